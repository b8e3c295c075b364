/*
 * hstu.h — C ABI of the B200 (sm_100a) HSTU layer library, libhstu.so.
 *
 * What it computes.  One HSTU layer over a jagged batch of user-action
 * sequences, and the pieces of it:
 *
 *   U, V, Q, K = Split(SiLU(f1(LayerNorm(X))))                  (pointwise projection)
 *   A V        = (SiLU(Q K^T + rab^{p,t}) / N  (.) mask) V       (pointwise aggregated attention)
 *   Y          = X + f2(LayerNorm(A V) (.) U)                    (pointwise transformation)
 *
 * Sources: "Actions Speak Louder than Words" summary, section 1.2 (three
 * sub-layers, attention without softmax, relative position/time bias) and
 * section 2.2 (6 linear layers fused into 2, LayerNorm and SiLU fused);
 * "生成式推荐（一）：HSTU", HSTU encoder section (f1, f2 single linear
 * layers; phi = SiLU; Norm = LayerNorm; Norm(A(X)V(X)) (.) U(X)) and its
 * M-FALCON section (mask and rab changed so that b_m candidates are scored in
 * one pass); "Meta HSTU" case study, "Что меняется внутри HSTU" and
 * "Разная длина истории" (real sequence lengths instead of padding).
 * The pages lost the equations themselves; the constants are fixed here:
 *   position bucket  pb = clamp(pos_i - pos_j, 0, 127)
 *   time bucket      tb = clamp(floor(ln(max(1, |t_i - t_j|)) / time_div), 0, 127),
 *                    time_div = 0.301, evaluated exactly as the fp64 formula
 *                    through integer thresholds (hstu_build_time_thresholds)
 *   rab_ij           = pos_bias[pb] + time_bias[tb]
 *   N                = history length of the sequence (tokens that are not
 *                      M-FALCON candidates), at least 1
 *   mask             = causal with the diagonal; an M-FALCON candidate (one of
 *                      the last num_targets[s] tokens of sequence s) sits at
 *                      position N and sees the history and itself only.
 *   No 1/sqrt(d) scaling of Q K^T.  LayerNorm: biased variance, affine.
 *
 * Conventions shared by every call.
 *   - Every pointer argument named as "device" is a device pointer owned by the
 *     caller; the library allocates no device memory on any of these calls.
 *     Scratch comes from the caller's `workspace` (device, 256-byte aligned),
 *     at least the size the matching *_workspace_size call reports.
 *   - Tensors are token-major.  A [T, H, dh] tensor has row stride `ld`
 *     (elements between consecutive tokens); head h starts at column h*dh.
 *     Rows must start 16-byte aligned (ld * element size a multiple of 16).
 *   - Element type is the descriptor's dtype: HSTU_DTYPE_F32 (float) or
 *     HSTU_DTYPE_BF16 (bfloat16, fp32 accumulation).  Bias tables, LayerNorm
 *     affine vectors, linear biases, statistics and weight gradients are float.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     is asynchronous on it and does no host/device synchronisation.
 *   - Return value: HSTU_OK or an HSTU_ERR_* code; nothing is launched when an
 *     argument check fails.  Errors detected on the device (a bounded wait that
 *     expired) are written to the status word at the start of the workspace;
 *     read it with hstu_workspace_status after synchronising.
 *   - `total_tokens` in hstu_jagged is the capacity (rows of every [T, .]
 *     buffer).  The rows actually used are seq_offsets[batch] <= total_tokens,
 *     read on the device; output rows beyond it are not written.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define HSTU_OK               0
#define HSTU_ERR_INVALID_ARG  1  /* null pointer, bad size or stride, misaligned buffer */
#define HSTU_ERR_UNSUPPORTED  2  /* head dim / dtype / bucket count not built */
#define HSTU_ERR_CUDA         3  /* a CUDA runtime error (launch or earlier async error) */
#define HSTU_ERR_TIMEOUT      4  /* a bounded device-side wait expired (device status) */
#define HSTU_ERR_WORKSPACE    5  /* workspace missing or smaller than required */
#define HSTU_ERR_BAD_OFFSETS  6  /* device-side validation: offsets not monotone / out of range */

#define HSTU_DTYPE_F32  0
#define HSTU_DTYPE_BF16 1

/* descriptor flags */
#define HSTU_FLAG_FORCE_SIMT 1   /* diagnostics: run the CUDA-core attention/GEMM kernels
                                    instead of the tcgen05 ones (bf16 only) */
#define HSTU_FLAG_SHORT_SEQUENCES 2
/* hstu_layer_fwd: the caller states that every sequence has at most 128 tokens,
 * and the layer runs as one kernel (every intermediate on the chip: LayerNorm,
 * f1, the attention of all heads, LayerNorm(A V) * U, f2 and the residual;
 * "Actions Speak Louder than Words" summary, 1.3: kernel fusion).  Its work units
 * are runs of at most 128 consecutive token rows holding whole sequences, so
 * several short sequences share one tile.
 * It applies to bf16 weights and activations (io_dtype bf16), head dimension 64,
 * d_model and num_heads * 64 at most 256 and multiples of 64, and inference
 * (saved == NULL); otherwise the flag is ignored.  A sequence longer than 128
 * tokens (or outside the buffers) is not computed and sets HSTU_ERR_BAD_OFFSETS
 * in the workspace status word. */
#define HSTU_FLAG_REUSE_PREP 4
/* hstu_layer_fwd / hstu_layer_bwd / hstu_attn_fwd / hstu_attn_bwd: the workspace
 * still holds the attention's work list and timestamp tile records from an
 * earlier call of the same entry point on the same jagged batch (the same
 * seq_offsets, num_targets and timestamps, contents and sizes) and the same head
 * count; they are not rebuilt (the layers of a stack share them within a step).
 * The relative-bias band, which depends on the bias tables, is rebuilt.  Offsets
 * that the earlier call found invalid stay without work, and only that call
 * reported them. */
/* seq_offsets and num_targets are always checked on the device by the
 * scheduler kernel that precedes every attention launch; a violation writes
 * HSTU_ERR_BAD_OFFSETS to the workspace status word and schedules no work. */

/* ---- descriptors ------------------------------------------------------- */
typedef struct hstu_attn_desc {
  int32_t num_heads;        /* H >= 1 */
  int32_t dqk;              /* head dim of Q and K: 32, 64 or 128 */
  int32_t dv;               /* head dim of V and of the output: must equal dqk */
  int32_t dtype;            /* HSTU_DTYPE_* */
  int32_t rab_head_stride;  /* 0: one bias table pair shared by all heads;
                               num_pos_buckets: head h uses table + h * 128 */
  int32_t num_pos_buckets;  /* must be 128 */
  int32_t num_time_buckets; /* must be 128 */
  int32_t flags;            /* HSTU_FLAG_* */
  double  time_div;         /* divisor of ln(dt) in the time bucket: 0.301 */
} hstu_attn_desc;

typedef struct hstu_layer_desc {
  int32_t d_model;          /* d; must be a multiple of 8, <= 1024 */
  float   ln_eps;           /* LayerNorm epsilon, 1e-5 */
  int32_t io_dtype;         /* element type of the residual stream X, Y (and dX, dY):
                               attn.dtype, or HSTU_DTYPE_F32 to keep the residual
                               stream in fp32 while activations and weights are bf16 */
  int32_t reserved;         /* must be 0 */
  hstu_attn_desc attn;      /* H * dv is the width of U, V, Q, K and of A V */
} hstu_layer_desc;

/* A jagged batch: sequence s holds tokens seq_offsets[s] .. seq_offsets[s+1]-1. */
typedef struct hstu_jagged {
  int32_t batch;               /* B >= 0 */
  int32_t total_tokens;        /* capacity T of every [T, .] buffer; seq_offsets[B] <= T */
  const int32_t* seq_offsets;  /* device [B+1], non-decreasing, seq_offsets[0] = 0 */
  const int32_t* num_targets;  /* device [B] or NULL: the last num_targets[s] tokens of
                                  sequence s are M-FALCON candidates (0 <= it <= n_s) */
  const int64_t* timestamps;   /* device [T], seconds */
} hstu_jagged;

/* Layer parameters.  Linear weights are (out, in) row-major: y = x W^T + b. */
typedef struct hstu_layer_weights {
  const void*  w1;          /* device [4*H*dv, d], dtype; output columns ordered U, V, Q, K */
  const float* b1;          /* device [4*H*dv] */
  const float* ln1_gamma;   /* device [d] */
  const float* ln1_beta;    /* device [d] */
  const float* ln2_gamma;   /* device [H*dv] */
  const float* ln2_beta;    /* device [H*dv] */
  const void*  w2;          /* device [d, H*dv], dtype */
  const float* b2;          /* device [d] */
  const float* pos_bias;    /* device [128] or [H,128] (rab_head_stride) */
  const float* time_bias;   /* device [128] or [H,128] */
} hstu_layer_weights;

/* Activations the forward pass keeps for the backward pass (all device, T rows). */
typedef struct hstu_layer_saved {
  void*  xhat;       /* [T, d] dtype: LayerNorm1(X) */
  float* ln1_mean;   /* [T] */
  float* ln1_rstd;   /* [T] */
  void*  z;          /* [T, 4*H*dv] dtype: f1 pre-activation */
  void*  uvqk;       /* [T, 4*H*dv] dtype: SiLU(z) = U | V | Q | K */
  void*  attn_out;   /* [T, H*dv] dtype: A V */
  float* ln2_mean;   /* [T] */
  float* ln2_rstd;   /* [T] */
  void*  gate;       /* [T, H*dv] dtype: LayerNorm2(A V) * U, the input of f2.  The
                        forward writes it when non-NULL and the backward then reads it
                        (so it must hold what the forward wrote); NULL: the forward
                        keeps it in its workspace and the backward recomputes it from
                        attn_out and uvqk */
} hstu_layer_saved;

/* Gradients of one layer (all device).  Weight gradients are overwritten (=). */
typedef struct hstu_layer_grads {
  float* dw1;         /* [4*H*dv, d] */
  float* db1;         /* [4*H*dv] */
  float* dln1_gamma;  /* [d] */
  float* dln1_beta;   /* [d] */
  float* dln2_gamma;  /* [H*dv] */
  float* dln2_beta;   /* [H*dv] */
  float* dw2;         /* [d, H*dv] */
  float* db2;         /* [d] */
  float* dpos_bias;   /* like pos_bias */
  float* dtime_bias;  /* like time_bias */
  void*  duvqk;       /* optional [T, 4*H*dv] dtype: gradients w.r.t. U | V | Q | K
                         (the SiLU outputs); NULL keeps them in the workspace */
} hstu_layer_grads;

/* ---- utilities ----------------------------------------------------------- */

/* Message for a status code (static storage, never NULL). */
const char* hstu_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int hstu_version(void);

/* Description of the last CUDA error that made a call of this thread return
 * HSTU_ERR_CUDA (the failing runtime call and CUDA's message); thread-local
 * static storage, never NULL. */
const char* hstu_last_cuda_error(void);

/* Integer thresholds of the time bucket (host only, no CUDA call):
 * out[0] = 0 and, for b >= 1, out[b] = the smallest dt >= 1 with
 * floor(ln(dt) / time_div) >= b in fp64 (INT64_MAX if none).  Then
 * tb(dt) = min(num_buckets - 1, #{b in 1..num_buckets-1 : out[b] <= max(|dt|, 1)}).
 * out has num_buckets entries.  Returns HSTU_ERR_INVALID_ARG for time_div <= 0,
 * num_buckets outside [2, 1024] or out == NULL. */
int hstu_build_time_thresholds(double time_div, int32_t num_buckets, int64_t* out);

/* Copy the device status word at the start of a workspace to *status (host).
 * Synchronises `stream`.  *status is HSTU_OK or an HSTU_ERR_* code. */
int hstu_workspace_status(const void* workspace, int32_t* status, void* stream);

/* ---- pointwise aggregated attention ------------------------------------ */

/* Workspace bytes for hstu_attn_fwd on a batch of `batch` sequences with
 * capacity `total_tokens`.  Writes *bytes; no CUDA call. */
int hstu_attn_fwd_workspace_size(const hstu_attn_desc* desc, int32_t batch,
                                 int32_t total_tokens, size_t* bytes);

/* out_i = (1/N_s) sum_{j in mask(i)} SiLU(q_i . k_j + rab_ij) v_j for every
 * token i of every sequence s and every head.
 *   q, k: device [T, H, dqk] with row strides ldq, ldk;  v: device [T, H, dv], ldv;
 *   pos_bias, time_bias: device float tables (desc->rab_head_stride);
 *   out: device [T, H, dv] with row stride ldo (may not alias q, k, v).
 * bf16 with dqk in {64, 128} runs on the tcgen05 tensor cores; f32 (and
 * HSTU_FLAG_FORCE_SIMT) runs on the CUDA cores. */
int hstu_attn_fwd(const hstu_attn_desc* desc, const hstu_jagged* jb,
                  const void* q, int64_t ldq, const void* k, int64_t ldk,
                  const void* v, int64_t ldv,
                  const float* pos_bias, const float* time_bias,
                  void* out, int64_t ldo,
                  void* workspace, size_t workspace_bytes, void* stream);

/* hstu_attn_fwd without a workspace argument, for callers that cannot allocate
 * device memory where they call it (an application whose device memory is
 * owned entirely by another allocator, or a serving loop that forbids
 * allocation once it runs).  The pages describe no such variant: it is a
 * property of this library, not of the method.
 *
 * Same arguments, layouts and result as hstu_attn_fwd.  The scratch it needs
 * lives in a 1 MiB array that the library keeps in the device memory of every
 * GPU it is loaded on, for the life of the process; the call itself allocates
 * nothing.  That scratch is the status word, the work list and, on the
 * tensor-core path, the per-kv-tile timestamp records; this entry point does
 * without the near-diagonal bias band of hstu_attn_fwd (it evaluates those
 * biases per element instead), so its results may differ from hstu_attn_fwd's
 * by bf16 rounding of the bias near the diagonal.  A problem whose scratch
 * exceeds the array is refused with HSTU_ERR_WORKSPACE before anything is
 * launched: with W = total_tokens/128 + batch + 1, the tensor-core path needs
 * about (16 * num_heads + 560) * W bytes + 1 KB (num_heads = 4: up to about
 * 1,700 tiles of 128 tokens, some 200,000 tokens in few sequences).
 *   - The first call on a device looks up the array's device address on that
 *     device (current device at the time of the call), and so does the first
 *     call from each further context of the device (a non-primary context, or
 *     the primary context recreated after cudaDeviceReset).
 *   - All calls share the one array and each call overwrites it.  Calls that
 *     may run at the same time on the GPU (different streams without ordering
 *     between them) race on it and give undefined results: order them.
 *   - Device-side wait timeouts of this call are recorded in the array's status
 *     word, which is not readable through this interface. */
int hstu_attn_fwd_noalloc(const hstu_attn_desc* desc, const hstu_jagged* jb,
                          const void* q, int64_t ldq, const void* k, int64_t ldk,
                          const void* v, int64_t ldv,
                          const float* pos_bias, const float* time_bias,
                          void* out, int64_t ldo, void* stream);

int hstu_attn_bwd_workspace_size(const hstu_attn_desc* desc, int32_t batch,
                                 int32_t total_tokens, size_t* bytes);

/* Backward of hstu_attn_fwd for the loss sum(out * dout):
 *   dq = dS k, dk = dS^T q, dv = P^T dout with P = mask SiLU(S)/N and
 *   dS = (dout v^T) (.) mask (.) SiLU'(S) / N;
 *   d_pos_bias[b] += sum of dS over pairs with position bucket b, d_time_bias
 *   likewise (ACCUMULATED: the caller zeroes them; the order of the float
 *   additions is not deterministic).
 * dq, dk, dv: device, dtype, same layouts as q, k, v (strides lddq, lddk, lddv);
 * they are overwritten. */
int hstu_attn_bwd(const hstu_attn_desc* desc, const hstu_jagged* jb,
                  const void* q, int64_t ldq, const void* k, int64_t ldk,
                  const void* v, int64_t ldv,
                  const float* pos_bias, const float* time_bias,
                  const void* dout, int64_t lddo,
                  void* dq, int64_t lddq, void* dk, int64_t lddk, void* dv, int64_t lddv,
                  float* d_pos_bias, float* d_time_bias,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ---- the layer ------------------------------------------------------------ */

int hstu_layer_fwd_workspace_size(const hstu_layer_desc* desc, int32_t batch,
                                  int32_t total_tokens, size_t* bytes);

/* Y = X + f2(LayerNorm2(A V) (.) U) with U, V, Q, K = Split(SiLU(f1(LayerNorm1(X)))).
 *   x, y: device [T, d] io_dtype, contiguous (row stride d); y may not alias x.
 *   saved: NULL for inference, else its buffers receive what hstu_layer_bwd needs.
 * The attention's preparation (work list, timestamp records, bias band) runs on a
 * library-owned side stream of the device, overlapping LayerNorm1 and f1; calls
 * from several host threads share that stream, which only orders their
 * preparations.  While `stream` is being captured into a CUDA graph the
 * preparation runs on `stream` itself, so the capture never reaches the shared
 * side stream. */
int hstu_layer_fwd(const hstu_layer_desc* desc, const hstu_layer_weights* w,
                   const hstu_jagged* jb, const void* x, void* y,
                   const hstu_layer_saved* saved,
                   void* workspace, size_t workspace_bytes, void* stream);

/* The layer forward from and to HOST memory: the sequences are split into
 * `num_chunks` groups of consecutive sequences with about equal token counts;
 * chunk c's X rows and timestamps are copied in while chunk c-1 is computed
 * and chunk c-2's Y rows are copied out (one copy stream each way), so that on
 * a full-duplex link the call takes about as long as the larger of the two
 * transfers.  Every row is computed exactly as hstu_layer_fwd computes it on
 * the whole batch (rows of different sequences do not interact), so Y is
 * bit-identical to that call's.
 *   seq_offsets [batch+1], num_targets [batch] (or NULL), timestamps [T]:
 *     HOST arrays, read during the call (T = seq_offsets[batch]);
 *   x [T, d], y [T, d]: HOST, io_dtype, contiguous; page-locked memory
 *     (cudaHostAlloc / cudaHostRegister) is needed for the copies to overlap
 *     the computation, pageable memory works but serialises them;
 *   num_chunks: 1 .. 64 (clamped to batch);
 *   workspace: device, hstu_layer_fwd_host_workspace_size bytes, 256-aligned.
 * The call returns once everything is enqueued; `stream` is complete when Y is
 * in host memory.  Errors: HSTU_ERR_INVALID_ARG (null pointers, batch < 0,
 * offsets not starting at 0 or decreasing, num_chunks < 1), HSTU_ERR_WORKSPACE,
 * HSTU_ERR_CUDA; device-side errors go to the workspace status word. */
int hstu_layer_fwd_host_workspace_size(const hstu_layer_desc* desc, int32_t batch,
                                       int32_t total_tokens, int32_t num_chunks, size_t* bytes);
int hstu_layer_fwd_host(const hstu_layer_desc* desc, const hstu_layer_weights* w, int32_t batch,
                        const int32_t* seq_offsets, const int32_t* num_targets,
                        const int64_t* timestamps, const void* x, void* y, int32_t num_chunks,
                        void* workspace, size_t workspace_bytes, void* stream);

int hstu_layer_bwd_workspace_size(const hstu_layer_desc* desc, int32_t batch,
                                  int32_t total_tokens, size_t* bytes);

/* Gradients of sum(Y * dy) for one layer, from the activations hstu_layer_fwd
 * saved.  x, dy, dx: device [T, d] io_dtype (dx may alias dy).  All gradients
 * in `g` are overwritten, rab gradients included.  Rows of the saved xhat beyond
 * seq_offsets[batch] (up to the next multiple of 64) are set to zero. */
int hstu_layer_bwd(const hstu_layer_desc* desc, const hstu_layer_weights* w,
                   const hstu_jagged* jb, const void* x, const hstu_layer_saved* saved,
                   const void* dy, void* dx, const hstu_layer_grads* g,
                   void* workspace, size_t workspace_bytes, void* stream);

/* ---- M-FALCON ranking ------------------------------------------------------ */

/* Workspace for mfalcon_rank: `hist_total` history tokens over `num_users`
 * users, candidates scored `microbatch` at a time through `num_layers` layers. */
int mfalcon_rank_workspace_size(const hstu_layer_desc* desc, int32_t num_layers,
                                int32_t num_users, int32_t hist_total, int32_t microbatch,
                                size_t* bytes);

/* Scores every candidate of every user ("2.3 M-FALCON算法"): for microbatch k,
 * user u's sequence is [history_u ; candidates_u[k*b_m, (k+1)*b_m)], run through
 * the `num_layers` layers with the candidates as M-FALCON targets (they see the
 * history and themselves, sit at position n_u, and N = n_u).  The final-layer rows
 * of the candidates are written to cand_out.
 *   layers: host array of num_layers weight structs (device pointers inside);
 *   hist_offsets [U+1], cand_offsets [U+1]: device; hist_x [hist_total, d],
 *   hist_ts [hist_total]; cand_x [cand_offsets[U], d], cand_ts [...]: device;
 *   max_candidates: host upper bound on any user's candidate count (sets the
 *   number of microbatches, ceil(max_candidates / microbatch)); a user with more
 *   candidates than those microbatches hold (or a negative count) sets the status
 *   word to HSTU_ERR_BAD_OFFSETS after the call's work, and its candidates past
 *   the last microbatch are not written;
 *   hist_x, cand_x, cand_out are in desc->io_dtype; cand_out: [cand_offsets[U], d].
 * The history rows do not depend on the candidates, so every layer's keys and
 * values of the history are computed once, with microbatch 0, and kept in the
 * workspace (one U|V|Q|K cache per layer, "the history's KV cache is reused
 * across microbatches"); every later microbatch computes only its candidates'
 * rows.  Each user keeps b_m candidate slots in every microbatch: slots past the
 * user's candidates are computed on zero rows and not written out.
 * Errors: HSTU_ERR_INVALID_ARG (null or misaligned pointers, bad counts),
 * HSTU_ERR_WORKSPACE (workspace too small or not 256-byte aligned),
 * HSTU_ERR_CUDA; errors found on the device go to the status word at the start
 * of the workspace (hstu_workspace_status). */
int mfalcon_rank(const hstu_layer_desc* desc, const hstu_layer_weights* layers,
                 int32_t num_layers, int32_t num_users, int32_t hist_total,
                 int32_t max_candidates, int32_t microbatch,
                 const int32_t* hist_offsets, const void* hist_x, const int64_t* hist_ts,
                 const int32_t* cand_offsets, const void* cand_x, const int64_t* cand_ts,
                 void* cand_out, void* workspace, size_t workspace_bytes, void* stream);

/* ---- data-parallel sharding ----------------------------------------------- */

/* Splits one jagged batch over `world` data-parallel ranks by sequence (rows of
 * different sequences never interact, so the ranks exchange nothing on the data
 * path; "Meta HSTU" case study, "Разная длина истории": a sequence costs what its
 * real length costs).  Host-only: no device work, usable without a GPU.
 * The cost of sequence s is its attended pairs, N(N+1)/2 + m(N+1) with N its
 * history length and m = num_targets[s] (NULL: 0), plus token_weight * n_s for
 * the row-wise work; the sequences go, in order of decreasing cost (equal costs:
 * lower index first), each to the rank with the smallest total so far (equal
 * totals: lower rank) -- greedy longest-processing-time first.  Every rank that
 * calls it with the same arguments gets the same assignment.
 *   seq_offsets [batch+1], num_targets [batch] or NULL: HOST arrays;
 *   rank_of [batch]: HOST, receives each sequence's rank;
 *   rank_cost [world]: HOST, receives each rank's total cost.
 * Errors: HSTU_ERR_INVALID_ARG (batch < 0, world < 1, null outputs, offsets not
 * starting at 0 or decreasing, negative token_weight). */
int hstu_lpt_partition(int32_t batch, const int32_t* seq_offsets, const int32_t* num_targets, int32_t world,
                       double token_weight, int32_t* rank_of, double* rank_cost);

/* ---- Stochastic Length ------------------------------------------------------ */

int hstu_stochastic_length_workspace_size(int32_t batch, int32_t total_tokens, size_t* bytes);

/* Stochastic Length subsampling ("2.1 随机长度": training on random sub-sequences
 * of long histories, sometimes on the whole history).  Sequence s with
 * n_s > max_len and coins[s] < prob_u32 keeps the max_len tokens whose keys are
 * smallest (ties to the lower index), in their original order; every other
 * sequence is kept whole.  coins [B] and keys [T] are caller-drawn uint32
 * random numbers (device).  Writes out_offsets [B+1] and out_index [T]
 * (source row of each kept token; the first out_offsets[B] entries are used). */
int hstu_stochastic_length(int32_t batch, int32_t total_tokens, const int32_t* seq_offsets,
                           const uint32_t* coins, const uint32_t* keys,
                           int32_t max_len, uint32_t prob_u32,
                           int32_t* out_offsets, int32_t* out_index,
                           void* workspace, size_t workspace_bytes, void* stream);

/* dst[r] = src[index[r]] for r < *count (device int32 read on the device),
 * rows of `row_bytes` bytes (a multiple of 4); at most `capacity` rows. */
int hstu_gather_rows(const void* src, void* dst, int64_t row_bytes,
                     const int32_t* index, const int32_t* count, int32_t capacity,
                     void* stream);

/* ---- tracing ------------------------------------------------------------------ */

/* enable != 0: from now on every kernel launch of the library is bracketed by a
 * pair of CUDA events on its stream (host-side event objects; no device memory).
 * Either value discards the records kept so far. */
int hstu_trace_enable(int enable);

/* Synchronises the recorded events and sums device time per kernel name:
 * names [max_kernels][32] (NUL-terminated), counts [max_kernels] launches,
 * total_ms [max_kernels]; *num_kernels receives the number of distinct names
 * (entries beyond max_kernels are not written). */
int hstu_trace_read(int32_t max_kernels, char* names, int32_t* counts, double* total_ms, int32_t* num_kernels);

/* ---- diagnostics ------------------------------------------------------------ */

/* For each query pair p: pairs[3p] = sequence, pairs[3p+1] = i, pairs[3p+2] = j
 * (indices inside the sequence), writes out[3p] = position bucket,
 * out[3p+1] = time bucket, out[3p+2] = 1 if (i, j) is attended, else 0 — using
 * the same device code as the attention kernels.  pairs/out: device int32. */
int hstu_debug_rab_buckets(const hstu_attn_desc* desc, const hstu_jagged* jb,
                           const int32_t* pairs, int32_t num_pairs, int32_t* out,
                           void* stream);

/* Runs one kernel whose mbarrier wait can never complete, using the bounded
 * wait of the library's kernels cut to `timeout_ns` nanoseconds (1 .. 2e9); it
 * must give up, write HSTU_ERR_TIMEOUT to *status_dev (device int32) and return.
 * The library's own kernels give up after 2 s per wait and report
 * HSTU_ERR_TIMEOUT in the workspace status word. */
int hstu_debug_timeout_probe(int64_t timeout_ns, int32_t* status_dev, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HSTU_H_ */
