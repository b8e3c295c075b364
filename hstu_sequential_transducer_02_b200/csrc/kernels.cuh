// Internal launcher interfaces of libhstu (not part of the C ABI).
#pragma once

#include "common.cuh"

namespace hstu {

// ---------------------------------------------------------------- scheduler
size_t work_list_capacity(int B, int T, int H, int tile);
// Also writes tile_base[s] = index of sequence s's first kv tile of width tk in a
// tiled per-tile array (tile_base[B] = total tiles) when tile_base is not null.
// With q_from_hist (forward modes), a sequence's q tiles start at the one holding
// its first target row: only the targets' rows are computed (their history rows'
// K and V must be in place).
cudaError_t launch_build_work_list(const int32_t* offs, const int32_t* num_targets, int B, int T, int H,
                                   int tm, int tk, int mode, int max_items, WorkItem* items,
                                   int32_t* count, int32_t* status, cudaStream_t stream,
                                   int32_t* tile_base = nullptr, int q_from_hist = 0);

// Per kv tile of 128 columns: timestamps as int32 offsets from the sequence's
// first timestamp, with per-32-column min/max and a flag when any offset
// leaves +-2^30 (record of kTsRecWords int32, 16-byte multiple).
constexpr int kTsRecWords = 140;   // rel[128] | min[4] | max[4] | wide | pad[3]
struct TsRec {
  int32_t rel[128];  // t_j - t_first(sequence), clamped to +-(2^30 - 1); 0 beyond the sequence
  int32_t mn[4];     // per 32-column segment: min / max of rel over the columns inside the sequence
  int32_t mx[4];
  int32_t wide;      // 1 if some column's offset left +-2^30 (then the 64-bit path is used)
  int32_t pad[3];
};
static_assert(sizeof(TsRec) == kTsRecWords * 4, "record layout");
constexpr int kBandChunks = 20;    // 8-column bf16 chunks per row of the near-diagonal bias band
size_t ts_tiles_capacity(int B, int T);

cudaError_t launch_ts_tiles(const int32_t* offs, const int64_t* ts, int B, const int32_t* tile_base, int tiles_cap,
                            int32_t* recs, cudaStream_t st);


// ---------------------------------------------------------------- attention
// time-bucket thresholds, passed by value (kernel parameter space)
struct Thresholds { int64_t v[kNumBuckets]; };

size_t band_bytes(int T);
cudaError_t launch_band_bias(const int32_t* offs, const int32_t* num_targets, const int64_t* ts, int B, int T,
                             const int32_t* tile_base, int tiles_cap, const float* pos_bias,
                             const float* time_bias, const Thresholds& thr, double time_div, const int32_t* status,
                             void* band, cudaStream_t st);


struct AttnFwdParams {
  const int32_t* seq_offsets;
  const int32_t* num_targets;
  const int64_t* timestamps;
  const void* q; int64_t ldq;
  const void* k; int64_t ldk;
  const void* v; int64_t ldv;
  void* out; int64_t ldo;
  const float* pos_bias;
  const float* time_bias;
  int rab_head_stride;
  int num_heads;
  int total_rows;             // capacity T of the [T, .] tensors
  Thresholds thr;
  const WorkItem* items;
  const int32_t* item_count;
  int32_t* status;
  long long timeout_ns;        // bound of every device-side wait
  const int32_t* tile_base;    // tensor-core path: first tile record of each sequence
  const int32_t* tile_recs;    // tensor-core path: timestamp tile records
  int32_t* item_cursor;        // tensor-core path: dynamic work-list cursor (zeroed by the scheduler)
  const void* band;            // tensor-core path: near-diagonal half-bias band (bf16), or null
};

// Near-diagonal band of the tensor-core backward: for kv row j of a sequence and the
// 160 q rows i in [floor32(j), floor32(j) + 160), one 32-bit word: the relative bias
// rab(i, j) as bf16 in the upper half (-1e30 where (i, j) is not attended, so that
// SiLU and its derivative vanish there) and the time bucket in bits 0-6.
constexpr int kBwdBandCols = 160;
size_t bwd_band_bytes(int T);
cudaError_t launch_bwd_band(const int32_t* offs, const int32_t* num_targets, const int64_t* ts, int B, int T,
                            const int32_t* tile_base, int tiles_cap, const float* pos_bias, const float* time_bias,
                            const Thresholds& thr, double time_div, const int32_t* status, uint32_t* band,
                            cudaStream_t st);

struct AttnBwdParams {
  const int32_t* seq_offsets;
  const int32_t* num_targets;
  const int64_t* timestamps;
  const void* q; int64_t ldq;
  const void* k; int64_t ldk;
  const void* v; int64_t ldv;
  const void* dout; int64_t lddo;
  float* dq_accum;            // [rows, H, dh] fp32, zeroed by the caller
  void* dk; int64_t lddk;
  void* dv; int64_t lddv;
  const float* pos_bias;
  const float* time_bias;
  float* d_pos_bias;
  float* d_time_bias;
  int rab_head_stride;
  int num_heads;
  int total_rows;
  Thresholds thr;
  const WorkItem* items;
  const int32_t* item_count;
  int32_t* status;
  long long timeout_ns;        // bound of every device-side wait
  const int32_t* tile_base;    // tensor-core path: first timestamp record of each sequence
  const int32_t* tile_recs;    // tensor-core path: timestamp records of the 128-row tiles
  const uint32_t* band;        // tensor-core path, bias shared by heads: near-diagonal band, or null
  int32_t* item_cursor;        // tensor-core path: dynamic work-list cursor (zeroed by the scheduler)
  float* rab_partial;          // tensor-core path: per-CTA partial rab gradients [grid][rab_tables][2][128], zeroed
  int rab_tables;              // 1 (tables shared by heads) or num_heads
};

int simt_tile_m();
cudaError_t launch_attn_fwd_simt(const AttnFwdParams& p, int dtype, int dh, int grid, cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const AttnBwdParams& p, int dtype, int dh, int grid, cudaStream_t st);
// tcgen05 (sm_100a) attention backward, bf16, dh = 64
bool tc_attn_bwd_supported(int dtype, int dh);
int tc_bwd_tile();
cudaError_t launch_attn_bwd_tc(const AttnBwdParams& p, int grid, cudaStream_t st, double time_div);
// d_pos[h * head_stride + b] += sum over CTAs of the partial tables, likewise d_time
cudaError_t launch_rab_reduce(const float* part, int ctas, int tables, int head_stride, float* d_pos, float* d_time,
                              cudaStream_t st);
cudaError_t launch_dq_finalize(const float* acc, const int32_t* offs, int B, int H, int dh, int dtype,
                               void* dq, int64_t lddq, int grid, cudaStream_t st);

// tcgen05 (sm_100a) attention forward, bf16 in/out, dh in {64, 128}
int tc_tile_m();
bool tc_attn_supported(int dtype, int dh);
cudaError_t launch_attn_fwd_tc(const AttnFwdParams& p, int dh, int grid, cudaStream_t st, double time_div);
int tc_attn_grid(int max_items);

cudaError_t launch_debug_buckets(const int32_t* offs, const int32_t* num_targets, const int64_t* ts,
                                 const Thresholds& thr, double time_div, const int32_t* pairs, int n, int32_t* out,
                                 cudaStream_t st);
cudaError_t launch_timeout_probe(long long timeout_ns, int32_t* status, cudaStream_t st);

// ---------------------------------------------------------------- fused short-sequence layer
struct FusedShortArgs {
  const int32_t* offs; const int32_t* num_targets; const int64_t* ts;
  const void* x; void* y;
  const void* w1; const float* b1; const float* ln1_g; const float* ln1_b;
  const float* ln2_g; const float* ln2_b; const void* w2; const float* b2;
  const float* pos_bias; const float* time_bias; int rab_head_stride;
  int B, T, d, H;
  float eps; double time_div; Thresholds thr;
  int32_t* cursor;             // zeroed before the launch
  int32_t* status;
  long long timeout_ns;
};
bool fused_short_supported(int d_model, int num_heads, int head_dim, int dtype, int io_dtype);
int fused_short_max_len();
cudaError_t launch_fused_short(const FusedShortArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- GEMM
// C[m, n] = sum_k A(m, k) B(n, k) with element strides; fp32 accumulation.
enum GemmEpilogue {
  EPI_STORE_F32 = 0,       // out_f32[m*ldo + n] = acc  (beta: += when accumulate)
  EPI_BIAS_SILU = 1,       // z = acc + bias[n]; out[m, n] = SiLU(z) (dtype); out2[m, n] = z if out2
  EPI_BIAS_RESIDUAL = 2,   // out[m, n] = acc + bias[n] + residual[m, n] (dtype)
  EPI_STORE = 3,           // out[m, n] = acc (dtype)
  EPI_SILU_BWD = 4,        // out[m, n] = acc * SiLU'(aux[m, n]) (dtype) — unused by the forward path
};

struct GemmParams {
  int M, N, K;
  const void* A; int64_t sam, sak;
  const void* B; int64_t sbn, sbk;
  int epi;
  const float* bias;
  const void* residual; int64_t ldr;
  void* out; int64_t ldo;
  void* out2; int64_t ldo2;
  const int32_t* rows_dev;   // if set: rows = min(M, *rows_dev)
  const int32_t* k_dev;      // if set: reduction length = min(K, *k_dev)
  int accumulate;            // EPI_STORE_F32: add to the existing value
  int out_f32;               // EPI_BIAS_RESIDUAL / EPI_STORE: output is fp32 (else the operand dtype)
  int res_f32;               // EPI_BIAS_RESIDUAL: residual is fp32 (else the operand dtype)
  int32_t* status;           // device status word for bounded-wait timeouts (tensor-core path)
  // EPI_BIAS_SILU on the tensor-core path: if set, output row m is written to row
  // out_slot_offs[m / out_slot_bm + 1] + m of out (rows at or past out_slot_cap are
  // dropped): the M-FALCON candidates' rows straight into their slots
  const int32_t* out_slot_offs; int out_slot_bm, out_slot_cap;
  // EPI_BIAS_RESIDUAL on the tensor-core path (whole 32-column chunks): if set, the
  // residual of row m is row res_map[m] and output row m goes to row out_map[m];
  // -1 means no residual / the row is dropped
  const int32_t* res_map; const int32_t* out_map;
};

cudaError_t launch_gemm_simt(const GemmParams& p, int dtype, cudaStream_t st);
// tcgen05 GEMM: A [M, K] and B [N, K] both K-major (sak = sbk = 1), bf16
bool tc_gemm_supported(const GemmParams& p, int dtype);
cudaError_t launch_gemm_tc(const GemmParams& p, cudaStream_t st);

// ---------------------------------------------------------------- row kernels
// xhat = LN(x) * gamma + beta; x in x_dtype, xhat in out_dtype
// (in_map: row m of x is row in_map[m], or a zero row where in_map[m] < 0)
cudaError_t launch_layer_norm(const void* x, int64_t ldx, int x_dtype, const float* gamma, const float* beta,
                              float eps, void* out, int64_t ldo, int out_dtype, float* mean, float* rstd,
                              int rows_cap, const int32_t* rows_dev, int d, cudaStream_t st,
                              const int32_t* in_map = nullptr);
// g = LN(o) * u; with in_slot_offs, row m of o and u is read from row
// in_slot_offs[m / in_slot_bm + 1] + m (row 0 if that reaches in_slot_cap)
cudaError_t launch_ln_gate(const void* o, int64_t ldo_in, const void* u, int64_t ldu, const float* gamma,
                           const float* beta, float eps, void* out, int64_t ldout, float* mean, float* rstd,
                           int rows_cap, const int32_t* rows_dev, int d, int dtype, cudaStream_t st,
                           const int32_t* in_slot_offs = nullptr, int in_slot_bm = 1, int in_slot_cap = 0);
// backward of g = (LN2(o) gamma + beta) * u: writes d_o and du = dg (LN2(o) gamma + beta)
// (dtype) and accumulates the affine gradients (atomics; the caller zeroes them)
cudaError_t launch_ln_gate_bwd(const void* o, int64_t ldo_in, const void* u, int64_t ldu, const float* gamma,
                               const float* beta, const float* mean, const float* rstd, const void* dg, int64_t lddg,
                               void* d_o, int64_t ld_do, void* du, int64_t lddu, float* dgamma, float* dbeta,
                               int rows_cap, const int32_t* rows_dev, int d, int dtype, cudaStream_t st);
// du = dg * (LN2(o) gamma + beta)
cudaError_t launch_ln_gate_du(const void* o, int64_t ldo_in, const float* gamma, const float* beta,
                              const float* mean, const float* rstd, const void* dg, int64_t lddg, void* du,
                              int64_t lddu, int rows_cap, const int32_t* rows_dev, int d, int dtype,
                              cudaStream_t st);
// backward of xhat = LN1(x): dx = dres + LNback(dxhat); accumulates dgamma/dbeta.
// x, dres and dx are in io_dtype, dxhat is fp32
cudaError_t launch_ln_bwd(const void* x, int64_t ldx, const float* gamma, const float* mean, const float* rstd,
                          const float* dxhat, int64_t lddxh, const void* dres, int64_t lddres, void* dx,
                          int64_t lddx, float* dgamma, float* dbeta, int rows_cap, const int32_t* rows_dev,
                          int d, int io_dtype, cudaStream_t st);
// dst (bf16 or fp32 per dst_dtype) = src (src_dtype) for rows < *rows_dev, zero for rows in
// [*rows_dev, min(cap, round_up(*rows_dev, pad_multiple)))
cudaError_t launch_convert_rows(const void* src, int64_t lds, int src_dtype, void* dst, int64_t ldd, int dst_dtype,
                                int cols, int rows_cap, const int32_t* rows_dev, int pad_multiple, cudaStream_t st);
// zero rows [*rows_dev, min(cap, round_up(*rows_dev, multiple))) of a row-major buffer
cudaError_t launch_zero_tail_rows(void* buf, int64_t ld_bytes, int64_t row_bytes, int rows_cap,
                                  const int32_t* rows_dev, int multiple, cudaStream_t st);
// dz = da * SiLU'(z) (dtype), elementwise on [rows, cols]; with dq, columns
// [q_col0, q_col0 + q_cols) take da from the fp32 matrix dq (row stride ldq)
cudaError_t launch_silu_bwd(const void* da, const void* z, void* dz, int64_t ld, int rows_cap,
                            const int32_t* rows_dev, int cols, int dtype, cudaStream_t st, const float* dq = nullptr,
                            int64_t ldq = 0, int q_col0 = 0, int q_cols = 0);
// floats of scratch the column-sum passes below need for `cols` columns
size_t col_partials_size(int cols);
// launch_silu_bwd and, in the same pass, col_sums = the column sums of dz as stored
// (overwritten); part: col_partials_size(cols) floats of scratch
cudaError_t launch_silu_bwd_colsum(const void* da, const void* z, void* dz, int64_t ld, int rows_cap,
                                   const int32_t* rows_dev, int cols, int dtype, float* col_sums, float* part,
                                   cudaStream_t st, const float* dq = nullptr, int64_t ldq = 0, int q_col0 = 0,
                                   int q_cols = 0);
// launch_convert_rows and, in the same pass, col_sums = the column sums of src's
// rows < *rows_dev (overwritten); part: col_partials_size(cols) floats of scratch
cudaError_t launch_convert_rows_colsum(const void* src, int64_t lds, int src_dtype, void* dst, int64_t ldd,
                                       int dst_dtype, int cols, int rows_cap, const int32_t* rows_dev,
                                       int pad_multiple, float* col_sums, float* part, cudaStream_t st);
// column sums of a [rows, cols] dtype matrix into fp32 out (overwrite)
cudaError_t launch_col_sum(const void* a, int64_t lda, int rows_cap, const int32_t* rows_dev, int cols,
                           int dtype, float* out, cudaStream_t st);

cudaError_t launch_gather_rows(const void* src, void* dst, int64_t row_bytes, const int32_t* index,
                               const int32_t* count, int capacity, cudaStream_t st);
cudaError_t launch_sl_select(int B, int T, const int32_t* offs, const uint32_t* coins, const uint32_t* keys,
                             int max_len, uint32_t prob, int32_t* out_offsets, int32_t* out_index,
                             int32_t* scratch_len, int32_t* status, cudaStream_t st);
// out[i] = offs[s0 + i] - offs[s0] for i in [0, nb]
cudaError_t launch_rebase_offsets(const int32_t* offs, int s0, int nb, int32_t* out, cudaStream_t st);
// rows r < *total_rows (total_rows null: r < cap_rows) with cand_row_map[r] >= 0 go to that row of cand_out
cudaError_t launch_mfalcon_scatter(const void* y, int d, int dtype, const int32_t* cand_row_map,
                                   const int32_t* total_rows, int cap_rows, void* cand_out, cudaStream_t st);
// M-FALCON with the history cached across microbatches (slot layout: user u's rows
// [history_u ; bm candidate slots] from row hist_offs[u] + u * bm; compact candidate
// row c = u * bm + j).  Offsets and num_targets (= bm) of the slot layout:
cudaError_t launch_mfalcon_slot_offsets(int U, int bm, const int32_t* hist_offs, int32_t* offs, int32_t* nt,
                                       cudaStream_t st);
// microbatch mb's candidates into the slot rows (x_slot, ts_slot) and/or the compact
// rows (x_c), zero rows past a user's candidates; cand_dst[c] = row of cand_out or -1.
// with_hist also copies the history rows; rows_cap = rows walked (all slot rows or U * bm);
// slot rows at or past cap (offsets larger than the workspace was sized for) are skipped.
cudaError_t launch_mfalcon_slot_pack(int U, int mb, int bm, int rows_cap, int cap, const int32_t* hist_offs,
                                     const void* hist_x, const int64_t* hist_ts, const int32_t* cand_offs,
                                     const void* cand_x, const int64_t* cand_ts, int d, int dtype, int with_hist,
                                     void* x_slot, int64_t* ts_slot, void* x_c, int32_t* cand_dst, cudaStream_t st);
// HSTU_ERR_BAD_OFFSETS into the status word when a user has a negative candidate
// count or more than `limit` candidates
cudaError_t launch_mfalcon_check_counts(int U, int limit, const int32_t* cand_offs, int32_t* status,
                                        cudaStream_t st);
// row_bytes of each candidate row between the compact and the slot layout (multiples of 16 bytes)
cudaError_t launch_mfalcon_slot_rows(int U, int bm, int cap, const int32_t* hist_offs, const void* src,
                                     int64_t lds_bytes, void* dst, int64_t ldd_bytes, int64_t row_bytes, int to_slot,
                                     cudaStream_t st);

}  // namespace hstu
