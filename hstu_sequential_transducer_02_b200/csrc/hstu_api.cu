// The C ABI of libhstu: argument validation, workspace carving and the launch
// sequence of each call.  Every step of the computation runs in this
// library's own kernels; nothing here computes on the host except the
// time-bucket threshold table.
#include <algorithm>
#include <cuda.h>
#include <math.h>
#include <stdio.h>
#include <mutex>
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"
#include "trace.cuh"

using namespace hstu;

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr long long kDefaultTimeoutNs = 2000000000ll;  // a device-side wait gives up after 2 s
constexpr int kMaxDevices = 64;                        // per-device caches (side stream, scratch address)

// ---------------------------------------------------------------- workspace carving
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base((char*)b) {}
  template <typename T>
  T* take(size_t count) {
    off = (off + 255) & ~(size_t)255;
    T* p = base ? (T*)(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
  size_t size() const { return (off + 255) & ~(size_t)255; }
};

size_t elem_size(int dtype) { return dtype == HSTU_DTYPE_F32 ? 4 : 2; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA; }

#define HSTU_TRY(expr)                      \
  do {                                      \
    int _s = (expr);                        \
    if (_s != HSTU_OK) return _s;           \
  } while (0)
thread_local char g_last_error[256] = "no error";

int record_cuda_error(cudaError_t e, const char* what) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
  return HSTU_ERR_CUDA;
}

#define HSTU_CUDA(expr)                                         \
  do {                                                          \
    cudaError_t _e = (expr);                                    \
    if (_e != cudaSuccess) return record_cuda_error(_e, #expr); \
  } while (0)

// ---------------------------------------------------------------- thresholds
int64_t bucket_floor(int64_t dt, double div) {
  double v = (double)(dt < 1 ? 1 : dt);
  return (int64_t)floor(log(v) / div);
}

void build_thresholds(double div, int nb, int64_t* out) {
  out[0] = 0;
  for (int b = 1; b < nb; ++b) {
    if (bucket_floor(INT64_MAX, div) < b) { out[b] = INT64_MAX; continue; }
    int64_t lo = 1, hi = INT64_MAX;  // f(hi) >= b
    if (bucket_floor(lo, div) >= b) { out[b] = lo; continue; }
    while (hi - lo > 1) {
      int64_t mid = lo + (hi - lo) / 2;
      if (bucket_floor(mid, div) >= b) hi = mid; else lo = mid;
    }
    out[b] = hi;
  }
}

std::mutex g_thr_mu;
double g_thr_div = -1.0;
Thresholds g_thr;

Thresholds thresholds_for(double div) {
  std::lock_guard<std::mutex> lk(g_thr_mu);
  if (div != g_thr_div) {
    build_thresholds(div, kNumBuckets, g_thr.v);
    g_thr_div = div;
  }
  return g_thr;
}

// ---------------------------------------------------------------- validation
int check_attn_desc(const hstu_attn_desc* d) {
  if (!d) return HSTU_ERR_INVALID_ARG;
  if (d->num_heads < 1 || d->num_heads > 1024) return HSTU_ERR_INVALID_ARG;
  if (d->num_pos_buckets != kNumBuckets || d->num_time_buckets != kNumBuckets) return HSTU_ERR_UNSUPPORTED;
  if (d->dtype != HSTU_DTYPE_F32 && d->dtype != HSTU_DTYPE_BF16) return HSTU_ERR_UNSUPPORTED;
  if (d->dqk != d->dv) return HSTU_ERR_UNSUPPORTED;
  if (d->dqk != 32 && d->dqk != 64 && d->dqk != 128) return HSTU_ERR_UNSUPPORTED;
  if (d->rab_head_stride != 0 && d->rab_head_stride != kNumBuckets) return HSTU_ERR_INVALID_ARG;
  if (!(d->time_div > 0.0) || !isfinite(d->time_div)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

int check_jagged(const hstu_jagged* jb) {
  if (!jb) return HSTU_ERR_INVALID_ARG;
  if (jb->batch < 0 || jb->total_tokens < 0) return HSTU_ERR_INVALID_ARG;
  if (!jb->seq_offsets || (jb->total_tokens > 0 && !jb->timestamps)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

int check_rows(const void* p, int64_t ld, int64_t min_ld, int dtype) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  if (ld < min_ld) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(p) || ((ld * (int64_t)elem_size(dtype)) % 16) != 0) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

// ---------------------------------------------------------------- attention
struct AttnWs {
  int32_t* status;
  int32_t* count;
  WorkItem* items;
  float* dq_accum;
  int capacity;
  int32_t* tile_base;   // tensor-core path: [B+1]
  int32_t* tile_recs;   // tensor-core path: timestamp records
  int tiles_cap;
  void* band;           // tensor-core path, rab shared by heads: near-diagonal bias band
  float* rab_partial;   // tensor-core backward: per-CTA partial rab gradients
  int rab_tables;
};

constexpr int kMaxBwdCtas = 256;   // the tensor-core backward runs at most this many CTAs

bool use_tc(const hstu_attn_desc* d) {
  return !(d->flags & HSTU_FLAG_FORCE_SIMT) && tc_attn_supported(d->dtype, d->dqk);
}

int attn_tile(const hstu_attn_desc* d) { return use_tc(d) ? tc_tile_m() : simt_tile_m(); }

bool use_tc_bwd(const hstu_attn_desc* d) {
  return !(d->flags & HSTU_FLAG_FORCE_SIMT) && tc_attn_bwd_supported(d->dtype, d->dqk) && d->dqk == d->dv;
}

int attn_bwd_tile(const hstu_attn_desc* d) { return use_tc_bwd(d) ? tc_bwd_tile() : simt_tile_m(); }

AttnWs carve_attn(Carver& c, const hstu_attn_desc* d, int B, int T, bool bwd, bool with_band = true) {
  AttnWs w;
  w.status = c.take<int32_t>(kStatusBytes / 4);
  w.count = c.take<int32_t>(64);
  const int tile = bwd ? attn_bwd_tile(d) : attn_tile(d);
  w.capacity = (int)work_list_capacity(B, T, d->num_heads, tile);
  w.items = c.take<WorkItem>(w.capacity);
  w.dq_accum = bwd ? c.take<float>((size_t)T * d->num_heads * d->dqk) : nullptr;
  w.tile_base = nullptr;
  w.tile_recs = nullptr;
  w.tiles_cap = 0;
  w.band = nullptr;
  w.rab_partial = nullptr;
  w.rab_tables = d->rab_head_stride ? d->num_heads : 1;
  if (!bwd && use_tc(d)) {
    w.tiles_cap = (int)ts_tiles_capacity(B, T);
    w.tile_base = c.take<int32_t>((size_t)B + 1);
    w.tile_recs = c.take<int32_t>((size_t)w.tiles_cap * kTsRecWords);
    if (with_band && d->rab_head_stride == 0) w.band = c.take<uint8_t>(band_bytes(T));
  }
  if (bwd && use_tc_bwd(d)) {
    // timestamp records of the 128-row tiles and, with one bias table for all heads,
    // the backward's near-diagonal band of bias and time-bucket words
    w.tiles_cap = (int)ts_tiles_capacity(B, T);
    w.tile_base = c.take<int32_t>((size_t)B + 1);
    w.tile_recs = c.take<int32_t>((size_t)w.tiles_cap * kTsRecWords);
    if (with_band && d->rab_head_stride == 0) w.band = c.take<uint8_t>(bwd_band_bytes(T));
    w.rab_partial = c.take<float>((size_t)kMaxBwdCtas * w.rab_tables * 2 * kNumBuckets);
  }
  return w;
}

// The attention's preparation (work list, timestamp tile records, bias band)
// depends only on the offsets, timestamps and bias tables, not on Q, K, V.
int run_attn_prep(const hstu_attn_desc* d, const hstu_jagged* jb, const float* pos_bias, const float* time_bias,
                  const AttnWs& w, cudaStream_t st) {
  const int tile = attn_tile(d);
  if (d->flags & HSTU_FLAG_REUSE_PREP) {
    // work list and tile records from an earlier call: only the fetch cursor restarts
    HSTU_CUDA(cudaMemsetAsync(w.count + 1, 0, sizeof(int32_t), st));
  } else {
    // tensor-core path: locality order, fetched dynamically (count[1] is the cursor)
    TraceScope tr("sched_fwd", st);
    HSTU_CUDA(launch_build_work_list(jb->seq_offsets, jb->num_targets, jb->batch, jb->total_tokens, d->num_heads,
                                     tile, tile, use_tc(d) ? 3 : 0, w.capacity, w.items, w.count, w.status, st,
                                     w.tile_base));
  }
  if (w.tile_recs && !(d->flags & HSTU_FLAG_REUSE_PREP)) {
    TraceScope tr("ts_tiles", st);
    HSTU_CUDA(launch_ts_tiles(jb->seq_offsets, jb->timestamps, jb->batch, w.tile_base, w.tiles_cap, w.tile_recs, st));
  }
  if (w.band) {
    TraceScope tr("band_bias", st);
    HSTU_CUDA(launch_band_bias(jb->seq_offsets, jb->num_targets, jb->timestamps, jb->batch, jb->total_tokens,
                               w.tile_base, w.tiles_cap, pos_bias, time_bias, thresholds_for(d->time_div),
                               d->time_div, w.status, w.band, st));
  }
  return HSTU_OK;
}

int run_attn_main(const hstu_attn_desc* d, const hstu_jagged* jb, const void* q, int64_t ldq, const void* k,
                  int64_t ldk, const void* v, int64_t ldv, const float* pos_bias, const float* time_bias, void* out,
                  int64_t ldo, const AttnWs& w, cudaStream_t st) {
  AttnFwdParams p;
  memset(&p, 0, sizeof(p));
  p.seq_offsets = jb->seq_offsets;
  p.num_targets = jb->num_targets;
  p.timestamps = jb->timestamps;
  p.q = q; p.ldq = ldq; p.k = k; p.ldk = ldk; p.v = v; p.ldv = ldv;
  p.out = out; p.ldo = ldo;
  p.pos_bias = pos_bias; p.time_bias = time_bias;
  p.rab_head_stride = d->rab_head_stride;
  p.num_heads = d->num_heads;
  p.total_rows = jb->total_tokens;
  p.thr = thresholds_for(d->time_div);
  p.items = w.items;
  p.item_count = w.count;
  p.status = w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  p.tile_base = w.tile_base;
  p.tile_recs = w.tile_recs;
  p.item_cursor = w.count + 1;
  p.band = w.band;
  if (use_tc(d)) {
    TraceScope tr("attn_fwd_tc", st);
    HSTU_CUDA(launch_attn_fwd_tc(p, d->dqk, tc_attn_grid(w.capacity), st, d->time_div));
  } else {
    TraceScope tr("attn_fwd_simt", st);
    int grid = w.capacity < 148 * 4 ? (w.capacity > 0 ? w.capacity : 1) : 148 * 4;
    HSTU_CUDA(launch_attn_fwd_simt(p, d->dtype, d->dqk, grid, st));
  }
  return HSTU_OK;
}

int run_attn_fwd(const hstu_attn_desc* d, const hstu_jagged* jb, const void* q, int64_t ldq, const void* k,
                 int64_t ldk, const void* v, int64_t ldv, const float* pos_bias, const float* time_bias, void* out,
                 int64_t ldo, const AttnWs& w, cudaStream_t st) {
  HSTU_TRY(run_attn_prep(d, jb, pos_bias, time_bias, w, st));
  return run_attn_main(d, jb, q, ldq, k, ldk, v, ldv, pos_bias, time_bias, out, ldo, w, st);
}

// ---------------------------------------------------------------- side stream
// One non-blocking stream per device on which the layer forward runs the
// attention preparation while LayerNorm1 and f1 run on the caller's stream;
// fork and join through events.  Record-and-wait pairs are made under a mutex;
// a join that waits for a later record (another caller's) still implies this
// caller's work, which precedes it on the same in-order stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
SideStream g_side[kMaxDevices];

int side_stream(SideStream** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
  SideStream& ss = g_side[dev];
  if (!ss.s) {
    SideStream n;   // becomes the device's only once every handle exists
    HSTU_CUDA(cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking));
    HSTU_CUDA(cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming));
    HSTU_CUDA(cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming));
    ss = n;
  }
  *out = &ss;
  return HSTU_OK;
}

// The attention backward's preparation: the work list (unless reused), the
// timestamp records, the band of bias and bucket words and the cleared dQ
// accumulator.  It needs only the batch and the bias tables, so the layer backward
// runs it on the side stream next to its first GEMMs.
int run_attn_bwd_prep(const hstu_attn_desc* d, const hstu_jagged* jb, const float* pos_bias,
                      const float* time_bias, const AttnWs& w, cudaStream_t st) {
  const int tile = attn_bwd_tile(d);
  const int H = d->num_heads, dh = d->dqk;
  const bool tc = use_tc_bwd(d);
  const Thresholds thr = thresholds_for(d->time_div);
  const bool reuse = (d->flags & HSTU_FLAG_REUSE_PREP) != 0;
  if (reuse) {
    // work list and tile records from an earlier call: only the fetch cursor restarts
    HSTU_CUDA(cudaMemsetAsync(w.count + 1, 0, sizeof(int32_t), st));
  } else {
    TraceScope tr("sched_bwd", st);
    HSTU_CUDA(launch_build_work_list(jb->seq_offsets, jb->num_targets, jb->batch, jb->total_tokens, H, tile, tile, 1,
                                     w.capacity, w.items, w.count, w.status, st, tc ? w.tile_base : nullptr));
  }
  if (tc) {
    TraceScope tr("bwd_prep", st);
    if (!reuse)
      HSTU_CUDA(launch_ts_tiles(jb->seq_offsets, jb->timestamps, jb->batch, w.tile_base, w.tiles_cap, w.tile_recs, st));
    if (w.band)
      HSTU_CUDA(launch_bwd_band(jb->seq_offsets, jb->num_targets, jb->timestamps, jb->batch, jb->total_tokens,
                                w.tile_base, w.tiles_cap, pos_bias, time_bias, thr, d->time_div, w.status,
                                (uint32_t*)w.band, st));
  }
  HSTU_CUDA(cudaMemsetAsync(w.dq_accum, 0, sizeof(float) * (size_t)jb->total_tokens * H * dh, st));
  return HSTU_OK;
}

// the attention backward proper, after run_attn_bwd_prep on the same workspace
int run_attn_bwd_main(const hstu_attn_desc* d, const hstu_jagged* jb, const void* q, int64_t ldq, const void* k,
                      int64_t ldk, const void* v, int64_t ldv, const float* pos_bias, const float* time_bias,
                      const void* dout, int64_t lddo, void* dq, int64_t lddq, void* dk, int64_t lddk, void* dv,
                      int64_t lddv, float* dpos, float* dtime, const AttnWs& w, cudaStream_t st) {
  const int H = d->num_heads, dh = d->dqk;
  const bool tc = use_tc_bwd(d);
  const Thresholds thr = thresholds_for(d->time_div);
  AttnBwdParams p;
  memset(&p, 0, sizeof(p));
  p.seq_offsets = jb->seq_offsets;
  p.num_targets = jb->num_targets;
  p.timestamps = jb->timestamps;
  p.q = q; p.ldq = ldq; p.k = k; p.ldk = ldk; p.v = v; p.ldv = ldv;
  p.dout = dout; p.lddo = lddo;
  p.dq_accum = w.dq_accum;
  p.dk = dk; p.lddk = lddk; p.dv = dv; p.lddv = lddv;
  p.pos_bias = pos_bias; p.time_bias = time_bias;
  p.d_pos_bias = dpos; p.d_time_bias = dtime;
  p.rab_head_stride = d->rab_head_stride;
  p.num_heads = H;
  p.total_rows = jb->total_tokens;
  p.thr = thr;
  p.items = w.items;
  p.item_count = w.count;
  p.status = w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  p.tile_base = w.tile_base;
  p.tile_recs = w.tile_recs;
  p.band = (const uint32_t*)w.band;
  p.item_cursor = w.count + 1;
  p.rab_partial = w.rab_partial;
  p.rab_tables = w.rab_tables;
  if (tc) {
    const int grid = std::min(tc_attn_grid(w.capacity), kMaxBwdCtas);
    HSTU_CUDA(cudaMemsetAsync(w.rab_partial, 0, sizeof(float) * (size_t)grid * w.rab_tables * 2 * kNumBuckets, st));
    {
      TraceScope tr("attn_bwd_tc", st);
      HSTU_CUDA(launch_attn_bwd_tc(p, grid, st, d->time_div));
    }
    HSTU_CUDA(launch_rab_reduce(w.rab_partial, grid, w.rab_tables, d->rab_head_stride, dpos, dtime, st));
  } else {
    TraceScope tr("attn_bwd_simt", st);
    const int grid = w.capacity < 148 * 2 ? (w.capacity > 0 ? w.capacity : 1) : 148 * 2;
    HSTU_CUDA(launch_attn_bwd_simt(p, d->dtype, dh, grid, st));
  }
  if (dq) {   // (without dq the caller reads the fp32 accumulator w.dq_accum itself)
    TraceScope tr("dq_finalize", st);
    HSTU_CUDA(launch_dq_finalize(w.dq_accum, jb->seq_offsets, jb->batch, H, dh, d->dtype, dq, lddq, 148 * 8, st));
  }
  return HSTU_OK;
}

int run_attn_bwd(const hstu_attn_desc* d, const hstu_jagged* jb, const void* q, int64_t ldq, const void* k,
                 int64_t ldk, const void* v, int64_t ldv, const float* pos_bias, const float* time_bias,
                 const void* dout, int64_t lddo, void* dq, int64_t lddq, void* dk, int64_t lddk, void* dv,
                 int64_t lddv, float* dpos, float* dtime, const AttnWs& w, cudaStream_t st) {
  HSTU_TRY(run_attn_bwd_prep(d, jb, pos_bias, time_bias, w, st));
  return run_attn_bwd_main(d, jb, q, ldq, k, ldk, v, ldv, pos_bias, time_bias, dout, lddo, dq, lddq, dk, lddk, dv,
                           lddv, dpos, dtime, w, st);
}

// ---------------------------------------------------------------- GEMM dispatch
int gemm(const GemmParams& p, int dtype, int flags, cudaStream_t st, const char* name) {
  if (!(flags & HSTU_FLAG_FORCE_SIMT) && tc_gemm_supported(p, dtype)) {
    TraceScope tr(name, st);
    return cuda_status(launch_gemm_tc(p, st));
  }
  TraceScope tr(name, st);
  return cuda_status(launch_gemm_simt(p, dtype, st));
}

// ---------------------------------------------------------------- layer
int check_layer(const hstu_layer_desc* d, const hstu_layer_weights* w) {
  if (!d || !w) return HSTU_ERR_INVALID_ARG;
  HSTU_TRY(check_attn_desc(&d->attn));
  const int dm = d->d_model, hv = d->attn.num_heads * d->attn.dv;
  if (dm < 8 || dm > 1024 || dm % 8) return HSTU_ERR_UNSUPPORTED;
  if (hv > 1024 || hv % 8) return HSTU_ERR_UNSUPPORTED;
  if (!(d->ln_eps >= 0.f)) return HSTU_ERR_INVALID_ARG;
  if (d->io_dtype != HSTU_DTYPE_F32 && d->io_dtype != d->attn.dtype) return HSTU_ERR_UNSUPPORTED;
  if (d->reserved != 0) return HSTU_ERR_INVALID_ARG;
  const void* ptrs[] = {w->w1, w->b1, w->ln1_gamma, w->ln1_beta, w->ln2_gamma, w->ln2_beta,
                        w->w2, w->b2, w->pos_bias, w->time_bias};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

struct LayerBufs {
  void* xhat; float* mu1; float* rs1; void* z; void* uvqk; void* o; float* mu2; float* rs2; void* g;
};

struct LayerFwdWs {
  AttnWs attn;
  LayerBufs b;
};

LayerFwdWs carve_layer_fwd(Carver& c, const hstu_layer_desc* d, int B, int T, bool need_all) {
  LayerFwdWs w;
  w.attn = carve_attn(c, &d->attn, B, T, false);
  const size_t es = elem_size(d->attn.dtype);
  const int dm = d->d_model, hv = d->attn.num_heads * d->attn.dv;
  (void)need_all;
  w.b.xhat = c.take<char>((size_t)T * dm * es);
  w.b.mu1 = c.take<float>(T);
  w.b.rs1 = c.take<float>(T);
  w.b.z = nullptr;
  w.b.uvqk = c.take<char>((size_t)T * 4 * hv * es);
  w.b.o = c.take<char>((size_t)T * hv * es);
  w.b.mu2 = c.take<float>(T);
  w.b.rs2 = c.take<float>(T);
  w.b.g = c.take<char>((size_t)T * hv * es);
  return w;
}

int run_layer_fwd(const hstu_layer_desc* d, const hstu_layer_weights* w, const hstu_jagged* jb, const void* x,
                  void* y, const hstu_layer_saved* saved, const LayerFwdWs& ws, cudaStream_t st) {
  const int dt = d->attn.dtype;
  const int dm = d->d_model, H = d->attn.num_heads, dh = d->attn.dv, hv = H * dh;
  const int T = jb->total_tokens;
  const int32_t* rows = jb->seq_offsets + jb->batch;  // device row count
  LayerBufs b = ws.b;
  if (saved) {
    b.xhat = saved->xhat; b.mu1 = saved->ln1_mean; b.rs1 = saved->ln1_rstd; b.z = saved->z;
    b.uvqk = saved->uvqk; b.o = saved->attn_out; b.mu2 = saved->ln2_mean; b.rs2 = saved->ln2_rstd;
    if (saved->gate) b.g = saved->gate;
  }
  // attention preparation on the side stream, overlapping LayerNorm1 and f1.  The
  // side stream is shared by every caller on the device, so a stream that is being
  // captured into a graph keeps the preparation on itself: the shared stream must
  // not join one caller's capture while other callers enqueue work on it.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  HSTU_CUDA(cudaStreamIsCapturing(st, &cap));
  SideStream* side = nullptr;
  if (cap == cudaStreamCaptureStatusNone) {
    std::lock_guard<std::mutex> lk(g_side_mu);
    HSTU_TRY(side_stream(&side));
    HSTU_CUDA(cudaEventRecord(side->fork, st));
    HSTU_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    HSTU_TRY(run_attn_prep(&d->attn, jb, w->pos_bias, w->time_bias, ws.attn, side->s));
    HSTU_CUDA(cudaEventRecord(side->join, side->s));
  } else {
    HSTU_TRY(run_attn_prep(&d->attn, jb, w->pos_bias, w->time_bias, ws.attn, st));
  }
  // (A1) LayerNorm1
  {
    TraceScope tr("ln1", st);
    HSTU_CUDA(launch_layer_norm(x, dm, d->io_dtype, w->ln1_gamma, w->ln1_beta, d->ln_eps, b.xhat, dm, dt, b.mu1,
                                b.rs1, T, rows, dm, st));
  }
  // (A1) f1 + SiLU, split layout U | V | Q | K
  GemmParams g1;
  memset(&g1, 0, sizeof(g1));
  g1.M = T; g1.N = 4 * hv; g1.K = dm;
  g1.A = b.xhat; g1.sam = dm; g1.sak = 1;
  g1.B = w->w1; g1.sbn = dm; g1.sbk = 1;
  g1.epi = EPI_BIAS_SILU; g1.bias = w->b1;
  g1.out = b.uvqk; g1.ldo = 4 * hv;
  g1.out2 = b.z; g1.ldo2 = 4 * hv;
  g1.rows_dev = rows;
  g1.status = ws.attn.status;
  HSTU_TRY(gemm(g1, dt, d->attn.flags, st, "gemm_f1_silu"));
  // (A2-A4) attention
  const size_t es = elem_size(dt);
  const char* uvqk = (const char*)b.uvqk;
  if (side) HSTU_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  HSTU_TRY(run_attn_main(&d->attn, jb, uvqk + 2 * hv * es, 4 * hv, uvqk + 3 * hv * es, 4 * hv, uvqk + 1 * hv * es,
                         4 * hv, w->pos_bias, w->time_bias, b.o, hv, ws.attn, st));
  // (A5) LayerNorm2(A V) * U
  {
    TraceScope tr("ln2_gate", st);
    HSTU_CUDA(launch_ln_gate(b.o, hv, b.uvqk, 4 * hv, w->ln2_gamma, w->ln2_beta, d->ln_eps, b.g, hv, b.mu2,
                             b.rs2, T, rows, hv, dt, st));
  }
  // (A6) f2 + residual
  GemmParams g2;
  memset(&g2, 0, sizeof(g2));
  g2.M = T; g2.N = dm; g2.K = hv;
  g2.A = b.g; g2.sam = hv; g2.sak = 1;
  g2.B = w->w2; g2.sbn = hv; g2.sbk = 1;
  g2.epi = EPI_BIAS_RESIDUAL; g2.bias = w->b2;
  g2.residual = x; g2.ldr = dm;
  g2.out = y; g2.ldo = dm;
  g2.rows_dev = rows;
  g2.res_f32 = d->io_dtype == HSTU_DTYPE_F32;
  g2.out_f32 = d->io_dtype == HSTU_DTYPE_F32;
  g2.status = ws.attn.status;
  HSTU_TRY(gemm(g2, dt, d->attn.flags, st, "gemm_f2_residual"));
  return HSTU_OK;
}

// backward workspace: attention bwd scratch + gradients of the intermediates
struct LayerBwdWs {
  AttnWs attn;
  void* g;       // [T, hv] recomputed gate output
  void* dg;      // [T, hv]
  void* d_o;     // [T, hv]
  void* duvqk;   // [T, 4hv]
  void* dz;      // [T, 4hv]
  float* dxhat;  // [T, dm] fp32
  void* dyb;     // [T, dm] dy in the activation dtype, zero-padded to a multiple of 64 rows
  float* colpart;  // column partial sums (db2 with dy's conversion, db1 with the SiLU backward)
};

LayerBwdWs carve_layer_bwd(Carver& c, const hstu_layer_desc* d, int B, int T) {
  LayerBwdWs w;
  w.attn = carve_attn(c, &d->attn, B, T, true);
  const size_t es = elem_size(d->attn.dtype);
  const int dm = d->d_model, hv = d->attn.num_heads * d->attn.dv;
  w.g = c.take<char>((size_t)T * hv * es);
  w.dg = c.take<char>((size_t)T * hv * es);
  w.d_o = c.take<char>((size_t)T * hv * es);
  w.duvqk = c.take<char>((size_t)T * 4 * hv * es);
  w.dz = c.take<char>((size_t)T * 4 * hv * es);
  w.dxhat = c.take<float>((size_t)T * dm);
  w.dyb = c.take<char>((size_t)T * dm * es);
  w.colpart = c.take<float>(col_partials_size(4 * hv > dm ? 4 * hv : dm));
  return w;
}

int run_layer_bwd(const hstu_layer_desc* d, const hstu_layer_weights* w, const hstu_jagged* jb, const void* x,
                  const hstu_layer_saved* sv, const void* dy, void* dx, const hstu_layer_grads* gr,
                  const LayerBwdWs& ws, cudaStream_t st) {
  const int dt = d->attn.dtype;
  const int io = d->io_dtype;
  const int dm = d->d_model, H = d->attn.num_heads, dh = d->attn.dv, hv = H * dh;
  const int T = jb->total_tokens;
  const int32_t* rows = jb->seq_offsets + jb->batch;
  const size_t es = elem_size(dt);
  const int fl = d->attn.flags;
  void* duvqk = gr->duvqk ? gr->duvqk : ws.duvqk;
  void* gate = sv->gate ? sv->gate : ws.g;
  int32_t* status = ws.attn.status;
  // without a caller buffer for dU|dV|dQ|dK, the SiLU' pass reads dQ from the
  // attention's fp32 accumulator (no conversion pass)
  const bool dq_direct = !gr->duvqk && hv % 8 == 0;
  // the attention backward's preparation on the side stream, next to the GEMMs
  // and row kernels before the attention (a stream being captured keeps it, as
  // in the forward)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  HSTU_CUDA(cudaStreamIsCapturing(st, &cap));
  SideStream* side = nullptr;
  if (cap == cudaStreamCaptureStatusNone) {
    std::lock_guard<std::mutex> lk(g_side_mu);
    HSTU_TRY(side_stream(&side));
    HSTU_CUDA(cudaEventRecord(side->fork, st));
    HSTU_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    HSTU_TRY(run_attn_bwd_prep(&d->attn, jb, w->pos_bias, w->time_bias, ws.attn, side->s));
    HSTU_CUDA(cudaEventRecord(side->join, side->s));
  } else {
    HSTU_TRY(run_attn_bwd_prep(&d->attn, jb, w->pos_bias, w->time_bias, ws.attn, st));
  }
  // The weight-gradient products reduce over tokens in 64-row slices: rows from the
  // device row count up to the next multiple of 64 of every token-major operand are zeroed.
  {
    TraceScope tr("bwd_prep", st);
    HSTU_CUDA(launch_convert_rows_colsum(dy, dm, io, ws.dyb, dm, dt, dm, T, rows, 64, gr->db2, ws.colpart, st));
    HSTU_CUDA(launch_zero_tail_rows(sv->xhat, (int64_t)dm * es, (int64_t)dm * es, T, rows, 64, st));
    // g = LN2(o) * U as the forward kept it, or recomputed
    if (!sv->gate)
      HSTU_CUDA(launch_ln_gate(sv->attn_out, hv, sv->uvqk, 4 * hv, w->ln2_gamma, w->ln2_beta, d->ln_eps, ws.g, hv,
                               nullptr, nullptr, T, rows, hv, dt, st));
    HSTU_CUDA(launch_zero_tail_rows(gate, (int64_t)hv * es, (int64_t)hv * es, T, rows, 64, st));
  }
  // y = x + g W2^T + b2:  dW2 = dy^T g, dg = dy W2 (db2 = colsum(dy) came with dy's conversion)
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = dm; p.N = hv; p.K = T;                 // dW2[m=out, n=in] = sum_t dy[t, m] g[t, n]
  p.A = ws.dyb; p.sam = 1; p.sak = dm;
  p.B = gate; p.sbn = 1; p.sbk = hv;
  p.epi = EPI_STORE_F32; p.out = gr->dw2; p.ldo = hv; p.k_dev = rows; p.status = status;
  HSTU_TRY(gemm(p, dt, fl, st, "gemm_dw2"));
  memset(&p, 0, sizeof(p));
  p.M = T; p.N = hv; p.K = dm;                 // dg[t, n] = sum_m dy[t, m] W2[m, n]
  p.A = ws.dyb; p.sam = dm; p.sak = 1;
  p.B = w->w2; p.sbn = 1; p.sbk = hv;
  p.epi = EPI_STORE; p.out = ws.dg; p.ldo = hv; p.rows_dev = rows; p.status = status;
  HSTU_TRY(gemm(p, dt, fl, st, "gemm_dg"));
  // g = (LN2(o) gamma2 + beta2) * U:  dU, d_o, dgamma2, dbeta2
  {
    TraceScope tr("ln2_gate_bwd", st);
    HSTU_CUDA(cudaMemsetAsync(gr->dln2_gamma, 0, sizeof(float) * hv, st));
    HSTU_CUDA(cudaMemsetAsync(gr->dln2_beta, 0, sizeof(float) * hv, st));
    HSTU_CUDA(launch_ln_gate_bwd(sv->attn_out, hv, sv->uvqk, 4 * hv, w->ln2_gamma, w->ln2_beta, sv->ln2_mean,
                                 sv->ln2_rstd, ws.dg, hv, ws.d_o, hv, duvqk, 4 * hv, gr->dln2_gamma,
                                 gr->dln2_beta, T, rows, hv, dt, st));
  }
  // attention backward -> dV, dQ, dK columns of duvqk, rab grads
  const size_t rab_n = (size_t)(d->attn.rab_head_stride ? H : 1) * kNumBuckets;
  HSTU_CUDA(cudaMemsetAsync(gr->dpos_bias, 0, sizeof(float) * rab_n, st));
  HSTU_CUDA(cudaMemsetAsync(gr->dtime_bias, 0, sizeof(float) * rab_n, st));
  const char* uvqk = (const char*)sv->uvqk;
  char* du = (char*)duvqk;
  if (side) HSTU_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  HSTU_TRY(run_attn_bwd_main(&d->attn, jb, uvqk + 2 * hv * es, 4 * hv, uvqk + 3 * hv * es, 4 * hv, uvqk + hv * es,
                             4 * hv, w->pos_bias, w->time_bias, ws.d_o, hv, dq_direct ? nullptr : du + 2 * hv * es,
                             4 * hv, du + 3 * hv * es, 4 * hv, du + hv * es, 4 * hv, gr->dpos_bias, gr->dtime_bias,
                             ws.attn, st));
  // a = SiLU(z): dz = da * SiLU'(z), and in the same pass db1 = colsum(dz)
  {
    TraceScope tr("silu_bwd", st);
    HSTU_CUDA(launch_silu_bwd_colsum(duvqk, sv->z, ws.dz, 4 * hv, T, rows, 4 * hv, dt, gr->db1, ws.colpart, st,
                                     dq_direct ? ws.attn.dq_accum : nullptr, hv, 2 * hv, hv));
    HSTU_CUDA(launch_zero_tail_rows(ws.dz, (int64_t)4 * hv * es, (int64_t)4 * hv * es, T, rows, 64, st));
  }
  // z = xhat W1^T + b1: dW1 = dz^T xhat, dxhat = dz W1
  memset(&p, 0, sizeof(p));
  p.M = 4 * hv; p.N = dm; p.K = T;
  p.A = ws.dz; p.sam = 1; p.sak = 4 * hv;
  p.B = sv->xhat; p.sbn = 1; p.sbk = dm;
  p.epi = EPI_STORE_F32; p.out = gr->dw1; p.ldo = dm; p.k_dev = rows; p.status = status;
  HSTU_TRY(gemm(p, dt, fl, st, "gemm_dw1"));
  memset(&p, 0, sizeof(p));
  p.M = T; p.N = dm; p.K = 4 * hv;
  p.A = ws.dz; p.sam = 4 * hv; p.sak = 1;
  p.B = w->w1; p.sbn = 1; p.sbk = dm;
  p.epi = EPI_STORE_F32; p.out = ws.dxhat; p.ldo = dm; p.rows_dev = rows; p.status = status;
  HSTU_TRY(gemm(p, dt, fl, st, "gemm_dxhat"));
  // xhat = LN1(x): dx = dy + LN1 backward
  {
    TraceScope tr("ln1_bwd", st);
    HSTU_CUDA(cudaMemsetAsync(gr->dln1_gamma, 0, sizeof(float) * dm, st));
    HSTU_CUDA(cudaMemsetAsync(gr->dln1_beta, 0, sizeof(float) * dm, st));
    HSTU_CUDA(launch_ln_bwd(x, dm, w->ln1_gamma, sv->ln1_mean, sv->ln1_rstd, ws.dxhat, dm, dy, dm, dx, dm,
                            gr->dln1_gamma, gr->dln1_beta, T, rows, dm, io, st));
  }
  return HSTU_OK;
}

}  // namespace

// =============================================================================
// exported entry points
// =============================================================================
extern "C" {

const char* hstu_status_string(int status) {
  switch (status) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARG: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported configuration";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_TIMEOUT: return "device wait timed out";
    case HSTU_ERR_WORKSPACE: return "workspace too small";
    case HSTU_ERR_BAD_OFFSETS: return "invalid sequence offsets or target counts";
    default: return "unknown status";
  }
}

int hstu_version(void) { return kVersion; }

const char* hstu_last_cuda_error(void) { return g_last_error; }

int hstu_build_time_thresholds(double time_div, int32_t num_buckets, int64_t* out) {
  if (!out || !(time_div > 0.0) || !isfinite(time_div) || num_buckets < 2 || num_buckets > 1024)
    return HSTU_ERR_INVALID_ARG;
  build_thresholds(time_div, num_buckets, out);
  return HSTU_OK;
}

int hstu_workspace_status(const void* workspace, int32_t* status, void* stream) {
  if (!workspace || !status) return HSTU_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  HSTU_CUDA(cudaMemcpyAsync(status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  HSTU_CUDA(cudaStreamSynchronize(st));
  return HSTU_OK;
}

int hstu_attn_fwd_workspace_size(const hstu_attn_desc* desc, int32_t batch, int32_t total_tokens, size_t* bytes) {
  HSTU_TRY(check_attn_desc(desc));
  if (!bytes || batch < 0 || total_tokens < 0) return HSTU_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_attn(c, desc, batch, total_tokens, false);
  *bytes = c.size();
  return HSTU_OK;
}

int hstu_attn_fwd(const hstu_attn_desc* desc, const hstu_jagged* jb, const void* q, int64_t ldq, const void* k,
                  int64_t ldk, const void* v, int64_t ldv, const float* pos_bias, const float* time_bias, void* out,
                  int64_t ldo, void* workspace, size_t workspace_bytes, void* stream) {
  HSTU_TRY(check_attn_desc(desc));
  HSTU_TRY(check_jagged(jb));
  const int hd = desc->num_heads * desc->dqk;
  HSTU_TRY(check_rows(q, ldq, hd, desc->dtype));
  HSTU_TRY(check_rows(k, ldk, hd, desc->dtype));
  HSTU_TRY(check_rows(v, ldv, hd, desc->dtype));
  HSTU_TRY(check_rows(out, ldo, hd, desc->dtype));
  if (!pos_bias || !time_bias) return HSTU_ERR_INVALID_ARG;
  size_t need;
  HSTU_TRY(hstu_attn_fwd_workspace_size(desc, jb->batch, jb->total_tokens, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(workspace);
  AttnWs w = carve_attn(c, desc, jb->batch, jb->total_tokens, false);
  HSTU_CUDA(cudaMemsetAsync(w.status, 0, kStatusBytes, st));
  return run_attn_fwd(desc, jb, q, ldq, k, ldk, v, ldv, pos_bias, time_bias, out, ldo, w, st);
}

int hstu_attn_bwd_workspace_size(const hstu_attn_desc* desc, int32_t batch, int32_t total_tokens, size_t* bytes) {
  HSTU_TRY(check_attn_desc(desc));
  if (!bytes || batch < 0 || total_tokens < 0) return HSTU_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_attn(c, desc, batch, total_tokens, true);
  *bytes = c.size();
  return HSTU_OK;
}

int hstu_attn_bwd(const hstu_attn_desc* desc, const hstu_jagged* jb, const void* q, int64_t ldq, const void* k,
                  int64_t ldk, const void* v, int64_t ldv, const float* pos_bias, const float* time_bias,
                  const void* dout, int64_t lddo, void* dq, int64_t lddq, void* dk, int64_t lddk, void* dv,
                  int64_t lddv, float* d_pos_bias, float* d_time_bias, void* workspace, size_t workspace_bytes,
                  void* stream) {
  HSTU_TRY(check_attn_desc(desc));
  HSTU_TRY(check_jagged(jb));
  const int hd = desc->num_heads * desc->dqk;
  HSTU_TRY(check_rows(q, ldq, hd, desc->dtype));
  HSTU_TRY(check_rows(k, ldk, hd, desc->dtype));
  HSTU_TRY(check_rows(v, ldv, hd, desc->dtype));
  HSTU_TRY(check_rows(dout, lddo, hd, desc->dtype));
  HSTU_TRY(check_rows(dq, lddq, hd, desc->dtype));
  HSTU_TRY(check_rows(dk, lddk, hd, desc->dtype));
  HSTU_TRY(check_rows(dv, lddv, hd, desc->dtype));
  if (!pos_bias || !time_bias || !d_pos_bias || !d_time_bias) return HSTU_ERR_INVALID_ARG;
  size_t need;
  HSTU_TRY(hstu_attn_bwd_workspace_size(desc, jb->batch, jb->total_tokens, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(workspace);
  AttnWs w = carve_attn(c, desc, jb->batch, jb->total_tokens, true);
  HSTU_CUDA(cudaMemsetAsync(w.status, 0, kStatusBytes, st));
  return run_attn_bwd(desc, jb, q, ldq, k, ldk, v, ldv, pos_bias, time_bias, dout, lddo, dq, lddq, dk, lddk, dv,
                      lddv, d_pos_bias, d_time_bias, w, st);
}

int hstu_layer_fwd_workspace_size(const hstu_layer_desc* desc, int32_t batch, int32_t total_tokens, size_t* bytes) {
  if (!desc || !bytes || batch < 0 || total_tokens < 0) return HSTU_ERR_INVALID_ARG;
  HSTU_TRY(check_attn_desc(&desc->attn));
  Carver c(nullptr);
  carve_layer_fwd(c, desc, batch, total_tokens, true);
  *bytes = c.size();
  return HSTU_OK;
}

int hstu_layer_fwd(const hstu_layer_desc* desc, const hstu_layer_weights* w, const hstu_jagged* jb, const void* x,
                   void* y, const hstu_layer_saved* saved, void* workspace, size_t workspace_bytes, void* stream) {
  HSTU_TRY(check_layer(desc, w));
  HSTU_TRY(check_jagged(jb));
  const int dm = desc->d_model;
  const int io = desc->io_dtype;
  HSTU_TRY(check_rows(x, dm, dm, io));
  HSTU_TRY(check_rows(y, dm, dm, io));
  if (x == y) return HSTU_ERR_INVALID_ARG;
  if (saved) {
    const void* ps[] = {saved->xhat, saved->ln1_mean, saved->ln1_rstd, saved->z, saved->uvqk,
                        saved->attn_out, saved->ln2_mean, saved->ln2_rstd};
    for (const void* p : ps)
      if (!p || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
    if (saved->gate && !aligned16(saved->gate)) return HSTU_ERR_INVALID_ARG;
  }
  size_t need;
  HSTU_TRY(hstu_layer_fwd_workspace_size(desc, jb->batch, jb->total_tokens, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(workspace);
  LayerFwdWs ws = carve_layer_fwd(c, desc, jb->batch, jb->total_tokens, true);
  HSTU_CUDA(cudaMemsetAsync(ws.attn.status, 0, kStatusBytes, st));
  if ((desc->attn.flags & HSTU_FLAG_SHORT_SEQUENCES) && !saved &&
      fused_short_supported(dm, desc->attn.num_heads, desc->attn.dqk, desc->attn.dtype, io) &&
      desc->attn.dv == desc->attn.dqk) {
    // the whole layer in one kernel, over units of at most 128 token rows holding whole sequences
    FusedShortArgs a;
    memset(&a, 0, sizeof(a));
    a.offs = jb->seq_offsets; a.num_targets = jb->num_targets; a.ts = jb->timestamps;
    a.x = x; a.y = y;
    a.w1 = w->w1; a.b1 = w->b1; a.ln1_g = w->ln1_gamma; a.ln1_b = w->ln1_beta;
    a.ln2_g = w->ln2_gamma; a.ln2_b = w->ln2_beta; a.w2 = w->w2; a.b2 = w->b2;
    a.pos_bias = w->pos_bias; a.time_bias = w->time_bias; a.rab_head_stride = desc->attn.rab_head_stride;
    a.B = jb->batch; a.T = jb->total_tokens; a.d = dm; a.H = desc->attn.num_heads;
    a.eps = desc->ln_eps; a.time_div = desc->attn.time_div; a.thr = thresholds_for(desc->attn.time_div);
    a.cursor = ws.attn.count + 2;
    a.status = ws.attn.status;
    a.timeout_ns = kDefaultTimeoutNs;
    HSTU_CUDA(cudaMemsetAsync(a.cursor, 0, sizeof(int32_t), st));
    TraceScope tr("fused_short_layer", st);
    HSTU_CUDA(launch_fused_short(a, st));
    return HSTU_OK;
  }
  return run_layer_fwd(desc, w, jb, x, y, saved, ws, st);
}

// ---------------------------------------------------------------- layer forward from host memory
namespace {
constexpr int kMaxChunks = 64;

// Per device: one copy stream each way and the events that chain a call's
// chunks; a call enqueues under the mutex, so calls do not share events while
// they are being recorded.
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kMaxChunks] = {}, out[kMaxChunks] = {};
};
std::mutex g_copy_mu;
CopyStreams g_copy[kMaxDevices];

int copy_streams(CopyStreams** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
  CopyStreams& cs = g_copy[dev];
  if (!cs.h2d) {
    // created into a copy that becomes the device's only once every handle exists
    CopyStreams n;
    HSTU_CUDA(cudaStreamCreateWithFlags(&n.h2d, cudaStreamNonBlocking));
    HSTU_CUDA(cudaStreamCreateWithFlags(&n.d2h, cudaStreamNonBlocking));
    HSTU_CUDA(cudaEventCreateWithFlags(&n.start, cudaEventDisableTiming));
    HSTU_CUDA(cudaEventCreateWithFlags(&n.done, cudaEventDisableTiming));
    for (int i = 0; i < kMaxChunks; ++i) {
      HSTU_CUDA(cudaEventCreateWithFlags(&n.in[i], cudaEventDisableTiming));
      HSTU_CUDA(cudaEventCreateWithFlags(&n.out[i], cudaEventDisableTiming));
    }
    cs = n;
  }
  *out = &cs;
  return HSTU_OK;
}

struct HostFwdWs {
  LayerFwdWs layer;
  void* x;            // [T, d] io_dtype
  void* y;            // [T, d]
  int64_t* ts;        // [T]
  int32_t* offs;      // [B+1] as given
  int32_t* nt;        // [B]
  int32_t* chunk_offs;  // kMaxChunks x [B+1], rebased per chunk
};

HostFwdWs carve_host_fwd(Carver& c, const hstu_layer_desc* d, int B, int T) {
  HostFwdWs w;
  w.layer = carve_layer_fwd(c, d, B, T, true);
  const size_t eio = elem_size(d->io_dtype);
  w.x = c.take<char>((size_t)T * d->d_model * eio);
  w.y = c.take<char>((size_t)T * d->d_model * eio);
  w.ts = c.take<int64_t>(T > 0 ? T : 1);
  w.offs = c.take<int32_t>((size_t)B + 1);
  w.nt = c.take<int32_t>(B > 0 ? B : 1);
  w.chunk_offs = c.take<int32_t>((size_t)kMaxChunks * (B + 1));
  return w;
}
}  // namespace

int hstu_layer_fwd_host_workspace_size(const hstu_layer_desc* desc, int32_t batch, int32_t total_tokens,
                                       int32_t num_chunks, size_t* bytes) {
  if (!desc || !bytes || batch < 0 || total_tokens < 0 || num_chunks < 1) return HSTU_ERR_INVALID_ARG;
  HSTU_TRY(check_attn_desc(&desc->attn));
  Carver c(nullptr);
  carve_host_fwd(c, desc, batch, total_tokens);
  *bytes = c.size();
  return HSTU_OK;
}

int hstu_layer_fwd_host(const hstu_layer_desc* desc, const hstu_layer_weights* w, int32_t batch,
                        const int32_t* seq_offsets, const int32_t* num_targets, const int64_t* timestamps,
                        const void* x, void* y, int32_t num_chunks, void* workspace, size_t workspace_bytes,
                        void* stream) {
  HSTU_TRY(check_layer(desc, w));
  if (batch < 0 || num_chunks < 1 || !seq_offsets || !x || !y) return HSTU_ERR_INVALID_ARG;
  if (seq_offsets[0] != 0) return HSTU_ERR_INVALID_ARG;
  for (int s = 0; s < batch; ++s)
    if (seq_offsets[s + 1] < seq_offsets[s]) return HSTU_ERR_INVALID_ARG;
  const int T = seq_offsets[batch];
  if (T > 0 && !timestamps) return HSTU_ERR_INVALID_ARG;
  size_t need;
  HSTU_TRY(hstu_layer_fwd_host_workspace_size(desc, batch, T, num_chunks, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(workspace);
  HostFwdWs ws = carve_host_fwd(c, desc, batch, T);
  HSTU_CUDA(cudaMemsetAsync(ws.layer.attn.status, 0, kStatusBytes, st));
  if (batch == 0 || T == 0) return HSTU_OK;
  const int dm = desc->d_model;
  const size_t row_bytes = (size_t)dm * elem_size(desc->io_dtype);
  // chunks of consecutive sequences with about T / nc tokens each
  const int nc = std::min(std::min(num_chunks, batch), kMaxChunks);
  int bounds[kMaxChunks + 1];
  bounds[0] = 0;
  for (int ch = 1, s = 0; ch < nc; ++ch) {
    const int64_t target = (int64_t)T * ch / nc;
    while (s < batch - (nc - ch) && seq_offsets[s + 1] <= target) ++s;
    if (s < bounds[ch - 1] + 1) s = bounds[ch - 1] + 1;
    bounds[ch] = s;
  }
  bounds[nc] = batch;
  std::lock_guard<std::mutex> lk(g_copy_mu);
  CopyStreams* cs = nullptr;
  HSTU_TRY(copy_streams(&cs));
  // the copies may overwrite the workspace only after the stream's earlier work
  HSTU_CUDA(cudaEventRecord(cs->start, st));
  HSTU_CUDA(cudaStreamWaitEvent(cs->h2d, cs->start, 0));
  HSTU_CUDA(cudaStreamWaitEvent(cs->d2h, cs->start, 0));
  HSTU_CUDA(cudaMemcpyAsync(ws.offs, seq_offsets, sizeof(int32_t) * (batch + 1), cudaMemcpyHostToDevice, cs->h2d));
  if (num_targets)
    HSTU_CUDA(cudaMemcpyAsync(ws.nt, num_targets, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, cs->h2d));
  for (int ch = 0; ch < nc; ++ch) {
    const int r0 = seq_offsets[bounds[ch]], r1 = seq_offsets[bounds[ch + 1]];
    if (r1 > r0) {
      HSTU_CUDA(cudaMemcpyAsync((char*)ws.x + r0 * row_bytes, (const char*)x + r0 * row_bytes,
                                (size_t)(r1 - r0) * row_bytes, cudaMemcpyHostToDevice, cs->h2d));
      HSTU_CUDA(cudaMemcpyAsync(ws.ts + r0, timestamps + r0, sizeof(int64_t) * (r1 - r0), cudaMemcpyHostToDevice,
                                cs->h2d));
    }
    HSTU_CUDA(cudaEventRecord(cs->in[ch], cs->h2d));
  }
  // every chunk is a batch of its own: its preparation is built, never reused
  hstu_layer_desc dc = *desc;
  dc.attn.flags &= ~HSTU_FLAG_REUSE_PREP;
  for (int ch = 0; ch < nc; ++ch) {
    const int s0 = bounds[ch], nb = bounds[ch + 1] - s0;
    const int r0 = seq_offsets[s0], r1 = seq_offsets[s0 + nb];
    HSTU_CUDA(cudaStreamWaitEvent(st, cs->in[ch], 0));
    int32_t* co = ws.chunk_offs + (size_t)ch * (batch + 1);
    HSTU_CUDA(launch_rebase_offsets(ws.offs, s0, nb, co, st));
    hstu_jagged jb;
    jb.batch = nb;
    jb.total_tokens = r1 - r0;
    jb.seq_offsets = co;
    jb.num_targets = num_targets ? ws.nt + s0 : nullptr;
    jb.timestamps = ws.ts + r0;
    HSTU_TRY(run_layer_fwd(&dc, w, &jb, (const char*)ws.x + r0 * row_bytes, (char*)ws.y + r0 * row_bytes, nullptr,
                           ws.layer, st));
    HSTU_CUDA(cudaEventRecord(cs->out[ch], st));
    HSTU_CUDA(cudaStreamWaitEvent(cs->d2h, cs->out[ch], 0));
    if (r1 > r0)
      HSTU_CUDA(cudaMemcpyAsync((char*)y + r0 * row_bytes, (const char*)ws.y + r0 * row_bytes,
                                (size_t)(r1 - r0) * row_bytes, cudaMemcpyDeviceToHost, cs->d2h));
  }
  HSTU_CUDA(cudaEventRecord(cs->done, cs->d2h));
  HSTU_CUDA(cudaStreamWaitEvent(st, cs->done, 0));
  return HSTU_OK;
}

int hstu_layer_bwd_workspace_size(const hstu_layer_desc* desc, int32_t batch, int32_t total_tokens, size_t* bytes) {
  if (!desc || !bytes || batch < 0 || total_tokens < 0) return HSTU_ERR_INVALID_ARG;
  HSTU_TRY(check_attn_desc(&desc->attn));
  Carver c(nullptr);
  carve_layer_bwd(c, desc, batch, total_tokens);
  *bytes = c.size();
  return HSTU_OK;
}

int hstu_layer_bwd(const hstu_layer_desc* desc, const hstu_layer_weights* w, const hstu_jagged* jb, const void* x,
                   const hstu_layer_saved* saved, const void* dy, void* dx, const hstu_layer_grads* g,
                   void* workspace, size_t workspace_bytes, void* stream) {
  HSTU_TRY(check_layer(desc, w));
  HSTU_TRY(check_jagged(jb));
  if (!saved || !g) return HSTU_ERR_INVALID_ARG;
  const int dm = desc->d_model;
  const int io = desc->io_dtype;
  HSTU_TRY(check_rows(x, dm, dm, io));
  HSTU_TRY(check_rows(dy, dm, dm, io));
  HSTU_TRY(check_rows(dx, dm, dm, io));
  const void* ps[] = {saved->xhat, saved->ln1_mean, saved->ln1_rstd, saved->z, saved->uvqk, saved->attn_out,
                      saved->ln2_mean, saved->ln2_rstd, g->dw1, g->db1, g->dln1_gamma, g->dln1_beta,
                      g->dln2_gamma, g->dln2_beta, g->dw2, g->db2, g->dpos_bias, g->dtime_bias};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  if (g->duvqk && !aligned16(g->duvqk)) return HSTU_ERR_INVALID_ARG;
  if (saved->gate && !aligned16(saved->gate)) return HSTU_ERR_INVALID_ARG;
  size_t need;
  HSTU_TRY(hstu_layer_bwd_workspace_size(desc, jb->batch, jb->total_tokens, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(workspace);
  LayerBwdWs ws = carve_layer_bwd(c, desc, jb->batch, jb->total_tokens);
  HSTU_CUDA(cudaMemsetAsync(ws.attn.status, 0, kStatusBytes, st));
  return run_layer_bwd(desc, w, jb, x, saved, dy, dx, g, ws, st);
}

// ---------------------------------------------------------------- M-FALCON
// The history rows of a user do not depend on its candidates (they attend only to
// the history), so their K and V are computed once and cached across microbatches
// ("2.3 M-FALCON算法": the history's keys and values are reused by every
// microbatch).  Every user keeps a fixed place in a slot layout,
// [history_u ; bm candidate slots]; microbatch 0 runs the full layer stack over
// it, writing each layer's U|V|Q|K into that layer's cache; every later
// microbatch computes only its candidate rows: LayerNorm1 and f1 on the compact
// candidate rows, their U|V|Q|K scattered into the cache's slot rows, the
// attention over the q tiles of the slots only (keys and values: the cached
// history and the slots), then LayerNorm2 * U and f2 on the compact rows.  The
// rows computed are the same rows as in a full pass over [history ; microbatch],
// with the same reduction order, so the candidates' outputs are too.
namespace {
struct MfalconWs {
  LayerFwdWs layer;       // full pass over the slot layout (microbatch 0)
  AttnWs attn_t;          // targets-only attention: own work list, shared records and status
  int32_t* offs;          // slot layout [U+1]
  int32_t* nt;            // [U], all bm
  int64_t* ts;            // [cap]
  void* x0;               // [cap, d] slot-layout layer input / output (microbatch 0)
  void* x1;
  char* uvqk_cache;       // num_layers x [cap, 4 hv]
  size_t uvqk_stride;     // bytes per layer
  void* o_slot;           // [cap, hv] attention output, slot layout
  void* xc0;              // [C, d] compact candidate rows
  void* xc1;
  void* xhat_c;           // [C, d]
  float* mu1c; float* rs1c; float* mu2c; float* rs2c;
  void* uvqk_c;           // [C, 4 hv]
  void* o_c;              // [C, hv]
  void* g_c;              // [C, hv]
  int32_t* cand_dst;      // [C]
  int cap;
  int C;
};

MfalconWs carve_mfalcon(Carver& c, const hstu_layer_desc* d, int L, int U, int hist_total, int bm) {
  MfalconWs w;
  w.cap = hist_total + U * bm;
  w.C = U * bm;
  w.layer = carve_layer_fwd(c, d, U, w.cap, true);
  const size_t es = elem_size(d->attn.dtype), eio = elem_size(d->io_dtype);
  const int dm = d->d_model, hv = d->attn.num_heads * d->attn.dv;
  // targets-only attention: a work list of its own; status, tile bases and timestamp
  // records are the full pass's (same offsets); no bias band (rewriting its candidate
  // groups for every microbatch costs more than it saves there: candidate segments
  // beyond the history's last 128 positions take the one-column path instead)
  w.attn_t = w.layer.attn;
  w.attn_t.count = c.take<int32_t>(64);
  w.attn_t.items = c.take<WorkItem>(w.layer.attn.capacity);
  w.attn_t.band = nullptr;
  w.offs = c.take<int32_t>(U + 1);
  w.nt = c.take<int32_t>(U > 0 ? U : 1);
  w.ts = c.take<int64_t>(w.cap > 0 ? w.cap : 1);
  w.x0 = c.take<char>((size_t)w.cap * dm * eio);
  w.x1 = c.take<char>((size_t)w.cap * dm * eio);
  w.uvqk_stride = (((size_t)w.cap * 4 * hv * es) + 255) & ~(size_t)255;
  w.uvqk_cache = c.take<char>(w.uvqk_stride * L);
  w.o_slot = c.take<char>((size_t)w.cap * hv * es);
  w.xc0 = c.take<char>((size_t)w.C * dm * eio);
  w.xc1 = c.take<char>((size_t)w.C * dm * eio);
  w.xhat_c = c.take<char>((size_t)w.C * dm * es);
  w.mu1c = c.take<float>(w.C);
  w.rs1c = c.take<float>(w.C);
  w.mu2c = c.take<float>(w.C);
  w.rs2c = c.take<float>(w.C);
  w.uvqk_c = c.take<char>((size_t)w.C * 4 * hv * es);
  w.o_c = c.take<char>((size_t)w.C * hv * es);
  w.g_c = c.take<char>((size_t)w.C * hv * es);
  w.cand_dst = c.take<int32_t>(w.C > 0 ? w.C : 1);
  return w;
}

// One layer over the compact candidate rows x_c -> y_c (C rows), the history's
// keys and values taken from `uvqk` (slot layout), whose slot rows receive the
// candidates' U|V|Q|K.
// x_map / y_map (optional): compact row c of the input is row x_map[c] of x_c,
// and compact output row c goes to row y_map[c] of y_c (-1: a zero input row /
// a dropped output row) -- the candidates' own rows of the caller's arrays
int run_layer_targets(const hstu_layer_desc* d, const hstu_layer_weights* w, const hstu_jagged* slot_jb, int U,
                      int bm, const int32_t* hist_offsets, const void* x_c, void* y_c, char* uvqk,
                      const MfalconWs& ws, cudaStream_t st, const int32_t* x_map = nullptr,
                      const int32_t* y_map = nullptr) {
  const int dt = d->attn.dtype;
  const int dm = d->d_model, hv = d->attn.num_heads * d->attn.dv;
  const int C = ws.C;
  const size_t es = elem_size(dt);
  {
    TraceScope tr("ln1", st);
    HSTU_CUDA(launch_layer_norm(x_c, dm, d->io_dtype, w->ln1_gamma, w->ln1_beta, d->ln_eps, ws.xhat_c, dm, dt,
                                ws.mu1c, ws.rs1c, C, nullptr, dm, st, x_map));
  }
  GemmParams g1;
  memset(&g1, 0, sizeof(g1));
  g1.M = C; g1.N = 4 * hv; g1.K = dm;
  g1.A = ws.xhat_c; g1.sam = dm; g1.sak = 1;
  g1.B = w->w1; g1.sbn = dm; g1.sbk = 1;
  g1.epi = EPI_BIAS_SILU; g1.bias = w->b1;
  g1.out = ws.uvqk_c; g1.ldo = 4 * hv;
  g1.status = ws.layer.attn.status;
  // on the tensor-core path f1 writes the candidates' U|V|Q|K rows straight into
  // their slots of the cache, and LN2 * U below reads A V and U from the slots:
  // no copies between the compact and the slot layouts
  const bool direct = !(d->attn.flags & HSTU_FLAG_FORCE_SIMT) && tc_gemm_supported(g1, dt);
  if (direct) {
    g1.out = uvqk;
    g1.out_slot_offs = hist_offsets; g1.out_slot_bm = bm; g1.out_slot_cap = ws.cap;
  }
  HSTU_TRY(gemm(g1, dt, d->attn.flags, st, "gemm_f1_silu"));
  if (!direct) {
    TraceScope tr("mfalcon_slot_rows", st);
    HSTU_CUDA(launch_mfalcon_slot_rows(U, bm, ws.cap, hist_offsets, ws.uvqk_c, (int64_t)4 * hv * es, uvqk,
                                       (int64_t)4 * hv * es, (int64_t)4 * hv * es, 1, st));
  }
  // the targets-only work list is reused: reset its fetch cursor
  HSTU_CUDA(cudaMemsetAsync(ws.attn_t.count + 1, 0, sizeof(int32_t), st));
  HSTU_TRY(run_attn_main(&d->attn, slot_jb, uvqk + 2 * hv * es, 4 * hv, uvqk + 3 * hv * es, 4 * hv,
                         uvqk + 1 * hv * es, 4 * hv, w->pos_bias, w->time_bias, ws.o_slot, hv, ws.attn_t, st));
  if (direct) {
    TraceScope tr("ln2_gate", st);
    HSTU_CUDA(launch_ln_gate(ws.o_slot, hv, uvqk, 4 * hv, w->ln2_gamma, w->ln2_beta, d->ln_eps, ws.g_c, hv,
                             ws.mu2c, ws.rs2c, C, nullptr, hv, dt, st, hist_offsets, bm, ws.cap));
  } else {
    {
      TraceScope tr("mfalcon_slot_rows", st);
      HSTU_CUDA(launch_mfalcon_slot_rows(U, bm, ws.cap, hist_offsets, ws.o_slot, (int64_t)hv * es, ws.o_c,
                                         (int64_t)hv * es, (int64_t)hv * es, 0, st));
    }
    TraceScope tr("ln2_gate", st);
    HSTU_CUDA(launch_ln_gate(ws.o_c, hv, ws.uvqk_c, 4 * hv, w->ln2_gamma, w->ln2_beta, d->ln_eps, ws.g_c, hv,
                             ws.mu2c, ws.rs2c, C, nullptr, hv, dt, st));
  }
  GemmParams g2;
  memset(&g2, 0, sizeof(g2));
  g2.M = C; g2.N = dm; g2.K = hv;
  g2.A = ws.g_c; g2.sam = hv; g2.sak = 1;
  g2.B = w->w2; g2.sbn = hv; g2.sbk = 1;
  g2.epi = EPI_BIAS_RESIDUAL; g2.bias = w->b2;
  g2.residual = x_c; g2.ldr = dm;
  g2.out = y_c; g2.ldo = dm;
  g2.res_f32 = d->io_dtype == HSTU_DTYPE_F32;
  g2.out_f32 = d->io_dtype == HSTU_DTYPE_F32;
  g2.status = ws.layer.attn.status;
  g2.res_map = x_map; g2.out_map = y_map;
  // the maps exist on the tensor-core path only (the caller checked targets_mapped_io)
  if ((x_map || y_map) && ((d->attn.flags & HSTU_FLAG_FORCE_SIMT) || !tc_gemm_supported(g2, dt)))
    return HSTU_ERR_UNSUPPORTED;
  HSTU_TRY(gemm(g2, dt, d->attn.flags, st, "gemm_f2_residual"));
  return HSTU_OK;
}

// whether a candidate-only pass can read its input rows from, and write its
// output rows to, the caller's candidate arrays directly (run_layer_targets'
// maps; the tensor-core f2 with whole 32-column chunks)
bool targets_mapped_io(const hstu_layer_desc* d, const void* cand_x, const void* cand_out) {
  const size_t eio = elem_size(d->io_dtype);
  return !(d->attn.flags & HSTU_FLAG_FORCE_SIMT) && d->attn.dtype == HSTU_DTYPE_BF16 && d->d_model % 32 == 0 &&
         (d->d_model * eio) % 16 == 0 && aligned16(cand_x) && aligned16(cand_out) &&
         d->attn.num_heads * d->attn.dv % 8 == 0;
}
}  // namespace

int mfalcon_rank_workspace_size(const hstu_layer_desc* desc, int32_t num_layers, int32_t num_users,
                                int32_t hist_total, int32_t microbatch, size_t* bytes) {
  if (!desc || !bytes || num_layers < 1 || num_users < 0 || hist_total < 0 || microbatch < 1)
    return HSTU_ERR_INVALID_ARG;
  HSTU_TRY(check_attn_desc(&desc->attn));
  if ((int64_t)hist_total + (int64_t)num_users * microbatch >= (1ll << 31)) return HSTU_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_mfalcon(c, desc, num_layers, num_users, hist_total, microbatch);
  *bytes = c.size();
  return HSTU_OK;
}

int mfalcon_rank(const hstu_layer_desc* desc, const hstu_layer_weights* layers, int32_t num_layers,
                 int32_t num_users, int32_t hist_total, int32_t max_candidates, int32_t microbatch,
                 const int32_t* hist_offsets, const void* hist_x, const int64_t* hist_ts,
                 const int32_t* cand_offsets, const void* cand_x, const int64_t* cand_ts, void* cand_out,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!layers || num_layers < 1 || max_candidates < 0 || microbatch < 1) return HSTU_ERR_INVALID_ARG;
  for (int l = 0; l < num_layers; ++l) HSTU_TRY(check_layer(desc, &layers[l]));
  if (!hist_offsets || !cand_offsets || !cand_ts || !cand_out || !cand_x) return HSTU_ERR_INVALID_ARG;
  if (hist_total > 0 && (!hist_x || !hist_ts)) return HSTU_ERR_INVALID_ARG;
  const int dt = desc->io_dtype;
  const int dm = desc->d_model;
  if ((hist_x && !aligned16(hist_x)) || !aligned16(cand_x) || !aligned16(cand_out)) return HSTU_ERR_INVALID_ARG;
  size_t need;
  HSTU_TRY(mfalcon_rank_workspace_size(desc, num_layers, num_users, hist_total, microbatch, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(workspace);
  const int U = num_users, bm = microbatch;
  MfalconWs w = carve_mfalcon(c, desc, num_layers, U, hist_total, bm);
  HSTU_CUDA(cudaMemsetAsync(w.layer.attn.status, 0, kStatusBytes, st));
  const int n_mb = (max_candidates + bm - 1) / bm;
  if (U == 0) return HSTU_OK;
  if (n_mb == 0) {
    HSTU_CUDA(launch_mfalcon_check_counts(U, 0, cand_offsets, w.layer.attn.status, st));
    return HSTU_OK;
  }
  HSTU_CUDA(launch_mfalcon_slot_offsets(U, bm, hist_offsets, w.offs, w.nt, st));
  hstu_jagged jb;
  jb.batch = U;
  jb.total_tokens = w.cap;
  jb.seq_offsets = w.offs;
  jb.num_targets = w.nt;
  jb.timestamps = w.ts;
  const hstu_attn_desc* ad = &desc->attn;
  const int tile = attn_tile(ad);
  const bool mapped = targets_mapped_io(desc, cand_x, cand_out);   // later microbatches: no pack or scatter of rows
  for (int mb = 0; mb < n_mb; ++mb) {
    void* cur = w.xc0;
    void* nxt = w.xc1;
    if (mb == 0) {
      // full pass over [history ; microbatch 0]: every layer's U|V|Q|K goes to its cache
      HSTU_CUDA(launch_mfalcon_slot_pack(U, 0, bm, w.cap, w.cap, hist_offsets, hist_x, hist_ts, cand_offsets, cand_x,
                                         cand_ts, dm, dt, 1, w.x0, w.ts, nullptr, w.cand_dst, st));
      void* xs = w.x0;
      void* ys = w.x1;
      // the layers after the first reuse the first one's work list and tile records
      hstu_layer_desc dl = *desc;
      for (int l = 0; l < num_layers; ++l) {
        LayerFwdWs lw = w.layer;
        lw.b.uvqk = w.uvqk_cache + (size_t)l * w.uvqk_stride;
        dl.attn.flags = l == 0 ? (desc->attn.flags & ~HSTU_FLAG_REUSE_PREP) : (desc->attn.flags | HSTU_FLAG_REUSE_PREP);
        HSTU_TRY(run_layer_fwd(&dl, &layers[l], &jb, xs, ys, nullptr, lw, st));
        void* t = xs; xs = ys; ys = t;
      }
      // the candidates' final rows, compact
      HSTU_CUDA(launch_mfalcon_slot_rows(U, bm, w.cap, hist_offsets, xs, (int64_t)dm * elem_size(dt), cur,
                                         (int64_t)dm * elem_size(dt), (int64_t)dm * elem_size(dt), 0, st));
      // work list of the later microbatches: the q tiles of the candidate slots only
      {
        TraceScope tr("sched_fwd", st);
        HSTU_CUDA(launch_build_work_list(w.offs, w.nt, U, w.cap, ad->num_heads, tile, tile, use_tc(ad) ? 3 : 0,
                                         w.attn_t.capacity, w.attn_t.items, w.attn_t.count, w.attn_t.status, st,
                                         nullptr, 1));
      }
    } else {
      // with mapped input and output rows the first layer reads the candidates' rows
      // of cand_x and the last writes cand_out's: the pack only places timestamps
      // and the row map, and no scatter follows
      HSTU_CUDA(launch_mfalcon_slot_pack(U, mb, bm, w.C, w.cap, hist_offsets, hist_x, hist_ts, cand_offsets, cand_x,
                                         cand_ts, dm, dt, 0, nullptr, w.ts, mapped ? nullptr : cur, w.cand_dst, st));
      if (w.attn_t.tile_recs) {
        // the candidates' timestamps changed: timestamp records of every kv tile
        TraceScope tr("ts_tiles", st);
        HSTU_CUDA(launch_ts_tiles(w.offs, w.ts, U, w.attn_t.tile_base, w.attn_t.tiles_cap, w.attn_t.tile_recs, st));
      }
      for (int l = 0; l < num_layers; ++l) {
        const bool first = mapped && l == 0, last = mapped && l == num_layers - 1;
        HSTU_TRY(run_layer_targets(desc, &layers[l], &jb, U, bm, hist_offsets, first ? cand_x : cur,
                                   last ? cand_out : nxt, w.uvqk_cache + (size_t)l * w.uvqk_stride, w, st,
                                   first ? w.cand_dst : nullptr, last ? w.cand_dst : nullptr));
        void* t = cur; cur = nxt; nxt = t;
      }
      if (mapped) continue;   // the last layer wrote cand_out
    }
    HSTU_CUDA(launch_mfalcon_scatter(cur, dm, dt, w.cand_dst, nullptr, w.C, cand_out, st));
  }
  // a user with more candidates than the n_mb microbatches hold had some left unscored
  HSTU_CUDA(launch_mfalcon_check_counts(U, n_mb * bm, cand_offsets, w.layer.attn.status, st));
  return HSTU_OK;
}

// ---------------------------------------------------------------- Stochastic Length
int hstu_stochastic_length_workspace_size(int32_t batch, int32_t total_tokens, size_t* bytes) {
  if (!bytes || batch < 0 || total_tokens < 0) return HSTU_ERR_INVALID_ARG;
  Carver c(nullptr);
  c.take<int32_t>(kStatusBytes / 4);
  *bytes = c.size();
  return HSTU_OK;
}

int hstu_stochastic_length(int32_t batch, int32_t total_tokens, const int32_t* seq_offsets, const uint32_t* coins,
                           const uint32_t* keys, int32_t max_len, uint32_t prob_u32, int32_t* out_offsets,
                           int32_t* out_index, void* workspace, size_t workspace_bytes, void* stream) {
  if (batch < 0 || total_tokens < 0 || max_len < 1 || !seq_offsets || !out_offsets) return HSTU_ERR_INVALID_ARG;
  if (batch > 0 && (!coins || (total_tokens > 0 && (!keys || !out_index)))) return HSTU_ERR_INVALID_ARG;
  size_t need;
  HSTU_TRY(hstu_stochastic_length_workspace_size(batch, total_tokens, &need));
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return HSTU_ERR_WORKSPACE;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  int32_t* status = (int32_t*)workspace;
  HSTU_CUDA(cudaMemsetAsync(status, 0, kStatusBytes, st));
  HSTU_CUDA(launch_sl_select(batch, total_tokens, seq_offsets, coins, keys, max_len, prob_u32, out_offsets, out_index,
                             nullptr, status, st));
  return HSTU_OK;
}

int hstu_gather_rows(const void* src, void* dst, int64_t row_bytes, const int32_t* index, const int32_t* count,
                     int32_t capacity, void* stream) {
  if (!src || !dst || !index || !count || capacity < 0 || row_bytes <= 0 || row_bytes % 4) return HSTU_ERR_INVALID_ARG;
  if (((uintptr_t)src & 3) || ((uintptr_t)dst & 3)) return HSTU_ERR_INVALID_ARG;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  return cuda_status(launch_gather_rows(src, dst, row_bytes, index, count, capacity, (cudaStream_t)stream));
}

// ---------------------------------------------------------------- diagnostics
int hstu_debug_rab_buckets(const hstu_attn_desc* desc, const hstu_jagged* jb, const int32_t* pairs,
                           int32_t num_pairs, int32_t* out, void* stream) {
  HSTU_TRY(check_attn_desc(desc));
  HSTU_TRY(check_jagged(jb));
  if (num_pairs < 0 || (num_pairs > 0 && (!pairs || !out))) return HSTU_ERR_INVALID_ARG;
  if (num_pairs == 0) return HSTU_OK;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  Thresholds thr = thresholds_for(desc->time_div);
  return cuda_status(launch_debug_buckets(jb->seq_offsets, jb->num_targets, jb->timestamps, thr, desc->time_div,
                                          pairs, num_pairs, out, (cudaStream_t)stream));
}

int hstu_debug_timeout_probe(int64_t timeout_ns, int32_t* status_dev, void* stream) {
  if (!status_dev || timeout_ns < 1 || timeout_ns > 2000000000ll) return HSTU_ERR_INVALID_ARG;
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  return cuda_status(launch_timeout_probe(timeout_ns, status_dev, (cudaStream_t)stream));
}

}  // extern "C"

// =============================================================================
// Attention forward without caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they run the
// attention: an embedding application whose device memory is entirely owned by
// another allocator, or a latency-bound serving loop that forbids any
// allocation once it has started.  For them this entry point takes its scratch
// (the status word and the cost-sorted work list) from a fixed array that the
// library itself places in device memory, instead of from a workspace.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes bytes;
// every GPU on which the library is loaded holds it until the process exits.
// In host code its name only stands for the variable, it is not a device
// address, so the address is looked up once per device (cudaGetSymbolAddress,
// with that device current) on the first call made on that device, and passed
// to the kernels from then on.
// =============================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = 1u << 20;  // 1 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};   // id of the context the address belongs to

// The CUDA driver API context calls, taken through the runtime's entry-point query so
// that the library has no link-time dependency on libcuda.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device, looked up once per
// device and context: the address is only valid in the context it was looked up
// in, so a call from another context of the device (a non-primary context, or
// the primary context again after cudaDeviceReset) looks it up afresh.  Context
// ids are never reused within a process.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSTU_ERR_UNSUPPORTED;
  unsigned long long id = current_context_id();   // 0: no context current yet
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev] || id == 0 || g_noalloc_ctx[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HSTU_ERR_CUDA;
    if (id == 0) id = current_context_id();   // the lookup made the device's primary context current
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = id;
  }
  *out = g_noalloc_ptr[dev];
  return HSTU_OK;
}

}  // namespace

extern "C" int hstu_attn_fwd_noalloc(const hstu_attn_desc* desc, const hstu_jagged* jb, const void* q, int64_t ldq,
                                     const void* k, int64_t ldk, const void* v, int64_t ldv,
                                     const float* pos_bias, const float* time_bias, void* out, int64_t ldo,
                                     void* stream) {
  HSTU_TRY(check_attn_desc(desc));
  HSTU_TRY(check_jagged(jb));
  const int hd = desc->num_heads * desc->dqk;
  HSTU_TRY(check_rows(q, ldq, hd, desc->dtype));
  HSTU_TRY(check_rows(k, ldk, hd, desc->dtype));
  HSTU_TRY(check_rows(v, ldv, hd, desc->dtype));
  HSTU_TRY(check_rows(out, ldo, hd, desc->dtype));
  if (!pos_bias || !time_bias) return HSTU_ERR_INVALID_ARG;
  Carver sizer(nullptr);
  carve_attn(sizer, desc, jb->batch, jb->total_tokens, false, false);  // without the bias band
  if (sizer.size() > kNoAllocScratchBytes) return HSTU_ERR_WORKSPACE;  // problem larger than the fixed array
  void* scratch = nullptr;
  HSTU_TRY(noalloc_scratch(&scratch));
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  Carver c(scratch);
  AttnWs w = carve_attn(c, desc, jb->batch, jb->total_tokens, false, false);  // no band: bounded scratch
  HSTU_CUDA(cudaMemsetAsync(w.status, 0, kStatusBytes, st));  // the previous call's status must not leak
  return run_attn_fwd(desc, jb, q, ldq, k, ldk, v, ldv, pos_bias, time_bias, out, ldo, w, st);
}
