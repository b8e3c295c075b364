// The whole HSTU layer in one kernel for short sequences (at most 128 tokens):
//
//   U, V, Q, K = Split(SiLU(f1(LayerNorm(X))))
//   A V        = (SiLU(Q K^T + rab) / N (.) mask) V
//   Y          = X + f2(LayerNorm(A V) (.) U)
//
// ("Actions Speak Louder than Words" summary, 1.3 and 2.2: the layer's linear
// maps are grouped and its element-wise work fused; for short histories the
// launches and the round trips through memory between the stages cost more than
// the arithmetic.)  The batch is cut into work units of at most 128 consecutive
// token rows that hold whole sequences (the sequences inside each 128-row window,
// and each sequence crossing a window boundary on its own), so short sequences
// share one tile: rows of different sequences never attend to each other, which
// the bias matrix masks.  One CTA takes one unit at a time from a shared cursor
// and keeps every intermediate on the chip:
//   shared memory  x-hat (later the gate LN2(A V) * U) as the A operand of f1 and
//                  f2; Q, K, V of the current head; the relative-bias matrix of
//                  the unit (bf16, -1e30 where masked, across sequences too); each
//                  row's sequence (first row, length, N); a ring of weight slices
//   TMEM           the f1 accumulator of one head (U|V|Q|K, 256 columns), reused
//                  by S, P and the head's A V; U and A V of all heads as bf16;
//                  finally the f2 accumulator
//   warp 0         finds the next unit (a warp-wide search of the offsets), then
//                  TMA: W1 slices (the 4 x 64 rows of one head's U, V, Q, K) and
//                  W2 slices, 64 input columns at a time
//   warp 1         tcgen05.mma (whole warp, one elected lane)
//   warps 2-17     LayerNorms, bias matrix, f1 epilogue (bias, SiLU, split),
//                  pointwise attention epilogue, gate, f2 epilogue (+ residual);
//                  four warps per TMEM lane quarter, each on a quarter of the columns
// Head dimension 64; d_model and H * 64 at most 256, multiples of 64; bf16.
// Every device-side wait is bounded (HSTU_ERR_TIMEOUT); a sequence longer than
// 128 tokens is skipped and reported as HSTU_ERR_BAD_OFFSETS, and so are offsets
// that are not non-decreasing from 0 to at most T (nothing outside [0, T) is read
// or written either way).
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
namespace {
using namespace sm100;

constexpr int R = 128;                   // rows (tokens) per sequence at most
constexpr int DH = 64;                   // head dimension
constexpr int kMaxD = 256;               // d_model and H * DH at most
constexpr int kEpiWarps = 16;
constexpr int kEpiWarp0 = 2;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kAtom = R * 128;           // [128 rows x 64] bf16, 128-byte swizzle: 16 KB
constexpr int kSlice = 4 * 64 * 128;     // one weight slice: 256 rows x 64 columns bf16 (32 KB)
constexpr int kRingStages = 2;
constexpr uint32_t kColAcc = 0, kColO = 128, kColU = 256, kColOb = 384, kTmemCols = 512;
constexpr float kMasked = -1e30f;

struct Bars {
  uint64_t it_full[2], it_empty[2];
  uint64_t ring_full[kRingStages], ring_empty[kRingStages];
  uint64_t xhat_ready, f1_full, qkv_ready, s_full, p_ready, o_full, o_done, gate_ready, f2_full;
  uint64_t epi_sync;
  uint64_t done;
};

struct Layout {
  static constexpr int kA = 0;                               // x-hat / gate: 4 atoms
  static constexpr int kQ = kA + 4 * kAtom;
  static constexpr int kK = kQ + kAtom;
  static constexpr int kV = kK + kAtom;
  static constexpr int kRing = kV + kAtom;
  static constexpr int kBias = kRing + kRingStages * kSlice;  // [128 x 128] bf16, 16-byte chunks swizzled
  static constexpr int kTs = kBias + R * R * 2;               // rel offsets int32[128] | abs int64[128]
  static constexpr int kRows = kTs + R * 4 + R * 8;           // per row: sequence start in the pack, n, N
  static constexpr int kPackOffs = kRows + 3 * R * 4;         // the pack's sequence offsets (up to 129)
  static constexpr int kThr = kPackOffs + (R + 4) * 4;
  static constexpr int kThr32 = kThr + kNumBuckets * 8;
  static constexpr int kPosB = kThr32 + (kNumBuckets + 4) * 4;
  static constexpr int kTimeB = kPosB + kNumBuckets * 4;
  static constexpr int kStats = kTimeB + kNumBuckets * 4;     // LN2 partial sums [4 parts][128 rows][2]
  static constexpr int kBar = kStats + 4 * R * 2 * 4;
  static constexpr int kMisc = kBar + (int)sizeof(Bars);
  static constexpr int kItems = kMisc + 16;
  static constexpr int kEnd = kItems + 2 * 8 * 4;
  static constexpr int kAlloc = kEnd + 1024;
};
static_assert(Layout::kAlloc <= 227 * 1024, "shared memory");

struct FusedParams {
  CUtensorMap map_w1;    // W1 [4 hv, d], box 64 columns x 64 rows
  CUtensorMap map_w2;    // W2 [d, hv], box 64 columns x 64 rows
  const int32_t* offs;
  const int32_t* num_targets;
  const int64_t* ts;
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  const float* b1;
  const float* ln1_g;
  const float* ln1_b;
  const float* ln2_g;
  const float* ln2_b;
  const float* b2;
  const float* pos_bias;
  const float* time_bias;
  int rab_head_stride;
  int B, T, d, H, hv;
  float eps;
  float ln2_over_div;
  Thresholds thr;
  int32_t* cursor;
  int32_t* status;
  long long timeout_ns;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// SiLU(x) = x sigma(x), sigma from 2^x and a reciprocal (accurate for every x;
// a masked score of -1e30 gives 0)
__device__ __forceinline__ float silu_acc(float x) {
  return x * rcp_approx(1.0f + ex2_approx(x * -1.4426950408889634f));
}
// SiLU(x) = h + h tanh(h), h = x / 2: one special-function op (the projection's SiLU,
// as the multi-kernel layer computes it)
__device__ __forceinline__ float silu_tanh(float x) {
  const float h = 0.5f * x;
  return fmaf(h, tanh_approx(h), h);
}

// first index in [0, cnt) with a[index] >= v (cnt if none), a non-decreasing; the
// whole warp searches, 32 probes at a time
__device__ __forceinline__ int warp_lower_bound(const int32_t* a, int cnt, int v, int lane) {
  int lo = 0, hi = cnt;   // the answer lies in [lo, hi]
  while (hi - lo > 31) {
    const int step = (hi - lo + 30) / 31;         // lane 31 probes at or beyond hi: some probe answers yes
    const int idx = lo + lane * step;
    const bool ge = idx < hi ? a[idx] >= v : true;
    const int f = __ffs(__ballot_sync(0xffffffffu, ge)) - 1;   // first probe at or above v
    const int idx_f = min(lo + f * step, hi);
    lo = f == 0 ? lo : lo + (f - 1) * step + 1;
    hi = idx_f;
  }
  const int idx = lo + lane;                      // hi - lo <= 31: lane 31 is at or beyond hi
  const bool ge = idx < hi ? a[idx] >= v : true;
  return lo + __ffs(__ballot_sync(0xffffffffu, ge)) - 1;
}

// A work unit: up to 128 consecutive token rows holding whole sequences.  With
// W = ceil(T_used / 128) windows of 128 rows, unit u < W takes the sequences that
// lie entirely inside window u, and unit W - 1 + b takes the sequence that crosses
// the boundary between windows b - 1 and b (a sequence of at most 128 tokens
// crosses at most one), so every sequence belongs to exactly one unit and no
// unit needs more than one 128-row tile.
struct Pack {
  int id;      // -1: no more units
  int row0;    // first token row
  int nrows;   // rows (0: nothing to compute)
  int s0;      // first sequence
  int count;   // sequences s0 .. s0 + count - 1
  int bad;     // a crossing sequence longer than 128 tokens, or inconsistent offsets
};

__device__ __forceinline__ Pack decode_pack(const FusedParams& p, int id, int lane) {
  Pack pk;
  pk.id = id; pk.row0 = 0; pk.nrows = 0; pk.s0 = 0; pk.count = 0; pk.bad = 0;
  const int t_used = p.offs[p.B];
  if (p.offs[0] != 0 || t_used < 0 || t_used > p.T) {
    pk.bad = id == 0 ? 1 : 0;   // reported once
    pk.id = id == 0 ? 0 : -1;
    return pk;
  }
  const int W = (t_used + R - 1) / R;
  if (id < 0 || id >= 2 * W - 1) { pk.id = -1; return pk; }
  if (id < W) {
    const int lo = id * R, hi = min(lo + R, t_used);
    const int sa = warp_lower_bound(p.offs, p.B + 1, lo, lane);          // first sequence starting at or after lo
    const int sb = warp_lower_bound(p.offs, p.B + 1, hi + 1, lane) - 1;  // last offset at or below hi
    if (sb > sa && sb <= p.B) {
      pk.row0 = p.offs[sa];
      pk.nrows = p.offs[sb] - pk.row0;
      pk.s0 = sa;
      pk.count = sb - sa;
    }
  } else {
    const int b = (id - W + 1) * R;
    const int s = warp_lower_bound(p.offs, p.B + 1, b, lane) - 1;      // last sequence starting before b
    if (s >= 0 && s < p.B && p.offs[s + 1] > b) {
      const int len = p.offs[s + 1] - p.offs[s];
      if (len <= R) {
        pk.row0 = p.offs[s];
        pk.nrows = len;
        pk.s0 = s;
        pk.count = 1;
      } else {
        pk.bad = 1;   // not this kernel's: reported
      }
    }
  }
  if (pk.nrows < 0 || pk.nrows > R || pk.row0 < 0 || pk.row0 + pk.nrows > p.T) {   // unsorted offsets
    pk.nrows = 0;
    pk.bad = 1;
  }
  return pk;
}

// byte offset of element (row r, column c) of a [128 x 64k] bf16 tile of 64-column
// atoms with the 128-byte swizzle (16-byte chunks permuted by the row's low bits)
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)((c >> 6) * kAtom + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}

__global__ void __launch_bounds__(kThreads, 1) fused_short_kernel(const __grid_constant__ FusedParams prm) {
  using L = Layout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* items = reinterpret_cast<volatile int*>(smem + L::kItems);
  int32_t* rel_s = reinterpret_cast<int32_t*>(smem + L::kTs);
  int64_t* abs_s = reinterpret_cast<int64_t*>(smem + L::kTs + R * 4);
  int32_t* row_sb = reinterpret_cast<int32_t*>(smem + L::kRows);          // first row of the row's sequence
  int32_t* row_n = row_sb + R;                                             // its length
  int32_t* row_hist = row_n + R;                                           // its N
  int32_t* pack_offs = reinterpret_cast<int32_t*>(smem + L::kPackOffs);   // the unit's sequence offsets
  int64_t* thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int32_t* thr32 = reinterpret_cast<int32_t*>(smem + L::kThr32);
  float* pos_b = reinterpret_cast<float*>(smem + L::kPosB);
  float* time_b = reinterpret_cast<float*>(smem + L::kTimeB);
  float* stats = reinterpret_cast<float*>(smem + L::kStats);
  const uint32_t sA = smem_u32(smem + L::kA);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  const uint32_t sV = smem_u32(smem + L::kV);
  const uint32_t sRing = smem_u32(smem + L::kRing);
  const uint32_t sBias = smem_u32(smem + L::kBias);

  const FusedParams& p = prm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tmo = p.timeout_ns;
  const int d = p.d, hv = p.hv, H = p.H;
  const int k_d = d / 64, k_hv = hv / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) { mbar_init(&bars->it_full[s], 1); mbar_init(&bars->it_empty[s], 1 + kEpiWarps); }
    for (int s = 0; s < kRingStages; ++s) { mbar_init(&bars->ring_full[s], 1); mbar_init(&bars->ring_empty[s], 1); }
    mbar_init(&bars->xhat_ready, kEpiWarps);
    mbar_init(&bars->f1_full, 1);
    mbar_init(&bars->qkv_ready, kEpiWarps);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_ready, kEpiWarps);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_done, kEpiWarps);
    mbar_init(&bars->gate_ready, kEpiWarps);
    mbar_init(&bars->f2_full, 1);
    mbar_init(&bars->epi_sync, kEpiWarps);
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&prm.map_w1);
    tma_prefetch_desc(&prm.map_w2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  for (int c = threadIdx.x; c < kNumBuckets + 4; c += kThreads) {
    if (c < kNumBuckets) {
      thr[c] = p.thr.v[c];
      thr32[c] = p.thr.v[c] > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)p.thr.v[c];
    } else {
      thr32[c] = 0x7FFFFFFF;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================================ work units and weight slices
    int r = 0;   // ring slot counter
    for (int k = 0;; ++k) {
      const int slot = k & 1;
      if (!warp_wait(&bars->it_empty[slot], ((k >> 1) & 1) ^ 1, tmo, abort_flag)) goto fail;
      int id = 0;
      if (lane == 0) id = *abort_flag ? -1 : atomicAdd(p.cursor, 1);
      id = __shfl_sync(0xffffffffu, id, 0);
      const Pack pk = decode_pack(p, id, lane);
      if (lane == 0) {
        items[8 * slot] = pk.id;
        items[8 * slot + 1] = pk.row0;
        items[8 * slot + 2] = pk.nrows;
        items[8 * slot + 3] = pk.s0;
        items[8 * slot + 4] = pk.count;
        items[8 * slot + 5] = pk.bad;
        mbar_arrive(&bars->it_full[slot]);
      }
      __syncwarp();
      if (pk.id < 0) break;
      if (pk.nrows == 0) continue;   // nothing to compute (a bad unit is reported by the epilogue)
      bool ok = true;
      if (lane == 0) {
        for (int h = 0; h < H && ok; ++h) {
          for (int ks = 0; ks < k_d; ++ks, ++r) {
            const int st = r % kRingStages;
            if (!mbar_wait(&bars->ring_empty[st], ((r / kRingStages) & 1) ^ 1, tmo, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars->ring_full[st], kSlice);
            // rows 64c .. 64c + 63 of the slice: W1 rows of block c (U, V, Q, K) for head h
            for (int c = 0; c < 4; ++c)
              tma_load_2d(smem + L::kRing + st * kSlice + c * 64 * 128, &prm.map_w1, &bars->ring_full[st], ks * 64,
                          c * hv + h * DH);
          }
        }
        for (int ks = 0; ks < k_hv && ok; ++ks, ++r) {
          const int st = r % kRingStages;
          if (!mbar_wait(&bars->ring_empty[st], ((r / kRingStages) & 1) ^ 1, tmo, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->ring_full[st], k_d * 64 * 128);
          for (int c = 0; c < k_d; ++c)
            tma_load_2d(smem + L::kRing + st * kSlice + c * 64 * 128, &prm.map_w2, &bars->ring_full[st], ks * 64,
                        c * 64);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) goto fail;
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    constexpr uint32_t id_f1 = make_idesc_bf16(R, 256, false, false);
    constexpr uint32_t id_s = make_idesc_bf16(R, R, false, false);
    constexpr uint32_t id_o = make_idesc_bf16(R, DH, false, true);
    const uint32_t id_f2 = make_idesc_bf16(R, d, false, false);
    const uint64_t dA = make_sw128_desc(sA, 16, 1024);
    const uint64_t dQd = make_sw128_desc(sQ, 16, 1024);
    const uint64_t dKd = make_sw128_desc(sK, 16, 1024);
    const uint64_t dVd = make_sw128_desc(sV, kAtom, 1024);
    const uint64_t dR = make_sw128_desc(sRing, 16, 1024);
    int r = 0, g = 0;
    for (int k = 0;; ++k) {
      const int slot = k & 1;
      if (!warp_wait(&bars->it_full[slot], (k >> 1) & 1, tmo, abort_flag)) goto fail;
      const int unit = items[8 * slot];
      const int unit_rows = items[8 * slot + 2];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->it_empty[slot]);
      if (unit < 0) break;
      if (unit_rows == 0) continue;
      if (!warp_wait(&bars->xhat_ready, k & 1, tmo, abort_flag)) goto fail;
      for (int h = 0; h < H; ++h, ++g) {
        // f1 of head h: [128 x d] x [d x 256] into the accumulator (after the previous
        // head's A V was read out of the same columns)
        if (h > 0 && !warp_wait(&bars->o_done, (g - 1) & 1, tmo, abort_flag)) goto fail;
        for (int ks = 0; ks < k_d; ++ks, ++r) {
          const int st = r % kRingStages;
          if (!warp_wait(&bars->ring_full[st], (r / kRingStages) & 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            umma_f16_ss_elect(tmem + kColAcc, desc_advance(dA, ks * kAtom + q * 32),
                              desc_advance(dR, st * kSlice + q * 32), id_f1, (ks > 0 || q > 0) ? 1u : 0u);
          umma_commit_elect(&bars->ring_empty[st]);
        }
        umma_commit_elect(&bars->f1_full);
        // S = Q K^T
        if (!warp_wait(&bars->qkv_ready, g & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < DH / 16; ++q)
          umma_f16_ss_elect(tmem + kColAcc, desc_advance(dQd, q * 32), desc_advance(dKd, q * 32), id_s,
                            q > 0 ? 1u : 0u);
        umma_commit_elect(&bars->s_full);
        // A V = P V, P from TMEM (over the S columns)
        if (!warp_wait(&bars->p_ready, g & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < R / 16; ++q)
          umma_f16_ts_elect(tmem + kColO, tmem + kColAcc + 32 * (q >> 1) + 8 * (q & 1),
                            desc_advance(dVd, q * 16 * 128), id_o, q > 0 ? 1u : 0u);
        umma_commit_elect(&bars->o_full);
      }
      // f2 once the gate is in place: [128 x hv] x [hv x d]
      if (!warp_wait(&bars->gate_ready, k & 1, tmo, abort_flag)) goto fail;
      tc_fence_after();
      for (int ks = 0; ks < k_hv; ++ks, ++r) {
        const int st = r % kRingStages;
        if (!warp_wait(&bars->ring_full[st], (r / kRingStages) & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          umma_f16_ss_elect(tmem + kColAcc, desc_advance(dA, ks * kAtom + q * 32),
                            desc_advance(dR, st * kSlice + q * 32), id_f2, (ks > 0 || q > 0) ? 1u : 0u);
        umma_commit_elect(&bars->ring_empty[st]);
      }
      umma_commit_elect(&bars->f2_full);
    }
    umma_commit_elect(&bars->done);
    warp_wait(&bars->done, 0, tmo, nullptr);
  } else {
    // ================================================================ epilogue warps
    const int ew = warp - kEpiWarp0;        // 0..7
    const int quarter = warp & 3;           // TMEM lane quarter
    const int part = ew >> 2;               // column quarter
    const int row = quarter * 32 + lane;    // this lane's row in TMEM-lane order
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int etid = threadIdx.x - 32 * kEpiWarp0;   // 0..255
    int epi_phase = 0;
    auto epi_barrier = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->epi_sync);
      const bool ok = warp_wait(&bars->epi_sync, epi_phase & 1, tmo, abort_flag);
      ++epi_phase;
      return ok;
    };
    int g = 0;
    int bias_head = -1;
    for (int k = 0;; ++k) {
      const int slot = k & 1;
      if (!warp_wait(&bars->it_full[slot], (k >> 1) & 1, tmo, abort_flag)) goto fail;
      const int unit = items[8 * slot];
      const int start = items[8 * slot + 1];    // first token row of the unit
      const int n = items[8 * slot + 2];        // its rows
      const int s0 = items[8 * slot + 3];
      const int count = items[8 * slot + 4];
      const int bad = items[8 * slot + 5];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->it_empty[slot]);
      if (unit < 0) break;
      if (bad && etid == 0) set_status(p.status, HSTU_ERR_BAD_OFFSETS);
      if (n == 0) continue;
      // ---- every row's sequence: its first row in the unit, its length and N (rows
      // beyond the unit: none).  The unit's sequence offsets go to shared memory first
      // when there are at most 128 of them (more only with empty sequences).
      if (count <= R)
        for (int t = etid; t <= count; t += 32 * kEpiWarps) pack_offs[t] = p.offs[s0 + t] - start;
      if (!epi_barrier()) goto fail;
      if (etid < R) {
        int sb = etid, nn = 0, hh = 0;
        if (etid < n) {
          int lo = 0, hi = count - 1;   // the last sequence of the unit starting at or before this row
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            const int st_mid = count <= R ? pack_offs[mid] : p.offs[s0 + mid] - start;
            if (st_mid <= etid) lo = mid; else hi = mid - 1;
          }
          const int sq = s0 + lo;
          sb = p.offs[sq] - start;
          nn = p.offs[sq + 1] - p.offs[sq];
          int nt = p.num_targets ? p.num_targets[sq] : 0;
          nt = nt < 0 ? 0 : (nt > nn ? nn : nt);
          hh = nn - nt;
        }
        row_sb[etid] = sb;
        row_n[etid] = nn;
        row_hist[etid] = hh;
      }
      // ---- timestamps of the unit: offsets from its first, clamped to +-(2^30 - 1)
      // (a pair with a clamped offset takes the 64-bit values)
      const int64_t t_first = p.ts[start];
      constexpr int32_t kLim = (1 << 30) - 1;
      for (int i = etid; i < R; i += 32 * kEpiWarps) {
        const int64_t t = i < n ? p.ts[start + i] : t_first;
        const int64_t rel = t - t_first;
        rel_s[i] = (int32_t)(rel < -kLim ? -kLim : (rel > kLim ? kLim : rel));
        abs_s[i] = t;
      }
      // ---- LayerNorm1: warp ew takes rows 8 ew .. 8 ew + 7, lanes over d (8 columns
      // each); the eight rows' loads are in flight together
      {
        const bool on = lane * 8 < d;
        uint4 raw[8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 8 * ew + rr;
          raw[rr] = (r < n && on) ? *reinterpret_cast<const uint4*>(p.x + (int64_t)(start + r) * d + lane * 8)
                                  : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 8 * ew + rr;
          float v[8];
          const uint32_t w[4] = {raw[rr].x, raw[rr].y, raw[rr].z, raw[rr].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
          }
          float sum = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sum += v[e];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          const float mu = sum / (float)d;
          float sq = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sq += on ? (v[e] - mu) * (v[e] - mu) : 0.f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
          const float rs = rsqrtf(sq / (float)d + p.eps);
          if (on) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = lane * 8 + 2 * e;
              const float a = r < n ? (v[2 * e] - mu) * rs * p.ln1_g[c] + p.ln1_b[c] : 0.f;
              const float b = r < n ? (v[2 * e + 1] - mu) * rs * p.ln1_g[c + 1] + p.ln1_b[c + 1] : 0.f;
              pk[e] = pack_bf16x2(a, b);
            }
            st_shared_v4(sA + sw_off(r, lane * 8), pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->xhat_ready);
      if (!epi_barrier()) goto fail;   // timestamps and row facts in shared memory for everyone
      const float inv_n = 1.0f / (float)(row_hist[row] > 1 ? row_hist[row] : 1);   // this lane's row
      // ---- relative-bias matrix of the sequence: bias(i, j) as bf16, -1e30 where the
      // pair is not attended.  Thread t: row t / 4, columns [32 (t % 4), +32).
      auto build_bias = [&](int head) {
        for (int e = etid; e < R * 4; e += 32 * kEpiWarps) {
          const int i = e >> 2, j0 = (e & 3) * 32;
          const int sbi = row_sb[i], ni = row_n[i], hi_ = row_hist[i];   // row i's sequence
          const int posi = token_pos(i - sbi, hi_);
#pragma unroll 1
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float bv[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int j = j0 + 8 * c8 + 2 * u + q;
                float b = kMasked;
                const int lj = j - sbi;   // column j inside row i's sequence (same sequence iff 0 <= lj < ni)
                if (i < n && lj >= 0 && lj < ni && attended(i - sbi, lj, ni, hi_)) {
                  const int pb = pos_bucket(posi, token_pos(lj, hi_));
                  const int32_t ri = rel_s[i], rj = rel_s[j];
                  const bool clamped = ri == kLim || ri == -kLim || rj == kLim || rj == -kLim;
                  const int tb = clamped ? time_bucket_exact(abs_diff_i64(abs_s[i], abs_s[j]), thr)
                                         : fast_bucket(abs(ri - rj), thr32, p.ln2_over_div);
                  b = pos_b[pb] + time_b[tb];
                }
                bv[q] = b;
              }
              pk[u] = pack_bf16x2(bv[0], bv[1]);
            }
            const int ch = (j0 >> 3) + c8;   // 16-byte chunk of the 256-byte row, swizzled by the row
            st_shared_v4(sBias + i * 256 + ((ch ^ (i & 15)) << 4), pk[0], pk[1], pk[2], pk[3]);
          }
        }
      };
      if (p.rab_head_stride == 0 && bias_head != 0) {
        for (int c = etid; c < kNumBuckets; c += 32 * kEpiWarps) {
          pos_b[c] = p.pos_bias[c];
          time_b[c] = p.time_bias[c];
        }
        if (!epi_barrier()) goto fail;
        bias_head = 0;
      }
      if (p.rab_head_stride == 0) build_bias(0);
      for (int h = 0; h < H; ++h, ++g) {
        if (p.rab_head_stride != 0) {
          if (!epi_barrier()) goto fail;   // everyone is done with the previous head's matrix and tables
          for (int c = etid; c < kNumBuckets; c += 32 * kEpiWarps) {
            pos_b[c] = p.pos_bias[h * p.rab_head_stride + c];
            time_b[c] = p.time_bias[h * p.rab_head_stride + c];
          }
          if (!epi_barrier()) goto fail;
          build_bias(h);
          bias_head = h;
        }
        // ---- f1 epilogue: column quarter 0 takes U of head h, 1 V, 2 Q, 3 K
        if (!warp_wait(&bars->f1_full, g & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        {
          const int cb = part;   // 0 U, 1 V, 2 Q, 3 K
          const float* bias1 = p.b1 + cb * hv + h * DH;
#pragma unroll 1
          for (int c16 = 0; c16 < 4; ++c16) {
            uint32_t raw[16];
            tmem_ld_32x32b_x16(tmem + kColAcc + lane_off + cb * 64 + 16 * c16, raw);
            tmem_ld_wait();
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = 16 * c16 + 2 * e;
              pk[e] = pack_bf16x2(silu_tanh(__uint_as_float(raw[2 * e]) + bias1[c]),
                                  silu_tanh(__uint_as_float(raw[2 * e + 1]) + bias1[c + 1]));
            }
            if (cb == 0) {
              // U of head h: packed into the U columns (32 per head)
              tmem_st_32x32b_x8(tmem + kColU + lane_off + 32 * h + 8 * c16, pk);
            } else {
              const uint32_t tile = cb == 1 ? sV : (cb == 2 ? sQ : sK);
              st_shared_v4(tile + sw_off(row, 16 * c16), pk[0], pk[1], pk[2], pk[3]);
              st_shared_v4(tile + sw_off(row, 16 * c16 + 8), pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        if (p.rab_head_stride != 0 || h == 0) {
          if (!epi_barrier()) goto fail;   // the bias matrix is complete before S is read
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->qkv_ready);
        // ---- attention epilogue: S + bias, SiLU (masked pairs give 0), P as bf16 over
        // the first 16 columns of each 32-column segment (the A operand of P V)
        if (!warp_wait(&bars->s_full, g & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        {
          const int seg = part;
          uint32_t raw[32];
          tmem_ld_32x32b_x32(tmem + kColAcc + lane_off + 32 * seg, raw);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const int ch = 4 * seg + c8;
            uint32_t bw[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(bw[0]), "=r"(bw[1]), "=r"(bw[2]), "=r"(bw[3])
                         : "r"(sBias + row * 256 + ((ch ^ (row & 15)) << 4)));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int e = 8 * c8 + 2 * u;
              const float x0 = __uint_as_float(raw[e]) + __uint_as_float(bw[u] << 16);
              const float x1 = __uint_as_float(raw[e + 1]) + __uint_as_float(bw[u] & 0xFFFF0000u);
              pk[4 * c8 + u] = pack_bf16x2(silu_acc(x0), silu_acc(x1));
            }
          }
          tmem_st_32x32b_x16(tmem + kColAcc + lane_off + 32 * seg, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready);
        // ---- A V of head h: (1/N), bf16, into the A V columns (32 per head)
        if (!warp_wait(&bars->o_full, g & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        {
          uint32_t raw[16];
          tmem_ld_32x32b_x16(tmem + kColO + lane_off + 16 * part, raw);
          tmem_ld_wait();
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * inv_n, __uint_as_float(raw[2 * e + 1]) * inv_n);
          tmem_st_32x32b_x8(tmem + kColOb + lane_off + 32 * h + 8 * part, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->o_done);
      }
      // ---- gate: LayerNorm2 over the row's H * 64 values of A V, times U.  Each column
      // quarter of the warps holds a quarter of the row's values; the partial sums
      // meet in shared memory.
      {
        const int ncol = hv / 4;            // values per part (16 .. 64)
        const int c0 = part * ncol;         // first value of this part
        float s1 = 0.f, s2 = 0.f;
        tc_fence_after();
#pragma unroll 1
        for (int c8 = 0; c8 < ncol / 16; ++c8) {
          uint32_t ob[8];
          tmem_ld_32x32b_x8(tmem + kColOb + lane_off + (c0 >> 1) + 8 * c8, ob);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = __uint_as_float(ob[e] << 16), b = __uint_as_float(ob[e] & 0xFFFF0000u);
            s1 += a + b;
            s2 += a * a + b * b;
          }
        }
        stats[(part * R + row) * 2] = s1;
        stats[(part * R + row) * 2 + 1] = s2;
        if (!epi_barrier()) goto fail;
        float t1 = 0.f, t2 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          t1 += stats[(q * R + row) * 2];
          t2 += stats[(q * R + row) * 2 + 1];
        }
        const float mu = t1 / (float)hv;
        const float var = fmaxf(t2 / (float)hv - mu * mu, 0.f);
        const float rs = rsqrtf(var + p.eps);
        // the gate goes over x-hat (every f1 is done: all A V were read after their f1)
#pragma unroll 1
        for (int c8 = 0; c8 < ncol / 16; ++c8) {
          uint32_t ob[8], ub[8];
          tmem_ld_32x32b_x8(tmem + kColOb + lane_off + (c0 >> 1) + 8 * c8, ob);
          tmem_ld_32x32b_x8(tmem + kColU + lane_off + (c0 >> 1) + 8 * c8, ub);
          tmem_ld_wait();
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = c0 + 16 * c8 + 2 * e;
            const float o0 = __uint_as_float(ob[e] << 16), o1 = __uint_as_float(ob[e] & 0xFFFF0000u);
            const float u0 = __uint_as_float(ub[e] << 16), u1 = __uint_as_float(ub[e] & 0xFFFF0000u);
            const float g0 = ((o0 - mu) * rs * p.ln2_g[c] + p.ln2_b[c]) * u0;
            const float g1 = ((o1 - mu) * rs * p.ln2_g[c + 1] + p.ln2_b[c + 1]) * u1;
            pk[e] = row < n ? pack_bf16x2(g0, g1) : 0u;
          }
#pragma unroll
          for (int q = 0; q < 2; ++q)
            st_shared_v4(sA + sw_off(row, c0 + 16 * c8 + 8 * q), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                         pk[4 * q + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->gate_ready);
      }
      // ---- f2 epilogue: + b2 + X, bf16, rows of the sequence only
      if (!warp_wait(&bars->f2_full, k & 1, tmo, abort_flag)) goto fail;
      tc_fence_after();
      {
        const int ncol = d / 4;             // 16 .. 64 columns per part
        const int c0 = part * ncol;
#pragma unroll 1
        for (int c16 = 0; c16 < ncol / 16; ++c16) {
          uint32_t raw[16];
          tmem_ld_32x32b_x16(tmem + kColAcc + lane_off + c0 + 16 * c16, raw);
          tmem_ld_wait();
          if (row < n) {
            const int c = c0 + 16 * c16;
            const __nv_bfloat16* xr = p.x + (int64_t)(start + row) * d + c;
            const uint4 xa = *reinterpret_cast<const uint4*>(xr);
            const uint4 xb = *reinterpret_cast<const uint4*>(xr + 8);
            const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float y0 = __uint_as_float(raw[2 * e]) + p.b2[c + 2 * e] + __uint_as_float(xw[e] << 16);
              const float y1 =
                  __uint_as_float(raw[2 * e + 1]) + p.b2[c + 2 * e + 1] + __uint_as_float(xw[e] & 0xFFFF0000u);
              pk[e] = pack_bf16x2(y0, y1);
            }
            __nv_bfloat16* yr = p.y + (int64_t)(start + row) * d + c;
            *reinterpret_cast<uint4*>(yr) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(yr + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
    }
  }
  goto teardown;
fail:
  set_status(prm.status, HSTU_ERR_TIMEOUT);
  *abort_flag = 1;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kRingStages; ++s) {
      mbar_wait(&bars->ring_full[s], 0, 100000000ll, nullptr);
      mbar_wait(&bars->ring_full[s], 1, 100000000ll, nullptr);
    }
  }
teardown:
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 weight [rows, cols] (row stride cols), box 64 columns x 64 rows, 128-byte swizzle
bool make_wmap(CUtensorMap* m, const void* base, int64_t cols, int64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms_fused() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

bool fused_short_supported(int d_model, int num_heads, int head_dim, int dtype, int io_dtype) {
  const int hv = num_heads * head_dim;
  return dtype == HSTU_DTYPE_BF16 && io_dtype == HSTU_DTYPE_BF16 && head_dim == DH && d_model % 64 == 0 &&
         d_model >= 64 && d_model <= kMaxD && hv % 64 == 0 && hv >= 64 && hv <= kMaxD;
}

int fused_short_max_len() { return R; }

cudaError_t launch_fused_short(const FusedShortArgs& a, cudaStream_t st) {
  FusedParams fp;
  memset(&fp, 0, sizeof(fp));
  fp.offs = a.offs; fp.num_targets = a.num_targets; fp.ts = a.ts;
  fp.x = (const __nv_bfloat16*)a.x; fp.y = (__nv_bfloat16*)a.y;
  fp.b1 = a.b1; fp.ln1_g = a.ln1_g; fp.ln1_b = a.ln1_b; fp.ln2_g = a.ln2_g; fp.ln2_b = a.ln2_b; fp.b2 = a.b2;
  fp.pos_bias = a.pos_bias; fp.time_bias = a.time_bias; fp.rab_head_stride = a.rab_head_stride;
  fp.B = a.B; fp.T = a.T; fp.d = a.d; fp.H = a.H; fp.hv = a.H * DH; fp.eps = a.eps;
  fp.ln2_over_div = (float)(0.69314718055994530942 / a.time_div);
  fp.thr = a.thr;
  fp.cursor = a.cursor; fp.status = a.status; fp.timeout_ns = a.timeout_ns;
  if (!make_wmap(&fp.map_w1, a.w1, a.d, 4 * fp.hv) || !make_wmap(&fp.map_w2, a.w2, fp.hv, a.d))
    return cudaErrorInvalidValue;
  const int smem = Layout::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(fused_short_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // units: ceil(T / 128) windows and the boundaries between them (an upper bound:
  // the kernel reads the used token count from the offsets)
  const int64_t units = 2 * (((int64_t)a.T + R - 1) / R) - 1;
  const int grid = units < num_sms_fused() ? (units > 0 ? (int)units : 1) : num_sms_fused();
  fused_short_kernel<<<grid, kThreads, smem, st>>>(fp);
  return cudaGetLastError();
}

}  // namespace hstu
