// Pointwise aggregated attention backward on the sm_100a tensor cores (bf16,
// head dim 64).
//
// Forward: O_i = (1/N) sum_{j in mask(i)} SiLU(s_ij) v_j, s_ij = q_i . k_j + rab_ij.
// With P_ij = SiLU(s_ij)/N and dS_ij = (dO_i . v_j) SiLU'(s_ij)/N on attended pairs:
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K,  d rab[bucket] = sum of dS over the bucket.
// ("Actions Speak Louder than Words" summary, 1.2 and 2.2: the attention is
// trained end to end; the relative bias tables receive gradients.)
//
// One persistent CTA per SM takes kv-tile work items (sequence, head, 128 kv
// rows; longest first) from a shared cursor.  For every q tile of 128 rows that
// attends to the kv tile:
//   warp 0      fetches the items; TMA: K, V and the kv tile's timestamp record
//               per item (two stages), Q, dO and the q tile's record per q tile
//               (two stages)
//   warp 1      issues tcgen05.mma (whole warp, one elected lane):
//                 S^T  = K Q^T    -> TMEM columns [0, 128)
//                 dP^T = V dO^T   -> [128, 256)
//                 dV  += P^T dO   (P^T from TMEM [256, 320))      -> [320, 384)
//                 dK  += dS^T Q   (dS^T from shared memory)       -> [384, 448)
//                 dQ   = dS K     (the same tile read transposed) -> [448, 512)
//               S^T and dP^T of the next q tile are issued as soon as the
//               epilogue has read this tile's, before this tile's dV, dK, dQ, so
//               the tensor core works on one tile while the epilogue works on
//               the other.
//   warps 2-17  epilogue, one warp per TMEM lane quarter (32 kv rows) and 32 q
//               columns.  Three kinds of segment:
//               far    every q row at least 127 positions past every kv row:
//                      the position bucket is the last one, and the timestamp
//                      records bound each lane's time buckets to at most four;
//                      their bias is per lane, their dS sums stay in registers
//               band   within 160 positions of the diagonal (history rows): bias,
//                      mask and time bucket come from a precomputed band (one
//                      word per pair); dS is summed per position bucket along
//                      diagonals (one shuffle per column) and per time bucket
//                      along runs
//               other  (candidates, per-head bias tables, 64-bit time offsets)
//                      everything per element
//               P^T (bf16) goes to TMEM, dS^T (bf16) to shared memory; the dQ
//               of a tile and the dK, dV of an item are read out while the
//               next tile's scores are already there (fp32 dQ with vector
//               atomics into an accumulator, dK and dV as bf16 rows).
// Every device-side wait is bounded (HSTU_ERR_TIMEOUT).
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
namespace {
using namespace sm100;

constexpr int BT = 128;                  // q rows and kv rows per tile
constexpr int DHB = 64;                  // head dimension of this kernel
constexpr int kEpiWarps = 16;
constexpr int kEpiWarp0 = 2;             // warp 0: loads, 1: MMA, 2..17: epilogue
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kTile = BT * DHB * 2;      // one [128 x 64] bf16 tile: 128 rows of 128 bytes (16 KB)
constexpr int kStages = 2;               // K/V stages and Q/dO stages
constexpr int kItemSlots = 4;
constexpr int kItemReaders = 1 + kEpiWarps;   // MMA warp and epilogue warps
constexpr int kRecBytes = kTsRecWords * 4;
constexpr uint32_t kColS = 0, kColDP = 128, kColP = 256, kColDV = 320, kColDK = 384, kColDQ = 448;
constexpr uint32_t kTmemCols = 512;
constexpr float kMaskedBias = -1e30f;    // a masked pair's bias: SiLU and SiLU' of it are 0

struct BwdBars {
  uint64_t it_full[kItemSlots], it_empty[kItemSlots];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[kStages], q_empty[kStages];
  uint64_t sp_full, sp_free, p_ready, pds_free, dq_full, dq_empty, acc_full, acc_empty;
  uint64_t epi_sync;   // barrier among the epilogue warps (bounded waits, unlike bar.sync)
  uint64_t done;
};

struct BwdLayout {
  static constexpr int kKV = 0;                                  // per stage: K tile, V tile
  static constexpr int kQ = kKV + kStages * 2 * kTile;           // per stage: Q tile, dO tile
  static constexpr int kDS = kQ + kStages * 2 * kTile;           // dS^T [128 kv x 128 q] bf16: two 64-column atoms
  static constexpr int kKRec = kDS + 2 * kTile;                  // kv tile records, per K/V stage
  static constexpr int kQRec = kKRec + kStages * kRecBytes;      // q tile records, per Q stage
  static constexpr int kThr = kQRec + kStages * kRecBytes;
  static constexpr int kThr32 = kThr + kNumBuckets * 8;
  static constexpr int kPosB = kThr32 + (kNumBuckets + 4) * 4;
  static constexpr int kTimeB = kPosB + kNumBuckets * 4;
  static constexpr int kBar = (kTimeB + kNumBuckets * 4 + 15) & ~15;
  static constexpr int kItems = kBar + (int)sizeof(BwdBars);
  static constexpr int kMisc = kItems + kItemSlots * 8 * 4;
  static constexpr int kDiag = kMisc + 16;                       // per epilogue warp: 32 completed diagonal sums
  static constexpr int kPend = kDiag + kEpiWarps * 32 * 4;        // per epilogue thread: pending readout rows
  static constexpr int kEnd = kPend + kEpiWarps * 32 * 8;
  static constexpr int kAlloc = kEnd + 1024;  // slack for 1024-byte alignment of the base
};
static_assert(BwdLayout::kAlloc <= 227 * 1024, "shared memory");

struct BwdTcParams {
  CUtensorMap map_q, map_k, map_v, map_do;
  AttnBwdParams p;
  float ln2_over_div;
};

// q tiles (of BT rows) holding a row that attends to kv tile kt
__device__ __forceinline__ bool q_tile_hits(const SeqInfo& si, int qt, int kt) {
  const int r0 = qt * BT;
  const KvRange kr = kv_tiles_for(r0, min(si.n, r0 + BT), si.hist, BT);
  return kt < kr.a || (kt >= kr.b0 && kt < kr.b1);
}

// A fetched work item and its sequence's facts, as the item ring holds them.
struct ItemInfo {
  int idx;   // -1: no more items
  WorkItem wi;
  SeqInfo si;
};

__device__ __forceinline__ void ring_put(volatile int* ring, int slot, const ItemInfo& x) {
  volatile int* w = ring + 8 * slot;
  w[0] = x.idx; w[1] = x.wi.seq; w[2] = x.wi.head; w[3] = x.wi.qtile;
  w[4] = x.si.start; w[5] = x.si.n; w[6] = x.si.hist; w[7] = __float_as_int(x.si.inv_n);
}

__device__ __forceinline__ ItemInfo ring_get(const volatile int* ring, int slot) {
  const volatile int* w = ring + 8 * slot;
  ItemInfo x;
  x.idx = w[0]; x.wi.seq = w[1]; x.wi.head = w[2]; x.wi.qtile = w[3]; x.wi.cost = 0;
  x.si.start = w[4]; x.si.n = w[5]; x.si.hist = w[6]; x.si.inv_n = __int_as_float(w[7]);
  return x;
}

// ---------------------------------------------------------------- packed fp32 pairs
__device__ __forceinline__ void mul2(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma2(float a0, float a1, float b0, float b1, float c0, float c1, float& r0,
                                     float& r1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
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

// For two scores x (bias included) and their dP: P = SiLU(x)/N as packed bf16 and
// dS = dP SiLU'(x)/N in fp32, from sigma(x) = 1 / (1 + 2^(-x log2 e)):
//   SiLU(x) = x sigma,  SiLU'(x) = sigma (1 + x (1 - sigma)).
// sigma is accurate to a few fp32 ulps everywhere (the relative-bias gradients
// sum dS over up to millions of pairs, so its error must not be systematic); a
// masked pair's bias of -1e30 gives sigma = 0, hence P = dS = 0.
__device__ __forceinline__ void p_ds2(float x0, float x1, float dp0, float dp1, float inv_n, uint32_t& pw,
                                      float& ds0, float& ds1) {
  float a0, a1;
  mul2(x0, x1, -1.4426950408889634f, -1.4426950408889634f, a0, a1);
  float d0, d1;
  add2(ex2_approx(a0), ex2_approx(a1), 1.0f, 1.0f, d0, d1);
  const float s0 = rcp_approx(d0), s1 = rcp_approx(d1);
  float sn0, sn1, p0, p1, om0, om1, t0, t1, u0, u1;
  mul2(s0, s1, inv_n, inv_n, sn0, sn1);              // sigma / N
  mul2(x0, x1, sn0, sn1, p0, p1);                    // P
  fma2(s0, s1, -1.0f, -1.0f, 1.0f, 1.0f, om0, om1);  // 1 - sigma
  fma2(x0, x1, om0, om1, 1.0f, 1.0f, t0, t1);        // 1 + x (1 - sigma)
  mul2(dp0, dp1, sn0, sn1, u0, u1);
  mul2(u0, u1, t0, t1, ds0, ds1);                    // dS
  pw = pack_bf16x2(p0, p1);
}

__device__ __forceinline__ void red_add(float* addr, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a) : "memory");
}
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void store_bf16_row16(__nv_bfloat16* dst, const uint32_t (&r)[16]) {
  uint4 w0, w1;
  w0.x = pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1]));
  w0.y = pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3]));
  w0.z = pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5]));
  w0.w = pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]));
  w1.x = pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9]));
  w1.y = pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11]));
  w1.z = pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13]));
  w1.w = pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15]));
  *reinterpret_cast<uint4*>(dst) = w0;
  *reinterpret_cast<uint4*>(dst + 8) = w1;
}

__global__ void __launch_bounds__(kThreads, 1) attn_bwd_tc_kernel(const __grid_constant__ BwdTcParams prm) {
  using L = BwdLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + L::kBar);
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::kItems);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int64_t* thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int32_t* thr32 = reinterpret_cast<int32_t*>(smem + L::kThr32);
  float* pos_b = reinterpret_cast<float*>(smem + L::kPosB);
  float* time_b = reinterpret_cast<float*>(smem + L::kTimeB);
  const TsRec* krecs = reinterpret_cast<const TsRec*>(smem + L::kKRec);
  const TsRec* qrecs = reinterpret_cast<const TsRec*>(smem + L::kQRec);
  const uint32_t sKV = smem_u32(smem + L::kKV);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sDS = smem_u32(smem + L::kDS);
  float* diag_all = reinterpret_cast<float*>(smem + L::kDiag);

  const AttnBwdParams& p = prm.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tmo = p.timeout_ns;
  const int count = *p.item_count;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kItemSlots; ++s) { mbar_init(&bars->it_full[s], 1); mbar_init(&bars->it_empty[s], kItemReaders); }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1 + kEpiWarps);
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1 + kEpiWarps);
    }
    mbar_init(&bars->sp_full, 1);
    mbar_init(&bars->sp_free, kEpiWarps);
    mbar_init(&bars->p_ready, kEpiWarps);
    mbar_init(&bars->pds_free, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, kEpiWarps);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kEpiWarps);
    mbar_init(&bars->epi_sync, kEpiWarps);
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&prm.map_q);
    tma_prefetch_desc(&prm.map_k);
    tma_prefetch_desc(&prm.map_v);
    tma_prefetch_desc(&prm.map_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  const int per_head_rab = p.rab_head_stride != 0;
  for (int c = threadIdx.x; c < kNumBuckets + 4; c += kThreads) {
    if (c < kNumBuckets) {
      thr[c] = p.thr.v[c];
      thr32[c] = p.thr.v[c] > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)p.thr.v[c];
      pos_b[c] = p.pos_bias[c];
      time_b[c] = p.time_bias[c];
    } else {
      thr32[c] = 0x7FFFFFFF;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================================ items and loads
    if (lane == 0) {
      const TsRec* grecs = reinterpret_cast<const TsRec*>(p.tile_recs);
      int g = 0;
      for (int k = 0;; ++k) {
        const int slot = k % kItemSlots;
        if (!mbar_wait(&bars->it_empty[slot], ((k / kItemSlots) & 1) ^ 1, tmo, abort_flag)) goto fail;
        ItemInfo x;
        x.idx = *abort_flag ? -1 : atomicAdd(p.item_cursor, 1);
        if (x.idx >= count) x.idx = -1;
        if (x.idx >= 0) {
          x.wi = p.items[x.idx];
          x.si = load_seq(p.seq_offsets, p.num_targets, x.wi.seq);
        }
        ring_put(item_ring, slot, x);
        mbar_arrive(&bars->it_full[slot]);
        if (x.idx < 0) break;
        const int kt = x.wi.qtile;   // backward items carry the kv tile
        const int h = x.wi.head;
        const TsRec* srec = grecs + p.tile_base[x.wi.seq];
        const int ks = k % kStages;
        if (!mbar_wait(&bars->kv_empty[ks], ((k / kStages) & 1) ^ 1, tmo, abort_flag)) goto fail;
        mbar_arrive_expect_tx(&bars->kv_full[ks], 2 * kTile + kRecBytes);
        tma_load_2d(smem + L::kKV + ks * 2 * kTile, &prm.map_k, &bars->kv_full[ks], h * DHB, x.si.start + kt * BT);
        tma_load_2d(smem + L::kKV + ks * 2 * kTile + kTile, &prm.map_v, &bars->kv_full[ks], h * DHB,
                    x.si.start + kt * BT);
        bulk_load(smem + L::kKRec + ks * kRecBytes, srec + kt, kRecBytes, &bars->kv_full[ks]);
        const int nq = (x.si.n + BT - 1) / BT;
        for (int qt = kt; qt < nq; ++qt) {
          if (!q_tile_hits(x.si, qt, kt)) continue;
          const int qs = g % kStages;
          if (!mbar_wait(&bars->q_empty[qs], ((g / kStages) & 1) ^ 1, tmo, abort_flag)) goto fail;
          mbar_arrive_expect_tx(&bars->q_full[qs], 2 * kTile + kRecBytes);
          tma_load_2d(smem + L::kQ + qs * 2 * kTile, &prm.map_q, &bars->q_full[qs], h * DHB, x.si.start + qt * BT);
          tma_load_2d(smem + L::kQ + qs * 2 * kTile + kTile, &prm.map_do, &bars->q_full[qs], h * DHB,
                      x.si.start + qt * BT);
          bulk_load(smem + L::kQRec + qs * kRecBytes, srec + qt, kRecBytes, &bars->q_full[qs]);
          ++g;
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    constexpr uint32_t id_s = make_idesc_bf16(BT, BT, false, false);      // S^T, dP^T
    constexpr uint32_t id_kv = make_idesc_bf16(BT, DHB, false, true);     // dV, dK: B MN-major
    constexpr uint32_t id_q = make_idesc_bf16(BT, DHB, true, true);       // dQ: A and B MN-major
    const uint64_t dDS_kmaj = make_sw128_desc(sDS, 16, 1024);
    const uint64_t dDS_mn = make_sw128_desc(sDS, 16384, 1024);
    // S^T and dP^T of q tile qt of the item in K/V stage ks, into the score buffers
    auto issue_sp = [&](int ks, int g) {
      const int qs = g % kStages;
      const uint32_t sk = sKV + ks * 2 * kTile, sv = sk + kTile;
      const uint32_t sq = sQ + qs * 2 * kTile, sdo = sq + kTile;
      const uint64_t dk = make_sw128_desc(sk, 16, 1024), dv = make_sw128_desc(sv, 16, 1024);
      const uint64_t dq = make_sw128_desc(sq, 16, 1024), ddo = make_sw128_desc(sdo, 16, 1024);
#pragma unroll
      for (int s = 0; s < DHB / 16; ++s)
        umma_f16_ss_elect(tmem + kColS, desc_advance(dk, s * 32), desc_advance(dq, s * 32), id_s, s > 0 ? 1u : 0u);
#pragma unroll
      for (int s = 0; s < DHB / 16; ++s)
        umma_f16_ss_elect(tmem + kColDP, desc_advance(dv, s * 32), desc_advance(ddo, s * 32), id_s, s > 0 ? 1u : 0u);
      umma_commit_elect(&bars->sp_full);
    };
    int k = 0, g = 0;
    // the current item (cur) and, once its last q tile is reached, the next one
    auto fetch = [&](int kk, ItemInfo& x) -> bool {
      const int slot = kk % kItemSlots;
      if (!warp_wait(&bars->it_full[slot], (kk / kItemSlots) & 1, tmo, abort_flag)) return false;
      x = ring_get(item_ring, slot);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->it_empty[slot]);
      return true;
    };
    ItemInfo cur;
    if (!fetch(0, cur)) goto fail;
    if (cur.idx >= 0) {
      {
        // the first item's first q tile
        if (!warp_wait(&bars->kv_full[0], 0, tmo, abort_flag)) goto fail;
        if (!warp_wait(&bars->q_full[0], 0, tmo, abort_flag)) goto fail;
        tc_fence_after();
        issue_sp(0, 0);
      }
      for (;;) {
        const int kt = cur.wi.qtile;
        const int nq = (cur.si.n + BT - 1) / BT;
        const int ks = k % kStages;
        const uint32_t sk = sKV + ks * 2 * kTile;
        const uint64_t dK_mn = make_sw128_desc(sk, 16384, 1024);
        // acc_empty: the epilogue has read the previous item's dK and dV
        if (!warp_wait(&bars->acc_empty, (k & 1) ^ 1, tmo, abort_flag)) goto fail;
        int qt = kt;
        while (qt < nq - 1 && !q_tile_hits(cur.si, qt, kt)) ++qt;   // the item's first q tile (issued already)
        bool first = true;
        ItemInfo nxt;
        nxt.idx = -1;
        bool have_next = false;
        for (;;) {
          int qn = qt + 1;
          while (qn < nq && !q_tile_hits(cur.si, qn, kt)) ++qn;
          const bool last = qn >= nq;
          // S^T, dP^T of the next q tile (this item's, or the next item's first), once
          // the epilogue has read this tile's scores
          if (!warp_wait(&bars->sp_free, g & 1, tmo, abort_flag)) goto fail;
          if (!last) {
            if (!warp_wait(&bars->q_full[(g + 1) % kStages], ((g + 1) / kStages) & 1, tmo, abort_flag)) goto fail;
            tc_fence_after();
            issue_sp(ks, g + 1);
          } else {
            if (!fetch(k + 1, nxt)) goto fail;
            have_next = nxt.idx >= 0;
            if (have_next) {
              const int ks2 = (k + 1) % kStages;
              if (!warp_wait(&bars->kv_full[ks2], ((k + 1) / kStages) & 1, tmo, abort_flag)) goto fail;
              if (!warp_wait(&bars->q_full[(g + 1) % kStages], ((g + 1) / kStages) & 1, tmo, abort_flag)) goto fail;
              tc_fence_after();
              issue_sp(ks2, g + 1);
            }
          }
          // dV, dK, dQ of this tile once the epilogue has written P^T and dS^T
          if (!warp_wait(&bars->p_ready, g & 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
          const int qs = g % kStages;
          const uint32_t sq = sQ + qs * 2 * kTile, sdo = sq + kTile;
          const uint64_t dq_mn = make_sw128_desc(sq, 16384, 1024), ddo_mn = make_sw128_desc(sdo, 16384, 1024);
#pragma unroll
          for (int s = 0; s < BT / 16; ++s)   // dV += P^T dO (reduction over the tile's 128 q rows)
            umma_f16_ts_elect(tmem + kColDV, tmem + kColP + 8 * s, desc_advance(ddo_mn, s * 2048), id_kv,
                              (!first || s > 0) ? 1u : 0u);
#pragma unroll
          for (int s = 0; s < BT / 16; ++s)   // dK += dS^T Q
            umma_f16_ss_elect(tmem + kColDK, desc_advance(dDS_kmaj, (s >> 2) * 16384 + (s & 3) * 32),
                              desc_advance(dq_mn, s * 2048), id_kv, (!first || s > 0) ? 1u : 0u);
          if (!warp_wait(&bars->dq_empty, (g & 1) ^ 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < BT / 16; ++s)   // dQ = dS K (reduction over the kv tile's 128 rows)
            umma_f16_ss_elect(tmem + kColDQ, desc_advance(dDS_mn, s * 2048), desc_advance(dK_mn, s * 2048), id_q,
                              s > 0 ? 1u : 0u);
          umma_commit_elect(&bars->pds_free);
          umma_commit_elect(&bars->dq_full);
          umma_commit_elect(&bars->q_empty[qs]);
          first = false;
          ++g;
          if (last) break;
          qt = qn;
        }
        umma_commit_elect(&bars->acc_full);
        umma_commit_elect(&bars->kv_empty[ks]);
        ++k;
        if (!have_next) break;
        cur = nxt;
      }
    }
    // every MMA issued completes before TMEM is released
    umma_commit_elect(&bars->done);
    warp_wait(&bars->done, 0, tmo, nullptr);
  } else {
    // ================================================================ epilogue
    const int ew = warp - kEpiWarp0;       // 0..15
    const int quarter = warp & 3;          // TMEM lane quarter: kv rows 32 quarter ..
    const int seg = ew >> 2;               // q columns [32 seg, 32 seg + 32) of the q tile
    const int jl = quarter * 32 + lane;    // kv row inside the tile
    float* const diag_w = diag_all + ew * 32;   // this warp's completed diagonal sums (band segments)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float k_lg = prm.ln2_over_div;
    const int etid = threadIdx.x - 32 * kEpiWarp0;
    int cur_head = -1;
    float far_pos = 0.f;                   // dS of pairs in the last position bucket (summed in registers)
    // deferred readouts: dQ of the previous q tile, dK and dV of the previous item
    bool pend_dq = false, pend_acc = false;
    // their destinations wait in shared memory (no registers while pending): the dQ
    // accumulator row and the dK/dV row, each as token * heads + head (-1: none)
    int2* const pend_rows = reinterpret_cast<int2*>(smem + L::kPend) + (threadIdx.x - 32 * kEpiWarp0);
    int acc_par = 0;
    // every epilogue warp at the same point: an mbarrier phase (a warp that gave up on
    // a bounded wait sets the abort flag, and the others' waits return)
    int epi_phase = 0;
    auto epi_barrier = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->epi_sync);
      const bool ok = warp_wait(&bars->epi_sync, epi_phase & 1, tmo, abort_flag);
      ++epi_phase;
      return ok;
    };
    // relative-bias gradients: this CTA's partial tables in global memory (fp32
    // reductions in L2; shared-memory float atomics would serialise), one pair of
    // 128-entry tables per bias table; a later pass adds the CTAs' partials up
    float* gpos = p.rab_partial + (size_t)blockIdx.x * p.rab_tables * 2 * kNumBuckets;
    float* gtime = gpos + kNumBuckets;
    auto flush_far = [&]() {
      float fp = far_pos;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) fp += __shfl_xor_sync(0xffffffffu, fp, o);
      if (lane == 0 && fp != 0.f) red_add(&gpos[kNumBuckets - 1], fp);
      far_pos = 0.f;
    };
    // the deferred readouts of the previous q tile's dQ and the previous item's dK
    // and dV, then the wait until the previous tile's P^T and dS^T are consumed
    int g = 0;
    auto readouts = [&]() -> bool {
      if (pend_dq) {
        if (!mbar_wait(&bars->dq_full, (g - 1) & 1, tmo, abort_flag)) return false;
        tc_fence_after();
        uint32_t qr[16];
        tmem_ld_32x32b_x16(tmem + kColDQ + lane_off + 16 * seg, qr);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->dq_empty);
        const int dq_r = pend_rows->x;
        if (dq_r >= 0) {
          float* dq_dst = p.dq_accum + (int64_t)dq_r * DHB + 16 * seg;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            red_add_v4(dq_dst + 4 * c, __uint_as_float(qr[4 * c]), __uint_as_float(qr[4 * c + 1]),
                       __uint_as_float(qr[4 * c + 2]), __uint_as_float(qr[4 * c + 3]));
        }
        pend_dq = false;
      }
      if (pend_acc) {
        if (!mbar_wait(&bars->acc_full, acc_par, tmo, abort_flag)) return false;
        tc_fence_after();
        {
          uint32_t vr[16];
          tmem_ld_32x32b_x16(tmem + kColDV + lane_off + 16 * seg, vr);
          tmem_ld_wait();
          const int kv_r = pend_rows->y;
          if (kv_r >= 0)
            store_bf16_row16(reinterpret_cast<__nv_bfloat16*>(p.dv) + (int64_t)(kv_r / p.num_heads) * p.lddv +
                                 (kv_r % p.num_heads) * DHB + 16 * seg, vr);
        }
        {
          uint32_t kr[16];
          tmem_ld_32x32b_x16(tmem + kColDK + lane_off + 16 * seg, kr);
          tmem_ld_wait();
          const int kv_r = pend_rows->y;
          if (kv_r >= 0)
            store_bf16_row16(reinterpret_cast<__nv_bfloat16*>(p.dk) + (int64_t)(kv_r / p.num_heads) * p.lddk +
                                 (kv_r % p.num_heads) * DHB + 16 * seg, kr);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty);
        pend_acc = false;
      }
      if (!mbar_wait(&bars->pds_free, (g & 1) ^ 1, tmo, abort_flag)) return false;
      tc_fence_after();
      return true;
    };
    for (int k = 0;; ++k) {
      const int slot = k % kItemSlots;
      if (!mbar_wait(&bars->it_full[slot], (k / kItemSlots) & 1, tmo, abort_flag)) goto fail;
      const ItemInfo x = ring_get(item_ring, slot);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->it_empty[slot]);
      if (x.idx < 0) break;
      const SeqInfo si = x.si;
      const int kt = x.wi.qtile, h = x.wi.head;
      if (per_head_rab && h != cur_head) {
        // this head's tables, and its partial gradient tables
        if (cur_head >= 0) flush_far();
        if (!epi_barrier()) goto fail;
        for (int c = etid; c < kNumBuckets; c += 32 * kEpiWarps) {
          pos_b[c] = p.pos_bias[h * p.rab_head_stride + c];
          time_b[c] = p.time_bias[h * p.rab_head_stride + c];
        }
        if (!epi_barrier()) goto fail;
        gpos = p.rab_partial + ((size_t)blockIdx.x * p.rab_tables + h) * 2 * kNumBuckets;
        gtime = gpos + kNumBuckets;
        cur_head = h;
      }
      const int ks = k % kStages;
      if (!mbar_wait(&bars->kv_full[ks], (k / kStages) & 1, tmo, abort_flag)) goto fail;
      const TsRec& krec = krecs[ks];
      const int j = kt * BT + jl;
      const int j0 = kt * BT + quarter * 32;    // first kv row of the warp
      const bool jlive = j < si.n;
      const int32_t rj = krec.rel[jl];
      const int posj = token_pos(j, si.hist);
      const int nq = (si.n + BT - 1) / BT;
      for (int qt = kt; qt < nq; ++qt) {
        if (!q_tile_hits(si, qt, kt)) continue;
        const int qs = g % kStages;
        if (!mbar_wait(&bars->q_full[qs], (g / kStages) & 1, tmo, abort_flag)) goto fail;
        const TsRec& qrec = qrecs[qs];
        // ---- classify this warp's segment (the records alone decide it)
        const int i0 = qt * BT + 32 * seg;     // first q row of the segment
        const int D = i0 - j0;                 // i - j = D + col - lane for column col, lane
        const bool narrow = !krec.wide && !qrec.wide;
        // kind: 0 masked, 1 far, 2 band, 3 per element
        int kind = 3;
        if (D + 31 < 0) kind = 0;                                           // every i < j
        else if (narrow && D >= 158 && (i0 + 31 < si.hist || (si.hist == si.n && i0 < si.n)))
          kind = 1;   // i - j >= 127 everywhere (q rows beyond a sequence without targets are masked)
        else if (p.band != nullptr && D >= 0 && D < kBwdBandCols && (i0 + 31 < si.hist || si.hist == si.n))
          kind = 2;
        // far: time buckets of this lane's row over the segment's q columns, from the
        // records' per-segment timestamp range
        int tlo = 0, lrank = 1;
        int32_t th1 = 0x7FFFFFFF, th2 = 0x7FFFFFFF, th3 = 0x7FFFFFFF;
        if (kind == 1) {
          const int32_t mn = qrec.mn[seg], mx = qrec.mx[seg];
          int32_t dlo, dhi;
          if (rj <= mn) { dlo = mn - rj; dhi = mx - rj; }
          else if (rj >= mx) { dlo = rj - mx; dhi = rj - mn; }
          else { dlo = 0; dhi = max(rj - mn, mx - rj); }
          tlo = fast_bucket(dlo, thr32, k_lg);
          th1 = thr32[tlo + 1];
          th2 = thr32[tlo + 2];
          th3 = thr32[tlo + 3];
          lrank = dhi < th1 ? 1 : (dhi < th2 ? 2 : (dhi < th3 ? 3 : (dhi < thr32[tlo + 4] ? 4 : 5)));
          if (__any_sync(0xffffffffu, lrank > 4)) kind = 3;
        }
        int wrank = kind == 1 ? __reduce_max_sync(0xffffffffu, lrank) : 0;
        // two buckets and every q row's timestamp at or after this lane's: the bucket of a
        // column is one compare of its timestamp offset with rj + th1
        if (wrank == 2 && __all_sync(0xffffffffu, rj <= qrec.mn[seg])) wrank = -2;
        const int64_t up64 = (int64_t)rj + th1;
        const int32_t up_at = up64 > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)up64;
        const float inv_n = si.inv_n;
        const uint32_t ds_atom = sDS + (seg >> 1) * kTile + jl * 128;   // dS^T row jl, q columns 32 seg ..
        const int ds_ch = (seg & 1) * 4;
        // far-segment state
        const float pb127 = pos_b[kNumBuckets - 1];
        const float hb0 = pb127 + time_b[tlo];
        const float hb1 = pb127 + time_b[min(tlo + 1, kNumBuckets - 1)];
        const float hb2 = pb127 + time_b[min(tlo + 2, kNumBuckets - 1)];
        const float hb3 = pb127 + time_b[min(tlo + 3, kNumBuckets - 1)];
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        // band-segment state: the diagonal running sum and the time-bucket run
        float dg = 0.f, at = 0.f;
        int cur_tb = -1;
        const uint4* bp = reinterpret_cast<const uint4*>(p.band + (int64_t)(si.start + (jlive ? j : 0)) * kBwdBandCols +
                                                         (D > 0 ? D : 0));
        // band words of the segment's first chunk, in flight while the scores are awaited
        // (kv rows beyond the sequence read none: masked)
        uint4 wn0 = make_uint4(0u, 0u, 0u, 0u), wn1 = wn0;
        const uint32_t kMaskedWord = __float_as_uint(kMaskedBias) & 0xFFFF0000u;
        if (kind == 2) {
          if (jlive) {
            wn0 = __ldg(bp);
            wn1 = __ldg(bp + 1);
          } else {
            wn0 = wn1 = make_uint4(kMaskedWord, kMaskedWord, kMaskedWord, kMaskedWord);
          }
        }
        if (!mbar_wait(&bars->sp_full, g & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        if (kind != 3) {
          // one copy of the chunk loop per kind (each with only its own state live)
          // the deferred readouts (their MMAs ran while the scores were awaited), then the
          // previous tile's P^T and dS^T must have been consumed before this tile's are written
          if (!readouts()) goto fail;
          auto chunks = [&](auto&& compute) -> bool {
          // ---- the segment in four chunks of 8 q columns: S^T and dP^T of the chunk into
          // registers (the last chunk's load frees the score buffers for the next tile's
          // MMAs), P and dS, then P^T into TMEM and dS^T into shared memory
#pragma unroll 1
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t sr[8], dr[8];
            tmem_ld_32x32b_x8(tmem + kColS + lane_off + 32 * seg + 8 * c8, sr);
            tmem_ld_32x32b_x8(tmem + kColDP + lane_off + 32 * seg + 8 * c8, dr);
            // band words of this chunk (loaded one chunk ahead), and the next chunk's in flight
            const uint32_t w[8] = {wn0.x, wn0.y, wn0.z, wn0.w, wn1.x, wn1.y, wn1.z, wn1.w};
            if (kind == 2 && c8 < 3 && jlive) {
              wn0 = __ldg(bp + 2 * c8 + 2);
              wn1 = __ldg(bp + 2 * c8 + 3);
            }
            tmem_ld_wait();
            if (c8 == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->sp_free);
            }
            if (kind == 1 && i0 + 8 * c8 + 7 >= si.n) {
              // the sequence ends inside this chunk: q rows beyond it are masked
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (i0 + 8 * c8 + e >= si.n) sr[e] = __float_as_uint(kMaskedBias);
            }
            uint32_t pk[4];   // P^T words (bf16 pairs) of the chunk's 8 q columns
            uint32_t dk[4];   // dS^T words
            compute(c8, sr, dr, w, pk, dk);
            tmem_st_32x32b_x4(tmem + kColP + lane_off + 16 * seg + 4 * c8, pk);
            st_shared_v4(ds_atom + (((ds_ch + c8) ^ (jl & 7)) << 4), dk[0], dk[1], dk[2], dk[3]);
          }
          return true;
          };
          bool chunks_ok;
          if (kind == 0) {
            chunks_ok = chunks([&](int c8, const uint32_t (&sr)[8], const uint32_t (&dr)[8], const uint32_t (&w)[8], uint32_t (&pk)[4], uint32_t (&dk)[4]) {
              (void)c8; (void)sr; (void)dr; (void)w;
    #pragma unroll
                  for (int e = 0; e < 4; ++e) { pk[e] = 0u; dk[e] = 0u; }
            });
          }
          else if (kind == 1 && wrank == 1) {
            chunks_ok = chunks([&](int c8, const uint32_t (&sr)[8], const uint32_t (&dr)[8], const uint32_t (&w)[8], uint32_t (&pk)[4], uint32_t (&dk)[4]) {
              (void)c8; (void)sr; (void)dr; (void)w;
    #pragma unroll
                  for (int e = 0; e < 8; e += 2) {
                    float ds0, ds1;
                    p_ds2(__uint_as_float(sr[e]) + hb0, __uint_as_float(sr[e + 1]) + hb0, __uint_as_float(dr[e]),
                          __uint_as_float(dr[e + 1]), inv_n, pk[e >> 1], ds0, ds1);
                    dk[e >> 1] = pack_bf16x2(ds0, ds1);
                    a0 += ds0 + ds1;
                  }
            });
          }
          else if (kind == 1 && wrank == -2) {
            chunks_ok = chunks([&](int c8, const uint32_t (&sr)[8], const uint32_t (&dr)[8], const uint32_t (&w)[8], uint32_t (&pk)[4], uint32_t (&dk)[4]) {
              (void)c8; (void)sr; (void)dr; (void)w;
                  float aup = 0.f;   // the upper bucket's part of what went into a0
    #pragma unroll
                  for (int e4 = 0; e4 < 2; ++e4) {
                    const int4 rel4 = *reinterpret_cast<const int4*>(&qrec.rel[32 * seg + 8 * c8 + 4 * e4]);
                    const int32_t rv[4] = {rel4.x, rel4.y, rel4.z, rel4.w};
                    bool up[4];
                    float xs[4];
    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                      up[u] = rv[u] >= up_at;
                      xs[u] = __uint_as_float(sr[4 * e4 + u]) + (up[u] ? hb1 : hb0);
                    }
    #pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2) {
                      float ds0, ds1;
                      const int e = 4 * e4 + 2 * q2;
                      p_ds2(xs[2 * q2], xs[2 * q2 + 1], __uint_as_float(dr[e]), __uint_as_float(dr[e + 1]), inv_n,
                            pk[e >> 1], ds0, ds1);
                      dk[e >> 1] = pack_bf16x2(ds0, ds1);
                      a0 += ds0 + ds1;
                      aup += (up[2 * q2] ? ds0 : 0.f) + (up[2 * q2 + 1] ? ds1 : 0.f);
                    }
                  }
                  a0 -= aup;
                  a1 += aup;
            });
          }
          else if (kind == 1) {
            chunks_ok = chunks([&](int c8, const uint32_t (&sr)[8], const uint32_t (&dr)[8], const uint32_t (&w)[8], uint32_t (&pk)[4], uint32_t (&dk)[4]) {
              (void)c8; (void)sr; (void)dr; (void)w;
    #pragma unroll
                  for (int e4 = 0; e4 < 2; ++e4) {
                    const int4 rel4 = *reinterpret_cast<const int4*>(&qrec.rel[32 * seg + 8 * c8 + 4 * e4]);
                    const int32_t rv[4] = {rel4.x, rel4.y, rel4.z, rel4.w};
                    float xs[4];
                    int bk[4];
    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                      const int32_t dd = abs(rv[u] - rj);
                      bk[u] = (dd >= th1 ? 1 : 0) + (dd >= th2 ? 1 : 0) + (dd >= th3 ? 1 : 0);
                      const float hb = bk[u] == 0 ? hb0 : (bk[u] == 1 ? hb1 : (bk[u] == 2 ? hb2 : hb3));
                      xs[u] = __uint_as_float(sr[4 * e4 + u]) + hb;
                    }
    #pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2) {
                      float ds0, ds1;
                      const int e = 4 * e4 + 2 * q2;
                      p_ds2(xs[2 * q2], xs[2 * q2 + 1], __uint_as_float(dr[e]), __uint_as_float(dr[e + 1]), inv_n,
                            pk[e >> 1], ds0, ds1);
                      dk[e >> 1] = pack_bf16x2(ds0, ds1);
                      const float dsv[2] = {ds0, ds1};
    #pragma unroll
                      for (int u = 0; u < 2; ++u) {
                        const int b = bk[2 * q2 + u];
                        a0 += b == 0 ? dsv[u] : 0.f;
                        a1 += b == 1 ? dsv[u] : 0.f;
                        a2 += b == 2 ? dsv[u] : 0.f;
                        a3 += b == 3 ? dsv[u] : 0.f;
                      }
                    }
                  }
            });
          }
          else {
            chunks_ok = chunks([&](int c8, const uint32_t (&sr)[8], const uint32_t (&dr)[8], const uint32_t (&w)[8], uint32_t (&pk)[4], uint32_t (&dk)[4]) {
              (void)c8; (void)sr; (void)dr; (void)w;
                  if (c8 == 0) cur_tb = w[0] & 0x7F;
    #pragma unroll
                  for (int e = 0; e < 8; e += 2) {
                    float ds0, ds1;
                    float x0, x1;
                    add2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1]), __uint_as_float(w[e] & 0xFFFF0000u),
                         __uint_as_float(w[e + 1] & 0xFFFF0000u), x0, x1);
                    p_ds2(x0, x1, __uint_as_float(dr[e]), __uint_as_float(dr[e + 1]), inv_n, pk[e >> 1], ds0, ds1);
                    dk[e >> 1] = pack_bf16x2(ds0, ds1);
                    const float dsv[2] = {ds0, ds1};
    #pragma unroll
                    for (int u = 0; u < 2; ++u) {
                      // time bucket: runs along the row
                      const int tb = w[e + u] & 0x7F;
                      const bool change = tb != cur_tb;
                      if (change) red_add(&gtime[cur_tb], at);
                      cur_tb = tb;
                      at = change ? dsv[u] : at + dsv[u];
                      // position bucket D + col - lane: the running sum of the diagonal col - lane
                      // moves one lane down per column, and lane 31's is complete: it is kept
                      // in shared memory until the segment's end
                      dg += dsv[u];
                      const int col = 8 * c8 + e + u;
                      if (lane == 31) diag_w[col] = dg;
                      dg = lane == 31 ? 0.f : dg;
                      dg = __shfl_sync(0xffffffffu, dg, (lane + 31) & 31);
                    }
                  }
            });
          }
          if (!chunks_ok) goto fail;
        } else {
          // ---- per element (candidates, per-head bias tables, 64-bit time offsets): the
          // scores are read 8 columns at a time and the score buffers freed at the end
          if (!readouts()) goto fail;
#pragma unroll 1
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t sr[8], dr[8];
            tmem_ld_32x32b_x8(tmem + kColS + lane_off + 32 * seg + 8 * c8, sr);
            tmem_ld_32x32b_x8(tmem + kColDP + lane_off + 32 * seg + 8 * c8, dr);
            tmem_ld_wait();
            uint32_t pk[4], dk[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float xs[2];
              bool att[2];
              int pbk[2], tbk[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int i = i0 + 8 * c8 + e + u;
                att[u] = jlive && attended(i, j, si.n, si.hist);
                pbk[u] = pos_bucket(token_pos(i, si.hist), posj);
                if (narrow) {
                  tbk[u] = fast_bucket(abs(qrec.rel[32 * seg + 8 * c8 + e + u] - rj), thr32, k_lg);
                } else {
                  const int ii = i < si.n ? i : si.n - 1;
                  const int jj = jlive ? j : 0;
                  tbk[u] = time_bucket_exact(abs_diff_i64(p.timestamps[si.start + ii], p.timestamps[si.start + jj]),
                                             thr);
                }
                xs[u] = att[u] ? __uint_as_float(sr[e + u]) + (pos_b[pbk[u]] + time_b[tbk[u]]) : kMaskedBias;
              }
              float ds0, ds1;
              p_ds2(xs[0], xs[1], __uint_as_float(dr[e]), __uint_as_float(dr[e + 1]), inv_n, pk[e >> 1], ds0, ds1);
              dk[e >> 1] = pack_bf16x2(ds0, ds1);
              const float dsv[2] = {ds0, ds1};
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                if (att[u]) {
                  if (pbk[u] == kNumBuckets - 1) far_pos += dsv[u];
                  else red_add(&gpos[pbk[u]], dsv[u]);
                  red_add(&gtime[tbk[u]], dsv[u]);
                }
              }
            }
            tmem_st_32x32b_x4(tmem + kColP + lane_off + 16 * seg + 4 * c8, pk);
            st_shared_v4(ds_atom + (((ds_ch + c8) ^ (jl & 7)) << 4), dk[0], dk[1], dk[2], dk[3]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sp_free);
        }
        if (kind == 1) {
          // lanes are kv rows of the sequence here (j < i < n)
          red_add(&gtime[tlo], a0);
          if (lrank > 1) red_add(&gtime[tlo + 1], a1);
          if (lrank > 2) red_add(&gtime[tlo + 2], a2);
          if (lrank > 3) red_add(&gtime[tlo + 3], a3);
          far_pos += (a0 + a1) + (a2 + a3);
        } else if (kind == 2) {
          if (at != 0.f) red_add(&gtime[cur_tb], at);
          // lane l >= 1 holds the diagonal 32 - l: position bucket D + 32 - l; the diagonal
          // completed at column l (position bucket D + l - 31; below 0 only for D = 0,
          // where its pairs are masked) waits in shared memory
          if (lane > 0 && dg != 0.f) red_add(&gpos[min(D + 32 - lane, kNumBuckets - 1)], dg);
          __syncwarp();
          const float dl = diag_w[lane];
          if ((D > 0 || lane == 31) && dl != 0.f) red_add(&gpos[min(D + lane - 31, kNumBuckets - 1)], dl);
          __syncwarp();   // read before the next band segment writes
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->p_ready);
          mbar_arrive(&bars->q_empty[qs]);
        }
        // this tile's dQ is read out at the start of the next tile (its MMA runs meanwhile)
        const int iq = qt * BT + jl;   // this lane's q row of the dQ tile
        pend_rows->x = iq < si.n ? (si.start + iq) * p.num_heads + h : -1;
        pend_dq = true;
        ++g;
      }
      // this item's dK and dV are read out during the next item's first tile
      if (jlive) {
        pend_rows->y = (si.start + j) * p.num_heads + h;
      } else {
        pend_rows->y = -1;
      }
      pend_acc = true;
      acc_par = k & 1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->kv_empty[ks]);   // done with the kv tile's record
    }
    // the last readouts
    if (pend_dq) {
      if (!mbar_wait(&bars->dq_full, (g - 1) & 1, tmo, abort_flag)) goto fail;
      tc_fence_after();
      uint32_t qr[16];
      tmem_ld_32x32b_x16(tmem + kColDQ + lane_off + 16 * seg, qr);
      tmem_ld_wait();
      const int dq_r = pend_rows->x;
      if (dq_r >= 0) {
        float* dq_dst = p.dq_accum + (int64_t)dq_r * DHB + 16 * seg;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          red_add_v4(dq_dst + 4 * c, __uint_as_float(qr[4 * c]), __uint_as_float(qr[4 * c + 1]),
                     __uint_as_float(qr[4 * c + 2]), __uint_as_float(qr[4 * c + 3]));
      }
    }
    if (pend_acc) {
      if (!mbar_wait(&bars->acc_full, acc_par, tmo, abort_flag)) goto fail;
      tc_fence_after();
      uint32_t vr[16], kr[16];
      tmem_ld_32x32b_x16(tmem + kColDV + lane_off + 16 * seg, vr);
      tmem_ld_32x32b_x16(tmem + kColDK + lane_off + 16 * seg, kr);
      tmem_ld_wait();
      const int kv_r = pend_rows->y;
      if (kv_r >= 0) {
        const int64_t tok = kv_r / p.num_heads, hh = kv_r % p.num_heads;
        store_bf16_row16(reinterpret_cast<__nv_bfloat16*>(p.dv) + tok * p.lddv + hh * DHB + 16 * seg, vr);
        store_bf16_row16(reinterpret_cast<__nv_bfloat16*>(p.dk) + tok * p.lddk + hh * DHB + 16 * seg, kr);
      }
    }
    flush_far();
  }
  goto teardown;
fail:
  set_status(p.status, HSTU_ERR_TIMEOUT);
  *abort_flag = 1;
  if (warp == 0 && lane == 0) {
    // let every copy this CTA may have issued land before it exits (bounded)
    for (int s = 0; s < kStages; ++s) {
      mbar_wait(&bars->kv_full[s], 0, 100000000ll, nullptr);
      mbar_wait(&bars->kv_full[s], 1, 100000000ll, nullptr);
      mbar_wait(&bars->q_full[s], 0, 100000000ll, nullptr);
      mbar_wait(&bars->q_full[s], 1, 100000000ll, nullptr);
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

// ---------------------------------------------------------------------------
// The near-diagonal band: one block per group of 32 kv rows (four per 128-row
// tile of tile_base), one thread per band column c (q row i = floor32(j) + c).
// Buckets follow the attention's rule: the 32-bit estimate with an exact compare
// near a boundary, the 64-bit threshold search where offsets leave +-2^30.
__device__ __noinline__ int band_bucket_wide64(int64_t ti, int64_t tj, const int64_t* thr) {
  return time_bucket_exact(abs_diff_i64(ti, tj), thr);
}

__global__ void __launch_bounds__(kBwdBandCols) bwd_band_kernel(const int32_t* __restrict__ offs,
                                                                const int32_t* __restrict__ num_targets,
                                                                const int64_t* __restrict__ ts, int B,
                                                                const int32_t* __restrict__ tile_base,
                                                                const float* __restrict__ pos_bias,
                                                                const float* __restrict__ time_bias,
                                                                const Thresholds thr_in, float ln2_over_div, int T,
                                                                const int32_t* __restrict__ status,
                                                                uint32_t* __restrict__ band) {
  __shared__ int64_t thr[kNumBuckets];
  __shared__ int32_t thr32[kNumBuckets + 4];
  __shared__ float pb_s[kNumBuckets], tb_s[kNumBuckets];
  __shared__ int32_t rel_s[32];
  __shared__ int64_t abs_s[32];
  __shared__ __align__(16) uint32_t out_s[32][kBwdBandCols];
  if (*status != 0) return;  // the scheduler found the offsets invalid
  const int grp = blockIdx.x;
  if (grp >= 4 * tile_base[B]) return;
  const int t = grp >> 2;
  int lo = 0, hi = B;  // sequence s with tile_base[s] <= t < tile_base[s + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_base[mid] <= t) lo = mid; else hi = mid;
  }
  const SeqInfo si = load_seq(offs, num_targets, lo);
  const int j0 = (t - tile_base[lo]) * 128 + 32 * (grp & 3);
  if (j0 >= si.n || si.start + si.n > T) return;
  const int c = threadIdx.x;
  for (int b = c; b < kNumBuckets + 4; b += kBwdBandCols) {
    if (b < kNumBuckets) {
      thr[b] = thr_in.v[b];
      thr32[b] = thr_in.v[b] > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)thr_in.v[b];
      pb_s[b] = pos_bias[b];
      tb_s[b] = time_bias[b];
    } else {
      thr32[b] = 0x7FFFFFFF;
    }
  }
  const int64_t t_first = ts[si.start];
  const int64_t lim = (1ll << 30) - 1;
  if (c < 32) {
    const int jj = j0 + c < si.n ? j0 + c : si.n - 1;
    const int64_t tj = ts[si.start + jj];
    const int64_t rel = tj - t_first;
    rel_s[c] = (int32_t)(rel < -lim ? -lim : (rel > lim ? lim : rel));
    abs_s[c] = tj;
  }
  const int i = j0 + c;
  const int64_t ti = i < si.n ? ts[si.start + i] : t_first;
  const int64_t reli = ti - t_first;
  const bool wide_i = reli < -lim || reli > lim;
  __syncthreads();
  bool wide = wide_i;
  for (int r = 0; r < 32; ++r) wide = wide || (abs_s[r] - t_first < -lim || abs_s[r] - t_first > lim);
  wide = __syncthreads_or(wide) != 0;
  const int32_t relc = (int32_t)(reli < -lim ? -lim : (reli > lim ? lim : reli));
  const int posi = token_pos(i, si.hist);
  const uint32_t masked = ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(kMaskedBias))) << 16;
  const int rows = si.n - j0 < 32 ? si.n - j0 : 32;
  for (int r = 0; r < rows; ++r) {
    const int j = j0 + r;
    uint32_t word = masked;
    if (i < si.n && attended(i, j, si.n, si.hist)) {
      const int pb = pos_bucket(posi, token_pos(j, si.hist));
      const int tb = wide ? band_bucket_wide64(ti, abs_s[r], thr)
                          : fast_bucket(abs(relc - rel_s[r]), thr32, ln2_over_div);
      const float bias = pb_s[pb] + tb_s[tb];
      word = ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(bias)) << 16) | (uint32_t)tb;
    }
    out_s[r][c] = word;
  }
  __syncthreads();
  for (int e = c; e < rows * (kBwdBandCols / 4); e += kBwdBandCols) {
    const int r = e / (kBwdBandCols / 4), q = e - r * (kBwdBandCols / 4);
    reinterpret_cast<uint4*>(band + (int64_t)(si.start + j0 + r) * kBwdBandCols)[q] =
        *reinterpret_cast<const uint4*>(&out_s[r][4 * q]);
  }
}

// The CTAs' partial relative-bias gradients added into the caller's tables:
// entry e of table t (t = 2 head + {0: position, 1: time}) over all CTAs, the
// CTAs split over blockIdx.y (each slice's sum added atomically)
__global__ void rab_reduce_kernel(const float* __restrict__ part, int ctas, int tables, int head_stride,
                                  float* __restrict__ d_pos, float* __restrict__ d_time) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // over tables * 2 * 128
  const int n = tables * 2 * kNumBuckets;
  if (e >= n) return;
  const int c0 = (int)((int64_t)ctas * blockIdx.y / gridDim.y), c1 = (int)((int64_t)ctas * (blockIdx.y + 1) / gridDim.y);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  int c = c0;
  for (; c + 3 < c1; c += 4) {
    s0 += part[(size_t)c * n + e];
    s1 += part[(size_t)(c + 1) * n + e];
    s2 += part[(size_t)(c + 2) * n + e];
    s3 += part[(size_t)(c + 3) * n + e];
  }
  for (; c < c1; ++c) s0 += part[(size_t)c * n + e];
  if (c1 <= c0) return;
  const int h = e / (2 * kNumBuckets), k = (e / kNumBuckets) & 1, b = e % kNumBuckets;
  float* dst = (k == 0 ? d_pos : d_time) + h * head_stride + b;
  atomicAdd(dst, (s0 + s1) + (s2 + s3));
}

// ---------------------------------------------------------------------------
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

// bf16 [rows, cols] with row stride ld elements; box 64 columns x 128 rows, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_attn_bwd_supported(int dtype, int dh) { return dtype == HSTU_DTYPE_BF16 && dh == DHB; }
int tc_bwd_tile() { return BT; }

size_t bwd_band_bytes(int T) { return (size_t)(T > 0 ? T : 0) * kBwdBandCols * 4; }

cudaError_t launch_bwd_band(const int32_t* offs, const int32_t* num_targets, const int64_t* ts, int B, int T,
                            const int32_t* tile_base, int tiles_cap, const float* pos_bias, const float* time_bias,
                            const Thresholds& thr, double time_div, const int32_t* status, uint32_t* band,
                            cudaStream_t st) {
  if (T <= 0 || B <= 0 || tiles_cap <= 0) return cudaSuccess;
  bwd_band_kernel<<<4 * tiles_cap, kBwdBandCols, 0, st>>>(offs, num_targets, ts, B, tile_base, pos_bias, time_bias,
                                                          thr, (float)(0.69314718055994530942 / time_div), T, status,
                                                          band);
  return cudaGetLastError();
}

cudaError_t launch_rab_reduce(const float* part, int ctas, int tables, int head_stride, float* d_pos, float* d_time,
                              cudaStream_t st) {
  const int n = tables * 2 * kNumBuckets;
  const int slices = ctas >= 64 ? 16 : (ctas >= 4 ? ctas / 4 : 1);   // about 4 .. 16 CTAs per thread
  rab_reduce_kernel<<<dim3((n + 255) / 256, slices), 256, 0, st>>>(part, ctas, tables, head_stride, d_pos, d_time);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(const AttnBwdParams& p, int grid, cudaStream_t st, double time_div) {
  BwdTcParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.p = p;
  tp.ln2_over_div = (float)(0.69314718055994530942 / time_div);
  if ((int64_t)p.total_rows * p.num_heads >= 0x7FFFFFFF) return cudaErrorInvalidValue;   // int32 row * head indices
  const int64_t hd = (int64_t)p.num_heads * DHB;
  if (!make_map(&tp.map_q, p.q, hd, p.total_rows, p.ldq) || !make_map(&tp.map_k, p.k, hd, p.total_rows, p.ldk) ||
      !make_map(&tp.map_v, p.v, hd, p.total_rows, p.ldv) ||
      !make_map(&tp.map_do, p.dout, hd, p.total_rows, p.lddo))
    return cudaErrorInvalidValue;
  const int smem = BwdLayout::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_bwd_tc_kernel<<<grid, kThreads, smem, st>>>(tp);
  return cudaGetLastError();
}

}  // namespace hstu
