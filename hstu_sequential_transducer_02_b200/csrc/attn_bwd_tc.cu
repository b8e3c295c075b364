// Pointwise aggregated attention backward on the sm_100a tensor cores (bf16,
// head dim 64).
//
// Forward: O_i = (1/N) sum_{j in mask(i)} SiLU(s_ij) v_j, s_ij = q_i . k_j + rab_ij.
// With P_ij = SiLU(s_ij)/N and dS_ij = (dO_i . v_j) SiLU'(s_ij)/N on attended pairs:
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K,  d rab[bucket] = sum of dS over the bucket.
// ("Actions Speak Louder than Words" summary, 1.2 and 2.2: the attention is
// trained end to end; the relative bias tables receive gradients.)
//
// One persistent CTA per SM walks kv-tile work items (sequence, head, 128 kv
// rows), longest first.  For every q tile of 128 rows that attends to the kv
// tile:
//   warp 0      TMA: K and V once per item, Q and dO per q tile (two stages)
//   warp 1      one thread issues tcgen05.mma:
//                 S^T  = K Q^T        -> TMEM columns [0, 128)
//                 dP^T = V dO^T       -> TMEM columns [128, 256)
//                 dV  += P^T dO       (P^T from TMEM)       -> [256, 320)
//                 dK  += dS^T Q       (dS^T from shared memory) -> [320, 384)
//                 dQ   = dS K         (the same tile, read as its transpose) -> [384, 448)
//   warps 2-17  epilogue, one warp per TMEM lane quarter (32 kv rows) and 32 q
//               columns: bias, SiLU, SiLU', mask; P^T (bf16) back into TMEM,
//               dS^T (bf16) into shared memory; relative-bias gradients summed
//               along runs of equal bucket into per-CTA histograms; dQ of the
//               tile added to an fp32 accumulator with vector atomics; at the
//               end of the item dK and dV -> bf16 -> global memory.
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
constexpr int kQStages = 2;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 320, kColDQ = 384, kTmemCols = 512;

struct BwdBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t sp_full, p_ready, dq_full, dq_empty, acc_full, acc_empty;
  uint64_t done;
};

struct BwdLayout {
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;                  // per stage: Q tile, then dO tile
  static constexpr int kDS = kQ + kQStages * 2 * kTile;  // dS^T [128 kv x 128 q] bf16: two 64-column atoms
  static constexpr int kThr = kDS + 2 * kTile;
  static constexpr int kThr32 = kThr + kNumBuckets * 8;
  static constexpr int kPosB = kThr32 + (kNumBuckets + 4) * 4;
  static constexpr int kTimeB = kPosB + kNumBuckets * 4;
  static constexpr int kGPos = kTimeB + kNumBuckets * 4;
  static constexpr int kGTime = kGPos + kNumBuckets * 4;
  static constexpr int kBar = (kGTime + kNumBuckets * 4 + 15) & ~15;
  static constexpr int kMisc = kBar + (int)sizeof(BwdBars);
  static constexpr int kEnd = kMisc + 16;
  static constexpr int kAlloc = kEnd + 1024;  // slack for 1024-byte alignment of the base
};

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

// SiLU and its derivative from sigma(x) = 1 / (1 + exp(-x)); the relative-bias
// gradients sum dS over up to millions of pairs, so a systematic error in
// SiLU' (as tanh.approx would leave, about 2^-11) must not enter them.
__device__ __forceinline__ void silu_and_grad(float x, float& f, float& g) {
  const float sg = __fdividef(1.0f, 1.0f + __expf(-x));
  f = x * sg;
  g = sg * fmaf(x, 1.0f - sg, 1.0f);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) attn_bwd_tc_kernel(const __grid_constant__ BwdTcParams prm) {
  using L = BwdLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int64_t* thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int32_t* thr32 = reinterpret_cast<int32_t*>(smem + L::kThr32);
  float* pos_b = reinterpret_cast<float*>(smem + L::kPosB);
  float* time_b = reinterpret_cast<float*>(smem + L::kTimeB);
  float* gpos = reinterpret_cast<float*>(smem + L::kGPos);
  float* gtime = reinterpret_cast<float*>(smem + L::kGTime);
  const uint32_t sK = smem_u32(smem + L::kK);
  const uint32_t sV = smem_u32(smem + L::kV);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sDS = smem_u32(smem + L::kDS);

  const AttnBwdParams& p = prm.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tmo = p.timeout_ns;
  const int count = *p.item_count;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < kQStages; ++s) { mbar_init(&bars->q_full[s], 1); mbar_init(&bars->q_empty[s], 1); }
    mbar_init(&bars->sp_full, 1);
    mbar_init(&bars->p_ready, kEpiWarps);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, kEpiWarps);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kEpiWarps);
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
  for (int c = threadIdx.x; c < kNumBuckets + 4; c += kThreads) {
    if (c < kNumBuckets) {
      thr[c] = p.thr.v[c];
      thr32[c] = p.thr.v[c] > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)p.thr.v[c];
      gpos[c] = 0.f;
      gtime[c] = 0.f;
    } else {
      thr32[c] = 0x7FFFFFFF;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================================ loads
    if (lane == 0) {
      int qi = 0, k = 0;
      for (int idx = blockIdx.x; idx < count; idx += gridDim.x, ++k) {
        const WorkItem wi = p.items[idx];
        const SeqInfo si = load_seq(p.seq_offsets, p.num_targets, wi.seq);
        const int kt = wi.qtile;  // backward items carry the kv tile
        if (!mbar_wait(&bars->kv_empty, (k & 1) ^ 1, tmo, abort_flag)) goto fail;
        mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile);
        tma_load_2d(smem + L::kK, &prm.map_k, &bars->kv_full, wi.head * DHB, si.start + kt * BT);
        tma_load_2d(smem + L::kV, &prm.map_v, &bars->kv_full, wi.head * DHB, si.start + kt * BT);
        const int nq = (si.n + BT - 1) / BT;
        for (int qt = kt; qt < nq; ++qt) {
          if (!q_tile_hits(si, qt, kt)) continue;
          const int st = qi % kQStages;
          if (!mbar_wait(&bars->q_empty[st], ((qi / kQStages) & 1) ^ 1, tmo, abort_flag)) goto fail;
          mbar_arrive_expect_tx(&bars->q_full[st], 2 * kTile);
          tma_load_2d(smem + L::kQ + st * 2 * kTile, &prm.map_q, &bars->q_full[st], wi.head * DHB, si.start + qt * BT);
          tma_load_2d(smem + L::kQ + st * 2 * kTile + kTile, &prm.map_do, &bars->q_full[st], wi.head * DHB,
                      si.start + qt * BT);
          ++qi;
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = make_idesc_bf16(BT, BT, false, false);      // S^T, dP^T
      constexpr uint32_t id_kv = make_idesc_bf16(BT, DHB, false, true);     // dV, dK: B MN-major
      constexpr uint32_t id_q = make_idesc_bf16(BT, DHB, true, true);       // dQ: A and B MN-major
      const uint64_t dK_kmaj = make_sw128_desc(sK, 16, 1024);
      const uint64_t dV_kmaj = make_sw128_desc(sV, 16, 1024);
      const uint64_t dK_mn = make_sw128_desc(sK, 16384, 1024);
      const uint64_t dDS_kmaj = make_sw128_desc(sDS, 16, 1024);
      const uint64_t dDS_mn = make_sw128_desc(sDS, 16384, 1024);
      int qi = 0, k = 0;
      for (int idx = blockIdx.x; idx < count; idx += gridDim.x, ++k) {
        const WorkItem wi = p.items[idx];
        const SeqInfo si = load_seq(p.seq_offsets, p.num_targets, wi.seq);
        const int kt = wi.qtile;
        if (!mbar_wait(&bars->kv_full, k & 1, tmo, abort_flag)) goto fail;
        if (!mbar_wait(&bars->acc_empty, (k & 1) ^ 1, tmo, abort_flag)) goto fail;
        bool first = true;
        const int nq = (si.n + BT - 1) / BT;
        for (int qt = kt; qt < nq; ++qt) {
          if (!q_tile_hits(si, qt, kt)) continue;
          const int st = qi % kQStages;
          if (!mbar_wait(&bars->q_full[st], (qi / kQStages) & 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
          const uint32_t sq = sQ + st * 2 * kTile, sdo = sq + kTile;
          const uint64_t dq_kmaj = make_sw128_desc(sq, 16, 1024), ddo_kmaj = make_sw128_desc(sdo, 16, 1024);
          const uint64_t dq_mn = make_sw128_desc(sq, 16384, 1024), ddo_mn = make_sw128_desc(sdo, 16384, 1024);
          // S^T = K Q^T and dP^T = V dO^T (reduction over the head dimension)
#pragma unroll
          for (int ks = 0; ks < DHB / 16; ++ks) {
            umma_f16_ss(tmem + kColS, desc_advance(dK_kmaj, ks * 32), desc_advance(dq_kmaj, ks * 32), id_s,
                        ks > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < DHB / 16; ++ks) {
            umma_f16_ss(tmem + kColDP, desc_advance(dV_kmaj, ks * 32), desc_advance(ddo_kmaj, ks * 32), id_s,
                        ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars->sp_full);
          if (!mbar_wait(&bars->p_ready, qi & 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
          // dV += P^T dO, dK += dS^T Q (reduction over the q tile's 128 rows)
#pragma unroll
          for (int ks = 0; ks < BT / 16; ++ks) {
            umma_f16_ts(tmem + kColDV, tmem + kColS + 32 * (ks >> 1) + 8 * (ks & 1), desc_advance(ddo_mn, ks * 2048),
                        id_kv, (!first || ks > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < BT / 16; ++ks) {
            umma_f16_ss(tmem + kColDK, desc_advance(dDS_kmaj, (ks >> 2) * 16384 + (ks & 3) * 32),
                        desc_advance(dq_mn, ks * 2048), id_kv, (!first || ks > 0) ? 1u : 0u);
          }
          // dQ = dS K (reduction over the kv tile's 128 rows), once the previous dQ was read
          if (!mbar_wait(&bars->dq_empty, (qi & 1) ^ 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BT / 16; ++ks) {
            umma_f16_ss(tmem + kColDQ, desc_advance(dDS_mn, ks * 2048), desc_advance(dK_mn, ks * 2048), id_q,
                        ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars->dq_full);
          umma_commit(&bars->q_empty[st]);
          first = false;
          ++qi;
        }
        umma_commit(&bars->acc_full);
        umma_commit(&bars->kv_empty);
      }
      umma_commit(&bars->done);
      mbar_wait(&bars->done, 0, tmo, nullptr);
    }
  } else {
    // ================================================================ epilogue
    const int ew = warp - kEpiWarp0;       // 0..15
    const int quarter = warp & 3;          // TMEM lane quarter: kv rows 32 quarter ..
    const int seg = ew >> 2;               // q columns [32 seg, 32 seg + 32) of the q tile
    const int jl = quarter * 32 + lane;    // kv row inside the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float k_lg = prm.ln2_over_div;
    const int etid = threadIdx.x - 32 * kEpiWarp0;
    int qi = 0, k = 0;
    for (int idx = blockIdx.x; idx < count; idx += gridDim.x, ++k) {
      const WorkItem wi = p.items[idx];
      const SeqInfo si = load_seq(p.seq_offsets, p.num_targets, wi.seq);
      const int kt = wi.qtile, h = wi.head;
      // relative-bias tables of this head
      named_bar_sync(1, 32 * kEpiWarps);
      for (int c = etid; c < kNumBuckets; c += 32 * kEpiWarps) {
        pos_b[c] = p.pos_bias[h * p.rab_head_stride + c];
        time_b[c] = p.time_bias[h * p.rab_head_stride + c];
      }
      named_bar_sync(1, 32 * kEpiWarps);
      const int j = kt * BT + jl;
      const int j0w = kt * BT + quarter * 32;   // first kv row of the warp
      const bool jlive = j < si.n;
      const int64_t t_first = p.timestamps[si.start];
      const int64_t tj = p.timestamps[si.start + (jlive ? j : 0)];
      const int64_t rj64 = tj - t_first;
      const bool rj_narrow = __all_sync(0xffffffffu, rj64 > -(1ll << 30) && rj64 < (1ll << 30));
      const int32_t rj = (int32_t)rj64;
      const int posj = token_pos(j, si.hist);
      float far_pos = 0.f;                       // dS of far segments (position bucket 127)
      const int nq = (si.n + BT - 1) / BT;
      int nhit = 0;
      for (int qt = kt; qt < nq; ++qt) {
        if (!q_tile_hits(si, qt, kt)) continue;
        ++nhit;
        // timestamp of q column 32 seg + lane of this tile (shared through shuffles),
        // as an offset from the sequence's first timestamp
        const int i0 = qt * BT + 32 * seg;    // first q row of this segment
        const int icol = i0 + lane;
        const int64_t relc64 = p.timestamps[si.start + (icol < si.n ? icol : si.n - 1)] - t_first;
        const bool wnarrow = __all_sync(0xffffffffu, relc64 > -(1ll << 30) && relc64 < (1ll << 30)) && rj_narrow;
        const int32_t relc = (int32_t)relc64;
        // far segment: history rows at least 127 positions past every kv row of the
        // warp, so the position bucket is the last one; with one time bucket per
        // lane the bias is constant and dS is summed in registers
        // (`two`: the same with at most two time buckets per lane, told apart by one
        // threshold compare per element, each summed in registers)
        bool fast = false, two = false;
        int tlo = 0;
        float hb = 0.f, hb1 = 0.f;
        int32_t th1 = 0x7FFFFFFF;
        if (wnarrow && i0 + 31 < si.hist && i0 - (j0w + 31) >= kNumBuckets - 1) {
          const int32_t mn = __reduce_min_sync(0xffffffffu, relc), mx = __reduce_max_sync(0xffffffffu, relc);
          int32_t dlo, dhi;
          if (rj >= mx) { dlo = rj - mx; dhi = rj - mn; }
          else if (rj <= mn) { dlo = mn - rj; dhi = mx - rj; }
          else { dlo = 0; dhi = max(rj - mn, mx - rj); }
          tlo = fast_bucket(dlo, thr32, k_lg);
          th1 = thr32[tlo + 1];
          fast = __all_sync(0xffffffffu, dhi < th1);
          two = !fast && __all_sync(0xffffffffu, dhi < thr32[tlo + 2]);   // tlo < 127 here
          hb = pos_b[kNumBuckets - 1] + time_b[tlo];
          if (two) hb1 = pos_b[kNumBuckets - 1] + time_b[tlo + 1];
        }
        if (!mbar_wait(&bars->sp_full, qi & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        int cur_tb = -1;
        float acc_t = 0.f, acc_fast = 0.f, acc_two = 0.f;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          const int cb = 32 * seg + 16 * hh;   // first q column of this half inside the tile
          uint32_t sr[16], dr[16];
          tmem_ld_32x32b_x16(tmem + kColS + lane_off + cb, sr);
          tmem_ld_32x32b_x16(tmem + kColDP + lane_off + cb, dr);
          tmem_ld_wait();
          float pv[16], dsv[16];
          if (fast) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float f, g;
              silu_and_grad(__uint_as_float(sr[e]) + hb, f, g);
              pv[e] = jlive ? f * si.inv_n : 0.f;
              dsv[e] = jlive ? __uint_as_float(dr[e]) * g * si.inv_n : 0.f;
              acc_fast += dsv[e];
            }
          } else if (two) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int32_t dd = abs(__shfl_sync(0xffffffffu, relc, 16 * hh + e) - rj);
              const bool up = dd >= th1;   // bucket tlo + 1, else tlo
              float f, g;
              silu_and_grad(__uint_as_float(sr[e]) + (up ? hb1 : hb), f, g);
              pv[e] = jlive ? f * si.inv_n : 0.f;
              dsv[e] = jlive ? __uint_as_float(dr[e]) * g * si.inv_n : 0.f;
              acc_fast += up ? 0.f : dsv[e];
              acc_two += up ? dsv[e] : 0.f;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int i = qt * BT + cb + e;
              const bool att = jlive && attended(i, j, si.n, si.hist);
              int tb;
              if (wnarrow) {
                tb = fast_bucket(abs(__shfl_sync(0xffffffffu, relc, 16 * hh + e) - rj), thr32, k_lg);
              } else {
                const int64_t ti = __shfl_sync(0xffffffffu, (long long)relc64, 16 * hh + e) + t_first;
                tb = time_bucket_exact(abs_diff_i64(ti, tj), thr);
              }
              const int pb = pos_bucket(token_pos(i, si.hist), posj);
              float f, g;
              silu_and_grad(__uint_as_float(sr[e]) + (pos_b[pb] + time_b[tb]), f, g);
              pv[e] = att ? f * si.inv_n : 0.f;
              dsv[e] = att ? __uint_as_float(dr[e]) * g * si.inv_n : 0.f;
              // relative-bias gradients: position buckets differ across the lanes of an
              // element near the diagonal; time buckets are summed along runs
              if (att) {
                if (pb == kNumBuckets - 1) far_pos += dsv[e];   // shared by all far lanes: summed in registers
                else atomicAdd(&gpos[pb], dsv[e]);
              }
              if (tb != cur_tb) {
                if (acc_t != 0.f) atomicAdd(&gtime[cur_tb], acc_t);
                cur_tb = tb;
                acc_t = 0.f;
              }
              acc_t += dsv[e];
            }
          }
          // P^T (bf16 pairs) over this half's consumed S^T columns (the A operand of dV)
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
          tmem_st_32x32b_x8(tmem + kColS + lane_off + 32 * seg + 8 * hh, pk);
          // dS^T row jl, q columns cb .. cb + 15: two 16-byte chunks of the 128-byte swizzled row
          uint32_t dk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) dk[e] = pack_bf16x2(dsv[2 * e], dsv[2 * e + 1]);
          const uint32_t atom = sDS + (cb >> 6) * kTile + jl * 128;
          const int ch = (cb & 63) >> 3;
          st_shared_v4(atom + (((ch) ^ (jl & 7)) << 4), dk[0], dk[1], dk[2], dk[3]);
          st_shared_v4(atom + (((ch + 1) ^ (jl & 7)) << 4), dk[4], dk[5], dk[6], dk[7]);
        }
        if (fast) {
          if (jlive) atomicAdd(&gtime[tlo], acc_fast);
          far_pos += acc_fast;   // position bucket 127, added once per item
        } else if (two) {
          if (jlive) {
            if (acc_fast != 0.f) atomicAdd(&gtime[tlo], acc_fast);
            if (acc_two != 0.f) atomicAdd(&gtime[tlo + 1], acc_two);
          }
          far_pos += acc_fast + acc_two;
        } else if (acc_t != 0.f) {
          atomicAdd(&gtime[cur_tb], acc_t);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready);
        // dQ of this q tile: q rows 32 quarter + lane, head columns [16 seg, 16 seg + 16)
        if (!mbar_wait(&bars->dq_full, qi & 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        uint32_t qr[16];
        tmem_ld_32x32b_x16(tmem + kColDQ + lane_off + 16 * seg, qr);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->dq_empty);
        const int iq = qt * BT + jl;   // this lane's q row
        if (iq < si.n) {
          float* dst = p.dq_accum + ((int64_t)(si.start + iq) * p.num_heads + h) * DHB + 16 * seg;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            red_add_v4(dst + 4 * c, __uint_as_float(qr[4 * c]), __uint_as_float(qr[4 * c + 1]),
                       __uint_as_float(qr[4 * c + 2]), __uint_as_float(qr[4 * c + 3]));
        }
        ++qi;
      }
      // dK and dV of this kv tile: kv row jl, head columns [16 seg, 16 seg + 16)
      if (!mbar_wait(&bars->acc_full, k & 1, tmo, abort_flag)) goto fail;
      tc_fence_after();
      uint32_t vr[16], kr[16];
      tmem_ld_32x32b_x16(tmem + kColDV + lane_off + 16 * seg, vr);
      tmem_ld_32x32b_x16(tmem + kColDK + lane_off + 16 * seg, kr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);
      if (jlive) {
        __nv_bfloat16* dvp = reinterpret_cast<__nv_bfloat16*>(p.dv) + (int64_t)(si.start + j) * p.lddv + h * DHB + 16 * seg;
        __nv_bfloat16* dkp = reinterpret_cast<__nv_bfloat16*>(p.dk) + (int64_t)(si.start + j) * p.lddk + h * DHB + 16 * seg;
        uint4 w[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t* src = &vr[8 * hf];
          w[hf] = make_uint4(pack_bf16x2(nhit ? __uint_as_float(src[0]) : 0.f, nhit ? __uint_as_float(src[1]) : 0.f),
                             pack_bf16x2(nhit ? __uint_as_float(src[2]) : 0.f, nhit ? __uint_as_float(src[3]) : 0.f),
                             pack_bf16x2(nhit ? __uint_as_float(src[4]) : 0.f, nhit ? __uint_as_float(src[5]) : 0.f),
                             pack_bf16x2(nhit ? __uint_as_float(src[6]) : 0.f, nhit ? __uint_as_float(src[7]) : 0.f));
        }
        *reinterpret_cast<uint4*>(dvp) = w[0];
        *reinterpret_cast<uint4*>(dvp + 8) = w[1];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t* src = &kr[8 * hf];
          w[hf] = make_uint4(pack_bf16x2(nhit ? __uint_as_float(src[0]) : 0.f, nhit ? __uint_as_float(src[1]) : 0.f),
                             pack_bf16x2(nhit ? __uint_as_float(src[2]) : 0.f, nhit ? __uint_as_float(src[3]) : 0.f),
                             pack_bf16x2(nhit ? __uint_as_float(src[4]) : 0.f, nhit ? __uint_as_float(src[5]) : 0.f),
                             pack_bf16x2(nhit ? __uint_as_float(src[6]) : 0.f, nhit ? __uint_as_float(src[7]) : 0.f));
        }
        *reinterpret_cast<uint4*>(dkp) = w[0];
        *reinterpret_cast<uint4*>(dkp + 8) = w[1];
      }
      // flush this item's relative-bias gradients (this head's tables)
      {
        float fp = far_pos;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) fp += __shfl_xor_sync(0xffffffffu, fp, o);
        if (lane == 0 && fp != 0.f) atomicAdd(&gpos[kNumBuckets - 1], fp);
      }
      named_bar_sync(1, 32 * kEpiWarps);
      for (int c = etid; c < kNumBuckets; c += 32 * kEpiWarps) {
        if (gpos[c] != 0.f) atomicAdd(&p.d_pos_bias[h * p.rab_head_stride + c], gpos[c]);
        if (gtime[c] != 0.f) atomicAdd(&p.d_time_bias[h * p.rab_head_stride + c], gtime[c]);
        gpos[c] = 0.f;
        gtime[c] = 0.f;
      }
    }
  }
  goto teardown;
fail:
  set_status(p.status, HSTU_ERR_TIMEOUT);
  *abort_flag = 1;
  if (warp == 0 && lane == 0) {
    // let every copy this CTA may have issued land before it exits (bounded)
    mbar_wait(&bars->kv_full, 0, 100000000ll, nullptr);
    mbar_wait(&bars->kv_full, 1, 100000000ll, nullptr);
    for (int s = 0; s < kQStages; ++s) {
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

cudaError_t launch_attn_bwd_tc(const AttnBwdParams& p, int grid, cudaStream_t st, double time_div) {
  BwdTcParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.p = p;
  tp.ln2_over_div = (float)(0.69314718055994530942 / time_div);
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
