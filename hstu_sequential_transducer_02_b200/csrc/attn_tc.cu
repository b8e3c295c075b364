// Pointwise aggregated attention forward on the sm_100a tensor cores.
//
//   O_i = (1/N) * sum_{j in mask(i)} SiLU(q_i . k_j + rab_ij) v_j
//
// ("Actions Speak Louder than Words" summary, 1.2; "生成式推荐（一）：HSTU",
// pointwise aggregated attention: no normalisation over the sequence.)
//
// One persistent CTA per SM takes (sequence, head, q tile) work items from a
// shared cursor over a list in locality order (long sequences first, then head,
// then q tile), so the CTAs running at the same time share K/V tiles in L2.
// Per q tile of 128 rows and each kv tile of 128 columns that holds an attended
// pair:
//   warp 0        TMA: Q once per item, K per kv tile into a ring of stages, and
//                 the kv tile's timestamp record (int32 offsets, per-segment
//                 min/max); it also fetches the work items for everyone
//   warp 2        TMA: V per kv tile into its own ring
//   warp 1        issues S = Q K^T (tcgen05.mma, operands in shared memory)
//                 into one of three TMEM buffers
//   warp 3        issues O += P V with P read from TMEM (the A operand) and V
//                 from shared memory (each issuer warp runs its loop
//                 warp-uniformly; one elected lane issues)
//   warps 4-19    epilogue, one warp per TMEM lane quarter and 32-column
//                 segment: S -> registers, rab bias (position and time buckets,
//                 bit-exact integer rule), SiLU, mask, bf16 P written back over
//                 the S columns; at the end of the item O * (1/N) -> bf16 ->
//                 global memory
// No softmax means no running max and no rescaling: O accumulates in TMEM
// across all kv tiles.  Fully masked kv tiles are never visited.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
namespace {
using namespace sm100;

constexpr int BM = 128;                    // q rows per tile (UMMA M)
constexpr int BN = 128;                    // kv columns per tile
constexpr int kEpiWarps = 16;              // four warps per TMEM lane quarter, one per 32-column segment
constexpr int kEpiWarp0 = 4;               // warps 0: Q/K loads, 1: S MMAs, 2: V loads, 3: P V MMAs, 4..19: epilogue
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kBoxBytes = 128 * 128;       // one TMA box: 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 512;
constexpr int kRecBytes = kTsRecWords * 4;

template <int DH>
struct Cfg {
  static constexpr int kKStages = DH == 128 ? 2 : 4;
  static constexpr int kVStages = DH == 128 ? 3 : 4;
  static constexpr int kBoxes = DH / 64;
  static constexpr int kTileBytes = BM * DH * 2;
};


constexpr int kRecStages = 8;              // timestamp records run up to 8 kv tiles ahead
constexpr int kSBufs = 3;                  // S/P buffers in TMEM: S runs two kv tiles ahead of P V

constexpr int kItemSlots = 4;              // work items fetched ahead by the Q/K producer
constexpr int kItemReaders = 3 + kEpiWarps;  // V producer, two MMA issuers, epilogue warps

struct Barriers {
  uint64_t it_full[kItemSlots], it_empty[kItemSlots];
  uint64_t q_full, q_empty;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t r_full[kRecStages], r_empty[kRecStages];
  uint64_t s_full[3], p_full[3], pv_done[3];
  uint64_t o_full, o_empty;
  uint64_t done, done_pv;
};

struct TcParams {
  CUtensorMap map_q;
  CUtensorMap map_k;
  CUtensorMap map_v;
  AttnFwdParams p;
  float ln2_over_div;   // ln(2) / time_div
};

template <int DH>
struct Layout {
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + Cfg<DH>::kTileBytes;
  static constexpr int kV = kK + Cfg<DH>::kKStages * Cfg<DH>::kTileBytes;
  static constexpr int kTs = kV + Cfg<DH>::kVStages * Cfg<DH>::kTileBytes;
  static constexpr int kThr = kTs + kRecStages * kRecBytes;
  static constexpr int kThr32 = kThr + kNumBuckets * 8;
  static constexpr int kPosB = kThr32 + (kNumBuckets + 4) * 4;
  static constexpr int kTimeB = kPosB + kNumBuckets * 4;
  static constexpr int kBar = (kTimeB + kNumBuckets * 4 + 15) & ~15;
  static constexpr int kMisc = kBar + (int)sizeof(Barriers);
  static constexpr int kItems = kMisc + 16;
  static constexpr int kPend = kItems + kItemSlots * 8 * 4;   // per epilogue thread: pending O readout
  static constexpr int kEnd = kPend + kEpiWarps * 32 * 16;
  static constexpr int kAlloc = kEnd + 1024;  // slack for 1024-byte alignment of the base
};

// A fetched work item and the facts of its sequence, as the item ring holds
// them (8 words per slot) so that no reader reloads them from global memory.
struct ItemInfo {
  int idx;       // -1: no more items
  WorkItem wi;
  SeqInfo si;
};

__device__ __forceinline__ void ring_put(volatile int* ring, int slot, const ItemInfo& x) {
  volatile int* w = ring + 8 * slot;
  w[0] = x.idx;
  w[1] = x.wi.seq;
  w[2] = x.wi.head;
  w[3] = x.wi.qtile;
  w[4] = x.si.start;
  w[5] = x.si.n;
  w[6] = x.si.hist;
  w[7] = __float_as_int(x.si.inv_n);
}

__device__ __forceinline__ ItemInfo ring_get(const volatile int* ring, int slot) {
  const volatile int* w = ring + 8 * slot;
  ItemInfo x;
  x.idx = w[0];
  x.wi.seq = w[1];
  x.wi.head = w[2];
  x.wi.qtile = w[3];
  x.wi.cost = 0;
  x.si.start = w[4];
  x.si.n = w[5];
  x.si.hist = w[6];
  x.si.inv_n = __int_as_float(w[7]);
  return x;
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Exact time bucket of 0 <= d < 2^31 in O(1): an approximate ln(d)/div rounded
// to the nearest integer is at most one bucket off, and one comparison with
// each neighbouring integer threshold corrects it (thr32[b] = min(threshold b,
// INT32_MAX), thr32[128] = INT32_MAX).
// Waits for outstanding tcgen05.ld into `r`; the register operands keep the
// compiler from reading them earlier.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
        "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// A deferred O readout of one epilogue thread: its output row (null for rows
// beyond the sequence) and 1/N.  Kept in shared memory, not in registers.
struct PendingO {
  __nv_bfloat16* out;
  float inv_n;
  int pad;
};

// O of a finished work item, once its last P V is done: this warp's kOc columns of
// its 32 rows -> (1/N) -> bf16 -> global memory.  Returns false on a timeout.
template <int kOc>
__device__ __forceinline__ bool o_readout(Barriers* bars, int parity, uint32_t taddr, const PendingO* pend,
                                          int lane, long long tmo, volatile int* abort_flag) {
  if (!mbar_wait(&bars->o_full, parity, tmo, abort_flag)) return false;
  tc_fence_after();
  __nv_bfloat16* out = pend->out;
  const float inv_n = pend->inv_n;
  // 16 columns at a time (few registers: the caller's tile state stays live)
#pragma unroll 1
  for (int h = 0; h < kOc / 16; ++h) {
    uint32_t oraw[16];
    tmem_ld_32x32b_x16(taddr + 16 * h, oraw);
    tmem_ld_wait();
    if (out != nullptr) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(oraw[8 * c + 0]) * inv_n, __uint_as_float(oraw[8 * c + 1]) * inv_n);
        v.y = pack_bf16x2(__uint_as_float(oraw[8 * c + 2]) * inv_n, __uint_as_float(oraw[8 * c + 3]) * inv_n);
        v.z = pack_bf16x2(__uint_as_float(oraw[8 * c + 4]) * inv_n, __uint_as_float(oraw[8 * c + 5]) * inv_n);
        v.w = pack_bf16x2(__uint_as_float(oraw[8 * c + 6]) * inv_n, __uint_as_float(oraw[8 * c + 7]) * inv_n);
        *reinterpret_cast<uint4*>(out + 16 * h + 8 * c) = v;
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&bars->o_empty);
  return true;
}

// ---------------------------------------------------------------------------
template <int DH>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_tc_kernel(const __grid_constant__ TcParams prm) {
  using C = Cfg<DH>;
  using L = Layout<DH>;
  constexpr int SK = C::kKStages;
  constexpr int SV = C::kVStages;
  constexpr int DV = DH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  Barriers* bars = reinterpret_cast<Barriers*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::kItems);
  int64_t* thr = reinterpret_cast<int64_t*>(smem + L::kThr);
  int32_t* thr32 = reinterpret_cast<int32_t*>(smem + L::kThr32);
  float* pos_b = reinterpret_cast<float*>(smem + L::kPosB);
  float* time_b = reinterpret_cast<float*>(smem + L::kTimeB);
  TsRec* recs = reinterpret_cast<TsRec*>(smem + L::kTs);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  const uint32_t sV = smem_u32(smem + L::kV);

  const AttnFwdParams& p = prm.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tmo = p.timeout_ns;

  // ---- set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < kItemSlots; ++s) { mbar_init(&bars->it_full[s], 1); mbar_init(&bars->it_empty[s], kItemReaders); }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < SK; ++s) { mbar_init(&bars->k_full[s], 1); mbar_init(&bars->k_empty[s], 1); }
    for (int s = 0; s < SV; ++s) { mbar_init(&bars->v_full[s], 1); mbar_init(&bars->v_empty[s], 1); }
    for (int s = 0; s < kRecStages; ++s) { mbar_init(&bars->r_full[s], 1); mbar_init(&bars->r_empty[s], kEpiWarps); }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], kEpiWarps);
      mbar_init(&bars->pv_done[s], 1);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_empty, kEpiWarps);
    mbar_init(&bars->done, 1);
    mbar_init(&bars->done_pv, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&prm.map_q);
    tma_prefetch_desc(&prm.map_k);
    tma_prefetch_desc(&prm.map_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
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
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_s0 = tmem_base;               // S / P buffers at columns 0, 128, 256
  const uint32_t tmem_o = tmem_base + kSBufs * BN;  // O accumulator at column 384

  const int count = *p.item_count;
  const int per_head_rab = p.rab_head_stride != 0;

  if (warp == 0 || warp == 2) {
    // =================================================================== producers (0: Q, K and records, 2: V)
    if (lane == 0) {
      const bool kside = warp == 0;
      int it = 0;
      for (int k = 0;; ++k) {
        // the Q/K producer fetches the next work item; everyone else reads it from the ring
        const int slot = k % kItemSlots;
        ItemInfo x;
        if (kside) {
          if (!mbar_wait(&bars->it_empty[slot], ((k / kItemSlots) & 1) ^ 1, tmo, abort_flag)) goto fail;
          x.idx = *abort_flag ? -1 : atomicAdd(p.item_cursor, 1);
          if (x.idx >= count) x.idx = -1;
          if (x.idx >= 0) {
            x.wi = p.items[x.idx];
            x.si = load_seq(p.seq_offsets, p.num_targets, x.wi.seq);
          }
          ring_put(item_ring, slot, x);
          mbar_arrive(&bars->it_full[slot]);
        } else {
          if (!mbar_wait(&bars->it_full[slot], (k / kItemSlots) & 1, tmo, abort_flag)) goto fail;
          x = ring_get(item_ring, slot);
          mbar_arrive(&bars->it_empty[slot]);
        }
        if (x.idx < 0) break;
        const WorkItem wi = x.wi;
        const SeqInfo si = x.si;
        const int r0 = wi.qtile * BM;
        const int r1 = min(si.n, r0 + BM);
        if (kside) {
          if (!mbar_wait(&bars->q_empty, (k & 1) ^ 1, tmo, abort_flag)) goto fail;
          mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
          for (int b = 0; b < C::kBoxes; ++b)
            tma_load_2d(smem + L::kQ + b * kBoxBytes, &prm.map_q, &bars->q_full, wi.head * DH + 64 * b,
                        si.start + r0);
        }
        const TsRec* grec = reinterpret_cast<const TsRec*>(p.tile_recs) + p.tile_base[wi.seq];
        const KvRange kr = kv_tiles_for(r0, r1, si.hist, BN);
        const int nk = kv_count(kr);
        for (int jj = 0; jj < nk; ++jj, ++it) {
          const int kt = kv_tile_at(kr, jj);
          if (kside) {
            const int rs = it % kRecStages;
            if (!mbar_wait(&bars->r_empty[rs], ((it / kRecStages) & 1) ^ 1, tmo, abort_flag)) goto fail;
            mbar_arrive_expect_tx(&bars->r_full[rs], kRecBytes);
            bulk_load(&recs[rs], grec + kt, kRecBytes, &bars->r_full[rs]);
            const int st = it % SK;
            if (!mbar_wait(&bars->k_empty[st], ((it / SK) & 1) ^ 1, tmo, abort_flag)) goto fail;
            mbar_arrive_expect_tx(&bars->k_full[st], C::kTileBytes);
            for (int b = 0; b < C::kBoxes; ++b)
              tma_load_2d(smem + L::kK + st * C::kTileBytes + b * kBoxBytes, &prm.map_k, &bars->k_full[st],
                          wi.head * DH + 64 * b, si.start + kt * BN);
          } else {
            const int st = it % SV;
            if (!mbar_wait(&bars->v_empty[st], ((it / SV) & 1) ^ 1, tmo, abort_flag)) goto fail;
            mbar_arrive_expect_tx(&bars->v_full[st], C::kTileBytes);
            for (int b = 0; b < C::kBoxes; ++b)
              tma_load_2d(smem + L::kV + st * C::kTileBytes + b * kBoxBytes, &prm.map_v, &bars->v_full[st],
                          wi.head * DV + 64 * b, si.start + kt * BN);
          }
        }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // =================================================================== MMA issuers
    // Issue is synchronous with the tensor pipe, so S = Q K^T (warp 1) and O += P V
    // (warp 3) have a warp each: S of a later kv tile only waits until P V has
    // consumed its TMEM buffer, not until the P V before it has been issued.  The
    // whole warp runs the loop (its waits, counters and descriptors stay
    // warp-uniform) and one elected lane issues each MMA and commit.
    {
      const bool s_side = warp == 1;
      constexpr uint32_t idesc_s = make_idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(BM, DV, false, true);
      // descriptors of stage 0; every MMA below adds compile-time offsets to these
      const uint64_t dq0 = make_sw128_desc(sQ, 16, 1024);
      const uint64_t dk0 = make_sw128_desc(sK, 16, 1024);
      const uint64_t dv0 = make_sw128_desc(sV, kBoxBytes, 1024);
      int n_it = 0;  // global kv-tile counter of this warp
      for (int k = 0;; ++k) {
        const int slot = k % kItemSlots;
        if (!warp_wait(&bars->it_full[slot], (k / kItemSlots) & 1, tmo, abort_flag)) goto fail;
        const ItemInfo x = ring_get(item_ring, slot);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->it_empty[slot]);
        if (x.idx < 0) break;
        const WorkItem wi = x.wi;
        const SeqInfo si = x.si;
        const int r0 = wi.qtile * BM;
        const KvRange kr = kv_tiles_for(r0, min(si.n, r0 + BM), si.hist, BN);
        const int nk = kv_count(kr);
        if (s_side) {
          if (!warp_wait(&bars->q_full, k & 1, tmo, abort_flag)) goto fail;
          for (int jj = 0; jj < nk; ++jj, ++n_it) {
            // S of kv tile n_it into buffer n_it % kSBufs once P V of tile n_it - kSBufs is done
            const int st = n_it % SK;
            const int sb = n_it % kSBufs;
            if (!warp_wait(&bars->k_full[st], (n_it / SK) & 1, tmo, abort_flag)) goto fail;
            if (!warp_wait(&bars->pv_done[sb], ((n_it / kSBufs) & 1) ^ 1, tmo, abort_flag)) goto fail;
            tc_fence_after();
            const uint64_t dk = desc_advance(dk0, st * C::kTileBytes);
            const uint32_t dS = tmem_s0 + sb * BN;
#pragma unroll
            for (int ks = 0; ks < DH / 16; ++ks) {
              const uint32_t off = (ks >> 2) * kBoxBytes + (ks & 3) * 32;
              umma_f16_ss_elect(dS, desc_advance(dq0, off), desc_advance(dk, off), idesc_s, ks > 0 ? 1u : 0u);
            }
            umma_commit_elect(&bars->s_full[sb]);
            umma_commit_elect(&bars->k_empty[st]);
            if (jj == nk - 1) umma_commit_elect(&bars->q_empty);
          }
        } else {
          for (int jj = 0; jj < nk; ++jj, ++n_it) {
            // O (+)= P V for kv tile n_it, P read from TMEM
            const int pb = n_it % kSBufs;
            const int vs = n_it % SV;
            if (!warp_wait(&bars->p_full[pb], (n_it / kSBufs) & 1, tmo, abort_flag)) goto fail;
            if (!warp_wait(&bars->v_full[vs], (n_it / SV) & 1, tmo, abort_flag)) goto fail;
            if (jj == 0 && !warp_wait(&bars->o_empty, (k & 1) ^ 1, tmo, abort_flag)) goto fail;
            tc_fence_after();
            const uint32_t pa = tmem_s0 + pb * BN;
            const uint64_t dv = desc_advance(dv0, vs * C::kTileBytes);
            const uint32_t acc0 = jj > 0 ? 1u : 0u;
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks) {
              // kv columns [16ks, 16ks+16) were written by segment ks/2 at columns 32*(ks/2) + 8*(ks%2)
              umma_f16_ts_elect(tmem_o, pa + 32 * (ks >> 1) + 8 * (ks & 1), desc_advance(dv, ks * 16 * 128), idesc_o,
                                ks > 0 ? 1u : acc0);
            }
            umma_commit_elect(&bars->v_empty[vs]);
            umma_commit_elect(&bars->pv_done[pb]);
          }
          umma_commit_elect(&bars->o_full);
        }
      }
      // all MMAs this warp issued complete before TMEM is released
      uint64_t* dbar = s_side ? &bars->done : &bars->done_pv;
      umma_commit_elect(dbar);
      warp_wait(dbar, 0, tmo, nullptr);
    }
  } else {
    // =================================================================== epilogue
    const int ew = warp - kEpiWarp0;       // 0..15
    const int quarter = warp & 3;          // TMEM lane quarter this warp may access
    const int seg = ew >> 2;               // 32-column segment of S (and of O)
    const int r = quarter * 32 + lane;     // row of the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float k_lg = prm.ln2_over_div;
    int it = 0;  // global kv-tile counter
    int cur_head = -1;
    // The O readout of an item is deferred: a warp that finishes its part of an
    // item early goes on with the next item's kv tiles (their S needs no O) and
    // reads O once the item's last P V is done, instead of idling until the
    // slowest warp has finished.  At most one readout is pending per warp: the
    // next item's O cannot complete before every warp has read this one.
    constexpr int kOc = DV / 4;
    int pend_par = -1;                       // parity of the pending readout's o_full phase; -1: none
    // this lane's output row (null beyond the sequence) and 1/N, kept in shared memory
const auto pend = [&]() { return reinterpret_cast<PendingO*>(smem + L::kPend) + (threadIdx.x - 32 * kEpiWarp0); };
    for (int k = 0;; ++k) {
      const int slot = k % kItemSlots;
      if (!mbar_wait(&bars->it_full[slot], (k / kItemSlots) & 1, tmo, abort_flag)) goto fail;
      const ItemInfo x = ring_get(item_ring, slot);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->it_empty[slot]);
      if (x.idx < 0) break;
      const WorkItem wi = x.wi;
      const SeqInfo si = x.si;
      if (per_head_rab && wi.head != cur_head) {
        named_bar_sync(1, 32 * kEpiWarps);
        for (int c = threadIdx.x - 32 * kEpiWarp0; c < kNumBuckets; c += 32 * kEpiWarps) {
          pos_b[c] = p.pos_bias[wi.head * p.rab_head_stride + c];
          time_b[c] = p.time_bias[wi.head * p.rab_head_stride + c];
        }
        named_bar_sync(1, 32 * kEpiWarps);
        cur_head = wi.head;
      }
      const int r0 = wi.qtile * BM;
      const int i = r0 + r;
      const bool live = i < si.n;
      const bool cand = i >= si.hist;
      const int64_t t_first = si.n > 0 ? p.timestamps[si.start] : 0;
      const int64_t ti = live ? p.timestamps[si.start + i] : t_first;
      const int64_t rel64 = ti - t_first;
      const bool row_narrow = rel64 > -(1ll << 30) && rel64 < (1ll << 30);
      const int32_t ri = (int32_t)rel64;
      const int posi = token_pos(i, si.hist);
      const KvRange kr = kv_tiles_for(r0, min(si.n, r0 + BM), si.hist, BN);
      const int nk = kv_count(kr);
      // rows of the warp with fewer than 128 attended columns: their outputs may rest on
      // a few small terms, whose SiLU the tanh form would not keep accurate
      const bool few_terms = __any_sync(0xffffffffu, live && i < kNumBuckets);
      // this row's last one-bucket segment: distances in [c_lo, c_hi) share the
      // bias 2 * c_hb (empty until the first one); far from the diagonal the bucket
      // rarely changes from one kv tile to the next
      int32_t c_lo = 0x7FFFFFFF, c_hi = 0;
      float c_hb = 0.f;
      for (int jj = 0; jj < nk; ++jj, ++it) {
        const int c0 = kv_tile_at(kr, jj) * BN;
        const int sb = it % kSBufs;
        const int rs = it % kRecStages;
        // S of this tile into registers: at once when it is ready (the load is then in
        // flight during the classification), else after the classification, which
        // needs only the timestamp record and so runs while S is being computed
        bool s_ready = __all_sync(0xffffffffu, mbar_try_wait(&bars->s_full[sb], (it / kSBufs) & 1));
        if (!s_ready && pend_par >= 0) {
          // S may depend on P V of this item, which waits until every warp has read
          // the previous item's O: the pending readout goes first
          if (!o_readout<kOc>(bars, pend_par, tmem_o + lane_off + seg * kOc, pend(), lane, tmo, abort_flag)) goto fail;
          pend_par = -1;
          s_ready = __all_sync(0xffffffffu, mbar_try_wait(&bars->s_full[sb], (it / kSBufs) & 1));
        }
        uint32_t raw[32];
        if (s_ready) {
          tc_fence_after();
          tmem_ld_32x32b_x32(tmem_s0 + sb * BN + lane_off + seg * 32, raw);
        }
        if (!mbar_wait(&bars->r_full[rs], (it / kRecStages) & 1, tmo, abort_flag)) goto fail;
        const TsRec& rec = recs[rs];
        // ---- classify this row's 32 columns:
        //   rank 0: nothing attended; 1: one time bucket (constant bias); 2: two buckets;
        //   3: three or four buckets (per-element threshold compares); 4: general
        //   (per-element mask and exact buckets).  Far from the diagonal the position
        //   bucket is the last one for every column.
        const int cl = c0 + seg * 32;   // first column of the segment
        const bool narrow = row_narrow && !rec.wide;
        const bool any_live = live && (cand ? (cl < si.hist || (i >= cl && i < cl + 32)) : (cl <= i));
        const bool full = live && (cand ? (cl + 31 < si.hist) : (cl + 31 <= i));
        int rank = any_live ? 4 : 0;
        float hb0 = 0.f, hb1 = 0.f, hb2 = 0.f, hb3 = 0.f;   // half of the bias values
        int32_t th1 = 0x7FFFFFFF, th2 = 0x7FFFFFFF, th3 = 0x7FFFFFFF;
        if (full && narrow && posi - (cl + 31) >= kNumBuckets - 1) {
          const int32_t mn = rec.mn[seg], mx = rec.mx[seg];
          int32_t dlo, dhi;
          if (ri >= mx) { dlo = ri - mx; dhi = ri - mn; }
          else if (ri <= mn) { dlo = mn - ri; dhi = mx - ri; }
          else { dlo = 0; dhi = max(ri - mn, mx - ri); }
          if (dlo >= c_lo && dhi < c_hi) {
            rank = 1;
            hb0 = c_hb;
          } else {
          const int tlo = fast_bucket(dlo, thr32, k_lg);
          const float pb127 = pos_b[kNumBuckets - 1];
          hb0 = 0.5f * (pb127 + time_b[tlo]);
          if (dhi < thr32[tlo + 1]) {
            rank = 1;
            c_lo = thr32[tlo];
            c_hi = thr32[tlo + 1];
            c_hb = hb0;
          } else {
            const int thi = fast_bucket(dhi, thr32, k_lg);
            if (thi - tlo <= 3) {
              rank = thi - tlo == 1 ? 2 : 3;
              hb1 = 0.5f * (pb127 + time_b[tlo + 1]);
              th1 = thr32[tlo + 1];
              if (thi - tlo >= 2) { hb2 = 0.5f * (pb127 + time_b[tlo + 2]); th2 = thr32[tlo + 2]; }
              if (thi - tlo >= 3) { hb3 = 0.5f * (pb127 + time_b[tlo + 3]); th3 = thr32[tlo + 3]; }
            }
          }
          }
        }
        // one path per warp: the highest rank of its rows (a lower rank's row is a
        // special case of a higher one; rows beyond the sequence are zeroed below)
        const int wrank = __reduce_max_sync(0xffffffffu, rank);
        // the band serves warps of history rows (rows beyond the sequence are zero)
        // in segments starting at or after i0 - 128, i0 = the warp's first row
        const int i0w = r0 + quarter * 32;
        const bool use_band = wrank == 4 && p.band != nullptr && cl >= i0w - 128 &&
                              !__any_sync(0xffffffffu, live && cand);
        // warps of candidate rows (every row at or after N): the band's candidate window
        // [floor32(N) - 128, floor32(N) + 32), and beyond it only each row's own column
        const bool cand_warp = wrank == 4 && i0w >= si.hist;
        const int cwb = (si.hist & ~31) - 128;
        const bool use_cband = cand_warp && p.band != nullptr && cl >= cwb && cl < cwb + 160;
        const bool self_only = cand_warp && cl >= cwb + 160;
        if (!s_ready) {
          if (!mbar_wait(&bars->s_full[sb], (it / kSBufs) & 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
          tmem_ld_32x32b_x32(tmem_s0 + sb * BN + lane_off + seg * 32, raw);
        }
        tmem_ld_wait_regs(raw);
        // ---- bias, SiLU, mask; packed bf16 pairs.  With h = (s + bias) / 2, SiLU = h + h tanh h,
        // except on rows whose outputs may rest on a few terms (the first 128 rows of a
        // sequence, candidates, which see one column beyond the history): the exact form
        uint32_t pk[16];
        if (wrank == 0) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        } else if (wrank == 1) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float h0, h1;
            half_plus2(__uint_as_float(raw[2 * e]), __uint_as_float(raw[2 * e + 1]), hb0, h0, h1);
            pk[e] = silu2_bf16(h0, h1);
          }
        } else if (wrank == 2) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const int4 rel4 = *reinterpret_cast<const int4*>(&rec.rel[seg * 32 + e4 * 4]);
            const int32_t rv[4] = {rel4.x, rel4.y, rel4.z, rel4.w};
            float h[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              h[u] = fmaf(__uint_as_float(raw[e4 * 4 + u]), 0.5f, abs(ri - rv[u]) >= th1 ? hb1 : hb0);
            pk[2 * e4] = silu2_bf16(h[0], h[1]);
            pk[2 * e4 + 1] = silu2_bf16(h[2], h[3]);
          }
        } else if (wrank == 3) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const int4 rel4 = *reinterpret_cast<const int4*>(&rec.rel[seg * 32 + e4 * 4]);
            const int32_t rv[4] = {rel4.x, rel4.y, rel4.z, rel4.w};
            float h[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int32_t dd = abs(ri - rv[u]);
              float hb = dd >= th1 ? hb1 : hb0;
              hb = dd >= th2 ? hb2 : hb;
              hb = dd >= th3 ? hb3 : hb;
              h[u] = fmaf(__uint_as_float(raw[e4 * 4 + u]), 0.5f, hb);
            }
            pk[2 * e4] = silu2_bf16(h[0], h[1]);
            pk[2 * e4 + 1] = silu2_bf16(h[2], h[3]);
          }
        } else if (use_band) {
          // near-diagonal segment of history rows: half biases from the band
          // (bf16 pairs), mask j <= i
          uint4 bb[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                         make_uint4(0, 0, 0, 0)};
          if (live) {
            const uint4* bp = reinterpret_cast<const uint4*>(p.band) + (int64_t)(si.start + i) * kBandChunks +
                              ((cl - (i0w - 128)) >> 3);
#pragma unroll
            for (int c = 0; c < 4; ++c) bb[c] = __ldg(bp + c);
          }
          const int lim = live ? i - cl : -1;   // column e of the segment is attended iff e <= lim
          const uint32_t* bw = reinterpret_cast<const uint32_t*>(bb);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float h0, h1;
            half_plus2c(__uint_as_float(raw[2 * q]), __uint_as_float(raw[2 * q + 1]), __uint_as_float(bw[q] << 16),
                        __uint_as_float(bw[q] & 0xFFFF0000u), h0, h1);
            const uint32_t v = few_terms ? silu2_exact_bf16(h0, h1) : silu2_bf16(h0, h1);
            pk[q] = (2 * q <= lim ? (v & 0xFFFFu) : 0u) | (2 * q + 1 <= lim ? (v & 0xFFFF0000u) : 0u);
          }
        } else if (use_cband) {
          // candidate rows near the end of the history: half biases from the band's
          // candidate window; a column is attended iff it is history or the row's own
          // (the exact SiLU: a candidate's output may rest on few terms)
          uint4 bb[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                         make_uint4(0, 0, 0, 0)};
          if (live) {
            const uint4* bp = reinterpret_cast<const uint4*>(p.band) + (int64_t)(si.start + i) * kBandChunks +
                              ((cl - cwb) >> 3);
#pragma unroll
            for (int c = 0; c < 4; ++c) bb[c] = __ldg(bp + c);
          }
          const int lim_h = live ? si.hist - 1 - cl : -1;   // columns e <= lim_h are history
          const int e_self = live ? i - cl : -1;
          const uint32_t* bw = reinterpret_cast<const uint32_t*>(bb);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float h0, h1;
            half_plus2c(__uint_as_float(raw[2 * q]), __uint_as_float(raw[2 * q + 1]), __uint_as_float(bw[q] << 16),
                        __uint_as_float(bw[q] & 0xFFFF0000u), h0, h1);
            const uint32_t v = silu2_exact_bf16(h0, h1);
            pk[q] = ((2 * q <= lim_h || 2 * q == e_self) ? (v & 0xFFFFu) : 0u) |
                    ((2 * q + 1 <= lim_h || 2 * q + 1 == e_self) ? (v & 0xFFFF0000u) : 0u);
          }
        } else if (self_only) {
          // candidate columns only: each row attends its own column (position bucket 0,
          // time difference 0), if it lies in this segment
          const int e_self = live ? i - cl : -1;
          float s_self = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) s_self = e == e_self ? __uint_as_float(raw[e]) : s_self;
          const float h = fmaf(s_self, 0.5f, 0.5f * (pos_b[0] + time_b[0]));
          const uint32_t v = silu2_exact_bf16(h, h);
#pragma unroll
          for (int q = 0; q < 16; ++q)
            pk[q] = (e_self >> 1) == q ? ((e_self & 1) ? (v & 0xFFFF0000u) : (v & 0xFFFFu)) : 0u;
        } else if (__all_sync(0xffffffffu, narrow)) {
          // general, 32-bit time offsets: per-element mask, position and time bucket
          // (shared-memory reads kept few: the tensor core is reading Q, K and V
          // from the same shared memory meanwhile)
#pragma unroll
          for (int g4 = 0; g4 < 8; ++g4) {
            const int4 rel4 = *reinterpret_cast<const int4*>(&rec.rel[seg * 32 + 4 * g4]);
            const int32_t rv[4] = {rel4.x, rel4.y, rel4.z, rel4.w};
            float h[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = cl + 4 * g4 + u;
              const int32_t dd = abs(ri - rv[u]);
              const int tb = exact_bucket(dd < 1 ? 1 : dd, thr32, k_lg);
              const int pb = pos_bucket(posi, token_pos(j, si.hist));
              h[u] = 0.5f * (__uint_as_float(raw[4 * g4 + u]) + (pos_b[pb] + time_b[tb]));
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int j = cl + 4 * g4 + 2 * q;
              const uint32_t v = silu2_exact_bf16(h[2 * q], h[2 * q + 1]);
              pk[2 * g4 + q] = (attended(i, j, si.n, si.hist) ? (v & 0xFFFFu) : 0u) |
                               (attended(i, j + 1, si.n, si.hist) ? (v & 0xFFFF0000u) : 0u);
            }
          }
        } else {
          // general with 64-bit time differences (a row or column offset beyond +-2^30)
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            float h[2];
            bool att[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int e = 2 * e2 + u;
              const int j = cl + e;
              att[u] = attended(i, j, si.n, si.hist);
              float bias = 0.f;
              if (att[u]) {
                const int pb = pos_bucket(posi, token_pos(j, si.hist));
                const int tb = time_bucket_exact(abs_diff_i64(ti, p.timestamps[si.start + j]), thr);
                bias = pos_b[pb] + time_b[tb];
              }
              h[u] = 0.5f * (__uint_as_float(raw[e]) + bias);
            }
            const uint32_t v = silu2_exact_bf16(h[0], h[1]);
            pk[e2] = (att[0] ? (v & 0xFFFFu) : 0u) | (att[1] ? (v & 0xFFFF0000u) : 0u);
          }
        }
        if (rank == 0 && wrank != 4) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        // ---- P -> TMEM, over this segment's own S columns (the A operand of P V)
        tmem_st_32x32b_x16(tmem_s0 + sb * BN + lane_off + seg * 32, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->p_full[sb]);
          mbar_arrive(&bars->r_empty[rs]);
        }
        // the pending readout as soon as the previous item's O is complete
        if (pend_par >= 0 && __all_sync(0xffffffffu, mbar_try_wait(&bars->o_full, pend_par))) {
          if (!o_readout<kOc>(bars, pend_par, tmem_o + lane_off + seg * kOc, pend(), lane, tmo, abort_flag)) goto fail;
          pend_par = -1;
        }
      }
      // ---- this item's O readout becomes the pending one (an older one is done first)
      if (pend_par >= 0) {
        if (!o_readout<kOc>(bars, pend_par, tmem_o + lane_off + seg * kOc, pend(), lane, tmo, abort_flag)) goto fail;
      }
      pend_par = k & 1;
      pend()->out = live ? reinterpret_cast<__nv_bfloat16*>(p.out) + (int64_t)(si.start + i) * p.ldo +
                             (int64_t)wi.head * DV + seg * kOc
                       : nullptr;
      pend()->inv_n = si.inv_n;
    }
    if (pend_par >= 0) {
      if (!o_readout<kOc>(bars, pend_par, tmem_o + lane_off + seg * kOc, pend(), lane, tmo, abort_flag)) goto fail;
    }
  }
  goto teardown;
fail:
  set_status(p.status, HSTU_ERR_TIMEOUT);
  *abort_flag = 1;
  if ((warp == 0 || warp == 2) && lane == 0) {
    // let every copy this CTA may have issued land before it exits (bounded)
    for (int s = 0; s < 4; ++s) {
      if (warp == 0 && s < SK) {
        mbar_wait(&bars->k_full[s], 0, 100000000ll, nullptr);
        mbar_wait(&bars->k_full[s], 1, 100000000ll, nullptr);
      }
      if (warp == 0) {
        for (int rr = s; rr < kRecStages; rr += 4) {
          mbar_wait(&bars->r_full[rr], 0, 100000000ll, nullptr);
          mbar_wait(&bars->r_full[rr], 1, 100000000ll, nullptr);
        }
      }
      if (warp == 2 && s < SV) {
        mbar_wait(&bars->v_full[s], 0, 100000000ll, nullptr);
        mbar_wait(&bars->v_full[s], 1, 100000000ll, nullptr);
      }
    }
    if (warp == 0) {
      mbar_wait(&bars->q_full, 0, 100000000ll, nullptr);
      mbar_wait(&bars->q_full, 1, 100000000ll, nullptr);
    }
  }
teardown:
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Timestamp records: one block of 128 threads per kv tile of the batch.
__global__ void __launch_bounds__(128) ts_tiles_kernel(const int32_t* __restrict__ offs,
                                                       const int64_t* __restrict__ ts, int B,
                                                       const int32_t* __restrict__ tile_base,
                                                       int32_t* __restrict__ recs) {
  const int t = blockIdx.x;
  if (t >= tile_base[B]) return;
  int lo = 0, hi = B;  // sequence s with tile_base[s] <= t < tile_base[s + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_base[mid] <= t) lo = mid; else hi = mid;
  }
  const int s = lo;
  const int start = offs[s], n = offs[s + 1] - start;
  const int c = (t - tile_base[s]) * BN + threadIdx.x;
  const bool ok = c < n;
  const int64_t d = ok ? ts[start + c] - ts[start] : 0;
  const int64_t lim = (1ll << 30) - 1;
  const int32_t rel = (int32_t)(d < -lim ? -lim : (d > lim ? lim : d));
  const bool wide = ok && (d < -lim || d > lim);
  int32_t mn = ok ? rel : 0x7FFFFFFF, mx = ok ? rel : (int32_t)0x80000000;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const int any_wide = __syncthreads_or(wide);
  int32_t* rec = recs + (int64_t)t * kTsRecWords;
  rec[threadIdx.x] = rel;
  if ((threadIdx.x & 31) == 0) {
    const int w = threadIdx.x >> 5;
    rec[BN + w] = mn > mx ? 0 : mn;
    rec[BN + 4 + w] = mn > mx ? 0 : mx;
  }
  if (threadIdx.x == 0) {
    rec[BN + 8] = any_wide ? 1 : 0;
    rec[BN + 9] = rec[BN + 10] = rec[BN + 11] = 0;
  }
}

// ---------------------------------------------------------------------------
// host side: tensor maps
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

// 2-D bf16 map over [rows, cols] with row stride `ld` elements; box 64 columns x 128 rows, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int DH>
cudaError_t launch_tc(const AttnFwdParams& p, int grid, cudaStream_t st, double time_div) {
  TcParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.p = p;
  tp.ln2_over_div = (float)(0.69314718055994530942 / time_div);
  const int64_t hd = (int64_t)p.num_heads * DH;
  if (!make_map(&tp.map_q, p.q, hd, p.total_rows, p.ldq) || !make_map(&tp.map_k, p.k, hd, p.total_rows, p.ldk) ||
      !make_map(&tp.map_v, p.v, hd, p.total_rows, p.ldv))
    return cudaErrorInvalidValue;
  auto kern = attn_fwd_tc_kernel<DH>;
  const int smem = Layout<DH>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(tp);
  return cudaGetLastError();
}

// Near-diagonal bias band: for token row i of a sequence and the 160 columns
// j in [floor32(i) - 128, floor32(i) + 32), half of rab(i, j) as bf16, 0 where
// (i, j) is not attended.  A warp of 32 rows starting at i0 (a multiple of 32)
// reaches columns within 127 positions of its rows only in segments starting at
// i0 - 128 ... i0, which the band covers, so the epilogue reads these biases
// instead of evaluating both buckets per element there.  A group of 32 candidate
// rows (i0 >= N, position N for all) takes the window [floor32(N) - 128,
// floor32(N) + 32) instead: the history columns within 127 positions of N, and
// its own column where that falls inside (a candidate's other columns there are
// candidates, not attended).
// One block per group of 32 rows (four per 128-row tile of tile_base), one
// thread per band column: timestamps become 32-bit offsets from the sequence's
// first one (the 64-bit threshold search serves blocks whose offsets leave
// +-2^30), buckets follow the 32-bit rule of the attention kernel, and the rows
// leave as 16-byte stores.
constexpr int kBandCols = kBandChunks * 8;   // 160
__device__ __noinline__ int band_bucket_wide(int64_t ti, int64_t tj, const int64_t* thr) {
  return time_bucket_exact(abs_diff_i64(ti, tj), thr);
}
__global__ void __launch_bounds__(kBandCols) band_bias_kernel(const int32_t* __restrict__ offs,
                                                              const int32_t* __restrict__ num_targets,
                                                              const int64_t* __restrict__ ts, int B,
                                                              const int32_t* __restrict__ tile_base,
                                                              const float* __restrict__ pos_bias,
                                                              const float* __restrict__ time_bias,
                                                              const Thresholds thr_in, float ln2_over_div, int T,
                                                              const int32_t* __restrict__ status,
                                                              uint4* __restrict__ band) {
  __shared__ int64_t thr[kNumBuckets];
  __shared__ int32_t thr32[kNumBuckets + 4];
  __shared__ float pb_s[kNumBuckets], tb_s[kNumBuckets];
  __shared__ int32_t rel_s[kBandCols];
  __shared__ int64_t abs_s[kBandCols];
  __shared__ int32_t rrel_s[32];   // the group's rows
  __shared__ int64_t rabs_s[32];
  __shared__ __align__(16) uint16_t out_s[32][kBandCols];
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
  const int i0 = (t - tile_base[lo]) * 128 + 32 * (grp & 3);
  if (i0 >= si.n || si.start + si.n > T) return;
  const bool cand_grp = i0 >= si.hist;   // every row of the group a candidate
  const int w = threadIdx.x;
  const int j = (cand_grp ? (si.hist & ~31) : i0) - 128 + w;   // this thread's window column
  for (int c = w; c < kNumBuckets + 4; c += kBandCols) {
    if (c < kNumBuckets) {
      thr[c] = thr_in.v[c];
      thr32[c] = thr_in.v[c] > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)thr_in.v[c];
      pb_s[c] = pos_bias[c];
      tb_s[c] = time_bias[c];
    } else {
      thr32[c] = 0x7FFFFFFF;
    }
  }
  const int64_t t_first = ts[si.start];
  const int64_t tj = (j >= 0 && j < si.n) ? ts[si.start + j] : t_first;
  const int64_t rel = tj - t_first;
  const int64_t lim = (1ll << 30) - 1;
  rel_s[w] = (int32_t)(rel < -lim ? -lim : (rel > lim ? lim : rel));
  abs_s[w] = tj;
  bool wide_t = rel < -lim || rel > lim;
  if (w < 32) {
    const int64_t ti = i0 + w < si.n ? ts[si.start + i0 + w] : t_first;
    const int64_t reli = ti - t_first;
    rrel_s[w] = (int32_t)(reli < -lim ? -lim : (reli > lim ? lim : reli));
    rabs_s[w] = ti;
    wide_t = wide_t || reli < -lim || reli > lim;
  }
  const bool wide = __syncthreads_or(wide_t) != 0;
  const int32_t relj = rel_s[w];
  const int posj = token_pos(j, si.hist);
  const int rows = si.n - i0 < 32 ? si.n - i0 : 32;
  for (int r = 0; r < rows; ++r) {
    const int i = i0 + r;
    float v = 0.f;
    if (j >= 0 && attended(i, j, si.n, si.hist)) {
      const int pb = pos_bucket(token_pos(i, si.hist), posj);
      const int tb = wide ? band_bucket_wide(rabs_s[r], tj, thr)
                          : fast_bucket(abs(rrel_s[r] - relj), thr32, ln2_over_div);
      v = 0.5f * (pb_s[pb] + tb_s[tb]);
    }
    out_s[r][w] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  __syncthreads();
  for (int e = w; e < rows * kBandChunks; e += kBandCols) {
    const int r = e / kBandChunks, c = e - r * kBandChunks;
    band[(int64_t)(si.start + i0 + r) * kBandChunks + c] = *reinterpret_cast<const uint4*>(&out_s[r][8 * c]);
  }
}

// ---------------------------------------------------------------------------
// diagnostics
__global__ void debug_buckets_kernel(const int32_t* offs, const int32_t* num_targets, const int64_t* ts,
                                     const Thresholds thr_in, float ln2_over_div, const int32_t* pairs, int n,
                                     int32_t* out) {
  __shared__ int64_t thr[kNumBuckets];
  __shared__ int32_t thr32[kNumBuckets + 4];
  for (int c = threadIdx.x; c < kNumBuckets + 4; c += blockDim.x) {
    if (c < kNumBuckets) {
      thr[c] = thr_in.v[c];
      thr32[c] = thr_in.v[c] > 0x7FFFFFFF ? 0x7FFFFFFF : (int32_t)thr_in.v[c];
    } else {
      thr32[c] = 0x7FFFFFFF;
    }
  }
  __syncthreads();
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const SeqInfo si = load_seq(offs, num_targets, pairs[3 * e]);
    const int i = pairs[3 * e + 1], j = pairs[3 * e + 2];
    int pb = -1, tb = -1, att = 0;
    if (i >= 0 && i < si.n && j >= 0 && j < si.n) {
      pb = pos_bucket(token_pos(i, si.hist), token_pos(j, si.hist));
      // the tensor-core kernel's rule: the 32-bit path below 2^31 - 1, else the
      // 64-bit threshold search
      const int64_t dt = abs_diff_i64(ts[si.start + i], ts[si.start + j]);
      tb = dt < 0x7FFFFFFF ? fast_bucket((int32_t)dt, thr32, ln2_over_div) : time_bucket_exact(dt, thr);
      att = attended(i, j, si.n, si.hist) ? 1 : 0;
    }
    out[3 * e] = pb;
    out[3 * e + 1] = tb;
    out[3 * e + 2] = att;
  }
}

__global__ void timeout_probe_kernel(long long timeout_ns, int32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the bounded wait must give up
  if (!mbar_wait(&bar, 0, timeout_ns, nullptr)) {
    if (threadIdx.x == 0) *status = HSTU_ERR_TIMEOUT;
  } else if (threadIdx.x == 0) {
    *status = HSTU_OK;
  }
}

}  // namespace

int tc_tile_m() { return BM; }

bool tc_attn_supported(int dtype, int dh) { return dtype == HSTU_DTYPE_BF16 && (dh == 64 || dh == 128); }

int tc_attn_grid(int max_items) {
  const int s = num_sms();
  return max_items < 1 ? 1 : (max_items < s ? max_items : s);
}

cudaError_t launch_attn_fwd_tc(const AttnFwdParams& p, int dh, int grid, cudaStream_t st, double time_div) {
  if (p.total_rows <= 0) return cudaSuccess;
  if (dh == 128) return launch_tc<128>(p, grid, st, time_div);
  if (dh == 64) return launch_tc<64>(p, grid, st, time_div);
  return cudaErrorInvalidValue;
}

size_t ts_tiles_capacity(int B, int T) { return (size_t)T / BN + (size_t)B + 1; }

size_t band_bytes(int T) { return (size_t)T * kBandChunks * 16; }

cudaError_t launch_band_bias(const int32_t* offs, const int32_t* num_targets, const int64_t* ts, int B, int T,
                             const int32_t* tile_base, int tiles_cap, const float* pos_bias,
                             const float* time_bias, const Thresholds& thr, double time_div, const int32_t* status,
                             void* band, cudaStream_t st) {
  if (T <= 0 || B <= 0 || tiles_cap <= 0) return cudaSuccess;
  band_bias_kernel<<<4 * tiles_cap, kBandCols, 0, st>>>(offs, num_targets, ts, B, tile_base, pos_bias, time_bias, thr,
                                                  (float)(0.69314718055994530942 / time_div), T, status,
                                                  reinterpret_cast<uint4*>(band));
  return cudaGetLastError();
}

cudaError_t launch_ts_tiles(const int32_t* offs, const int64_t* ts, int B, const int32_t* tile_base, int tiles_cap,
                            int32_t* recs, cudaStream_t st) {
  if (tiles_cap <= 0) return cudaSuccess;
  ts_tiles_kernel<<<tiles_cap, 128, 0, st>>>(offs, ts, B, tile_base, recs);
  return cudaGetLastError();
}

cudaError_t launch_debug_buckets(const int32_t* offs, const int32_t* num_targets, const int64_t* ts,
                                 const Thresholds& thr, double time_div, const int32_t* pairs, int n, int32_t* out,
                                 cudaStream_t st) {
  const int grid = (n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024;
  debug_buckets_kernel<<<grid, 256, 0, st>>>(offs, num_targets, ts, thr, (float)(0.69314718055994530942 / time_div),
                                             pairs, n, out);
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(long long timeout_ns, int32_t* status, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(timeout_ns, status);
  return cudaGetLastError();
}

}  // namespace hstu
