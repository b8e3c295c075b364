// tcgen05 GEMM with the layer's fused epilogues (sm_100a).
//
//   D[m, n] = sum_k A(m, k) B(n, k)        bf16 operands, fp32 accumulation in TMEM
//
// A and B may each be K-major (k contiguous) or MN-major (m or n contiguous);
// the MN-major forms serve the weight-gradient products of the backward pass
// without transposing activations.  One persistent CTA per SM walks the output
// tiles (128 x BN, BN = 256 or 128); a long reduction may be split over
// `split` CTAs whose partial tiles are added into an fp32 output with atomics.
//
//   warp 0     TMA producer: A and B k-slices (64 deep) into a ring of stages
//   warp 1     one thread issues tcgen05.mma into one of two TMEM accumulators
//   warps 2-17 epilogue: TMEM -> registers -> bias / SiLU / residual -> global;
//              four warps per TMEM lane quarter, each on a quarter of the columns,
//              so every SM sub-partition has four warps to hide the latencies
// The two accumulators let the epilogue of one tile overlap the main loop of
// the next.  ("Actions Speak Louder than Words" summary, 2.2: the linear layers
// are fused with LayerNorm and SiLU; f1 and f2 are single linear layers.)
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
namespace {
using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;                       // one 128-byte swizzle atom of bf16
constexpr int kEpiWarps = 16;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kABytes = BM * BK * 2;         // 16 KB

template <int BN>
struct GCfg {
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kXpose = kBarOff + 256;                  // per epilogue warp: a 32 x 64-byte transpose tile
  static constexpr int kAlloc = kXpose + kEpiWarps * 2048 + 1024;
  static constexpr uint32_t kTmemCols = 2 * BN <= 32 ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
};

struct GBars {
  uint64_t full[6], empty[6];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t done;
};

struct TcGemmParams {
  CUtensorMap map_a;
  CUtensorMap map_b;
  GemmParams p;
  int a_mn;          // A is MN-major
  int b_mn;          // B is MN-major
  int split;         // K splits
  int k_chunk;       // K elements per split (multiple of BK)
  int out_f32;       // output element type (EPI_BIAS_RESIDUAL / EPI_STORE): 1 = fp32
  int res_f32;       // residual element type: 1 = fp32
  long long timeout_ns;
  int32_t* status;
};

struct Unit {
  int m0, n0, k0, k1;
};

__device__ __forceinline__ bool unit_of(const TcGemmParams& tp, int u, int n_tiles, int M_eff, int K_eff, int BN,
                                        Unit& out) {
  const int per_m = n_tiles * tp.split;
  const int mt = u / per_m;
  const int rem = u % per_m;
  const int nt = rem / tp.split;
  const int ks = rem % tp.split;
  out.m0 = mt * BM;
  out.n0 = nt * BN;
  out.k0 = ks * tp.k_chunk;
  out.k1 = min(K_eff, out.k0 + tp.k_chunk);
  return out.m0 < M_eff;
}

__device__ __forceinline__ float silu_fast(float v) {
  const float h = 0.5f * v;
  return fmaf(h, tanh_approx(h), h);
}

// One thread's 32 consecutive accumulator columns [n0, n0+32) of row m -> output.
// A warp's 32 rows x 32 bf16 columns (64 bytes a row, one row per lane in w) to
// global memory through its shared-memory tile: every store instruction then
// writes 8 whole 64-byte row pieces (4 lanes a row) instead of 32 scattered
// 16-byte pieces.  The tile's 16-byte chunks are XOR-swizzled by row so that
// both the row-wise writes and the transposed reads are free of bank conflicts.
// (base: the first of the 64 bytes of row m_first; ld_bytes: the row stride)
__device__ __forceinline__ void store_rows_xpose(uint4* tile, const uint4 (&w)[4], char* base, int64_t ld_bytes,
                                                 int m_first, int m_end, int lane) {
#pragma unroll
  for (int k = 0; k < 4; ++k) tile[lane * 4 + (k ^ ((lane >> 1) & 3))] = w[k];
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = 8 * j + (lane >> 2), pc = lane & 3;
    const uint4 v = tile[r * 4 + (pc ^ ((r >> 1) & 3))];
    if (m_first + r < m_end) *reinterpret_cast<uint4*>(base + (int64_t)r * ld_bytes + 16 * pc) = v;
  }
  __syncwarp();
}
// store_rows_xpose with a destination per row: my_row is the address of this
// lane's row (row m_first + lane) at the chunk's first column, or nullptr to drop
// it; the storing lanes take the addresses by shuffle
__device__ __forceinline__ void store_rows_xpose_mapped(uint4* tile, const uint4 (&w)[4], char* my_row, int lane) {
#pragma unroll
  for (int k = 0; k < 4; ++k) tile[lane * 4 + (k ^ ((lane >> 1) & 3))] = w[k];
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = 8 * j + (lane >> 2), pc = lane & 3;
    const uint4 v = tile[r * 4 + (pc ^ ((r >> 1) & 3))];
    char* rb = reinterpret_cast<char*>(
        __shfl_sync(0xffffffffu, static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(my_row)), r));
    if (rb) *reinterpret_cast<uint4*>(rb + 16 * pc) = v;
  }
  __syncwarp();
}
__device__ __forceinline__ void pack8_bf16(const float* v, uint4& w) {
  w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
}

// The EPI_BIAS_RESIDUAL / EPI_STORE outputs of a warp's 32 rows x 32 columns (full,
// no split, no accumulate): the output through the warp's transpose tile, 8 whole
// row pieces per store instruction.
__device__ __forceinline__ void epilogue_chunk_xpose(const TcGemmParams& tp, uint4* tile, int m_first, int m_end,
                                                     int n0, const uint32_t (&raw)[32], bool has_k, int lane) {
  const GemmParams& p = tp.p;
  float v[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = has_k ? __uint_as_float(raw[e]) : 0.f;
  if (p.epi == EPI_BIAS_RESIDUAL && p.bias) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + n0 + e));
      v[e] += b.x; v[e + 1] += b.y; v[e + 2] += b.z; v[e + 3] += b.w;
    }
  }
  int64_t m = m_first + lane < m_end ? m_first + lane : -1;   // this lane's residual row
  if (m >= 0 && p.res_map) m = p.res_map[m];
  if (p.epi == EPI_BIAS_RESIDUAL && p.residual && m >= 0) {
    // the residual row by its own lane (all its loads in flight together)
    if (tp.res_f32) {
      const float* rs = (const float*)p.residual + m * p.ldr + n0;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 w = *reinterpret_cast<const float4*>(rs + e);
        v[e] += w.x; v[e + 1] += w.y; v[e + 2] += w.z; v[e + 3] += w.w;
      }
    } else {
      const __nv_bfloat16* rs = (const __nv_bfloat16*)p.residual + m * p.ldr + n0;
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        const uint4 w = *reinterpret_cast<const uint4*>(rs + e);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(h[q]);
          v[e + 2 * q] += f.x;
          v[e + 2 * q + 1] += f.y;
        }
      }
    }
  }
  // with out_map: this lane's output row, or -1 (dropped)
  const int64_t mo = p.out_map ? (m_first + lane < m_end ? p.out_map[m_first + lane] : -1) : 0;
  if (tp.out_f32 || p.epi == EPI_STORE_F32) {
    char* ob = (char*)((float*)p.out + (int64_t)m_first * p.ldo + n0);
    char* my = mo >= 0 ? (char*)((float*)p.out + mo * p.ldo + n0) : nullptr;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        w[k] = make_uint4(__float_as_uint(v[16 * h + 4 * k]), __float_as_uint(v[16 * h + 4 * k + 1]),
                          __float_as_uint(v[16 * h + 4 * k + 2]), __float_as_uint(v[16 * h + 4 * k + 3]));
      if (p.out_map) store_rows_xpose_mapped(tile, w, my ? my + 64 * h : nullptr, lane);
      else store_rows_xpose(tile, w, ob + 64 * h, p.ldo * 4, m_first, m_end, lane);
    }
  } else {
    uint4 w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) pack8_bf16(v + 8 * k, w[k]);
    if (p.out_map)
      store_rows_xpose_mapped(tile, w, mo >= 0 ? (char*)((__nv_bfloat16*)p.out + mo * p.ldo + n0) : nullptr, lane);
    else
      store_rows_xpose(tile, w, (char*)((__nv_bfloat16*)p.out + (int64_t)m_first * p.ldo + n0), p.ldo * 2, m_first,
                       m_end, lane);
  }
}

__device__ __forceinline__ void epilogue_chunk(const TcGemmParams& tp, int m, int n0, const uint32_t (&raw)[32],
                                               bool has_k) {
  const GemmParams& p = tp.p;
  float v[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = has_k ? __uint_as_float(raw[e]) : 0.f;
  const bool full32 = n0 + 32 <= p.N;
  if (p.epi == EPI_STORE_F32) {
    float* o = (float*)p.out + (int64_t)m * p.ldo + n0;
    if (tp.split > 1) {
      if (has_k) {
        if (full32 && ((uintptr_t)o & 15) == 0) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) red_add_f32x4(o + e, v[e], v[e + 1], v[e + 2], v[e + 3]);
        } else {
          for (int e = 0; e < 32; ++e)
            if (n0 + e < p.N) atomicAdd(o + e, v[e]);
        }
      }
    } else if (full32) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        float4 w = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        if (p.accumulate) {
          const float4 old = *reinterpret_cast<const float4*>(o + e);
          w.x += old.x; w.y += old.y; w.z += old.z; w.w += old.w;
        }
        *reinterpret_cast<float4*>(o + e) = w;
      }
    } else {
      for (int e = 0; e < 32 && n0 + e < p.N; ++e) o[e] = p.accumulate ? o[e] + v[e] : v[e];
    }
    return;
  }
  if (p.epi == EPI_BIAS_RESIDUAL && p.bias) {
    if (full32) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + n0 + e));
        v[e] += b.x; v[e + 1] += b.y; v[e + 2] += b.z; v[e + 3] += b.w;
      }
    } else {
      for (int e = 0; e < 32 && n0 + e < p.N; ++e) v[e] += p.bias[n0 + e];
    }
  }
  if (p.epi == EPI_BIAS_RESIDUAL && p.residual) {
    if (tp.res_f32) {
      const float* rs = (const float*)p.residual + (int64_t)m * p.ldr + n0;
      if (full32) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 w = *reinterpret_cast<const float4*>(rs + e);
          v[e] += w.x; v[e + 1] += w.y; v[e + 2] += w.z; v[e + 3] += w.w;
        }
      } else {
        for (int e = 0; e < 32 && n0 + e < p.N; ++e) v[e] += rs[e];
      }
    } else {
      const __nv_bfloat16* rs = (const __nv_bfloat16*)p.residual + (int64_t)m * p.ldr + n0;
      if (full32) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          const uint4 w = *reinterpret_cast<const uint4*>(rs + e);
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h[q]);
            v[e + 2 * q] += f.x;
            v[e + 2 * q + 1] += f.y;
          }
        }
      } else {
        for (int e = 0; e < 32 && n0 + e < p.N; ++e) v[e] += __bfloat162float(rs[e]);
      }
    }
  }
  // EPI_BIAS_RESIDUAL / EPI_STORE in the output type
  if (tp.out_f32) {
    float* o = (float*)p.out + (int64_t)m * p.ldo + n0;
    if (full32) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    } else {
      for (int e = 0; e < 32 && n0 + e < p.N; ++e) o[e] = v[e];
    }
  } else {
    __nv_bfloat16* o = (__nv_bfloat16*)p.out + (int64_t)m * p.ldo + n0;
    if (full32) {
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 w;
        w.x = pack_bf16x2(v[e], v[e + 1]); w.y = pack_bf16x2(v[e + 2], v[e + 3]);
        w.z = pack_bf16x2(v[e + 4], v[e + 5]); w.w = pack_bf16x2(v[e + 6], v[e + 7]);
        *reinterpret_cast<uint4*>(o + e) = w;
      }
    } else {
      for (int e = 0; e < 32 && n0 + e < p.N; ++e) o[e] = __float2bfloat16_rn(v[e]);
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ TcGemmParams tp) {
  using C = GCfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  GBars* bars = reinterpret_cast<GBars*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + sizeof(GBars));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + sizeof(GBars) + 4);
  const GemmParams& p = tp.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tmo = tp.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&bars->full[s], 1); mbar_init(&bars->empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&bars->acc_full[s], 1); mbar_init(&bars->acc_empty[s], kEpiWarps); }
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tp.map_a);
    tma_prefetch_desc(&tp.map_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int M_eff = p.rows_dev ? min(p.M, *p.rows_dev) : p.M;
  const int K_eff = p.k_dev ? min(p.K, *p.k_dev) : p.K;
  const int m_tiles = (p.M + BM - 1) / BM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int units = m_tiles * n_tiles * tp.split;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      for (int u = blockIdx.x; u < units; u += gridDim.x) {
        Unit un;
        if (!unit_of(tp, u, n_tiles, M_eff, K_eff, BN, un)) continue;
        for (int k = un.k0; k < un.k1; k += BK, ++it) {
          const int st = it % S;
          if (!mbar_wait(&bars->empty[st], ((it / S) & 1) ^ 1, tmo, abort_flag)) goto fail;
          uint8_t* sa = smem + st * C::kStageBytes;
          uint8_t* sb = sa + kABytes;
          mbar_arrive_expect_tx(&bars->full[st], C::kStageBytes);
          if (tp.a_mn) {
            for (int b = 0; b < BM / 64; ++b) tma_load_2d(sa + b * 8192, &tp.map_a, &bars->full[st], un.m0 + 64 * b, k);
          } else {
            tma_load_2d(sa, &tp.map_a, &bars->full[st], k, un.m0);
          }
          if (tp.b_mn) {
            for (int b = 0; b < BN / 64; ++b) tma_load_2d(sb + b * 8192, &tp.map_b, &bars->full[st], un.n0 + 64 * b, k);
          } else {
            tma_load_2d(sb, &tp.map_b, &bars->full[st], k, un.n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(BM, BN, tp.a_mn != 0, tp.b_mn != 0);
      int it = 0, t = 0;
      for (int u = blockIdx.x; u < units; u += gridDim.x) {
        Unit un;
        if (!unit_of(tp, u, n_tiles, M_eff, K_eff, BN, un)) continue;
        const int ab = t & 1;
        if (!mbar_wait(&bars->acc_empty[ab], ((t >> 1) & 1) ^ 1, tmo, abort_flag)) goto fail;
        tc_fence_after();
        const uint32_t dacc = tmem_base + ab * BN;
        bool first = true;
        for (int k = un.k0; k < un.k1; k += BK, ++it) {
          const int st = it % S;
          if (!mbar_wait(&bars->full[st], (it / S) & 1, tmo, abort_flag)) goto fail;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * C::kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t da = tp.a_mn ? make_sw128_desc(sa + ks * 2048, 8192, 1024)
                                        : make_sw128_desc(sa + ks * 32, 16, 1024);
            const uint64_t db = tp.b_mn ? make_sw128_desc(sb + ks * 2048, 8192, 1024)
                                        : make_sw128_desc(sb + ks * 32, 16, 1024);
            umma_f16_ss(dacc, da, db, idesc, first ? 0u : 1u);
            first = false;
          }
          umma_commit(&bars->empty[st]);
        }
        umma_commit(&bars->acc_full[ab]);
        ++t;
      }
      umma_commit(&bars->done);
      mbar_wait(&bars->done, 0, tmo, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;          // TMEM lane quarter this warp may access
    const int group = (warp - 2) >> 2;     // quarter of the tile's columns
    uint4* const xtile = reinterpret_cast<uint4*>(smem + C::kXpose) + (warp - 2) * 128;   // 2 KB
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    constexpr int kCols = BN / 4;
    int t = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      Unit un;
      if (!unit_of(tp, u, n_tiles, M_eff, K_eff, BN, un)) continue;
      const int ab = t & 1;
      const int m = un.m0 + r;
      const bool row_ok = m < M_eff;
      const int64_t rm = row_ok && p.res_map ? p.res_map[m] : m;   // the residual row (-1: none)
      if (p.epi == EPI_BIAS_RESIDUAL && p.residual && row_ok && rm >= 0 && un.n0 + group * kCols < p.N) {
        // this lane's residual row piece (kCols columns) on its way to L2 while
        // the main loop still fills the accumulator
        const int c0 = un.n0 + group * kCols, es = tp.res_f32 ? 4 : 2;
        const int bytes = (p.N - c0 < kCols ? p.N - c0 : kCols) * es;   // inside the row
        const char* rp = (const char*)p.residual + (rm * p.ldr + c0) * es;
#pragma unroll
        for (int b = 0; b < kCols * 4; b += 128)
          if (b < bytes) prefetch_l2(rp + b);
      }
      int64_t slot_row = -1;   // this lane's output row in the slot layout (out_slot_offs)
      if (p.out_slot_offs && row_ok) {
        const int64_t sr = (int64_t)p.out_slot_offs[m / p.out_slot_bm + 1] + m;
        slot_row = sr < p.out_slot_cap ? sr : -1;
      }
      if (!mbar_wait(&bars->acc_full[ab], (t >> 1) & 1, tmo, abort_flag)) goto fail;
      tc_fence_after();
      const bool has_k = un.k1 > un.k0;  // an empty K range never wrote the accumulator
#pragma unroll 1
      for (int c = group * kCols; c < (group + 1) * kCols; c += 32) {
        __syncwarp();
        uint32_t raw[32];
        tmem_ld_32x32b_x32(tmem_base + ab * BN + lane_off + c, raw);
        tmem_ld_wait();
        const int n0 = un.n0 + c;
        if (p.epi == EPI_BIAS_SILU) {
          // (N % 32 == 0 on this path) bias, z = pre-activation and U|V|Q|K = SiLU(z) as bf16,
          // stored through the warp's transpose tile
          if (n0 < p.N) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 b = p.bias ? __ldg(reinterpret_cast<const float4*>(p.bias + n0 + e))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
              v[e] = (has_k ? __uint_as_float(raw[e]) : 0.f) + b.x;
              v[e + 1] = (has_k ? __uint_as_float(raw[e + 1]) : 0.f) + b.y;
              v[e + 2] = (has_k ? __uint_as_float(raw[e + 2]) : 0.f) + b.z;
              v[e + 3] = (has_k ? __uint_as_float(raw[e + 3]) : 0.f) + b.w;
            }
            const int m_first = un.m0 + quarter * 32;
            uint4 w[4];
            if (p.out2) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int e = 8 * k;
                w[k].x = pack_bf16x2(v[e], v[e + 1]); w[k].y = pack_bf16x2(v[e + 2], v[e + 3]);
                w[k].z = pack_bf16x2(v[e + 4], v[e + 5]); w[k].w = pack_bf16x2(v[e + 6], v[e + 7]);
              }
              store_rows_xpose(xtile, w, (char*)((__nv_bfloat16*)p.out2 + (int64_t)m_first * p.ldo2 + n0),
                               p.ldo2 * 2, m_first, M_eff, lane);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int e = 8 * k;
              w[k].x = pack_bf16x2(silu_fast(v[e]), silu_fast(v[e + 1]));
              w[k].y = pack_bf16x2(silu_fast(v[e + 2]), silu_fast(v[e + 3]));
              w[k].z = pack_bf16x2(silu_fast(v[e + 4]), silu_fast(v[e + 5]));
              w[k].w = pack_bf16x2(silu_fast(v[e + 6]), silu_fast(v[e + 7]));
            }
            if (p.out_slot_offs)
              store_rows_xpose_mapped(xtile, w,
                                      slot_row >= 0 ? (char*)((__nv_bfloat16*)p.out + slot_row * p.ldo + n0) : nullptr,
                                      lane);
            else
              store_rows_xpose(xtile, w, (char*)((__nv_bfloat16*)p.out + (int64_t)m_first * p.ldo + n0), p.ldo * 2,
                               m_first, M_eff, lane);
          }
        } else if ((p.epi == EPI_BIAS_RESIDUAL || p.epi == EPI_STORE ||
                    (p.epi == EPI_STORE_F32 && tp.split == 1 && !p.accumulate)) && n0 + 32 <= p.N) {
          // whole 32-column chunks: the rows through the warp's transpose tile
          epilogue_chunk_xpose(tp, xtile, un.m0 + quarter * 32, M_eff, n0, raw, has_k, lane);
        } else if (row_ok && n0 < p.N && !p.res_map && !p.out_map) {
          epilogue_chunk(tp, m, n0, raw, has_k);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[ab]);
      ++t;
    }
  }
  goto teardown;
fail:
  set_status(tp.status, HSTU_ERR_TIMEOUT);
  *abort_flag = 1;
  if (warp == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_wait(&bars->full[s], 0, 100000000ll, nullptr);
      mbar_wait(&bars->full[s], 1, 100000000ll, nullptr);
    }
  }
teardown:
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
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

// bf16 matrix with `inner` contiguous elements per line and `outer` lines `ld` elements apart;
// box: 64 inner elements x `box_outer` lines, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld, int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)(outer > 0 ? outer : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

template <int BN>
cudaError_t launch_bn(TcGemmParams& tp, cudaStream_t st) {
  const GemmParams& p = tp.p;
  const int m_tiles = (p.M + BM - 1) / BM, n_tiles = (p.N + BN - 1) / BN;
  // A: K-major -> inner K, outer M, box {64, 128}; MN-major -> inner M, outer K, box {64, 64}
  bool ok = tp.a_mn ? make_map(&tp.map_a, p.A, p.M, p.K, p.sak, 64) : make_map(&tp.map_a, p.A, p.K, p.M, p.sam, BM);
  ok = ok && (tp.b_mn ? make_map(&tp.map_b, p.B, p.N, p.K, p.sbk, 64) : make_map(&tp.map_b, p.B, p.K, p.N, p.sbn, BN));
  if (!ok) return cudaErrorInvalidValue;
  const int units = m_tiles * n_tiles * tp.split;
  const int grid = units < sm_count() ? units : sm_count();
  auto kern = gemm_tc_kernel<BN>;
  const int smem = GCfg<BN>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(tp);
  return cudaGetLastError();
}

}  // namespace

bool tc_gemm_supported(const GemmParams& p, int dtype) {
  if (dtype != HSTU_DTYPE_BF16) return false;
  if (p.M <= 0 || p.N <= 0 || p.K <= 0) return false;
  if (!(p.sak == 1 || p.sam == 1) || !(p.sbk == 1 || p.sbn == 1)) return false;
  if (!aligned16(p.A) || !aligned16(p.B) || !aligned16(p.out)) return false;
  const int64_t lda = p.sak == 1 ? p.sam : p.sak, ldb = p.sbk == 1 ? p.sbn : p.sbk;
  if ((lda * 2) % 16 || (ldb * 2) % 16) return false;
  if (p.epi == EPI_SILU_BWD) return false;
  if (p.epi == EPI_BIAS_SILU && p.N % 32) return false;
  if ((p.res_map || p.out_map) && (p.epi != EPI_BIAS_RESIDUAL || p.N % 32)) return false;
  if (p.out_slot_offs && p.epi != EPI_BIAS_SILU) return false;
  if ((p.sak != 1 && p.M % 64) || (p.sbk != 1 && p.N % 64)) return false;
  return true;
}

cudaError_t launch_gemm_tc(const GemmParams& p, cudaStream_t st) {
  TcGemmParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.p = p;
  tp.a_mn = p.sak != 1;
  tp.b_mn = p.sbk != 1;
  tp.out_f32 = p.out_f32;
  tp.res_f32 = p.res_f32;
  tp.timeout_ns = 2000000000ll;
  tp.status = p.status;
  const int BN = p.N >= 256 ? 256 : 128;
  const int m_tiles = (p.M + BM - 1) / BM, n_tiles = (p.N + BN - 1) / BN;
  // split the reduction when the output tiles alone cannot fill the GPU
  int split = 1;
  if (p.epi == EPI_STORE_F32 && !p.accumulate) {
    const int tiles = m_tiles * n_tiles;
    const int k_steps = (p.K + BK - 1) / BK;
    while (tiles * split * 2 <= sm_count() && k_steps / (split * 2) >= 4) split *= 2;
    if (split > 1) {
      // the fp32 output is accumulated with atomics: start from zero
      cudaError_t e = cudaMemset2DAsync(p.out, sizeof(float) * p.ldo, 0, sizeof(float) * p.N, p.M, st);
      if (e != cudaSuccess) return e;
    }
  }
  const int k_steps = (p.K + BK - 1) / BK;
  tp.split = split;
  tp.k_chunk = ((k_steps + split - 1) / split) * BK;
  return BN == 256 ? launch_bn<256>(tp, st) : launch_bn<128>(tp, st);
}

}  // namespace hstu
