// Memory-bound row kernels of the HSTU layer: LayerNorm (forward/backward),
// LayerNorm(A V) (.) U gating and its backward, SiLU backward, column sums,
// row gathers, Stochastic Length selection and M-FALCON packing.
//
// Every row kernel assigns one warp per row and moves 8 elements per lane per
// access (16-byte vectors for bf16), with warp-shuffle reductions.
// ("Actions Speak Louder than Words" summary, 2.2: LayerNorm and SiLU fused
// into the two linear layers; "Meta HSTU", "Что меняется внутри HSTU":
// normalisation after aggregation, element-wise product with U.)
#include <cub/block/block_scan.cuh>

#include "common.cuh"
#include "kernels.cuh"

namespace hstu {
namespace {

constexpr int kRowWarps = 8;          // warps (rows) per block
constexpr int kMaxChunks = 4;         // 8-element chunks per lane: d <= 32*8*4 = 1024
constexpr int kColPartBlocks = 1024;  // row blocks of the SiLU backward's column partial sums

__device__ __forceinline__ void load8(const float* p, float v[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float v[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(float* p, const float v[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float v[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// source row of row m when rows are read from the M-FALCON slot layout (see launch_ln_gate)
struct SlotMap {
  const int32_t* offs;
  int bm, cap;
};
__device__ __forceinline__ int64_t src_row(const SlotMap& m, int row) {
  if (!m.offs) return row;
  const int64_t s = (int64_t)m.offs[row / m.bm + 1] + row;
  return s < m.cap ? s : 0;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int rows_of(int cap, const int32_t* rows_dev) {
  if (!rows_dev) return cap;
  int r = *rows_dev;
  return r < cap ? r : cap;
}

// ---------------------------------------------------------------- LayerNorm
template <typename T, typename TO>
__global__ void __launch_bounds__(kRowWarps * 32)
layer_norm_kernel(const T* __restrict__ x, int64_t ldx, const float* __restrict__ gamma,
                  const float* __restrict__ beta, float eps, TO* __restrict__ out, int64_t ldo,
                  float* __restrict__ mean_out, float* __restrict__ rstd_out, int rows_cap,
                  const int32_t* __restrict__ rows_dev, int d, const int32_t* __restrict__ in_map) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int nch = d / 8;
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    const int src = in_map ? in_map[row] : row;   // < 0: a zero row
    float v[kMaxChunks][8];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        if (src >= 0) {
          load8(x + (int64_t)src * ldx + ch * 8, v[c]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[c][e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) s += v[c][e];
      }
    }
    const float mean = warp_sum(s) / d;
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      if (lane + 32 * c < nch) {
#pragma unroll
        for (int e = 0; e < 8; ++e) { float t = v[c][e] - mean; q += t * t; }
      }
    }
    const float rstd = 1.0f / sqrtf(warp_sum(q) / d + eps);
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float o[8];
        float g[8], b[8];
        load8(gamma + ch * 8, g);
        load8(beta + ch * 8, b);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = (v[c][e] - mean) * rstd * g[e] + b[e];
        store8(out + (int64_t)row * ldo + ch * 8, o);
      }
    }
    if (lane == 0) {
      if (mean_out) mean_out[row] = mean;
      if (rstd_out) rstd_out[row] = rstd;
    }
  }
}

// g = LN(o) * u
template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32)
ln_gate_kernel(const T* __restrict__ o, int64_t ldo_in, const T* __restrict__ u, int64_t ldu,
               const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
               T* __restrict__ out, int64_t ldout, float* __restrict__ mean_out, float* __restrict__ rstd_out,
               int rows_cap, const int32_t* __restrict__ rows_dev, int d, SlotMap sm) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int nch = d / 8;
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    const int64_t srow = src_row(sm, row);
    float v[kMaxChunks][8];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        load8(o + srow * ldo_in + ch * 8, v[c]);
#pragma unroll
        for (int e = 0; e < 8; ++e) s += v[c][e];
      }
    }
    const float mean = warp_sum(s) / d;
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      if (lane + 32 * c < nch) {
#pragma unroll
        for (int e = 0; e < 8; ++e) { float t = v[c][e] - mean; q += t * t; }
      }
    }
    const float rstd = 1.0f / sqrtf(warp_sum(q) / d + eps);
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float g[8], b[8], uu[8], r[8];
        load8(gamma + ch * 8, g);
        load8(beta + ch * 8, b);
        load8(u + srow * ldu + ch * 8, uu);
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = ((v[c][e] - mean) * rstd * g[e] + b[e]) * uu[e];
        store8(out + (int64_t)row * ldout + ch * 8, r);
      }
    }
    if (lane == 0) {
      if (mean_out) mean_out[row] = mean;
      if (rstd_out) rstd_out[row] = rstd;
    }
  }
}

// per-block column partials of dgamma/dbeta reduced through shared memory,
// then one atomic per column per block
__device__ __forceinline__ void flush_affine_grads(float (*pg)[8], float (*pb)[8], int nch, float* dgamma,
                                                   float* dbeta, float* red /* smem [2][1024] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 2 * 1024; i += blockDim.x) red[i] = 0.f;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        atomicAdd(&red[ch * 8 + e], pg[c][e]);
        atomicAdd(&red[1024 + ch * 8 + e], pb[c][e]);
      }
    }
  }
  (void)warp;
  __syncthreads();
  for (int i = threadIdx.x; i < nch * 8; i += blockDim.x) {
    if (dgamma) atomicAdd(&dgamma[i], red[i]);
    if (dbeta) atomicAdd(&dbeta[i], red[1024 + i]);
  }
}

// backward of g = (LN(o) gamma + beta) * u for d_o and the affine gradients
template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32)
ln_gate_bwd_kernel(const T* __restrict__ o, int64_t ldo_in, const T* __restrict__ u, int64_t ldu,
                   const float* __restrict__ gamma, const float* __restrict__ mean_in,
                   const float* __restrict__ rstd_in, const T* __restrict__ dg, int64_t lddg,
                   T* __restrict__ d_o, int64_t ld_do, float* __restrict__ dgamma, float* __restrict__ dbeta,
                   int rows_cap, const int32_t* __restrict__ rows_dev, int d) {
  __shared__ float red[2 * 1024];
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int nch = d / 8;
  float pg[kMaxChunks][8], pb[kMaxChunks][8];
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) { pg[c][e] = 0.f; pb[c][e] = 0.f; }
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    const float mean = mean_in[row], rstd = rstd_in[row];
    float xh[kMaxChunks][8], dxh[kMaxChunks][8];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float ov[8], uu[8], gg[8], g[8];
        load8(o + (int64_t)row * ldo_in + ch * 8, ov);
        load8(u + (int64_t)row * ldu + ch * 8, uu);
        load8(dg + (int64_t)row * lddg + ch * 8, gg);
        load8(gamma + ch * 8, g);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          xh[c][e] = (ov[e] - mean) * rstd;
          const float don = gg[e] * uu[e];
          pg[c][e] += don * xh[c][e];
          pb[c][e] += don;
          dxh[c][e] = don * g[e];
          s1 += dxh[c][e];
          s2 += dxh[c][e] * xh[c][e];
        }
      }
    }
    s1 = warp_sum(s1) / d;
    s2 = warp_sum(s2) / d;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = rstd * (dxh[c][e] - s1 - xh[c][e] * s2);
        store8(d_o + (int64_t)row * ld_do + ch * 8, r);
      }
    }
  }
  flush_affine_grads(pg, pb, nch, dgamma, dbeta, red);
}

// du = dg * LN(o) (separate pass keeps the register footprint of the kernel above small)
template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32)
ln_gate_du_kernel(const T* __restrict__ o, int64_t ldo_in, const float* __restrict__ gamma,
                  const float* __restrict__ beta, const float* __restrict__ mean_in,
                  const float* __restrict__ rstd_in, const T* __restrict__ dg, int64_t lddg,
                  T* __restrict__ du, int64_t lddu, int rows_cap, const int32_t* __restrict__ rows_dev, int d) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int nch = d / 8;
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    const float mean = mean_in[row], rstd = rstd_in[row];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float ov[8], gg[8], g[8], b[8], r[8];
        load8(o + (int64_t)row * ldo_in + ch * 8, ov);
        load8(dg + (int64_t)row * lddg + ch * 8, gg);
        load8(gamma + ch * 8, g);
        load8(beta + ch * 8, b);
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = gg[e] * ((ov[e] - mean) * rstd * g[e] + b[e]);
        store8(du + (int64_t)row * lddu + ch * 8, r);
      }
    }
  }
}

// dx = dres + rstd * (dxh*gamma - mean(dxh*gamma) - xhat * mean(dxh*gamma*xhat)), dxh fp32
template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32)
ln_bwd_kernel(const T* __restrict__ x, int64_t ldx, const float* __restrict__ gamma,
              const float* __restrict__ mean_in, const float* __restrict__ rstd_in,
              const float* __restrict__ dxhat, int64_t lddxh, const T* __restrict__ dres, int64_t lddres,
              T* __restrict__ dx, int64_t lddx, float* __restrict__ dgamma, float* __restrict__ dbeta,
              int rows_cap, const int32_t* __restrict__ rows_dev, int d) {
  __shared__ float red[2 * 1024];
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int nch = d / 8;
  float pg[kMaxChunks][8], pb[kMaxChunks][8];
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) { pg[c][e] = 0.f; pb[c][e] = 0.f; }
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    const float mean = mean_in[row], rstd = rstd_in[row];
    float xh[kMaxChunks][8], dg[kMaxChunks][8];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float xv[8], dv8[8], g[8];
        load8(x + (int64_t)row * ldx + ch * 8, xv);
        load8(dxhat + (int64_t)row * lddxh + ch * 8, dv8);
        load8(gamma + ch * 8, g);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          xh[c][e] = (xv[e] - mean) * rstd;
          pg[c][e] += dv8[e] * xh[c][e];
          pb[c][e] += dv8[e];
          dg[c][e] = dv8[e] * g[e];
          s1 += dg[c][e];
          s2 += dg[c][e] * xh[c][e];
        }
      }
    }
    s1 = warp_sum(s1) / d;
    s2 = warp_sum(s2) / d;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nch) {
        float r[8], rs[8];
        load8(dres + (int64_t)row * lddres + ch * 8, rs);
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = rs[e] + rstd * (dg[c][e] - s1 - xh[c][e] * s2);
        store8(dx + (int64_t)row * lddx + ch * 8, r);
      }
    }
  }
  flush_affine_grads(pg, pb, nch, dgamma, dbeta, red);
}

// (columns [q_col0, q_col0 + q_cols) take da from the fp32 matrix dq, row stride ldq,
// when dq is given)
template <typename T>
__global__ void silu_bwd_kernel(const T* __restrict__ da, const T* __restrict__ z, T* __restrict__ dz,
                                int64_t ld, int rows_cap, const int32_t* __restrict__ rows_dev, int cols,
                                const float* __restrict__ dq, int64_t ldq, int q_col0, int q_cols) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int nch = cols / 8;
  const int64_t total = (int64_t)rows * nch;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / nch;
    const int ch = (int)(e % nch);
    float a[8], zz[8], r[8];
    if (dq != nullptr && ch * 8 >= q_col0 && ch * 8 < q_col0 + q_cols) load8(dq + row * ldq + (ch * 8 - q_col0), a);
    else load8(da + row * ld + ch * 8, a);
    load8(z + row * ld + ch * 8, zz);
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = a[i] * silu_grad_f(zz[i]);
    store8(dz + row * ld + ch * 8, r);
  }
}

// column sums: block handles a chunk of rows for 256 columns (one column per thread)
template <typename T>
__global__ void col_sum_kernel(const T* __restrict__ a, int64_t lda, int rows_cap,
                               const int32_t* __restrict__ rows_dev, int cols, float* __restrict__ out) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  if (col >= cols) return;
  const int chunk = (rows + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * chunk, r1 = min(rows, r0 + chunk);
  // four independent partial sums keep several loads in flight per thread
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  int r = r0;
  for (; r + 3 < r1; r += 4) {
    s0 += Elem<T>::to_f(a[(int64_t)r * lda + col]);
    s1 += Elem<T>::to_f(a[(int64_t)(r + 1) * lda + col]);
    s2 += Elem<T>::to_f(a[(int64_t)(r + 2) * lda + col]);
    s3 += Elem<T>::to_f(a[(int64_t)(r + 3) * lda + col]);
  }
  for (; r < r1; ++r) s0 += Elem<T>::to_f(a[(int64_t)r * lda + col]);
  if (r1 > r0) atomicAdd(&out[col], (s0 + s1) + (s2 + s3));
}

__global__ void gather_rows_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst, int64_t words,
                                   const int32_t* __restrict__ index, const int32_t* __restrict__ count,
                                   int capacity) {
  const int n = min(*count, capacity);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < (int64_t)n * words;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / words, w = e % words;
    dst[r * words + w] = src[(int64_t)index[r] * words + w];
  }
}

// rows of 16-byte multiples: a warp per row, 16-byte vectors, no division per element
__global__ void gather_rows_vec_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int vecs,
                                       const int32_t* __restrict__ index, const int32_t* __restrict__ count,
                                       int capacity) {
  const int n = min(*count, capacity);
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += gridDim.x * wpb) {
    const uint4* s = src + (int64_t)index[r] * vecs;
    uint4* d = dst + (int64_t)r * vecs;
    for (int w = lane; w < vecs; w += 32) d[w] = s[w];
  }
}

// ---------------------------------------------------------------- Stochastic Length
constexpr int kSlThreads = 1024;

__global__ void __launch_bounds__(kSlThreads)
sl_offsets_kernel(int B, int T, const int32_t* __restrict__ offs, const uint32_t* __restrict__ coins, int max_len,
                  uint32_t prob, int32_t* __restrict__ out_offs, int32_t* __restrict__ status) {
  using Scan = cub::BlockScan<int, kSlThreads>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int carry;
  if (threadIdx.x == 0) {
    carry = 0;
    if (offs[0] != 0 || offs[B] > T) set_status(status, HSTU_ERR_BAD_OFFSETS);
  }
  __syncthreads();
  for (int base = 0; base < B; base += kSlThreads) {
    const int s = base + threadIdx.x;
    int len = 0;
    if (s < B) {
      const int n = max(0, offs[s + 1] - offs[s]);
      len = (n > max_len && coins[s] < prob) ? max_len : n;
    }
    int ex, tot;
    Scan(tmp).ExclusiveSum(len, ex, tot);
    if (s < B) out_offs[s] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) out_offs[B] = carry;
}

// one block per sequence: keep the max_len smallest (key, index) pairs in index order
__global__ void __launch_bounds__(kSlThreads)
sl_select_kernel(int B, const int32_t* __restrict__ offs, const uint32_t* __restrict__ coins,
                 const uint32_t* __restrict__ keys, int max_len, uint32_t prob,
                 const int32_t* __restrict__ out_offs, int32_t* __restrict__ out_index) {
  using Scan = cub::BlockScan<int, kSlThreads>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int red[32];
  __shared__ int carry;
  const int s = blockIdx.x;
  if (s >= B) return;
  const int a = offs[s], n = max(0, offs[s + 1] - a);
  const int dst0 = out_offs[s];
  const bool sub = n > max_len && coins[s] < prob;
  if (!sub) {
    for (int i = threadIdx.x; i < n; i += kSlThreads) out_index[dst0 + i] = a + i;
    return;
  }
  // composite value (key << 32 | local index) is unique; find the max_len-th smallest by
  // deciding its bits from the top: prefix search over 64 bits
  uint64_t prefix = 0;
  int need = max_len;  // rank (1-based) of the threshold among values with the current prefix
  for (int bit = 63; bit >= 0; --bit) {
    // count values whose bits above `bit` equal prefix's and whose `bit` is 0
    const uint64_t hi_mask = bit == 63 ? 0ull : (~0ull << (bit + 1));
    int cnt = 0;
    for (int i = threadIdx.x; i < n; i += kSlThreads) {
      const uint64_t v = ((uint64_t)keys[a + i] << 32) | (uint32_t)i;
      if ((v & hi_mask) == (prefix & hi_mask) && !((v >> bit) & 1ull)) ++cnt;
    }
    // block reduce
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = cnt;
    __syncthreads();
    if (threadIdx.x < 32) {
      int t = red[threadIdx.x];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    const int zeros = red[0];
    __syncthreads();
    if (need > zeros) { prefix |= (1ull << bit); need -= zeros; }
  }
  // prefix is the max_len-th smallest value: keep v <= prefix, in index order
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kSlThreads) {
    const int i = base + threadIdx.x;
    int keep = 0;
    if (i < n) keep = ((((uint64_t)keys[a + i] << 32) | (uint32_t)i) <= prefix) ? 1 : 0;
    int ex, tot;
    Scan(tmp).ExclusiveSum(keep, ex, tot);
    if (keep) out_index[dst0 + carry + ex] = a + i;
    __syncthreads();
    if (threadIdx.x == 0) carry += tot;
    __syncthreads();
  }
}

// ---------------------------------------------------------------- M-FALCON output rows
template <typename T>
__global__ void mfalcon_scatter_kernel(const T* __restrict__ y, int d, const int32_t* __restrict__ row_map,
                                       const int32_t* __restrict__ total_rows, int cap, T* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int total = total_rows ? min(*total_rows, cap) : cap;
  for (int r = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < total; r += gridDim.x * (blockDim.x / 32)) {
    const int dst = row_map[r];
    if (dst < 0) continue;
    for (int e = lane * 8; e < d; e += 32 * 8) {
      float v[8];
      load8(y + (int64_t)r * d + e, v);
      store8(out + (int64_t)dst * d + e, v);
    }
  }
}

// ---------------------------------------------------------------- M-FALCON with a history cache
// Slot layout: user u's rows sit at a fixed place across microbatches,
// [history_u ; a slot of bm candidate rows], from row hist_offs[u] + u * bm; the
// compact candidate layout has row c = u * bm + j for slot row j of user u.
__global__ void mfalcon_slot_offsets_kernel(int U, int bm, const int32_t* __restrict__ hist_offs,
                                            int32_t* __restrict__ offs, int32_t* __restrict__ nt) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u <= U; u += gridDim.x * blockDim.x) {
    offs[u] = hist_offs[u] + u * bm;
    if (u < U) nt[u] = bm;
  }
}

// Microbatch mb in the slot layout, one warp per row: candidate j of user u is
// candidate mb * bm + j of that user, or a zero row (timestamp of the user's last
// history token, else of its last candidate, else 0) past the user's candidates.  With with_hist the history
// rows are written too (x and timestamps) and the rows walked are all slot-layout
// rows; otherwise only the candidate rows.  x_slot and x_c may each be null.
template <typename T>
__global__ void mfalcon_slot_pack_kernel(int U, int mb, int bm, const int32_t* __restrict__ hist_offs,
                                         const T* __restrict__ hist_x, const int64_t* __restrict__ hist_ts,
                                         const int32_t* __restrict__ cand_offs, const T* __restrict__ cand_x,
                                         const int64_t* __restrict__ cand_ts, int d, int with_hist, int cap,
                                         T* __restrict__ x_slot, int64_t* __restrict__ ts_slot, T* __restrict__ x_c,
                                         int32_t* __restrict__ cand_dst) {
  const int lane = threadIdx.x & 31;
  const int total = with_hist ? hist_offs[U] + U * bm : U * bm;   // rows walked
  for (int r = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < total; r += gridDim.x * (blockDim.x / 32)) {
    int u, j;          // user, and slot row (j < 0: history row -j - 1)
    if (with_hist) {
      int lo = 0, hi = U;  // slot-layout start of user lo <= r < start of user hi
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (hist_offs[mid] + mid * bm <= r) lo = mid; else hi = mid;
      }
      u = lo;
      const int l = r - (hist_offs[u] + u * bm);
      const int n = hist_offs[u + 1] - hist_offs[u];
      j = l < n ? -l - 1 : l - n;
    } else {
      u = r / bm;
      j = r - u * bm;
    }
    const T* src = nullptr;
    int64_t ts = 0;
    int slot_row;
    if (j < 0) {
      const int h = hist_offs[u] + (-j - 1);
      src = hist_x + (int64_t)h * d;
      ts = hist_ts[h];
      slot_row = r;
    } else {
      const int m = cand_offs[u + 1] - cand_offs[u];
      const int ci = mb * bm + j;
      slot_row = hist_offs[u + 1] + u * bm + j;
      if (ci < m) {
        src = cand_x + (int64_t)(cand_offs[u] + ci) * d;
        ts = cand_ts[cand_offs[u] + ci];
      } else if (hist_offs[u + 1] > hist_offs[u]) {
        ts = hist_ts[hist_offs[u + 1] - 1];
      } else if (m > 0) {
        ts = cand_ts[cand_offs[u + 1] - 1];   // no history: keep the sequence's offsets small
      }
      if (lane == 0) cand_dst[u * bm + j] = ci < m ? cand_offs[u] + ci : -1;
    }
    if (slot_row >= cap) continue;   // offsets beyond the sizes the workspace was made for
    if (x_slot || (x_c && j >= 0))
      for (int e = lane * 8; e < d; e += 32 * 8) {
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (src) load8(src + e, v);
        if (x_slot) store8(x_slot + (int64_t)slot_row * d + e, v);
        if (x_c && j >= 0) store8(x_c + (int64_t)(u * bm + j) * d + e, v);
      }
    if (lane == 0) ts_slot[slot_row] = ts;
  }
}

// Rows between the compact candidate layout and the slot layout: `words`
// 16-byte words of each row (to_slot: compact -> slot, else slot -> compact);
// one warp per row.
__global__ void mfalcon_slot_rows_kernel(int U, int bm, const int32_t* __restrict__ hist_offs,
                                         const uint4* __restrict__ src, int64_t lds, uint4* __restrict__ dst,
                                         int64_t ldd, int words, int to_slot, int cap) {
  const int lane = threadIdx.x & 31;
  const int rows = U * bm;
  for (int c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); c < rows; c += gridDim.x * (blockDim.x / 32)) {
    const int u = c / bm, j = c - u * bm;
    const int64_t slot_row = hist_offs[u + 1] + (int64_t)u * bm + j;
    if (slot_row >= cap) continue;   // offsets beyond the sizes the workspace was made for
    const uint4* s_row = src + (to_slot ? (int64_t)c * lds : slot_row * lds);
    uint4* d_row = dst + (to_slot ? slot_row * ldd : (int64_t)c * ldd);
    for (int w = lane; w < words; w += 32) d_row[w] = s_row[w];
  }
}

// offsets of sequences [s0, s0 + nb] rebased to start at row 0
__global__ void rebase_offsets_kernel(const int32_t* __restrict__ offs, int s0, int nb, int32_t* __restrict__ out) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= nb; i += gridDim.x * blockDim.x)
    out[i] = offs[s0 + i] - offs[s0];
}

template <typename TS, typename TD>
__global__ void convert_rows_kernel(const TS* __restrict__ src, int64_t lds, TD* __restrict__ dst, int64_t ldd,
                                    int cols, int rows_cap, const int32_t* __restrict__ rows_dev, int pad_multiple) {
  const int rows = rows_of(rows_cap, rows_dev);
  int pad_end = ((rows + pad_multiple - 1) / pad_multiple) * pad_multiple;
  pad_end = pad_end < rows_cap ? pad_end : rows_cap;
  const int nch = cols / 8;
  const int64_t total = (int64_t)pad_end * nch;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / nch;
    const int ch = (int)(e % nch);
    float v[8];
    if (r < rows) {
      load8(src + r * lds + ch * 8, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    store8(dst + r * ldd + ch * 8, v);
  }
}

__global__ void zero_tail_rows_kernel(uint32_t* __restrict__ buf, int64_t ld_words, int64_t row_words, int rows_cap,
                                      const int32_t* __restrict__ rows_dev, int multiple) {
  const int rows = rows_of(rows_cap, rows_dev);
  int end = ((rows + multiple - 1) / multiple) * multiple;
  end = end < rows_cap ? end : rows_cap;
  const int64_t total = (int64_t)(end - rows) * row_words;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x)
    buf[(rows + e / row_words) * ld_words + e % row_words] = 0u;
}


// ---------------------------------------------------------------- LayerNorm, d = 256 * NCH
// One warp per row as above, but gamma and beta stay in registers for all of the
// warp's rows and the next row is loaded (as raw 16-byte vectors) while the
// current one is normalised, so each warp keeps two rows of loads in flight.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void get(float v[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void load(const float* p) {
    a = *reinterpret_cast<const float4*>(p);
    b = *reinterpret_cast<const float4*>(p + 4);
  }
  __device__ __forceinline__ void get(float v[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

template <int NCH>
__device__ __forceinline__ void row_stats(const float (&v)[NCH][8], float eps, float& mean, float& rstd) {
  constexpr float inv_d = 1.0f / (256 * NCH);
  float sm = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) sm += v[c][e];
  mean = warp_sum(sm) * inv_d;
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) { const float t = v[c][e] - mean; q = fmaf(t, t, q); }
  rstd = 1.0f / sqrtf(warp_sum(q) * inv_d + eps);
}

template <typename T, typename TO, int NCH>
__global__ void __launch_bounds__(kRowWarps * 32, NCH > 2 ? 1 : (sizeof(T) == 2 ? 3 : 2))   // registers for two rows in flight
layer_norm_rows(const T* __restrict__ x, int64_t ldx, const float* __restrict__ gamma, const float* __restrict__ beta,
                float eps, TO* __restrict__ out, int64_t ldo, float* __restrict__ mean_out,
                float* __restrict__ rstd_out, int rows_cap, const int32_t* __restrict__ rows_dev,
                const int32_t* __restrict__ in_map) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * kRowWarps;
  float g[NCH][8], b[NCH][8];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    load8(gamma + (lane + 32 * c) * 8, g[c]);
    load8(beta + (lane + 32 * c) * 8, b[c]);
  }
  // two rows in flight ahead of the one being normalised: the warp's rows
  // alternate between two register buffers
  auto fetch = [&](Raw8<T> (&r)[NCH], int row) {
    if (row < rows) {
      const int src = in_map ? in_map[row] : row;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        if (src >= 0) r[c].load(x + (int64_t)src * ldx + (lane + 32 * c) * 8);
        else r[c].zero();
      }
    }
  };
  auto normalise = [&](Raw8<T> (&r)[NCH], int row) {
    float v[NCH][8];
#pragma unroll
    for (int c = 0; c < NCH; ++c) r[c].get(v[c]);
    fetch(r, row + 2 * stride);   // the buffer's next row, issued before the arithmetic
    float mean, rstd;
    row_stats<NCH>(v, eps, mean, rstd);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = fmaf((v[c][e] - mean) * rstd, g[c][e], b[c][e]);
      store8(out + (int64_t)row * ldo + (lane + 32 * c) * 8, o);
    }
    if (lane == 0) {
      if (mean_out) mean_out[row] = mean;
      if (rstd_out) rstd_out[row] = rstd;
    }
  };
  int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  Raw8<T> r0[NCH], r1[NCH];
  fetch(r0, row);
  fetch(r1, row + stride);
  for (; row < rows; row += 2 * stride) {
    normalise(r0, row);
    if (row + stride >= rows) break;
    normalise(r1, row + stride);
  }
}

// g = LN(o) * u, d = 256 * NCH
template <typename T, int NCH>
__global__ void __launch_bounds__(kRowWarps * 32, sizeof(T) == 2 && NCH <= 2 ? 2 : 1)   // two rows in flight
ln_gate_rows(const T* __restrict__ o, int64_t ldo_in, const T* __restrict__ u, int64_t ldu,
             const float* __restrict__ gamma, const float* __restrict__ beta, float eps, T* __restrict__ out,
             int64_t ldout, float* __restrict__ mean_out, float* __restrict__ rstd_out, int rows_cap,
             const int32_t* __restrict__ rows_dev, SlotMap sm) {
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * kRowWarps;
  // two rows of O and U in flight ahead of the one being normalised (two register
  // buffers, as in layer_norm_rows); gamma and beta come from L1 per row
  auto fetch = [&](Raw8<T> (&ro)[NCH], Raw8<T> (&ru)[NCH], int row) {
    if (row < rows) {
      const int64_t sr = src_row(sm, row);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        ro[c].load(o + sr * ldo_in + (lane + 32 * c) * 8);
        ru[c].load(u + sr * ldu + (lane + 32 * c) * 8);
      }
    }
  };
  auto gate = [&](Raw8<T> (&ro)[NCH], Raw8<T> (&ru)[NCH], int row) {
    float v[NCH][8], uu[NCH][8];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      ro[c].get(v[c]);
      ru[c].get(uu[c]);
    }
    fetch(ro, ru, row + 2 * stride);   // the buffers' next row, issued before the arithmetic
    float mean, rstd;
    row_stats<NCH>(v, eps, mean, rstd);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      float g[8], b[8], r[8];
      load8(gamma + (lane + 32 * c) * 8, g);
      load8(beta + (lane + 32 * c) * 8, b);
#pragma unroll
      for (int e = 0; e < 8; ++e) r[e] = fmaf((v[c][e] - mean) * rstd, g[e], b[e]) * uu[c][e];
      store8(out + (int64_t)row * ldout + (lane + 32 * c) * 8, r);
    }
    if (lane == 0) {
      if (mean_out) mean_out[row] = mean;
      if (rstd_out) rstd_out[row] = rstd;
    }
  };
  int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  Raw8<T> o0[NCH], u0[NCH], o1[NCH], u1[NCH];
  fetch(o0, u0, row);
  fetch(o1, u1, row + stride);
  for (; row < rows; row += 2 * stride) {
    gate(o0, u0, row);
    if (row + stride >= rows) break;
    gate(o1, u1, row + stride);
  }
}

// per-block column partials of dgamma/dbeta for d = 256 * NCH: summed through
// shared memory (stored column-chunk-minor, so a warp's 32 lanes hit 32 banks),
// then one atomic per column per block
template <int NCH>
__device__ __forceinline__ void flush_affine_grads_n(const float (&pg)[NCH][8], const float (&pb)[NCH][8],
                                                     float* dgamma, float* dbeta, float* red /* [2][256 NCH] */) {
  constexpr int D = 256 * NCH, NC = 32 * NCH;   // columns, 8-column chunks
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 2 * D; i += blockDim.x) red[i] = 0.f;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      atomicAdd(&red[e * NC + lane + 32 * c], pg[c][e]);
      atomicAdd(&red[D + e * NC + lane + 32 * c], pb[c][e]);
    }
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const int k = (i & 7) * NC + (i >> 3);   // column i = chunk (i / 8), element (i % 8)
    if (dgamma) atomicAdd(&dgamma[i], red[k]);
    if (dbeta) atomicAdd(&dbeta[i], red[D + k]);
  }
}

// LayerNorm1 backward for d = 256 * NCH: dx = dres + rstd (dxh gamma - mean(dxh gamma)
// - xhat mean(dxh gamma xhat)) with the dgamma/dbeta partials.  A warp takes a row
// at a time and loads its three inputs (x, dxhat, dres) before any arithmetic, so
// they are in flight together; gamma is read from L1 per row (registers go to the
// partial sums).
template <typename T, int NCH>
__global__ void __launch_bounds__(kRowWarps * 32, NCH > 2 ? 1 : 2)
ln_bwd_rows(const T* __restrict__ x, int64_t ldx, const float* __restrict__ gamma,
            const float* __restrict__ mean_in, const float* __restrict__ rstd_in, const float* __restrict__ dxhat,
            int64_t lddxh, const T* __restrict__ dres, int64_t lddres, T* __restrict__ dx, int64_t lddx,
            float* __restrict__ dgamma, float* __restrict__ dbeta, int rows_cap, const int32_t* __restrict__ rows_dev) {
  __shared__ float red[2 * 256 * NCH];
  constexpr int D = 256 * NCH;
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  float pg[NCH][8], pb[NCH][8];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) { pg[c][e] = 0.f; pb[c][e] = 0.f; }
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    Raw8<T> xr[NCH], rr[NCH];
    float dv[NCH][8];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      xr[c].load(x + (int64_t)row * ldx + col);
      load8(dxhat + (int64_t)row * lddxh + col, dv[c]);
      rr[c].load(dres + (int64_t)row * lddres + col);
    }
    const float mean = mean_in[row], rstd = rstd_in[row];
    float xh[NCH][8];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      float g[8];
      load8(gamma + (lane + 32 * c) * 8, g);
      xr[c].get(xh[c]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        xh[c][e] = (xh[c][e] - mean) * rstd;
        pg[c][e] += dv[c][e] * xh[c][e];
        pb[c][e] += dv[c][e];
        dv[c][e] *= g[e];
        s1 += dv[c][e];
        s2 += dv[c][e] * xh[c][e];
      }
    }
    s1 = warp_sum(s1) / D;
    s2 = warp_sum(s2) / D;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      float r[8];
      rr[c].get(r);
#pragma unroll
      for (int e = 0; e < 8; ++e) r[e] += rstd * (dv[c][e] - s1 - xh[c][e] * s2);
      store8(dx + (int64_t)row * lddx + (lane + 32 * c) * 8, r);
    }
  }
  flush_affine_grads_n<NCH>(pg, pb, dgamma, dbeta, red);
}

// Backward of g = (LN2(o) gamma + beta) * u for d = 256 * NCH in one pass: d_o,
// du = dg (LN2(o) gamma + beta) and the dgamma/dbeta partials.  A warp loads a
// row's o, u and dg before any arithmetic; gamma and beta are read from L1.
template <typename T, int NCH>
__global__ void __launch_bounds__(kRowWarps * 32, NCH > 2 ? 1 : 2)
ln_gate_bwd_rows(const T* __restrict__ o, int64_t ldo_in, const T* __restrict__ u, int64_t ldu,
                 const float* __restrict__ gamma, const float* __restrict__ beta, const float* __restrict__ mean_in,
                 const float* __restrict__ rstd_in, const T* __restrict__ dg, int64_t lddg, T* __restrict__ d_o,
                 int64_t ld_do, T* __restrict__ du, int64_t lddu, float* __restrict__ dgamma,
                 float* __restrict__ dbeta, int rows_cap, const int32_t* __restrict__ rows_dev) {
  __shared__ float red[2 * 256 * NCH];
  constexpr int D = 256 * NCH;
  const int rows = rows_of(rows_cap, rows_dev);
  const int lane = threadIdx.x & 31;
  float pg[NCH][8], pb[NCH][8];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) { pg[c][e] = 0.f; pb[c][e] = 0.f; }
  for (int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < rows; row += gridDim.x * kRowWarps) {
    Raw8<T> orw[NCH], urw[NCH], grw[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      orw[c].load(o + (int64_t)row * ldo_in + col);
      urw[c].load(u + (int64_t)row * ldu + col);
      grw[c].load(dg + (int64_t)row * lddg + col);
    }
    const float mean = mean_in[row], rstd = rstd_in[row];
    float xh[NCH][8], dxh[NCH][8];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      float uu[8], gg[8], g[8], b[8], r[8];
      orw[c].get(xh[c]);
      urw[c].get(uu);
      grw[c].get(gg);
      load8(gamma + col, g);
      load8(beta + col, b);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        xh[c][e] = (xh[c][e] - mean) * rstd;
        r[e] = gg[e] * (xh[c][e] * g[e] + b[e]);
        const float don = gg[e] * uu[e];
        pg[c][e] += don * xh[c][e];
        pb[c][e] += don;
        dxh[c][e] = don * g[e];
        s1 += dxh[c][e];
        s2 += dxh[c][e] * xh[c][e];
      }
      store8(du + (int64_t)row * lddu + col, r);
    }
    s1 = warp_sum(s1) / D;
    s2 = warp_sum(s2) / D;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      float r[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) r[e] = rstd * (dxh[c][e] - s1 - xh[c][e] * s2);
      store8(d_o + (int64_t)row * ld_do + (lane + 32 * c) * 8, r);
    }
  }
  flush_affine_grads_n<NCH>(pg, pb, dgamma, dbeta, red);
}

// Thread layout of the column-sum passes below: a block's 256 threads take cpr =
// min(256, cols / 8) 8-column vectors of a row and rpi = 256 / cpr rows at a time
// (narrow matrices keep every thread busy); with 256 vectors a row, block y takes
// the columns [2048 y, 2048 y + 2048).  Thread (sub, vector) writes its column sums
// to partial row x rpi + sub.
struct ColSumLayout {
  int cpr, rpi, sub, col;
  __host__ __device__ static int vectors(int cols) { return (cols + 7) / 8 < 256 ? (cols + 7) / 8 : 256; }
  __device__ explicit ColSumLayout(int cols) {
    cpr = vectors(cols);
    rpi = 256 / cpr;
    sub = threadIdx.x / cpr;
    col = (blockIdx.y * 256 + threadIdx.x % cpr) * 8;
  }
};

// dz = da * SiLU'(z) with the column sums of dz (as stored) in one pass: block x
// takes the x-th range of rows, two rows a thread in flight (layout above), and
// writes its column sums to the partial rows; col_partials_reduce adds them up.
template <typename T>
__global__ void __launch_bounds__(256)
silu_bwd_colsum_kernel(const T* __restrict__ da, const T* __restrict__ z, T* __restrict__ dz, int64_t ld,
                       int rows_cap, const int32_t* __restrict__ rows_dev, int cols, const float* __restrict__ dq,
                       int64_t ldq, int q_col0, int q_cols, float* __restrict__ part) {
  const int rows = rows_of(rows_cap, rows_dev);
  const ColSumLayout L(cols);
  if (L.sub >= L.rpi) return;
  const int col = L.col;
  if (col >= cols) return;
  const bool from_q = dq != nullptr && col >= q_col0 && col < q_col0 + q_cols;
  const int chunk = (rows + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * chunk, r1 = min(rows, r0 + chunk);
  float s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = 0.f;
  auto load_a = [&](int row, float (&a)[8]) {
    if (from_q) load8(dq + (int64_t)row * ldq + (col - q_col0), a);
    else load8(da + (int64_t)row * ld + col, a);
  };
  auto finish = [&](int row, const float (&a)[8], const float (&zz)[8]) {
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = a[i] * silu_grad_f(zz[i]);
    store8(dz + (int64_t)row * ld + col, r);
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] += Elem<T>::to_f(Elem<T>::from_f(r[i]));   // the value stored
  };
  int row = r0 + L.sub;
  for (; row + L.rpi < r1; row += 2 * L.rpi) {
    float a0[8], z0[8], a1[8], z1[8];
    load_a(row, a0);
    load8(z + (int64_t)row * ld + col, z0);
    load_a(row + L.rpi, a1);
    load8(z + (int64_t)(row + L.rpi) * ld + col, z1);
    finish(row, a0, z0);
    finish(row + L.rpi, a1, z1);
  }
  if (row < r1) {
    float a0[8], z0[8];
    load_a(row, a0);
    load8(z + (int64_t)row * ld + col, z0);
    finish(row, a0, z0);
  }
  float* pp = part + ((int64_t)blockIdx.x * L.rpi + L.sub) * cols + col;
  *reinterpret_cast<float4*>(pp) = make_float4(s[0], s[1], s[2], s[3]);
  *reinterpret_cast<float4*>(pp + 4) = make_float4(s[4], s[5], s[6], s[7]);
}

// out[c] = sum over b < nb of part[b][c]: block (x, y) adds partials
// [y nb / gridDim.y, (y + 1) nb / gridDim.y) of 256 columns (about 8 per thread);
// out starts at zero
__global__ void col_partials_reduce_kernel(const float* __restrict__ part, int nb, int cols, float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int b0 = (int)((int64_t)nb * blockIdx.y / gridDim.y), b1 = (int)((int64_t)nb * (blockIdx.y + 1) / gridDim.y);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  int b = b0;
  for (; b + 3 < b1; b += 4) {
    s0 += part[(int64_t)b * cols + c];
    s1 += part[(int64_t)(b + 1) * cols + c];
    s2 += part[(int64_t)(b + 2) * cols + c];
    s3 += part[(int64_t)(b + 3) * cols + c];
  }
  for (; b < b1; ++b) s0 += part[(int64_t)b * cols + c];
  if (b1 > b0) atomicAdd(&out[c], (s0 + s1) + (s2 + s3));
}

// dst = src (converted) for rows < *rows_dev and zero up to the next multiple of
// pad_multiple (at most rows_cap), with the column sums of src in the same pass:
// blocks laid out as in silu_bwd_colsum_kernel
template <typename TS, typename TD>
__global__ void __launch_bounds__(256)
convert_rows_colsum_kernel(const TS* __restrict__ src, int64_t lds, TD* __restrict__ dst, int64_t ldd, int cols,
                           int rows_cap, const int32_t* __restrict__ rows_dev, int pad_multiple,
                           float* __restrict__ part) {
  const int rows = rows_of(rows_cap, rows_dev);
  int pad_end = ((rows + pad_multiple - 1) / pad_multiple) * pad_multiple;
  pad_end = pad_end < rows_cap ? pad_end : rows_cap;
  const ColSumLayout L(cols);
  if (L.sub >= L.rpi) return;
  const int col = L.col;
  if (col >= cols) return;
  const int chunk = (pad_end + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * chunk, r1 = min(pad_end, r0 + chunk);
  float s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = 0.f;
  auto load = [&](int row, float (&v)[8]) {
    if (row < rows) {
      load8(src + (int64_t)row * lds + col, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
  };
  auto finish = [&](int row, const float (&v)[8]) {
    store8(dst + (int64_t)row * ldd + col, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] += v[i];
  };
  int row = r0 + L.sub;
  for (; row + L.rpi < r1; row += 2 * L.rpi) {
    float v0[8], v1[8];
    load(row, v0);
    load(row + L.rpi, v1);
    finish(row, v0);
    finish(row + L.rpi, v1);
  }
  if (row < r1) {
    float v0[8];
    load(row, v0);
    finish(row, v0);
  }
  float* pp = part + ((int64_t)blockIdx.x * L.rpi + L.sub) * cols + col;
  *reinterpret_cast<float4*>(pp) = make_float4(s[0], s[1], s[2], s[3]);
  *reinterpret_cast<float4*>(pp + 4) = make_float4(s[4], s[5], s[6], s[7]);
}

// grid of the register-resident row kernels: the blocks that are resident at
// once (one wave), each warp walking rows with a grid-sized stride
int row_sms() {
  static const int n = [] {
    int dev = 0, c = 0;
    cudaGetDevice(&dev);
    return cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && c > 0 ? c : 148;
  }();
  return n;
}
// slices of the column-partial reduce: about 8 partials per thread
int partial_slices(int nb) { return nb >= 512 ? 64 : (nb >= 8 ? nb / 8 : 1); }
template <auto K>
int rows_grid(int rows_cap) {
  static const int occ = [] {
    int o = 0;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, K, kRowWarps * 32, 0) == cudaSuccess && o > 0 ? o : 1;
  }();
  const int g = (rows_cap + kRowWarps - 1) / kRowWarps;
  const int cap = row_sms() * occ;
  return g < 1 ? 1 : (g > cap ? cap : g);
}

template <typename T, typename TO>
cudaError_t launch_ln_rows(const T* x, int64_t ldx, const float* gamma, const float* beta, float eps, TO* out,
                           int64_t ldo, float* mean, float* rstd, int rows_cap, const int32_t* rows_dev, int d,
                           cudaStream_t st, const int32_t* in_map) {
  const int t = kRowWarps * 32;
  switch (d / 256) {
    case 1: layer_norm_rows<T, TO, 1><<<rows_grid<layer_norm_rows<T, TO, 1>>(rows_cap), t, 0, st>>>(x, ldx, gamma, beta, eps, out, ldo, mean, rstd, rows_cap, rows_dev, in_map); break;
    case 2: layer_norm_rows<T, TO, 2><<<rows_grid<layer_norm_rows<T, TO, 2>>(rows_cap), t, 0, st>>>(x, ldx, gamma, beta, eps, out, ldo, mean, rstd, rows_cap, rows_dev, in_map); break;
    case 3: layer_norm_rows<T, TO, 3><<<rows_grid<layer_norm_rows<T, TO, 3>>(rows_cap), t, 0, st>>>(x, ldx, gamma, beta, eps, out, ldo, mean, rstd, rows_cap, rows_dev, in_map); break;
    default: layer_norm_rows<T, TO, 4><<<rows_grid<layer_norm_rows<T, TO, 4>>(rows_cap), t, 0, st>>>(x, ldx, gamma, beta, eps, out, ldo, mean, rstd, rows_cap, rows_dev, in_map); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ln_gate_rows(const T* o, int64_t ldo_in, const T* u, int64_t ldu, const float* gamma,
                                const float* beta, float eps, T* out, int64_t ldout, float* mean, float* rstd,
                                int rows_cap, const int32_t* rows_dev, int d, cudaStream_t st, SlotMap sm) {
  const int t = kRowWarps * 32;
  switch (d / 256) {
    case 1: ln_gate_rows<T, 1><<<rows_grid<ln_gate_rows<T, 1>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, eps, out, ldout, mean, rstd, rows_cap, rows_dev, sm); break;
    case 2: ln_gate_rows<T, 2><<<rows_grid<ln_gate_rows<T, 2>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, eps, out, ldout, mean, rstd, rows_cap, rows_dev, sm); break;
    case 3: ln_gate_rows<T, 3><<<rows_grid<ln_gate_rows<T, 3>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, eps, out, ldout, mean, rstd, rows_cap, rows_dev, sm); break;
    default: ln_gate_rows<T, 4><<<rows_grid<ln_gate_rows<T, 4>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, eps, out, ldout, mean, rstd, rows_cap, rows_dev, sm); break;
  }
  return cudaGetLastError();
}

bool fast_rows_ok(int d, const void* a, int64_t lda, const void* b, int64_t ldb, const void* c, int64_t ldc,
                  int esize_ab, int esize_c) {
  if (d % 256 || d / 256 < 1 || d / 256 > 4) return false;
  auto al = [](const void* p) { return ((uintptr_t)p & 15) == 0; };
  if (!al(a) || !al(c) || (b && !al(b))) return false;
  if ((lda * esize_ab) % 16 || (ldc * esize_c) % 16 || (b && (ldb * esize_ab) % 16)) return false;
  return true;
}

int row_grid(int rows_cap) {
  int g = (rows_cap + kRowWarps - 1) / kRowWarps;
  return g < 1 ? 1 : (g > 148 * 16 ? 148 * 16 : g);
}

}  // namespace

cudaError_t launch_layer_norm(const void* x, int64_t ldx, int x_dtype, const float* gamma, const float* beta,
                              float eps, void* out, int64_t ldo, int out_dtype, float* mean, float* rstd,
                              int rows_cap, const int32_t* rows_dev, int d, cudaStream_t st, const int32_t* in_map) {
  if (rows_cap <= 0) return cudaSuccess;
  using bf = __nv_bfloat16;
  const int xs = x_dtype == HSTU_DTYPE_F32 ? 4 : 2, os = out_dtype == HSTU_DTYPE_F32 ? 4 : 2;
  if (fast_rows_ok(d, x, ldx, nullptr, 0, out, ldo, xs, os) && gamma && beta) {
    if (x_dtype == HSTU_DTYPE_F32 && out_dtype == HSTU_DTYPE_F32)
      return launch_ln_rows<float, float>((const float*)x, ldx, gamma, beta, eps, (float*)out, ldo, mean, rstd,
                                          rows_cap, rows_dev, d, st, in_map);
    if (x_dtype == HSTU_DTYPE_F32)
      return launch_ln_rows<float, bf>((const float*)x, ldx, gamma, beta, eps, (bf*)out, ldo, mean, rstd, rows_cap,
                                       rows_dev, d, st, in_map);
    if (out_dtype == HSTU_DTYPE_F32)
      return launch_ln_rows<bf, float>((const bf*)x, ldx, gamma, beta, eps, (float*)out, ldo, mean, rstd, rows_cap,
                                       rows_dev, d, st, in_map);
    return launch_ln_rows<bf, bf>((const bf*)x, ldx, gamma, beta, eps, (bf*)out, ldo, mean, rstd, rows_cap,
                                  rows_dev, d, st, in_map);
  }
  const int g = row_grid(rows_cap);
  const int t = kRowWarps * 32;
  if (x_dtype == HSTU_DTYPE_F32 && out_dtype == HSTU_DTYPE_F32)
    layer_norm_kernel<float, float><<<g, t, 0, st>>>((const float*)x, ldx, gamma, beta, eps, (float*)out, ldo, mean,
                                                     rstd, rows_cap, rows_dev, d, in_map);
  else if (x_dtype == HSTU_DTYPE_F32)
    layer_norm_kernel<float, bf><<<g, t, 0, st>>>((const float*)x, ldx, gamma, beta, eps, (bf*)out, ldo, mean, rstd,
                                                  rows_cap, rows_dev, d, in_map);
  else if (out_dtype == HSTU_DTYPE_F32)
    layer_norm_kernel<bf, float><<<g, t, 0, st>>>((const bf*)x, ldx, gamma, beta, eps, (float*)out, ldo, mean, rstd,
                                                  rows_cap, rows_dev, d, in_map);
  else
    layer_norm_kernel<bf, bf><<<g, t, 0, st>>>((const bf*)x, ldx, gamma, beta, eps, (bf*)out, ldo, mean, rstd,
                                               rows_cap, rows_dev, d, in_map);
  return cudaGetLastError();
}

cudaError_t launch_ln_gate(const void* o, int64_t ldo_in, const void* u, int64_t ldu, const float* gamma,
                           const float* beta, float eps, void* out, int64_t ldout, float* mean, float* rstd,
                           int rows_cap, const int32_t* rows_dev, int d, int dtype, cudaStream_t st,
                           const int32_t* in_slot_offs, int in_slot_bm, int in_slot_cap) {
  if (rows_cap <= 0) return cudaSuccess;
  if (in_slot_offs && (in_slot_bm < 1 || in_slot_cap < 1)) return cudaErrorInvalidValue;
  const SlotMap sm{in_slot_offs, in_slot_bm, in_slot_cap};
  const int es = dtype == HSTU_DTYPE_F32 ? 4 : 2;
  if (fast_rows_ok(d, o, ldo_in, u, ldu, out, ldout, es, es) && gamma && beta) {
    if (dtype == HSTU_DTYPE_F32)
      return launch_ln_gate_rows<float>((const float*)o, ldo_in, (const float*)u, ldu, gamma, beta, eps, (float*)out,
                                        ldout, mean, rstd, rows_cap, rows_dev, d, st, sm);
    return launch_ln_gate_rows<__nv_bfloat16>((const __nv_bfloat16*)o, ldo_in, (const __nv_bfloat16*)u, ldu, gamma,
                                              beta, eps, (__nv_bfloat16*)out, ldout, mean, rstd, rows_cap, rows_dev,
                                              d, st, sm);
  }
  const int g = row_grid(rows_cap);
  if (dtype == HSTU_DTYPE_F32)
    ln_gate_kernel<float><<<g, kRowWarps * 32, 0, st>>>((const float*)o, ldo_in, (const float*)u, ldu, gamma, beta,
                                                        eps, (float*)out, ldout, mean, rstd, rows_cap, rows_dev, d, sm);
  else
    ln_gate_kernel<__nv_bfloat16><<<g, kRowWarps * 32, 0, st>>>(
        (const __nv_bfloat16*)o, ldo_in, (const __nv_bfloat16*)u, ldu, gamma, beta, eps, (__nv_bfloat16*)out,
        ldout, mean, rstd, rows_cap, rows_dev, d, sm);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ln_gate_bwd_rows(const T* o, int64_t ldo_in, const T* u, int64_t ldu, const float* gamma,
                                    const float* beta, const float* mean, const float* rstd, const T* dg,
                                    int64_t lddg, T* d_o, int64_t ld_do, T* du, int64_t lddu, float* dgamma,
                                    float* dbeta, int rows_cap, const int32_t* rows_dev, int d, cudaStream_t st) {
  const int t = kRowWarps * 32;
  switch (d / 256) {
    case 1: ln_gate_bwd_rows<T, 1><<<rows_grid<ln_gate_bwd_rows<T, 1>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, mean, rstd, dg, lddg, d_o, ld_do, du, lddu, dgamma, dbeta, rows_cap, rows_dev); break;
    case 2: ln_gate_bwd_rows<T, 2><<<rows_grid<ln_gate_bwd_rows<T, 2>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, mean, rstd, dg, lddg, d_o, ld_do, du, lddu, dgamma, dbeta, rows_cap, rows_dev); break;
    case 3: ln_gate_bwd_rows<T, 3><<<rows_grid<ln_gate_bwd_rows<T, 3>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, mean, rstd, dg, lddg, d_o, ld_do, du, lddu, dgamma, dbeta, rows_cap, rows_dev); break;
    default: ln_gate_bwd_rows<T, 4><<<rows_grid<ln_gate_bwd_rows<T, 4>>(rows_cap), t, 0, st>>>(o, ldo_in, u, ldu, gamma, beta, mean, rstd, dg, lddg, d_o, ld_do, du, lddu, dgamma, dbeta, rows_cap, rows_dev); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ln_bwd_rows(const T* x, int64_t ldx, const float* gamma, const float* mean, const float* rstd,
                               const float* dxhat, int64_t lddxh, const T* dres, int64_t lddres, T* dx,
                               int64_t lddx, float* dgamma, float* dbeta, int rows_cap, const int32_t* rows_dev,
                               int d, cudaStream_t st) {
  const int t = kRowWarps * 32;
  switch (d / 256) {
    case 1: ln_bwd_rows<T, 1><<<rows_grid<ln_bwd_rows<T, 1>>(rows_cap), t, 0, st>>>(x, ldx, gamma, mean, rstd, dxhat, lddxh, dres, lddres, dx, lddx, dgamma, dbeta, rows_cap, rows_dev); break;
    case 2: ln_bwd_rows<T, 2><<<rows_grid<ln_bwd_rows<T, 2>>(rows_cap), t, 0, st>>>(x, ldx, gamma, mean, rstd, dxhat, lddxh, dres, lddres, dx, lddx, dgamma, dbeta, rows_cap, rows_dev); break;
    case 3: ln_bwd_rows<T, 3><<<rows_grid<ln_bwd_rows<T, 3>>(rows_cap), t, 0, st>>>(x, ldx, gamma, mean, rstd, dxhat, lddxh, dres, lddres, dx, lddx, dgamma, dbeta, rows_cap, rows_dev); break;
    default: ln_bwd_rows<T, 4><<<rows_grid<ln_bwd_rows<T, 4>>(rows_cap), t, 0, st>>>(x, ldx, gamma, mean, rstd, dxhat, lddxh, dres, lddres, dx, lddx, dgamma, dbeta, rows_cap, rows_dev); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_ln_gate_bwd(const void* o, int64_t ldo_in, const void* u, int64_t ldu, const float* gamma,
                               const float* beta, const float* mean, const float* rstd, const void* dg, int64_t lddg,
                               void* d_o, int64_t ld_do, void* du, int64_t lddu, float* dgamma, float* dbeta,
                               int rows_cap, const int32_t* rows_dev, int d, int dtype, cudaStream_t st) {
  if (rows_cap <= 0) return cudaSuccess;
  const int es = dtype == HSTU_DTYPE_F32 ? 4 : 2;
  if (fast_rows_ok(d, o, ldo_in, u, ldu, d_o, ld_do, es, es) && fast_rows_ok(d, dg, lddg, du, lddu, du, lddu, es, es)) {
    if (dtype == HSTU_DTYPE_F32)
      return launch_ln_gate_bwd_rows<float>((const float*)o, ldo_in, (const float*)u, ldu, gamma, beta, mean, rstd,
                                            (const float*)dg, lddg, (float*)d_o, ld_do, (float*)du, lddu, dgamma,
                                            dbeta, rows_cap, rows_dev, d, st);
    using bf = __nv_bfloat16;
    return launch_ln_gate_bwd_rows<bf>((const bf*)o, ldo_in, (const bf*)u, ldu, gamma, beta, mean, rstd,
                                       (const bf*)dg, lddg, (bf*)d_o, ld_do, (bf*)du, lddu, dgamma, dbeta, rows_cap,
                                       rows_dev, d, st);
  }
  cudaError_t e = launch_ln_gate_du(o, ldo_in, gamma, beta, mean, rstd, dg, lddg, du, lddu, rows_cap, rows_dev, d,
                                    dtype, st);
  if (e != cudaSuccess) return e;
  const int g = row_grid(rows_cap) < 296 ? row_grid(rows_cap) : 296;
  if (dtype == HSTU_DTYPE_F32)
    ln_gate_bwd_kernel<float><<<g, kRowWarps * 32, 0, st>>>((const float*)o, ldo_in, (const float*)u, ldu, gamma,
                                                            mean, rstd, (const float*)dg, lddg, (float*)d_o, ld_do,
                                                            dgamma, dbeta, rows_cap, rows_dev, d);
  else
    ln_gate_bwd_kernel<__nv_bfloat16><<<g, kRowWarps * 32, 0, st>>>(
        (const __nv_bfloat16*)o, ldo_in, (const __nv_bfloat16*)u, ldu, gamma, mean, rstd,
        (const __nv_bfloat16*)dg, lddg, (__nv_bfloat16*)d_o, ld_do, dgamma, dbeta, rows_cap, rows_dev, d);
  return cudaGetLastError();
}

cudaError_t launch_ln_gate_du(const void* o, int64_t ldo_in, const float* gamma, const float* beta,
                              const float* mean, const float* rstd, const void* dg, int64_t lddg, void* du,
                              int64_t lddu, int rows_cap, const int32_t* rows_dev, int d, int dtype,
                              cudaStream_t st) {
  if (rows_cap <= 0) return cudaSuccess;
  const int g = row_grid(rows_cap);
  if (dtype == HSTU_DTYPE_F32)
    ln_gate_du_kernel<float><<<g, kRowWarps * 32, 0, st>>>((const float*)o, ldo_in, gamma, beta, mean, rstd,
                                                           (const float*)dg, lddg, (float*)du, lddu, rows_cap,
                                                           rows_dev, d);
  else
    ln_gate_du_kernel<__nv_bfloat16><<<g, kRowWarps * 32, 0, st>>>(
        (const __nv_bfloat16*)o, ldo_in, gamma, beta, mean, rstd, (const __nv_bfloat16*)dg, lddg,
        (__nv_bfloat16*)du, lddu, rows_cap, rows_dev, d);
  return cudaGetLastError();
}

cudaError_t launch_ln_bwd(const void* x, int64_t ldx, const float* gamma, const float* mean, const float* rstd,
                          const float* dxhat, int64_t lddxh, const void* dres, int64_t lddres, void* dx,
                          int64_t lddx, float* dgamma, float* dbeta, int rows_cap, const int32_t* rows_dev,
                          int d, int io_dtype, cudaStream_t st) {
  if (rows_cap <= 0) return cudaSuccess;
  const int es = io_dtype == HSTU_DTYPE_F32 ? 4 : 2;
  if (fast_rows_ok(d, x, ldx, dres, lddres, dx, lddx, es, es) && fast_rows_ok(d, dxhat, lddxh, nullptr, 0, dxhat, lddxh, 4, 4)) {
    if (io_dtype == HSTU_DTYPE_F32)
      return launch_ln_bwd_rows<float>((const float*)x, ldx, gamma, mean, rstd, dxhat, lddxh, (const float*)dres,
                                       lddres, (float*)dx, lddx, dgamma, dbeta, rows_cap, rows_dev, d, st);
    using bf = __nv_bfloat16;
    return launch_ln_bwd_rows<bf>((const bf*)x, ldx, gamma, mean, rstd, dxhat, lddxh, (const bf*)dres, lddres,
                                  (bf*)dx, lddx, dgamma, dbeta, rows_cap, rows_dev, d, st);
  }
  const int g = row_grid(rows_cap) < 296 ? row_grid(rows_cap) : 296;
  if (io_dtype == HSTU_DTYPE_F32)
    ln_bwd_kernel<float><<<g, kRowWarps * 32, 0, st>>>((const float*)x, ldx, gamma, mean, rstd, dxhat, lddxh,
                                                       (const float*)dres, lddres, (float*)dx, lddx, dgamma, dbeta,
                                                       rows_cap, rows_dev, d);
  else
    ln_bwd_kernel<__nv_bfloat16><<<g, kRowWarps * 32, 0, st>>>(
        (const __nv_bfloat16*)x, ldx, gamma, mean, rstd, dxhat, lddxh, (const __nv_bfloat16*)dres, lddres,
        (__nv_bfloat16*)dx, lddx, dgamma, dbeta, rows_cap, rows_dev, d);
  return cudaGetLastError();
}

cudaError_t launch_silu_bwd(const void* da, const void* z, void* dz, int64_t ld, int rows_cap,
                            const int32_t* rows_dev, int cols, int dtype, cudaStream_t st, const float* dq,
                            int64_t ldq, int q_col0, int q_cols) {
  if (rows_cap <= 0) return cudaSuccess;
  if (dq && (q_col0 % 8 || q_cols % 8 || ldq % 4)) return cudaErrorInvalidValue;
  const int g = 148 * 8;
  if (dtype == HSTU_DTYPE_F32)
    silu_bwd_kernel<float><<<g, 256, 0, st>>>((const float*)da, (const float*)z, (float*)dz, ld, rows_cap,
                                              rows_dev, cols, dq, ldq, q_col0, q_cols);
  else
    silu_bwd_kernel<__nv_bfloat16><<<g, 256, 0, st>>>((const __nv_bfloat16*)da, (const __nv_bfloat16*)z,
                                                      (__nv_bfloat16*)dz, ld, rows_cap, rows_dev, cols, dq, ldq,
                                                      q_col0, q_cols);
  return cudaGetLastError();
}

size_t col_partials_size(int cols) { return (size_t)kColPartBlocks * (cols > 0 ? cols : 1); }

cudaError_t launch_silu_bwd_colsum(const void* da, const void* z, void* dz, int64_t ld, int rows_cap,
                                   const int32_t* rows_dev, int cols, int dtype, float* col_sums, float* part,
                                   cudaStream_t st, const float* dq, int64_t ldq, int q_col0, int q_cols) {
  cudaError_t e = cudaMemsetAsync(col_sums, 0, sizeof(float) * (cols > 0 ? cols : 0), st);
  if (e != cudaSuccess || rows_cap <= 0 || cols <= 0) return e;
  const int es = dtype == HSTU_DTYPE_F32 ? 4 : 2;
  const bool vec = cols % 8 == 0 && (ld * es) % 16 == 0 && ((uintptr_t)da & 15) == 0 && ((uintptr_t)z & 15) == 0 &&
                   ((uintptr_t)dz & 15) == 0 && ((uintptr_t)part & 15) == 0 &&
                   (!dq || (((uintptr_t)dq & 15) == 0 && ldq % 4 == 0 && q_col0 % 8 == 0 && q_cols % 8 == 0));
  if (!vec) {
    e = launch_silu_bwd(da, z, dz, ld, rows_cap, rows_dev, cols, dtype, st, dq, ldq, q_col0, q_cols);
    if (e != cudaSuccess) return e;
    return launch_col_sum(dz, ld, rows_cap, rows_dev, cols, dtype, col_sums, st);
  }
  dim3 grid(1, (cols + 2047) / 2048);
  const int rpi = 256 / ColSumLayout::vectors(cols), cap_x = kColPartBlocks / rpi;
  const int bx = row_sms() * 4 / (int)grid.y;
  grid.x = bx < 1 ? 1 : (bx > cap_x ? cap_x : bx);
  if (grid.x > (unsigned)rows_cap) grid.x = rows_cap;
  if (dtype == HSTU_DTYPE_F32)
    silu_bwd_colsum_kernel<float><<<grid, 256, 0, st>>>((const float*)da, (const float*)z, (float*)dz, ld, rows_cap,
                                                        rows_dev, cols, dq, ldq, q_col0, q_cols, part);
  else
    silu_bwd_colsum_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)da, (const __nv_bfloat16*)z,
                                                                (__nv_bfloat16*)dz, ld, rows_cap, rows_dev, cols, dq,
                                                                ldq, q_col0, q_cols, part);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  col_partials_reduce_kernel<<<dim3((cols + 255) / 256, partial_slices((int)grid.x * rpi)), 256, 0, st>>>(
      part, (int)grid.x * rpi, cols, col_sums);
  return cudaGetLastError();
}

cudaError_t launch_convert_rows_colsum(const void* src, int64_t lds, int src_dtype, void* dst, int64_t ldd,
                                       int dst_dtype, int cols, int rows_cap, const int32_t* rows_dev,
                                       int pad_multiple, float* col_sums, float* part, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(col_sums, 0, sizeof(float) * (cols > 0 ? cols : 0), st);
  if (e != cudaSuccess || rows_cap <= 0 || cols <= 0) return e;
  const int ss = src_dtype == HSTU_DTYPE_F32 ? 4 : 2, ds = dst_dtype == HSTU_DTYPE_F32 ? 4 : 2;
  const bool vec = cols % 8 == 0 && (lds * ss) % 16 == 0 && (ldd * ds) % 16 == 0 && ((uintptr_t)src & 15) == 0 &&
                   ((uintptr_t)dst & 15) == 0 && ((uintptr_t)part & 15) == 0;
  if (!vec) {
    e = launch_convert_rows(src, lds, src_dtype, dst, ldd, dst_dtype, cols, rows_cap, rows_dev, pad_multiple, st);
    if (e != cudaSuccess) return e;
    return launch_col_sum(src, lds, rows_cap, rows_dev, cols, src_dtype, col_sums, st);
  }
  dim3 grid(1, (cols + 2047) / 2048);
  const int rpi = 256 / ColSumLayout::vectors(cols), cap_x = kColPartBlocks / rpi;
  const int bx = row_sms() * 4 / (int)grid.y;
  grid.x = bx < 1 ? 1 : (bx > cap_x ? cap_x : bx);
  if (grid.x > (unsigned)rows_cap) grid.x = rows_cap;
  using bf = __nv_bfloat16;
  if (src_dtype == HSTU_DTYPE_F32 && dst_dtype == HSTU_DTYPE_F32)
    convert_rows_colsum_kernel<float, float><<<grid, 256, 0, st>>>((const float*)src, lds, (float*)dst, ldd, cols,
                                                                   rows_cap, rows_dev, pad_multiple, part);
  else if (src_dtype == HSTU_DTYPE_F32)
    convert_rows_colsum_kernel<float, bf><<<grid, 256, 0, st>>>((const float*)src, lds, (bf*)dst, ldd, cols, rows_cap,
                                                                rows_dev, pad_multiple, part);
  else if (dst_dtype == HSTU_DTYPE_F32)
    convert_rows_colsum_kernel<bf, float><<<grid, 256, 0, st>>>((const bf*)src, lds, (float*)dst, ldd, cols, rows_cap,
                                                                rows_dev, pad_multiple, part);
  else
    convert_rows_colsum_kernel<bf, bf><<<grid, 256, 0, st>>>((const bf*)src, lds, (bf*)dst, ldd, cols, rows_cap,
                                                             rows_dev, pad_multiple, part);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  col_partials_reduce_kernel<<<dim3((cols + 255) / 256, partial_slices((int)grid.x * rpi)), 256, 0, st>>>(
      part, (int)grid.x * rpi, cols, col_sums);
  return cudaGetLastError();
}

cudaError_t launch_col_sum(const void* a, int64_t lda, int rows_cap, const int32_t* rows_dev, int cols,
                           int dtype, float* out, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * cols, st);
  if (e != cudaSuccess || rows_cap <= 0) return e;
  // about 64 rows per thread
  const int chunks = rows_cap / 64 < 1 ? 1 : (rows_cap / 64 > 4096 ? 4096 : rows_cap / 64);
  dim3 grid((cols + 255) / 256, chunks);
  if (dtype == HSTU_DTYPE_F32)
    col_sum_kernel<float><<<grid, 256, 0, st>>>((const float*)a, lda, rows_cap, rows_dev, cols, out);
  else
    col_sum_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)a, lda, rows_cap, rows_dev, cols,
                                                        out);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, void* dst, int64_t row_bytes, const int32_t* index,
                               const int32_t* count, int capacity, cudaStream_t st) {
  if (capacity <= 0) return cudaSuccess;
  if (row_bytes % 16 == 0 && ((uintptr_t)src & 15) == 0 && ((uintptr_t)dst & 15) == 0 &&
      row_bytes / 16 < (1ll << 31)) {
    gather_rows_vec_kernel<<<row_sms() * 8, 256, 0, st>>>((const uint4*)src, (uint4*)dst, (int)(row_bytes / 16), index,
                                                           count, capacity);
    return cudaGetLastError();
  }
  gather_rows_kernel<<<148 * 8, 256, 0, st>>>((const uint32_t*)src, (uint32_t*)dst, row_bytes / 4, index, count,
                                              capacity);
  return cudaGetLastError();
}

cudaError_t launch_sl_select(int B, int T, const int32_t* offs, const uint32_t* coins, const uint32_t* keys,
                             int max_len, uint32_t prob, int32_t* out_offsets, int32_t* out_index,
                             int32_t* scratch_len, int32_t* status, cudaStream_t st) {
  (void)scratch_len;
  sl_offsets_kernel<<<1, kSlThreads, 0, st>>>(B, T, offs, coins, max_len, prob, out_offsets, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || B == 0) return e;
  sl_select_kernel<<<B, kSlThreads, 0, st>>>(B, offs, coins, keys, max_len, prob, out_offsets, out_index);
  return cudaGetLastError();
}

cudaError_t launch_rebase_offsets(const int32_t* offs, int s0, int nb, int32_t* out, cudaStream_t st) {
  rebase_offsets_kernel<<<(nb + 256) / 256, 256, 0, st>>>(offs, s0, nb, out);
  return cudaGetLastError();
}

cudaError_t launch_mfalcon_slot_offsets(int U, int bm, const int32_t* hist_offs, int32_t* offs, int32_t* nt,
                                       cudaStream_t st) {
  mfalcon_slot_offsets_kernel<<<(U + 256) / 256, 256, 0, st>>>(U, bm, hist_offs, offs, nt);
  return cudaGetLastError();
}

// A user whose candidate count is negative or exceeds the n_mb * bm slots of the
// microbatches the caller asked for: the status word records it (candidates past
// the last microbatch were not scored).  Runs after the scoring, so the status
// word stays clear while the layers run.
__global__ void mfalcon_check_counts_kernel(int U, int limit, const int32_t* __restrict__ cand_offs,
                                            int32_t* __restrict__ status) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < U; u += gridDim.x * blockDim.x) {
    const int m = cand_offs[u + 1] - cand_offs[u];
    if (m < 0 || m > limit) set_status(status, HSTU_ERR_BAD_OFFSETS);
  }
}

cudaError_t launch_mfalcon_check_counts(int U, int limit, const int32_t* cand_offs, int32_t* status,
                                        cudaStream_t st) {
  if (U <= 0) return cudaSuccess;
  mfalcon_check_counts_kernel<<<(U + 255) / 256, 256, 0, st>>>(U, limit, cand_offs, status);
  return cudaGetLastError();
}

cudaError_t launch_mfalcon_slot_pack(int U, int mb, int bm, int rows_cap, int cap, const int32_t* hist_offs,
                                     const void* hist_x, const int64_t* hist_ts, const int32_t* cand_offs,
                                     const void* cand_x, const int64_t* cand_ts, int d, int dtype, int with_hist,
                                     void* x_slot, int64_t* ts_slot, void* x_c, int32_t* cand_dst, cudaStream_t st) {
  if (rows_cap <= 0) return cudaSuccess;
  const int g = min(148 * 8, (rows_cap + 7) / 8);
  if (dtype == HSTU_DTYPE_F32)
    mfalcon_slot_pack_kernel<float><<<g, 256, 0, st>>>(U, mb, bm, hist_offs, (const float*)hist_x, hist_ts, cand_offs,
                                                       (const float*)cand_x, cand_ts, d, with_hist, cap, (float*)x_slot,
                                                       ts_slot, (float*)x_c, cand_dst);
  else
    mfalcon_slot_pack_kernel<__nv_bfloat16><<<g, 256, 0, st>>>(
        U, mb, bm, hist_offs, (const __nv_bfloat16*)hist_x, hist_ts, cand_offs, (const __nv_bfloat16*)cand_x,
        cand_ts, d, with_hist, cap, (__nv_bfloat16*)x_slot, ts_slot, (__nv_bfloat16*)x_c, cand_dst);
  return cudaGetLastError();
}

cudaError_t launch_mfalcon_slot_rows(int U, int bm, int cap, const int32_t* hist_offs, const void* src,
                                     int64_t lds_bytes, void* dst, int64_t ldd_bytes, int64_t row_bytes, int to_slot,
                                     cudaStream_t st) {
  if ((int64_t)U * bm == 0) return cudaSuccess;
  mfalcon_slot_rows_kernel<<<148 * 8, 256, 0, st>>>(U, bm, hist_offs, (const uint4*)src, lds_bytes / 16, (uint4*)dst,
                                                    ldd_bytes / 16, (int)(row_bytes / 16), to_slot, cap);
  return cudaGetLastError();
}

cudaError_t launch_mfalcon_scatter(const void* y, int d, int dtype, const int32_t* cand_row_map,
                                   const int32_t* total_rows, int cap_rows, void* cand_out, cudaStream_t st) {
  const int g = 148 * 4;
  if (dtype == HSTU_DTYPE_F32)
    mfalcon_scatter_kernel<float><<<g, 256, 0, st>>>((const float*)y, d, cand_row_map, total_rows, cap_rows,
                                                     (float*)cand_out);
  else
    mfalcon_scatter_kernel<__nv_bfloat16><<<g, 256, 0, st>>>((const __nv_bfloat16*)y, d, cand_row_map, total_rows,
                                                             cap_rows, (__nv_bfloat16*)cand_out);
  return cudaGetLastError();
}

cudaError_t launch_convert_rows(const void* src, int64_t lds, int src_dtype, void* dst, int64_t ldd, int dst_dtype,
                                int cols, int rows_cap, const int32_t* rows_dev, int pad_multiple, cudaStream_t st) {
  if (rows_cap <= 0) return cudaSuccess;
  using bf = __nv_bfloat16;
  const int g = 148 * 8;
  if (src_dtype == HSTU_DTYPE_F32 && dst_dtype == HSTU_DTYPE_F32)
    convert_rows_kernel<float, float><<<g, 256, 0, st>>>((const float*)src, lds, (float*)dst, ldd, cols, rows_cap,
                                                         rows_dev, pad_multiple);
  else if (src_dtype == HSTU_DTYPE_F32)
    convert_rows_kernel<float, bf><<<g, 256, 0, st>>>((const float*)src, lds, (bf*)dst, ldd, cols, rows_cap, rows_dev,
                                                      pad_multiple);
  else if (dst_dtype == HSTU_DTYPE_F32)
    convert_rows_kernel<bf, float><<<g, 256, 0, st>>>((const bf*)src, lds, (float*)dst, ldd, cols, rows_cap, rows_dev,
                                                      pad_multiple);
  else
    convert_rows_kernel<bf, bf><<<g, 256, 0, st>>>((const bf*)src, lds, (bf*)dst, ldd, cols, rows_cap, rows_dev,
                                                   pad_multiple);
  return cudaGetLastError();
}

cudaError_t launch_zero_tail_rows(void* buf, int64_t ld_bytes, int64_t row_bytes, int rows_cap,
                                  const int32_t* rows_dev, int multiple, cudaStream_t st) {
  if (rows_cap <= 0) return cudaSuccess;
  zero_tail_rows_kernel<<<64, 256, 0, st>>>((uint32_t*)buf, ld_bytes / 4, row_bytes / 4, rows_cap, rows_dev,
                                            multiple);
  return cudaGetLastError();
}

}  // namespace hstu
