// CUDA-core GEMM with the layer's fused epilogues: the path for fp32 tensors
// and for operand layouts the tcgen05 GEMM does not take (transposed operands
// of the weight-gradient products).  C[m, n] = sum_k A(m, k) B(n, k) with
// arbitrary element strides, fp32 accumulation, 64x64 tiles, 4x4 per thread.
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void epilogue_store(const GemmParams& p, int m, int n, float acc) {
  switch (p.epi) {
    case EPI_STORE_F32: {
      float* o = (float*)p.out + (int64_t)m * p.ldo + n;
      *o = p.accumulate ? *o + acc : acc;
      break;
    }
    case EPI_BIAS_SILU: {
      const float z = acc + (p.bias ? p.bias[n] : 0.f);
      ((T*)p.out)[(int64_t)m * p.ldo + n] = Elem<T>::from_f(silu_f(z));
      if (p.out2) ((T*)p.out2)[(int64_t)m * p.ldo2 + n] = Elem<T>::from_f(z);
      break;
    }
    case EPI_BIAS_RESIDUAL: {
      float y = acc + (p.bias ? p.bias[n] : 0.f);
      if (p.residual) {
        if (p.res_f32) y += ((const float*)p.residual)[(int64_t)m * p.ldr + n];
        else y += Elem<T>::to_f(((const T*)p.residual)[(int64_t)m * p.ldr + n]);
      }
      if (p.out_f32) ((float*)p.out)[(int64_t)m * p.ldo + n] = y;
      else ((T*)p.out)[(int64_t)m * p.ldo + n] = Elem<T>::from_f(y);
      break;
    }
    default:
      if (p.out_f32) ((float*)p.out)[(int64_t)m * p.ldo + n] = acc;
      else ((T*)p.out)[(int64_t)m * p.ldo + n] = Elem<T>::from_f(acc);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) gemm_simt_kernel(GemmParams p) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int M = p.rows_dev ? min(p.M, *p.rows_dev) : p.M;
  const int K = p.k_dev ? min(p.K, *p.k_dev) : p.K;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  if (m0 >= M) return;
  const T* A = (const T*)p.A;
  const T* B = (const T*)p.B;
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  const bool a_kmajor = p.sak == 1;
  const bool b_kmajor = p.sbk == 1;
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int r = 0; r < (BM * BK) / kThreads; ++r) {
      const int e = tid + r * kThreads;
      int mm, kk;
      if (a_kmajor) { mm = e / BK; kk = e % BK; } else { mm = e % BM; kk = e / BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? Elem<T>::to_f(A[(int64_t)gm * p.sam + (int64_t)gk * p.sak]) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < (BN * BK) / kThreads; ++r) {
      const int e = tid + r * kThreads;
      int nn, kk;
      if (b_kmajor) { nn = e / BK; kk = e % BK; } else { nn = e % BN; kk = e / BN; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < p.N && gk < K) ? Elem<T>::to_f(B[(int64_t)gn * p.sbn + (int64_t)gk * p.sbk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) av[a] = As[kk][tr * 4 + a];
#pragma unroll
      for (int b = 0; b < 4; ++b) bv[b] = Bs[kk][tc * 4 + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int m = m0 + tr * 4 + a;
    if (m >= M) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int n = n0 + tc * 4 + b;
      if (n < p.N) epilogue_store<T>(p, m, n, acc[a][b]);
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmParams& p, int dtype, cudaStream_t st) {
  if (p.M <= 0 || p.N <= 0) return cudaSuccess;
  dim3 grid((p.N + BN - 1) / BN, (p.M + BM - 1) / BM);
  if (grid.y > 65535) return cudaErrorInvalidValue;
  if (dtype == HSTU_DTYPE_F32)
    gemm_simt_kernel<float><<<grid, kThreads, 0, st>>>(p);
  else
    gemm_simt_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace hstu
