// Pointwise aggregated attention on the CUDA cores (fp32 math): the path for
// fp32 tensors (and a diagnostic path for bf16).  Forward and backward.
//
// Forward, per work item (sequence s, head h, q tile of 64 rows), for every kv
// tile of 64 columns that holds an attended pair:
//   S = Q K^T + rab, P = SiLU(S) masked, O += P V; at the end O *= 1/N.
// Backward, per (sequence, head, kv tile of 64 columns), over the q tiles that
// attend to it: recompute S and P, dV += P^T dO, dP = dO V^T,
// dS = dP SiLU'(S) mask / N, dK += dS^T Q, dQ += dS K (fp32 atomics), and the
// rab gradients via per-CTA bucket histograms.
// ("Actions Speak Louder than Words" summary, 1.2: attention without softmax,
// relative position/time bias.)
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {
namespace {

constexpr int TM = 64;
constexpr int TK = 64;
constexpr int kThreads = 256;

template <int DH>
struct SimtSmem {
  float q[TM][DH + 1];
  float k[TK][DH + 1];
  float v[TK][DH + 1];
  float p[TM][TK + 1];
  int64_t thr[kNumBuckets];
  float pos_b[kNumBuckets];
  float time_b[kNumBuckets];
  int64_t ts_q[TM];
  int64_t ts_k[TK];
};

template <int DH>
struct SimtBwdSmem {
  float q[TM][DH + 1];
  float k[TK][DH + 1];
  float v[TK][DH + 1];
  float dout[TM][DH + 1];
  float ds[TM][TK + 1];
  float p[TM][TK + 1];
  int64_t thr[kNumBuckets];
  float pos_b[kNumBuckets];
  float time_b[kNumBuckets];
  float gpos[kNumBuckets];
  float gtime[kNumBuckets];
  int64_t ts_q[TM];
  int64_t ts_k[TK];
};

// rows [row0, row0+rows) of a [T, H, DH] tensor at head h into dst[rows][DH+1] (zero beyond valid)
template <typename T, int DH, int LD>
__device__ __forceinline__ void load_rows(float (*dst)[LD], const T* __restrict__ src, int64_t ld, int head,
                                          int row0, int valid) {
  for (int e = threadIdx.x; e < 64 * DH; e += kThreads) {
    int r = e / DH, c = e % DH;
    float val = 0.f;
    if (r < valid) val = Elem<T>::to_f(src[(int64_t)(row0 + r) * ld + (int64_t)head * DH + c]);
    dst[r][c] = val;
  }
}

__device__ __forceinline__ float rab_value(int i, int j, const SeqInfo& si, int64_t ti, int64_t tj,
                                           const int64_t* thr, const float* pos_b, const float* time_b) {
  int pb = pos_bucket(token_pos(i, si.hist), token_pos(j, si.hist));
  int tb = time_bucket_exact(abs_diff_i64(ti, tj), thr);
  return pos_b[pb] + time_b[tb];
}

template <typename T, int DH>
__global__ void __launch_bounds__(kThreads)
attn_fwd_simt_kernel(AttnFwdParams prm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto& sm = *reinterpret_cast<SimtSmem<DH>*>(smem_raw);
  const int tid = threadIdx.x;
  const int count = *prm.item_count;
  for (int c = tid; c < kNumBuckets; c += kThreads) sm.thr[c] = prm.thr.v[c];

  for (int it = blockIdx.x; it < count; it += gridDim.x) {
    const WorkItem wi = prm.items[it];
    const SeqInfo si = load_seq(prm.seq_offsets, prm.num_targets, wi.seq);
    const int h = wi.head;
    const int r0 = wi.qtile * TM;
    const int qvalid = min(TM, si.n - r0);
    __syncthreads();  // previous item done with smem
    for (int c = tid; c < kNumBuckets; c += kThreads) {
      sm.pos_b[c] = prm.pos_bias[h * prm.rab_head_stride + c];
      sm.time_b[c] = prm.time_bias[h * prm.rab_head_stride + c];
    }
    for (int r = tid; r < TM; r += kThreads) sm.ts_q[r] = r < qvalid ? prm.timestamps[si.start + r0 + r] : 0;
    load_rows<T, DH, DH + 1>(sm.q, (const T*)prm.q, prm.ldq, h, si.start + r0, qvalid);

    // output accumulators: thread owns rows orow*4..+3, cols ocol*(DH/16)..
    constexpr int OC = DH / 16;
    const int orow = tid / 16, ocol = tid % 16;
    float acc[4][OC];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < OC; ++b) acc[a][b] = 0.f;

    const KvRange kr = kv_tiles_for(r0, r0 + qvalid, si.hist, TK);
    const int nkv = kv_count(kr);
    for (int kt_i = 0; kt_i < nkv; ++kt_i) {
      const int c0 = kv_tile_at(kr, kt_i) * TK;
      const int kvalid = min(TK, si.n - c0);
      __syncthreads();
      load_rows<T, DH, DH + 1>(sm.k, (const T*)prm.k, prm.ldk, h, si.start + c0, kvalid);
      load_rows<T, DH, DH + 1>(sm.v, (const T*)prm.v, prm.ldv, h, si.start + c0, kvalid);
      for (int r = tid; r < TK; r += kThreads) sm.ts_k[r] = r < kvalid ? prm.timestamps[si.start + c0 + r] : 0;
      __syncthreads();
      // S tile: thread computes rows srow*4.., cols scol*4..
      {
        const int srow = tid / 16, scol = tid % 16;
        float s[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) s[a][b] = 0.f;
        for (int d = 0; d < DH; ++d) {
          float qa[4], kb[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) qa[a] = sm.q[srow * 4 + a][d];
#pragma unroll
          for (int b = 0; b < 4; ++b) kb[b] = sm.k[scol * 4 + b][d];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) s[a][b] = fmaf(qa[a], kb[b], s[a][b]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int ri = srow * 4 + a, i = r0 + ri;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int cj = scol * 4 + b, j = c0 + cj;
            float pv = 0.f;
            if (ri < qvalid && cj < kvalid && attended(i, j, si.n, si.hist)) {
              float sv = s[a][b] + rab_value(i, j, si, sm.ts_q[ri], sm.ts_k[cj], sm.thr, sm.pos_b, sm.time_b);
              pv = silu_f(sv);
            }
            sm.p[ri][cj] = pv;
          }
        }
      }
      __syncthreads();
      // O += P V
      for (int j = 0; j < TK; ++j) {
        float vb[OC];
#pragma unroll
        for (int b = 0; b < OC; ++b) vb[b] = sm.v[j][ocol * OC + b];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          float pa = sm.p[orow * 4 + a][j];
#pragma unroll
          for (int b = 0; b < OC; ++b) acc[a][b] = fmaf(pa, vb[b], acc[a][b]);
        }
      }
    }
    // store O * 1/N
    T* out = (T*)prm.out;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int ri = orow * 4 + a;
      if (ri >= qvalid) continue;
      const int64_t row = si.start + r0 + ri;
#pragma unroll
      for (int b = 0; b < OC; ++b)
        out[row * prm.ldo + (int64_t)h * DH + ocol * OC + b] = Elem<T>::from_f(acc[a][b] * si.inv_n);
    }
  }
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------
template <typename T, int DH>
__global__ void __launch_bounds__(kThreads)
attn_bwd_simt_kernel(AttnBwdParams prm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto& sm = *reinterpret_cast<SimtBwdSmem<DH>*>(smem_raw);
  const int tid = threadIdx.x;
  const int count = *prm.item_count;
  for (int c = tid; c < kNumBuckets; c += kThreads) sm.thr[c] = prm.thr.v[c];

  for (int it = blockIdx.x; it < count; it += gridDim.x) {
    const WorkItem wi = prm.items[it];
    const SeqInfo si = load_seq(prm.seq_offsets, prm.num_targets, wi.seq);
    const int h = wi.head;
    const int c0 = wi.qtile * TK;  // in backward items, "qtile" is the kv tile
    const int kvalid = min(TK, si.n - c0);
    __syncthreads();
    for (int c = tid; c < kNumBuckets; c += kThreads) {
      sm.pos_b[c] = prm.pos_bias[h * prm.rab_head_stride + c];
      sm.time_b[c] = prm.time_bias[h * prm.rab_head_stride + c];
      sm.gpos[c] = 0.f;
      sm.gtime[c] = 0.f;
    }
    load_rows<T, DH, DH + 1>(sm.k, (const T*)prm.k, prm.ldk, h, si.start + c0, kvalid);
    load_rows<T, DH, DH + 1>(sm.v, (const T*)prm.v, prm.ldv, h, si.start + c0, kvalid);
    for (int r = tid; r < TK; r += kThreads) sm.ts_k[r] = r < kvalid ? prm.timestamps[si.start + c0 + r] : 0;

    constexpr int OC = DH / 16;
    const int orow = tid / 16, ocol = tid % 16;  // dK/dV: rows orow*4.. (kv rows), cols ocol*OC..
    float dk_acc[4][OC], dv_acc[4][OC];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < OC; ++b) { dk_acc[a][b] = 0.f; dv_acc[a][b] = 0.f; }

    const int nq = (si.n + TM - 1) / TM;
    const int qt_begin = c0 / TM;
    for (int qt = qt_begin; qt < nq; ++qt) {
      const int r0 = qt * TM;
      const int qvalid = min(TM, si.n - r0);
      // skip q tiles without an attended pair in this kv tile
      {
        const KvRange kr = kv_tiles_for(r0, r0 + qvalid, si.hist, TK);
        const int kt = c0 / TK;
        bool hit = kt < kr.a || (kt >= kr.b0 && kt < kr.b1);
        if (!hit) continue;
      }
      __syncthreads();
      load_rows<T, DH, DH + 1>(sm.q, (const T*)prm.q, prm.ldq, h, si.start + r0, qvalid);
      load_rows<T, DH, DH + 1>(sm.dout, (const T*)prm.dout, prm.lddo, h, si.start + r0, qvalid);
      for (int r = tid; r < TM; r += kThreads) sm.ts_q[r] = r < qvalid ? prm.timestamps[si.start + r0 + r] : 0;
      __syncthreads();
      {
        const int srow = tid / 16, scol = tid % 16;
        float s[4][4], dp[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) { s[a][b] = 0.f; dp[a][b] = 0.f; }
        for (int d = 0; d < DH; ++d) {
          float qa[4], kb[4], da[4], vb[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) { qa[a] = sm.q[srow * 4 + a][d]; da[a] = sm.dout[srow * 4 + a][d]; }
#pragma unroll
          for (int b = 0; b < 4; ++b) { kb[b] = sm.k[scol * 4 + b][d]; vb[b] = sm.v[scol * 4 + b][d]; }
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              s[a][b] = fmaf(qa[a], kb[b], s[a][b]);
              dp[a][b] = fmaf(da[a], vb[b], dp[a][b]);
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int ri = srow * 4 + a, i = r0 + ri;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int cj = scol * 4 + b, j = c0 + cj;
            float pv = 0.f, dsv = 0.f;
            if (ri < qvalid && cj < kvalid && attended(i, j, si.n, si.hist)) {
              int pb = pos_bucket(token_pos(i, si.hist), token_pos(j, si.hist));
              int tb = time_bucket_exact(abs_diff_i64(sm.ts_q[ri], sm.ts_k[cj]), sm.thr);
              float sv = s[a][b] + sm.pos_b[pb] + sm.time_b[tb];
              pv = silu_f(sv) * si.inv_n;
              dsv = dp[a][b] * silu_grad_f(sv) * si.inv_n;
              atomicAdd(&sm.gpos[pb], dsv);
              atomicAdd(&sm.gtime[tb], dsv);
            }
            sm.p[ri][cj] = pv;
            sm.ds[ri][cj] = dsv;
          }
        }
      }
      __syncthreads();
      // dV += P^T dO, dK += dS^T Q (kv rows orow*4.., cols ocol*OC..)
      for (int i = 0; i < TM; ++i) {
        float qv[OC], dov[OC];
#pragma unroll
        for (int b = 0; b < OC; ++b) { qv[b] = sm.q[i][ocol * OC + b]; dov[b] = sm.dout[i][ocol * OC + b]; }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          float pa = sm.p[i][orow * 4 + a], da = sm.ds[i][orow * 4 + a];
#pragma unroll
          for (int b = 0; b < OC; ++b) {
            dv_acc[a][b] = fmaf(pa, dov[b], dv_acc[a][b]);
            dk_acc[a][b] = fmaf(da, qv[b], dk_acc[a][b]);
          }
        }
      }
      // dQ += dS K (q rows orow*4.., cols ocol*OC..), fp32 atomics into the workspace
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int ri = orow * 4 + a;
        if (ri >= qvalid) continue;
        float dq[OC];
#pragma unroll
        for (int b = 0; b < OC; ++b) dq[b] = 0.f;
        for (int j = 0; j < TK; ++j) {
          float dsv = sm.ds[ri][j];
#pragma unroll
          for (int b = 0; b < OC; ++b) dq[b] = fmaf(dsv, sm.k[j][ocol * OC + b], dq[b]);
        }
        float* dst = prm.dq_accum + ((int64_t)(si.start + r0 + ri) * prm.num_heads + h) * DH + ocol * OC;
#pragma unroll
        for (int b = 0; b < OC; ++b) atomicAdd(dst + b, dq[b]);
      }
    }
    // store dK, dV
    T* dk = (T*)prm.dk;
    T* dv = (T*)prm.dv;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = orow * 4 + a;
      if (r >= kvalid) continue;
      const int64_t row = si.start + c0 + r;
#pragma unroll
      for (int b = 0; b < OC; ++b) {
        dk[row * prm.lddk + (int64_t)h * DH + ocol * OC + b] = Elem<T>::from_f(dk_acc[a][b]);
        dv[row * prm.lddv + (int64_t)h * DH + ocol * OC + b] = Elem<T>::from_f(dv_acc[a][b]);
      }
    }
    __syncthreads();
    for (int c = tid; c < kNumBuckets; c += kThreads) {
      if (sm.gpos[c] != 0.f) atomicAdd(&prm.d_pos_bias[h * prm.rab_head_stride + c], sm.gpos[c]);
      if (sm.gtime[c] != 0.f) atomicAdd(&prm.d_time_bias[h * prm.rab_head_stride + c], sm.gtime[c]);
    }
  }
}

template <typename T>
__global__ void dq_finalize_kernel(const float* __restrict__ acc, const int32_t* __restrict__ offs, int B,
                                   int H, int dh, T* __restrict__ dq, int64_t lddq) {
  const int rows = offs[B];
  const int64_t total = (int64_t)rows * H * dh;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    int64_t row = e / (H * dh);
    int col = (int)(e % (H * dh));
    dq[row * lddq + col] = Elem<T>::from_f(acc[e]);
  }
}

template <typename T, int DH>
cudaError_t fwd_dispatch(const AttnFwdParams& p, int grid, cudaStream_t st) {
  size_t smem = sizeof(SimtSmem<DH>);
  auto kern = attn_fwd_simt_kernel<T, DH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int DH>
cudaError_t bwd_dispatch(const AttnBwdParams& p, int grid, cudaStream_t st) {
  size_t smem = sizeof(SimtBwdSmem<DH>);
  auto kern = attn_bwd_simt_kernel<T, DH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int simt_tile_m() { return TM; }

cudaError_t launch_attn_fwd_simt(const AttnFwdParams& p, int dtype, int dh, int grid, cudaStream_t st) {
  if (dtype == HSTU_DTYPE_F32) {
    if (dh == 32) return fwd_dispatch<float, 32>(p, grid, st);
    if (dh == 64) return fwd_dispatch<float, 64>(p, grid, st);
    if (dh == 128) return fwd_dispatch<float, 128>(p, grid, st);
  } else {
    if (dh == 32) return fwd_dispatch<__nv_bfloat16, 32>(p, grid, st);
    if (dh == 64) return fwd_dispatch<__nv_bfloat16, 64>(p, grid, st);
    if (dh == 128) return fwd_dispatch<__nv_bfloat16, 128>(p, grid, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_simt(const AttnBwdParams& p, int dtype, int dh, int grid, cudaStream_t st) {
  if (dtype == HSTU_DTYPE_F32) {
    if (dh == 32) return bwd_dispatch<float, 32>(p, grid, st);
    if (dh == 64) return bwd_dispatch<float, 64>(p, grid, st);
    if (dh == 128) return bwd_dispatch<float, 128>(p, grid, st);
  } else {
    if (dh == 32) return bwd_dispatch<__nv_bfloat16, 32>(p, grid, st);
    if (dh == 64) return bwd_dispatch<__nv_bfloat16, 64>(p, grid, st);
    if (dh == 128) return bwd_dispatch<__nv_bfloat16, 128>(p, grid, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_dq_finalize(const float* acc, const int32_t* offs, int B, int H, int dh, int dtype,
                               void* dq, int64_t lddq, int grid, cudaStream_t st) {
  if (dtype == HSTU_DTYPE_F32)
    dq_finalize_kernel<float><<<grid, 256, 0, st>>>(acc, offs, B, H, dh, (float*)dq, lddq);
  else
    dq_finalize_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(acc, offs, B, H, dh, (__nv_bfloat16*)dq, lddq);
  return cudaGetLastError();
}

}  // namespace hstu
