// Shared device/host helpers of libhstu: element types, status word, the
// exact rab bucket rule and the M-FALCON mask rule.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/hstu.h"

namespace hstu {

constexpr int kNumBuckets = 128;

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }
__device__ __forceinline__ float silu_grad_f(float x) {
  float s = __frcp_rn(1.0f + __expf(-x));   // the correctly rounded 1 / (1 + e^-x)
  return s * (1.0f + x * (1.0f - s));
}

// ---------------------------------------------------------------------------
// status word: first 256 bytes of every workspace
// ---------------------------------------------------------------------------
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// rab buckets.  The time bucket is clamp(floor(ln(max(1,|dt|))/div), 0, 127);
// it equals the number of thresholds thr[1..127] that are <= max(|dt|, 1),
// where thr[b] is the smallest dt whose fp64 formula value reaches b (built on
// the host by hstu_build_time_thresholds).  Binary search over 128 entries.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int time_bucket_exact(uint64_t adt, const int64_t* thr) {
  // thr[0] = 0, thr non-decreasing; returns max{b : thr[b] <= adt} (adt >= 0)
  int lo = 0;
#pragma unroll
  for (int step = 64; step >= 1; step >>= 1) {
    int c = lo + step;
    if (c < kNumBuckets && (uint64_t)thr[c] <= adt) lo = c;
  }
  return lo;
}

__device__ __forceinline__ uint64_t abs_diff_i64(int64_t a, int64_t b) {
  return a >= b ? (uint64_t)a - (uint64_t)b : (uint64_t)b - (uint64_t)a;
}

__device__ __forceinline__ int pos_bucket(int pi, int pj) {
  int d = pi - pj;
  return d < 0 ? 0 : (d > kNumBuckets - 1 ? kNumBuckets - 1 : d);
}

// Sequence-level facts every attention kernel needs.
struct SeqInfo {
  int start;    // first token row
  int n;        // length
  int hist;     // N: history length (n - num_targets), tokens < hist are history
  float inv_n;  // 1 / max(hist, 1)
};

__device__ __forceinline__ SeqInfo load_seq(const int32_t* offs, const int32_t* num_targets, int s) {
  SeqInfo si;
  si.start = offs[s];
  si.n = offs[s + 1] - si.start;
  int nt = num_targets ? num_targets[s] : 0;
  nt = nt < 0 ? 0 : (nt > si.n ? si.n : nt);
  si.hist = si.n - nt;
  si.inv_n = 1.0f / (float)(si.hist > 1 ? si.hist : 1);
  return si;
}

// position index used by the position bias: history i, every candidate N
__device__ __forceinline__ int token_pos(int i, int hist) { return i < hist ? i : hist; }

// attended(i, j): causal with the diagonal; a candidate sees history and itself
__device__ __forceinline__ bool attended(int i, int j, int n, int hist) {
  return j <= i && i < n && (j < hist || j == i);
}

// Exact time bucket floor(ln(d) / div) of 1 <= d < 2^31 with few shared-memory
// reads.  y = log2(d) * ln2/div comes from the special-function unit; its error
// is below 2e-4 (the log2 approximation, float rounding of y < 72, and for
// d >= 2^23 the eight dropped low bits), so floor(y) is the bucket unless y lies
// within 2^-9 of an integer.  Only such lanes read one threshold (thr32[b] =
// smallest d of bucket b, clamped to INT32_MAX; thr32[128] = INT32_MAX) and
// settle the bucket with an exact integer compare.
__device__ __forceinline__ int exact_bucket(int32_t d, const int32_t* thr32, float ln2_over_div) {
  const bool big = d >= (1 << 23);
  const float f = __int_as_float(0x4B000000 | (big ? d >> 8 : d)) - 8388608.0f;  // exact: < 2^23
  const float y = (__log2f(f) + (big ? 8.0f : 0.0f)) * ln2_over_div;
  const float t = (y - 0.5f) + 12582912.0f;                 // round(y - 1/2) = floor(y) off the integers
  const float fr = y - (t - 12582912.0f);                   // y - floor(y)
  int b = __float_as_int(t) - 0x4B400000;
  b = b < 0 ? 0 : (b > kNumBuckets - 1 ? kNumBuckets - 1 : b);
  if (fr < 0.001953125f || fr > 0.998046875f) {
    const bool up = fr > 0.5f;
    const int32_t th = thr32[up ? b + 1 : b];
    b += up ? (d >= th ? 1 : 0) : (d < th ? -1 : 0);
    b = b < 0 ? 0 : (b > kNumBuckets - 1 ? kNumBuckets - 1 : b);
  }
  return b;
}
__device__ __forceinline__ int fast_bucket(int32_t d, const int32_t* thr32, float ln2_over_div) {
  return exact_bucket(d < 1 ? 1 : d, thr32, ln2_over_div);
}

// ---------------------------------------------------------------------------
// kv-tile range of a q tile [r0, r1) (in-sequence rows; r1 <= n).
// Returns the number of kv tiles of width tk that hold an attended pair and
// fills first/second ranges: tiles [0, a) and [b0, b1) (b0 >= a).
// ---------------------------------------------------------------------------
struct KvRange { int a; int b0; int b1; };

__host__ __device__ __forceinline__ KvRange kv_tiles_for(int r0, int r1, int hist, int tk) {
  // History rows need columns [0, min(r1, hist)); candidate rows need [0, hist)
  // plus their own diagonal column; both prefixes are [0, min(r1, hist)).
  KvRange k;
  int cols_a = r1 < hist ? r1 : hist;
  k.a = (cols_a + tk - 1) / tk;
  k.b0 = k.b1 = k.a;
  if (r1 > hist) {
    int c0 = r0 > hist ? r0 : hist;  // first candidate row of the tile
    int t0 = c0 / tk, t1 = (r1 - 1) / tk + 1;
    if (t0 < k.a) t0 = k.a;
    k.b0 = t0;
    k.b1 = t1 > t0 ? t1 : t0;
  }
  return k;
}

__host__ __device__ __forceinline__ int kv_count(const KvRange& k) { return k.a + (k.b1 - k.b0); }
__host__ __device__ __forceinline__ int kv_tile_at(const KvRange& k, int idx) {
  return idx < k.a ? idx : k.b0 + (idx - k.a);
}

// Work item of the jagged schedule: (sequence, head, q tile) and its cost in kv tiles.
struct WorkItem { int seq; int head; int qtile; int cost; };

}  // namespace hstu
