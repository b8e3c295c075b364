// Jagged-batch scheduler: builds the (sequence, head, q tile) work list of the
// attention kernels ("Разная длина истории": real lengths, no padding to a
// common maximum).  Two orders: by cost (number of kv tiles) in descending order,
// for persistent CTAs that take items in snake order (an approximation of LPT);
// and a locality order for CTAs that fetch items dynamically (mode 3).
#include <cub/block/block_scan.cuh>

#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

namespace {
constexpr int kSchedThreads = 1024;
constexpr int kCostBins = 2048;  // costs >= kCostBins - 1 share the top bin
constexpr int kSeqSmem = 4096;   // sequences whose list offsets fit in shared memory (locality order)

// cost of one item: kv tiles for a forward q tile (mode 0) or for a pair of
// q tiles of width tk (mode 2, tm = 2 tk), q tiles for a backward kv tile (mode 1)
__device__ __forceinline__ int item_cost(int mode, int t, int n, int hist, int tm, int tk) {
  if (mode == 0) {
    int r0 = t * tm, r1 = min(n, r0 + tm);
    return kv_count(kv_tiles_for(r0, r1, hist, tk));
  }
  if (mode == 2) {
    const int r0 = t * tm, rb = r0 + tk;
    int c = kv_count(kv_tiles_for(r0, min(n, rb), hist, tk));
    if (rb < n) c += kv_count(kv_tiles_for(rb, min(n, r0 + tm), hist, tk));
    return c;
  }
  // backward: q tiles that hold a row attending to kv tile t (columns [c0, c1))
  int c0 = t * tk, c1 = min(n, c0 + tk);
  int qt_end = (n + tm - 1) / tm;
  if (c0 < hist) return qt_end - c0 / tm;
  return (c1 - 1) / tm - c0 / tm + 1;
}

__global__ void __launch_bounds__(kSchedThreads)
build_work_list_kernel(const int32_t* __restrict__ offs, const int32_t* __restrict__ num_targets,
                       int B, int T, int H, int tm, int tk, int mode, int max_items,
                       WorkItem* __restrict__ items, int32_t* __restrict__ count,
                       int32_t* __restrict__ status, int32_t* __restrict__ tile_base, int q_from_hist) {
  using Scan = cub::BlockScan<int, kSchedThreads>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int hist_bins[kCostBins];
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int c = tid; c < kCostBins; c += kSchedThreads) hist_bins[c] = 0;
  __syncthreads();
  // validation of the jagged description
  if (tid == 0 && (offs[0] != 0 || offs[B] > T || offs[B] < 0)) bad = 1;
  for (int s = tid; s < B; s += kSchedThreads) {
    int n = offs[s + 1] - offs[s];
    int nt = num_targets ? num_targets[s] : 0;
    if (n < 0 || nt < 0 || nt > n) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      *count = 0;
      set_status(status, HSTU_ERR_BAD_OFFSETS);
      if (tile_base) tile_base[B] = 0;
    }
    return;
  }
  // first kv tile (of width tk) of every sequence in a tiled per-tile array
  if (tile_base) {
    __shared__ int carry;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < B; base += kSchedThreads) {
      const int s = base + tid;
      const int v = s < B ? (offs[s + 1] - offs[s] + tk - 1) / tk : 0;
      int ex, tot;
      Scan(scan_tmp).ExclusiveSum(v, ex, tot);
      if (s < B) tile_base[s] = carry + ex;
      __syncthreads();
      if (tid == 0) carry += tot;
      __syncthreads();
    }
    if (tid == 0) tile_base[B] = carry;
    __syncthreads();
  }
  if (mode == 3) {
    // Locality order for dynamically fetched forward items: sequences by number of
    // q tiles (descending), then head, then q tile (descending).  CTAs that run at
    // the same time then share the K/V tiles of a few (sequence, head) pairs.
    // (with q_from_hist, only the q tiles from the one holding the first target row on)
    for (int s = tid; s < B; s += kSchedThreads) {
      const int n = offs[s + 1] - offs[s];
      const int t0 = q_from_hist ? (n - (num_targets ? num_targets[s] : 0)) / tm : 0;
      const int tiles = (n + tm - 1) / tm - t0;
      if (tiles > 0) atomicAdd(&hist_bins[min(tiles, kCostBins - 1)], tiles * H);
    }
    __syncthreads();
    constexpr int kPer3 = kCostBins / kSchedThreads;
    int loc[kPer3];
    int sum3 = 0;
#pragma unroll
    for (int r = 0; r < kPer3; ++r) {
      loc[r] = hist_bins[kCostBins - 1 - (tid * kPer3 + r)];
      sum3 += loc[r];
    }
    int base3, total3;
    Scan(scan_tmp).ExclusiveSum(sum3, base3, total3);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kPer3; ++r) {
      hist_bins[kCostBins - 1 - (tid * kPer3 + r)] = base3;
      base3 += loc[r];
    }
    __syncthreads();
    if (total3 > max_items) {
      if (tid == 0) { *count = 0; set_status(status, HSTU_ERR_WORKSPACE); }
      return;
    }
    // every sequence's place in the list; the items themselves are then written by
    // all threads (flat index over sequences in order, H * tiles items each)
    __shared__ int seq_base[kSeqSmem];
    const bool flat = tile_base != nullptr && tm == tk && B <= kSeqSmem && !q_from_hist;
    for (int s = tid; s < B; s += kSchedThreads) {
      const SeqInfo si = load_seq(offs, num_targets, s);
      const int t0 = q_from_hist ? si.hist / tm : 0;
      const int tiles = (si.n + tm - 1) / tm - t0;
      if (tiles <= 0) continue;
      const int base_s = atomicAdd(&hist_bins[min(tiles, kCostBins - 1)], tiles * H);
      if (flat) {
        seq_base[s] = base_s;
        continue;
      }
      for (int h = 0; h < H; ++h)
        for (int t = 0; t < tiles; ++t)
          items[base_s + h * tiles + (tiles - 1 - t)] =
              WorkItem{s, h, t0 + t, item_cost(0, t0 + t, si.n, si.hist, tm, tk)};
    }
    if (flat) {
      __syncthreads();
      // tile_base[s] (q tiles before sequence s, tm == tk) orders the flat index
      for (int f = tid; f < total3; f += kSchedThreads) {
        int lo = 0, hi = B - 1;  // last s with tile_base[s] * H <= f
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if ((int64_t)tile_base[mid] * H <= f) lo = mid; else hi = mid - 1;
        }
        const int s = lo;
        const SeqInfo si = load_seq(offs, num_targets, s);
        const int tiles = tile_base[s + 1] - tile_base[s];
        const int local = f - tile_base[s] * H;
        const int h = local / tiles, t = local - h * tiles;
        items[seq_base[s] + h * tiles + (tiles - 1 - t)] = WorkItem{s, h, t, item_cost(0, t, si.n, si.hist, tm, tk)};
      }
    }
    if (tid == 0) {
      *count = total3;
      count[1] = 0;  // dynamic fetch cursor
    }
    return;
  }
  // pass 1: histogram of costs
  for (int s = tid; s < B; s += kSchedThreads) {
    SeqInfo si = load_seq(offs, num_targets, s);
    int tiles = mode != 1 ? (si.n + tm - 1) / tm : (si.n + tk - 1) / tk;
    const int t0 = (q_from_hist && mode != 1) ? si.hist / tm : 0;
    for (int t = t0; t < tiles; ++t) {
      int c = item_cost(mode, t, si.n, si.hist, tm, tk);
      if (c <= 0) continue;
      atomicAdd(&hist_bins[min(c, kCostBins - 1)], H);
    }
  }
  __syncthreads();
  // exclusive scan in descending cost order: bin c starts after all bins > c
  constexpr int kPer = kCostBins / kSchedThreads;
  int local[kPer];
  int sum = 0;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    int c = kCostBins - 1 - (tid * kPer + r);
    local[r] = hist_bins[c];
    sum += local[r];
  }
  int base, total;
  Scan(scan_tmp).ExclusiveSum(sum, base, total);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    int c = kCostBins - 1 - (tid * kPer + r);
    hist_bins[c] = base;  // becomes the cursor of bin c
    base += local[r];
  }
  __syncthreads();
  if (total > max_items) {  // cannot happen for consistent sizes; refuse rather than overflow
    if (tid == 0) { *count = 0; set_status(status, HSTU_ERR_WORKSPACE); }
    return;
  }
  // pass 2: scatter
  for (int s = tid; s < B; s += kSchedThreads) {
    SeqInfo si = load_seq(offs, num_targets, s);
    int tiles = mode != 1 ? (si.n + tm - 1) / tm : (si.n + tk - 1) / tk;
    const int t0 = (q_from_hist && mode != 1) ? si.hist / tm : 0;
    for (int t = t0; t < tiles; ++t) {
      int c = item_cost(mode, t, si.n, si.hist, tm, tk);
      if (c <= 0) continue;
      int pos = atomicAdd(&hist_bins[min(c, kCostBins - 1)], H);
      for (int h = 0; h < H; ++h) items[pos + h] = WorkItem{s, h, t, c};
    }
  }
  if (tid == 0) {
    *count = total;
    count[1] = 0;  // dynamic fetch cursor
  }
}
}  // namespace

size_t work_list_capacity(int B, int T, int H, int tile) {
  return ((size_t)T / tile + (size_t)B + 1) * (size_t)H;
}

cudaError_t launch_build_work_list(const int32_t* offs, const int32_t* num_targets, int B, int T, int H,
                                   int tm, int tk, int mode, int max_items, WorkItem* items,
                                   int32_t* count, int32_t* status, cudaStream_t stream, int32_t* tile_base,
                                   int q_from_hist) {
  build_work_list_kernel<<<1, kSchedThreads, 0, stream>>>(offs, num_targets, B, T, H, tm, tk, mode,
                                                          max_items, items, count, status, tile_base, q_from_hist);
  return cudaGetLastError();
}

}  // namespace hstu
