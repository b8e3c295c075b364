// Host-side sharding of one jagged batch over data-parallel ranks.
//
// Sequences are independent units of the layer (rows of different sequences do
// not interact), so a batch shards by sequence with no exchange on the data
// path ("Meta HSTU" case study, "Разная длина истории превращается в выигрыш по
// ресурсам": real lengths instead of padding make the cost of a sequence its
// own).  The cost of a sequence is its attended (i, j) pairs, which grow as n^2,
// plus a per-token weight for the row-wise work (LayerNorm, the projections),
// and the sequences are dealt out longest-processing-time first: in order of
// decreasing cost, each to the rank whose total cost is smallest so far.
#include <stdint.h>

#include <algorithm>
#include <vector>

#include "../../include/hstu.h"

extern "C" int hstu_lpt_partition(int32_t batch, const int32_t* seq_offsets, const int32_t* num_targets,
                                  int32_t world, double token_weight, int32_t* rank_of, double* rank_cost) {
  if (batch < 0 || world < 1 || !rank_of || !rank_cost || (batch > 0 && !seq_offsets) || !(token_weight >= 0.0))
    return HSTU_ERR_INVALID_ARG;
  if (batch > 0 && seq_offsets[0] != 0) return HSTU_ERR_INVALID_ARG;
  std::vector<double> cost((size_t)batch);
  for (int32_t s = 0; s < batch; ++s) {
    const int64_t n = (int64_t)seq_offsets[s + 1] - seq_offsets[s];
    if (n < 0) return HSTU_ERR_INVALID_ARG;
    int64_t nt = num_targets ? num_targets[s] : 0;
    nt = nt < 0 ? 0 : (nt > n ? n : nt);
    const int64_t N = n - nt;                          // history tokens
    const int64_t pairs = N * (N + 1) / 2 + nt * (N + 1);
    cost[(size_t)s] = (double)pairs + token_weight * (double)n;
  }
  std::vector<int32_t> order((size_t)batch);
  for (int32_t s = 0; s < batch; ++s) order[(size_t)s] = s;
  // decreasing cost; equal costs keep the lower index first (deterministic on every rank)
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return cost[(size_t)a] > cost[(size_t)b]; });
  for (int32_t r = 0; r < world; ++r) rank_cost[r] = 0.0;
  for (int32_t s : order) {
    int32_t best = 0;
    for (int32_t r = 1; r < world; ++r)
      if (rank_cost[r] < rank_cost[best]) best = r;   // the lowest rank among equal loads
    rank_of[s] = best;
    rank_cost[best] += cost[(size_t)s];
  }
  return HSTU_OK;
}
