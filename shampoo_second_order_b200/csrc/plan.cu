// Host-only planner for the block-sharded data-parallel step: which rank owns
// which parameter.  The blocks of a weight are independent (podcast
// transcript, segment 16, Lemma 2), so ranks can split the optimizer work by
// parameter with no exchange beyond the gradients coming in and the updated
// weights going out; keeping whole parameters on one rank keeps the
// layer-wise graft norms local.
#include <algorithm>
#include <cstdint>
#include <numeric>
#include <string>
#include <vector>

#include "../../include/shampoo.h"

namespace shampoo {
void set_global_error(const std::string& msg);   // api.cu
}

namespace {

// Work of one parameter per optimizer step, in flop-like units: statistics
// and apply GEMMs every step (3 mn(m+n) per m x n block, both factors), and
// the root iteration every root_interval steps (about 10 steps of 4
// products, 2 n^3 each, per factor).  A 1-D segment of length l: l^2 per step
// and 60 l^3 per root step.
double param_cost(int64_t rows, int64_t cols, int ndim, int b, int root_interval) {
  const double iv = (double)std::max(root_interval, 1);
  double c = 0.0;
  if (ndim == 2) {
    for (int64_t r0 = 0; r0 < rows; r0 += b)
      for (int64_t c0 = 0; c0 < cols; c0 += b) {
        const double m = (double)std::min<int64_t>(b, rows - r0), n = (double)std::min<int64_t>(b, cols - c0);
        c += 3.0 * m * n * (m + n) + 80.0 * (m * m * m + n * n * n) / iv;
      }
  } else {
    const int64_t len = rows * cols;
    for (int64_t s0 = 0; s0 < len; s0 += b) {
      const double l = (double)std::min<int64_t>(b, len - s0);
      c += 3.0 * l * l + 60.0 * l * l * l / iv;
    }
  }
  // the elementwise passes (accumulator, graft norms, update) scale with size
  return c + 64.0 * (double)rows * (double)cols;
}

}  // namespace

extern "C" shampoo_status shampoo_plan_shards(int nparams, const int64_t* shapes, const int32_t* ndims,
                                              int block_size, int root_interval, int nranks, int32_t* owner,
                                              double* rank_cost) {
  if (nparams < 1 || !shapes || !owner || nranks < 1 || block_size < 1 || root_interval < 1) {
    shampoo::set_global_error("bad argument to shampoo_plan_shards");
    return SHAMPOO_EINVAL;
  }
  std::vector<double> cost(nparams);
  for (int i = 0; i < nparams; ++i) {
    const int64_t r = shapes[2 * i], c = shapes[2 * i + 1];
    const int nd = ndims ? ndims[i] : 2;
    if (r < 1 || c < 1 || (nd != 1 && nd != 2)) {
      shampoo::set_global_error("bad shape for parameter " + std::to_string(i));
      return SHAMPOO_EINVAL;
    }
    cost[i] = param_cost(r, c, nd, block_size, root_interval);
  }
  // longest processing time first: the costliest parameter goes to the least
  // loaded rank (ties: the lower index), in a fixed order so every rank
  // computes the same plan
  std::vector<int> order(nparams);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<double> load(nranks, 0.0);
  for (int i : order) {
    const int r = (int)(std::min_element(load.begin(), load.end()) - load.begin());
    owner[i] = r;
    load[r] += cost[i];
  }
  if (rank_cost)
    for (int r = 0; r < nranks; ++r) rank_cost[r] = load[r];
  return SHAMPOO_OK;
}
