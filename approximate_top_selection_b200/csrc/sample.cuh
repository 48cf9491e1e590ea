// sample.cuh -- the sampling tail of vocabulary sampling: one token per row
// drawn from the softmax, at temperature T, of the row's selected logits.
//
// Workload: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
// pith.science review page, "Core claim" and Fig. 4 (left): top-k vocabulary
// sampling over n = 128,256 logits.  The pages leave the tail implicit; this
// is plain top-k sampling.  From the selected pairs of a row (best-first, as
// the selection writes them) index idx[i] is drawn with probability
// w_i / sum_j w_j, w_i = exp((v_i - v_0) / T), by inverse CDF with the
// caller's uniform u in [0, 1): the first i whose running sum of w exceeds
// u * sum w, else (rounding) the last entry of positive weight.  Padding
// (index -1) and -inf values weigh 0; a row whose best value is NaN or +inf
// draws idx[0]; a row without candidates draws -1.
//
// One warp per row (sample_row_warp, shared with the selection kernels, which
// run it on each row right after Stage 2 when a sampling tail is requested).
#pragma once

#include "select_core.cuh"

namespace tk {

constexpr int kSampleWarps = 8;

__global__ void __launch_bounds__(32 * kSampleWarps)
    sample_rows_kernel(const float* vals, const int32_t* idx, int64_t rows, int k, float inv_t,
                       const float* u, int32_t* token) {
  pdl_wait_then_release();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kSampleWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  sample_row_warp<float>(vals + r * k, idx + r * k, k, inv_t, __ldg(u + r), token + r);
}

}  // namespace tk
