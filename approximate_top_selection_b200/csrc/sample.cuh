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
// One warp per row: each lane sums a contiguous slice of the k weights in
// fp32, a shuffle scan gives every lane the weight before its slice, and the
// lane whose running sum crosses the target names the token.
#pragma once

#include "common.cuh"

namespace tk {

constexpr int kSampleWarps = 8;

__global__ void __launch_bounds__(32 * kSampleWarps)
    sample_rows_kernel(const float* vals, const int32_t* idx, int64_t rows, int k, float inv_t,
                       const float* u, int32_t* token) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kSampleWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  const float* v = vals + r * k;
  const int32_t* ix = idx + r * k;
  const int32_t i0 = ix[0];
  const float v0 = v[0];
  if (i0 < 0 || v0 != v0 || v0 == __int_as_float(0x7f800000)) {
    if (lane == 0) token[r] = i0;  // -1 (no candidate), or the NaN / +inf entry
    return;
  }
  const int per = (k + 31) / 32;
  const int beg = min(lane * per, k), end = min(beg + per, k);
  float part = 0.0f;
  for (int i = beg; i < end; ++i)
    if (ix[i] >= 0) part += expf((v[i] - v0) * inv_t);
  float incl = part;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const float total = __shfl_sync(0xffffffffu, incl, 31);
  const float target = u[r] * total;
  float run = incl - part;
  int32_t pick = -1, last = -1;
  for (int i = beg; i < end; ++i) {
    if (ix[i] < 0) continue;
    const float w = expf((v[i] - v0) * inv_t);
    if (w > 0.0f) last = ix[i];
    run += w;
    if (run > target) {
      pick = ix[i];
      break;
    }
  }
  const unsigned picked = __ballot_sync(0xffffffffu, pick >= 0);
  const unsigned lasted = __ballot_sync(0xffffffffu, last >= 0);
  const int src = picked ? __ffs(picked) - 1 : (lasted ? 31 - __clz(lasted) : 0);
  const int32_t t = __shfl_sync(0xffffffffu, picked ? pick : last, src);
  if (lane == 0) token[r] = t;
}

}  // namespace tk
