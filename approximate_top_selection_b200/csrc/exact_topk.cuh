// exact_topk.cuh -- exact top-k per row (the baseline the bucketed method is
// compared with, and the general form of its Stage 2).
//
// "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358): Fig. 1
// compares against exact top-k implementations; Fig. 12 (RADIXSELECT) finds
// the k-th value digit by digit and notes that a tied k-th value needs a
// second "collect" step.  This kernel does that on the CTA level:
//   * rows of at most kSortCap elements: bitonic sort of the packed
//     (key, index) candidates in shared memory;
//   * longer rows: up to three radix levels (11, 11, 10 bits of the
//     order-preserving key) with shared-memory histograms narrow the k-th key;
//     as soon as the elements sharing the current digit prefix fit in shared
//     memory they are gathered and sorted there; if a full key is still tied
//     beyond that, the tied elements are taken in index order (collect step).
// One CTA of 1024 threads per row.
#pragma once

#include "select_core.cuh"

namespace tk {

constexpr int kExactThreads = 1024;
constexpr int kSortCap = 8192;
constexpr int kCandCap = 4096;
constexpr int kHistBins = 2048;

struct ExactSmem {
  int n_sort;  // next_pow2(n) when n <= kSortCap, else 0
  int sel_cap; // next_pow2(k) for the radix path
  __host__ __device__ size_t total() const {
    if (n_sort) return static_cast<size_t>(n_sort) * 8;
    return static_cast<size_t>(kHistBins) * 4 + static_cast<size_t>(kCandCap) * 8 +
           static_cast<size_t>(sel_cap) * 8 + 128;
  }
};

__global__ void __launch_bounds__(kExactThreads) exact_topk_kernel(const float* x, int64_t n, int k,
                                                                   int sel_cap, float* out_vals,
                                                                   int32_t* out_idx) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int64_t r = blockIdx.x;
  const float* row = x + r * n;
  float* ov = out_vals + r * static_cast<int64_t>(k);
  int32_t* oi = out_idx + r * static_cast<int64_t>(k);
  const int tid = threadIdx.x;
  const int T = blockDim.x;
  pdl_wait_then_release();

  if (n <= kSortCap) {
    uint64_t* s = reinterpret_cast<uint64_t*>(smem);
    const int nn = static_cast<int>(n);
    for (int i = tid; i < nn; i += T) s[i] = pack(order_key(__ldg(row + i)), i);
    finalize_row<kGatherInput, float>(s, nn, k, row, ov, oi, T);
    return;
  }

  uint32_t* hist = reinterpret_cast<uint32_t*>(smem);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + kHistBins * 4);
  uint64_t* sel = cand + kCandCap;
  int* misc = reinterpret_cast<int*>(sel + sel_cap);  // 32 ints of scratch
  __shared__ int s_digit, s_gt, s_eq, s_nsel, s_ncand;

  if (k >= n) {
    // Every element is selected; the sort orders them and pads the rest.
    const int nn = static_cast<int>(n);
    for (int i = tid; i < nn; i += T) sel[i] = pack(order_key(__ldg(row + i)), i);
    finalize_row<kGatherInput, float>(sel, nn, k, row, ov, oi, T);
    return;
  }


  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  uint32_t prefix = 0;  // digits fixed so far
  int need = k;         // elements still to take from those matching prefix
  int level = 0;
  int eq = 0;
  for (; level < 3; ++level) {
    const int sh = shifts[level], wd = widths[level];
    const int bins = 1 << wd;
    for (int i = tid; i < bins; i += T) hist[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < n; i += T) {
      const uint32_t key = order_key(__ldg(row + i));
      if ((static_cast<uint64_t>(key) >> (sh + wd)) == prefix)
        atomicAdd(hist + ((key >> sh) & (bins - 1)), 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // Walk the bins from the top, 32 at a time: find the digit holding the
      // need-th largest key among the elements matching the prefix.
      int above = 0;
      for (int base = bins - 32; base >= 0; base -= 32) {
        const int bin = base + 31 - tid;  // lane 0 holds the highest bin of the chunk
        const int h = static_cast<int>(hist[bin]);
        int incl = h;  // inclusive prefix over lanes 0..tid (descending bins)
        for (int m = 1; m < 32; m <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, m);
          if (tid >= m) incl += y;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (above + total >= need) {
          const unsigned hit = __ballot_sync(0xffffffffu, above + incl >= need);
          const int lane = __ffs(hit) - 1;
          if (tid == lane) {
            s_digit = bin;
            s_gt = above + incl - h;
            s_eq = h;
          }
          break;
        }
        above += total;
      }
    }
    __syncthreads();
    prefix = (prefix << wd) | static_cast<uint32_t>(s_digit);
    need -= s_gt;
    eq = s_eq;
    __syncthreads();
    if (eq <= kCandCap) break;
  }
  if (level == 3) level = 2;
  const int sh = shifts[level];

  // Gather: everything strictly above the prefix is selected; the elements on
  // the prefix are candidates for the remaining `need` slots.
  if (tid == 0) {
    s_nsel = 0;
    s_ncand = 0;
  }
  __syncthreads();
  const bool fits = eq <= kCandCap;
  for (int64_t i = tid; i < n; i += T) {
    const uint32_t key = order_key(__ldg(row + i));
    const uint32_t top = key >> sh;
    if (top > prefix) {
      sel[atomicAdd(&s_nsel, 1)] = pack(key, static_cast<uint32_t>(i));
    } else if (fits && top == prefix) {
      cand[atomicAdd(&s_ncand, 1)] = pack(key, static_cast<uint32_t>(i));
    }
  }
  __syncthreads();
  const int base = k - need;  // == s_nsel
  if (fits) {
    const int m = s_ncand;
    const int N = next_pow2(m);
    for (int i = m + tid; i < N; i += T) cand[i] = 0;
    __syncthreads();
    bitonic_desc(cand, N, T);
    for (int i = tid; i < need; i += T) sel[base + i] = cand[i];
  } else {
    // Full 32-bit key tied beyond the buffer: take the tied elements in index
    // order (lowest indices first), `need` of them.
    int taken = 0;
    for (int64_t c0 = 0; c0 < n && taken < need; c0 += T) {
      const int64_t i = c0 + tid;
      const bool tie = i < n && order_key(__ldg(row + i)) == prefix;
      const unsigned bal = __ballot_sync(0xffffffffu, tie);
      const int lane = tid & 31, warp = tid >> 5;
      const int before_in_warp = __popc(bal & ((1u << lane) - 1u));
      __syncthreads();
      if (lane == 0) misc[warp] = __popc(bal);
      __syncthreads();
      int before = 0, total = 0;
      for (int w = 0; w < (T >> 5); ++w) {
        const int cw = misc[w];
        if (w < warp) before += cw;
        total += cw;
      }
      const int rank = taken + before + before_in_warp;
      if (tie && rank < need) sel[base + rank] = pack(prefix, static_cast<uint32_t>(i));
      taken += total;
    }
  }
  __syncthreads();
  finalize_row<kGatherInput, float>(sel, k, k, row, ov, oi, T);
}

}  // namespace tk
