// merge_select.cuh -- bucketed selection over lists of (value, index) pairs.
//
// Method: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
// pith.science review page, "What carries the argument": the bucket of an
// element is its index modulo b ("The reading"), each bucket keeps its top-k_b
// and the final exact top-k keeps the k best candidates.  Here the elements
// arrive as candidate lists with global indices -- the per-slice results of a
// row cut into column slices (several CTAs, or several GPUs, each holding part
// of a vocabulary or of an entity table) -- and the same selection runs on
// their union.  When every slice's list is that slice's bucketed top-k (with
// global indices), the result is the bucketed top-k of the whole row, bit for
// bit: a kept element is in its slice's top-k (k slice candidates above it
// would give k row candidates above it), and the per-bucket top-k_b of the
// union of the slices' per-bucket lists is the row's.
//
// One CTA per row.  The bucket lists live in shared memory as packed words
// (order key << 32 | ~index, 0 = empty) and every pair is inserted by a
// cascade of 64-bit atomicMax operations: slot 0 of a bucket keeps the
// largest word offered to it and hands the smaller of (old, new) to slot 1,
// and so on, so slot s ends with the (s+1)-th largest word ever offered to
// the bucket whatever the interleaving.  Stage 2 is the shared one.
#pragma once

#include "select_core.cuh"

namespace tk {

constexpr int kMergeMaxParts = 64;

struct MergeArgs {
  const float* vals;    // [parts][rows][m]
  const int32_t* idx;   // [parts][rows][m]; -1 = empty slot
  int parts, m, k, b;
  int64_t rows, n_total;
  float* out_vals;      // [rows][k]
  int32_t* out_idx;     // [rows][k]
  int64_t offs[kMergeMaxParts];  // added to every index of a part
};

__device__ __forceinline__ uint64_t umin64_m(uint64_t a, uint64_t b) { return a < b ? a : b; }

template <int KB>
__global__ void __launch_bounds__(kThreads) bucket_merge_kernel(MergeArgs p) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem);  // [b][KB] lists, then Stage-2 room
  const int tid = threadIdx.x;
  const int C = p.b * KB;
  const int cap = sort_capacity(C);
  pdl_wait_then_release();
  const int64_t r = blockIdx.x;
  for (int i = tid; i < cap; i += kThreads) cand[i] = 0ull;
  group_sync(kThreads);

  bool bad = false;
  for (int part = 0; part < p.parts; ++part) {
    const size_t base = (static_cast<size_t>(part) * p.rows + r) * p.m;
    const float* v = p.vals + base;
    const int32_t* ix = p.idx + base;
    const int64_t off = p.offs[part];
    for (int e = tid; e < p.m; e += kThreads) {
      const int32_t li = __ldg(ix + e);
      if (li < 0) continue;  // empty slot
      const int64_t g = static_cast<int64_t>(li) + off;
      if (g >= p.n_total) {
        bad = true;
        continue;
      }
      uint64_t c = pack(order_key(__ldg(v + e)), static_cast<uint32_t>(g));
      uint64_t* slot = cand + static_cast<size_t>(g % p.b) * KB;
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        const uint64_t old = atomicMax(reinterpret_cast<unsigned long long*>(slot + s),
                                       static_cast<unsigned long long>(c));
        c = umin64_m(old, c);
        if (c == 0ull) break;
      }
    }
  }
  if (bad) atomicOr(&g_device_status, 2);
  group_sync(kThreads);

  float* ov = p.out_vals + r * static_cast<int64_t>(p.k);
  int32_t* oi = p.out_idx + r * static_cast<int64_t>(p.k);
  stage2<kFromKey, float>(cand, C, p.k, nullptr, ov, oi);

  // Values came back from their keys, which fold -0.0 into +0.0 and every NaN
  // into one; restore the input bits of such outputs.  The outputs are sorted
  // by packed word, so each zero or NaN pair finds its slot by binary search
  // in a shared-memory copy of that order.
  const int kept = C < p.k ? C : p.k;
  for (int s = tid; s < kept; s += kThreads)
    cand[s] = oi[s] >= 0 ? pack(order_key(ov[s]), static_cast<uint32_t>(oi[s])) : 0ull;
  group_sync(kThreads);
  for (int part = 0; part < p.parts; ++part) {
    const size_t base = (static_cast<size_t>(part) * p.rows + r) * p.m;
    const float* v = p.vals + base;
    const int32_t* ix = p.idx + base;
    const int64_t off = p.offs[part];
    for (int e = tid; e < p.m; e += kThreads) {
      const float x = __ldg(v + e);
      if (!(x == 0.0f || x != x)) continue;
      const int32_t li = __ldg(ix + e);
      if (li < 0) continue;
      const int64_t g = static_cast<int64_t>(li) + off;
      if (g >= p.n_total) continue;
      const uint64_t w = pack(order_key(x), static_cast<uint32_t>(g));
      int lo = 0, hi = kept;  // descending: find w
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cand[mid] > w)
          lo = mid + 1;
        else
          hi = mid;
      }
      if (lo < kept && cand[lo] == w) ov[lo] = x;
    }
  }
}

}  // namespace tk
