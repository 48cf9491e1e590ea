// select_core.cuh -- the pieces every selection kernel shares:
//   * per-thread register bucket queues (Stage 1 state, k_b <= 4 entries each),
//   * the merge of queues that cover the same bucket,
//   * Stage 2 (exact top-k over the bucket candidates, best-first) in shared memory,
//   * the cross-CTA merge of a row split over several CTAs.
//
// Method: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
// pith.science review page, "What carries the argument" (per-thread priority
// queues of size k_b <= 4 in registers; optional final exact top-k) and Fig. 2.
//
// Split rows: a CTA that holds only part of a row ("piece") writes the per-bucket
// top-k_b of its piece to the workspace; the last CTA to finish a piece of that
// row (atomic ticket, nobody waits) takes, per bucket, the top-k_b of all pieces'
// lists and runs Stage 2.  This equals the single-pass result because the top-k_b
// of a bucket is the top-k_b of the union of the per-piece top-k_b lists.
#pragma once

#include "common.cuh"

namespace tk {

// ------------------------------------------------------------------ queues
// Four register queues per thread.  Queue v keeps the best KB (key, index)
// pairs offered to it, best-first.  Inside one queue indices arrive in
// increasing order, so a strict comparison resolves ties by lowest index
// without looking at the index.
//
// k_b = 1: the queue is a running maximum kept in the float domain: thr[v] is
// the best value so far (NaN before the first element), idx[v][0] its index,
// and open[v] stays true until the queue holds a NaN (nothing can beat a NaN
// that came first).  One offer costs a predicated compare and two selects:
// the unordered test !(x <= thr) is true for x > thr, for a NaN x, and while
// the queue is still empty; IEEE equality makes -0 tie +0 for free.
// k_b > 1: keys are kept sorted in registers; thr[v] is the float value of the
// worst kept entry (NaN while the queue is not full or when that entry is a
// NaN), so the common case costs one float comparison.
template <int KB>
struct Queues {
  uint32_t key[4][KB];
  uint32_t idx[4][KB];
  float thr[4];
  bool open[4];

  static constexpr uint32_t kEmptyIdx = 0xffffffffu;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        key[v][s] = 0u;
        idx[v][s] = kEmptyIdx;
      }
      thr[v] = __uint_as_float(0x7fffffffu);
      open[v] = true;
    }
  }

  template <int V>
  __device__ __forceinline__ void take1(float x, uint32_t i) {
    const bool p = open[V] && !(x <= thr[V]);
    thr[V] = p ? x : thr[V];
    idx[V][0] = p ? i : idx[V][0];
    open[V] = open[V] && !(p && (x != x));
  }

  template <int V>
  __device__ __forceinline__ void insert(float x, uint32_t i) {
    const uint32_t kx = order_key(x);
    if (kx <= key[V][KB - 1]) return;
    bool placed = false;
#pragma unroll
    for (int s = KB - 1; s >= 0; --s) {
      const int up_s = s > 0 ? s - 1 : 0;
      const bool up = (s > 0) && (kx > key[V][up_s]);
      const uint32_t nk = up ? key[V][up_s] : kx;
      const uint32_t ni = up ? idx[V][up_s] : i;
      if (!placed) {
        key[V][s] = nk;
        idx[V][s] = ni;
      }
      placed = placed || !up;
    }
    thr[V] = key[V][KB - 1] ? key_value(key[V][KB - 1]) : __uint_as_float(0x7fffffffu);
  }

  template <int V>
  __device__ __forceinline__ void offer(float x, uint32_t i) {
    if (KB == 1) {
      take1<V>(x, i);
    } else if (!(x <= thr[V])) {
      insert<V>(x, i);
    }
  }

  // Four consecutive positions i0..i0+3 (one per queue).
  __device__ __forceinline__ void offer4(const float4 x, uint32_t i0) {
    offer<0>(x.x, i0);
    offer<1>(x.y, i0 + 1);
    offer<2>(x.z, i0 + 2);
    offer<3>(x.w, i0 + 3);
  }

  // U float4 values x[u] at positions i0[u]..i0[u]+3, in increasing position
  // order per queue; valid[u] false skips x[u].  For k_b > 1 the threshold tests
  // of one queue are combined so that a queue whose U values all fail costs a
  // single branch.
  template <int U>
  __device__ __forceinline__ void offer_rows(const float4 (&x)[U], const uint32_t (&i0)[U],
                                             const bool (&valid)[U]) {
    if (KB == 1) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (valid[u]) offer4(x[u], i0[u]);
      return;
    }
    bool any0 = false, any1 = false, any2 = false, any3 = false;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      any0 |= valid[u] && !(x[u].x <= thr[0]);
      any1 |= valid[u] && !(x[u].y <= thr[1]);
      any2 |= valid[u] && !(x[u].z <= thr[2]);
      any3 |= valid[u] && !(x[u].w <= thr[3]);
    }
    if (any0) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (valid[u]) offer<0>(x[u].x, i0[u]);
    }
    if (any1) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (valid[u]) offer<1>(x[u].y, i0[u] + 1);
    }
    if (any2) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (valid[u]) offer<2>(x[u].z, i0[u] + 2);
    }
    if (any3) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (valid[u]) offer<3>(x[u].w, i0[u] + 3);
    }
  }

  // Store queue v as packed candidates at dst[0..KB).
  __device__ __forceinline__ void store(int v, uint64_t* dst) const {
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      uint64_t p = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        if (w == v) {
          if (KB == 1)
            p = idx[w][0] != kEmptyIdx ? pack(order_key(thr[w]), idx[w][0]) : 0ull;
          else
            p = pack(key[w][s], idx[w][s]);
        }
      }
      dst[s] = p;
    }
  }
};

// Insert packed candidate c into best[0..KB) (best-first, strict order).
template <int KB>
__device__ __forceinline__ void keep_best(uint64_t (&best)[KB], uint64_t c) {
  if (c <= best[KB - 1]) return;
  bool placed = false;
#pragma unroll
  for (int s = KB - 1; s >= 0; --s) {
    const int up_s = s > 0 ? s - 1 : 0;
    const bool up = (s > 0) && (c > best[up_s]);
    const uint64_t nv = up ? best[up_s] : c;
    if (!placed) best[s] = nv;
    placed = placed || !up;
  }
}

// Lane slot l (0 <= l < kLanes) holds the top-KB of the piece positions
// congruent to l modulo L*b, with L = kLanes / b lanes per bucket (b <= kLanes),
// so its bucket is (a + l) mod b for a piece starting at row position a.
// Writes dst[j*KB + s], j = absolute bucket.  dst may be shared or global.
template <int KB>
__device__ __forceinline__ void merge_lanes(const uint64_t* lanebuf, int b, int64_t a,
                                            uint64_t* dst, int T) {
  const int L = kLanes / b;
  const int a_mod = static_cast<int>(a % b);
  for (int beta = threadIdx.x; beta < b; beta += T) {
    uint64_t best[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s) best[s] = 0;
    for (int m = 0; m < L; ++m) {
      const uint64_t* src = lanebuf + static_cast<size_t>(beta + m * b) * KB;
#pragma unroll
      for (int s = 0; s < KB; ++s) keep_best<KB>(best, src[s]);
    }
    int j = beta + a_mod;
    if (j >= b) j -= b;
#pragma unroll
    for (int s = 0; s < KB; ++s) dst[static_cast<size_t>(j) * KB + s] = best[s];
  }
}

// ------------------------------------------------------------------ Stage 2
__device__ __forceinline__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Bitonic sort of s[0..N) (N a power of two) into descending order by the
// first T threads of the CTA.
__device__ __forceinline__ void bitonic_desc(uint64_t* s, int N, int T) {
  for (int size = 2; size <= N; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (N >> 1); t += T) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t x = s[lo], y = s[hi];
        if (desc ? (x < y) : (x > y)) {
          s[lo] = y;
          s[hi] = x;
        }
      }
      group_sync(T);
    }
  }
}

enum ValueSource { kGatherInput = 0, kFromKey = 1 };

// cand[0..C) holds the Stage-1 candidates (0 = empty).  Sorts them best-first
// and writes the first k (Stage 2: only the k best survive when C > k), padding
// with -inf / -1.  Values either come from the input row (exact input bits)
// or from the key (fused scores).  cand must have room for next_pow2(C).
template <ValueSource VS>
__device__ __forceinline__ void finalize_row(uint64_t* cand, int C, int k, const float* xrow,
                                             float* ov, int32_t* oi, int T) {
  const int N = next_pow2(C);
  for (int i = C + threadIdx.x; i < N; i += T) cand[i] = 0;
  group_sync(T);
  bitonic_desc(cand, N, T);
  for (int s = threadIdx.x; s < k; s += T) {
    const uint64_t p = s < N ? cand[s] : 0ull;
    if (p) {
      const uint32_t i = packed_idx(p);
      float v;
      if (VS == kGatherInput)
        v = __ldg(xrow + i);
      else
        v = key_value(packed_key(p));
      ov[s] = v;
      oi[s] = static_cast<int32_t>(i);
    } else {
      ov[s] = __int_as_float(0xff800000);
      oi[s] = -1;
    }
  }
  group_sync(T);
}

// ------------------------------------------------------------------ pieces
struct RowSplit {
  int64_t rows, n;  // row length in elements (scores or keys)
  int64_t E;        // rows * n
  int64_t units;    // E / align
  int G, align;
  uint32_t* tickets;  // [rows], zero between calls
  uint64_t* slots;    // [G][2][b*KB]
};

__device__ __forceinline__ int64_t cta_start(const RowSplit& rs, int c) {
  return part_start(rs.units, rs.G, c, rs.align, rs.E);
}

// Finish one piece [a, a+len) of row r whose per-lane queues are in lanebuf,
// by the first kThreads threads of the CTA.  A whole-row piece runs Stage 2 at
// once; a partial piece publishes its per-bucket lists and the last piece of
// the row to finish runs the merge (and clears what it read).
template <int KB, ValueSource VS>
__device__ void finish_piece(const RowSplit& rs, int b, int k, int64_t r, int64_t a, int64_t len,
                             const uint64_t* lanebuf, uint64_t* cand, const float* xrow,
                             float* out_vals, int32_t* out_idx, int* s_flag) {
  constexpr int T = kThreads;
  const int C = b * KB;
  float* ov = out_vals + r * static_cast<int64_t>(k);
  int32_t* oi = out_idx + r * static_cast<int64_t>(k);
  if (a == 0 && len == rs.n) {
    merge_lanes<KB>(lanebuf, b, 0, cand, T);
    group_sync(T);
    finalize_row<VS>(cand, C, k, xrow, ov, oi, T);
    return;
  }
  const int64_t row0 = r * rs.n;
  const int me = blockIdx.x;
  const int slot = (cta_start(rs, me) / rs.n == r) ? 0 : 1;
  uint64_t* mine = rs.slots + (static_cast<size_t>(me) * 2 + slot) * C;
  merge_lanes<KB>(lanebuf, b, a, mine, T);
  __threadfence();
  group_sync(T);
  const int c_first = part_of(row0, rs.units, rs.G, rs.align);
  const int c_last = part_of(row0 + rs.n - 1, rs.units, rs.G, rs.align);
  if (threadIdx.x == 0) {
    const unsigned pieces = static_cast<unsigned>(c_last - c_first + 1);
    const unsigned old = atomicAdd(rs.tickets + r, 1u);
    *s_flag = (old == pieces - 1) ? 1 : 0;
  }
  group_sync(T);
  const bool last = *s_flag != 0;
  group_sync(T);  // everyone has read the flag before it can be reused
  if (!last) return;
  __threadfence();
  for (int j = threadIdx.x; j < b; j += T) {
    uint64_t best[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s) best[s] = 0;
    for (int c = c_first; c <= c_last; ++c) {
      const int sl = (cta_start(rs, c) / rs.n == r) ? 0 : 1;
      uint64_t* src = rs.slots + (static_cast<size_t>(c) * 2 + sl) * C + static_cast<size_t>(j) * KB;
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        keep_best<KB>(best, __ldcg(src + s));
        __stcg(src + s, 0ull);  // leave the workspace zeroed
      }
    }
#pragma unroll
    for (int s = 0; s < KB; ++s) cand[static_cast<size_t>(j) * KB + s] = best[s];
  }
  group_sync(T);
  finalize_row<VS>(cand, C, k, xrow, ov, oi, T);
  if (threadIdx.x == 0) rs.tickets[r] = 0u;  // leave the workspace zeroed
}

}  // namespace tk
