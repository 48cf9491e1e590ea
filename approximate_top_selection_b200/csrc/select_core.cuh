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
// Register queues per thread.  Queue v keeps the best KB elements offered
// to it, best-first, as (value, index) in the float domain; an empty slot holds
// -inf with index kEmpty.  Elements reach a queue in increasing index order, so
// "x ranks above slot s" needs no index comparison: with x neither NaN nor -inf
// it is exactly the IEEE test x > val[s] (ties, -0 == +0 included, keep the
// earlier element; a NaN slot is never beaten; an empty slot's -inf always is).
// That fast update is branch-free: KB compares and 4 selects per slot.  NaN or
// -inf values take the exact update, which compares order-preserving keys.
//
// Stored indices are "base" positions: queue v of a thread stores p - v for an
// element at position p, so one base per float4 serves its four queues; the
// true position is restored in store().
//
// NQ queues per thread: four for the float4 layout (k_b <= 2), one or two for
// the wide k_b > 2 kernel.  The four-queue members (offer4, offer_tile, ...)
// exist only for NQ == 4.
#ifndef TOPK_MINMAX_QUEUES
#define TOPK_MINMAX_QUEUES 1
#endif

template <int KB, int NQ = 4>
struct Queues {
  float val[NQ][KB];
  uint32_t idx[NQ][KB];

  static constexpr uint32_t kEmpty = 0xffffffffu;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int v = 0; v < NQ; ++v) {
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        val[v][s] = __int_as_float(0xff800000);
        idx[v][s] = kEmpty;
      }
    }
  }

  // Shift-insert given the monotone flags above[s] ("x ranks above slot s").
  template <int V>
  __device__ __forceinline__ void place(const bool (&above)[KB], float x, uint32_t base) {
#pragma unroll
    for (int s = KB - 1; s >= 0; --s) {
      if (s > 0) {
        const bool up = above[s > 0 ? s - 1 : 0];
        const float vs = above[s] ? x : val[V][s];
        const uint32_t is = above[s] ? base : idx[V][s];
        val[V][s] = up ? val[V][s > 0 ? s - 1 : 0] : vs;
        idx[V][s] = up ? idx[V][s > 0 ? s - 1 : 0] : is;
      } else {
        val[V][0] = above[0] ? x : val[V][0];
        idx[V][0] = above[0] ? base : idx[V][0];
      }
    }
  }

  // x is neither NaN nor -inf.
  template <int V>
  __device__ __forceinline__ void insert_fast(float x, uint32_t base) {
    bool above[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s) above[s] = x > val[V][s];
#if TOPK_MINMAX_QUEUES
    if constexpr (KB <= 2) {
    // The values as a max/min insertion network: slot s keeps the larger of
    // itself and what the slots above pass down, and passes the smaller on.
    // A NaN slot (only ever at the top) stays (max.NaN) and passes x on
    // (fminf returns the non-NaN operand); with no NaN and x not -inf this
    // is the sorted insert.  Each value depends on its own slot through one
    // operation only, which shortens the chain between consecutive elements.
    // Indices follow the strict comparisons, so ties keep the earlier element.
    // Used for k_b <= 2 (the branch-free update of every element).
#pragma unroll
    for (int s = KB - 1; s > 0; --s)
      idx[V][s] = above[s - 1] ? idx[V][s - 1] : (above[s] ? base : idx[V][s]);
    idx[V][0] = above[0] ? base : idx[V][0];
    float carry = x;
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      const float v = val[V][s];
      val[V][s] = fmax_nan(v, carry);
      if (s + 1 < KB) carry = fminf(v, carry);
    }
    } else {
      place<V>(above, x, base);  // longer queues: the select chain measured faster
    }
#else
    place<V>(above, x, base);
#endif
  }

  // Any x (NaN ranks above +inf; all NaNs tie).
  template <int V>
  __device__ __forceinline__ void insert_exact(float x, uint32_t base) {
    const uint32_t kx = order_key(x);
    bool above[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s)
      above[s] = (idx[V][s] == kEmpty) || kx > order_key(val[V][s]);
    place<V>(above, x, base);
  }

  template <int V>
  __device__ __forceinline__ void offer(float x, uint32_t base) {
    if (x > __int_as_float(0xff800000))
      insert_fast<V>(x, base);
    else
      insert_exact<V>(x, base);
  }

  __device__ __forceinline__ static bool special(const float4 x) {
    const float ninf = __int_as_float(0xff800000);
    return !(x.x > ninf) | !(x.y > ninf) | !(x.z > ninf) | !(x.w > ninf);
  }

  __device__ __forceinline__ void fast4(const float4 x, uint32_t base) {
    insert_fast<0>(x.x, base);
    insert_fast<1>(x.y, base);
    insert_fast<2>(x.z, base);
    insert_fast<3>(x.w, base);
  }

  __device__ __forceinline__ void exact4(const float4 x, uint32_t base, int valid = 4) {
    if (valid > 0) insert_exact<0>(x.x, base);
    if (valid > 1) insert_exact<1>(x.y, base);
    if (valid > 2) insert_exact<2>(x.z, base);
    if (valid > 3) insert_exact<3>(x.w, base);
  }

  // Positions base..base+3, one per queue.
  __device__ __forceinline__ void offer4(const float4 x, uint32_t base) {
    if (special(x))
      exact4(x, base);
    else
      fast4(x, base);
  }

  // U float4 values at bases base[u] (increasing), all valid.  One NaN-keeping
  // min over all 4U values decides whether any of them is NaN or -inf.
  template <int U>
  __device__ __forceinline__ void offer_tile(const float4 (&x)[U], const uint32_t (&base)[U]) {
    float all[4 * U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      all[4 * u] = x[u].x;
      all[4 * u + 1] = x[u].y;
      all[4 * u + 2] = x[u].z;
      all[4 * u + 3] = x[u].w;
    }
    const bool sp = !(min_nan_all<4 * U>(all) > __int_as_float(0xff800000));
    if (!sp) {
#pragma unroll
      for (int u = 0; u < U; ++u) fast4(x[u], base[u]);
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) exact4(x[u], base[u]);
    }
  }

  // Store queue v as packed candidates at dst[0..KB).
  __device__ __forceinline__ void store(int v, uint64_t* dst) const {
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      uint64_t p = 0;
#pragma unroll
      for (int w = 0; w < NQ; ++w) {
        if (w == v && idx[w][s] != kEmpty)
          p = pack(order_key(val[w][s]), idx[w][s] + static_cast<uint32_t>(w));
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

// Lane slot l (0 <= l < nl) holds the top-KB of the piece positions
// congruent to l modulo L*b, with L = nl / b lanes per bucket (b <= nl),
// so its bucket is (a + l) mod b for a piece starting at row position a.
// Writes dst[j*KB + s], j = absolute bucket.  dst may be shared or global.
template <int KB>
__device__ __forceinline__ void merge_lanes(const uint64_t* lanebuf, int b, int64_t a,
                                            uint64_t* dst, int T, int nl = kLanes) {
  const int L = nl / b;
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

// ------------------------------------------------------------------ register sort
// Bitonic sort into descending order of the N = kThreads * EPT packed keys held
// by the first kThreads threads, blocked (thread t holds elements t*EPT + j).
// Exchanges inside a thread use registers, exchanges inside a warp use
// shuffles, and only strides that cross warps go through shared memory (xchg,
// N entries), so a 512-key sort needs 6 shared-memory rounds instead of 45.
__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a > b ? b : a; }

// One compare-exchange round of the network (SIZE, STRIDE fixed at compile time).
// Rounds whose stride crosses warps exchange through shared memory: with one
// buffer (xchg2 == nullptr) each such round needs a barrier after its writes
// and another after its reads (the next round rewrites the buffer); with two
// buffers used in turn, the barrier after the next round's writes already
// orders this round's reads before any rewrite, so one barrier per round.
template <int EPT, int SIZE, int STRIDE>
__device__ __forceinline__ void bitonic_round(uint64_t (&v)[EPT], uint64_t* xchg, uint64_t* xchg2,
                                              int& flip) {
  const int t = threadIdx.x;
  if constexpr (STRIDE >= 32 * EPT) {
    uint64_t* xb = (xchg2 != nullptr && flip) ? xchg2 : xchg;
#pragma unroll
    for (int j = 0; j < EPT; ++j) xb[t * EPT + j] = v[j];
    group_sync(kThreads);
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = t * EPT + j;
      const uint64_t o = xb[e ^ STRIDE];
      const bool keep_max = ((e & SIZE) == 0) == ((e & STRIDE) == 0);
      v[j] = keep_max ? umax64(v[j], o) : umin64(v[j], o);
    }
    if (xchg2 == nullptr)
      group_sync(kThreads);
    else
      flip ^= 1;
  } else if constexpr (STRIDE >= EPT) {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = t * EPT + j;
      const uint64_t o = __shfl_xor_sync(0xffffffffu, v[j], STRIDE / EPT);
      const bool keep_max = ((e & SIZE) == 0) == ((e & STRIDE) == 0);
      v[j] = keep_max ? umax64(v[j], o) : umin64(v[j], o);
    }
  } else {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      if ((j & STRIDE) == 0) {
        const int jj = j | STRIDE;
        const int e = t * EPT + j;
        const uint64_t a = v[j], b = v[jj];
        const bool desc = (e & SIZE) == 0;
        v[j] = desc ? umax64(a, b) : umin64(a, b);
        v[jj] = desc ? umin64(a, b) : umax64(a, b);
      }
    }
  }
  if constexpr (STRIDE > 1) bitonic_round<EPT, SIZE, STRIDE / 2>(v, xchg, xchg2, flip);
}

template <int EPT, int SIZE>
__device__ __forceinline__ void bitonic_sizes(uint64_t (&v)[EPT], uint64_t* xchg, uint64_t* xchg2,
                                              int& flip) {
  bitonic_round<EPT, SIZE, SIZE / 2>(v, xchg, xchg2, flip);
  if constexpr (SIZE < kThreads * EPT) bitonic_sizes<EPT, SIZE * 2>(v, xchg, xchg2, flip);
}

// xchg2: nullable second exchange buffer of kThreads * EPT entries.
template <int EPT>
__device__ __forceinline__ void block_sort_desc(uint64_t (&v)[EPT], uint64_t* xchg,
                                                uint64_t* xchg2 = nullptr) {
  int flip = 0;
  bitonic_sizes<EPT, 2>(v, xchg, xchg2, flip);
  if (xchg2 != nullptr) group_sync(kThreads);  // the last round's reads, before any reuse
}

// Bitonic network on the 32 * EPT keys of one warp, strided (lane l holds
// elements j * 32 + l): strides below 32 are shuffles, larger ones register
// swaps; no shared memory, no block barrier.
template <int EPT, int SIZE, int STRIDE>
__device__ __forceinline__ void warp_bitonic_round(uint64_t (&v)[EPT], int lane) {
  if constexpr (STRIDE >= 32) {
    constexpr int DJ = STRIDE / 32;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      if ((j & DJ) == 0) {
        const bool desc = ((j * 32) & SIZE) == 0;
        const uint64_t a = v[j], b = v[j | DJ];
        v[j] = desc ? umax64(a, b) : umin64(a, b);
        v[j | DJ] = desc ? umin64(a, b) : umax64(a, b);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = j * 32 + lane;
      const uint64_t o = __shfl_xor_sync(0xffffffffu, v[j], STRIDE);
      const bool keep_max = ((e & SIZE) == 0) == ((lane & STRIDE) == 0);
      v[j] = keep_max ? umax64(v[j], o) : umin64(v[j], o);
    }
  }
  if constexpr (STRIDE > 1) warp_bitonic_round<EPT, SIZE, STRIDE / 2>(v, lane);
}

template <int EPT, int SIZE>
__device__ __forceinline__ void warp_bitonic_sizes(uint64_t (&v)[EPT], int lane) {
  warp_bitonic_round<EPT, SIZE, SIZE / 2>(v, lane);
  if constexpr (SIZE < 32 * EPT) warp_bitonic_sizes<EPT, SIZE * 2>(v, lane);
}

// Value of an output candidate: from its key, except that a zero or NaN is
// re-read from the input row so that -0.0 and NaN payloads keep their bits.
// V is the element type of the output: float, or uint16_t holding bf16 bits
// (a bf16 widened to float is exact, so its upper 16 bits give it back).
template <int VS, typename V>
__device__ __forceinline__ V candidate_value(uint64_t p, const V* xrow) {
  const float v = key_value(packed_key(p));
  if constexpr (sizeof(V) == 4) {
    if (VS == 0 && (v == 0.0f || v != v)) return __ldg(xrow + packed_idx(p));
    return v;
  } else {
    if (VS == 0 && (v == 0.0f || v != v)) return xrow[packed_idx(p)];
    return static_cast<V>(__float_as_uint(v) >> 16);
  }
}

template <typename V>
__device__ __forceinline__ V negative_infinity() {
  if constexpr (sizeof(V) == 4)
    return __int_as_float(0xff800000);
  else
    return static_cast<V>(0xff80u);
}

template <int EPT, int VS, typename V>
__device__ __noinline__ void finalize_row_regs(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                               int32_t* oi, uint64_t* xchg2) {
  constexpr int N = kThreads * EPT;
  const int t = threadIdx.x;
  uint64_t v[EPT];
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = t * EPT + j;
    v[j] = e < C ? cand[e] : 0ull;
  }
  group_sync(kThreads);  // cand is reused as the exchange buffer
  block_sort_desc<EPT>(v, cand, xchg2);
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = t * EPT + j;
    if (e < k) {
      if (v[j]) {
        ov[e] = candidate_value<VS, V>(v[j], xrow);
        oi[e] = static_cast<int32_t>(packed_idx(v[j]));
      } else {
        ov[e] = negative_infinity<V>();
        oi[e] = -1;
      }
    }
  }
  for (int e = N + t; e < k; e += kThreads) {
    ov[e] = negative_infinity<V>();
    oi[e] = -1;
  }
  group_sync(kThreads);
}

// Candidate buffer entries the register sort needs for C candidates.
__host__ __device__ __forceinline__ int sort_capacity(int C) {
  int n = kThreads;
  while (n < C) n <<= 1;
  return n;
}

// Shared-memory bytes of the Stage-2 buffer for C candidates: the sort
// buffer plus the radix-select histogram and counters behind it.
constexpr int kStage2Extra = 2048;
__host__ __device__ __forceinline__ size_t stage2_bytes(int C) {
  return static_cast<size_t>(sort_capacity(C)) * 8 + kStage2Extra;
}

template <ValueSource VS, typename V>
__device__ __forceinline__ void finalize_row_fast(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                                  int32_t* oi, uint64_t* xchg2 = nullptr,
                                                  int xchg2_cap = 0);

// Stage 2 for a small k (k <= M = 32 * EPT, C <= 8 M): every warp sorts its M
// candidates in registers, then in three rounds warp w < h takes the list of
// warp w + h from shared memory and keeps the M best of the two (the bitonic
// merge: max(own[e], partner[M-1-e]) is a bitonic sequence holding the M
// best, and log2(M) more rounds sort it).  Warp 0 ends with the M best,
// sorted, and writes the first k.  Fewer exchanges and barriers than sorting
// all C when only k of them are wanted.
template <int EPT, int VS, typename V>
__device__ __noinline__ void finalize_row_topk_warps(uint64_t* cand, int C, int k, const V* xrow,
                                                     V* ov, int32_t* oi) {
  constexpr int M = 32 * EPT;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  uint64_t v[EPT];
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = w * M + j * 32 + lane;
    v[j] = e < C ? cand[e] : 0ull;
  }
  warp_bitonic_sizes<EPT, 2>(v, lane);
  group_sync(kThreads);  // every candidate has been read
#pragma unroll
  for (int h = kThreads / 64; h >= 1; h >>= 1) {
    if (w >= h && w < 2 * h) {
#pragma unroll
      for (int j = 0; j < EPT; ++j) cand[(w - h) * M + j * 32 + lane] = v[j];
    }
    group_sync(kThreads);
    if (w < h) {
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        const int e = j * 32 + lane;
        v[j] = umax64(v[j], cand[w * M + (M - 1 - e)]);
      }
      warp_bitonic_round<EPT, 2 * M, M / 2>(v, lane);  // descending merge of a bitonic sequence
    }
    group_sync(kThreads);
  }
  if (w == 0) {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = j * 32 + lane;
      if (e < k) {
        if (v[j]) {
          ov[e] = candidate_value<VS, V>(v[j], xrow);
          oi[e] = static_cast<int32_t>(packed_idx(v[j]));
        } else {
          ov[e] = negative_infinity<V>();
          oi[e] = -1;
        }
      }
    }
  }
  group_sync(kThreads);
}

// Stage 2 when the candidates far outnumber k: find the k-th largest packed
// key with 8-bit radix histograms (most significant digit first; keys are
// unique, so at most 8 passes, and the walk stops as soon as the boundary
// digit holds exactly the elements still needed), gather the selected keys
// and sort only those.  Same result as sorting all C and keeping k.
template <int EPT, int VS, typename V>
__device__ __noinline__ void finalize_row_select(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                                 int32_t* oi, uint64_t* xchg2, int xchg2_cap) {
  const int t = threadIdx.x;
  uint32_t* hist = reinterpret_cast<uint32_t*>(cand + sort_capacity(C));  // 256 bins
  int* misc = reinterpret_cast<int*>(hist + 256);                        // digit, above, count, n
  uint64_t v[EPT];
  uint64_t any_bits = 0ull, all_bits = ~0ull;
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = j * kThreads + t;
    v[j] = e < C ? cand[e] : 0ull;
    if (v[j] != 0ull) {
      any_bits |= v[j];
      all_bits &= v[j];
    }
  }
  // The bytes above the highest bit in which the real keys differ are common
  // to all of them: the digit walk starts below them.
  uint32_t* red = reinterpret_cast<uint32_t*>(misc + 4);  // OR lo/hi, AND lo/hi
  if (t == 0) {
    red[0] = 0u;
    red[1] = 0u;
    red[2] = ~0u;
    red[3] = ~0u;
  }
  group_sync(kThreads);
  {
    const uint32_t o0 = __reduce_or_sync(0xffffffffu, static_cast<uint32_t>(any_bits));
    const uint32_t o1 = __reduce_or_sync(0xffffffffu, static_cast<uint32_t>(any_bits >> 32));
    const uint32_t a0 = __reduce_and_sync(0xffffffffu, static_cast<uint32_t>(all_bits));
    const uint32_t a1 = __reduce_and_sync(0xffffffffu, static_cast<uint32_t>(all_bits >> 32));
    if ((t & 31) == 0) {
      atomicOr(red, o0);
      atomicOr(red + 1, o1);
      atomicAnd(red + 2, a0);
      atomicAnd(red + 3, a1);
    }
  }
  group_sync(kThreads);
  const uint64_t common_and = red[2] | (static_cast<uint64_t>(red[3]) << 32);
  const uint64_t differ = (red[0] | (static_cast<uint64_t>(red[1]) << 32)) ^ common_and;
  int shift = differ ? ((63 - __clzll(static_cast<long long>(differ))) & ~7) : 0;
  uint64_t prefix = shift < 56 ? (common_and & ~((1ull << (shift + 8)) - 1ull)) : 0ull;
  int need = k;
  bool all_real = false;
  for (; shift >= 0; shift -= 8) {
    for (int i = t; i < 256; i += kThreads) hist[i] = 0u;
    group_sync(kThreads);
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const bool match = v[j] != 0ull && (shift == 56 || (v[j] >> (shift + 8)) == (prefix >> (shift + 8)));
      // Candidates are often concentrated in a few bins: one atomic per
      // distinct bin of the warp instead of one per lane.
      const uint32_t bin = match ? static_cast<uint32_t>((v[j] >> shift) & 255u) : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (match && (t & 31) == __ffs(peers) - 1) atomicAdd(hist + bin, static_cast<uint32_t>(__popc(peers)));
    }
    group_sync(kThreads);
    if (t < 32) {
      // Lane l holds bins 255-8l down to 248-8l; find the digit that holds the
      // need-th largest key.
      int c8[8];
      int local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c8[i] = static_cast<int>(hist[255 - 8 * t - i]);
        local += c8[i];
      }
      int incl = local;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, m);
        if (t >= m) incl += y;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
      if (t == 0) misc[3] = total;
      if (hit) {
        const int l = __ffs(hit) - 1;
        if (t == l) {
          int above = incl - local;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (above + c8[i] >= need) {
              misc[0] = 255 - 8 * t - i;
              misc[1] = above;
              misc[2] = c8[i];
              break;
            }
            above += c8[i];
          }
        }
      }
    }
    group_sync(kThreads);
    if (misc[3] < need) {  // fewer candidates than still needed: take them all
      all_real = true;
      group_sync(kThreads);
      break;
    }
    const int d = misc[0], above = misc[1], cnt = misc[2];
    group_sync(kThreads);  // misc is rewritten by the next pass
    prefix |= static_cast<uint64_t>(d) << shift;
    need -= above;
    if (cnt == need) break;  // every key on this prefix is selected
  }
  // Selected: keys whose digits down to `shift` are >= the prefix (or, when
  // there were fewer than needed, every real key matching the prefix so far).
  if (t == 0) misc[3] = 0;
  group_sync(kThreads);
  const int sh = shift < 0 ? 0 : shift;
  const int lane = t & 31;
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    bool sel;
    if (all_real)
      sel = v[j] != 0ull && (sh == 56 ? true : (v[j] >> (sh + 8)) >= (prefix >> (sh + 8)));
    else
      sel = v[j] != 0ull && (v[j] >> sh) >= (prefix >> sh);
    // One counter update per warp, not per selected key.
    const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel_mask) {
      const int leader = __ffs(sel_mask) - 1;
      int at = 0;
      if (lane == leader) at = atomicAdd(misc + 3, __popc(sel_mask));
      at = __shfl_sync(0xffffffffu, at, leader);
      if (sel) cand[at + __popc(sel_mask & ((1u << lane) - 1u))] = v[j];
    }
  }
  group_sync(kThreads);
  const int kept = misc[3];
  group_sync(kThreads);
  finalize_row_fast<static_cast<ValueSource>(VS), V>(cand, kept, k, xrow, ov, oi, xchg2, xchg2_cap);
}

template <ValueSource VS, typename V>
__device__ __forceinline__ void finalize_row(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                             int32_t* oi, int T);

template <int EPT, int VS, typename V>
__device__ __noinline__ void finalize_row_select(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                                 int32_t* oi, uint64_t* xchg2, int xchg2_cap);

// Stage 2 for the streaming kernels (kThreads threads): up to 8 keys per
// thread are sorted in registers; larger candidate sets use the shared-memory
// network.  xchg2 (nullable, xchg2_cap entries): spare shared memory for a
// second exchange buffer of the register sort.
template <ValueSource VS, typename V>
__device__ __forceinline__ void finalize_row_fast(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                                  int32_t* oi, uint64_t* xchg2, int xchg2_cap) {
  const int ept = sort_capacity(C) / kThreads;
  uint64_t* x2 = ept * kThreads <= xchg2_cap ? xchg2 : nullptr;
  switch (ept) {
    case 1: finalize_row_regs<1, VS, V>(cand, C, k, xrow, ov, oi, x2); break;
    case 2: finalize_row_regs<2, VS, V>(cand, C, k, xrow, ov, oi, x2); break;
    case 4: finalize_row_regs<4, VS, V>(cand, C, k, xrow, ov, oi, x2); break;
    case 8: finalize_row_regs<8, VS, V>(cand, C, k, xrow, ov, oi, x2); break;
    default: finalize_row<VS, V>(cand, C, k, xrow, ov, oi, kThreads); break;
  }
}

// cand[0..C) holds the Stage-1 candidates (0 = empty).  Sorts them best-first
// and writes the first k (Stage 2: only the k best survive when C > k), padding
// with -inf / -1.  Values either come from the input row (exact input bits)
// or from the key (fused scores).  cand must have room for next_pow2(C).
template <ValueSource VS, typename V>
__device__ __forceinline__ void finalize_row(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                             int32_t* oi, int T) {
  const int N = next_pow2(C);
  for (int i = C + threadIdx.x; i < N; i += T) cand[i] = 0;
  group_sync(T);
  bitonic_desc(cand, N, T);
  for (int s = threadIdx.x; s < k; s += T) {
    const uint64_t p = s < N ? cand[s] : 0ull;
    if (p) {
      const uint32_t i = packed_idx(p);
      ov[s] = VS == kGatherInput ? xrow[i] : candidate_value<VS, V>(p, xrow);
      oi[s] = static_cast<int32_t>(i);
    } else {
      ov[s] = negative_infinity<V>();
      oi[s] = -1;
    }
  }
  group_sync(T);
}

// Stage 2 entry of the streaming kernels: select first when that shrinks the
// sort (at least 1024 candidates and k under half of them), else sort all.
#ifndef TOPK_WARP_TOPK
#define TOPK_WARP_TOPK 1
#endif
// xchg2 (nullable, xchg2_cap entries): shared memory the caller no longer
// needs, used as a second exchange buffer by the register sort.
template <ValueSource VS, typename V>
__device__ __forceinline__ void stage2(uint64_t* cand, int C, int k, const V* xrow, V* ov,
                                       int32_t* oi, uint64_t* xchg2 = nullptr, int xchg2_cap = 0) {
  if (TOPK_WARP_TOPK && C > k && C <= 8 * kThreads) {
    const int ept = sort_capacity(C) / kThreads;
    if (k <= 32 * ept) {
      switch (ept) {
        case 2: finalize_row_topk_warps<2, VS, V>(cand, C, k, xrow, ov, oi); return;
        case 4: finalize_row_topk_warps<4, VS, V>(cand, C, k, xrow, ov, oi); return;
        case 8: finalize_row_topk_warps<8, VS, V>(cand, C, k, xrow, ov, oi); return;
        default: break;
      }
    }
  }
  if (C >= 1024 && 2 * k <= C && C <= 16 * kThreads) {
    switch (sort_capacity(C) / kThreads) {
      case 4: finalize_row_select<4, VS, V>(cand, C, k, xrow, ov, oi, xchg2, xchg2_cap); return;
      case 8: finalize_row_select<8, VS, V>(cand, C, k, xrow, ov, oi, xchg2, xchg2_cap); return;
      default: finalize_row_select<16, VS, V>(cand, C, k, xrow, ov, oi, xchg2, xchg2_cap); return;
    }
  }
  finalize_row_fast<VS, V>(cand, C, k, xrow, ov, oi, xchg2, xchg2_cap);
}

// ------------------------------------------------------------------ sampling tail
// Top-k sampling of one row by one warp: from the k selected pairs (v, ix),
// best-first, index ix[i] is drawn with probability w_i / sum w,
// w_i = exp((v_i - v_0) * inv_t), by inverse CDF with the uniform u: the
// first i whose running sum exceeds u * sum w, else (rounding) the last entry
// of positive weight.  Padding (-1) and -inf weigh 0; a NaN or +inf best
// entry is drawn outright; no candidate draws -1.  Each lane sums a contiguous
// slice in fp32 and a shuffle scan gives it the weight before its slice.
// v and ix are plain loads: they may have been written by this CTA.  V is
// float, or uint16_t holding bf16 bits (widened to fp32 exactly).
__device__ __forceinline__ float sample_value(const float* v, int i) { return v[i]; }
__device__ __forceinline__ float sample_value(const uint16_t* v, int i) {
  return __uint_as_float(static_cast<uint32_t>(v[i]) << 16);
}

template <typename V>
__device__ __forceinline__ void sample_row_warp(const V* v, const int32_t* ix, int k, float inv_t,
                                                float u, int32_t* token) {
  const int lane = threadIdx.x & 31;
  const int32_t i0 = ix[0];
  const float v0 = sample_value(v, 0);
  if (i0 < 0 || v0 != v0 || v0 == __int_as_float(0x7f800000)) {
    if (lane == 0) *token = i0;  // -1 (no candidate), or the NaN / +inf entry
    return;
  }
  const int per = (k + 31) / 32;
  const int beg = min(lane * per, k), end = min(beg + per, k);
  float part = 0.0f;
  for (int i = beg; i < end; ++i)
    if (ix[i] >= 0) part += expf((sample_value(v, i) - v0) * inv_t);
  float incl = part;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const float total = __shfl_sync(0xffffffffu, incl, 31);
  const float target = u * total;
  float run = incl - part;
  int32_t pick = -1, last = -1;
  for (int i = beg; i < end; ++i) {
    if (ix[i] < 0) continue;
    const float w = expf((sample_value(v, i) - v0) * inv_t);
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
  if (lane == 0) *token = t;
}

// Optional sampling tail of a selection call (token == nullptr: none).
struct SampleTail {
  const float* u;  // [rows] uniforms
  int32_t* token;  // [rows]
  float inv_t;     // 1 / temperature
};

// Out of line so that the streaming loop of the selection kernels keeps its
// registers: the draw runs once per row, after Stage 2.
template <typename V>
__device__ __noinline__ void sample_row_warp_call(const V* v, const int32_t* ix, int k,
                                                  float inv_t, float u, int32_t* token) {
  sample_row_warp<V>(v, ix, k, inv_t, u, token);
}

// After Stage 2 of row r wrote ov / oi (and the CTA met at a barrier): warp 0
// draws the row's token.
template <typename V>
__device__ __forceinline__ void run_sample_tail(const SampleTail& tail, int64_t r, int k,
                                                const V* ov, const int32_t* oi) {
  if (tail.token != nullptr && threadIdx.x < 32)
    sample_row_warp_call<V>(ov, oi, k, tail.inv_t, __ldg(tail.u + r), tail.token + r);
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
template <int KB, ValueSource VS, typename V>
__device__ void finish_piece(const RowSplit& rs, int b, int k, int64_t r, int64_t a, int64_t len,
                             const uint64_t* lanebuf, uint64_t* cand, const V* xrow, V* out_vals,
                             int32_t* out_idx, int* s_flag, int nl = kLanes,
                             const SampleTail& tail = SampleTail{nullptr, nullptr, 1.0f}) {
  constexpr int T = kThreads;
  const int C = b * KB;
  V* ov = out_vals + r * static_cast<int64_t>(k);
  int32_t* oi = out_idx + r * static_cast<int64_t>(k);
  // After the lanes are merged their buffer is free: Stage 2 may use it.
  uint64_t* spare = const_cast<uint64_t*>(lanebuf);
  const int spare_cap = nl * KB;
  if (a == 0 && len == rs.n) {
    merge_lanes<KB>(lanebuf, b, 0, cand, T, nl);
    group_sync(T);
    stage2<VS, V>(cand, C, k, xrow, ov, oi, spare, spare_cap);
    run_sample_tail<V>(tail, r, k, ov, oi);
    return;
  }
  const int64_t row0 = r * rs.n;
  const int me = blockIdx.x;
  const int slot = (cta_start(rs, me) / rs.n == r) ? 0 : 1;
  uint64_t* mine = rs.slots + (static_cast<size_t>(me) * 2 + slot) * C;
  merge_lanes<KB>(lanebuf, b, a, mine, T, nl);
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
  stage2<VS, V>(cand, C, k, xrow, ov, oi, spare, spare_cap);
  run_sample_tail<V>(tail, r, k, ov, oi);
  if (threadIdx.x == 0) rs.tickets[r] = 0u;  // leave the workspace zeroed
}

}  // namespace tk
