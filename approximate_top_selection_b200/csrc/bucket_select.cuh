// bucket_select.cuh -- Stage 1 + Stage 2 of bucketed top-k over float32 or
// bfloat16 score rows.
//
// Method: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
// pith.science review page, "What carries the argument": interleaved buckets
// (element i -> bucket i mod b), exact top-k_b per bucket kept in per-thread
// register queues (k_b <= 4), final exact top-k when b*k_b > k.
//
// Work decomposition (ours, not the page's): one CTA per row when the rows
// fill one resident wave, else the rows*n elements are cut into G equal
// contiguous CTA ranges; a row that straddles CTA ranges is merged by the last
// CTA to finish it (select_core.cuh).
//
// Fast kernel (n % 4 == 0 for fp32 / 8 for bf16, 16-byte aligned rows,
// b | 1024): a producer warp streams 32 KB tiles of the row into a ring of
// shared-memory stages (cp.async.bulk + mbarrier).  k_b <= 2: thread t owns
// the four consecutive positions 4t..4t+3 of every 1024-element stripe, so
// each of its four queues sees a single bucket ((a + 4t + v) mod b), updated
// branch-free.  k_b > 2: queue q of thread t covers positions t + 256 q modulo
// max(256, b); each element is tested against its queue's k_b-th value and
// only survivors take the sorted insert.  An optional sampling tail (template
// flag) draws one token per row after Stage 2.
// General kernel (any n, alignment, b <= 1024): direct coalesced scalar loads,
// thread t owns stripe positions t + 256 v of a stripe of L*b elements.
#pragma once

#include "select_core.cuh"

namespace tk {

constexpr int kTileBytes = 32768;  // bytes per bulk copy
constexpr int kTile = 8192;        // fp32 elements per tile

// Element types of score rows: float, or uint16_t holding bfloat16 bits.  A
// bf16 widened to fp32 is exact and keeps the order, ties, -0 and NaN, so the
// queues always compare fp32 values.
template <typename T>
struct Elem {
  static constexpr int kPerTile = kTileBytes / static_cast<int>(sizeof(T));
  static constexpr int kAlign = 16 / static_cast<int>(sizeof(T));  // elements per 16 bytes
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
// Four consecutive elements (16 or 8 bytes, aligned) as fp32.
__device__ __forceinline__ float4 load4_f32(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4_f32(const uint16_t* p) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                     __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
}

template <typename T>
struct SelectArgs {
  const T* x;
  int k, b;
  T* out_vals;
  int32_t* out_idx;
  RowSplit rs;
  SampleTail tail;  // token == nullptr: no sampling tail
};

// Shared-memory layouts of the streaming kernels:
//  kLayoutSeparate  tile ring, lane buffer (every queue, stored for the
//                   merge), Stage-2 candidate buffer and barriers side by side.
//  kLayoutAliased   every CTA streams exactly one piece, so the lane and
//                   candidate buffers are only needed once the ring has been
//                   consumed for good: they live inside it, and the ring gets
//                   their room (more tile stages in flight).
enum SelectLayout { kLayoutSeparate = 0, kLayoutAliased = 1 };

struct SelectSmem {
  int stages, kb, cand_cap, nl;  // nl: register queues (lanes) per CTA
  int layout = kLayoutSeparate;
  __host__ __device__ size_t lane_bytes() const { return static_cast<size_t>(nl) * kb * 8; }
  __host__ __device__ size_t cand_bytes() const {
    return static_cast<size_t>(cand_cap) * 8 + kStage2Extra;
  }
  __host__ __device__ size_t ring_bytes() const {
    const size_t r = static_cast<size_t>(stages) * kTileBytes;
    const size_t lc = lane_bytes() + cand_bytes();
    return layout == kLayoutAliased && lc > r ? lc : r;
  }
  __host__ __device__ size_t lane_off() const {
    return layout == kLayoutAliased ? 0 : ring_bytes();
  }
  __host__ __device__ size_t cand_off() const { return lane_off() + lane_bytes(); }
  __host__ __device__ size_t bar_off() const {
    return layout == kLayoutAliased ? ring_bytes() : ring_bytes() + lane_bytes() + cand_bytes();
  }
  __host__ __device__ size_t bar_bytes() const { return 16 * static_cast<size_t>(stages) + 16; }
  __host__ __device__ size_t total() const { return bar_off() + bar_bytes(); }
};

// Survivor masks on the FMA pipe (the k_b > 2 update saturates the ALU pipe):
// FSET turns x > thr into 1.0 or 0.0 and an FMA adds it times 2^bit to 2^23,
// exactly (the sum stays below 2^24), so the float's low mantissa bits are the
// mask.  mask_acc_init / mask_acc_bits bracket the accumulation.
__device__ __forceinline__ float mask_acc_init() { return 8388608.0f; }
__device__ __forceinline__ float mask_acc_add(float acc, float x, float thr, int bit) {
  return fmaf(x > thr ? 1.0f : 0.0f, static_cast<float>(1u << bit), acc);
}
__device__ __forceinline__ uint32_t mask_acc_bits(float acc) {
  return __float_as_uint(acc) - 0x4B000000u;
}

// 0 * x is NaN exactly when x is NaN or infinite: false when any of the N
// values is NaN or +-inf (FMA-pipe chains, two of them).
template <int N>
__device__ __forceinline__ bool all_finite(const float (&x)[N]) {
  float a = 0.0f, b = 0.0f;
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    a = fmaf(x[i], 0.0f, a);
    if (i + 1 < N) b = fmaf(x[i + 1], 0.0f, b);
  }
  const float s = a + b;
  return s == s;
}

// k_b > 2: one tile (c valid floats at row positions pos_tile ...) for the
// queues of this thread: element u sits at tile offset t + 256 u and feeds
// queue u mod nq.  Each element is first compared with its queue's worst
// entry; only the survivors -- typically a few per thread per tile once the
// queues have filled -- go through the sorted insert, re-read from shared
// memory, so a warp pays for its busiest thread's survivors rather than for
// every element.  A tile holding NaN or -inf takes the exact update instead.
template <int KB, typename T>
__device__ __forceinline__ void select_tile_sparse(Queues<KB>& q, const T* tile, uint32_t c,
                                                   uint32_t pos_tile, int nq) {
  constexpr int U = kTile / kThreads;  // 32 elements per thread (8192 per call)
  const int t = threadIdx.x;
  float x[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const bool valid = static_cast<uint32_t>(t + kThreads * u) < c;
    x[u] = valid ? to_f32(tile[t + kThreads * u]) : __int_as_float(0x7f800000);
  }
  const uint32_t base = pos_tile + static_cast<uint32_t>(t);
  const bool full = c >= static_cast<uint32_t>(kTile);
  if (full ? !all_finite<U>(x) : !(min_nan_all<U>(x) > __int_as_float(0xff800000))) {
    // NaN or -inf (a full tile: or +inf) in this thread's elements: exact
    // update, in order.
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (static_cast<uint32_t>(t + kThreads * u) >= c) continue;
      const uint32_t pos = base + static_cast<uint32_t>(kThreads * u);
      const int qq = u % nq;
      if (qq == 0) q.template insert_exact<0>(x[u], pos);
      if (qq == 1) q.template insert_exact<1>(x[u], pos - 1);
      if (qq == 2) q.template insert_exact<2>(x[u], pos - 2);
      if (qq == 3) q.template insert_exact<3>(x[u], pos - 3);
    }
    return;
  }
  // Survivor masks per queue (queue of element u is u mod nq; nq is 1, 2 or 4).
  uint32_t mask[4] = {0u, 0u, 0u, 0u};
  const float thr[4] = {q.val[0][KB - 1], q.val[1][KB - 1], q.val[2][KB - 1], q.val[3][KB - 1]};
  if (full) {
    // Every element valid: the masks on the FMA pipe, 16 bits per accumulator.
    float lo[4], hi[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) lo[v] = hi[v] = mask_acc_init();
    if (nq == 1) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u < 16) lo[0] = mask_acc_add(lo[0], x[u], thr[0], u);
        else hi[0] = mask_acc_add(hi[0], x[u], thr[0], u - 16);
      }
    } else if (nq == 2) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u < 16) lo[u & 1] = mask_acc_add(lo[u & 1], x[u], thr[u & 1], u);
        else hi[u & 1] = mask_acc_add(hi[u & 1], x[u], thr[u & 1], u - 16);
      }
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u < 16) lo[u & 3] = mask_acc_add(lo[u & 3], x[u], thr[u & 3], u);
        else hi[u & 3] = mask_acc_add(hi[u & 3], x[u], thr[u & 3], u - 16);
      }
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) mask[v] = mask_acc_bits(lo[v]) | (mask_acc_bits(hi[v]) << 16);
  } else if (nq == 1) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      mask[0] |= (static_cast<uint32_t>(t + kThreads * u) < c && x[u] > thr[0]) ? (1u << u) : 0u;
  } else if (nq == 2) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      mask[u & 1] |=
          (static_cast<uint32_t>(t + kThreads * u) < c && x[u] > thr[u & 1]) ? (1u << u) : 0u;
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u)
      mask[u & 3] |=
          (static_cast<uint32_t>(t + kThreads * u) < c && x[u] > thr[u & 3]) ? (1u << u) : 0u;
  }
  // Survivors of each queue in turn, re-read from shared memory.  The loop is
  // software-pipelined: the next survivor's value is loaded before the
  // current one is inserted, so the load latency overlaps the insert.
  const T* tt = tile + t;
#define TK_SURVIVORS(Q)                                                                   \
  if (mask[Q]) {                                                                          \
    int u = __ffs(mask[Q]) - 1;                                                           \
    mask[Q] &= mask[Q] - 1u;                                                              \
    float xc = to_f32(tt[kThreads * u]);                                                  \
    for (;;) {                                                                            \
      const bool more = mask[Q] != 0u;                                                    \
      const int un = more ? __ffs(mask[Q]) - 1 : u;                                       \
      const float xn = to_f32(tt[kThreads * un]);                                         \
      q.template insert_fast<Q>(xc, base + static_cast<uint32_t>(kThreads * u) - (Q));    \
      if (!more) break;                                                                   \
      mask[Q] &= mask[Q] - 1u;                                                            \
      u = un;                                                                             \
      xc = xn;                                                                            \
    }                                                                                     \
  }
  TK_SURVIVORS(0)
  if (nq > 1) {
    TK_SURVIVORS(1)
  }
  if (nq > 2) {
    TK_SURVIVORS(2)
    TK_SURVIVORS(3)
  }
#undef TK_SURVIVORS
}

// ------------------------------------------------------------------ bf16 order keys
// bfloat16 rows with k_b >= 2.  A bf16 value and its place in its queue fit in
// one 32-bit word whose unsigned order is the method's total order: the high
// half is a 16-bit order code of the value, the low half 0xFFFF minus the
// element's ordinal in its queue (queues see their elements in increasing
// position, so among equal values the earlier one compares larger).  A queue
// is then KB such words, best first, and an element enters it through an
// unsigned max/min insertion network -- 2 KB - 1 integer operations, no
// comparison of indices and no branch, exact for every input.
//
// Order codes: a positive h codes as h ^ 0x8000 and a negative one as
// (h ^ 0xFFFF) + 1, so that -0 and +0 share 0x8000, -inf codes 0x0080 and +inf
// 0xFF80; every NaN codes 0xFFFF (all NaNs tie, above +inf).  No value codes 0,
// so the word 0 marks an empty slot.  A queue's ordinal must fit 16 bits: the
// path is taken for pieces of at most kKeyMaxPiece elements.
constexpr int64_t kKeyMaxPiece = static_cast<int64_t>(kLanes) << 16;

// Codes of the two bf16 in w (one per 16-bit half), w holding no NaN.  The
// byte permute replicates each half's sign bit over that half (0xFFFF where
// negative), so a negative half becomes (h ^ 0xFFFF) + 1 and a positive one
// h ^ 0x8000; the +1 never carries across the halves.
__device__ __forceinline__ uint32_t bf16x2_codes(uint32_t w) {
  uint32_t m;  // selector nibbles 9 and B: bytes 1 and 3 with their sign bit replicated
  asm("prmt.b32 %0, %1, 0, 0xBB99;" : "=r"(m) : "r"(w));
  return (w ^ (m | 0x80008000u)) + (m & 0x00010001u);
}

// Codes of any two bf16 (NaN halves code 0xFFFF).
__device__ __forceinline__ uint32_t bf16x2_codes_exact(uint32_t w) {
  uint32_t c = bf16x2_codes(w);
  if ((w & 0x7FFFu) > 0x7F80u) c |= 0x0000FFFFu;
  if (((w >> 16) & 0x7FFFu) > 0x7F80u) c |= 0xFFFF0000u;
  return c;
}

// acc + 0 * w on bf16 pairs (an FMA-pipe instruction): a half of the result is
// NaN once any w offered to it held NaN or +-inf in that half.
__device__ __forceinline__ uint32_t bf16x2_nonfinite_acc(uint32_t w, uint32_t acc) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(0u), "r"(acc));
  return d;
}

__device__ __forceinline__ bool bf16x2_has_nan(uint32_t w) {
  return ((w & 0x7FFFu) > 0x7F80u) | (((w >> 16) & 0x7FFFu) > 0x7F80u);
}

// k_b <= 2 on bf16 rows: a thread's four queues (the float4 layout) as, per
// slot, two bf16x2 value words (queues 0, 1 and 2, 3) and two words of 16-bit
// stripe ordinals (0xFFFF: empty), so that packed compares and bit-selects
// update two queues at once.  A finite element enters a slot when it is
// strictly larger (ties keep the earlier stripe; -0 and +0 compare equal);
// entries start at -inf, which every finite element beats.  A slice that
// holds a NaN or +-inf takes the element-wise update under the total order
// (16-bit order codes: NaN above +inf, -0 = +0, an empty queue takes anything).
__device__ __forceinline__ uint32_t bf16x2_gt_mask(uint32_t a, uint32_t b) {
  uint32_t d;  // per half: 0xFFFF where a > b, else 0
  asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf16_order_code(uint32_t h) {
  if ((h & 0x7FFFu) > 0x7F80u) return 0xFFFFu;      // NaN
  return (h & 0x8000u) ? ((h ^ 0xFFFFu) + 1u) & 0xFFFFu : (h ^ 0x8000u);
}

template <int KB>
struct PairQueues {
  uint32_t val[KB][2], ord[KB][2];  // slot s of queues (0, 1) and (2, 3)

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      val[s][0] = val[s][1] = 0xFF80FF80u;  // -inf, -inf
      ord[s][0] = ord[s][1] = 0xFFFFFFFFu;  // empty, empty
    }
  }

  // Four consecutive finite bf16 (w.x: queues 0, 1; w.y: queues 2, 3) at
  // stripe ordinal o.  The slots are sorted, so x above slot s implies x
  // above every later slot: slot s takes slot s-1 where x beats it, else x
  // where x beats slot s, else keeps its entry.
  __device__ __forceinline__ void offer4(uint2 w, uint32_t o) {
    const uint32_t o2 = o * 0x00010001u;
    const uint32_t xs[2] = {w.x, w.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t x = xs[i];
      uint32_t m[KB];
#pragma unroll
      for (int s = 0; s < KB; ++s) m[s] = bf16x2_gt_mask(x, val[s][i]);
#pragma unroll
      for (int s = KB - 1; s >= 0; --s) {
        const uint32_t tv = (x & m[s]) | (val[s][i] & ~m[s]);
        const uint32_t to = (o2 & m[s]) | (ord[s][i] & ~m[s]);
        if (s > 0) {
          val[s][i] = (val[s - 1][i] & m[s - 1]) | (tv & ~m[s - 1]);
          ord[s][i] = (ord[s - 1][i] & m[s - 1]) | (to & ~m[s - 1]);
        } else {
          val[s][i] = tv;
          ord[s][i] = to;
        }
      }
    }
  }

  __device__ __forceinline__ void offer4_exact(uint2 w, uint32_t o) {
    const uint32_t in[2] = {w.x, w.y};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = e >> 1, sh = (e & 1) * 16;
      const uint32_t lane_mask = 0xFFFFu << sh;
      const uint32_t h = (in[i] >> sh) & 0xFFFFu;
      // The first slot that is empty or holds a smaller entry takes the
      // element; every later entry moves down one slot (the last drops out).
      bool placed = false;
      uint32_t mv = h, mo = o;  // the entry to write next (ordinal 0xFFFF: none)
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        const uint32_t cur = (val[s][i] >> sh) & 0xFFFFu;
        const uint32_t co = (ord[s][i] >> sh) & 0xFFFFu;
        if (!placed) placed = co == 0xFFFFu || bf16_order_code(h) > bf16_order_code(cur);
        if (placed && mo != 0xFFFFu) {
          val[s][i] = (val[s][i] & ~lane_mask) | (mv << sh);
          ord[s][i] = (ord[s][i] & ~lane_mask) | (mo << sh);
          mv = cur;
          mo = co;
        }
      }
    }
  }

  // Queue v as KB packed (order key, ~position) words, position = pos_thread
  // + v + ordinal * kLanes (0: empty).
  __device__ __forceinline__ void store(int v, uint64_t* dst, uint32_t pos_thread) const {
    const int i = v >> 1, sh = (v & 1) * 16;
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      const uint32_t o = (ord[s][i] >> sh) & 0xFFFFu;
      const uint32_t h = (val[s][i] >> sh) & 0xFFFFu;
      dst[s] = o == 0xFFFFu ? 0ull
                            : pack(order_key(__uint_as_float(h << 16)),
                                   pos_thread + static_cast<uint32_t>(v) + o * static_cast<uint32_t>(kLanes));
    }
  }
};

// Four queues per thread (the float4 layout: queue v of thread t takes the
// positions congruent to 4t + v modulo kLanes), as order keys.  A key carries
// its own tie-break, so the top-KB of a queue does not depend on the order in
// which its elements are inserted: each queue is kept as SUB sub-queues that
// take alternate stripes -- independent insertion chains, more work in flight
// per thread -- and the sub-queues are combined when the piece ends.
template <int KB, int SUB = 2>
struct KeyQueues {
  uint32_t key[4][SUB][KB];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int v = 0; v < 4; ++v)
#pragma unroll
      for (int j = 0; j < SUB; ++j)
#pragma unroll
        for (int s = 0; s < KB; ++s) key[v][j][s] = 0u;
  }

  template <int V, int J>
  __device__ __forceinline__ void insert(uint32_t x) {
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      const uint32_t k = key[V][J][s];
      key[V][J][s] = max(k, x);
      if (s + 1 < KB) x = min(k, x);
    }
  }

  // Four consecutive bf16 (w.x: elements 0, 1; w.y: elements 2, 3), one per
  // queue, at queue ordinal `ord`, into sub-queue J.
  template <int J>
  __device__ __forceinline__ void offer4(uint2 w, uint32_t ord, bool nan) {
    const uint32_t lo = 0xFFFFu - ord;
    const uint32_t cx = nan ? bf16x2_codes_exact(w.x) : bf16x2_codes(w.x);
    const uint32_t cy = nan ? bf16x2_codes_exact(w.y) : bf16x2_codes(w.y);
    // (low code << 16) | lo as cx * 2^16 + lo: a multiply-add, on the FMA pipe
    // (the ALU pipe is the one the update saturates); the high code by a byte
    // permute.
    insert<0, J>(cx * 0x10000u + lo);
    insert<1, J>(__byte_perm(cx, lo, 0x3254u));
    insert<2, J>(cy * 0x10000u + lo);
    insert<3, J>(__byte_perm(cy, lo, 0x3254u));
  }

  // Folds sub-queues 1.. into sub-queue 0.
  __device__ __forceinline__ void combine() {
#pragma unroll
    for (int j = 1; j < SUB; ++j)
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        insert<0, 0>(key[0][j][s]);
        insert<1, 0>(key[1][j][s]);
        insert<2, 0>(key[2][j][s]);
        insert<3, 0>(key[3][j][s]);
      }
  }

  // Queue v (after combine()) as packed candidates at dst[0..KB); pos0 is the
  // row position of its ordinal 0.
  __device__ __forceinline__ void store(int v, uint64_t* dst, uint32_t pos0) const {
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      uint32_t k = 0u;
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (w == v) k = key[w][0][s];
      uint64_t out = 0ull;
      if (k != 0u) {
        const uint32_t code = k >> 16;
        const uint32_t h = code >= 0x8000u ? (code ^ 0x8000u) : (((code - 1u) ^ 0xFFFFu) & 0xFFFFu);
        const uint32_t ord = 0xFFFFu - (k & 0xFFFFu);
        out = pack(order_key(__uint_as_float(h << 16)), pos0 + static_cast<uint32_t>(kLanes) * ord);
      }
      dst[s] = out;
    }
  }
};

#ifndef TOPK_BF16_KEYS
#define TOPK_BF16_KEYS 1
#endif
#ifndef TOPK_BF16_KEYS_MIN_KB  // smallest k_b that takes the key path
#define TOPK_BF16_KEYS_MIN_KB 1
#endif
#ifndef TOPK_BF16_PAIR_MAX_KB  // largest k_b on packed bf16x2 queues (PairQueues)
#define TOPK_BF16_PAIR_MAX_KB 2
#endif

#ifndef TOPK_SPARSE_MIN_KB  // smallest k_b that takes the survivor (sparse / wide) update
#define TOPK_SPARSE_MIN_KB 3
#endif

// Register queues per CTA of the TMA kernel: four per thread (float4 layout)
// for the branch-free update (k_b < TOPK_SPARSE_MIN_KB) and for the bf16 key
// path, max(256, b) for the sparse survivor layout.
__host__ __device__ __forceinline__ int select_lanes(int kb, int b, bool keys = false) {
  return kb < TOPK_SPARSE_MIN_KB || keys ? kLanes : (b > kThreads ? b : kThreads);
}

constexpr int kConsumerWarps = kThreads / 32;
constexpr int kPipeThreads = kThreads + 32;  // consumers + one producer warp

// Warp-specialised streaming: warp kConsumerWarps issues the bulk copies of
// the CTA's tiles into a ring of `stages` shared-memory stages (full barrier:
// bytes landed; empty barrier: every consumer warp is done with the stage);
// the kThreads consumer threads never wait for each other inside a piece.
// SAMPLE: the instantiation that also draws each row's token after Stage 2
// (p.tail); without it the sampling code is not compiled in at all.
// KEYS: bf16 rows on 16-bit codes -- k_b <= TOPK_BF16_PAIR_MAX_KB in
// PairQueues, larger k_b in KeyQueues (see bf16 order keys).
template <typename T, int KB, bool SAMPLE = false, bool KEYS = false>
__global__ void __launch_bounds__(kPipeThreads, 2) bucket_select_tma(SelectArgs<T> p, int stages,
                                                                  int cand_cap, int layout) {
  constexpr int kTileElems = Elem<T>::kPerTile;
  static_assert(!KEYS || sizeof(T) == 2, "the key path is for bf16 rows");
  extern __shared__ __align__(128) unsigned char smem[];
  const SelectSmem L{stages, KB, cand_cap, select_lanes(KB, p.b, KEYS), layout};
  T* ring = reinterpret_cast<T*>(smem);
  uint64_t* lanebuf = reinterpret_cast<uint64_t*>(smem + L.lane_off());
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + L.cand_off());
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off());
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  int* piece_flag = reinterpret_cast<int*>(empty + stages) + 1;
  volatile int* skip_flag = reinterpret_cast<volatile int*>(empty + stages) + 2;

  const RowSplit& rs = p.rs;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t s0 = cta_start(rs, blockIdx.x);
  const int64_t e0 = cta_start(rs, blockIdx.x + 1);
  const int64_t n = rs.n;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait_then_release();

  // Tile t of this CTA covers [g, g + len) with len = min(tile, e0 - g,
  // end of g's row - g): tiles never straddle rows.
  auto tile_len = [&](int64_t g) -> int64_t {
    const int64_t rowend = (g / n + 1) * n;
    int64_t c = e0 - g;
    if (rowend - g < c) c = rowend - g;
    return c < kTileElems ? c : kTileElems;
  };

  if (warp == kConsumerWarps) {  // ---------------- producer
    if (lane == 0) {
      int64_t g = s0, t = 0;
      int st = 0;       // stage of tile t
      uint32_t ph = 0;  // parity of t / stages
      while (g < e0) {
        const int64_t c = tile_len(g);
        if (t >= stages && !mbar_wait_or_abort(empty + st, ph ^ 1u, abort_flag)) break;
        const uint32_t bytes = static_cast<uint32_t>(c * static_cast<int64_t>(sizeof(T)));
        mbar_expect_tx(full + st, bytes);
        bulk_g2s(ring + static_cast<size_t>(st) * kTileElems, p.x + g, bytes, full + st);
        g += c;
        ++t;
        if (++st == stages) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA can go away.
        drain_copies(full, stages, t > stages ? t - stages : 0, t);
      }
    }
    return;
  }

  // ---------------- consumers
  // k_b <= 2: four queues per thread over 4-element groups (kLanes lanes),
  // updated branch-free.  k_b > 2: queue q of thread t covers positions
  // t + 256 q modulo nl = max(256, b) (select_tile_sparse), so each queue sees
  // four times more elements and only the survivors of a threshold test pay
  // for the sorted insert.
  const int nl = select_lanes(KB, p.b, KEYS);
  const int nq = nl / kThreads;
  Queues<KB> q;
  KeyQueues<KB> kq;  // bf16 key path, k_b >= 2
  PairQueues<(KB <= 2 ? KB : 1)> pq;  // bf16 key path, packed queues
  int st = 0;       // ring stage of the next tile
  uint32_t ph = 0;  // its full-barrier parity
  int64_t g = s0;
  while (g < e0) {
    const int64_t r = g / n;
    const int64_t row0 = r * n;
    const int64_t a = g - row0;
    const int64_t pend = (row0 + n < e0) ? row0 + n : e0;
    const uint32_t len = static_cast<uint32_t>(pend - g);  // < 2^31
    const uint32_t pos_thread = static_cast<uint32_t>(a) + 4u * tid;
    if constexpr (KEYS && KB <= TOPK_BF16_PAIR_MAX_KB)
      pq.reset();
    else if constexpr (KEYS)
      kq.reset();
    else
      q.reset();
    for (uint32_t done = 0; done < len;) {
      const uint32_t c =
          (len - done) < static_cast<uint32_t>(kTileElems) ? (len - done) : kTileElems;
      // Warp-uniform: if any lane saw the stage complete, its bytes have landed.
      const bool ok = __any_sync(0xffffffffu,
                                 !*abort_flag && mbar_wait_or_abort(full + st, ph, abort_flag));
      if (ok) {
        const T* stage_tile = ring + static_cast<size_t>(st) * kTileElems;
        if constexpr (KEYS && KB <= TOPK_BF16_PAIR_MAX_KB) {
          // Slices of kTile elements as in the order-key path; a slice with
          // a NaN or +-inf takes the element-wise update.
          constexpr int U = kTile / kLanes;
#pragma unroll
          for (int h = 0; h < kTileElems / kTile; ++h) {
            const uint32_t hoff = static_cast<uint32_t>(h * kTile);
            const T* tile = stage_tile + hoff + 4 * tid;
            const uint32_t ord0 = (done + hoff) / static_cast<uint32_t>(kLanes);
            if (hoff + kTile <= c) {
              uint2 w[U];
#pragma unroll
              for (int u = 0; u < U; ++u) w[u] = *reinterpret_cast<const uint2*>(tile + kLanes * u);
              uint32_t mx = 0u, my = 0u;
#pragma unroll
              for (int u = 0; u < U; ++u) {
                mx = bf16x2_nonfinite_acc(w[u].x, mx);
                my = bf16x2_nonfinite_acc(w[u].y, my);
              }
              if (!(bf16x2_has_nan(mx) | bf16x2_has_nan(my))) {
#pragma unroll
                for (int u = 0; u < U; ++u) pq.offer4(w[u], ord0 + u);
              } else {
#pragma unroll
                for (int u = 0; u < U; ++u) pq.offer4_exact(w[u], ord0 + u);
              }
            } else {
#pragma unroll
              for (int u = 0; u < U; ++u) {
                const uint32_t off = hoff + 4u * tid + static_cast<uint32_t>(kLanes * u);
                if (off < c)
                  pq.offer4_exact(*reinterpret_cast<const uint2*>(tile + kLanes * u), ord0 + u);
              }
            }
          }
        } else if constexpr (KEYS) {
          // In slices of kTile elements: stripe u of a slice is queue ordinal
          // (done + hoff) / kLanes + u.  A pair NaN check per slice picks the
          // cheap or the NaN-aware codes.
          constexpr int U = kTile / kLanes;
#pragma unroll
          for (int h = 0; h < kTileElems / kTile; ++h) {
            const uint32_t hoff = static_cast<uint32_t>(h * kTile);
            const T* tile = stage_tile + hoff + 4 * tid;
            const uint32_t ord0 = (done + hoff) / static_cast<uint32_t>(kLanes);
            if (hoff + kTile <= c) {
              uint2 w[U];
#pragma unroll
              for (int u = 0; u < U; ++u) w[u] = *reinterpret_cast<const uint2*>(tile + kLanes * u);
              uint32_t mx = 0u, my = 0u;  // NaN or +-inf anywhere: the NaN-aware codes
#pragma unroll
              for (int u = 0; u < U; ++u) {
                mx = bf16x2_nonfinite_acc(w[u].x, mx);
                my = bf16x2_nonfinite_acc(w[u].y, my);
              }
              const bool nan = bf16x2_has_nan(mx) | bf16x2_has_nan(my);
#pragma unroll
              for (int u = 0; u < U; u += 2) {
                kq.template offer4<0>(w[u], ord0 + u, nan);
                kq.template offer4<1>(w[u + 1], ord0 + u + 1, nan);
              }
            } else {
#pragma unroll
              for (int u = 0; u < U; ++u) {
                const uint32_t off = hoff + 4u * tid + static_cast<uint32_t>(kLanes * u);
                if (off < c) {
                  const uint2 w = *reinterpret_cast<const uint2*>(tile + kLanes * u);
                  kq.template offer4<0>(w, ord0 + u, true);
                }
              }
            }
          }
        } else if constexpr (KB < TOPK_SPARSE_MIN_KB) {
          // In slices of kTile elements (a bf16 tile holds two of them).
          constexpr int U = kTile / kLanes;
#pragma unroll
          for (int h = 0; h < kTileElems / kTile; ++h) {
            const uint32_t hoff = static_cast<uint32_t>(h * kTile);
            const T* tile = stage_tile + hoff + 4 * tid;
            const uint32_t pos0 = pos_thread + done + hoff;
            if (hoff + kTile <= c) {
              float4 x[U];
              uint32_t base[U];
#pragma unroll
              for (int u = 0; u < U; ++u) {
                x[u] = load4_f32(tile + kLanes * u);
                base[u] = pos0 + static_cast<uint32_t>(kLanes * u);
              }
              q.template offer_tile<U>(x, base);
            } else {
#pragma unroll
              for (int u = 0; u < U; ++u) {
                const uint32_t off = hoff + 4u * tid + static_cast<uint32_t>(kLanes * u);
                if (off < c)
                  q.offer4(load4_f32(tile + kLanes * u), pos0 + static_cast<uint32_t>(kLanes * u));
              }
            }
          }
        } else {
#pragma unroll
          for (int h = 0; h < kTileElems / kTile; ++h) {
            const uint32_t hoff = static_cast<uint32_t>(h * kTile);
            if (hoff < c)
              select_tile_sparse<KB, T>(q, stage_tile + hoff, c - hoff,
                                        static_cast<uint32_t>(a) + done + hoff, nq);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);
      if (++st == stages) {
        st = 0;
        ph ^= 1u;
      }
      done += c;
    }
    g = pend;
    // Piece done: publish the queues and finish (Stage 2 or cross-CTA merge).
    // With the lane buffer inside the ring, every consumer must be done with
    // the ring first (the piece is the CTA's last: no copy is in flight).  An
    // aborted CTA may still have copies landing there: it stops here, all
    // consumers together (one thread reads the flag for all of them).
    if (layout == kLayoutAliased) {
      group_sync(kThreads);
      if (tid == 0) *skip_flag = *abort_flag;
      group_sync(kThreads);
      if (*skip_flag) break;
    }
    if constexpr (KEYS && KB <= TOPK_BF16_PAIR_MAX_KB) {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        pq.store(v, lanebuf + static_cast<size_t>(4 * tid + v) * KB, pos_thread);
    } else if constexpr (KEYS) {
      kq.combine();
#pragma unroll
      for (int v = 0; v < 4; ++v)
        kq.store(v, lanebuf + static_cast<size_t>(4 * tid + v) * KB, pos_thread + v);
    } else if constexpr (KB < TOPK_SPARSE_MIN_KB) {
#pragma unroll
      for (int v = 0; v < 4; ++v) q.store(v, lanebuf + static_cast<size_t>(4 * tid + v) * KB);
    } else {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        if (v < nq) q.store(v, lanebuf + static_cast<size_t>(tid + kThreads * v) * KB);
    }
    group_sync(kThreads);
    finish_piece<KB, kGatherInput, T>(rs, p.b, p.k, r, a, static_cast<int64_t>(len), lanebuf, cand,
                                      p.x + row0, p.out_vals, p.out_idx, piece_flag, nl,
                                      SAMPLE ? p.tail : SampleTail{nullptr, nullptr, 1.0f});
    group_sync(kThreads);
  }
}

// ------------------------------------------------------------------ k_b > 2, 16 warps
// The k_b > 2 update is a chain of survivor inserts per queue, so it is bound
// by latency rather than bandwidth: this kernel runs 16 consumer warps per CTA
// (two CTAs per SM) and gives each thread NQ = b / 512 queues over positions
// t + 512 q modulo b (used for b >= 512, one lane per bucket).  A thread sees
// 16 elements per 8192-element tile, half the chain of the 8-warp layout, and
// an SM holds twice the warps to overlap the chains.  Stage 2 and the merge
// run on the first kThreads threads.
constexpr int kWideConsumers = 512;
constexpr int kWideWarps = kWideConsumers / 32;
constexpr int kWideThreads = kWideConsumers + 32;  // consumers + one producer warp

__device__ __forceinline__ void consumer_sync_wide() {
  asm volatile("bar.sync 2, %0;" ::"r"(kWideConsumers) : "memory");
}

template <int KB, typename T, int NQ>
__device__ __forceinline__ void select_tile_wide(Queues<KB, NQ>& q, const T* tile, uint32_t c,
                                                 uint32_t pos_tile) {
  constexpr int CT = kWideConsumers;
  constexpr int U = kTile / CT;  // 16 elements per thread
  const int t = threadIdx.x;
  float x[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const bool valid = static_cast<uint32_t>(t + CT * u) < c;
    x[u] = valid ? to_f32(tile[t + CT * u]) : __int_as_float(0x7f800000);
  }
  const uint32_t base = pos_tile + static_cast<uint32_t>(t);
  const bool full = c >= static_cast<uint32_t>(kTile);
  if (full ? !all_finite<U>(x) : !(min_nan_all<U>(x) > __int_as_float(0xff800000))) {
    // NaN or -inf (a full tile: or +inf) in this thread's elements: exact
    // update, in order.
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (static_cast<uint32_t>(t + CT * u) >= c) continue;
      const uint32_t pos = base + static_cast<uint32_t>(CT * u);
      if (u % NQ == 0)
        q.template insert_exact<0>(x[u], pos);
      else
        q.template insert_exact<(NQ > 1 ? 1 : 0)>(x[u], pos - 1u);
    }
    return;
  }
  uint32_t mask[NQ];
  float thr[NQ];
#pragma unroll
  for (int v = 0; v < NQ; ++v) {
    mask[v] = 0u;
    thr[v] = q.val[v][KB - 1];
  }
  if (full) {  // every element valid: the masks on the FMA pipe (U = 16 bits)
    float acc[NQ];
#pragma unroll
    for (int v = 0; v < NQ; ++v) acc[v] = mask_acc_init();
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u % NQ] = mask_acc_add(acc[u % NQ], x[u], thr[u % NQ], u);
#pragma unroll
    for (int v = 0; v < NQ; ++v) mask[v] = mask_acc_bits(acc[v]);
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u)
      mask[u % NQ] |=
          (static_cast<uint32_t>(t + CT * u) < c && x[u] > thr[u % NQ]) ? (1u << u) : 0u;
  }
  // Survivors, software-pipelined as in select_tile_sparse.
  const T* tt = tile + t;
#pragma unroll
  for (int v = 0; v < NQ; ++v) {
    if (mask[v]) {
      int u = __ffs(mask[v]) - 1;
      mask[v] &= mask[v] - 1u;
      float xc = to_f32(tt[CT * u]);
      for (;;) {
        const bool more = mask[v] != 0u;
        const int un = more ? __ffs(mask[v]) - 1 : u;
        const float xn = to_f32(tt[CT * un]);
        if (v == 0)
          q.template insert_fast<0>(xc, base + static_cast<uint32_t>(CT * u));
        else
          q.template insert_fast<(NQ > 1 ? 1 : 0)>(xc, base + static_cast<uint32_t>(CT * u) - 1u);
        if (!more) break;
        mask[v] &= mask[v] - 1u;
        u = un;
        xc = xn;
      }
    }
  }
}

template <typename T, int KB, int NQ, bool SAMPLE = false>
__global__ void __launch_bounds__(kWideThreads, 2) bucket_select_wide(SelectArgs<T> p, int stages,
                                                                   int cand_cap, int layout) {
  constexpr int kTileElems = Elem<T>::kPerTile;
  constexpr int NL = kWideConsumers * NQ;  // register queues (lanes) per CTA
  extern __shared__ __align__(128) unsigned char smem[];
  const SelectSmem L{stages, KB, cand_cap, NL, layout};
  T* ring = reinterpret_cast<T*>(smem);
  uint64_t* lanebuf = reinterpret_cast<uint64_t*>(smem + L.lane_off());
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + L.cand_off());
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off());
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  int* piece_flag = reinterpret_cast<int*>(empty + stages) + 1;
  volatile int* skip_flag = reinterpret_cast<volatile int*>(empty + stages) + 2;

  const RowSplit& rs = p.rs;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t s0 = cta_start(rs, blockIdx.x);
  const int64_t e0 = cta_start(rs, blockIdx.x + 1);
  const int64_t n = rs.n;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kWideWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait_then_release();

  auto tile_len = [&](int64_t g) -> int64_t {
    const int64_t rowend = (g / n + 1) * n;
    int64_t c = e0 - g;
    if (rowend - g < c) c = rowend - g;
    return c < kTileElems ? c : kTileElems;
  };

  if (warp == kWideWarps) {  // ---------------- producer
    if (lane == 0) {
      int64_t g = s0, t = 0;
      int st = 0;
      uint32_t ph = 0;
      while (g < e0) {
        const int64_t c = tile_len(g);
        if (t >= stages && !mbar_wait_or_abort(empty + st, ph ^ 1u, abort_flag)) break;
        const uint32_t bytes = static_cast<uint32_t>(c * static_cast<int64_t>(sizeof(T)));
        mbar_expect_tx(full + st, bytes);
        bulk_g2s(ring + static_cast<size_t>(st) * kTileElems, p.x + g, bytes, full + st);
        g += c;
        ++t;
        if (++st == stages) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        drain_copies(full, stages, t > stages ? t - stages : 0, t);
      }
    }
    return;
  }

  // ---------------- consumers
  Queues<KB, NQ> q;
  int st = 0;
  uint32_t ph = 0;
  int64_t g = s0;
  while (g < e0) {
    const int64_t r = g / n;
    const int64_t row0 = r * n;
    const int64_t a = g - row0;
    const int64_t pend = (row0 + n < e0) ? row0 + n : e0;
    const uint32_t len = static_cast<uint32_t>(pend - g);
    q.reset();
    for (uint32_t done = 0; done < len;) {
      const uint32_t c =
          (len - done) < static_cast<uint32_t>(kTileElems) ? (len - done) : kTileElems;
      const bool ok = __any_sync(0xffffffffu,
                                 !*abort_flag && mbar_wait_or_abort(full + st, ph, abort_flag));
      if (ok) {
        const T* stage_tile = ring + static_cast<size_t>(st) * kTileElems;
#pragma unroll
        for (int h = 0; h < kTileElems / kTile; ++h) {
          const uint32_t hoff = static_cast<uint32_t>(h * kTile);
          if (hoff < c)
            select_tile_wide<KB, T, NQ>(q, stage_tile + hoff, c - hoff,
                                        static_cast<uint32_t>(a) + done + hoff);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);
      if (++st == stages) {
        st = 0;
        ph ^= 1u;
      }
      done += c;
    }
    g = pend;
    if (layout == kLayoutAliased) {  // lane buffer inside the ring (see bucket_select_tma)
      consumer_sync_wide();
      if (tid == 0) *skip_flag = *abort_flag;
      consumer_sync_wide();
      if (*skip_flag) break;
    }
#pragma unroll
    for (int v = 0; v < NQ; ++v)
      q.store(v, lanebuf + static_cast<size_t>(tid + kWideConsumers * v) * KB);
    consumer_sync_wide();
    if (tid < kThreads)
      finish_piece<KB, kGatherInput, T>(rs, p.b, p.k, r, a, static_cast<int64_t>(len), lanebuf,
                                        cand, p.x + row0, p.out_vals, p.out_idx, piece_flag, NL,
                                        SAMPLE ? p.tail : SampleTail{nullptr, nullptr, 1.0f});
    consumer_sync_wide();
  }
}

template <typename T, int KB>
__global__ void __launch_bounds__(kThreads) bucket_select_general(SelectArgs<T> p, int cand_cap) {
  extern __shared__ __align__(128) unsigned char smem[];
  const SelectSmem L{0, KB, cand_cap, kLanes};
  uint64_t* lanebuf = reinterpret_cast<uint64_t*>(smem + L.lane_off());
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + L.cand_off());
  __shared__ int piece_flag;

  const RowSplit& rs = p.rs;
  const int tid = threadIdx.x;
  const int64_t s0 = cta_start(rs, blockIdx.x);
  const int64_t e0 = cta_start(rs, blockIdx.x + 1);
  const int64_t n = rs.n;
  const int b = p.b;
  const int W = (kLanes / b) * b;  // stripe: lanes per bucket times b
  pdl_wait_then_release();

  Queues<KB> q;
  int64_t g = s0;
  while (g < e0) {
    const int64_t r = g / n;
    const int64_t row0 = r * n;
    const int64_t a = g - row0;
    const int64_t pend = (row0 + n < e0) ? row0 + n : e0;
    const int64_t len = pend - g;
    const T* src = p.x + g;
    q.reset();
    constexpr int U = 4;  // stripes in flight per thread
    for (int64_t base = 0; base < len; base += static_cast<int64_t>(W) * U) {
      float v[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int l = tid + kThreads * w;
          const int64_t off = base + static_cast<int64_t>(W) * u + l;
          v[u][w] = (l < W && off < len) ? to_f32(src[off]) : __uint_as_float(0xff800000u);
        }
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int l = tid + kThreads * w;
          const int64_t off = base + static_cast<int64_t>(W) * u + l;
          if (l < W && off < len) {
            // queue w stores position - w (see Queues)
            const uint32_t base = static_cast<uint32_t>(a + off) - static_cast<uint32_t>(w);
            if (w == 0) q.template offer<0>(v[u][0], base);
            if (w == 1) q.template offer<1>(v[u][1], base);
            if (w == 2) q.template offer<2>(v[u][2], base);
            if (w == 3) q.template offer<3>(v[u][3], base);
          }
        }
      }
    }
#pragma unroll
    for (int w = 0; w < 4; ++w)
      q.store(w, lanebuf + static_cast<size_t>(tid + kThreads * w) * KB);
    group_sync(kThreads);
    finish_piece<KB, kGatherInput, T>(rs, b, p.k, r, a, len, lanebuf, cand, p.x + row0, p.out_vals,
                                      p.out_idx, &piece_flag, kLanes, p.tail);
    group_sync(kThreads);
    g = pend;
  }
}

}  // namespace tk
