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
  if (!(min_nan_all<U>(x) > __int_as_float(0xff800000))) {
    // NaN or -inf somewhere in this thread's elements: exact update, in order.
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
  if (nq == 1) {
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

// Register queues per CTA of the TMA kernel: four per thread (float4 layout)
// for k_b <= 2, max(256, b) for the sparse k_b > 2 layout.
__host__ __device__ __forceinline__ int select_lanes(int kb, int b) {
  return kb <= 2 ? kLanes : (b > kThreads ? b : kThreads);
}

constexpr int kConsumerWarps = kThreads / 32;
constexpr int kPipeThreads = kThreads + 32;  // consumers + one producer warp

// Warp-specialised streaming: warp kConsumerWarps issues the bulk copies of
// the CTA's tiles into a ring of `stages` shared-memory stages (full barrier:
// bytes landed; empty barrier: every consumer warp is done with the stage);
// the kThreads consumer threads never wait for each other inside a piece.
// SAMPLE: the instantiation that also draws each row's token after Stage 2
// (p.tail); without it the sampling code is not compiled in at all.
template <typename T, int KB, bool SAMPLE = false>
__global__ void __launch_bounds__(kPipeThreads, 2) bucket_select_tma(SelectArgs<T> p, int stages,
                                                                  int cand_cap, int layout) {
  constexpr int kTileElems = Elem<T>::kPerTile;
  extern __shared__ __align__(128) unsigned char smem[];
  const SelectSmem L{stages, KB, cand_cap, select_lanes(KB, p.b), layout};
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
  const int nl = select_lanes(KB, p.b);
  const int nq = nl / kThreads;
  Queues<KB> q;
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
    q.reset();
    for (uint32_t done = 0; done < len;) {
      const uint32_t c =
          (len - done) < static_cast<uint32_t>(kTileElems) ? (len - done) : kTileElems;
      // Warp-uniform: if any lane saw the stage complete, its bytes have landed.
      const bool ok = __any_sync(0xffffffffu,
                                 !*abort_flag && mbar_wait_or_abort(full + st, ph, abort_flag));
      if (ok) {
        const T* stage_tile = ring + static_cast<size_t>(st) * kTileElems;
        if (KB <= 2) {
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
    if (KB <= 2) {
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
  if (!(min_nan_all<U>(x) > __int_as_float(0xff800000))) {
    // NaN or -inf somewhere in this thread's elements: exact update, in order.
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
#pragma unroll
  for (int u = 0; u < U; ++u)
    mask[u % NQ] |=
        (static_cast<uint32_t>(t + CT * u) < c && x[u] > thr[u % NQ]) ? (1u << u) : 0u;
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
