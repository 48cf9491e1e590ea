// rerank.cuh -- exact re-scoring of a given candidate index set, then the
// exact top-k of those scores.
//
// Source: "Recall Before You Rank" (ReTopK, arXiv 2607.27692, abstract):
// instead of scoring the current query against the whole key cache, the
// selector reuses the supports retrieved for similar earlier queries; the
// union of those supports is a candidate index set, and the candidates are
// scored exactly against the current query before the top-K is kept.  The
// pages give no kernel; this is the plain reading: score_i = q . K[i] (bf16
// inputs, fp32 accumulation, no 1/sqrt(d)) for every distinct valid candidate
// index i, and the k best (score, index) pairs under the library's total order
// (larger score first, ties by lower index, NaN above +inf), best-first.
//
// Three steps per row:
//  - list: duplicate indices (overlapping supports) are dropped by a bitmap
//    over the n keys (or, for large n, a hash set) in shared memory -- first
//    insert wins; duplicates carry identical scores, so which copy survives
//    does not matter -- and the distinct candidates are listed densely, so no
//    gather is spent on an empty or repeated slot and Stage 2 sees only real
//    candidates;
//  - score: a group of D/16 lanes scores one candidate: each lane holds 16
//    query values in registers and loads 16 key values with two 16-byte loads
//    (R candidates per group in flight), and the group sums with shuffles.
//    Scores become packed (order key, ~index) words in place of the list;
//  - select: the shared Stage 2 keeps the top k, radix-selecting the k best
//    first when that halves the sort.
//
// One CTA per row (four per SM, so that 512 rows fit one wave).
#pragma once

#include "select_core.cuh"

namespace tk {

constexpr int kRerankMaxC = 16 * kThreads;  // 4096 candidates per row

struct RerankArgs {
  const uint16_t* q;   // [rows][d] bf16 bits
  const uint16_t* K;   // bf16 bits; row r uses K + r * kstride, [n][d]
  const int32_t* cand_idx;  // [rows][c], -1 = empty
  int64_t rows, n, kstride;
  int c, k;
  float* out_vals;    // [rows][k]
  int32_t* out_idx;   // [rows][k]
  float* out_scores;  // nullable [rows][c]: score of each slot (-inf: empty, duplicate or invalid)
};

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// Words of the list step's scratch (hash set of 2c slots, or a bitmap of n
// bits when that is no larger); Stage 2 reuses it as its exchange buffer.
__host__ __device__ __forceinline__ int rerank_table_size(int c) {
  int h = 64;
  while (h < 2 * c) h <<= 1;
  return h;
}

#ifndef TOPK_RERANK_INFLIGHT
#define TOPK_RERANK_INFLIGHT 3
#endif
#ifndef TOPK_RERANK_MIN_CTAS
#define TOPK_RERANK_MIN_CTAS 4
#endif
#ifndef TOPK_RERANK_SELECT
#define TOPK_RERANK_SELECT 1
#endif

// List step of row r by threads 0..kThreads-1 (named barrier 1).  cand[0..cap)
// is cleared, then the e-th slot j that owns its index i (the first to insert
// it) is recorded as cand[e] = (j << 32) | i; *count ends at the number of
// distinct valid indices.  Empty, repeated and out-of-range slots get -inf in
// out_scores; an out-of-range index sets device status bit 2.  table: H words.
__device__ __forceinline__ void rerank_list_row(const RerankArgs& p, int64_t r, uint64_t* cand,
                                                uint32_t* table, int H, int* count) {
  constexpr int kPer = kRerankMaxC / kThreads;  // slots per thread
  const int C = p.c;
  const int cap = sort_capacity(C);
  const int tid = threadIdx.x, lane = tid & 31;
  const int32_t* ci = p.cand_idx + r * static_cast<int64_t>(C);
  // Every slot's index is loaded before the scratch is cleared, so the loads
  // are in flight together (slot j = tid + t * kThreads).
  int32_t slot_idx[kPer];
#pragma unroll
  for (int t = 0; t < kPer; ++t) {
    const int j = tid + t * kThreads;
    slot_idx[t] = j < C ? __ldg(ci + j) : -1;
  }
  const bool bitmap = p.n <= 32LL * H;
  const int words = bitmap ? static_cast<int>((p.n + 31) >> 5) : H;
  const uint32_t empty = bitmap ? 0u : 0xffffffffu;
  for (int i = tid; i < words; i += kThreads) table[i] = empty;
  for (int i = tid; i < cap; i += kThreads) cand[i] = 0ull;
  if (tid == 0) *count = 0;
  group_sync(kThreads);
  bool bad = false;
#pragma unroll
  for (int t = 0; t < kPer; ++t) {
    if (t * kThreads >= C) break;  // uniform across the group
    const int j = tid + t * kThreads;
    const int32_t i = slot_idx[t];
    bool own = false;
    if (j < C && i >= 0) {
      if (static_cast<int64_t>(i) >= p.n) {
        bad = true;
      } else if (bitmap) {
        const uint32_t bit = 1u << (i & 31);
        own = (atomicOr(table + (i >> 5), bit) & bit) == 0u;
      } else {
        int* hs = reinterpret_cast<int*>(table);
        uint32_t h = (static_cast<uint32_t>(i) * 2654435761u) & static_cast<uint32_t>(H - 1);
        for (int probe = 0; probe < H; ++probe) {
          const int32_t prev = atomicCAS(hs + h, -1, i);
          if (prev == -1) {
            own = true;
            break;
          }
          if (prev == i) break;  // a duplicate
          h = (h + 1u) & static_cast<uint32_t>(H - 1);
        }
      }
    }
    const unsigned mk = __ballot_sync(0xffffffffu, own);
    int at = 0;
    if (lane == 0 && mk) at = atomicAdd(count, __popc(mk));
    at = __shfl_sync(0xffffffffu, at, 0) + __popc(mk & ((1u << lane) - 1u));
    if (own)
      cand[at] = (static_cast<uint64_t>(j) << 32) | static_cast<uint32_t>(i);
    else if (j < C && p.out_scores)
      p.out_scores[r * static_cast<int64_t>(C) + j] = __int_as_float(0xff800000);
  }
  if (bad) atomicOr(&g_device_status, 2);
  group_sync(kThreads);
}

// Score step of row r by nwarps warps (w = this warp's rank among them): the
// m listed (slot, index) words become packed (order key, ~index) words, and
// the score is written to out_scores at its slot.
template <int D, int R>
__device__ __forceinline__ void rerank_score_row(const RerankArgs& p, int64_t r, uint64_t* cand,
                                                 int m, int w, int nwarps) {
  constexpr int G = D / 16;         // lanes per candidate
  constexpr int PER_WARP = 32 / G;  // candidates per warp per pass
  const int lane = threadIdx.x & 31;
  const int g = lane / G, gl = lane % G;
  const uint16_t* qr = p.q + r * static_cast<int64_t>(D) + gl * 16;
  float qv[16];
  {
    const uint4 a = *reinterpret_cast<const uint4*>(qr);
    const uint4 b = *reinterpret_cast<const uint4*>(qr + 8);
    const uint32_t wq[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      qv[2 * t] = bf16_bits_to_float(wq[t] & 0xffffu);
      qv[2 * t + 1] = bf16_bits_to_float(wq[t] >> 16);
    }
  }
  const uint16_t* Kr = p.K + r * p.kstride;
  // R candidates per lane group in flight: their key loads are all issued
  // before any is used, so a warp keeps 2R 16-byte loads per lane outstanding.
  const int step = nwarps * PER_WARP;  // candidates per pass of the warps
  for (int base = w * PER_WARP; base < m; base += R * step) {
    uint4 ka[R], kb[R];
    int32_t ii[R], slot[R];
    bool live[R];
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int e = base + u * step + g;
      live[u] = e < m;
      const uint64_t ent = live[u] ? cand[e] : 0ull;
      ii[u] = static_cast<int32_t>(static_cast<uint32_t>(ent));
      slot[u] = static_cast<int32_t>(ent >> 32);
      const uint16_t* kr = Kr + static_cast<int64_t>(ii[u]) * D + gl * 16;
      ka[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(kr)) : make_uint4(0, 0, 0, 0);
      kb[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(kr + 8)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int e = base + u * step + g;
      const uint32_t wk[8] = {ka[u].x, ka[u].y, ka[u].z, ka[u].w, kb[u].x, kb[u].y, kb[u].z, kb[u].w};
      float s = 0.0f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        s = fmaf(qv[2 * t], bf16_bits_to_float(wk[t] & 0xffffu), s);
        s = fmaf(qv[2 * t + 1], bf16_bits_to_float(wk[t] >> 16), s);
      }
#pragma unroll
      for (int o = G / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      // Every lane of the group read cand[e] before the shuffles above, so
      // lane 0 of the group may overwrite it now.
      if (gl == 0 && live[u]) {
        s = s + 0.0f;  // -0 -> +0: a zero score is +0
        cand[e] = pack(order_key(s), static_cast<uint32_t>(ii[u]));
        if (p.out_scores) p.out_scores[r * static_cast<int64_t>(p.c) + slot[u]] = s;
      }
    }
  }
}

// Select step of row r by threads 0..kThreads-1: the exact top-k of the m
// scored candidates.  x2 (x2_cap entries) is scratch the sort may use as its
// second exchange buffer.  When keeping k shrinks the sort (k under the next
// power of two below m's), the k best are radix-selected first and only they
// are sorted.
__device__ __forceinline__ void rerank_select_row(const RerankArgs& p, int64_t r, uint64_t* cand,
                                                  int m, uint64_t* x2, int x2_cap) {
  float* ov = p.out_vals + r * static_cast<int64_t>(p.k);
  int32_t* oi = p.out_idx + r * static_cast<int64_t>(p.k);
  const int ept = sort_capacity(m) / kThreads;
  const bool warp_topk = TOPK_WARP_TOPK && m > p.k && m <= 8 * kThreads && p.k <= 32 * ept;
  if (TOPK_RERANK_SELECT && !warp_topk && m > p.k && sort_capacity(p.k) < sort_capacity(m)) {
    switch (ept) {
      case 2: finalize_row_select<2, kFromKey, float>(cand, m, p.k, nullptr, ov, oi, x2, x2_cap); break;
      case 4: finalize_row_select<4, kFromKey, float>(cand, m, p.k, nullptr, ov, oi, x2, x2_cap); break;
      case 8: finalize_row_select<8, kFromKey, float>(cand, m, p.k, nullptr, ov, oi, x2, x2_cap); break;
      default: finalize_row_select<16, kFromKey, float>(cand, m, p.k, nullptr, ov, oi, x2, x2_cap); break;
    }
  } else {
    stage2<kFromKey, float>(cand, m, p.k, nullptr, ov, oi, x2, x2_cap);
  }
}

// One CTA (kThreads threads) per row: list, score with all 8 warps, select.
// Shared memory: stage2_bytes(c) candidate buffer, H scratch words, a counter.
template <int D>
__global__ void __launch_bounds__(kThreads, TOPK_RERANK_MIN_CTAS) rerank_kernel(RerankArgs p) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem);
  uint32_t* table = reinterpret_cast<uint32_t*>(smem + stage2_bytes(p.c));
  const int H = rerank_table_size(p.c);
  int* count = reinterpret_cast<int*>(table + H);
  pdl_wait_then_release();
  const int64_t r = blockIdx.x;
  rerank_list_row(p, r, cand, table, H, count);
  const int m = *count;
  rerank_score_row<D, TOPK_RERANK_INFLIGHT>(p, r, cand, m, threadIdx.x >> 5, kThreads / 32);
  group_sync(kThreads);
  rerank_select_row(p, r, cand, m, reinterpret_cast<uint64_t*>(table), H / 2);
}

}  // namespace tk
