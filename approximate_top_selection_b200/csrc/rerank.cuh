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
// One CTA per row.  Duplicate indices (overlapping supports) are dropped by a
// shared-memory hash set (first insert wins; duplicates carry identical
// scores, so which copy survives does not matter) and the distinct candidates
// are listed densely, so no gather pass is spent on an empty or repeated slot
// and Stage 2 sees only real candidates.  A group of D/16 lanes
// scores one candidate: each lane holds 16 query values in registers and
// loads 16 key values with two 16-byte loads (two candidates in flight per
// group; four CTAs per SM so that 512 rows fit one wave), and the group sums with
// shuffles.  Scores become packed (order key, ~index) words, and the shared
// Stage 2 keeps the top k.
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

__host__ __device__ __forceinline__ int rerank_table_size(int c) {
  int h = 64;
  while (h < 2 * c) h <<= 1;
  return h;
}

#ifndef TOPK_RERANK_INFLIGHT
#define TOPK_RERANK_INFLIGHT 2
#endif
#ifndef TOPK_RERANK_MIN_CTAS
#define TOPK_RERANK_MIN_CTAS 4
#endif

template <int D>
__global__ void __launch_bounds__(kThreads, TOPK_RERANK_MIN_CTAS) rerank_kernel(RerankArgs p) {
  constexpr int G = D / 16;          // lanes per candidate
  constexpr int PER_WARP = 32 / G;   // candidates per warp per pass
  extern __shared__ __align__(128) unsigned char smem[];
  const int C = p.c;
  const int cap = sort_capacity(C);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem);                      // [cap]
  int32_t* table = reinterpret_cast<int32_t*>(smem + stage2_bytes(C));  // hash set, then the list
  const int H = rerank_table_size(C);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait_then_release();
  const int64_t r = blockIdx.x;
  const int32_t* ci = p.cand_idx + r * static_cast<int64_t>(C);
  for (int i = tid; i < H; i += kThreads) table[i] = -1;
  for (int i = tid; i < cap; i += kThreads) cand[i] = 0ull;
  group_sync(kThreads);

  // 1. distinct valid indices: cand[j] = 1 marks the slot that owns its index
  bool bad = false;
  for (int j = tid; j < C; j += kThreads) {
    const int32_t i = __ldg(ci + j);
    uint64_t mark = 0ull;
    if (i >= 0 && static_cast<int64_t>(i) < p.n) {
      uint32_t h = (static_cast<uint32_t>(i) * 2654435761u) & static_cast<uint32_t>(H - 1);
      for (int probe = 0; probe < H; ++probe) {
        const int32_t prev = atomicCAS(table + h, -1, i);
        if (prev == -1) {
          mark = 1ull;  // this slot owns index i
          break;
        }
        if (prev == i) break;  // a duplicate
        h = (h + 1u) & static_cast<uint32_t>(H - 1);
      }
    } else if (i >= 0) {
      bad = true;
    }
    cand[j] = mark;
  }
  if (bad) atomicOr(&g_device_status, 2);
  group_sync(kThreads);

  // 2. the (slot, index) list of the owned slots replaces the hash set, and
  //    the marks are cleared so that cand can take the packed words densely
  int* owned_count = reinterpret_cast<int*>(table + H);
  if (tid == 0) *owned_count = 0;
  group_sync(kThreads);
  int32_t* olist = table;  // [2 m]
  for (int base = warp * 32; base < C; base += kThreads) {
    const int j = base + lane;
    const bool own = j < C && cand[j] != 0ull;
    const unsigned mk = __ballot_sync(0xffffffffu, own);
    int at = 0;
    if (lane == 0 && mk) at = atomicAdd(owned_count, __popc(mk));
    at = __shfl_sync(0xffffffffu, at, 0) + __popc(mk & ((1u << lane) - 1u));
    if (own) {
      olist[2 * at] = j;
      olist[2 * at + 1] = __ldg(ci + j);
    }
    if (j < C) {
      cand[j] = 0ull;
      if (!own && p.out_scores)
        p.out_scores[r * static_cast<int64_t>(C) + j] = __int_as_float(0xff800000);
    }
  }
  group_sync(kThreads);
  const int m = *owned_count;

  // 3. exact scores of the m distinct candidates
  const int g = lane / G, gl = lane % G;
  const uint16_t* qr = p.q + r * static_cast<int64_t>(D) + gl * 16;
  float qv[16];
  {
    const uint4 a = *reinterpret_cast<const uint4*>(qr);
    const uint4 b = *reinterpret_cast<const uint4*>(qr + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      qv[2 * t] = bf16_bits_to_float(w[t] & 0xffffu);
      qv[2 * t + 1] = bf16_bits_to_float(w[t] >> 16);
    }
  }
  const uint16_t* Kr = p.K + r * p.kstride;
  // R candidates per lane group in flight: their key loads are all issued
  // before any is used, so a warp keeps 2R 16-byte loads per lane outstanding.
  constexpr int R = TOPK_RERANK_INFLIGHT;
  constexpr int STEP = (kThreads / 32) * PER_WARP;  // candidates per CTA pass
  for (int base = warp * PER_WARP; base < m; base += R * STEP) {
    uint4 ka[R], kb[R];
    int32_t ii[R];
    bool live[R];
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int e = base + u * STEP + g;
      live[u] = e < m;
      ii[u] = live[u] ? olist[2 * e + 1] : 0;
      const uint16_t* kr = Kr + static_cast<int64_t>(ii[u]) * D + gl * 16;
      ka[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(kr)) : make_uint4(0, 0, 0, 0);
      kb[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(kr + 8)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int e = base + u * STEP + g;
      const uint32_t w[8] = {ka[u].x, ka[u].y, ka[u].z, ka[u].w, kb[u].x, kb[u].y, kb[u].z, kb[u].w};
      float s = 0.0f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        s = fmaf(qv[2 * t], bf16_bits_to_float(w[t] & 0xffffu), s);
        s = fmaf(qv[2 * t + 1], bf16_bits_to_float(w[t] >> 16), s);
      }
#pragma unroll
      for (int o = G / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (gl == 0 && live[u]) {
        s = s + 0.0f;  // -0 -> +0: a zero score is +0
        cand[e] = pack(order_key(s), static_cast<uint32_t>(ii[u]));
        if (p.out_scores) p.out_scores[r * static_cast<int64_t>(C) + olist[2 * e]] = s;
      }
    }
  }
  group_sync(kThreads);

  // 4. exact top-k of the m scored candidates
  stage2<kFromKey, float>(cand, m, p.k, nullptr, p.out_vals + r * static_cast<int64_t>(p.k),
                          p.out_idx + r * static_cast<int64_t>(p.k));
}

}  // namespace tk
