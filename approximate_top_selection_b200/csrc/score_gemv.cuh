// score_gemv.cuh -- fused selector: score_i = q . K_i (bf16 in, fp32 accumulate)
// streamed straight into the bucket queues; the score matrix never reaches HBM.
//
// Selector: "Recall Before You Rank" (ReTopK), abstract -- identifying the
// top-K subset scores the current query against the full KV cache before a
// global top-K, so selector cost is linear in context length; STARC page,
// Fig. 3 -- q in R^{1 x d_h}, K in R^{L x d_h} per head.  Selection:
// "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
// "What carries the argument" (bucketed two-stage top-k).
//
// One query against its key matrix is a GEMV (about 1 flop per byte of keys),
// bound by HBM bandwidth, so the dot products run on the CUDA cores: D/32
// threads share a key, each holding 32 query values in registers, and a
// 2- or 3-step shuffle sums their partial products.  Keys arrive through the
// TMA engine (cp.async.bulk) in 16 KB tiles into a ring of shared-memory
// stages.  Thread (key j, part p) reads its four 16-byte chunks of the key in
// an order rotated by j, which keeps the shared-memory reads conflict-free;
// its query registers are loaded in the same rotated order once per row.
// Scores go to a 1024-entry shared buffer, which the same bucket queues as
// the float32 kernel consume (thread t owns positions 4t..4t+3).
#pragma once

#include "select_core.cuh"

namespace tk {

constexpr int kKeyTileBytes = 16384;

struct ScoreArgs {
  const uint16_t* q;  // [rows][D]
  const uint16_t* K;  // row r: K + r*kstride, [n][D]
  int64_t kstride;
  int k, b;
  float* out_vals;
  int32_t* out_idx;
  float* out_scores;  // nullable [rows][n]
  RowSplit rs;        // over keys
};

struct ScoreSmem {
  int stages, kb, cand_cap;
  __host__ __device__ size_t ring_bytes() const {
    return static_cast<size_t>(stages) * kKeyTileBytes;
  }
  // The score blocks (streaming) and the lane lists (end of a piece) are never
  // live at the same time, so they share one region.
  __host__ __device__ size_t sbuf_bytes() const { return 2 * kLanes * 4; }
  __host__ __device__ size_t lane_bytes() const { return static_cast<size_t>(kLanes) * kb * 8; }
  __host__ __device__ size_t shared_region() const {
    return sbuf_bytes() > lane_bytes() ? sbuf_bytes() : lane_bytes();
  }
  __host__ __device__ size_t cand_bytes() const {
    return static_cast<size_t>(cand_cap) * 8 + kStage2Extra;
  }
  __host__ __device__ size_t bar_bytes() const { return 16 * static_cast<size_t>(stages) + 16; }
  __host__ __device__ size_t total() const {
    return ring_bytes() + shared_region() + cand_bytes() + bar_bytes();
  }
};

constexpr int kScoreConsumerWarps = kThreads / 32;
constexpr int kScorePipeThreads = kThreads + 32;

template <int KB, int D>
__global__ void __launch_bounds__(kScorePipeThreads, 2)
    score_select_gemv(ScoreArgs p, int stages, int cand_cap) {
  constexpr int TPK = D / 32;            // threads per key
  constexpr int KR = kThreads / TPK;     // keys per tile
  constexpr int KEY_BYTES = D * 2;
  static_assert(KR * KEY_BYTES == kKeyTileBytes, "tile size");
  static_assert(kLanes % KR == 0, "score block must hold whole tiles");

  extern __shared__ __align__(128) unsigned char smem[];
  const ScoreSmem L{stages, KB, cand_cap};
  unsigned char* ring = smem;
  float* sbuf = reinterpret_cast<float*>(smem + L.ring_bytes());
  uint64_t* lanebuf = reinterpret_cast<uint64_t*>(smem + L.ring_bytes());  // aliases sbuf
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + L.ring_bytes() + L.shared_region());
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.ring_bytes() + L.shared_region() +
                                               L.cand_bytes());
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  int* piece_flag = reinterpret_cast<int*>(empty + stages) + 1;

  const RowSplit& rs = p.rs;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t s0 = cta_start(rs, blockIdx.x);
  const int64_t e0 = cta_start(rs, blockIdx.x + 1);
  const int64_t n = rs.n;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kScoreConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait_then_release();

  if (warp == kScoreConsumerWarps) {  // ---------------- producer
    if (lane == 0) {
      int64_t g = s0, t = 0;
      int st = 0;       // stage of tile t
      uint32_t ph = 0;  // parity of t / stages
      while (g < e0) {
        const int64_t r = g / n;
        const int64_t rowend = (r + 1) * n;
        int64_t c = e0 - g;
        if (rowend - g < c) c = rowend - g;
        if (c > KR) c = KR;
        if (t >= stages && !mbar_wait_or_abort(empty + st, ph ^ 1u, abort_flag)) break;
        const uint32_t bytes = static_cast<uint32_t>(c * KEY_BYTES);
        const uint16_t* src = p.K + r * p.kstride + (g - r * n) * D;
        mbar_expect_tx(full + st, bytes);
        bulk_g2s(ring + static_cast<size_t>(st) * kKeyTileBytes, src, bytes, full + st);
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
  const int j = tid / TPK;     // key slot within a tile
  const int part = tid % TPK;  // which share of the key's chunks
  Queues<KB> q;
  float qf[4][8];
  int st = 0;       // ring stage of the next tile
  uint32_t ph = 0;  // its full-barrier parity
  int64_t g = s0;
  while (g < e0) {
    const int64_t r = g / n;
    const int64_t row0 = r * n;
    const int64_t a = g - row0;
    const int64_t pend = (row0 + n < e0) ? row0 + n : e0;
    const int64_t len = pend - g;
    // This thread's 32 query values, in the rotated chunk order it reads keys in.
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int chunk = part + TPK * ((c + j) & 3);
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.q + r * D + chunk * 8));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        qf[c][2 * h] = __uint_as_float(ws[h] << 16);
        qf[c][2 * h + 1] = __uint_as_float(ws[h] & 0xffff0000u);
      }
    }
    q.reset();
    int64_t done = 0;  // keys of this piece already scored
    while (done < len) {

      const int64_t c = (len - done) < KR ? (len - done) : KR;
      // Warp-uniform: if any lane saw the stage complete, its bytes have landed.
      const bool ok = __any_sync(0xffffffffu,
                                 !*abort_flag &&
                                     mbar_wait_or_abort(full + st, ph, abort_flag));
      if (ok) {
        const unsigned char* key = ring + static_cast<size_t>(st) * kKeyTileBytes + j * KEY_BYTES;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int chunk = part + TPK * ((cc + j) & 3);
          const uint4 w = *reinterpret_cast<const uint4*>(key + chunk * 16);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            acc0 = fmaf(__uint_as_float(ws[h] << 16), qf[cc][2 * h], acc0);
            acc1 = fmaf(__uint_as_float(ws[h] & 0xffff0000u), qf[cc][2 * h + 1], acc1);
          }
        }
        float acc = acc0 + acc1;
#pragma unroll
        for (int m = 1; m < TPK; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        if (part == 0 && j < c) {
          const int64_t pos = done + j;  // piece-relative
          sbuf[((pos / kLanes) & 1) * kLanes + (pos % kLanes)] = acc;
          if (p.out_scores) p.out_scores[row0 + a + pos] = acc;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);
      if (++st == stages) {
        st = 0;
        ph ^= 1u;
      }
      done += c;
      if (done % kLanes == 0 || done == len) {
        // A block of up to 1024 scores is complete: feed the bucket queues.
        group_sync(kThreads);
        const int64_t blk = (done - 1) / kLanes;
        const int64_t valid = done - blk * kLanes;
        const int off = 4 * tid;
        if (off < valid) {
          const float4 v = *reinterpret_cast<const float4*>(sbuf + (blk & 1) * kLanes + off);
          const uint32_t pos0 = static_cast<uint32_t>(a + blk * kLanes + off);
          if (off + 4 <= valid)
            q.offer4(v, pos0);
          else
            q.exact4(v, pos0, static_cast<int>(valid - off));
        }
      }
    }
    group_sync(kThreads);  // the last score block has been read: lanebuf may overwrite it
#pragma unroll
    for (int v = 0; v < 4; ++v) q.store(v, lanebuf + static_cast<size_t>(4 * tid + v) * KB);
    group_sync(kThreads);
    finish_piece<KB, kFromKey, float>(rs, p.b, p.k, r, a, len, lanebuf, cand, nullptr, p.out_vals,
                               p.out_idx, piece_flag);
    group_sync(kThreads);
    g = pend;
  }
}

}  // namespace tk
