// score_umma.cuh -- fused link-prediction selector: S = Q K^T on the 5th-gen
// tensor cores (tcgen05.mma, bf16 in, fp32 accumulators in TMEM), each score
// pushed straight into its bucket queue by the epilogue; S never reaches HBM.
//
// Application: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
// "Core claim" and Fig. 4 (right): knowledge-graph link prediction scores every
// query against millions of entities and keeps the top k = 100 with k_b = 1.
// Selection: the bucketed two-stage top-k of "What carries the argument".
//
// Work unit = (128 queries, group of 8 buckets).  Entity e = t*b + j belongs to
// bucket j, so a unit walks the entities t*b + 8g + jj (jj < 8) for all t.  The
// TMA engine fetches, per bucket jj, the box {64 d, 1, 32 t} of the key matrix
// viewed as [T][b][d], one after the other: 256 key rows of 128 B with the
// 128-byte swizzle, bucket-major -- exactly a K-major UMMA B operand.
// Accumulator column c of a 128 x 256 tile is then entity
// (t0 + c%32)*b + 8g + c/32: each 32-column TMEM load is one bucket's 32
// stripes, so an epilogue warp owns whole buckets and needs no merge.
//
// Warp roles (576 threads for k_b <= 2, 320 for k_b > 2): warp 0 issues TMA
// loads (Q tile once per unit, key stages through a ring), warp 1 owns TMEM
// (512 columns = two 128x256 fp32 accumulators) and issues the MMAs from one
// thread, and the epilogue warps -- 2..17 (16 warps) for k_b <= 2, 2..9 (8
// warps, more registers per thread for the longer queues) for k_b > 2 -- drain
// TMEM (tcgen05.ld) and update the queues: H warps per TMEM lane quarter, each
// owning 8/H buckets (H = 4 for k_b <= 2, 2 for larger queues).  Per-unit
// results (top-k_b per bucket) go to the workspace; umma_finish runs Stage 2.
//
// The units of one bucket group are consecutive, so the 8 query tiles that read
// the same key rows run at about the same time and share them through L2.
#pragma once

#include <cuda.h>

#include "select_core.cuh"

namespace tk {

constexpr int kUmmaM = 128;            // queries per tile (TMEM lanes)
constexpr int kUmmaN = 256;            // entities per tile (accumulator columns)
constexpr int kUmmaGroup = 8;          // buckets per unit
constexpr int kUmmaTPerTile = kUmmaN / kUmmaGroup;  // 32 stripes per tile
constexpr int kUmmaChunkBytes = 16384;              // 128 rows x 64 bf16 (A chunk)
constexpr int kUmmaStageBytes = 32768;              // 256 rows x 64 bf16 (B stage)
#ifndef TOPK_UMMA_STAGES
#define TOPK_UMMA_STAGES 4
#endif
constexpr int kUmmaStages = TOPK_UMMA_STAGES;
// Epilogue warps: 8 (k_b > 2, more registers per thread) or 16 (k_b <= 2).
__host__ __device__ constexpr int umma_epi_warps(int kb) { return kb <= 2 ? 16 : 8; }
__host__ __device__ constexpr int umma_threads(int kb) { return 64 + 32 * umma_epi_warps(kb); }

struct UmmaArgs {
  int64_t rows, n;   // queries, entities
  int b, T;          // buckets, stripes (n = T * b)
  int mtiles, groups, tiles_per_unit, units;
  float* out_scores;  // nullable [rows][n]
  uint64_t* cand;     // [rows][b][KB]
};

template <int D>
struct UmmaSmem {
  static constexpr int kChunks = D / 64;
  static constexpr size_t a_bytes = static_cast<size_t>(kChunks) * kUmmaChunkBytes;
  static constexpr size_t b_bytes = static_cast<size_t>(kUmmaStages) * kUmmaStageBytes;
  static constexpr size_t bar_bytes = 1024;
  static constexpr size_t total = 1024 /* alignment slack */ + a_bytes + b_bytes + bar_bytes;
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle:
// rows of 128 B, 8-row groups 1024 B apart (stride byte offset), sm_100 form.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                   // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                   // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                   // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: D = f32, A = B = bf16, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// CTA-pair forms (cta_group::2).  The two CTAs of a cluster of 2 form the
// pair; rank 0 (the leader) issues the MMAs, which read the A rows and the B
// half in each CTA's shared memory (same offsets) and write each CTA's TMEM.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_addr(p)), "r"(rank));
  return a;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (either CTA).
// Default (CTA-scope) semantics: what the arrival publishes is the end of
// this warp's TMEM reads, ordered by tcgen05.fence::before_thread_sync; a
// cluster-scope release would add a memory barrier per arrival for nothing.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cbar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cbar) : "memory");
}

// Bulk tensor copies into this CTA's shared memory whose completion is
// counted on an mbarrier of either CTA of the pair (cbar: shared::cluster).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* tm, int c0, int c1,
                                                 uint32_t cbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(cbar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* tm, int c0, int c1,
                                                 int c2, uint32_t cbar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(cbar)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives (once each) on the mbarrier at this offset in both CTAs of the pair
// when the leader's MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], "
      "%1;" ::"r"(smem_addr(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair_own(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ queues
#ifndef TOPK_UMMA_TILE_MAX  // k_b = 1: the maximum of each 32-score load first
#define TOPK_UMMA_TILE_MAX 1
#endif

// NQ bucket queues of KB entries (value domain, as Queues in select_core.cuh),
// storing true entity indices.
template <int NQ, int KB>
struct BucketQueues {
  float val[NQ][KB];
  uint32_t idx[NQ][KB];
  static constexpr uint32_t kEmpty = 0xffffffffu;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int s = 0; s < KB; ++s) {
        val[q][s] = __int_as_float(0xff800000);
        idx[q][s] = kEmpty;
      }
  }

  template <int Q>
  __device__ __forceinline__ void place(const bool (&above)[KB], float x, uint32_t i) {
#pragma unroll
    for (int s = KB - 1; s >= 0; --s) {
      if (s > 0) {
        const bool up = above[s > 0 ? s - 1 : 0];
        const float vs = above[s] ? x : val[Q][s];
        const uint32_t is = above[s] ? i : idx[Q][s];
        val[Q][s] = up ? val[Q][s > 0 ? s - 1 : 0] : vs;
        idx[Q][s] = up ? idx[Q][s > 0 ? s - 1 : 0] : is;
      } else {
        val[Q][0] = above[0] ? x : val[Q][0];
        idx[Q][0] = above[0] ? i : idx[Q][0];
      }
    }
  }

  template <int Q>
  __device__ __forceinline__ void insert_fast(float x, uint32_t i) {
    bool above[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s) above[s] = x > val[Q][s];
    place<Q>(above, x, i);
  }

  template <int Q>
  __device__ __forceinline__ void insert_exact(float x, uint32_t i) {
    const uint32_t kx = order_key(x);
    bool above[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s) above[s] = (idx[Q][s] == kEmpty) || kx > order_key(val[Q][s]);
    place<Q>(above, x, i);
  }
};

// Feeds the 32 scores of one tcgen05.ld -- bucket jb's stripes t0 .. t0+31 --
// to queue QI (a runtime index unrolled by the caller).  Queues store the
// stripe t; the entity t*b + jb is formed when the queue is written out.
template <int KB, int NQ, int QI>
__device__ __forceinline__ void umma_feed_bucket(BucketQueues<NQ, KB>& q, const uint32_t (&r)[32],
                                                 int t0, int T, uint32_t b, uint32_t jb, int64_t row,
                                                 int64_t rows, int64_t n, float* out_scores) {
  float all[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) all[i] = __uint_as_float(r[i]);
  const int valid = T - t0 < 32 ? T - t0 : 32;  // stripes of this tile inside the tensor
  if (out_scores != nullptr && row < rows) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid)
        out_scores[row * n + static_cast<int64_t>(t0 + i) * b + jb] = __uint_as_float(r[i]);
  }
  if constexpr (KB == 1 && TOPK_UMMA_TILE_MAX) {
    // One queue entry takes the best of the 32: the load's maximum (a NaN-
    // keeping max tree, about one ALU instruction per two scores) replaces
    // the queue's entry only if it is strictly larger, at its first position
    // among the 32 (the lowest stripe: ties go to the lower index).  The
    // element-wise path below takes loads whose maximum is NaN or -inf (NaN
    // ranks above everything, -inf must still fill an empty queue) or zero
    // (the element holding it may be -0 while the maximum reads +0); any
    // other maximum has the bits of the elements equal to it.
    const float m = max_nan_all<32>(all);
    if (valid == 32 && m > __int_as_float(0xff800000) && m != 0.0f) {
      if (m > q.val[QI][0]) {
        uint32_t hit = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) hit |= (all[i] == m ? 1u : 0u) << i;
        q.val[QI][0] = m;
        q.idx[QI][0] = static_cast<uint32_t>(t0 + __ffs(static_cast<int>(hit)) - 1);
      }
      return;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid) q.template insert_exact<QI>(__uint_as_float(r[i]), static_cast<uint32_t>(t0 + i));
    return;
  }
  const bool special = !(min_nan_all<32>(all) > __int_as_float(0xff800000));
  if (!special && valid == 32) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      q.template insert_fast<QI>(__uint_as_float(r[i]), static_cast<uint32_t>(t0 + i));
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid) q.template insert_exact<QI>(__uint_as_float(r[i]), static_cast<uint32_t>(t0 + i));
  }
}

// All NQ buckets of a warp, one 32-column TMEM load at a time (queue index
// fixed at compile time).  After the last load the accumulator buffer is
// handed back to the MMA warp before the last bucket is processed.
// PAIR: the buffer's empty barrier is the leader CTA's (acc_empty_cbar, a
// shared::cluster address); else this CTA's (acc_empty_buf).
template <int KB, int NQ, int J, bool PAIR = false>
__device__ __forceinline__ void umma_feed_all(BucketQueues<NQ, KB>& q, uint32_t taddr,
                                              uint64_t* acc_empty_buf, int t0, int T, uint32_t b,
                                              uint32_t jbase, int64_t row, int64_t rows, int64_t n,
                                              float* out_scores, uint32_t acc_empty_cbar = 0) {
  uint32_t r[32];
  tmem_ld_x32(taddr + J * 32, r);
  if constexpr (J + 1 == NQ) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      if constexpr (PAIR)
        mbar_arrive_cluster(acc_empty_cbar);
      else
        mbar_arrive(acc_empty_buf);
    }
  }
  umma_feed_bucket<KB, NQ, J>(q, r, t0, T, b, jbase + J, row, rows, n, out_scores);
  if constexpr (J + 1 < NQ)
    umma_feed_all<KB, NQ, J + 1, PAIR>(q, taddr, acc_empty_buf, t0, T, b, jbase, row, rows, n,
                                       out_scores, acc_empty_cbar);
}

template <int KB, int D>
__global__ void __launch_bounds__(umma_threads(KB), 1)
    score_select_umma(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      UmmaArgs p) {
  constexpr int kEpiWarps = umma_epi_warps(KB);
  constexpr int H = kEpiWarps / 4;             // warps sharing one TMEM lane quarter
  using L = UmmaSmem<D>;
  constexpr int kChunks = L::kChunks;
  constexpr uint32_t kIdesc = umma_idesc_bf16(kUmmaM, kUmmaN);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles.
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* a_tile = smem;
  unsigned char* b_ring = smem + L::a_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::a_bytes + L::b_bytes);
  uint64_t* a_full = bars + 0;
  uint64_t* a_empty = bars + 1;
  uint64_t* full_b = bars + 2;                   // [kUmmaStages]
  uint64_t* empty_b = bars + 2 + kUmmaStages;    // [kUmmaStages]
  uint64_t* acc_full = bars + 2 + 2 * kUmmaStages;   // [2]
  uint64_t* acc_empty = bars + 4 + 2 * kUmmaStages;  // [2]
  uint64_t* mma_done = bars + 6 + 2 * kUmmaStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7 + 2 * kUmmaStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < kUmmaStages; ++s) {
      mbar_init(full_b + s, 1);
      mbar_init(empty_b + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(acc_full + s, 1);
      mbar_init(acc_empty + s, kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_then_release();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0;
      int64_t bt = 0;  // key stages issued
      int iu = 0;
      for (int u = blockIdx.x; u < p.units && !*abort_flag; u += gridDim.x, ++iu) {
        const int m = u % p.mtiles, g = u / p.mtiles;
        if (iu > 0 && !mbar_wait_or_abort(a_empty, static_cast<uint32_t>((iu - 1) & 1), abort_flag))
          break;
        mbar_expect_tx(a_full, static_cast<uint32_t>(L::a_bytes));
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(a_tile + c * kUmmaChunkBytes, &tmQ, c * 64, m * kUmmaM, a_full);
        bool ok = true;
        for (int tile = 0; tile < p.tiles_per_unit && ok; ++tile) {
          for (int c = 0; c < kChunks; ++c) {
            if (bt >= kUmmaStages && !mbar_wait_or_abort(empty_b + st, ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_expect_tx(full_b + st, kUmmaStageBytes);
#pragma unroll
            for (int jj = 0; jj < kUmmaGroup; ++jj)
              tma_load_3d(b_ring + st * kUmmaStageBytes + jj * (kUmmaStageBytes / kUmmaGroup), &tmK,
                          c * 64, g * kUmmaGroup + jj, tile * kUmmaTPerTile, full_b + st);
            ++bt;
            if (++st == kUmmaStages) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA can go away.
        const unsigned long long start = global_ns();
        bool drained = true;
        for (int64_t x = (bt > kUmmaStages ? bt - kUmmaStages : 0); drained && x < bt; ++x)
          drained = drain_wait(full_b + (x % kUmmaStages),
                               static_cast<uint32_t>((x / kUmmaStages) & 1), start);
        if (drained && iu > 0) drain_wait(a_full, static_cast<uint32_t>((iu - 1) & 1), start);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0;
      int64_t tg = 0;  // tiles issued by this CTA
      int iu = 0;
      const uint32_t a_base = smem_addr(a_tile), b_base = smem_addr(b_ring);
      for (int u = blockIdx.x; u < p.units && !*abort_flag; u += gridDim.x, ++iu) {
        if (!mbar_wait_or_abort(a_full, static_cast<uint32_t>(iu & 1), abort_flag)) break;
        bool ok = true;
        for (int tile = 0; tile < p.tiles_per_unit && ok; ++tile, ++tg) {
          const int buf = static_cast<int>(tg & 1);
          if (tg >= 2 &&
              !mbar_wait_or_abort(acc_empty + buf, static_cast<uint32_t>(((tg >> 1) - 1) & 1),
                                  abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * kUmmaN);
          for (int c = 0; c < kChunks; ++c) {
            if (!mbar_wait_or_abort(full_b + st, ph, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = umma_desc_sw128(a_base + c * kUmmaChunkBytes + kk * 32);
              const uint64_t bd = umma_desc_sw128(b_base + st * kUmmaStageBytes + kk * 32);
              umma_bf16(d_tmem, ad, bd, kIdesc, (c | kk) != 0 ? 1u : 0u);
            }
            umma_commit(empty_b + st);  // the stage is free once these MMAs are done
            if (++st == kUmmaStages) {
              st = 0;
              ph ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(acc_full + buf);
        }
        if (!ok) break;
        umma_commit(a_empty);
      }
      // Every MMA this thread issued has completed before TMEM is released.
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, 1000000000ull);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;            // TMEM lanes this warp may read
    const int slice = ew >> 2;               // which buckets of the group (0 .. H-1)
    constexpr int kBucketsPerWarp = kUmmaGroup / H;
    const int64_t row_in_tile = quarter * 32 + lane;
    BucketQueues<kBucketsPerWarp, KB> q;
    int64_t tg = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
      const int m = u % p.mtiles, g = u / p.mtiles;
      const int64_t row = static_cast<int64_t>(m) * kUmmaM + row_in_tile;
      const uint32_t jbase = static_cast<uint32_t>(g * kUmmaGroup + slice * kBucketsPerWarp);
      q.reset();
      bool ok = true;
      for (int tile = 0; tile < p.tiles_per_unit; ++tile, ++tg) {
        const int buf = static_cast<int>(tg & 1);
        ok = __any_sync(0xffffffffu,
                        !*abort_flag && mbar_wait_or_abort(acc_full + buf,
                                                           static_cast<uint32_t>((tg >> 1) & 1),
                                                           abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int t0 = tile * kUmmaTPerTile;
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(buf * kUmmaN + slice * kBucketsPerWarp * 32);
        umma_feed_all<KB, kBucketsPerWarp, 0>(q, taddr, acc_empty + buf, t0, p.T,
                                              static_cast<uint32_t>(p.b), jbase, row, p.rows, p.n,
                                              p.out_scores);
      }
      if (!ok) break;
      if (row < p.rows) {
        uint64_t* dst = p.cand + (static_cast<size_t>(row) * p.b + jbase) * KB;
#pragma unroll
        for (int jj = 0; jj < kBucketsPerWarp; ++jj)
#pragma unroll
          for (int s2 = 0; s2 < KB; ++s2)
            dst[static_cast<size_t>(jj) * KB + s2] =
                q.idx[jj][s2] != BucketQueues<kBucketsPerWarp, KB>::kEmpty
                    ? pack(order_key(q.val[jj][s2]),
                           q.idx[jj][s2] * static_cast<uint32_t>(p.b) + jbase + jj)
                    : 0ull;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

// ------------------------------------------------------------------ CTA pair
// The same selector on a pair of CTAs (a cluster of 2 on neighbouring SMs)
// with tcgen05.mma.cta_group::2: work unit = 256 queries x one group of 8
// buckets.  Each CTA loads its own 128 query rows (A) and half of every key
// tile -- CTA r the 4 buckets 4r .. 4r+3 of the group, 128 key rows -- into
// its own shared memory, so each key tile crosses L2 once per 256 queries
// instead of once per 128, and each SM reads half the B operand per MMA.  The
// leader (rank 0) issues M=256, N=256 MMAs; accumulator rows 0..127 land in
// CTA 0's TMEM and rows 128..255 in CTA 1's, all 256 columns each, so each
// CTA's epilogue drains its own TMEM exactly as in score_select_umma.  Both
// CTAs' copies count on the leader's full barriers (the cta_group::2 form of
// the bulk tensor copy; no multicast load anywhere); the leader's commits
// arrive on both CTAs' barriers; the peer's epilogue hands accumulators back
// through the leader's empty barrier.  Every wait is bounded; both CTAs meet
// at a cluster barrier before the TMEM is freed and the CTAs exit.
constexpr int kUmmaPairM = 2 * kUmmaM;                           // 256 queries per unit
constexpr int kUmmaPairStageBytes = kUmmaStageBytes / 2;         // 128 key rows x 64 bf16
#ifndef TOPK_UMMA_PAIR_STAGES
#define TOPK_UMMA_PAIR_STAGES 4
#endif
constexpr int kUmmaPairStages = TOPK_UMMA_PAIR_STAGES;
// Accumulator buffers of 256 TMEM columns (2: the epilogue drains one while
// the MMAs fill the other).
#ifndef TOPK_UMMA_PAIR_ACC_BUFS
#define TOPK_UMMA_PAIR_ACC_BUFS 2
#endif
constexpr int kUmmaPairAccBufs = TOPK_UMMA_PAIR_ACC_BUFS;
constexpr int kUmmaPairTmemCols = kUmmaPairAccBufs * kUmmaN;

template <int D>
struct UmmaPairSmem {
  static constexpr int kChunks = D / 64;
  static constexpr size_t a_bytes = static_cast<size_t>(kChunks) * kUmmaChunkBytes;
  static constexpr size_t b_bytes = static_cast<size_t>(kUmmaPairStages) * kUmmaPairStageBytes;
  static constexpr size_t bar_bytes = 1024;
  static constexpr size_t total = 1024 /* alignment slack */ + a_bytes + b_bytes + bar_bytes;
};

template <int KB, int D>
__global__ void __launch_bounds__(umma_threads(KB), 1)
    score_select_umma_pair(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK, UmmaArgs p) {
  constexpr int kEpiWarps = umma_epi_warps(KB);
  constexpr int H = kEpiWarps / 4;
  using L = UmmaPairSmem<D>;
  constexpr int kChunks = L::kChunks;
  constexpr int kHalf = kUmmaGroup / 2;  // buckets whose key rows this CTA loads
  constexpr uint32_t kIdesc = umma_idesc_bf16(kUmmaPairM, kUmmaN);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* a_tile = smem;
  unsigned char* b_ring = smem + L::a_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::a_bytes + L::b_bytes);
  uint64_t* a_full = bars + 0;                          // leader's counts both CTAs' A copies
  uint64_t* a_empty = bars + 1;                         // both CTAs (commit multicast)
  uint64_t* full_b = bars + 2;                          // [stages], leader's
  uint64_t* empty_b = bars + 2 + kUmmaPairStages;       // [stages], both CTAs
  uint64_t* acc_full = bars + 2 + 2 * kUmmaPairStages;  // [2], both CTAs
  uint64_t* acc_empty = bars + 4 + 2 * kUmmaPairStages; // [2], leader's (both epilogues)
  uint64_t* mma_done = bars + 6 + 2 * kUmmaPairStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7 + 2 * kUmmaPairStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = static_cast<int>(blockIdx.x >> 1), pairs = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < kUmmaPairStages; ++s) {
      mbar_init(full_b + s, 1);
      mbar_init(empty_b + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(acc_full + s, 1);
      mbar_init(acc_empty + s, 2 * kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kUmmaPairTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised and their TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_then_release();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t a_full_c = cluster_addr(a_full, 0);
      int st = 0;
      uint32_t ph = 0;
      int64_t bt = 0;  // key stages issued
      int iu = 0;
      for (int u = pair; u < p.units && !*abort_flag; u += pairs, ++iu) {
        const int m = u % p.mtiles, g = u / p.mtiles;
        if (iu > 0 && !mbar_wait_or_abort(a_empty, static_cast<uint32_t>((iu - 1) & 1), abort_flag))
          break;
        if (rank == 0) mbar_expect_tx(a_full, static_cast<uint32_t>(2 * L::a_bytes));
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d_pair(a_tile + c * kUmmaChunkBytes, &tmQ, c * 64,
                           m * kUmmaPairM + static_cast<int>(rank) * kUmmaM, a_full_c);
        bool ok = true;
        for (int tile = 0; tile < p.tiles_per_unit && ok; ++tile) {
          for (int c = 0; c < kChunks; ++c) {
            if (bt >= kUmmaPairStages && !mbar_wait_or_abort(empty_b + st, ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            if (rank == 0) mbar_expect_tx(full_b + st, 2 * kUmmaPairStageBytes);
            const uint32_t full_c = cluster_addr(full_b + st, 0);
#pragma unroll
            for (int jj = 0; jj < kHalf; ++jj)
              tma_load_3d_pair(b_ring + st * kUmmaPairStageBytes + jj * (kUmmaPairStageBytes / kHalf),
                               &tmK, c * 64, g * kUmmaGroup + static_cast<int>(rank) * kHalf + jj,
                               tile * kUmmaTPerTile, full_c);
            ++bt;
            if (++st == kUmmaPairStages) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // The leader can tell when the copies it counted have landed; the
        // peer's completions count on the leader's barriers, so the peer
        // waits on the stages' release by the leader (bounded) instead.
        const unsigned long long start = global_ns();
        bool drained = true;
        for (int64_t x = (bt > kUmmaPairStages ? bt - kUmmaPairStages : 0); drained && x < bt; ++x)
          drained = rank == 0 ? drain_wait(full_b + (x % kUmmaPairStages),
                                           static_cast<uint32_t>((x / kUmmaPairStages) & 1), start)
                              : true;
        if (drained && iu > 0 && rank == 0)
          drain_wait(a_full, static_cast<uint32_t>((iu - 1) & 1), start);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      int st = 0;
      uint32_t ph = 0;
      int64_t tg = 0;
      int iu = 0;
      const uint32_t a_base = smem_addr(a_tile), b_base = smem_addr(b_ring);
      for (int u = pair; u < p.units && !*abort_flag; u += pairs, ++iu) {
        if (!mbar_wait_or_abort(a_full, static_cast<uint32_t>(iu & 1), abort_flag)) break;
        bool ok = true;
        for (int tile = 0; tile < p.tiles_per_unit && ok; ++tile, ++tg) {
          const int buf = static_cast<int>(tg % kUmmaPairAccBufs);
          const int64_t use = tg / kUmmaPairAccBufs;  // earlier uses of this buffer
          if (use >= 1 &&
              !mbar_wait_or_abort(acc_empty + buf, static_cast<uint32_t>((use - 1) & 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * kUmmaN);
          for (int c = 0; c < kChunks; ++c) {
            if (!mbar_wait_or_abort(full_b + st, ph, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = umma_desc_sw128(a_base + c * kUmmaChunkBytes + kk * 32);
              const uint64_t bd = umma_desc_sw128(b_base + st * kUmmaPairStageBytes + kk * 32);
              umma_bf16_pair(d_tmem, ad, bd, kIdesc, (c | kk) != 0 ? 1u : 0u);
            }
            umma_commit_pair_both(empty_b + st);  // both CTAs' halves of the stage are free
            if (++st == kUmmaPairStages) {
              st = 0;
              ph ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit_pair_both(acc_full + buf);
        }
        if (!ok) break;
        umma_commit_pair_both(a_empty);
      }
      umma_commit_pair_own(mma_done);
      mbar_wait(mma_done, 0, 1000000000ull);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int slice = ew >> 2;
    constexpr int kBucketsPerWarp = kUmmaGroup / H;
    const int64_t row_in_tile = static_cast<int64_t>(rank) * kUmmaM + quarter * 32 + lane;
    const uint32_t acc_empty_c[2] = {cluster_addr(acc_empty, 0),
                                     cluster_addr(acc_empty + (kUmmaPairAccBufs - 1), 0)};
    BucketQueues<kBucketsPerWarp, KB> q;
    int64_t tg = 0;
    for (int u = pair; u < p.units; u += pairs) {
      const int m = u % p.mtiles, g = u / p.mtiles;
      const int64_t row = static_cast<int64_t>(m) * kUmmaPairM + row_in_tile;
      const uint32_t jbase = static_cast<uint32_t>(g * kUmmaGroup + slice * kBucketsPerWarp);
      q.reset();
      bool ok = true;
      for (int tile = 0; tile < p.tiles_per_unit; ++tile, ++tg) {
        const int buf = static_cast<int>(tg % kUmmaPairAccBufs);
        ok = __any_sync(0xffffffffu,
                        !*abort_flag &&
                            mbar_wait_or_abort(acc_full + buf,
                                               static_cast<uint32_t>((tg / kUmmaPairAccBufs) & 1),
                                               abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int t0 = tile * kUmmaTPerTile;
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(buf * kUmmaN + slice * kBucketsPerWarp * 32);
        umma_feed_all<KB, kBucketsPerWarp, 0, true>(q, taddr, acc_empty + buf, t0, p.T,
                                                    static_cast<uint32_t>(p.b), jbase, row, p.rows,
                                                    p.n, p.out_scores, acc_empty_c[buf]);
      }
      if (!ok) break;
      if (row < p.rows) {
        uint64_t* dst = p.cand + (static_cast<size_t>(row) * p.b + jbase) * KB;
#pragma unroll
        for (int jj = 0; jj < kBucketsPerWarp; ++jj)
#pragma unroll
          for (int s2 = 0; s2 < KB; ++s2)
            dst[static_cast<size_t>(jj) * KB + s2] =
                q.idx[jj][s2] != BucketQueues<kBucketsPerWarp, KB>::kEmpty
                    ? pack(order_key(q.val[jj][s2]),
                           q.idx[jj][s2] * static_cast<uint32_t>(p.b) + jbase + jj)
                    : 0ull;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs are done and no CTA touches the other's memory any more
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kUmmaPairTmemCols)
                 : "memory");
  }
}

// Stage 2 of the tensor-core path: per query, the exact top-k of the b*k_b
// bucket candidates (the workspace is cleared behind the reads).
#ifndef TOPK_FINISH_MIN_CTAS  // resident CTAs per SM the register budget is cut for
#define TOPK_FINISH_MIN_CTAS 6
#endif
template <int KB>
__global__ void __launch_bounds__(kThreads, TOPK_FINISH_MIN_CTAS)
    umma_finish(uint64_t* cand_ws, int64_t rows, int b,
                                                        int k, float* out_vals, int32_t* out_idx) {

  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem);
  const int64_t r = blockIdx.x;
  pdl_wait_then_release();
  for (int j = threadIdx.x; j < b; j += kThreads) {
    uint64_t best[KB];
#pragma unroll
    for (int s = 0; s < KB; ++s) best[s] = 0;
    uint64_t* src = cand_ws + (static_cast<size_t>(r) * b + j) * KB;
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      keep_best<KB>(best, src[s]);
      src[s] = 0ull;  // leave the workspace zeroed for the next call
    }
#pragma unroll
    for (int s = 0; s < KB; ++s) cand[static_cast<size_t>(j) * KB + s] = best[s];
  }
  group_sync(kThreads);
  stage2<kFromKey, float>(cand, b * KB, k, nullptr, out_vals + r * k, out_idx + r * k);
}

}  // namespace tk
