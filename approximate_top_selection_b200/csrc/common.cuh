// common.cuh -- shared device helpers: order-preserving keys, packed candidates,
// bounded mbarrier waits and the bulk (TMA) global->shared copy.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tk {

constexpr int kThreads = 256;         // threads per CTA of the streaming kernels
constexpr int kLanes = 4 * kThreads;  // register queues per CTA (4 per thread)
constexpr int kMaxKb = 4;
constexpr int kMaxB = 1024;
constexpr int kMaxK = 16384;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

// Device status word (bit set of TOPK_DEV_* codes), read by topk_device_status().
// The library is one translation unit, so this is its only definition.
__device__ int g_device_status = 0;

// ---------------------------------------------------------------- ordering keys
// Total order of the method's readings: larger value first; -0 ties +0; NaN
// above +inf; ties by lower index.  order_key maps a float to a uint32 whose
// unsigned order is that value order (index excluded).  Key 0 is never produced
// (it would be a negative NaN, and NaNs are all mapped to 0xFFFFFFFF), so 0
// marks an empty queue slot.
__device__ __forceinline__ uint32_t order_key(float v) {
  const float z = __fadd_rn(v, 0.0f);  // -0 + 0 = +0 under round-to-nearest
  const uint32_t u = __float_as_uint(z);
  const uint32_t key = u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
  return (v != v) ? 0xFFFFFFFFu : key;
}

__device__ __forceinline__ float key_value(uint32_t key) {
  const uint32_t u = (key & 0x80000000u) ? (key ^ 0x80000000u) : ~key;
  return __uint_as_float(u);
}

// A candidate packs (key, index) so that a larger 64-bit integer ranks first:
// key in the high word, the complement of the index in the low word.
__device__ __forceinline__ uint64_t pack(uint32_t key, uint32_t idx) {
  return key ? ((static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(~idx)) : 0ull;
}
__device__ __forceinline__ uint32_t packed_key(uint64_t p) { return static_cast<uint32_t>(p >> 32); }
__device__ __forceinline__ uint32_t packed_idx(uint64_t p) { return ~static_cast<uint32_t>(p); }

// min that returns NaN when either operand is NaN (PTX min.NaN, sm_80+).
__device__ __forceinline__ float fmin_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// max that returns NaN when either operand is NaN (PTX max.NaN).
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Programmatic dependent launch.  Kernels are launched so that they may start
// while the previous kernel of the stream finishes; every thread waits here
// (until that kernel has completed and its writes are visible) before it
// touches global memory, and then lets the next kernel of the stream start
// its own set-up early in the same way.
__device__ __forceinline__ void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Three-input form (sm_100).
__device__ __forceinline__ float fmin3_nan(float a, float b, float c) {
  float d;
  asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Three-input max that keeps NaN (sm_100).
__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// NaN-keeping maximum of N values (three-input steps).
template <int N>
__device__ __forceinline__ float max_nan_all(const float (&v)[N]) {
  float m[(N + 2) / 3];
#pragma unroll
  for (int i = 0; i < (N + 2) / 3; ++i) {
    const float a = v[3 * i];
    const float b = 3 * i + 1 < N ? v[3 * i + 1] : a;
    const float c = 3 * i + 2 < N ? v[3 * i + 2] : a;
    m[i] = fmax3_nan(a, b, c);
  }
  if constexpr ((N + 2) / 3 == 1)
    return m[0];
  else
    return max_nan_all<(N + 2) / 3>(m);
}

// NaN-keeping minimum of N values (three-input steps).
template <int N>
__device__ __forceinline__ float min_nan_all(const float (&v)[N]) {
  float m[(N + 2) / 3];
#pragma unroll
  for (int i = 0; i < (N + 2) / 3; ++i) {
    const float a = v[3 * i];
    const float b = 3 * i + 1 < N ? v[3 * i + 1] : a;
    const float c = 3 * i + 2 < N ? v[3 * i + 2] : a;
    m[i] = fmin3_nan(a, b, c);
  }
  if constexpr ((N + 2) / 3 == 1)
    return m[0];
  else
    return min_nan_all<(N + 2) / 3>(m);
}

// ---------------------------------------------------------------- mbarrier / bulk copy
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase with the given parity to complete, for at most `limit`
// nanoseconds.  Returns false (and records TOPK_DEV_WAIT_TIMEOUT) on expiry.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit) {
      atomicOr(&g_device_status, 1);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// As mbar_wait, but also gives up as soon as *abort (shared) becomes non-zero,
// and raises *abort itself when the time limit expires.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_device_status, 1);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// Device status bit of a drain that expired (TOPK_DEV_DRAIN_TIMEOUT).
constexpr int kDevDrainTimeout = 4;

// One wait of the drain that follows an abort: all waits of one drain share a
// single deadline, kWaitLimitNs after `start`.  On expiry records
// TOPK_DEV_DRAIN_TIMEOUT and returns false.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity,
                                           unsigned long long start) {
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - start > kWaitLimitNs) {
      atomicOr(&g_device_status, kDevDrainTimeout);
      return false;
    }
  }
  return true;
}

// After an abort, the producer waits until the bulk copies it already issued
// -- tiles [t0, t1) of a ring of `stages` stages with full barriers `full` --
// have landed, so that the CTA never exits while a copy still writes into its
// shared memory.  If even that drain runs out of time, the status says so and
// the CTA exits anyway: the context is then to be treated as unusable.
__device__ __forceinline__ void drain_copies(uint64_t* full, int stages, int64_t t0, int64_t t1) {
  const unsigned long long start = global_ns();
  for (int64_t u = t0; u < t1; ++u)
    if (!drain_wait(full + (u % stages), static_cast<uint32_t>((u / stages) & 1), start)) return;
}

// Barrier over the first `nthreads` threads of the CTA (named barrier 1), so a
// producer warp outside that group never has to take part.
__device__ __forceinline__ void group_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Bulk asynchronous copy global -> shared (the TMA engine, non-tensor form).
// dst, src 16-byte aligned; bytes a multiple of 16.  Completion is signalled as
// transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------- partition
// The flattened element space [0, E) of all rows is cut into G contiguous CTA
// ranges of equal size (to within one unit of `align` elements).
__host__ __device__ __forceinline__ int64_t part_start(int64_t units, int G, int c, int align,
                                                       int64_t E) {
  return c >= G ? E : (units * c / G) * align;
}

// CTA whose range holds element g.
__host__ __device__ __forceinline__ int part_of(int64_t g, int64_t units, int G, int align) {
  const int64_t w = g / align;
  int64_t c = ((w + 1) * G - 1) / units;
  if (c > G - 1) c = G - 1;
  return static_cast<int>(c);
}

// Bounded-wait self-test: one thread waits on an mbarrier that nothing will
// complete, for at most limit_ns, then returns; the expiry is recorded in the
// device status like any other expired wait.  Exercises the failure path of
// every bounded wait without a fault, a trap or a hang.
__global__ void wait_timeout_probe(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait(&bar, 0u, limit_ns);
  }
}

}  // namespace tk
