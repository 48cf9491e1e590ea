// topk_api.cu -- the C ABI (include/topk_b200.h): argument checks, launch
// plans and kernel launches.  All device work lives in the included kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/topk_b200.h"
#include "bucket_select.cuh"
#include "exact_topk.cuh"
#include "merge_select.cuh"
#include "rerank.cuh"
#include "sample.cuh"
#include "score_gemv.cuh"
#include "score_umma.cuh"

namespace tk {
namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxN = 2147483647LL;       // indices are int32
constexpr int64_t kMaxElems = 1LL << 50;      // keeps the partition arithmetic in int64
constexpr int64_t kSelectMinPiece = 16384;    // elements per CTA before splitting pays
constexpr int64_t kScoreMinPiece = 1024;      // keys per CTA

// Ring depth: as many tile stages (32 KB for score rows, 16 KB for key tiles)
// as fit while kCtasPerSm CTAs share an SM's shared memory (bytes in flight
// per SM are what keeps HBM busy), clamped.
#ifndef TOPK_CTAS_PER_SM
#define TOPK_CTAS_PER_SM 2
#endif
#ifndef TOPK_MAX_STAGES
#define TOPK_MAX_STAGES 8
#endif
constexpr size_t kSmemPerSm = 228 * 1024;
constexpr size_t kSmemReservedPerCta = 1024;

template <typename Layout>
int fit_stages(Layout L, int min_stages) {
  const size_t budget = kSmemPerSm / TOPK_CTAS_PER_SM - kSmemReservedPerCta;
  int st = TOPK_MAX_STAGES;
  for (; st > min_stages; --st) {
    L.stages = st;
    if (L.total() <= budget) break;
  }
  return st;
}

struct DeviceInfo {
  bool init = false;
  int sms = 0;
  int max_smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TOPK_ECUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return TOPK_ECUDA;
    if (cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
      return TOPK_ECUDA;
    d.init = true;
  }
  *out = d;
  return TOPK_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int host_next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Launch plan shared by topk_bucketed / score_topk and their workspace query.
struct Plan {
  int G = 0;
  int align = 1;
  int stages = 0;
  int cand_cap = 0;
  size_t smem = 0;
  int64_t units = 0;
  size_t ws_tickets = 0;  // bytes
  size_t ws_slots = 0;    // bytes
  int wide_nq = 0;        // k_b > 2 fast path: queues per thread of the 16-warp kernel
  int layout = kLayoutSeparate;  // shared-memory layout of the streaming kernel (SelectLayout)
  bool keys = false;      // bf16 rows with k_b >= 2 in order-key queues (KeyQueues)
  size_t workspace() const { return ws_tickets + ws_slots; }
};

// Resident CTAs per SM of (kernel, dynamic smem) on a device, cached: the
// attribute call and the occupancy query cost microseconds of host time.
struct OccKey {
  int dev;
  const void* fn;
  size_t smem;
  int blocks;
};
constexpr int kOccSlots = 256;
OccKey g_occ[kOccSlots];
int g_occ_n = 0;
std::mutex g_occ_mu;

// Kernels whose dynamic shared-memory limit has been raised, per device.  The
// limit is raised once to the device's opt-in maximum, so any later launch of
// the kernel may use any size up to it (a per-size setting would be undone by
// the next call that asks for less).
struct AttrKey {
  int dev;
  const void* fn;
};
AttrKey g_attr[kOccSlots];
int g_attr_n = 0;

template <typename KernelT>
int raise_smem_limit_locked(KernelT kernel, int dev, int max_optin) {
  const void* fn = reinterpret_cast<const void*>(kernel);
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].dev == dev && g_attr[i].fn == fn) return TOPK_OK;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return TOPK_ECUDA;
  const int dyn_max = max_optin - static_cast<int>(fa.sharedSizeBytes);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) !=
      cudaSuccess)
    return TOPK_ECUDA;
  if (g_attr_n >= kOccSlots) return TOPK_ECUDA;
  g_attr[g_attr_n++] = AttrKey{dev, fn};
  return TOPK_OK;
}

template <typename KernelT>
int prepare_kernel(KernelT kernel) {
  int dev = 0, max_optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TOPK_ECUDA;
  if (cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
      cudaSuccess)
    return TOPK_ECUDA;
  std::lock_guard<std::mutex> lk(g_occ_mu);
  return raise_smem_limit_locked(kernel, dev, max_optin);
}

template <typename KernelT>
int occupancy(KernelT kernel, int block, size_t smem, int* blocks) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TOPK_ECUDA;
  const void* fn = reinterpret_cast<const void*>(kernel);
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    for (int i = 0; i < g_occ_n; ++i) {
      if (g_occ[i].dev == dev && g_occ[i].fn == fn && g_occ[i].smem == smem) {
        *blocks = g_occ[i].blocks;
        return TOPK_OK;
      }
    }
  }
  int rc = prepare_kernel(kernel);
  if (rc) return rc;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, kernel, block, smem) != cudaSuccess)
    return TOPK_ECUDA;
  if (*blocks < 1) return TOPK_EUNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_occ_mu);
  if (g_occ_n < kOccSlots) g_occ[g_occ_n++] = OccKey{dev, fn, smem, *blocks};
  return TOPK_OK;
}

// Number of CTAs: one per row when the rows alone fill the GPU and fit in one
// resident wave (no row is split); otherwise the flattened element space is cut
// into equal ranges, as many as fit in one wave, but no smaller than min_piece.
int choose_grid(int64_t rows, int64_t E, int align, int64_t min_piece, int sms, int per_sm) {
  const int64_t cap = static_cast<int64_t>(sms) * per_sm;
  const int64_t units = E / align;
  int64_t G;
#ifndef TOPK_GRID_ONE_ROW_PER_CTA
#define TOPK_GRID_ONE_ROW_PER_CTA 1
#endif
  if (TOPK_GRID_ONE_ROW_PER_CTA && rows <= cap && (rows >= sms || rows * min_piece >= E)) {
    G = rows;  // one row per CTA: no row is split
  } else {
    G = std::min<int64_t>(cap, std::max<int64_t>(1, (E + min_piece - 1) / min_piece));
    G = std::max<int64_t>(G, std::min<int64_t>(rows, cap));
  }
  G = std::max<int64_t>(1, std::min<int64_t>(G, units));
  return static_cast<int>(G);
}

#ifndef TOPK_WIDE_SPARSE
#define TOPK_WIDE_SPARSE 1
#endif

#ifndef TOPK_ALIAS_RING
#define TOPK_ALIAS_RING 1
#endif

// Ring stages, shared memory and resident CTAs of a fast-path plan with the
// given shared-memory layout (SelectLayout).
template <typename KernelT>
int fit_fast(KernelT kernel, int threads, int KB, int nl, int layout, Plan* pl,
             const DeviceInfo& dev, int* per_sm) {
  SelectSmem L{0, KB, pl->cand_cap, nl, layout};
  pl->stages = fit_stages(L, 2);
  L.stages = pl->stages;
  pl->smem = L.total();
  pl->layout = layout;
  if (pl->smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
  return occupancy(kernel, threads, pl->smem, per_sm);
}

template <typename T, int KB>
int plan_select_kb(bool fast, int64_t rows, int64_t n, int b, const DeviceInfo& dev, Plan* pl) {
  const int C = b * KB;
  pl->cand_cap = sort_capacity(C);
  pl->align = fast ? Elem<T>::kAlign : 1;
  pl->wide_nq = 0;
  pl->layout = kLayoutSeparate;
  pl->keys = false;
  int per_sm = 0;
  const int64_t E = rows * n;
  if (fast) {
    // bf16 rows (short enough for 16-bit queue ordinals): packed bf16x2 queues
    // (k_b <= 2) or order-key queues (k_b > 2) in the float4 layout.  Otherwise k_b > 2 with b >= 512:
    // the 16-warp kernel, one lane per bucket (b lanes); smaller b keeps the
    // 8-warp kernel, whose 256 lanes split a bucket over fewer queues (fewer
    // inserts).
    constexpr bool kKeyType = sizeof(T) == 2 && KB >= TOPK_BF16_KEYS_MIN_KB;
    // The packed queues keep ordinal 0xFFFF for an empty slot: one stripe less.
    const bool keys = kKeyType && TOPK_BF16_KEYS &&
                      n <= (KB <= TOPK_BF16_PAIR_MAX_KB ? kKeyMaxPiece - kLanes : kKeyMaxPiece);
    pl->keys = keys;
    const bool wide = !keys && KB >= TOPK_SPARSE_MIN_KB && TOPK_WIDE_SPARSE && b >= kWideConsumers;
    pl->wide_nq = wide ? (b > kWideConsumers ? b / kWideConsumers : 1) : 0;
    const int nl = wide ? kWideConsumers * pl->wide_nq : select_lanes(KB, b, keys);
    auto fit = [&](int layout) -> int {
      if constexpr (kKeyType) {
        if (keys)
          return fit_fast(bucket_select_tma<T, KB, false, true>, kPipeThreads, KB, nl, layout, pl,
                          dev, &per_sm);
      }
      if (!wide)
        return fit_fast(bucket_select_tma<T, KB>, kPipeThreads, KB, nl, layout, pl, dev, &per_sm);
      if (pl->wide_nq == 1)
        return fit_fast(bucket_select_wide<T, (KB >= TOPK_SPARSE_MIN_KB ? KB : 3), 1>, kWideThreads, KB, nl, layout,
                        pl, dev, &per_sm);
      return fit_fast(bucket_select_wide<T, (KB >= TOPK_SPARSE_MIN_KB ? KB : 3), 2>, kWideThreads, KB, nl, layout, pl,
                      dev, &per_sm);
    };
    // One whole row per CTA (n a multiple of the alignment): every CTA streams
    // a single piece, so its lane and Stage-2 buffers can share the ring.  The
    // aliased layout is tried first (its smaller footprint can be what makes
    // a row per CTA fit), the plain one otherwise.
    int rc = TOPK_EUNSUPPORTED;
    if (TOPK_ALIAS_RING && n % pl->align == 0) {
      rc = fit(kLayoutAliased);
      if (!rc && choose_grid(rows, E, pl->align, kSelectMinPiece, dev.sms, per_sm) != rows)
        rc = TOPK_EUNSUPPORTED;
    }
    if (rc) rc = fit(kLayoutSeparate);
    if (rc) return rc;
  } else {
    pl->stages = 0;
    SelectSmem L{0, KB, pl->cand_cap, kLanes};
    pl->smem = L.total();
    if (pl->smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
    int rc = occupancy(bucket_select_general<T, KB>, kThreads, pl->smem, &per_sm);
    if (rc) return rc;
  }
  pl->G = choose_grid(rows, E, pl->align, kSelectMinPiece, dev.sms, per_sm);
  pl->units = E / pl->align;
  pl->ws_tickets = align_up(static_cast<size_t>(rows) * 4, 256);
  pl->ws_slots = static_cast<size_t>(pl->G) * 2 * C * 8;
  return TOPK_OK;
}

template <typename T = float>
int plan_select(bool fast, int64_t rows, int64_t n, int b, int kb, const DeviceInfo& dev,
                Plan* pl) {
  switch (kb) {
    case 1: return plan_select_kb<T, 1>(fast, rows, n, b, dev, pl);
    case 2: return plan_select_kb<T, 2>(fast, rows, n, b, dev, pl);
    case 3: return plan_select_kb<T, 3>(fast, rows, n, b, dev, pl);
    case 4: return plan_select_kb<T, 4>(fast, rows, n, b, dev, pl);
  }
  return TOPK_EINVAL;
}

template <int KB, int D>
int plan_score_kd(int64_t rows, int64_t n, int b, const DeviceInfo& dev, Plan* pl) {
  const int C = b * KB;
  pl->cand_cap = sort_capacity(C);
  pl->align = 1;
  pl->stages = fit_stages(ScoreSmem{0, KB, pl->cand_cap}, 2);
  ScoreSmem L{pl->stages, KB, pl->cand_cap};
  pl->smem = L.total();
  if (pl->smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
  int per_sm = 0;
  int rc = occupancy(score_select_gemv<KB, D>, kScorePipeThreads, pl->smem, &per_sm);
  if (rc) return rc;
  const int64_t E = rows * n;
  pl->G = choose_grid(rows, E, 1, kScoreMinPiece, dev.sms, per_sm);
  pl->units = E;
  pl->ws_tickets = align_up(static_cast<size_t>(rows) * 4, 256);
  pl->ws_slots = static_cast<size_t>(pl->G) * 2 * C * 8;
  return TOPK_OK;
}

template <int KB>
int plan_score_k(int64_t rows, int64_t n, int b, int d, const DeviceInfo& dev, Plan* pl) {
  if (d == 128) return plan_score_kd<KB, 128>(rows, n, b, dev, pl);
  if (d == 256) return plan_score_kd<KB, 256>(rows, n, b, dev, pl);
  return TOPK_EUNSUPPORTED;
}

int plan_score(int64_t rows, int64_t n, int b, int kb, int d, const DeviceInfo& dev, Plan* pl) {
  switch (kb) {
    case 1: return plan_score_k<1>(rows, n, b, d, dev, pl);
    case 2: return plan_score_k<2>(rows, n, b, d, dev, pl);
    case 3: return plan_score_k<3>(rows, n, b, d, dev, pl);
    case 4: return plan_score_k<4>(rows, n, b, d, dev, pl);
  }
  return TOPK_EINVAL;
}

int check_common(int64_t rows, int64_t n, int k, int b, int kb) {
  if (rows < 1 || n < 1 || k < 1 || b < 1 || kb < 1 || kb > kMaxKb) return TOPK_EINVAL;
  if (n > kMaxN) return TOPK_EINVAL;
  if (rows > kMaxElems / n) return TOPK_EUNSUPPORTED;
  if (b > kMaxB || k > kMaxK) return TOPK_EUNSUPPORTED;
  return TOPK_OK;
}

// The TMA kernel needs 16-byte aligned rows (bulk copies) and b | 1024 (each
// register queue sees a single bucket).
template <typename T>
bool select_fast(const T* x, int64_t n, int b) {
  return aligned16(x) && (n % Elem<T>::kAlign) == 0 && (kLanes % b) == 0;
}

RowSplit make_split(const Plan& pl, int64_t rows, int64_t n, void* ws) {
  RowSplit rs;
  rs.rows = rows;
  rs.n = n;
  rs.E = rows * n;
  rs.units = pl.units;
  rs.G = pl.G;
  rs.align = pl.align;
  rs.tickets = static_cast<uint32_t*>(ws);
  rs.slots = reinterpret_cast<uint64_t*>(static_cast<unsigned char*>(ws) + pl.ws_tickets);
  return rs;
}

// A row is split iff the plan gives it to more than one CTA; only then is the
// workspace touched.  With G == rows and one row per CTA no workspace is needed.
bool plan_needs_workspace(const Plan& pl, int64_t rows, int64_t n) {
  if (pl.G == rows && pl.align == 1) return false;
  if (pl.G == rows && (n % pl.align) == 0) return false;
  return true;
}

// Launch errors are read right after the launch; a non-sticky error left by
// an earlier, unrelated runtime call is cleared first (clear_launch_error) so
// that it is not reported as this launch's failure.
void clear_launch_error() { (void)cudaGetLastError(); }

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TOPK_OK : TOPK_ECUDA;
}

// Launch with programmatic stream serialisation: the kernel may begin while
// the previous kernel on the stream finishes; it waits on the device
// (griddepcontrol.wait) before reading or writing global memory.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  clear_launch_error();
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    (void)cudaGetLastError();
    return TOPK_ECUDA;
  }
  return launch_status();
}

// launch_pdl for a kernel launched in clusters of cluster_x CTAs (along x).
template <typename... KArgs, typename... Args>
int launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  clear_launch_error();
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    (void)cudaGetLastError();
    return TOPK_ECUDA;
  }
  return launch_status();
}

template <typename T, int KB>
int launch_select_kb(bool fast, const Plan& pl, const SelectArgs<T>& a, cudaStream_t st) {
  const bool sample = a.tail.token != nullptr;
  if constexpr (KB >= TOPK_SPARSE_MIN_KB) {
    if (fast && pl.wide_nq > 0) {
      auto go = [&](auto kernel) -> int {
        int rc = prepare_kernel(kernel);
        if (rc) return rc;
        return launch_pdl(kernel, dim3(pl.G), dim3(kWideThreads), pl.smem, st, a, pl.stages,
                          pl.cand_cap, pl.layout);
      };
      if (sample)
        return pl.wide_nq == 1 ? go(bucket_select_wide<T, KB, 1, true>)
                               : go(bucket_select_wide<T, KB, 2, true>);
      return pl.wide_nq == 1 ? go(bucket_select_wide<T, KB, 1>) : go(bucket_select_wide<T, KB, 2>);
    }
  }
  if constexpr (sizeof(T) == 2 && KB >= TOPK_BF16_KEYS_MIN_KB) {
    if (fast && pl.keys) {
      auto go = [&](auto kernel) -> int {
        int rc = prepare_kernel(kernel);
        if (rc) return rc;
        return launch_pdl(kernel, dim3(pl.G), dim3(kPipeThreads), pl.smem, st, a, pl.stages,
                          pl.cand_cap, pl.layout);
      };
      return sample ? go(bucket_select_tma<T, KB, true, true>)
                    : go(bucket_select_tma<T, KB, false, true>);
    }
  }
  if (fast && sample) {
    int rc = prepare_kernel(bucket_select_tma<T, KB, true>);
    if (rc) return rc;
    return launch_pdl(bucket_select_tma<T, KB, true>, dim3(pl.G), dim3(kPipeThreads), pl.smem, st,
                      a, pl.stages, pl.cand_cap, pl.layout);
  }
  if (fast)
    return launch_pdl(bucket_select_tma<T, KB>, dim3(pl.G), dim3(kPipeThreads), pl.smem, st, a,
                      pl.stages, pl.cand_cap, pl.layout);
  return launch_pdl(bucket_select_general<T, KB>, dim3(pl.G), dim3(kThreads), pl.smem, st, a,
                    pl.cand_cap);
}

template <typename T>
int launch_select(int kb, bool fast, const Plan& pl, const SelectArgs<T>& a, cudaStream_t st) {
  switch (kb) {
    case 1: return launch_select_kb<T, 1>(fast, pl, a, st);
    case 2: return launch_select_kb<T, 2>(fast, pl, a, st);
    case 3: return launch_select_kb<T, 3>(fast, pl, a, st);
    default: return launch_select_kb<T, 4>(fast, pl, a, st);
  }
}

// topk_bucketed for either element type.
template <typename T>
int run_bucketed(const T* scores, int64_t rows, int64_t n, int k, int b, int kb, T* out_vals,
                 int32_t* out_idx, void* workspace, size_t workspace_bytes, void* stream,
                 const SampleTail& tail = SampleTail{nullptr, nullptr, 1.0f}) {
  if (!scores || !out_vals || !out_idx) return TOPK_EINVAL;
  int rc = check_common(rows, n, k, b, kb);
  if (rc) return rc;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev))) return rc;
  const bool fast = select_fast(scores, n, b);
  Plan pl;
  if ((rc = plan_select<T>(fast, rows, n, b, kb, dev, &pl))) return rc;
  if (plan_needs_workspace(pl, rows, n)) {
    if (!workspace || workspace_bytes < pl.workspace()) return TOPK_EWORKSPACE;
    if (!aligned16(workspace)) return TOPK_EINVAL;
  }
  SelectArgs<T> a;
  a.x = scores;
  a.k = k;
  a.b = b;
  a.out_vals = out_vals;
  a.out_idx = out_idx;
  a.rs = make_split(pl, rows, n, workspace);
  a.tail = tail;
  return launch_select<T>(kb, fast, pl, a, static_cast<cudaStream_t>(stream));
}

// Workspace of topk_bucketed for either element type: enough for the fast and
// the general plan, whichever the pointer's alignment selects.
template <typename T>
size_t bucketed_workspace(int64_t rows, int64_t n, int b, int kb, const DeviceInfo& dev) {
  Plan p1, p2;
  size_t need = 0;
  bool any = false;
  if (plan_select<T>(true, rows, n, b, kb, dev, &p1) == TOPK_OK) {
    need = p1.workspace();
    any = true;
  }
  if (plan_select<T>(false, rows, n, b, kb, dev, &p2) == TOPK_OK) {
    need = std::max(need, p2.workspace());
    any = true;
  }
  return any ? need : 0;
}

template <int KB, int D>
int launch_score_kd(const Plan& pl, const ScoreArgs& a, cudaStream_t st) {
  return launch_pdl(score_select_gemv<KB, D>, dim3(pl.G), dim3(kScorePipeThreads), pl.smem, st, a,
                    pl.stages, pl.cand_cap);
}

template <int KB>
int launch_score_k(int d, const Plan& pl, const ScoreArgs& a, cudaStream_t st) {
  if (d == 128) return launch_score_kd<KB, 128>(pl, a, st);
  return launch_score_kd<KB, 256>(pl, a, st);
}

// ---------------------------------------------------------------- tensor-core path
// Fused link-prediction selector on tcgen05 (score_umma.cuh): one key matrix
// shared by all rows, b a multiple of 8 dividing n, enough rows to fill M tiles.
constexpr int64_t kUmmaMinRows = 32;

bool umma_eligible(int64_t rows, int64_t n, int64_t kstride, int b, int d) {
  return kstride == 0 && rows >= kUmmaMinRows && (b % kUmmaGroup) == 0 && (n % b) == 0 &&
         (d == 128 || d == 256) && rows <= (1LL << 31) - 1;
}

size_t umma_workspace(int64_t rows, int b, int kb) {
  return static_cast<size_t>(rows) * b * kb * 8;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;

int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  std::lock_guard<std::mutex> lk(g_encode_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || fn == nullptr)
      return TOPK_ECUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_encode;
  return TOPK_OK;
}

// The CTA-pair selector (score_select_umma_pair) serves 256 or more queries.
#ifndef TOPK_UMMA_PAIR
#define TOPK_UMMA_PAIR 1
#endif
constexpr int64_t kUmmaPairMinRows = 2 * kUmmaM;

// Clusters of two CTAs of the pair kernel that can be resident at once on the
// current device (cached per device and kernel): the grid's number of pairs.
// 0 when the kernel does not fit.
struct PairSlots {
  int dev;
  const void* fn;
  int pairs;
};
PairSlots g_pair_slots[kOccSlots];
int g_pair_n = 0;
std::mutex g_pair_mu;

template <typename KernelT>
int umma_pair_slots(KernelT kernel, int threads, size_t smem, const DeviceInfo& dev, int* pairs) {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return TOPK_ECUDA;
  const void* fn = reinterpret_cast<const void*>(kernel);
  {
    std::lock_guard<std::mutex> lk(g_pair_mu);
    for (int i = 0; i < g_pair_n; ++i)
      if (g_pair_slots[i].dev == d && g_pair_slots[i].fn == fn) {
        *pairs = g_pair_slots[i].pairs;
        return TOPK_OK;
      }
  }
  *pairs = 0;
  if (smem <= static_cast<size_t>(dev.max_smem_optin)) {
    int rc = prepare_kernel(kernel);
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * dev.sms));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      clusters = 0;  // no pair form on this device: the single-CTA kernel serves
    }
    *pairs = clusters;
  }
  std::lock_guard<std::mutex> lk(g_pair_mu);
  if (g_pair_n < kOccSlots) g_pair_slots[g_pair_n++] = PairSlots{d, fn, *pairs};
  return TOPK_OK;
}

template <int KB, int D>
int launch_umma_kd(const uint16_t* q, int64_t rows, const uint16_t* K, int64_t n, int b, int k,
                   float* out_vals, int32_t* out_idx, float* out_scores, void* ws,
                   const DeviceInfo& dev, cudaStream_t st) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  int rc = tensor_map_encoder(&encode);
  if (rc) return rc;
  const int64_t T = n / b;
  CUtensorMap tmQ, tmK;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, kUmmaM};
    const cuuint32_t es[2] = {1, 1};
    if (encode(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(q), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return TOPK_ECUDA;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(b),
                                static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(b) * D * 2};
    const cuuint32_t box[3] = {64, 1, kUmmaTPerTile};  // one bucket's 32 stripes per load
    const cuuint32_t es[3] = {1, 1, 1};
    if (encode(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(K), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return TOPK_ECUDA;
  }
  UmmaArgs a;
  a.rows = rows;
  a.n = n;
  a.b = b;
  a.T = static_cast<int>(T);
  a.groups = b / kUmmaGroup;
  a.tiles_per_unit = static_cast<int>((T + kUmmaTPerTile - 1) / kUmmaTPerTile);
  a.out_scores = out_scores;
  a.cand = static_cast<uint64_t*>(ws);
  if ((rc = prepare_kernel(umma_finish<KB>))) return rc;
  int pairs = 0;
  if (TOPK_UMMA_PAIR && rows >= kUmmaPairMinRows &&
      (rc = umma_pair_slots(score_select_umma_pair<KB, D>, umma_threads(KB), UmmaPairSmem<D>::total,
                            dev, &pairs)))
    return rc;
  if (pairs > 0) {
    // A pair of CTAs per 256-query tile (cta_group::2).
    a.mtiles = static_cast<int>((rows + kUmmaPairM - 1) / kUmmaPairM);
    a.units = a.mtiles * a.groups;
    const int grid = 2 * std::min(a.units, pairs);
    if ((rc = launch_pdl_cluster(score_select_umma_pair<KB, D>, dim3(grid), dim3(umma_threads(KB)),
                                 UmmaPairSmem<D>::total, st, 2, tmQ, tmK, a)))
      return rc;
  } else {
    a.mtiles = static_cast<int>((rows + kUmmaM - 1) / kUmmaM);
    a.units = a.mtiles * a.groups;
    const size_t smem = UmmaSmem<D>::total;
    if (smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
    if ((rc = prepare_kernel(score_select_umma<KB, D>))) return rc;
    const int grid = std::min(a.units, dev.sms);
    if ((rc = launch_pdl(score_select_umma<KB, D>, dim3(grid), dim3(umma_threads(KB)), smem, st,
                         tmQ, tmK, a)))
      return rc;
  }
  const size_t fsmem = stage2_bytes(b * KB);
  return launch_pdl(umma_finish<KB>, dim3(static_cast<unsigned>(rows)), dim3(kThreads), fsmem, st,
                    a.cand, rows, b, k, out_vals, out_idx);
}

template <int KB>
int launch_umma_k(int d, const uint16_t* q, int64_t rows, const uint16_t* K, int64_t n, int b,
                  int k, float* ov, int32_t* oi, float* os, void* ws, const DeviceInfo& dev,
                  cudaStream_t st) {
  if (d == 128) return launch_umma_kd<KB, 128>(q, rows, K, n, b, k, ov, oi, os, ws, dev, st);
  return launch_umma_kd<KB, 256>(q, rows, K, n, b, k, ov, oi, os, ws, dev, st);
}

// ---------------------------------------------------------------- no-alloc scratch
// Built-in scratch of topk_bucketed_noalloc.  In host code this name is only a
// stand-in for the symbol: the device address is looked up per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TOPK_NOALLOC_SCRATCH_BYTES];

struct ScratchAddr {
  bool init = false;
  CUcontext ctx = nullptr;  // the context the address belongs to
  void* ptr = nullptr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device and context: after a device reset the runtime creates a new
// context in which the buffer has a new address, so the lookup is redone.
int noalloc_scratch_ptr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TOPK_ECUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_ctx_current) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || fn == nullptr)
      return TOPK_ECUDA;
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  CUcontext ctx = nullptr;  // null until the runtime has bound the device's context
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return TOPK_ECUDA;
  ScratchAddr& s = g_scratch_addr[dev];
  if (!s.init || ctx == nullptr || s.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return TOPK_ECUDA;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return TOPK_ECUDA;
    s.ptr = p;
    s.ctx = ctx;
    s.init = true;
  }
  *out = s.ptr;
  return TOPK_OK;
}

}  // namespace
}  // namespace tk

using namespace tk;

extern "C" {

const char* topk_status_string(int status) {
  switch (status) {
    case TOPK_OK: return "TOPK_OK";
    case TOPK_EINVAL: return "TOPK_EINVAL: invalid argument";
    case TOPK_EUNSUPPORTED: return "TOPK_EUNSUPPORTED: valid but not implemented by this build";
    case TOPK_ECUDA: return "TOPK_ECUDA: CUDA call or kernel launch failed";
    case TOPK_EWORKSPACE: return "TOPK_EWORKSPACE: workspace missing or too small";
    case TOPK_ESCRATCH:
      return "TOPK_ESCRATCH: the call needs more scratch than the built-in buffer of "
             "topk_bucketed_noalloc holds";
  }
  return "unknown topk status";
}

size_t topk_workspace_bytes(int op, int64_t rows, int64_t n, int k, int b, int kb, int d) {
  DeviceInfo dev;
  if (current_device_info(&dev)) return 0;
  Plan pl;
  if (op == TOPK_OP_EXACT) return 0;
  if (check_common(rows, n, k, b, kb)) return 0;
  if (op == TOPK_OP_BUCKETED) return bucketed_workspace<float>(rows, n, b, kb, dev);
  if (op == TOPK_OP_BUCKETED_BF16) return bucketed_workspace<uint16_t>(rows, n, b, kb, dev);
  if (op == TOPK_OP_SCORE) {
    if (kLanes % b) return 0;
    if (plan_score(rows, n, b, kb, d, dev, &pl)) return 0;
    size_t need = pl.workspace();
    if (umma_eligible(rows, n, 0, b, d)) need = std::max(need, umma_workspace(rows, b, kb));
    return need;
  }
  return 0;
}

int topk_bucketed(const float* scores, int64_t rows, int64_t n, int k, int b, int kb,
                  float* out_vals, int32_t* out_idx, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return run_bucketed<float>(scores, rows, n, k, b, kb, out_vals, out_idx, workspace,
                             workspace_bytes, stream);
}

int topk_bucketed_bf16(const uint16_t* scores, int64_t rows, int64_t n, int k, int b, int kb,
                       uint16_t* out_vals, int32_t* out_idx, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return run_bucketed<uint16_t>(scores, rows, n, k, b, kb, out_vals, out_idx, workspace,
                                workspace_bytes, stream);
}

int topk_bucketed_noalloc(const float* scores, int64_t rows, int64_t n, int k, int b, int kb,
                          float* out_vals, int32_t* out_idx, void* stream) {
  if (!scores || !out_vals || !out_idx) return TOPK_EINVAL;
  int rc = check_common(rows, n, k, b, kb);
  if (rc) return rc;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev))) return rc;
  const bool fast = select_fast(scores, n, b);
  Plan pl;
  if ((rc = plan_select<float>(fast, rows, n, b, kb, dev, &pl))) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch_ptr(&scratch))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (plan_needs_workspace(pl, rows, n)) {
    if (pl.workspace() > static_cast<size_t>(TOPK_NOALLOC_SCRATCH_BYTES)) return TOPK_ESCRATCH;
    // The tickets must start at zero whatever an earlier call left behind.
    if (cudaMemsetAsync(scratch, 0, pl.ws_tickets, st) != cudaSuccess) return TOPK_ECUDA;
  }
  SelectArgs<float> a;
  a.x = scores;
  a.k = k;
  a.b = b;
  a.out_vals = out_vals;
  a.out_idx = out_idx;
  a.rs = make_split(pl, rows, n, scratch);
  a.tail = SampleTail{nullptr, nullptr, 1.0f};
  return launch_select<float>(kb, fast, pl, a, st);
}

int topk_exact(const float* scores, int64_t rows, int64_t n, int k, float* out_vals,
               int32_t* out_idx, void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!scores || !out_vals || !out_idx) return TOPK_EINVAL;
  if (rows < 1 || n < 1 || k < 1 || n > kMaxN) return TOPK_EINVAL;
  if (k > kMaxK || rows > 2147483647LL) return TOPK_EUNSUPPORTED;
  DeviceInfo dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  ExactSmem L{n <= kSortCap ? host_next_pow2(static_cast<int>(n)) : 0,
              host_next_pow2(k)};
  const size_t smem = L.total();
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
  if ((rc = prepare_kernel(exact_topk_kernel))) return rc;
  return launch_pdl(exact_topk_kernel, dim3(static_cast<unsigned>(rows)), dim3(kExactThreads), smem,
                    static_cast<cudaStream_t>(stream), scores, n, k, L.sel_cap, out_vals, out_idx);
}

int topk_bucketed_merge(const float* vals, const int32_t* idx, int parts, int64_t rows, int m,
                        const int64_t* part_offset, int64_t n_total, int k, int b, int kb,
                        float* out_vals, int32_t* out_idx, void* stream) {
  if (!vals || !idx || !out_vals || !out_idx) return TOPK_EINVAL;
  if (parts < 1 || m < 1) return TOPK_EINVAL;
  int rc = check_common(rows, n_total, k, b, kb);
  if (rc) return rc;
  if (parts > kMergeMaxParts || rows > 2147483647LL) return TOPK_EUNSUPPORTED;
  if (static_cast<int64_t>(parts) * m > kMaxElems / rows) return TOPK_EUNSUPPORTED;
  MergeArgs a{};
  a.vals = vals;
  a.idx = idx;
  a.parts = parts;
  a.m = m;
  a.k = k;
  a.b = b;
  a.rows = rows;
  a.n_total = n_total;
  a.out_vals = out_vals;
  a.out_idx = out_idx;
  for (int i = 0; i < parts; ++i) {
    const int64_t o = part_offset ? part_offset[i] : 0;
    if (o < 0 || o >= n_total) return TOPK_EINVAL;
    a.offs[i] = o;
  }
  DeviceInfo dev;
  if ((rc = current_device_info(&dev))) return rc;
  const size_t smem = stage2_bytes(b * kb);
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(rows)), block(kThreads);
  switch (kb) {
    case 1:
      if ((rc = prepare_kernel(bucket_merge_kernel<1>))) return rc;
      return launch_pdl(bucket_merge_kernel<1>, grid, block, smem, st, a);
    case 2:
      if ((rc = prepare_kernel(bucket_merge_kernel<2>))) return rc;
      return launch_pdl(bucket_merge_kernel<2>, grid, block, smem, st, a);
    case 3:
      if ((rc = prepare_kernel(bucket_merge_kernel<3>))) return rc;
      return launch_pdl(bucket_merge_kernel<3>, grid, block, smem, st, a);
    default:
      if ((rc = prepare_kernel(bucket_merge_kernel<4>))) return rc;
      return launch_pdl(bucket_merge_kernel<4>, grid, block, smem, st, a);
  }
}

int score_rerank(const uint16_t* q, int64_t rows, int d, const uint16_t* K, int64_t n,
                 int64_t k_batch_stride, const int32_t* cand_idx, int c, int k, float* out_vals,
                 int32_t* out_idx, float* out_scores, void* stream) {
  if (!q || !K || !cand_idx || !out_vals || !out_idx) return TOPK_EINVAL;
  if (rows < 1 || n < 1 || n > kMaxN || c < 1 || k < 1 || k_batch_stride < 0) return TOPK_EINVAL;
  if (d != 128 && d != 256) return TOPK_EUNSUPPORTED;
  if (c > kRerankMaxC || k > kMaxK || rows > 2147483647LL) return TOPK_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(K) || (k_batch_stride % 8) != 0) return TOPK_EINVAL;
  DeviceInfo dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  RerankArgs a{q, K, cand_idx, rows, n, k_batch_stride, c, k, out_vals, out_idx, out_scores};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t smem = stage2_bytes(c) + static_cast<size_t>(rerank_table_size(c)) * 4 + 16;
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return TOPK_EUNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(rows)), block(kThreads);
  if (d == 128) {
    if ((rc = prepare_kernel(rerank_kernel<128>))) return rc;
    return launch_pdl(rerank_kernel<128>, grid, block, smem, st, a);
  }
  if ((rc = prepare_kernel(rerank_kernel<256>))) return rc;
  return launch_pdl(rerank_kernel<256>, grid, block, smem, st, a);
}

int topk_sample_rows(const float* vals, const int32_t* idx, int64_t rows, int k, float temperature,
                     const float* u, int32_t* token, void* stream) {
  if (!vals || !idx || !u || !token) return TOPK_EINVAL;
  if (rows < 1 || k < 1) return TOPK_EINVAL;
  if (!(temperature > 0.0f) || !std::isfinite(temperature) || !std::isfinite(1.0f / temperature))
    return TOPK_EINVAL;
  if (k > kMaxK) return TOPK_EUNSUPPORTED;
  const int64_t blocks = (rows + kSampleWarps - 1) / kSampleWarps;
  if (blocks > 2147483647LL) return TOPK_EUNSUPPORTED;
  int rc;
  if ((rc = prepare_kernel(sample_rows_kernel))) return rc;
  return launch_pdl(sample_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * kSampleWarps),
                    0, static_cast<cudaStream_t>(stream), vals, idx, rows, k, 1.0f / temperature, u,
                    token);
}

int topk_sample(const float* logits, int64_t rows, int64_t n, int k, int b, int kb,
                float temperature, const float* u, int32_t* token, float* out_vals,
                int32_t* out_idx, void* workspace, size_t workspace_bytes, void* stream) {
  if (!u || !token) return TOPK_EINVAL;
  if (!(temperature > 0.0f) || !std::isfinite(temperature) || !std::isfinite(1.0f / temperature))
    return TOPK_EINVAL;
  if (k > kMaxK) return TOPK_EUNSUPPORTED;
  // The draw runs inside the selection kernel, right after each row's Stage 2.
  return run_bucketed<float>(logits, rows, n, k, b, kb, out_vals, out_idx, workspace,
                             workspace_bytes, stream, SampleTail{u, token, 1.0f / temperature});
}

int topk_sample_bf16(const uint16_t* logits, int64_t rows, int64_t n, int k, int b, int kb,
                     float temperature, const float* u, int32_t* token, uint16_t* out_vals,
                     int32_t* out_idx, void* workspace, size_t workspace_bytes, void* stream) {
  if (!u || !token) return TOPK_EINVAL;
  if (!(temperature > 0.0f) || !std::isfinite(temperature) || !std::isfinite(1.0f / temperature))
    return TOPK_EINVAL;
  if (k > kMaxK) return TOPK_EUNSUPPORTED;
  return run_bucketed<uint16_t>(logits, rows, n, k, b, kb, out_vals, out_idx, workspace,
                                workspace_bytes, stream, SampleTail{u, token, 1.0f / temperature});
}

int score_topk(const uint16_t* q, int64_t rows, int d, const uint16_t* K, int64_t n,
               int64_t k_batch_stride, int k, int b, int kb, float* out_vals, int32_t* out_idx,
               float* out_scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !K || !out_vals || !out_idx) return TOPK_EINVAL;
  int rc = check_common(rows, n, k, b, kb);
  if (rc) return rc;
  if (k_batch_stride < 0) return TOPK_EINVAL;
  if (d != 128 && d != 256) return TOPK_EUNSUPPORTED;
  if (kLanes % b) return TOPK_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(K) || (k_batch_stride % 8) != 0) return TOPK_EINVAL;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev))) return rc;
  cudaStream_t sst = static_cast<cudaStream_t>(stream);
  if (umma_eligible(rows, n, k_batch_stride, b, d)) {
    const size_t need = umma_workspace(rows, b, kb);
    if (!workspace || workspace_bytes < need) return TOPK_EWORKSPACE;
    if (!aligned16(workspace)) return TOPK_EINVAL;
    switch (kb) {
      case 1: return launch_umma_k<1>(d, q, rows, K, n, b, k, out_vals, out_idx, out_scores, workspace, dev, sst);
      case 2: return launch_umma_k<2>(d, q, rows, K, n, b, k, out_vals, out_idx, out_scores, workspace, dev, sst);
      case 3: return launch_umma_k<3>(d, q, rows, K, n, b, k, out_vals, out_idx, out_scores, workspace, dev, sst);
      default: return launch_umma_k<4>(d, q, rows, K, n, b, k, out_vals, out_idx, out_scores, workspace, dev, sst);
    }
  }
  Plan pl;
  if ((rc = plan_score(rows, n, b, kb, d, dev, &pl))) return rc;
  if (plan_needs_workspace(pl, rows, n)) {
    if (!workspace || workspace_bytes < pl.workspace()) return TOPK_EWORKSPACE;
    if (!aligned16(workspace)) return TOPK_EINVAL;
  }
  ScoreArgs a;
  a.q = q;
  a.K = K;
  a.kstride = k_batch_stride;
  a.k = k;
  a.b = b;
  a.out_vals = out_vals;
  a.out_idx = out_idx;
  a.out_scores = out_scores;
  a.rs = make_split(pl, rows, n, workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (kb) {
    case 1: return launch_score_k<1>(d, pl, a, st);
    case 2: return launch_score_k<2>(d, pl, a, st);
    case 3: return launch_score_k<3>(d, pl, a, st);
    default: return launch_score_k<4>(d, pl, a, st);
  }
}

int topk_selftest_wait_timeout(unsigned long long limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > kWaitLimitNs) return TOPK_EINVAL;
  clear_launch_error();
  wait_timeout_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? TOPK_OK : TOPK_ECUDA;
}

int topk_device_status(int* status_out) {
  if (!status_out) return TOPK_EINVAL;
  if (cudaDeviceSynchronize() != cudaSuccess) return TOPK_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return TOPK_ECUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return TOPK_ECUDA;
  *status_out = v;
  return TOPK_OK;
}

}  // extern "C"
