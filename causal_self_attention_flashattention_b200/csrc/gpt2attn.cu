// Host side of the library: argument checks, TMA tensor maps over the packed
// layouts, launch configuration and the extern "C" entry points declared in
// include/gpt2attn.h.
//
// Nothing here allocates device memory. The only process-wide state is a
// per-device cache of the SM count and of the kernels' shared-memory opt-in,
// guarded by a mutex, a cache of encoded tensor maps (its own mutex), the
// device status word the kernels write when a bounded wait gives up, and the
// code of the last failed CUDA call.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "gpt2attn.h"
#include "checks.h"

#include "common.cuh"
#include "ptx.cuh"
#include "fwd.cuh"
#include "bwd.cuh"
#include "bwd_fused.cuh"
#include "decode.cuh"
#include "selftest.cuh"
#include "linear.cuh"
#include "fp8.cuh"

namespace ga_host {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ga_status check_shape(int B, int T, int H, int D) {
  if (B < 1 || T < 1 || H < 1 || D < 1) return GA_ERR_INVALID_ARG;
  if (D != ga::kD) return GA_ERR_UNSUPPORTED;
  const long double elems = static_cast<long double>(B) * T * 3 * H * D;
  if (elems >= 2147483648.0L) return GA_ERR_INVALID_ARG;
  return GA_OK;
}

ga_status check_scale(float scale) {
  if (!std::isfinite(scale) || !(scale > 0.f)) return GA_ERR_INVALID_ARG;
  return GA_OK;
}

}  // namespace ga_host

namespace {

using ga::kD;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int pair_clusters = 0;  // CTA pairs of the pair GEMM resident at once
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_get_current = nullptr;

// The last CUDA failure behind a GA_ERR_CUDA: the failing step in the high 32
// bits (kCudaErr*), its cudaError_t or CUresult in the low 32 bits.
std::atomic<unsigned long long> g_cuda_error{0};
constexpr unsigned long long kCudaErrSetup = 1, kCudaErrTensorMap = 2, kCudaErrLaunch = 3;

void record_cuda_error(unsigned long long step, unsigned int code) {
  g_cuda_error.store((step << 32) | code, std::memory_order_relaxed);
}

// Opts one forward kernel into its dynamic shared memory and checks that it
// was compiled for the register count its setmaxnreg split assumes.
template <class Kernel>
bool setup_fwd_kernel(Kernel kernel, bool fp8) {
  const int smem = static_cast<int>(fp8 ? ga::fwd::kSmemBytes<true> : ga::fwd::kSmemBytes<false>);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return false;
  cudaFuncAttributes fa;
  return cudaFuncGetAttributes(&fa, kernel) == cudaSuccess &&
         fa.numRegs >= static_cast<int>(ga::fwd::kLaunchRegs);
}

// With g_mutex held: fills g_devices[dev] on its first use (SM count, the
// dynamic shared-memory opt-in of every kernel). Returns nullptr on failure.
const DeviceInfo* setup_device(int dev) {
  DeviceInfo& info = g_devices[dev];
  if (info.ready) return &info;
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return nullptr;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (g_ctx_get_current == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return nullptr;
    g_ctx_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  if (cudaDeviceGetAttribute(&info.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return nullptr;
  // The forward kernels (bf16, FP8, fp16-v; small and large item tables).
  // Their setmaxnreg split (warpgroup budgets that add up to the block's
  // allocation) is only safe if they launch with the register count the split
  // was sized for.
  if (!setup_fwd_kernel(ga::fwd::attn_fwd_kernel<false, false, ga::fwd::kSchedSmall>, false) ||
      !setup_fwd_kernel(ga::fwd::attn_fwd_kernel<false, false, ga::fwd::kSchedMaxItems>, false) ||
      !setup_fwd_kernel(ga::fwd::attn_fwd_kernel<true, false, ga::fwd::kSchedSmall>, true) ||
      !setup_fwd_kernel(ga::fwd::attn_fwd_kernel<true, false, ga::fwd::kSchedMaxItems>, true) ||
      !setup_fwd_kernel(ga::fwd::attn_fwd_kernel<false, true, ga::fwd::kSchedSmall>, false) ||
      !setup_fwd_kernel(ga::fwd::attn_fwd_kernel<false, true, ga::fwd::kSchedMaxItems>, false))
    return nullptr;

  if (cudaFuncSetAttribute(ga::bwd::dkdv::attn_bwd_dkdv_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(ga::bwd::dkdv::kSmemBytes)) != cudaSuccess ||
      cudaFuncSetAttribute(ga::bwd::dq::attn_bwd_dq_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(ga::bwd::dq::kSmemBytes)) != cudaSuccess)
    return nullptr;
  if (cudaFuncSetAttribute(ga::bwd::fused::attn_bwd_fused_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(ga::bwd::fused::kSmemBytes)) != cudaSuccess)
    return nullptr;
  if (cudaFuncSetAttribute(ga::linear::linear_pair_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(ga::linear::kPairSmemBytes)) != cudaSuccess)
    return nullptr;
  {
    // How many two-CTA clusters fit at once (a pair must share a GPC, so an
    // odd SM count in a GPC leaves one SM out).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (info.num_sms / 2));
    cfg.blockDim = dim3(ga::linear::kThreads);
    cfg.dynamicSmemBytes = ga::linear::kPairSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, ga::linear::linear_pair_kernel, &cfg) != cudaSuccess ||
        n < 1)
      return nullptr;
    info.pair_clusters = n;
  }
  info.ready = true;
  return &info;
}

// The current device's set-up, done once. Returns nullptr on failure (the
// failing CUDA call's code is recorded; 0 if a non-CUDA check failed).
const DeviceInfo* device_info() {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    record_cuda_error(kCudaErrSetup, static_cast<unsigned int>(e));
    return nullptr;
  }
  const DeviceInfo* ready = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    ready = setup_device(dev);
  }
  if (ready == nullptr) {
    const cudaError_t le = cudaGetLastError();
    record_cuda_error(kCudaErrSetup, static_cast<unsigned int>(le));
    return nullptr;
  }
  // Tensor-map encoding is a driver call and needs a current context. A host
  // thread whose CUDA runtime calls so far needed none (a framework's worker
  // thread, say) has none bound yet: bind the device's primary context, as
  // the runtime itself would at its first launch. A context the caller made
  // current is left alone.
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
    const cudaError_t se = cudaSetDevice(dev);
    if (se != cudaSuccess) {
      record_cuda_error(kCudaErrSetup, static_cast<unsigned int>(se));
      return nullptr;
    }
  }
  return ready;
}

// Tensor maps are cached: a map is a pure function of its description (base
// address, data type, extents, box, swizzle), so a call that describes the
// same tensor as an earlier one reuses the earlier encoding instead of asking
// the driver again. The cache is a fixed table replaced round-robin under its
// own mutex; it allocates nothing.
struct MapKey {
  const void* base;
  uint64_t dims[3];
  uint32_t box[3];
  int rank, dtype, swizzle;
  bool operator==(const MapKey& o) const {
    return base == o.base && dims[0] == o.dims[0] && dims[1] == o.dims[1] &&
           dims[2] == o.dims[2] && box[0] == o.box[0] && box[1] == o.box[1] &&
           box[2] == o.box[2] && rank == o.rank && dtype == o.dtype && swizzle == o.swizzle;
  }
};

constexpr int kMapCacheSize = 64;
struct MapCacheEntry {
  bool used = false;
  MapKey key;
  CUtensorMap map;
};
std::mutex g_map_mutex;
MapCacheEntry g_map_cache[kMapCacheSize];
int g_map_next = 0;

// Row-major tensor of `rank` <= 3 dims (innermost first) with `elem` bytes per
// element and no padding between rows; box {box[0..rank)}; zero fill past
// the edges. Returns false (recording the driver's code) if encoding fails.
bool encode_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint32_t elem,
                int rank, const uint64_t (&dims)[3], const uint32_t (&box)[3],
                CUtensorMapSwizzle swizzle) {
  MapKey key;
  key.base = base;
  key.rank = rank;
  key.dtype = static_cast<int>(dtype);
  key.swizzle = static_cast<int>(swizzle);
  for (int d = 0; d < 3; ++d) {
    key.dims[d] = d < rank ? dims[d] : 0;
    key.box[d] = d < rank ? box[d] : 0;
  }
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (const MapCacheEntry& e : g_map_cache)
      if (e.used && e.key == key) {
        *map = e.map;
        return true;
      }
  }
  cuuint64_t gdims[3], strides[2];
  cuuint32_t gbox[3], elem_strides[3] = {1, 1, 1};
  uint64_t stride = elem;
  for (int d = 0; d < rank; ++d) {
    gdims[d] = dims[d];
    gbox[d] = box[d];
    if (d > 0) strides[d - 1] = stride;
    stride *= dims[d];
  }
  const CUresult r = g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                              gdims, strides, gbox, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    record_cuda_error(kCudaErrTensorMap, static_cast<unsigned int>(r));
    return false;
  }
  std::lock_guard<std::mutex> lock(g_map_mutex);
  MapCacheEntry& e = g_map_cache[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCacheSize;
  e.used = true;
  e.key = key;
  e.map = *map;
  return true;
}

// 3-D bf16 tensor map {inner, T, B} with a {64, 128, 1} box, 128-byte swizzle
// and zero fill outside the tensor (rows past T read as 0).
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, int T, int B) {
  const uint64_t dims[3] = {inner, static_cast<uint64_t>(T), static_cast<uint64_t>(B)};
  const uint32_t box[3] = {static_cast<uint32_t>(kD), static_cast<uint32_t>(ga::kBlockM), 1};
  return encode_map(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3, dims, box,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// 3-D byte tensor map {inner, T, B} (e4m3 data) with a {64, 128, 1} box (64
// bytes by 128 rows), the given swizzle and zero fill past the edges.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t inner, int T, int B,
                 CUtensorMapSwizzle swizzle) {
  const uint64_t dims[3] = {inner, static_cast<uint64_t>(T), static_cast<uint64_t>(B)};
  const uint32_t box[3] = {64, static_cast<uint32_t>(ga::kBlockM), 1};
  return encode_map(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 3, dims, box, swizzle);
}

// 2-D bf16 tensor map {inner, rows} (row-major, `inner` contiguous) with a
// {64, box_rows} box, 128-byte swizzle and zero fill past the edges.
bool make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                 uint32_t box_rows) {
  const uint64_t dims[3] = {inner, rows, 0};
  const uint32_t box[3] = {64, box_rows, 0};
  return encode_map(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2, dims, box,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// After a launch: GA_OK, or GA_ERR_CUDA with the launch error recorded.
ga_status check_launch() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return GA_OK;
  record_cuda_error(kCudaErrLaunch, static_cast<unsigned int>(e));
  return GA_ERR_CUDA;
}

using ga_host::aligned16;
using ga_host::check_scale;
using ga_host::check_shape;

ga::AttnShape make_shape(int B, int T, int H, float scale) {
  ga::AttnShape sh;
  sh.B = B;
  sh.T = T;
  sh.H = H;
  sh.scale = scale;
  sh.scale_log2 = scale * 1.4426950408889634f;
  return sh;
}

int grid_for(int items, int num_sms) { return items < num_sms ? items : num_sms; }

// Item deals (ga::ItemSchedule), longest processing time first. Items come
// heaviest first (their numbering in the kernel); each goes to the CTA with
// the least work so far, the lowest index on ties. An item's work is counted
// in half-tile steps: 2n for its n tiles plus a constant that stands for what
// an item costs beyond its tiles (the forward's first S product, the previous
// item's output and the swap of its warpgroups' tiles), chosen by A/B at
// B=16 T=1024 H=12 among 0, 1.26 and 2.5 tile steps (2.5 was fastest).
constexpr long kFwdItemCost2 = 5;

// Deals items [k0, k1) to `grid` CTAs into *s; cost(k) is item k's work.
// False if a CTA would get more than kSchedSlots items (the caller then deals
// fewer items per launch).
template <int kItems, class Cost>
bool build_schedule(ga::ItemSchedule<kItems>* s, long k0, long k1, int grid, Cost cost) {
  const long n = k1 - k0;
  if (grid <= 0 || grid > ga::kSchedMaxCtas || n <= 0 || n > kItems) return false;
  using Load = std::pair<long, int>;  // (work so far, CTA)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < grid; ++c) heap.push(Load(0, c));
  std::vector<int> owner(n), count(grid, 0);
  for (long k = k0; k < k1; ++k) {
    const Load least = heap.top();
    heap.pop();
    owner[k - k0] = least.second;
    if (++count[least.second] > ga::kSchedSlots) return false;
    heap.push(Load(least.first + cost(k), least.second));
  }
  int off = 0;
  for (int c = 0; c < grid; ++c) {
    s->start[c] = static_cast<uint16_t>(off);
    off += count[c];
    count[c] = s->start[c];  // next free place in CTA c's list
  }
  s->start[grid] = static_cast<uint16_t>(off);
  for (long t = 0; t < n; ++t) s->item[count[owner[t]]++] = static_cast<uint16_t>(t);
  s->base = static_cast<int>(k0);
  return true;
}

// One-launch deals, cached per (query tiles, heads, SMs) in a fixed table
// replaced round-robin under its own mutex.
template <int kItems>
struct SchedCache {
  struct Entry {
    bool used = false;
    int n_qt = 0, bh = 0, num_sms = 0;
    ga::ItemSchedule<kItems> sched;
    int grid = 0;
    int n = 0;  // items in the launch
  };
  static constexpr int kSize = 8;
  std::mutex mutex;
  Entry entries[kSize];
  int next = 0;
};
SchedCache<ga::fwd::kSchedMaxItems> g_fwd_sched;

// Calls launch(schedule, grid, items) once per launch of a kernel over
// `items` items of n_qt query tiles and bh heads on num_sms SMs, in item
// order: one launch unless the items do not fit one table. Returns false if a
// launch failed (launch() returned false).
template <int kItems, class Cost, class Launch>
bool for_each_launch(SchedCache<kItems>& cache, int n_qt, int bh, long items, int num_sms,
                     Cost cost, Launch launch) {
  ga::ItemSchedule<kItems> sched;
  int cached_grid = 0, cached_n = 0;
  {
    std::lock_guard<std::mutex> lock(cache.mutex);
    for (const auto& e : cache.entries)
      if (e.used && e.n_qt == n_qt && e.bh == bh && e.num_sms == num_sms) {
        cached_grid = e.grid;
        cached_n = e.n;
        sched.base = e.sched.base;
        std::copy(e.sched.start, e.sched.start + cached_grid + 1, sched.start);
        std::copy(e.sched.item, e.sched.item + cached_n, sched.item);
        break;
      }
  }
  if (cached_grid > 0) return launch(sched, cached_grid, cached_n);
  long chunk = kItems;
  for (long k0 = 0; k0 < items;) {
    const long k1 = std::min(items, k0 + chunk);
    const int grid = static_cast<int>(
        std::min<long>(k1 - k0, std::min(num_sms, ga::kSchedMaxCtas)));
    if (!build_schedule(&sched, k0, k1, grid, cost)) {
      chunk /= 2;  // fits at the latest once chunk <= kSchedSlots
      continue;
    }
    if (k0 == 0 && k1 == items) {
      std::lock_guard<std::mutex> lock(cache.mutex);
      auto& e = cache.entries[cache.next];
      cache.next = (cache.next + 1) % SchedCache<kItems>::kSize;
      e.sched = sched;
      e.grid = grid;
      e.n = static_cast<int>(k1 - k0);
      e.n_qt = n_qt;
      e.bh = bh;
      e.num_sms = num_sms;
      e.used = true;
    }
    if (!launch(sched, grid, static_cast<int>(k1 - k0))) return false;
    k0 = k1;
  }
  return true;
}

// The forward: item k is a pair of query tiles with n_kv(k) key tiles.
template <class Launch>
bool for_each_fwd_launch(int B, int T, int H, int num_sms, Launch launch) {
  const int n_qt = ga::ceil_div(T, ga::kBlockM), bh = B * H, n_pairs = (n_qt + 1) / 2;
  auto cost = [=](long k) {
    const int p = n_pairs - 1 - static_cast<int>(k / bh);
    const int n_kv = (2 * p + 1) < n_qt ? 2 * p + 2 : 2 * p + 1;
    return 2L * n_kv + kFwdItemCost2;
  };
  return for_each_launch(g_fwd_sched, n_qt, bh, static_cast<long>(bh) * n_pairs, num_sms, cost,
                         launch);
}

// Calls fn(table) with the deal of `sched` (n items on grid CTAs) in the
// smaller table type that holds it: every launch copies its whole parameter.
template <int kSmall, int kLarge, class Fn>
void with_table(const ga::ItemSchedule<kLarge>& sched, int grid, int n, Fn fn) {
  if (n <= kSmall) {
    ga::ItemSchedule<kSmall> small;
    small.base = sched.base;
    std::copy(sched.start, sched.start + grid + 1, small.start);
    std::copy(sched.item, sched.item + n, small.item);
    fn(small);
  } else {
    fn(sched);
  }
}

template <class Table>
constexpr int table_items() {
  return static_cast<int>(sizeof(Table::item) / sizeof(Table::item[0]));
}

// Writes the deal of each launch into launch/cta/pos (indexed by item).
struct DealWriter {
  int* launch;
  int* cta;
  int* pos;
  int n_launch = 0;
  template <class Sched>
  bool operator()(const Sched& sched, int grid, int) {
    for (int c = 0; c < grid; ++c)
      for (int t = sched.start[c]; t < sched.start[c + 1]; ++t) {
        const long k = sched.base + static_cast<long>(sched.item[t]);
        launch[k] = n_launch;
        cta[k] = c;
        pos[k] = t - sched.start[c];
      }
    ++n_launch;
    return true;
  }
};

bool deal_args_ok(int B, int T, int H, int num_sms, const int* launch, const int* cta,
                  const int* pos) {
  return launch != nullptr && cta != nullptr && pos != nullptr && B > 0 && T > 0 && H > 0 &&
         num_sms > 0;
}


// Launches attn_fwd_kernel<kFp8, kV16> over the n items of `sched` on `grid`
// CTAs.
template <bool kFp8, bool kV16, class... Args>
void launch_fwd_kernel(const ga::ItemSchedule<ga::fwd::kSchedMaxItems>& sched, int grid, int n,
                       cudaStream_t stream, Args... args) {
  const size_t smem = kFp8 ? ga::fwd::kSmemBytes<true> : ga::fwd::kSmemBytes<false>;
  with_table<ga::fwd::kSchedSmall>(sched, grid, n, [&](const auto& table) {
    constexpr int kN = table_items<std::decay_t<decltype(table)>>();
    ga::fwd::attn_fwd_kernel<kFp8, kV16, kN><<<grid, ga::fwd::kThreads, smem, stream>>>(args...,
                                                                                        table);
  });
}

size_t delta_bytes(int B, int T, int H) {
  const size_t n = static_cast<size_t>(B) * H * T * sizeof(float);
  return (n + 255) & ~static_cast<size_t>(255);
}

}  // namespace

extern "C" {

namespace {

// The bf16 forward, with v read as bf16 (converted in the kernel) or, for
// v16, as fp16 already.
ga_status launch_fwd(const void* qkv, void* out, float* lse, int B, int T, int H, int D,
                     float scale, gpt2attn_stream_t stream, bool v16) {
  if (qkv == nullptr || out == nullptr || lse == nullptr) return GA_ERR_INVALID_ARG;
  ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if ((st = check_scale(scale)) != GA_OK) return st;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(lse)) return GA_ERR_ALIGNMENT;
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;

  // One 16-bit map serves q, k and v: a TMA copy moves bytes, whatever the
  // 16-bit type.
  CUtensorMap map_qkv;
  if (!make_map(&map_qkv, qkv, static_cast<uint64_t>(3) * H * kD, T, B)) return GA_ERR_CUDA;
  const ga::AttnShape sh = make_shape(B, T, H, scale);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ga_status ls = GA_OK;
  for_each_fwd_launch(B, T, H, info->num_sms, [&](const auto& sched, int grid, int n) {
    if (v16)
      launch_fwd_kernel<false, true>(sched, grid, n, s, map_qkv, map_qkv,
                                     static_cast<__nv_bfloat16*>(out), lse, sh,
                                     static_cast<const float*>(nullptr));
    else
      launch_fwd_kernel<false, false>(sched, grid, n, s, map_qkv, map_qkv,
                                      static_cast<__nv_bfloat16*>(out), lse, sh,
                                      static_cast<const float*>(nullptr));
    return (ls = check_launch()) == GA_OK;
  });
  return ls;
}

}  // namespace

ga_status gpt2_attn_fwd(const void* qkv, void* out, float* lse, int B, int T, int H, int D,
                        float scale, gpt2attn_stream_t stream) {
  return launch_fwd(qkv, out, lse, B, T, H, D, scale, stream, false);
}

ga_status gpt2_attn_fwd_v16(const void* qkv, void* out, float* lse, int B, int T, int H, int D,
                            float scale, gpt2attn_stream_t stream) {
  return launch_fwd(qkv, out, lse, B, T, H, D, scale, stream, true);
}

ga_status gpt2_attn_fp8_quantize(const void* qkv, void* qkv8, float* scales, int B, int T, int H,
                                 int D, gpt2attn_stream_t stream) {
  if (qkv == nullptr || qkv8 == nullptr || scales == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if (!aligned16(qkv) || !aligned16(qkv8) || !aligned16(scales)) return GA_ERR_ALIGNMENT;
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;
  const int C = H * kD;
  const long long n_chunks = static_cast<long long>(B) * T * 3 * C / 8;
  const long long want = (n_chunks + ga::fp8::kThreads - 1) / ga::fp8::kThreads;
  const long long cap = 8LL * info->num_sms;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ga::fp8::fp8_zero_kernel<<<1, 32, 0, s>>>(scales);
  ga::fp8::fp8_amax_kernel<<<blocks, ga::fp8::kThreads, 0, s>>>(
      static_cast<const uint4*>(qkv), n_chunks, C, scales);
  ga::fp8::fp8_quantize_kernel<<<blocks, ga::fp8::kThreads, 0, s>>>(
      static_cast<const uint4*>(qkv), static_cast<uint2*>(qkv8), n_chunks, C, scales);
  return check_launch();
}

ga_status gpt2_attn_fwd_fp8(const void* qkv8, const float* scales, void* out, float* lse, int B,
                            int T, int H, int D, float scale, gpt2attn_stream_t stream) {
  if (qkv8 == nullptr || scales == nullptr || out == nullptr || lse == nullptr)
    return GA_ERR_INVALID_ARG;
  ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if ((st = check_scale(scale)) != GA_OK) return st;
  if (!aligned16(qkv8) || !aligned16(scales) || !aligned16(out) || !aligned16(lse))
    return GA_ERR_ALIGNMENT;
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;
  CUtensorMap map_qk, map_v;
  const uint64_t inner = static_cast<uint64_t>(3) * H * kD;
  if (!make_map_u8(&map_qk, qkv8, inner, T, B, CU_TENSOR_MAP_SWIZZLE_64B)) return GA_ERR_CUDA;
  if (!make_map_u8(&map_v, qkv8, inner, T, B, CU_TENSOR_MAP_SWIZZLE_NONE)) return GA_ERR_CUDA;
  const ga::AttnShape sh = make_shape(B, T, H, scale);
  ga_status ls = GA_OK;
  for_each_fwd_launch(B, T, H, info->num_sms, [&](const auto& sched, int grid, int n) {
    launch_fwd_kernel<true, false>(sched, grid, n, reinterpret_cast<cudaStream_t>(stream), map_qk,
                                   map_v, static_cast<__nv_bfloat16*>(out), lse, sh,
                                   scales + ga::fp8::kDequantOffset);
    return (ls = check_launch()) == GA_OK;
  });
  return ls;
}

ga_status gpt2_attn_bwd_workspace_size(int B, int T, int H, int D, size_t* bytes) {
  if (bytes == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  *bytes = delta_bytes(B, T, H);
  return GA_OK;
}

ga_status gpt2_attn_bwd_fused_workspace_size(int B, int T, int H, int D, size_t* bytes) {
  if (bytes == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  *bytes = ga::bwd::fused::ws_bytes(B, T, H);
  return GA_OK;
}

namespace {

ga_status launch_pre(const void* out, const void* dout, float* delta, uint32_t* counters,
                     int n_counters, int B, int T, int H, gpt2attn_stream_t stream) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;
  const ga::AttnShape sh = make_shape(B, T, H, 1.f);
  const long long rows = static_cast<long long>(B) * T * H;
  const long long blocks_needed = (rows * 8 + 255) / 256;
  const long long cap = 16LL * info->num_sms;
  const int blocks = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  ga::bwd::attn_bwd_pre_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), delta,
      counters, n_counters, sh);
  return check_launch();
}

}  // namespace

ga_status gpt2_attn_bwd_preprocess(const void* out, const void* dout, float* delta, int B,
                                   int T, int H, int D, gpt2attn_stream_t stream) {
  if (out == nullptr || dout == nullptr || delta == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(delta)) return GA_ERR_ALIGNMENT;
  return launch_pre(out, dout, delta, nullptr, 0, B, T, H, stream);
}

ga_status gpt2_attn_bwd_prepare(const void* out, const void* dout, void* workspace,
                                size_t workspace_bytes, int B, int T, int H, int D,
                                gpt2attn_stream_t stream) {
  if (out == nullptr || dout == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if (workspace == nullptr || workspace_bytes < ga::bwd::fused::ws_bytes(B, T, H))
    return GA_ERR_WORKSPACE;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(workspace)) return GA_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return launch_pre(out, dout, reinterpret_cast<float*>(ws),
                    reinterpret_cast<uint32_t*>(ws + ga::bwd::fused::ws_cnt_offset(B, T, H)),
                    B * H * ga::ceil_div(T, ga::kBlockM), B, T, H, stream);
}

namespace {

// Shared checks and tensor maps of the two tensor-core backward steps.
struct BwdLaunch {
  CUtensorMap map_qkv, map_do;
  ga::AttnShape sh;
  int grid;
};

ga_status prepare_bwd(const void* qkv, const void* dout, const float* lse, const float* delta,
                      void* dqkv, int B, int T, int H, int D, float scale, BwdLaunch* L) {
  if (qkv == nullptr || dout == nullptr || lse == nullptr || delta == nullptr || dqkv == nullptr)
    return GA_ERR_INVALID_ARG;
  ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if ((st = check_scale(scale)) != GA_OK) return st;
  if (!aligned16(qkv) || !aligned16(dout) || !aligned16(lse) || !aligned16(delta) ||
      !aligned16(dqkv))
    return GA_ERR_ALIGNMENT;
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;
  if (!make_map(&L->map_qkv, qkv, static_cast<uint64_t>(3) * H * kD, T, B)) return GA_ERR_CUDA;
  if (!make_map(&L->map_do, dout, static_cast<uint64_t>(H) * kD, T, B)) return GA_ERR_CUDA;
  L->sh = make_shape(B, T, H, scale);
  L->grid = grid_for(B * H * ga::ceil_div(T, ga::kBlockM), info->num_sms);
  return GA_OK;
}

}  // namespace

ga_status gpt2_attn_bwd_dkdv(const void* qkv, const void* dout, const float* lse,
                             const float* delta, void* dqkv, int B, int T, int H, int D,
                             float scale, gpt2attn_stream_t stream) {
  BwdLaunch L;
  const ga_status st = prepare_bwd(qkv, dout, lse, delta, dqkv, B, T, H, D, scale, &L);
  if (st != GA_OK) return st;
  CUtensorMap map_dqkv;
  if (!make_map(&map_dqkv, dqkv, static_cast<uint64_t>(3) * H * kD, T, B)) return GA_ERR_CUDA;
  ga::bwd::dkdv::attn_bwd_dkdv_kernel<<<L.grid, ga::bwd::kThreads, ga::bwd::dkdv::kSmemBytes,
                                        reinterpret_cast<cudaStream_t>(stream)>>>(
      L.map_qkv, L.map_do, map_dqkv, lse, delta, L.sh);
  return check_launch();
}

ga_status gpt2_attn_bwd_dq(const void* qkv, const void* out, const void* dout,
                           const float* lse, float* delta, void* dqkv, int B, int T, int H,
                           int D, float scale, gpt2attn_stream_t stream) {
  if (out == nullptr) return GA_ERR_INVALID_ARG;
  if (!aligned16(out)) return GA_ERR_ALIGNMENT;
  BwdLaunch L;
  const ga_status st = prepare_bwd(qkv, dout, lse, delta, dqkv, B, T, H, D, scale, &L);
  if (st != GA_OK) return st;
  CUtensorMap map_o;
  if (!make_map(&map_o, out, static_cast<uint64_t>(H) * kD, T, B)) return GA_ERR_CUDA;
  ga::bwd::dq::attn_bwd_dq_kernel<<<L.grid, ga::bwd::kThreads, ga::bwd::dq::kSmemBytes,
                                    reinterpret_cast<cudaStream_t>(stream)>>>(
      L.map_qkv, L.map_do, map_o, lse, delta, static_cast<__nv_bfloat16*>(dqkv), L.sh);
  return check_launch();
}

ga_status gpt2_attn_bwd_fused(const void* qkv, const void* dout, const float* lse,
                              void* workspace, size_t workspace_bytes, void* dqkv, int B, int T,
                              int H, int D, float scale, gpt2attn_stream_t stream) {
  if (workspace == nullptr) return GA_ERR_WORKSPACE;
  BwdLaunch L;
  const ga_status st = prepare_bwd(qkv, dout, lse, static_cast<const float*>(workspace), dqkv, B,
                                   T, H, D, scale, &L);
  if (st != GA_OK) return st;
  if (workspace_bytes < ga::bwd::fused::ws_bytes(B, T, H)) return GA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  ga::bwd::fused::attn_bwd_fused_kernel<<<L.grid, ga::bwd::fused::kFusedThreads,
                                          ga::bwd::fused::kSmemBytes,
                                          reinterpret_cast<cudaStream_t>(stream)>>>(
      L.map_qkv, L.map_do, lse, reinterpret_cast<const float*>(ws),
      reinterpret_cast<float*>(ws + ga::bwd::fused::ws_dq_offset(B, T, H)),
      reinterpret_cast<uint32_t*>(ws + ga::bwd::fused::ws_cnt_offset(B, T, H)),
      static_cast<__nv_bfloat16*>(dqkv), L.sh);
  return check_launch();
}

ga_status gpt2_attn_bwd(const void* qkv, const void* out, const void* dout, const float* lse,
                        void* dqkv, void* workspace, size_t workspace_bytes, int B, int T, int H,
                        int D, float scale, gpt2attn_stream_t stream) {
  if (qkv == nullptr || out == nullptr || dout == nullptr || lse == nullptr || dqkv == nullptr)
    return GA_ERR_INVALID_ARG;
  ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if ((st = check_scale(scale)) != GA_OK) return st;
  if (workspace == nullptr || workspace_bytes < delta_bytes(B, T, H)) return GA_ERR_WORKSPACE;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dqkv) || !aligned16(workspace))
    return GA_ERR_ALIGNMENT;
  float* delta = static_cast<float*>(workspace);
  if ((st = gpt2_attn_bwd_dq(qkv, out, dout, lse, delta, dqkv, B, T, H, D, scale, stream)) !=
      GA_OK)
    return st;
  return gpt2_attn_bwd_dkdv(qkv, dout, lse, delta, dqkv, B, T, H, D, scale, stream);
}

ga_status gpt2_attn_decode_workspace_size(int B, int T, int H, int D, size_t* bytes) {
  if (bytes == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  *bytes = ga::decode::ws_bytes(B, T, H);
  return GA_OK;
}

ga_status gpt2_attn_decode(const void* qkv, int t, void* out, float* lse, void* workspace,
                           size_t workspace_bytes, int B, int T, int H, int D, float scale,
                           gpt2attn_stream_t stream) {
  if (qkv == nullptr || out == nullptr || lse == nullptr) return GA_ERR_INVALID_ARG;
  ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if ((st = check_scale(scale)) != GA_OK) return st;
  if (t < 0 || t >= T || B > 65535 || H > 65535) return GA_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < ga::decode::ws_bytes(B, T, H))
    return GA_ERR_WORKSPACE;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(lse) || !aligned16(workspace))
    return GA_ERR_ALIGNMENT;
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;
  const ga::AttnShape sh = make_shape(B, T, H, scale);
  const int n_chunks = ga::decode::num_chunks(t);
  float* partials = static_cast<float*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap map_qkv;
  if (!make_map(&map_qkv, qkv, static_cast<uint64_t>(3) * H * kD, T, B)) return GA_ERR_CUDA;
  ga::decode::attn_decode_partial_kernel<<<dim3(n_chunks, H, B), ga::decode::kWarps * 32,
                                           ga::decode::kSmemBytes, s>>>(
      map_qkv, static_cast<const __nv_bfloat16*>(qkv), t, partials, sh);
  // The combine is a programmatic dependent of the partial kernel: its
  // launch overlaps the partials' tail, and it waits for them on the device.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(H, B);
  cfg.blockDim = dim3(ga::kD);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // A refused launch leaves its error for check_launch to record.
  (void)cudaLaunchKernelEx(&cfg, ga::decode::attn_decode_combine_kernel,
                           static_cast<const float*>(partials), n_chunks,
                           static_cast<__nv_bfloat16*>(out), lse, sh);
  return check_launch();
}

namespace {

// y (M, N) = a (M, K) w (N, K)^T + bias (N): the shared body of the two dense
// layers. K and N are multiples of 64 here (C = H * 64).
ga_status launch_linear(const void* a, const void* w, const void* bias, void* y, long long M,
                        int N, int K, int f16_from, gpt2attn_stream_t stream) {
  if (static_cast<long double>(M) * (N > K ? N : K) >= 2147483648.0L) return GA_ERR_INVALID_ARG;
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GA_ERR_CUDA;
  CUtensorMap map_a, map_w;
  if (!make_map_2d(&map_a, a, static_cast<uint64_t>(K), static_cast<uint64_t>(M), 128))
    return GA_ERR_CUDA;
  if (!make_map_2d(&map_w, w, static_cast<uint64_t>(K), static_cast<uint64_t>(N), 128))
    return GA_ERR_CUDA;
  CUtensorMap map_y;  // 16-bit y (bf16 or fp16 columns): the store only moves bits
  if (!make_map_2d(&map_y, y, static_cast<uint64_t>(N), static_cast<uint64_t>(M), 32))
    return GA_ERR_CUDA;
  ga::linear::GemmShape g;
  g.M = static_cast<int>(M);
  g.N = N;
  g.K = K;
  g.f16_from = f16_from;
  // CTA pairs, each on 256 x 256 tiles of y.
  const int tiles = ga::linear::num_pair_tiles(g);
  const int clusters = tiles < info->pair_clusters ? tiles : info->pair_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(ga::linear::kThreads);
  cfg.dynamicSmemBytes = ga::linear::kPairSmemBytes;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // A refused launch leaves its error for check_launch to record.
  (void)cudaLaunchKernelEx(&cfg, ga::linear::linear_pair_kernel, map_a, map_w, map_y,
                           static_cast<const uint16_t*>(bias), g);
  return check_launch();
}

ga_status check_linear_args(const void* a, const void* w, const void* bias, const void* y, int B,
                            int T, int H, int D) {
  if (a == nullptr || w == nullptr || bias == nullptr || y == nullptr) return GA_ERR_INVALID_ARG;
  const ga_status st = check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if (!aligned16(a) || !aligned16(w) || !aligned16(bias) || !aligned16(y)) return GA_ERR_ALIGNMENT;
  return GA_OK;
}

}  // namespace

ga_status gpt2_attn_qkv_proj(const void* x, const void* w_attn, const void* b_attn, void* qkv,
                             int B, int T, int H, int D, gpt2attn_stream_t stream) {
  const ga_status st = check_linear_args(x, w_attn, b_attn, qkv, B, T, H, D);
  if (st != GA_OK) return st;
  const int C = H * D;
  return launch_linear(x, w_attn, b_attn, qkv, static_cast<long long>(B) * T, 3 * C, C, 3 * C,
                       stream);
}

ga_status gpt2_attn_qkv_proj_v16(const void* x, const void* w_attn, const void* b_attn,
                                 void* qkv, int B, int T, int H, int D,
                                 gpt2attn_stream_t stream) {
  const ga_status st = check_linear_args(x, w_attn, b_attn, qkv, B, T, H, D);
  if (st != GA_OK) return st;
  const int C = H * D;
  // Columns [2C, 3C) are the v slot.
  return launch_linear(x, w_attn, b_attn, qkv, static_cast<long long>(B) * T, 3 * C, C, 2 * C,
                       stream);
}

ga_status gpt2_attn_out_proj(const void* out, const void* w_proj, const void* b_proj, void* y,
                             int B, int T, int H, int D, gpt2attn_stream_t stream) {
  const ga_status st = check_linear_args(out, w_proj, b_proj, y, B, T, H, D);
  if (st != GA_OK) return st;
  const int C = H * D;
  return launch_linear(out, w_proj, b_proj, y, static_cast<long long>(B) * T, C, C, C, stream);
}

ga_status gpt2_attn_selftest_wait_timeout(unsigned long long limit_ns, gpt2attn_stream_t stream) {
  if (limit_ns == 0 || limit_ns > ga::kMaxSelftestLimitNs) return GA_ERR_INVALID_ARG;
  if (device_info() == nullptr) return GA_ERR_CUDA;
  ga::selftest::wait_timeout_kernel<<<1, ga::selftest::kThreads, 0,
                                      reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  return check_launch();
}

ga_status gpt2_attn_last_device_status(gpt2attn_stream_t stream, unsigned long long* detail) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GA_ERR_CUDA;
  unsigned long long word = 0;
  if (cudaMemcpyFromSymbol(&word, ga::g_device_status, sizeof(word)) != cudaSuccess)
    return GA_ERR_CUDA;
  if (word != 0) {
    const unsigned long long zero = 0;
    if (cudaMemcpyToSymbol(ga::g_device_status, &zero, sizeof(zero)) != cudaSuccess)
      return GA_ERR_CUDA;
  }
  if (detail != nullptr) *detail = word;
  if (word == 0) return GA_OK;
  return (word >> 32) == ga::kFwdValueRange ? GA_ERR_RANGE : GA_ERR_TIMEOUT;
}

unsigned long long gpt2_attn_last_cuda_error(void) {
  return g_cuda_error.exchange(0, std::memory_order_relaxed);
}

const char* gpt2_attn_status_string(ga_status s) {
  switch (s) {
    case GA_OK: return "GA_OK";
    case GA_ERR_INVALID_ARG: return "GA_ERR_INVALID_ARG: null pointer, bad size or bad scale";
    case GA_ERR_UNSUPPORTED: return "GA_ERR_UNSUPPORTED: only head dimension D = 64 is implemented";
    case GA_ERR_ALIGNMENT: return "GA_ERR_ALIGNMENT: every pointer must be 16-byte aligned";
    case GA_ERR_WORKSPACE: return "GA_ERR_WORKSPACE: workspace missing or too small";
    case GA_ERR_CUDA: return "GA_ERR_CUDA: a CUDA call failed";
    case GA_ERR_TIMEOUT: return "GA_ERR_TIMEOUT: a device-side wait gave up";
    case GA_ERR_RANGE: return "GA_ERR_RANGE: a v entry outside the fp16 range (|v| > 65504)";
  }
  return "unknown ga_status";
}

int gpt2_attn_version(void) { return 100; }

int gpt2_attn_fwd_item_schedule(int B, int T, int H, int num_sms, int* launch, int* cta,
                                int* pos, long n) {
  if (!deal_args_ok(B, T, H, num_sms, launch, cta, pos)) return -GA_ERR_INVALID_ARG;
  const int n_qt = ga::ceil_div(T, ga::kBlockM);
  const long items = static_cast<long>(B) * H * ((n_qt + 1) / 2);
  if (n < items || items > INT32_MAX) return -GA_ERR_INVALID_ARG;
  DealWriter w{launch, cta, pos};
  for_each_fwd_launch(B, T, H, num_sms, [&](const auto& s, int g, int m) { return w(s, g, m); });
  return w.n_launch;
}

}  // extern "C"
