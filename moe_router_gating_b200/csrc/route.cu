// C ABI of the routing-metadata operator (declared in include/tk_gating.h):
// validation, launch planning, the stream-ordered workspace and the
// launches.  The kernels are in route.cuh.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "tk_gating.h"
#include "route.cuh"

namespace tkg {
uint32_t* device_error_word();  // tk_gating.cu: the device error word of the current device
}

namespace {

int64_t round_up64(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

tk_status validate_route(int64_t T, int32_t k, int32_t E) {
  if (T < 0 || k < 1 || E < 1) return TK_ERR_INVALID_ARG;
  if (E > TK_ROUTE_MAX_EXPERTS) return TK_ERR_UNSUPPORTED;
  if (T > 0 && T > static_cast<int64_t>(INT32_MAX) / k) return TK_ERR_UNSUPPORTED;  // positions are int32
  return TK_OK;
}

int32_t count_smem_bytes(int32_t E) { return tkg::ROUTE_WARPS * (E + 1) * 4; }

int32_t scatter_smem_bytes(int32_t E) {
  const int32_t E4 = static_cast<int32_t>(round_up64(E, 4));
  return (tkg::ROUTE_WARPS * (E + 1) + 2 * E4 + 36) * 4 + 2 * tkg::ROUTE_THREADS * 16;
}

tk_status route_plan_impl(int64_t T, int32_t k, int32_t E, int32_t num_sms, tk_route_plan* plan) {
  if (plan == nullptr || num_sms < 1) return TK_ERR_INVALID_ARG;
  std::memset(plan, 0, sizeof(*plan));
  const tk_status st = validate_route(T, k, E);
  if (st != TK_OK) return st;
  const int64_t n = T * k;
  // Spread the slots over at most one CTA per SM, each warp taking at least
  // ROUTE_MIN_WARP_SLOTS of them (a multiple of 32).
  const int64_t warps_max = static_cast<int64_t>(num_sms) * tkg::ROUTE_WARPS;
  int64_t L = round_up64((n + warps_max - 1) / warps_max, 32);
  if (L < tkg::ROUTE_MIN_WARP_SLOTS) L = tkg::ROUTE_MIN_WARP_SLOTS;
  const int64_t cta_slots = L * tkg::ROUTE_WARPS;
  int64_t G = (n + cta_slots - 1) / cta_slots;
  if (G < 1) G = 1;
  plan->ctas = static_cast<int32_t>(G);
  plan->threads = tkg::ROUTE_THREADS;
  plan->warp_slots = L;
  plan->workspace_bytes = G > 1 ? G * round_up64(E, 4) * 4 : 0;  // one CTA needs no table
  // counts from the gating: the table, then the scatter CTAs' arrival counter
  // (16 bytes keep the size a multiple of 16)
  plan->fused_workspace_bytes = G > 1 ? plan->workspace_bytes + 16 : 0;
  plan->count_smem_bytes = count_smem_bytes(E);
  plan->scatter_smem_bytes = scatter_smem_bytes(E);
  return TK_OK;
}

// Per-device set-up, done on the first call made with that device current:
// the SM count, the sm_100 check and the kernels' shared-memory limits.
struct RouteDevice {
  bool ready = false;
  tk_status status = TK_OK;
  int num_sms = 0;
};

constexpr int kMaxDevices = 64;
RouteDevice g_route_devices[kMaxDevices];
std::mutex g_route_mutex;

template <typename Kernel>
bool set_route_smem(Kernel kernel, int32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

template <int NB>
bool set_scatter_smem(int32_t bytes) {
  return set_route_smem(tkg::route_scatter_kernel<NB, tkg::ROUTE_ONE_CTA>, bytes) &&
         set_route_smem(tkg::route_scatter_kernel<NB, tkg::ROUTE_TABLE>, bytes) &&
         set_route_smem(tkg::route_scatter_kernel<NB, tkg::ROUTE_FUSED>, bytes);
}

const RouteDevice* route_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  RouteDevice& d = g_route_devices[dev];
  std::lock_guard<std::mutex> lock(g_route_mutex);
  if (d.ready) return &d;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (major != 10 || minor != 0) {
    d.status = TK_ERR_UNSUPPORTED;
    d.ready = true;
    return &d;
  }
  if (!set_route_smem(tkg::route_count_kernel, count_smem_bytes(TK_ROUTE_MAX_EXPERTS)) ||
      !set_scatter_smem<4>(scatter_smem_bytes(16)) || !set_scatter_smem<6>(scatter_smem_bytes(64)) ||
      !set_scatter_smem<8>(scatter_smem_bytes(256)) ||
      !set_scatter_smem<10>(scatter_smem_bytes(TK_ROUTE_MAX_EXPERTS))) {
    cudaGetLastError();
    return nullptr;  // not cached: a later call retries
  }
  d.status = TK_OK;
  d.ready = true;
  return &d;
}

template <int NB>
tk_status launch_scatter(const tk_route_plan& pl, const tkg::RouteParams& p, bool fused, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.ctas);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.scatter_smem_bytes;
  cfg.stream = stream;
  // programmatic dependent launch.  One CTA: the kernel may start while the
  // previous kernel (typically the gating) finishes, and waits for it before
  // reading ids.  Several: the scatter kernel may start once every count CTA has
  // passed its own dependency wait; it waits (griddepcontrol.wait) for the count
  // kernel's completion before reading the counts table
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err;
  if (pl.ctas == 1)
    err = cudaLaunchKernelEx(&cfg, tkg::route_scatter_kernel<NB, tkg::ROUTE_ONE_CTA>, p);
  else if (fused)
    err = cudaLaunchKernelEx(&cfg, tkg::route_scatter_kernel<NB, tkg::ROUTE_FUSED>, p);
  else
    err = cudaLaunchKernelEx(&cfg, tkg::route_scatter_kernel<NB, tkg::ROUTE_TABLE>, p);
  return err == cudaSuccess ? TK_OK : TK_ERR_CUDA;
}

// The launches on `stream`: the scatter kernel alone for one CTA, else the
// count kernel and the scatter kernel; `counts` holds plan.workspace_bytes.
// fused: the gating launch before has filled the counts table (and `counts`
// holds plan.fused_workspace_bytes: the table, then the arrival counter), so
// only the scatter kernel runs.
tk_status launch_route(const tk_route_plan& pl, const int32_t* ids, int64_t n, int32_t E, int32_t* counts,
                       int32_t* offsets, int32_t* sorted_slots, int32_t* slot_pos, bool fused, cudaStream_t stream) {
  tkg::RouteParams p;
  p.ids = ids;
  p.n = n;
  p.E = E;
  p.E4 = static_cast<int32_t>(round_up64(E, 4));
  p.Ep = E + 1;
  p.G = pl.ctas;
  p.warp_slots = pl.warp_slots;
  p.counts = counts;
  p.done = fused && counts != nullptr
               ? reinterpret_cast<uint32_t*>(counts + static_cast<int64_t>(pl.ctas) * p.E4)
               : nullptr;
  p.offsets = offsets;
  p.sorted_slots = sorted_slots;
  p.slot_pos = slot_pos;
  p.err_word = tkg::device_error_word();
  if (p.err_word == nullptr) return TK_ERR_CUDA;

  if (pl.ctas > 1 && !fused) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.ctas);
    cfg.blockDim = dim3(pl.threads);
    cfg.dynamicSmemBytes = pl.count_smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];  // a programmatic dependent of the previous kernel (see route_count_kernel)
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, tkg::route_count_kernel, p) != cudaSuccess) return TK_ERR_CUDA;
  }
  if (E <= 16) return launch_scatter<4>(pl, p, fused, stream);
  if (E <= 64) return launch_scatter<6>(pl, p, fused, stream);
  if (E <= 256) return launch_scatter<8>(pl, p, fused, stream);
  return launch_scatter<10>(pl, p, fused, stream);
}

tk_status route_checked(const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                        int32_t* sorted_slots, int32_t* slot_pos, const RouteDevice** dev_out,
                        tk_route_plan* pl) {
  tk_status st = validate_route(T, k, E);
  if (st != TK_OK) return st;
  const int64_t n = T * static_cast<int64_t>(k);
  if (offsets == nullptr || (n > 0 && (ids == nullptr || sorted_slots == nullptr || slot_pos == nullptr)))
    return TK_ERR_INVALID_ARG;
  if (!aligned4(offsets) || !aligned4(ids) || !aligned4(sorted_slots) || !aligned4(slot_pos))
    return TK_ERR_ALIGNMENT;
  const RouteDevice* dev = route_device();
  if (dev == nullptr) return TK_ERR_CUDA;
  if (dev->status != TK_OK) return dev->status;
  *dev_out = dev;
  return route_plan_impl(T, k, E, dev->num_sms, pl);
}

// ---- tk_gating_route_static: the counts table in a fixed device array ----
//
// For callers that cannot let the library allocate device memory.  The
// several-CTA path needs G x round_up(E, 4) int32 of scratch (the counts
// table); here it lives in this file-scope array instead of a stream-ordered
// allocation.  Every word the placing kernel reads is written by the counting
// kernel of the same call first, so nothing in it has to start at zero.  One
// array per device serves every call: calls that overlap on the device (other
// streams, other host threads) race on it.
static __device__ __align__(256) int32_t g_route_static_scratch[TK_ROUTE_STATIC_SCRATCH_BYTES / 4];

struct StaticScratch {
  bool ready = false;
  int32_t* ptr = nullptr;  // device address of g_route_static_scratch on that device
};

StaticScratch g_static_scratch[kMaxDevices];
std::mutex g_static_scratch_mutex;

// Set-up on the first call made with a device current: the array's device
// address (cudaGetSymbolAddress may load the module onto the device).
int32_t* static_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  StaticScratch& sc = g_static_scratch[dev];
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (sc.ready) return sc.ptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_static_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return nullptr;  // not cached: a later call retries
  }
  sc.ptr = static_cast<int32_t*>(p);
  sc.ready = true;
  return sc.ptr;
}

}  // namespace

namespace tkg {

// The routing half of tk_gating_fused_topk_route (tk_gating.cu): validation and
// the plan on the current device, then the placing launch after the gating.
tk_status route_fused_plan(int64_t T, int32_t k, int32_t E, tk_route_plan* pl) {
  const tk_status st = validate_route(T, k, E);
  if (st != TK_OK) return st;
  const RouteDevice* dev = route_device();
  if (dev == nullptr) return TK_ERR_CUDA;
  if (dev->status != TK_OK) return dev->status;
  return route_plan_impl(T, k, E, dev->num_sms, pl);
}

tk_status route_fused_launch(const tk_route_plan& pl, const int32_t* ids, int64_t n, int32_t E, int32_t* workspace,
                             int32_t* offsets, int32_t* sorted_slots, int32_t* slot_pos, cudaStream_t stream) {
  return launch_route(pl, ids, n, E, pl.ctas > 1 ? workspace : nullptr, offsets, sorted_slots, slot_pos, pl.ctas > 1,
                      stream);
}

}  // namespace tkg

extern "C" {

tk_status tk_gating_route_plan(int64_t T, int32_t k, int32_t E, int32_t num_sms, tk_route_plan* plan) {
  return route_plan_impl(T, k, E, num_sms, plan);
}

tk_status tk_gating_route(const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                          int32_t* sorted_slots, int32_t* slot_pos, void* stream) {
  const RouteDevice* dev = nullptr;
  tk_route_plan pl;
  tk_status st = route_checked(ids, T, k, E, offsets, sorted_slots, slot_pos, &dev, &pl);
  if (st != TK_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pl.workspace_bytes == 0)
    return launch_route(pl, ids, T * static_cast<int64_t>(k), E, nullptr, offsets, sorted_slots, slot_pos, false, s);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, static_cast<size_t>(pl.workspace_bytes), s) != cudaSuccess) {
    cudaGetLastError();
    return TK_ERR_CUDA;
  }
  st = launch_route(pl, ids, T * static_cast<int64_t>(k), E, static_cast<int32_t*>(ws), offsets, sorted_slots,
                    slot_pos, false, s);
  if (cudaFreeAsync(ws, s) != cudaSuccess && st == TK_OK) st = TK_ERR_CUDA;
  return st;
}

tk_status tk_gating_route_static(const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                                 int32_t* sorted_slots, int32_t* slot_pos, void* stream) {
  const RouteDevice* dev = nullptr;
  tk_route_plan pl;
  tk_status st = route_checked(ids, T, k, E, offsets, sorted_slots, slot_pos, &dev, &pl);
  if (st != TK_OK) return st;
  if (pl.workspace_bytes > TK_ROUTE_STATIC_SCRATCH_BYTES) return TK_ERR_UNSUPPORTED;
  int32_t* scratch = static_scratch();
  if (scratch == nullptr) return TK_ERR_CUDA;
  return launch_route(pl, ids, T * static_cast<int64_t>(k), E, pl.workspace_bytes > 0 ? scratch : nullptr, offsets,
                      sorted_slots, slot_pos, false, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
