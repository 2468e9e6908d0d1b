// C ABI of expert-parallel dispatch and combine (declared in include/tk_gating.h):
// validation, launch sizing, and the inter-process memory handles that let a
// rank address another rank's expert buffers.  The kernels are in ep.cuh.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "tk_gating.h"
#include "ep.cuh"

namespace tkg {
uint32_t* device_error_word();  // tk_gating.cu: the device error word of the current device
}

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

tk_status validate_ep(int64_t T, int64_t H, int32_t k, int32_t E) {
  if (T < 0 || H < 1 || k < 1 || E < 1) return TK_ERR_INVALID_ARG;
  if (H % 8 != 0 || k > TK_GATING_MAX_TOPK || E > TK_ROUTE_MAX_EXPERTS) return TK_ERR_UNSUPPORTED;
  if (T > 0 && T > static_cast<int64_t>(INT32_MAX) / k) return TK_ERR_UNSUPPORTED;
  return TK_OK;
}

int current_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

// As many CTAs as the SMs hold at once (every warp resident, each looping over
// the work items), or fewer when there are fewer items (one per warp).
template <typename Kernel>
int resident_grid(Kernel kernel, int64_t items, int num_sms) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, tkg::EP_THREADS, 0) != cudaSuccess || per_sm < 1)
    return 0;
  const int64_t warps_per_cta = tkg::EP_THREADS / 32;
  int64_t grid = (items + warps_per_cta - 1) / warps_per_cta;
  if (grid > static_cast<int64_t>(num_sms) * per_sm) grid = static_cast<int64_t>(num_sms) * per_sm;
  return static_cast<int>(grid < 1 ? 1 : grid);
}

// Row parts of about EP_PART_VECS vectors: parts per row and vectors per part
// (a multiple of 32 when the row has several parts; the last part shorter).
// A part never exceeds EP_PART_VECS (a multiple of 32), so a lane holds at most
// EP_LANE_VECS vectors of it.
bool row_parts(int64_t vec_per_row, int32_t* parts, int64_t* part_vecs) {
  *parts = static_cast<int32_t>((vec_per_row + tkg::EP_PART_VECS - 1) / tkg::EP_PART_VECS);
  *part_vecs = (vec_per_row + *parts - 1) / *parts;
  if (*parts > 1) *part_vecs = (*part_vecs + 31) / 32 * 32;
  return *part_vecs <= tkg::EP_PART_VECS && static_cast<int64_t>(*parts) * *part_vecs >= vec_per_row;
}

template <int KMAX>
tk_status launch_combine(const tkg::EpCombineParams& p, int num_sms, cudaStream_t s) {
  const int grid = resident_grid(tkg::ep_combine_kernel<KMAX>, p.T * p.parts, num_sms);
  if (grid == 0) return TK_ERR_CUDA;
  tkg::ep_combine_kernel<KMAX><<<grid, tkg::EP_THREADS, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? TK_OK : TK_ERR_CUDA;
}

template <int KMAX>
tk_status launch_dispatch(const tkg::EpDispatchParams& p, int num_sms, cudaStream_t s) {
  const int grid = resident_grid(tkg::ep_dispatch_kernel<KMAX>, p.T * p.parts, num_sms);
  if (grid == 0) return TK_ERR_CUDA;
  tkg::ep_dispatch_kernel<KMAX><<<grid, tkg::EP_THREADS, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? TK_OK : TK_ERR_CUDA;
}

// ---- inter-process handles: an allocation's handle plus the offset into it ----
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  });
  return fn;
}

struct IpcHandle {
  cudaIpcMemHandle_t mem;  // of the allocation that contains the pointer
  uint64_t offset;         // of the pointer into that allocation
};
static_assert(sizeof(IpcHandle) <= TK_EP_IPC_HANDLE_BYTES, "handle size");

}  // namespace

extern "C" {

tk_status tk_gating_fused_dispatch(const void* tokens, int64_t T, int64_t H, int32_t k, int32_t E, const int32_t* ids,
                                   const int32_t* offsets, const int32_t* slot_pos, const uint64_t* rows,
                                   void* stream) {
  tk_status st = validate_ep(T, H, k, E);
  if (st != TK_OK) return st;
  if (T == 0) return TK_OK;
  if (!tokens || !ids || !offsets || !slot_pos || !rows) return TK_ERR_INVALID_ARG;
  if (!aligned(tokens, 16) || !aligned(ids, 4) || !aligned(offsets, 4) || !aligned(slot_pos, 4) || !aligned(rows, 8))
    return TK_ERR_ALIGNMENT;
  uint32_t* err = tkg::device_error_word();
  const int sms = current_sms();
  if (err == nullptr || sms == 0) return TK_ERR_CUDA;
  tkg::EpDispatchParams p;
  p.tokens = static_cast<const uint4*>(tokens);
  p.ids = ids;
  p.offsets = offsets;
  p.slot_pos = slot_pos;
  p.rows = rows;
  p.err_word = err;
  p.T = T;
  p.vec_per_row = H / 8;
  if (!row_parts(p.vec_per_row, &p.parts, &p.part_vecs)) return TK_ERR_UNSUPPORTED;
  p.k = k;
  p.E = E;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k <= 4) return launch_dispatch<4>(p, sms, s);
  if (k <= 8) return launch_dispatch<8>(p, sms, s);
  if (k <= 16) return launch_dispatch<16>(p, sms, s);
  return launch_dispatch<32>(p, sms, s);
}

tk_status tk_gating_fused_combine(const uint64_t* rows, int64_t T, int64_t H, int32_t k, int32_t E, const int32_t* ids,
                                  const int32_t* offsets, const int32_t* slot_pos, const float* scores, void* out,
                                  void* stream) {
  tk_status st = validate_ep(T, H, k, E);
  if (st != TK_OK) return st;
  if (T == 0) return TK_OK;
  if (!rows || !ids || !offsets || !slot_pos || !scores || !out) return TK_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(ids, 4) || !aligned(offsets, 4) || !aligned(slot_pos, 4) ||
      !aligned(scores, 4) || !aligned(rows, 8))
    return TK_ERR_ALIGNMENT;
  uint32_t* err = tkg::device_error_word();
  const int sms = current_sms();
  if (err == nullptr || sms == 0) return TK_ERR_CUDA;
  tkg::EpCombineParams p;
  p.rows = rows;
  p.ids = ids;
  p.offsets = offsets;
  p.slot_pos = slot_pos;
  p.scores = scores;
  p.out = static_cast<uint4*>(out);
  p.err_word = err;
  p.T = T;
  p.vec_per_row = H / 8;
  if (!row_parts(p.vec_per_row, &p.parts, &p.part_vecs)) return TK_ERR_UNSUPPORTED;
  p.k = k;
  p.E = E;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k <= 4) return launch_combine<4>(p, sms, s);
  if (k <= 8) return launch_combine<8>(p, sms, s);
  if (k <= 16) return launch_combine<16>(p, sms, s);
  return launch_combine<32>(p, sms, s);
}

tk_status tk_gating_ep_rows_table(const int32_t* offsets_all, int32_t R, int32_t E, int32_t rank, const uint64_t* bases,
                                  const uint64_t* out_bases, int64_t H, uint64_t* rows, uint64_t* out_rows,
                                  int32_t* recv_offsets, void* stream) {
  if (R < 1 || E < 1 || rank < 0 || rank >= R || H < 1) return TK_ERR_INVALID_ARG;
  if (E > TK_ROUTE_MAX_EXPERTS || E % R != 0 || H % 8 != 0) return TK_ERR_UNSUPPORTED;
  if (!offsets_all || !bases || !rows || !recv_offsets || (out_rows != nullptr && out_bases == nullptr))
    return TK_ERR_INVALID_ARG;
  if (!aligned(offsets_all, 4) || !aligned(recv_offsets, 4) || !aligned(bases, 8) || !aligned(rows, 8) ||
      !aligned(out_bases, 8) || !aligned(out_rows, 8))
    return TK_ERR_ALIGNMENT;
  if (current_sms() == 0) return TK_ERR_CUDA;
  tkg::ep_rows_table_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      offsets_all, R, E, rank, bases, out_bases, H * 2, rows, out_rows, recv_offsets);
  return cudaGetLastError() == cudaSuccess ? TK_OK : TK_ERR_CUDA;
}

tk_status tk_gating_ep_ipc_handle(const void* dev_ptr, void* handle) {
  if (dev_ptr == nullptr || handle == nullptr) return TK_ERR_INVALID_ARG;
  AddressRangeFn range = address_range_fn();
  if (range == nullptr) return TK_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return TK_ERR_INVALID_ARG;
  IpcHandle h;
  std::memset(&h, 0, sizeof(h));
  if (cudaIpcGetMemHandle(&h.mem, reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return TK_ERR_CUDA;
  }
  h.offset = static_cast<uint64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  std::memset(handle, 0, TK_EP_IPC_HANDLE_BYTES);
  std::memcpy(handle, &h, sizeof(h));
  return TK_OK;
}

tk_status tk_gating_ep_ipc_open(const void* handle, void** dev_ptr) {
  if (handle == nullptr || dev_ptr == nullptr) return TK_ERR_INVALID_ARG;
  IpcHandle h;
  std::memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h.mem, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return TK_ERR_CUDA;
  }
  *dev_ptr = static_cast<uint8_t*>(base) + h.offset;
  return TK_OK;
}

tk_status tk_gating_ep_ipc_close(void* dev_ptr, const void* handle) {
  if (dev_ptr == nullptr || handle == nullptr) return TK_ERR_INVALID_ARG;
  IpcHandle h;
  std::memcpy(&h, handle, sizeof(h));
  if (cudaIpcCloseMemHandle(static_cast<uint8_t*>(dev_ptr) - h.offset) != cudaSuccess) {
    cudaGetLastError();
    return TK_ERR_CUDA;
  }
  return TK_OK;
}

}  // extern "C"
