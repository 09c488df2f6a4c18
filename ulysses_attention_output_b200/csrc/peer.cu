// CUDA IPC export and mapping of device memory, for the multi-GPU form of the fused exchange:
// every GPU of a Ulysses layer holds its own sequence-shard slabs, and the other GPUs' fused
// calls store their finished output tiles straight into them through these mappings (NVLink
// peer stores).  Host-side only; no kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "xs.h"
#include "xs_internal.cuh"

static_assert(sizeof(cudaIpcMemHandle_t) == XS_IPC_HANDLE_BYTES, "IPC handle size mismatch");

namespace {

std::once_flag g_range_once;
PFN_cuMemGetAddressRange_v3020 g_range = nullptr;

PFN_cuMemGetAddressRange_v3020 range_fn() {
  std::call_once(g_range_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 3020, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  });
  return g_range;
}

xs_status cuda_fail(cudaError_t e, const char *what) {
  return static_cast<xs_status>(xs::record_error(XS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e)));
}

xs_status invalid(const char *what) {
  return static_cast<xs_status>(xs::record_error(XS_ERR_INVALID_ARG, "%s", what));
}

}  // namespace

extern "C" {

xs_status xs_ipc_export(const void *ptr, unsigned char *handle, long long *offset) {
  if (!ptr || !handle || !offset) return invalid("ptr, handle and offset must be non-null");
  auto range = range_fn();
  if (!range)
    return static_cast<xs_status>(xs::record_error(XS_ERR_CUDA, "driver entry point cuMemGetAddressRange not found"));
  CUdeviceptr base = 0;
  size_t size = 0;
  const CUresult r = range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr));
  if (r != CUDA_SUCCESS)
    return static_cast<xs_status>(
        xs::record_error(XS_ERR_CUDA, "cuMemGetAddressRange failed (%d): not device memory", static_cast<int>(r)));
  cudaIpcMemHandle_t h;
  const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base));
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
  std::memcpy(handle, &h, sizeof(h));
  xs::clear_error();
  *offset = static_cast<long long>(reinterpret_cast<uintptr_t>(ptr) - static_cast<uintptr_t>(base));
  return XS_OK;
}

xs_status xs_ipc_open(const unsigned char *handle, void **base) {
  if (!handle || !base) return invalid("handle and base must be non-null");
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void *p = nullptr;
  const cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
  *base = p;
  xs::clear_error();
  return XS_OK;
}

xs_status xs_ipc_close(void *base) {
  if (!base) return invalid("base must be non-null");
  const cudaError_t e = cudaIpcCloseMemHandle(base);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
  xs::clear_error();
  return XS_OK;
}

}  // extern "C"
