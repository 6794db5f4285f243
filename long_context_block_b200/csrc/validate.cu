// Host-side checks of the device buffers every entry point is given: non-null, aligned,
// allocated on the current CUDA device, and (for plain device allocations) long enough
// for the bytes the call will touch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"
#include "misa.h"

namespace misa {
namespace {

using GetRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

GetRangeFn get_range_fn() {
  static GetRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetRangeFn>(p);
    cudaGetLastError();
  });
  return fn;
}

}  // namespace

int check_dev(const void* p, size_t bytes, size_t align) {
  if (p == nullptr) return MISA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p) % align) return MISA_ERR_INVALID_ARG;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return MISA_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return MISA_ERR_INVALID_ARG;
  if (a.type == cudaMemoryTypeDevice) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || a.device != dev) {
      cudaGetLastError();
      return MISA_ERR_INVALID_ARG;   // another GPU's buffer
    }
    if (GetRangeFn fn = get_range_fn()) {
      CUdeviceptr base = 0;
      size_t size = 0;
      if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(p)) == CUDA_SUCCESS) {
        if (reinterpret_cast<uintptr_t>(p) + bytes > (uintptr_t)base + size)
          return MISA_ERR_INVALID_ARG;
      }
    }
  }
  return MISA_OK;
}

int check_opt(const void* p, size_t bytes, size_t align) {
  return p == nullptr ? MISA_OK : check_dev(p, bytes, align);
}

}  // namespace misa
