// misa_score_topk_noalloc: the routed score + top-k entry point for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code that
// runs inside an allocator-free region of a serving engine (for example between a
// memory-pool snapshot and its replay, where any new allocation would break the
// pool's accounting), or plugins whose host framework owns every device allocation
// and exposes none to them.  This entry point needs no workspace: its scratch is a
// fixed array in the library's own device memory, reserved on every GPU that loads
// the library and held until the process exits.
//
// Limits and sharing rules:
//  * The scratch holds the routed scores of one call, nseq * T * L fp32 values, at
//    most kNoAllocScoreCapacity of them (16 MiB); larger calls are rejected with
//    MISA_ERR_STATIC_SCRATCH_TOO_SMALL before anything is enqueued.
//  * Every call on a device uses the same array, and the array keeps what the last
//    call left in it.  Calls whose GPU work overlaps (different streams, or several
//    host threads) race on it and must be serialised by the caller.
//  * The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call before
//    any stream capture.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"
#include "misa.h"

namespace {

constexpr size_t kNoAllocScoreCapacity = size_t(4) << 20;   // fp32 scores (16 MiB)
constexpr size_t kNoAllocBytes = misa::kStatusBytes + kNoAllocScoreCapacity * sizeof(float);
constexpr int kMaxDevices = 64;

// Scratch of the no-allocation entry point: status word (first 256 bytes), then scores.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MISA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MISA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MISA_OK;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (p == nullptr || cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" int misa_score_topk_noalloc(const uint16_t* q, const float* w, const uint16_t* k,
                                       const int32_t* heads, const int32_t* pos, int nseq, int T,
                                       int H, int d, int64_t L, int h, int topk, int32_t* idx,
                                       float* vals, int32_t* device_status, void* stream) {
  if (nseq < 1 || T < 1 || H < 1 || d < 1 || L < 1 || L >= INT32_MAX) return MISA_ERR_INVALID_ARG;
  if (d != MISA_HEAD_DIM || H > MISA_MAX_HEADS) return MISA_ERR_UNSUPPORTED;
  if (h < 1 || h > H || topk < 1) return MISA_ERR_INVALID_ARG;
  if (h > MISA_MAX_ROUTED || topk > MISA_MAX_TOPK) return MISA_ERR_UNSUPPORTED;
  if (q == nullptr || w == nullptr || k == nullptr || heads == nullptr || pos == nullptr ||
      idx == nullptr)
    return MISA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) % 16)
    return MISA_ERR_INVALID_ARG;
  const size_t rows = (size_t)nseq * T;
  if (rows * (size_t)L > kNoAllocScoreCapacity) return MISA_ERR_STATIC_SCRATCH_TOO_SMALL;
  for (const void* p : {(const void*)q, (const void*)w, (const void*)k, (const void*)heads,
                        (const void*)pos, (const void*)idx})
    if (!is_device_ptr(p)) return MISA_ERR_INVALID_ARG;
  if ((vals && !is_device_ptr(vals)) || (device_status && !is_device_ptr(device_status)))
    return MISA_ERR_INVALID_ARG;

  void* scratch = nullptr;
  const int s = scratch_for_current_device(&scratch);
  if (s != MISA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  int* status = reinterpret_cast<int*>(scratch);
  float* scores = reinterpret_cast<float*>(reinterpret_cast<char*>(scratch) + misa::kStatusBytes);
  // the status word must start each call at zero; the scores are fully written before read
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return MISA_ERR_CUDA;
  if (misa::launch_score_simt(q, w, k, heads, h, pos, nullptr, nullptr, nseq, T, H, L, scores, L,
                              status, st) != cudaSuccess)
    return MISA_ERR_CUDA;
  if (misa::launch_topk(scores, L, pos, L, nullptr, nullptr, (int)rows, topk, idx, vals, status,
                        st) != cudaSuccess)
    return MISA_ERR_CUDA;
  if (device_status &&
      cudaMemcpyAsync(device_status, status, sizeof(int), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return MISA_ERR_CUDA;
  return MISA_OK;
}
