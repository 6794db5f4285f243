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
//  * Every call looks up the array's device address (cudaGetSymbolAddress) with the
//    caller's device current; the first call on a device also loads the library's
//    device image there, so make that first call before any stream capture.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "misa.h"

namespace {

constexpr size_t kNoAllocScoreCapacity = size_t(4) << 20;   // fp32 scores (16 MiB)
constexpr size_t kNoAllocBytes = misa::kStatusBytes + kNoAllocScoreCapacity * sizeof(float);
// Scratch of the no-allocation entry point: status word (first 256 bytes), then scores.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of the scratch array on the current device.  Looked up on every call (it
// allocates nothing), so the address is never stale, e.g. after a cudaDeviceReset.
int scratch_for_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return MISA_ERR_CUDA;
  }
  *out = p;
  return MISA_OK;
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
  const size_t rows = (size_t)nseq * T;
  if (rows * (size_t)L > kNoAllocScoreCapacity) return MISA_ERR_STATIC_SCRATCH_TOO_SMALL;
  // the same buffer checks as misa_score_topk: every pointer on the current device,
  // aligned, and long enough for what the kernels read and write
  using misa::check_dev;
  using misa::check_opt;
  int s = MISA_OK;
  if ((s = check_dev(q, rows * H * d * 2, 16)) != MISA_OK ||
      (s = check_dev(w, rows * H * 4, 4)) != MISA_OK ||
      (s = check_dev(k, (size_t)nseq * L * d * 2, 16)) != MISA_OK ||
      (s = check_dev(heads, rows * h * 4, 4)) != MISA_OK ||
      (s = check_dev(pos, rows * 4, 4)) != MISA_OK ||
      (s = check_dev(idx, rows * topk * 4, 4)) != MISA_OK ||
      (s = check_opt(vals, rows * topk * 4, 4)) != MISA_OK ||
      (s = check_opt(device_status, 4, 4)) != MISA_OK)
    return s;

  void* scratch = nullptr;
  if ((s = scratch_for_current_device(&scratch)) != MISA_OK) return s;
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
