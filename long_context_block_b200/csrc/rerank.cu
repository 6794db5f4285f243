// K7 (preparation): MISA-dagger candidate lists -- Eq. (12) of the MISA paper summary
// (Methodology section 2) re-scores the coarse candidates Omega_t with all heads and
// keeps the top k.  To make that final TopK resolve equal scores by token index with
// the ordinary index-order pass, each row's candidates are first sorted ascending.
// Empty slots (-1) and ids outside the query's prefix are dropped (the latter are
// recorded as bad device input); `count` receives the number of valid candidates.
#include "blocksort.cuh"
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kThreads = kSortThreads;

__global__ void __launch_bounds__(kThreads) sort_candidates_kernel(
    const int32_t* __restrict__ cand, const int32_t* __restrict__ pos, int64_t L, int kprime,
    int sortn, int32_t* __restrict__ sorted, int32_t* __restrict__ count, int* status,
    int64_t row0) {
  extern __shared__ uint64_t buf[];   // [sortn]
  const int tid = threadIdx.x;
  const int64_t row = row0 + blockIdx.x;
  const int P = prefix_len(pos, row, L, tid == 0 ? status : nullptr);
  __shared__ int s_count;
  if (tid == 0) s_count = 0;
  __syncthreads();
  int valid_local = 0;
  // ascending token order = descending order of the complemented id; empty slots are 0
  for (int i = tid; i < sortn; i += kThreads) {
    uint64_t v = 0;
    if (i < kprime) {
      const int32_t c = cand[row * kprime + i];
      if (c >= 0 && c < P) {
        v = (uint64_t)(~(uint32_t)c) << 32;
        ++valid_local;
      } else if (c != -1) {
        set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
      }
    }
    buf[i] = v;
  }
  if (valid_local) atomicAdd(&s_count, valid_local);
  sort_buf_desc(buf, sortn);
  for (int i = tid; i < kprime; i += kThreads) {
    const uint64_t v = buf[i];
    sorted[row * kprime + i] = v ? (int32_t)(~(uint32_t)(v >> 32)) : -1;
  }
  if (tid == 0) count[row] = s_count;
}

}  // namespace

cudaError_t launch_sort_candidates(const int32_t* cand, const int32_t* pos, int rows,
                                   int64_t L, int kprime, int32_t* sorted, int32_t* count,
                                   int* status, cudaStream_t st) {
  const int sortn = topk_sort_size(kprime);
  const size_t smem = (size_t)sortn * sizeof(uint64_t);
  cudaError_t e = cudaFuncSetAttribute(sort_candidates_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    sort_candidates_kernel<<<(unsigned)nr, kThreads, smem, st>>>(cand, pos, L, kprime, sortn,
                                                                 sorted, count, status, row0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace misa
