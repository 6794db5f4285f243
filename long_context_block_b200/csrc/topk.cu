// K5: per-row top-k token selection -- TopK of Eqs. (2), (10), (11), (12) of the MISA
// paper summary.  Output order: descending score, equal scores by ascending token
// index; rows shorter than k are padded with index -1 and value -inf.
//
// One CTA (1024 threads) per row.  Scores are mapped to order-preserving uint32 keys
// and the k-th largest key is found exactly by a three-pass radix select (11, 11 and
// 10 bits; shared-memory histograms, a block-wide suffix scan picks the bin).  A
// final pass in index order gathers every key above that threshold plus the lowest-
// index keys equal to it, so that exactly k (key, index) pairs remain; a bitonic sort
// of those 64-bit pairs in shared memory produces the output order.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;

__device__ __forceinline__ uint64_t compose(uint32_t key, int32_t id) {
  return ((uint64_t)key << 32) | (uint64_t)(~(uint32_t)id);
}

// Block-wide exclusive prefix sum over one value per thread (all threads must call).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums,
                                                    uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t ws = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, ws, off);
      if (lane >= off) ws += o;
    }
    warp_sums[lane] = ws;
  }
  __syncthreads();
  const uint32_t base = warp > 0 ? warp_sums[warp - 1] : 0u;
  total = warp_sums[31];
  __syncthreads();
  return base + incl - v;
}

__global__ void __launch_bounds__(kThreads) topk_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const int32_t* __restrict__ gather_len, const int32_t* __restrict__ index_map, int topk,
    int sortn, int32_t* __restrict__ idx, float* __restrict__ vals, int64_t row0) {
  extern __shared__ uint64_t sel[];   // [sortn]
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_digit, s_above, s_cnt;
  const int tid = threadIdx.x;
  const int64_t row = row0 + blockIdx.x;
  const int n = gather_len ? gather_len[row] : prefix_len(pos, row, L, nullptr);
  const float* x = scores + row * stride;
  const int32_t* imap = index_map ? index_map + row * stride : nullptr;

  if (n <= topk) {
    for (int i = tid; i < sortn; i += kThreads)
      sel[i] = i < n ? compose(score_key(x[i]), imap ? imap[i] : i) : 0ull;
  } else {
    uint32_t prefix = 0, mask = 0, kneed = (uint32_t)topk;
    for (int p = 0; p < 3; ++p) {
      const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
      const int nb = p == 2 ? 1024 : 2048;
      for (int b = tid; b < kBins; b += kThreads) hist[b] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kThreads) {
        const uint32_t key = score_key(x[i]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
      }
      __syncthreads();
      // suffix scan: thread t covers bins nb-1-2t (hi) and nb-2-2t (lo)
      const bool act = 2 * tid < nb;
      const uint32_t c_hi = act ? hist[nb - 1 - 2 * tid] : 0u;
      const uint32_t c_lo = act ? hist[nb - 2 - 2 * tid] : 0u;
      uint32_t total;
      const uint32_t excl = block_excl_scan(c_hi + c_lo, warp_sums, total);
      if (act) {
        if (excl < kneed && kneed <= excl + c_hi) {
          s_digit = nb - 1 - 2 * tid;
          s_above = excl;
        } else if (excl + c_hi < kneed && kneed <= excl + c_hi + c_lo) {
          s_digit = nb - 2 - 2 * tid;
          s_above = excl + c_hi;
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= (uint32_t)(nb - 1) << shift;
      kneed -= s_above;
      __syncthreads();
    }
    const uint32_t thr = prefix;
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    uint32_t eq_taken = 0;
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      const uint32_t key = i < n ? score_key(x[i]) : 0u;
      const bool gt = i < n && key > thr;
      const bool eq = i < n && key == thr;
      if (gt) sel[atomicAdd(&s_cnt, 1u)] = compose(key, imap ? imap[i] : i);
      uint32_t total;
      const uint32_t rank = block_excl_scan(eq ? 1u : 0u, warp_sums, total);
      if (eq && eq_taken + rank < kneed) sel[atomicAdd(&s_cnt, 1u)] = compose(key, imap ? imap[i] : i);
      eq_taken += total;
    }
    __syncthreads();
    for (int i = topk + tid; i < sortn; i += kThreads) sel[i] = 0ull;
  }
  __syncthreads();

  // bitonic sort, descending
  for (int kk = 2; kk <= sortn; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < (sortn >> 1); i += kThreads) {
        const int lo = ((i & ~(j - 1)) << 1) | (i & (j - 1));
        const int hi = lo | j;
        const uint64_t a = sel[lo], b = sel[hi];
        const bool desc = (lo & kk) == 0;
        if (desc ? (a < b) : (a > b)) { sel[lo] = b; sel[hi] = a; }
      }
      __syncthreads();
    }
  }

  const int nvalid = n < topk ? n : topk;
  for (int i = tid; i < topk; i += kThreads) {
    const int64_t o = row * topk + i;
    if (i < nvalid) {
      const uint64_t v = sel[i];
      idx[o] = (int32_t)(~(uint32_t)(v & 0xffffffffu));
      if (vals) vals[o] = key_score((uint32_t)(v >> 32));
    } else {
      idx[o] = -1;
      if (vals) vals[o] = __int_as_float(0xff800000);
    }
  }
}

}  // namespace

int topk_sort_size(int topk) {
  int s = 2;
  while (s < topk) s <<= 1;
  return s;
}

cudaError_t launch_topk(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                        const int32_t* gather_len, const int32_t* index_map, int rows,
                        int topk, int32_t* idx, float* vals, int* status, cudaStream_t st) {
  (void)status;
  const int sortn = topk_sort_size(topk);
  const size_t smem = (size_t)sortn * sizeof(uint64_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    topk_kernel<<<(unsigned)nr, kThreads, smem, st>>>(scores, stride, pos, L, gather_len,
                                                      index_map, topk, sortn, idx, vals, row0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace misa
