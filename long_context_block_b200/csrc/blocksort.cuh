// Block-wide bitonic sort of 64-bit values held in registers (1024-thread blocks).
#pragma once

#include <cstdint>

namespace misa {

constexpr int kSortThreads = 1024;

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort into descending order of kSortThreads * E 64-bit values, E consecutive slots
// per thread held in registers.  Compare-exchange partners inside a thread stay in
// registers, partners inside a warp are exchanged by shuffles, and only partners in
// other warps go through `xbuf` (kSortThreads * E slots of shared memory).  All threads of
// the block must call it.
template <int E, int NT = kSortThreads>
__device__ __forceinline__ void bitonic_desc_regs(uint64_t (&v)[E], uint64_t* xbuf) {
  const int t = threadIdx.x;
  constexpr int N = NT * E;
#pragma unroll 1
  for (int kk = 2; kk <= N; kk <<= 1) {
    // strides j >= E pair slots of different threads (run-time loop)
#pragma unroll 1
    for (int j = kk >> 1; j >= E; j >>= 1) {
      const int tm = j / E;
      const bool lower = (t & tm) == 0;
      if (j < 32 * E) {   // partner in the same warp
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const bool desc = ((t * E + i) & kk) == 0;
          const uint64_t o = shfl_xor64(v[i], tm);
          v[i] = (desc == lower) ? (v[i] > o ? v[i] : o) : (v[i] < o ? v[i] : o);
        }
      } else {            // partner in another warp
#pragma unroll
        for (int i = 0; i < E; ++i) xbuf[t * E + i] = v[i];
        __syncthreads();
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const bool desc = ((t * E + i) & kk) == 0;
          const uint64_t o = xbuf[(t ^ tm) * E + i];
          v[i] = (desc == lower) ? (v[i] > o ? v[i] : o) : (v[i] < o ? v[i] : o);
        }
        __syncthreads();
      }
    }
    // strides j < E stay inside a thread; unrolled so every register index is static
#pragma unroll
    for (int j = E / 2; j > 0; j >>= 1) {
      if (j < kk) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
          if ((i & j) == 0) {
            const int p = i | j;
            const bool desc = ((t * E + i) & kk) == 0;
            const uint64_t a = v[i], b = v[p];
            if (desc ? (a < b) : (a > b)) { v[i] = b; v[p] = a; }
          }
        }
      }
    }
  }
}

template <int E, int NT = kSortThreads>
__device__ __forceinline__ void sort_buf_desc_e(uint64_t* buf) {
  uint64_t v[E];
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] = buf[threadIdx.x * E + i];
  __syncthreads();
  bitonic_desc_regs<E, NT>(v, buf);
#pragma unroll
  for (int i = 0; i < E; ++i) buf[threadIdx.x * E + i] = v[i];
  __syncthreads();
}

// Sort buf[0 .. sortn) (shared memory, sortn = NT * {1,2,4,8,16,32}) descending with a
// block of NT threads.
template <int NT>
__device__ __forceinline__ void sort_buf_desc_nt(uint64_t* buf, int sortn) {
  __syncthreads();
  switch (sortn / NT) {
    case 1: sort_buf_desc_e<1, NT>(buf); break;
    case 2: sort_buf_desc_e<2, NT>(buf); break;
    case 4: sort_buf_desc_e<4, NT>(buf); break;
    case 8: sort_buf_desc_e<8, NT>(buf); break;
    case 16: sort_buf_desc_e<16, NT>(buf); break;
    default: sort_buf_desc_e<32, NT>(buf); break;
  }
}

// Sort buf[0 .. sortn) (shared memory, sortn = kSortThreads * {1,2,4,8,16}) descending.
__device__ __forceinline__ void sort_buf_desc(uint64_t* buf, int sortn) {
  __syncthreads();
  switch (sortn / kSortThreads) {
    case 1: sort_buf_desc_e<1>(buf); break;
    case 2: sort_buf_desc_e<2>(buf); break;
    case 4: sort_buf_desc_e<4>(buf); break;
    case 8: sort_buf_desc_e<8>(buf); break;
    default: sort_buf_desc_e<16>(buf); break;
  }
}

}  // namespace misa
