// K1: block mean pooling of indexer keys -- Eq. (4) of the MISA paper summary
// (Methodology section 1), with Pool read as the arithmetic mean of a block's keys.
//
// HBM-bound: every key is read once (256 B per token) and each pooled key (512 B
// fp32) is written once.  One warp owns one (sequence, block): its two half-warps
// walk the even and odd tokens of the block, each lane owning one 16-byte slice
// (8 dims) of the 256-byte key row, so every warp-wide load covers two whole rows
// (512 contiguous bytes).  Eight token pairs are loaded before any is accumulated to
// keep enough bytes in flight per SM.
//
// The same kernel refreshes a range of blocks: in decode a sequence gains one key per
// step, so only the block holding it changes and the rest of the pooled keys are reused.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

__device__ __forceinline__ void acc8(float (&a)[8], const uint4& v) {
  a[0] += bf16lo(v.x); a[1] += bf16hi(v.x);
  a[2] += bf16lo(v.y); a[3] += bf16hi(v.y);
  a[4] += bf16lo(v.z); a[5] += bf16hi(v.z);
  a[6] += bf16lo(v.w); a[7] += bf16hi(v.w);
}

// Blocks b0 .. b0 + Mu - 1 of every sequence (M blocks per sequence in `out`).  W warps
// share one block: W = 1 for short blocks (a warp per block), W = 8 for long ones, whose
// tokens the CTA's warps split before a shared-memory reduction.
template <int W>
__global__ void __launch_bounds__(256) pool_mean_kernel(const uint4* __restrict__ k, int nseq,
                                                        int64_t L, int B, int M, int b0, int Mu,
                                                        float* __restrict__ out) {
  pdl_prologue();
  __shared__ float red[W > 1 ? W : 1][kHeadDim];
  const int lane = threadIdx.x & 31;
  const int wic = (threadIdx.x >> 5) % W;   // warp within its block's group
  const int64_t team = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / (32 * W);
  const int64_t nteams = ((int64_t)gridDim.x * blockDim.x) / (32 * W);
  const int half = lane >> 4;   // 0: even tokens of the pair, 1: odd tokens
  const int vec = lane & 15;    // which 16-byte slice of the key row
  const int64_t items = (int64_t)nseq * Mu;
  for (int64_t base_it = blockIdx.x * ((int64_t)blockDim.x / (32 * W)); base_it < items;
       base_it += nteams) {
    const int64_t it = base_it + (team - blockIdx.x * ((int64_t)blockDim.x / (32 * W)));
    const bool live = it < items;
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int64_t n = 0, b = 0, s0 = 0, s1 = 0;
    if (live) {
      n = it / Mu;
      b = b0 + (it - n * Mu);
      s0 = b * B;
      s1 = min(s0 + (int64_t)B, L);
      const uint4* base = k + n * L * 16 + vec;   // a key row is 16 uint4
      const int64_t step = 2 * W;                 // tokens between this warp's pairs
      int64_t s = s0 + 2 * wic + half;
      for (; s + 7 * step < s1; s += 8 * step) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcs(base + (s + u * step) * 16);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc8(a, v[u]);
      }
      for (; s < s1; s += step) acc8(a, __ldcs(base + s * 16));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] += __shfl_down_sync(0xffffffffu, a[i], 16);
    if constexpr (W > 1) {
      if (half == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) red[wic][vec * 8 + i] = a[i];
      }
      __syncthreads();
      if (wic == 0 && half == 0) {
        for (int w2 = 1; w2 < W; ++w2)
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] += red[w2][vec * 8 + i];
      }
      __syncthreads();
    }
    if (live && wic == 0 && half == 0) {
      const float inv = 1.0f / (float)(s1 - s0);
      float4* o = reinterpret_cast<float4*>(out + (n * M + b) * kHeadDim + vec * 8);
      o[0] = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
      o[1] = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
    }
  }
}

}  // namespace

cudaError_t launch_pool_mean(const uint16_t* k, int nseq, int64_t L, int B, float* k_pool,
                             cudaStream_t st, int64_t s_begin, int64_t s_end) {
  const int M = (int)((L + B - 1) / B);
  if (s_end < 0) s_end = L;
  const int b0 = (int)(s_begin / B);
  const int Mu = (int)((s_end + B - 1) / B) - b0;   // blocks meeting [s_begin, s_end)
  if (Mu <= 0) return cudaSuccess;
  const int64_t items = (int64_t)nseq * Mu;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (B >= 256) {   // a CTA of 8 warps per block
    const int grid = (int)(items < (int64_t)sms * 8 ? items : (int64_t)sms * 8);
    return launch_pdl(pool_mean_kernel<8>, dim3(grid), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(k), nseq, L, B, M, b0, Mu, k_pool);
  } else {          // a warp per block
    const int64_t want = (items + 7) / 8;
    const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    return launch_pdl(pool_mean_kernel<1>, dim3(grid), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(k), nseq, L, B, M, b0, Mu, k_pool);
  }
}

}  // namespace misa
