// K2: block-pooled head router -- Eqs. (7)-(8) of the MISA paper summary
// (Methodology section 1).
//
//   A[t,j,b] = w[t,j] * ReLU(q[t,j] . kp_b),   E[t,j] = (1/M_t) * sum_b |A[t,j,b]|
//   heads_t  = the h largest E[t,j]  (ties: lower j)
//
// kp_b are the pooled keys of query t's own prefix: full blocks come from the
// pooled-key tensor, and when the prefix ends inside a block that block's pooled
// key is the mean of its valid keys only, computed here from the raw keys.
//
// Pass 1 (route_partial_kernel): grid = (chunks of kRouteChunk blocks, query rows).
//   A CTA stages its chunk of pooled keys in shared memory (fp32) and each thread
//   keeps one head's query vector in registers; G thread groups split the chunk's
//   blocks.  It writes sum_b ReLU(q_j . kp_b) for its chunk to the workspace.
//   |w_j| / M_t is applied once, in pass 2, since it is common to all blocks.
// Pass 2 (route_select_kernel): one warp per query row sums the chunk partials,
//   forms E and selects the top-h heads by repeated warp arg-max.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kCh = kRouteChunk;

__global__ void __launch_bounds__(256) route_partial_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const float* __restrict__ k_pool, const int32_t* __restrict__ pos, int T, int H,
    int64_t L, int B, int Mpool, int G, float* __restrict__ partial, int nchunk,
    int* status, int64_t row0) {
  __shared__ __align__(16) float kp[kCh][kHeadDim];
  __shared__ float red[256];
  const int64_t row = row0 + blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x;
  const int P = prefix_len(pos, row, L, chunk == 0 && tid == 0 ? status : nullptr);
  const int M = (P + B - 1) / B;
  const int Mfull = P / B;
  const int b0 = chunk * kCh;
  if (b0 >= M) return;
  const int b1 = min(b0 + kCh, M);
  const int nb = b1 - b0;
  const int64_t n = row / T;
  const int nthreads = blockDim.x;

  // stage pooled keys of full blocks
  for (int e = tid; e < nb * (kHeadDim / 4); e += nthreads) {
    const int bb = e / (kHeadDim / 4), c = e % (kHeadDim / 4);
    const int b = b0 + bb;
    if (b < Mfull) {
      reinterpret_cast<float4*>(kp[bb])[c] =
          reinterpret_cast<const float4*>(k_pool + ((int64_t)n * Mpool + b) * kHeadDim)[c];
    }
  }
  // the partial last block of this prefix: mean of keys Mfull*B .. P-1
  if (Mfull < M && Mfull >= b0 && Mfull < b1) {
    const int s0 = Mfull * B, cnt = P - s0;
    const int dim = tid % kHeadDim, part = tid / kHeadDim, nparts = nthreads / kHeadDim;
    float a = 0.f;
    if (part < nparts) {
      const uint16_t* kr = k + ((int64_t)n * L + s0) * kHeadDim + dim;
      for (int s = part; s < cnt; s += nparts) a += bf16_to_f32(kr[(int64_t)s * kHeadDim]);
    }
    red[tid] = a;
    __syncthreads();
    if (tid < kHeadDim) {
      float sum = 0.f;
      for (int p = 0; p < nparts; ++p) sum += red[p * kHeadDim + tid];
      kp[Mfull - b0][tid] = sum / (float)cnt;
    }
  }
  __syncthreads();

  const int j = tid % H, g = tid / H;
  float acc = 0.f;
  if (g < G) {
    float qr[kHeadDim];
    const uint4* qv = reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim);
#pragma unroll
    for (int c = 0; c < kHeadDim / 8; ++c) {
      const uint4 v = qv[c];
      qr[8 * c + 0] = bf16lo(v.x); qr[8 * c + 1] = bf16hi(v.x);
      qr[8 * c + 2] = bf16lo(v.y); qr[8 * c + 3] = bf16hi(v.y);
      qr[8 * c + 4] = bf16lo(v.z); qr[8 * c + 5] = bf16hi(v.z);
      qr[8 * c + 6] = bf16lo(v.w); qr[8 * c + 7] = bf16hi(v.w);
    }
    for (int bb = g; bb < nb; bb += G) {
      const float4* kv = reinterpret_cast<const float4*>(kp[bb]);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int c = 0; c < kHeadDim / 4; c += 2) {
        const float4 x = kv[c], y = kv[c + 1];
        d0 = fmaf(qr[4 * c + 0], x.x, d0); d0 = fmaf(qr[4 * c + 1], x.y, d0);
        d0 = fmaf(qr[4 * c + 2], x.z, d0); d0 = fmaf(qr[4 * c + 3], x.w, d0);
        d1 = fmaf(qr[4 * c + 4], y.x, d1); d1 = fmaf(qr[4 * c + 5], y.y, d1);
        d1 = fmaf(qr[4 * c + 6], y.z, d1); d1 = fmaf(qr[4 * c + 7], y.w, d1);
      }
      acc += fmaxf(d0 + d1, 0.f);
    }
  }
  __syncthreads();
  red[tid] = acc;
  __syncthreads();
  if (tid < H) {
    float sum = 0.f;
    for (int gg = 0; gg < G; ++gg) sum += red[gg * H + tid];
    partial[(row * nchunk + chunk) * H + tid] = sum;
  }
}

// (value desc, index asc) ordering for the warp arg-max.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(256) route_select_kernel(
    const float* __restrict__ w, const int32_t* __restrict__ pos, int rows, int H, int64_t L,
    int B, int h, const float* __restrict__ partial, int nchunk, int32_t* __restrict__ heads,
    float* __restrict__ E) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  const int P = prefix_len(pos, row, L, nullptr);
  const int M = (P + B - 1) / B;
  const int nch = (M + kCh - 1) / kCh;
  constexpr int kPer = MISA_MAX_HEADS / 32;
  float e[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = lane + 32 * i;
    e[i] = -1.f;   // E >= 0, so -1 marks "absent or already taken"
    if (j < H) {
      float s = 0.f;
      for (int c = 0; c < nch; ++c) s += partial[(row * nchunk + c) * H + j];
      const float v = fabsf(w[row * H + j]) * s / (float)M;
      e[i] = v;
      if (E) E[row * H + j] = v;
    }
  }
  for (int r = 0; r < h; ++r) {
    float bv = -1.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int j = lane + 32 * i;
      if (e[i] >= 0.f && better(e[i], j, bv, bi)) { bv = e[i]; bi = j; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) heads[row * h + r] = bi;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (lane + 32 * i == bi) e[i] = -1.f;
  }
}

}  // namespace

cudaError_t launch_route(const uint16_t* q, const float* w, const uint16_t* k,
                         const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                         int64_t L, int B, int h, int32_t* heads, float* E, float* partial,
                         int nchunk, int* status, cudaStream_t st) {
  const int rows = nseq * T;
  const int Mpool = (int)((L + B - 1) / B);
  int G = 256 / H;
  if (G < 1) G = 1;
  const int threads = ((H * G + 31) / 32) * 32 < kHeadDim ? kHeadDim : ((H * G + 31) / 32) * 32;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    dim3 grid(nchunk, (unsigned)nr);
    route_partial_kernel<<<grid, threads, 0, st>>>(q, k, k_pool, pos, T, H, L, B, Mpool, G,
                                                   partial, nchunk, status, row0);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const int sel_blocks = (rows * 32 + 255) / 256;
  route_select_kernel<<<sel_blocks, 256, 0, st>>>(w, pos, rows, H, L, B, h, partial, nchunk,
                                                  heads, E);
  return cudaGetLastError();
}

}  // namespace misa
