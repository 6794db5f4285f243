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
// One kernel, grid = (chunks of kRouteChunk blocks, query rows).  A CTA stages its
// chunk of pooled keys in shared memory (fp32) and each thread keeps one head's query
// vector in registers; G thread groups split the chunk's blocks.  It writes
// sum_b ReLU(q_j . kp_b) for its chunk to the workspace and bumps the row's counter;
// the last CTA of a row to finish sums the chunk partials, applies |w_j| / M_t (common
// to all blocks, so applied once), writes E and selects the top-h heads by repeated
// warp arg-max.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kCh = kRouteChunk;

// (value desc, index asc) ordering for the warp arg-max.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// One warp: the h largest of ev[0..H) (all >= 0), by descending value, ties to the
// lower index, written to out[0..h).
__device__ __forceinline__ void select_top_h(const float* ev, int H, int h, int32_t* out) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = MISA_MAX_HEADS / 32;
  float e[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = lane + 32 * i;
    e[i] = j < H ? ev[j] : -1.f;   // -1 marks "absent or already taken"
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
    if (lane == 0) out[r] = bi;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (lane + 32 * i == bi) e[i] = -1.f;
  }
}

// Chunk of kRouteChunk blocks x up to 32*HG heads.  Thread (hp, bq) owns heads
// hp + 32*m (m < HG) and blocks 4*bq .. 4*bq+3 of the chunk: a register-tiled
// dot-product microkernel over d with q and pooled keys in shared memory (fp32).
constexpr int kRouteThreads = 256;
constexpr int kQStride = kHeadDim + 4;   // padded fp32 row: conflict-free 16-byte reads

template <int HG>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const float* __restrict__ k_pool, const int32_t* __restrict__ pos, int T, int H,
    int64_t L, int B, int Mpool, float* __restrict__ partial, int nchunk, int* status,
    int64_t row0, const float* __restrict__ w, int h, int* __restrict__ counters,
    int32_t* __restrict__ heads, float* __restrict__ E) {
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                                   // [32*HG][kQStride]
  float* kp = sm + 32 * HG * kQStride;              // [kCh][kQStride]
  __shared__ float red[kRouteThreads / 32][32 * HG];
  __shared__ float ev[MISA_MAX_HEADS];
  __shared__ int s_last;
  const int64_t row = row0 + blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x;
  const int P = prefix_len(pos, row, L, chunk == 0 && tid == 0 ? status : nullptr);
  const int M = (P + B - 1) / B;
  const int Mfull = P / B;
  const int b0 = chunk * kCh;
  if (b0 >= M) return;
  const int nb = min(b0 + kCh, M) - b0;
  const int64_t n = row / T;

  // q rows of this query (bf16 -> fp32), zero rows past H
  for (int e = tid; e < 32 * HG * (kHeadDim / 8); e += kRouteThreads) {
    const int j = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j < H) v = reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim)[c];
    float* d = qs + j * kQStride + c * 8;
    reinterpret_cast<float4*>(d)[0] = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
    reinterpret_cast<float4*>(d)[1] = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
  }
  // pooled keys of the chunk's full blocks; unused slots are zero
  for (int e = tid; e < kCh * (kHeadDim / 4); e += kRouteThreads) {
    const int bb = e / (kHeadDim / 4), c = e % (kHeadDim / 4);
    const int b = b0 + bb;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (bb < nb && b < Mfull)
      v = reinterpret_cast<const float4*>(k_pool + ((int64_t)n * Mpool + b) * kHeadDim)[c];
    reinterpret_cast<float4*>(kp + bb * kQStride)[c] = v;
  }
  __syncthreads();
  // the partial last block of this prefix: mean of keys Mfull*B .. P-1
  if (Mfull < M && Mfull >= b0 && Mfull < b0 + nb) {
    const int s0 = Mfull * B, cnt = P - s0;
    const int dim = tid % kHeadDim, part = tid / kHeadDim;   // 2 parts
    float a = 0.f;
    const uint16_t* kr = k + ((int64_t)n * L + s0) * kHeadDim + dim;
    for (int s = part; s < cnt; s += kRouteThreads / kHeadDim) a += bf16_to_f32(kr[(int64_t)s * kHeadDim]);
    float* tmp = ev;   // 128 floats of scratch
    if (part == 1) tmp[dim] = a;
    __syncthreads();
    if (part == 0) kp[(Mfull - b0) * kQStride + dim] = (a + tmp[dim]) / (float)cnt;
    __syncthreads();
  }

  const int hp = tid & 31, bq = tid >> 5;   // bq: 8 groups of 4 blocks
  float acc[HG][4];
#pragma unroll
  for (int m = 0; m < HG; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
#pragma unroll 4
  for (int d = 0; d < kHeadDim; d += 4) {
    float4 qv[HG], kv[4];
#pragma unroll
    for (int m = 0; m < HG; ++m) qv[m] = *reinterpret_cast<const float4*>(qs + (hp + 32 * m) * kQStride + d);
#pragma unroll
    for (int i = 0; i < 4; ++i) kv[i] = *reinterpret_cast<const float4*>(kp + (4 * bq + i) * kQStride + d);
#pragma unroll
    for (int m = 0; m < HG; ++m)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float x = acc[m][i];
        x = fmaf(qv[m].x, kv[i].x, x); x = fmaf(qv[m].y, kv[i].y, x);
        x = fmaf(qv[m].z, kv[i].z, x); x = fmaf(qv[m].w, kv[i].w, x);
        acc[m][i] = x;
      }
  }
  // sum_b ReLU(q_j . kp_b) over this thread's blocks, then over the 8 block groups
#pragma unroll
  for (int m = 0; m < HG; ++m) {
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (4 * bq + i < nb) sum += fmaxf(acc[m][i], 0.f);
    red[bq][hp + 32 * m] = sum;
  }
  __syncthreads();
  if (tid < H) {
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < kRouteThreads / 32; ++g) sum += red[g][tid];
    partial[(row * nchunk + chunk) * H + tid] = sum;
    __threadfence();
  }
  __syncthreads();
  const int nch = (M + kCh - 1) / kCh;
  if (tid == 0) s_last = atomicAdd(&counters[row], 1) == nch - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last CTA of this row: E[j] = |w_j| / M * sum over chunks, then the top-h heads.  The
  // chunk partials are summed by all threads (kRouteThreads / 32 groups of 32 heads), so
  // their L2 loads are in flight together rather than one after another.
  constexpr int kGroups = kRouteThreads / 32;
  {
    const int jj = tid & 31, grp = tid >> 5;
    for (int j0 = 0; j0 < H; j0 += 32) {
      const int j = j0 + jj;
      float sum = 0.f;
      if (j < H)
        for (int c = grp; c < nch; c += kGroups) sum += __ldcg(partial + (row * nchunk + c) * H + j);
      red[grp][jj] = sum;
      __syncthreads();
      if (grp == 0 && j < H) {
        float tot = 0.f;
#pragma unroll
        for (int g = 0; g < kGroups; ++g) tot += red[g][jj];
        const float v = fabsf(w[row * H + j]) * tot / (float)M;
        ev[j] = v;
        if (E) E[row * H + j] = v;
      }
      __syncthreads();
    }
  }
  if (tid < 32) select_top_h(ev, H, h, heads + row * h);
}

template <int HG>
static cudaError_t launch_hg(const uint16_t* q, const float* w, const uint16_t* k,
                             const float* k_pool, const int32_t* pos, int rows, int T, int H,
                             int64_t L, int B, int h, int32_t* heads, float* E, float* partial,
                             int nchunk, int* counters, int* status, cudaStream_t st) {
  const int Mpool = (int)((L + B - 1) / B);
  const size_t smem = (size_t)(32 * HG + kCh) * kQStride * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(route_kernel<HG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    dim3 grid(nchunk, (unsigned)nr);
    route_kernel<HG><<<grid, kRouteThreads, smem, st>>>(q, k, k_pool, pos, T, H, L, B, Mpool,
                                                        partial, nchunk, status, row0, w, h,
                                                        counters, heads, E);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_route(const uint16_t* q, const float* w, const uint16_t* k,
                         const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                         int64_t L, int B, int h, int32_t* heads, float* E, float* partial,
                         int nchunk, int* counters, int* status, cudaStream_t st) {
  const int rows = nseq * T;
  cudaError_t err = cudaMemsetAsync(counters, 0, (size_t)rows * sizeof(int), st);
  if (err != cudaSuccess) return err;
  switch ((H + 31) / 32) {
    case 1: return launch_hg<1>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, partial, nchunk, counters, status, st);
    case 2: return launch_hg<2>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, partial, nchunk, counters, status, st);
    case 3: return launch_hg<3>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, partial, nchunk, counters, status, st);
    default: return launch_hg<4>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, partial, nchunk, counters, status, st);
  }
}

}  // namespace misa
