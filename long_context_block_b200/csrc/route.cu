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
// One kernel, grid = (chunks of kRouteChunk blocks, query rows), for queries that do not
// share a sequence with many others (decode).  A CTA stages the query's head vectors and
// its chunk of pooled keys in shared memory and computes q_j . kp_b on the tensor cores
// (mma.sync, bf16 operands, fp32 pooled keys split into hi + lo parts).  It writes
// sum_b ReLU(q_j . kp_b) for its chunk to the workspace and bumps the row's counter;
// the last CTA of a row to finish sums the chunk partials, applies |w_j| / M_t (common
// to all blocks, so applied once), writes E and selects the top-h heads by repeated
// warp arg-max.
//
// The same kernel, in its block-score mode, reduces the affinities along the other axis
// for the HISA-style token-axis filter (MISA page, "Key distinction from HISA"):
// G[t,b] = sum_j A[t,j,b] = sum_j w[t,j] * ReLU(q[t,j] . kp_b), one value per block of
// the query's prefix, written straight to G (each CTA owns its chunk's blocks).
#include <cuda_bf16.h>

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

// One CTA = one (chunk of kCh blocks, query row): 4 warps; warp w takes the 16-head row
// tiles w, w+4 (of ceil(H/16)).  The contraction S[j, b] = q_j . kp_b runs on the tensor
// cores as mma.sync m16n8k16 with bf16 operands and fp32 accumulators: A = the query's
// head vectors (bf16 as given), B = the chunk's pooled keys split into bf16 hi + lo
// (hi = bf16(kp), lo = bf16(kp - hi)), so the two products reproduce the fp32 pooled key
// to about 2^-16 relative.  Operands sit in shared memory as rows of 128 bf16 padded by
// 16 bytes (fragment loads conflict-free).
constexpr int kRouteThreads = 128;
constexpr int kRowPad = kHeadDim + 8;   // bf16 elements per padded shared row

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// kBlockScores: write G[row, b] = sum_j w_j * ReLU(q_j . kp_b) for the chunk's blocks to
// `partial` (row stride Mpool) and M_t - 1 to counters[row] (the last block index), instead
// of the head energies.
template <int MT, bool kBlockScores>   // MT: 16-head row tiles per warp (ceil(ceil(H/16)/4))
__global__ void __launch_bounds__(kRouteThreads) route_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const float* __restrict__ k_pool, const int32_t* __restrict__ pos, int T, int H,
    int64_t L, int B, int Mpool, float* __restrict__ partial, int nchunk, int* status,
    int64_t row0, const float* __restrict__ w, int h, int* __restrict__ counters,
    int32_t* __restrict__ heads, float* __restrict__ E) {
  pdl_prologue();
  extern __shared__ __align__(16) uint16_t rsm[];
  uint16_t* qs = rsm;                                  // [16 * 4 * MT][kRowPad] bf16
  uint16_t* khi = qs + 16 * 4 * MT * kRowPad;          // [kCh][kRowPad]
  uint16_t* klo = khi + kCh * kRowPad;                 // [kCh][kRowPad]
  __shared__ float kpart[kHeadDim];                    // partial block's pooled key
  __shared__ float rsum[MISA_MAX_HEADS];
  __shared__ float red[kRouteThreads / 32][32];
  __shared__ float ev[MISA_MAX_HEADS];
  __shared__ int s_last;
  const int64_t row = row0 + blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = prefix_len(pos, row, L, chunk == 0 && tid == 0 ? status : nullptr);
  const int M = (P + B - 1) / B;
  const int Mfull = P / B;
  const int b0 = chunk * kCh;
  if (b0 >= M) return;
  const int nb = min(b0 + kCh, M) - b0;
  const int64_t n = row / T;
  const bool has_part = Mfull < M && Mfull >= b0 && Mfull < b0 + nb;
  if (kBlockScores && chunk == 0 && tid == 0) counters[row] = M - 1;

  // the partial last block of this prefix: mean of keys Mfull*B .. P-1 (fp32)
  if (has_part) {
    const int s0 = Mfull * B, cnt = P - s0;
    const uint16_t* kr = k + ((int64_t)n * L + s0) * kHeadDim + tid;
    float a = 0.f;
    for (int s = 0; s < cnt; ++s) a += bf16_to_f32(kr[(int64_t)s * kHeadDim]);
    kpart[tid] = a / (float)cnt;
  }
  // stage q rows (16-byte copies) and the chunk's pooled keys as bf16 hi/lo; every load
  // of a thread is issued before any is stored
  constexpr int kQPer = 16 * 4 * MT * (kHeadDim / 8) / kRouteThreads;
  constexpr int kKPer = kCh * (kHeadDim / 4) / kRouteThreads;
  uint4 qv[kQPer];
  float4 kv[kKPer];
#pragma unroll
  for (int i = 0; i < kQPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int j = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    qv[i] = j < H ? reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim)[c]
                  : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kKPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int bb = e / (kHeadDim / 4), c = e % (kHeadDim / 4);
    const int b = b0 + bb;
    kv[i] = (bb < nb && b < Mfull)
                ? reinterpret_cast<const float4*>(k_pool + ((int64_t)n * Mpool + b) * kHeadDim)[c]
                : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < kQPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int j = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    *reinterpret_cast<uint4*>(qs + j * kRowPad + c * 8) = qv[i];
  }
  __syncthreads();   // kpart complete
#pragma unroll
  for (int i = 0; i < kKPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int bb = e / (kHeadDim / 4), c = e % (kHeadDim / 4);
    float4 v = kv[i];
    if (has_part && bb == Mfull - b0) v = reinterpret_cast<const float4*>(kpart)[c];
    const float hx = __bfloat162float(__float2bfloat16_rn(v.x));
    const float hy = __bfloat162float(__float2bfloat16_rn(v.y));
    const float hz = __bfloat162float(__float2bfloat16_rn(v.z));
    const float hw = __bfloat162float(__float2bfloat16_rn(v.w));
    uint2 hi, lo;
    hi.x = pack_bf16(hx, hy);
    hi.y = pack_bf16(hz, hw);
    lo.x = pack_bf16(v.x - hx, v.y - hy);
    lo.y = pack_bf16(v.z - hz, v.w - hw);
    *reinterpret_cast<uint2*>(khi + bb * kRowPad + c * 4) = hi;
    *reinterpret_cast<uint2*>(klo + bb * kRowPad + c * 4) = lo;
  }
  __syncthreads();

  // S = Q K^T on the tensor cores; thread (g = lane/4, c = lane%4) holds rows g, g+8 and
  // columns 2c, 2c+1 of every 16 x 8 tile
  const int g = lane >> 2, c4 = lane & 3;
  constexpr int kNT = kCh / 8;
  float acc[MT][kNT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int t = 0; t < kNT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][t][i] = 0.f;
#pragma unroll
  for (int k0 = 0; k0 < kHeadDim; k0 += 16) {
    uint32_t bh[kNT][2], bl[kNT][2];
#pragma unroll
    for (int t = 0; t < kNT; ++t) {
      const uint16_t* ph = khi + (t * 8 + g) * kRowPad + k0 + 2 * c4;
      const uint16_t* pl = klo + (t * 8 + g) * kRowPad + k0 + 2 * c4;
      bh[t][0] = *reinterpret_cast<const uint32_t*>(ph);
      bh[t][1] = *reinterpret_cast<const uint32_t*>(ph + 8);
      bl[t][0] = *reinterpret_cast<const uint32_t*>(pl);
      bl[t][1] = *reinterpret_cast<const uint32_t*>(pl + 8);
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int r0 = (warp + 4 * m) * 16;
      const uint16_t* pa = qs + (r0 + g) * kRowPad + k0 + 2 * c4;
      uint32_t a[4];
      a[0] = *reinterpret_cast<const uint32_t*>(pa);
      a[1] = *reinterpret_cast<const uint32_t*>(pa + 8 * kRowPad);
      a[2] = *reinterpret_cast<const uint32_t*>(pa + 8);
      a[3] = *reinterpret_cast<const uint32_t*>(pa + 8 * kRowPad + 8);
#pragma unroll
      for (int t = 0; t < kNT; ++t) {
        mma_bf16_16816(acc[m][t], a, bh[t][0], bh[t][1]);
        mma_bf16_16816(acc[m][t], a, bl[t][0], bl[t][1]);
      }
    }
  }
  if constexpr (kBlockScores) {
    // G[b] = sum_j w_j * ReLU(S[j, b]): this thread's heads (rows g, g + 8 of each of its
    // tiles), then the 8 lanes sharing its columns, then the 4 warps
    float gs[kNT][2];
#pragma unroll
    for (int t = 0; t < kNT; ++t) gs[t][0] = gs[t][1] = 0.f;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int r0 = (warp + 4 * m) * 16;
      const float wa = r0 + g < H ? w[row * H + r0 + g] : 0.f;
      const float wb = r0 + g + 8 < H ? w[row * H + r0 + g + 8] : 0.f;
#pragma unroll
      for (int t = 0; t < kNT; ++t)
#pragma unroll
        for (int i = 0; i < 2; ++i)
          gs[t][i] += wa * fmaxf(acc[m][t][i], 0.f) + wb * fmaxf(acc[m][t][2 + i], 0.f);
    }
#pragma unroll
    for (int t = 0; t < kNT; ++t)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float v = gs[t][i];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        if (g == 0) red[warp][t * 8 + 2 * c4 + i] = v;
      }
    __syncthreads();
    if (tid < nb) {
      float v = 0.f;
#pragma unroll
      for (int wv = 0; wv < kRouteThreads / 32; ++wv) v += red[wv][tid];
      partial[row * Mpool + b0 + tid] = v;
    }
  } else {
  // sum_b ReLU(q_j . kp_b) over the chunk's valid blocks, per head
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float s_lo = 0.f, s_hi = 0.f;   // rows g and g + 8
#pragma unroll
    for (int t = 0; t < kNT; ++t)
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (t * 8 + 2 * c4 + i < nb) {
          s_lo += fmaxf(acc[m][t][i], 0.f);
          s_hi += fmaxf(acc[m][t][2 + i], 0.f);
        }
    s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
    s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
    s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
    s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
    const int r0 = (warp + 4 * m) * 16;
    if (c4 == 0) {
      if (r0 + g < H) rsum[r0 + g] = s_lo;
      if (r0 + g + 8 < H) rsum[r0 + g + 8] = s_hi;
    }
  }
  __syncthreads();
  for (int j = tid; j < H; j += kRouteThreads) partial[(row * nchunk + chunk) * H + j] = rsum[j];
  __threadfence();
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
  }   // energies (not kBlockScores)
}

template <int MT, bool kBlockScores>
static cudaError_t launch_mt(const uint16_t* q, const float* w, const uint16_t* k,
                             const float* k_pool, const int32_t* pos, int rows, int T, int H,
                             int64_t L, int B, int h, int32_t* heads, float* E, float* partial,
                             int nchunk, int* counters, int* status, cudaStream_t st) {
  const int Mpool = (int)((L + B - 1) / B);
  const size_t smem = (size_t)(16 * 4 * MT + 2 * kCh) * kRowPad * sizeof(uint16_t);
  cudaError_t err = cudaFuncSetAttribute(route_kernel<MT, kBlockScores>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    dim3 grid(nchunk, (unsigned)nr);
    err = launch_pdl(route_kernel<MT, kBlockScores>, grid, dim3(kRouteThreads), smem, st, q, k,
                     k_pool, pos, T, H, L, B, Mpool, partial, nchunk, status, row0, w, h,
                     counters, heads, E);
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
  if (H <= 64)
    return launch_mt<1, false>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, partial,
                               nchunk, counters, status, st);
  return launch_mt<2, false>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, partial,
                             nchunk, counters, status, st);
}

cudaError_t launch_block_scores(const uint16_t* q, const float* w, const uint16_t* k,
                                const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                                int64_t L, int B, float* G, int32_t* last_block, int* status,
                                cudaStream_t st) {
  const int rows = nseq * T;
  const int64_t M = (L + B - 1) / B;
  const int nchunk = (int)((M + kRouteChunk - 1) / kRouteChunk);
  if (H <= 64)
    return launch_mt<1, true>(q, w, k, k_pool, pos, rows, T, H, L, B, 1, nullptr, nullptr, G,
                              nchunk, last_block, status, st);
  return launch_mt<2, true>(q, w, k, k_pool, pos, rows, T, H, L, B, 1, nullptr, nullptr, G,
                            nchunk, last_block, status, st);
}

}  // namespace misa
