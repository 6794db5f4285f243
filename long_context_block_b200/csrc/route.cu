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
// For queries that do not share a sequence with many others (decode): every query row is
// a thread-block cluster of up to 16 CTAs (8 where a device cannot hold 16).  Each CTA
// stages the query's head vectors once and walks its share of the prefix's chunks of
// kRouteChunk blocks: the chunk's pooled keys go to shared memory split into bf16 hi + lo
// parts, q_j . kp_b runs on the tensor cores (mma.sync, fp32 accumulators), and the CTA
// adds sum_b ReLU(q_j . kp_b) into its per-head sums.  CTA 0 of the cluster then sums the
// members' partial sums through distributed shared memory, applies |w_j| / M_t (common to
// all blocks, so applied once), writes E and selects the top-h heads.
//
// The same products, in the block-score mode, reduce the affinities along the other axis
// for the HISA-style token-axis filter (MISA page, "Key distinction from HISA"):
// G[t,b] = sum_j A[t,j,b] = sum_j w[t,j] * ReLU(q[t,j] . kp_b), one value per block of
// the query's prefix, written straight to G (one CTA per chunk and query).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

namespace cg = cooperative_groups;

constexpr int kCh = kRouteChunk;
constexpr int kMaxCluster = 16;  // CTAs per query row (16: non-portable, where it fits)
constexpr int kPortableCluster = 8;

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

// 4 warps per CTA; warp w takes the 16-head row tiles w, w+4 (of ceil(H/16)).  The
// contraction S[j, b] = q_j . kp_b runs as mma.sync m16n8k16 with bf16 operands and fp32
// accumulators: A = the query's head vectors (bf16 as given), B = a chunk's pooled keys
// split into bf16 hi + lo (hi = bf16(kp), lo = bf16(kp - hi)), so the two products
// reproduce the fp32 pooled key to about 2^-16 relative.  Operands sit in shared memory as
// rows of 128 bf16 padded by 16 bytes (fragment loads conflict-free).
constexpr int kRouteThreads = 128;
constexpr int kRowPad = kHeadDim + 8;   // bf16 elements per padded shared row
constexpr int kNT = kCh / 8;            // 8-column MMA tiles per chunk

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

template <int MT>
constexpr size_t route_smem_bytes() {
  return (size_t)(16 * 4 * MT + 2 * kCh) * kRowPad * sizeof(uint16_t);
}

// The query's head vectors into qs (16-byte copies; rows past H are zero).
template <int MT>
__device__ __forceinline__ void stage_q(uint16_t* qs, const uint16_t* q, int64_t row, int H) {
  const int tid = threadIdx.x;
  constexpr int kQPer = 16 * 4 * MT * (kHeadDim / 8) / kRouteThreads;
  uint4 qv[kQPer];
#pragma unroll
  for (int i = 0; i < kQPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int j = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    qv[i] = j < H ? reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim)[c]
                  : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kQPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int j = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    *reinterpret_cast<uint4*>(qs + j * kRowPad + c * 8) = qv[i];
  }
}

// Blocks [b0, b0 + nb) of the prefix's pooled keys into khi / klo: full blocks (b < Mfull)
// from k_pool, the partial block (b = Mfull, when inside the chunk) as the mean of keys
// Mfull*B .. P-1, the rest zero.  Starts and ends with a barrier of the CTA.
__device__ __forceinline__ void stage_chunk(uint16_t* khi, uint16_t* klo, float* kpart,
                                            const float* k_pool, const uint16_t* k, int64_t n,
                                            int64_t L, int B, int Mpool, int P, int b0, int nb) {
  const int tid = threadIdx.x;
  const int M = (P + B - 1) / B, Mfull = P / B;
  const bool has_part = Mfull < M && Mfull >= b0 && Mfull < b0 + nb;
  __syncthreads();   // the previous chunk's operands are no longer read
  if (has_part) {
    const int s0 = Mfull * B, cnt = P - s0;
    const uint16_t* kr = k + ((int64_t)n * L + s0) * kHeadDim + tid;
    float a = 0.f;
    for (int s = 0; s < cnt; ++s) a += bf16_to_f32(kr[(int64_t)s * kHeadDim]);
    kpart[tid] = a / (float)cnt;
  }
  constexpr int kKPer = kCh * (kHeadDim / 4) / kRouteThreads;
  float4 kv[kKPer];
#pragma unroll
  for (int i = 0; i < kKPer; ++i) {
    const int e = tid + i * kRouteThreads;
    const int bb = e / (kHeadDim / 4), c = e % (kHeadDim / 4);
    const int b = b0 + bb;
    kv[i] = (bb < nb && b < Mfull)
                ? reinterpret_cast<const float4*>(k_pool + ((int64_t)n * Mpool + b) * kHeadDim)[c]
                : make_float4(0.f, 0.f, 0.f, 0.f);
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
}

// S = Q K^T for the staged chunk; thread (g = lane/4, c = lane%4) holds rows g, g+8 and
// columns 2c, 2c+1 of every 16 x 8 tile.
template <int MT>
__device__ __forceinline__ void chunk_products(const uint16_t* qs, const uint16_t* khi,
                                               const uint16_t* klo, float (&acc)[MT][kNT][4]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c4 = lane & 3;
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
}

// Head energies: grid (CS, query rows), clusters of CS CTAs along x (one per query row).
template <int MT>   // MT: 16-head row tiles per warp (ceil(ceil(H/16) / 4))
__global__ void __launch_bounds__(kRouteThreads) route_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const float* __restrict__ k_pool, const int32_t* __restrict__ pos, int T, int H,
    int64_t L, int B, int Mpool, int* status, int64_t row0, const float* __restrict__ w, int h,
    int32_t* __restrict__ heads, float* __restrict__ E) {
  pdl_prologue();
  extern __shared__ __align__(16) uint16_t rsm[];
  uint16_t* qs = rsm;                                  // [16 * 4 * MT][kRowPad] bf16
  uint16_t* khi = qs + 16 * 4 * MT * kRowPad;          // [kCh][kRowPad]
  uint16_t* klo = khi + kCh * kRowPad;                 // [kCh][kRowPad]
  __shared__ float kpart[kHeadDim];                    // partial block's pooled key
  __shared__ float rsum[MISA_MAX_HEADS];               // this CTA's sum_b ReLU(q_j . kp_b)
  __shared__ float ev[MISA_MAX_HEADS];
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks(), crank = (int)cluster.block_rank();
  const int64_t row = row0 + blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = prefix_len(pos, row, L, crank == 0 && tid == 0 ? status : nullptr);
  const int M = (P + B - 1) / B;
  const int64_t n = row / T;
  rsum[tid] = 0.f;   // kRouteThreads == MISA_MAX_HEADS
  stage_q<MT>(qs, q, row, H);
  const int g = lane >> 2, c4 = lane & 3;
  for (int c = crank; c * kCh < M; c += CS) {
    const int b0 = c * kCh, nb = min(b0 + kCh, M) - b0;
    stage_chunk(khi, klo, kpart, k_pool, k, n, L, B, Mpool, P, b0, nb);
    float acc[MT][kNT][4];
    chunk_products<MT>(qs, khi, klo, acc);
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
      if (c4 == 0) {   // each (warp, tile, g) owns its two heads
        rsum[r0 + g] += s_lo;
        rsum[r0 + g + 8] += s_hi;
      }
    }
  }
  cluster.sync();   // every member's sums are complete
  if (crank == 0) {
    // E[j] = |w_j| / M * the cluster's sums, then the top-h heads
    for (int j = tid; j < H; j += kRouteThreads) {
      float tot = 0.f;
      for (int r = 0; r < CS; ++r) tot += cluster.map_shared_rank(rsum, r)[j];
      const float v = fabsf(w[row * H + j]) * tot / (float)M;
      ev[j] = v;
      if (E) E[row * H + j] = v;
    }
    __syncthreads();
    if (tid < 32) select_top_h(ev, H, h, heads + row * h);
  }
  cluster.sync();   // no member leaves while CTA 0 still reads its sums
}

// Block scores for the HISA-style filter: grid (chunks, query rows), one chunk per CTA;
// G[row, b] = sum_j w_j * ReLU(q_j . kp_b) for the chunk's blocks (row stride Mpool), and
// last_block[row] = M_t - 1.
template <int MT>
__global__ void __launch_bounds__(kRouteThreads) block_score_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const float* __restrict__ k_pool, const int32_t* __restrict__ pos, int T, int H,
    int64_t L, int B, int Mpool, float* __restrict__ G, int* status, int64_t row0,
    const float* __restrict__ w, int32_t* __restrict__ last_block) {
  pdl_prologue();
  extern __shared__ __align__(16) uint16_t rsm[];
  uint16_t* qs = rsm;
  uint16_t* khi = qs + 16 * 4 * MT * kRowPad;
  uint16_t* klo = khi + kCh * kRowPad;
  __shared__ float kpart[kHeadDim];
  __shared__ float red[kRouteThreads / 32][32];
  const int64_t row = row0 + blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = prefix_len(pos, row, L, chunk == 0 && tid == 0 ? status : nullptr);
  const int M = (P + B - 1) / B;
  if (chunk == 0 && tid == 0) last_block[row] = M - 1;
  const int b0 = chunk * kCh;
  if (b0 >= M) return;
  const int nb = min(b0 + kCh, M) - b0;
  stage_q<MT>(qs, q, row, H);
  stage_chunk(khi, klo, kpart, k_pool, k, row / T, L, B, Mpool, P, b0, nb);
  float acc[MT][kNT][4];
  chunk_products<MT>(qs, khi, klo, acc);
  // this thread's heads (rows g, g + 8 of each of its tiles), then the 8 lanes sharing its
  // columns, then the 4 warps
  const int g = lane >> 2, c4 = lane & 3;
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
    G[row * Mpool + b0 + tid] = v;
  }
}

template <int MT>
cudaError_t launch_route_mt(const uint16_t* q, const float* w, const uint16_t* k,
                            const float* k_pool, const int32_t* pos, int rows, int T, int H,
                            int64_t L, int B, int h, int32_t* heads, float* E, int* status,
                            cudaStream_t st) {
  const int Mpool = (int)((L + B - 1) / B);
  const int nchunk = (Mpool + kCh - 1) / kCh;
  // 16 CTAs per row only for few rows (else the extra members cost more than they share)
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cap = (int64_t)rows * kMaxCluster <= 4LL * sms ? kMaxCluster : kPortableCluster;
  int CS = nchunk < cap ? nchunk : cap;
  const size_t smem = route_smem_bytes<MT>();
  cudaError_t err = cudaFuncSetAttribute(route_kernel<MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (CS > kPortableCluster) {
    // clusters of more than 8 CTAs only where the device can hold one
    int nclusters = 0;
    cudaLaunchConfig_t q16 = {};
    q16.gridDim = dim3((unsigned)CS, 1, 1);
    q16.blockDim = dim3(kRouteThreads, 1, 1);
    q16.dynamicSmemBytes = smem;
    cudaLaunchAttribute a16[1];
    a16[0].id = cudaLaunchAttributeClusterDimension;
    a16[0].val.clusterDim.x = (unsigned)CS;
    a16[0].val.clusterDim.y = 1;
    a16[0].val.clusterDim.z = 1;
    q16.attrs = a16;
    q16.numAttrs = 1;
    if (cudaFuncSetAttribute(route_kernel<MT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&nclusters, route_kernel<MT>, &q16) != cudaSuccess ||
        nclusters < 1) {
      cudaGetLastError();
      CS = kPortableCluster;
    }
  }
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)CS, (unsigned)nr, 1);
    cfg.blockDim = dim3(kRouteThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    err = cudaLaunchKernelEx(&cfg, route_kernel<MT>, q, k, k_pool, pos, T, H, L, B, Mpool, status,
                             row0, w, h, heads, E);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

template <int MT>
cudaError_t launch_block_scores_mt(const uint16_t* q, const float* w, const uint16_t* k,
                                   const float* k_pool, const int32_t* pos, int rows, int T,
                                   int H, int64_t L, int B, float* G, int32_t* last_block,
                                   int* status, cudaStream_t st) {
  const int Mpool = (int)((L + B - 1) / B);
  const int nchunk = (Mpool + kCh - 1) / kCh;
  const size_t smem = route_smem_bytes<MT>();
  cudaError_t err = cudaFuncSetAttribute(block_score_kernel<MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    err = launch_pdl(block_score_kernel<MT>, dim3(nchunk, (unsigned)nr), dim3(kRouteThreads), smem,
                     st, q, k, k_pool, pos, T, H, L, B, Mpool, G, status, row0, w, last_block);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_route(const uint16_t* q, const float* w, const uint16_t* k,
                         const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                         int64_t L, int B, int h, int32_t* heads, float* E, int* status,
                         cudaStream_t st) {
  const int rows = nseq * T;
  if (H <= 64)
    return launch_route_mt<1>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, status, st);
  return launch_route_mt<2>(q, w, k, k_pool, pos, rows, T, H, L, B, h, heads, E, status, st);
}

cudaError_t launch_block_scores(const uint16_t* q, const float* w, const uint16_t* k,
                                const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                                int64_t L, int B, float* G, int32_t* last_block, int* status,
                                cudaStream_t st) {
  const int rows = nseq * T;
  if (H <= 64)
    return launch_block_scores_mt<1>(q, w, k, k_pool, pos, rows, T, H, L, B, G, last_block,
                                     status, st);
  return launch_block_scores_mt<2>(q, w, k, k_pool, pos, rows, T, H, L, B, G, last_block, status,
                                   st);
}

}  // namespace misa
