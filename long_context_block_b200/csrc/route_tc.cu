// K2 (tensor-core form): the block-pooled router, Eqs. (7)-(8) of the MISA paper summary
// (Methodology section 1), for sequences with many queries (prefill):
//
//   E[t,j] = |w[t,j]| / M_t * ( sum_{b < Mfull_t} ReLU(q[t,j] . kp_b) + ReLU(q[t,j] . kpart_t) )
//
// where Mfull_t = floor(P_t / B) full blocks come from the pooled keys and kpart_t, the
// mean of the keys of query t's partial last block (present when P_t mod B != 0), is
// added on CUDA cores.  The full-block part is a GEMM: A = the (query, head) rows of q
// (128 rows = 128 / H queries per tile, streamed by TMA), B = the sequence's pooled keys
// (up to 256 blocks, resident in shared memory).  Pooled keys are fp32; they are split
// into bf16 hi + lo (hi = bf16(kp), lo = bf16(kp - hi)) so that two bf16 MMAs reproduce
// the fp32 products to about 2^-16 relative.  Accumulators live in TMEM (N = the tile's
// largest full-block count, rounded up to 16); the epilogue masks each row's columns to
// its own causal block count, adds the partial block and writes E.  The top-h selection
// runs afterwards, one warp per query.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace misa {
namespace {

using namespace sm100;

constexpr int kRows = 128;                          // (query, head) rows per tile
constexpr int kATileBytes = kRows * kHeadDim * 2;   // 32 KB
constexpr int kAHalf = kATileBytes / 2;
constexpr int kMaxBlocks = 256;                     // pooled keys held for one sequence
constexpr int kBBytes = kMaxBlocks * kHeadDim * 2;  // 64 KB per part (hi or lo)
constexpr int kBHalf = kBBytes / 2;
constexpr int kStages = 2;
constexpr int kAcc = 2;
constexpr int kCols = 512;
constexpr int kThreads = 192;
constexpr long long kWaitCycles = 4000000000LL;

constexpr int kStageBase = 0;
constexpr int kBBase = kStages * kATileBytes;         // hi then lo
constexpr int kBarBase = kBBase + 2 * kBBytes;
// full[S], empty[S], bfull, bempty, accfull[A], accempty[A], drain
constexpr int kNumBars = 2 * kStages + 2 + 2 * kAcc + 1;
constexpr int kMiscBase = kBarBase + kNumBars * 8;
constexpr int kSmemBytes = kMiscBase + 16 + 1024;

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  volatile int never = 0;
  mbar_wait(bar, parity, &never, status, kWaitCycles);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, status, kWaitCycles);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

struct RouteGeo {
  int T, H, B, QT;   // queries per sequence, heads, block size, queries per tile
  int64_t L;
  int tiles_per_seq;
};

// Largest full-block count among the queries of tile i (0 .. 256).
__device__ __forceinline__ int tile_blocks(const int32_t* pos, const RouteGeo& g, int i) {
  const int n = i / g.tiles_per_seq;
  const int ta = (i % g.tiles_per_seq) * g.QT;
  int mf = 0;
  for (int qq = 0; qq < g.QT && ta + qq < g.T; ++qq)
    mf = max(mf, prefix_len(pos, (int64_t)n * g.T + ta + qq, g.L, nullptr) / g.B);
  return min(mf, kMaxBlocks);
}

__global__ void __launch_bounds__(kThreads, 1) route_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_hi,
    const __grid_constant__ CUtensorMap tm_lo, const uint16_t* __restrict__ q,
    const float* __restrict__ w, const float* __restrict__ kpart, const int32_t* __restrict__ pos,
    RouteGeo g, int total_tiles, float* __restrict__ E, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = (int)((int64_t)total_tiles * blockIdx.x / gridDim.x);
  const int t1 = (int)((int64_t)total_tiles * (blockIdx.x + 1) / gridDim.x);
  if (t0 >= t1) return;
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kBarBase);
  uint64_t* empty = full + kStages;
  uint64_t* bfull = empty + kStages;
  uint64_t* bempty = bfull + 1;
  uint64_t* accfull = bempty + 1;
  uint64_t* accempty = accfull + kAcc;
  uint64_t* drain = accempty + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kMiscBase);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kMiscBase + 4);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(bfull, 1);
    mbar_init(bempty, 1);
    for (int a = 0; a < kAcc; ++a) { mbar_init(&accfull[a], 1); mbar_init(&accempty[a], 128); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0, bissued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int cur_seq = -1;
      for (int i = t0; i < t1; ++i) {
        const int n = i / g.tiles_per_seq;
        if (n != cur_seq) {   // pooled keys of a new sequence (after the last MMAs on the old)
          if (!mbar_wait(bempty, (bissued & 1) ^ 1, abort_flag, status, kWaitCycles)) break;
          mbar_arrive_expect_tx(bfull, 2 * kBBytes);
          uint8_t* hb = base + kBBase;
          tma_load_2d(hb, &tm_hi, bfull, 0, n * kMaxBlocks);
          tma_load_2d(hb + kBHalf, &tm_hi, bfull, 64, n * kMaxBlocks);
          tma_load_2d(hb + kBBytes, &tm_lo, bfull, 0, n * kMaxBlocks);
          tma_load_2d(hb + kBBytes + kBHalf, &tm_lo, bfull, 64, n * kMaxBlocks);
          ++bissued;
          cur_seq = n;
        }
        const int s = issued % kStages;
        if (!mbar_wait(&empty[s], ((issued / kStages) & 1) ^ 1, abort_flag, status, kWaitCycles))
          break;
        uint8_t* ab = base + kStageBase + s * kATileBytes;
        mbar_arrive_expect_tx(&full[s], kATileBytes);
        tma_load_2d(ab, &tm_q, &full[s], 0, i * kRows);
        tma_load_2d(ab + kAHalf, &tm_q, &full[s], 64, i * kRows);
        ++issued;
      }
    }
    __syncthreads();   // (A)
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i)
        drain_wait(&full[i % kStages], (i / kStages) & 1, status);
      if (bissued) drain_wait(bfull, (bissued - 1) & 1, status);
    }
    __syncthreads();   // (B)
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t smem0 = smem_u32(base);
      int it = 0, bseen = 0, cur_seq = -1;
      bool ok = true;
      for (int i = t0; i < t1 && ok; ++i) {
        const int n = i / g.tiles_per_seq;
        if (n != cur_seq) {
          if (cur_seq >= 0) mma_commit(bempty);   // the old pooled keys may be replaced
          if (!mbar_wait(bfull, bseen & 1, abort_flag, status, kWaitCycles)) break;
          ++bseen;
          cur_seq = n;
        }
        const int s = it % kStages;
        const int acc = it % kAcc;
        if (!mbar_wait(&full[s], (it / kStages) & 1, abort_flag, status, kWaitCycles) ||
            !mbar_wait(&accempty[acc], ((it / kAcc) & 1) ^ 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nb = tile_blocks(pos, g, i);
        const int N = (nb + 15) & ~15;
        if (N > 0) {
          const uint32_t idesc = idesc_bf16_f32(128, N);
          const uint32_t aaddr = smem0 + kStageBase + s * kATileBytes;
          const uint32_t d = tmem_base + (uint32_t)(acc * 256);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t baddr = smem0 + kBBase + part * kBBytes;
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk) {
              const uint32_t ao = (kk >> 2) * kAHalf + (kk & 3) * 32;
              const uint32_t bo = (kk >> 2) * kBHalf + (kk & 3) * 32;
              mma_bf16(d, desc_kmajor_sw128(aaddr + ao), desc_kmajor_sw128(baddr + bo), idesc,
                       (part | kk) ? 1u : 0u);
            }
          }
        }
        mma_commit(&empty[s]);
        mma_commit(&accfull[acc]);
        ++it;
      }
      mma_commit(drain);
      drain_wait(drain, 0, status);
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
    tc_fence_after();
    tmem_dealloc(tmem_base, kCols);
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // row of the tile
    bool ok = true;
    int it = 0;
    for (int i = t0; i < t1 && ok; ++i, ++it) {
      const int acc = it % kAcc;
      if (!warp_wait(&accfull[acc], (it / kAcc) & 1, abort_flag, status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int n = i / g.tiles_per_seq;
      const int tq = (i % g.tiles_per_seq) * g.QT + r / g.H;   // query index in the sequence
      const int j = r % g.H;
      const bool valid = tq < g.T;
      const int64_t qrow = (int64_t)n * g.T + (valid ? tq : 0);
      const int P = prefix_len(pos, qrow, g.L, nullptr);
      const int mfull = min(P / g.B, kMaxBlocks);
      // warp-uniform column count (queries of a warp may differ when H < 32)
      int mwarp = mfull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mwarp = max(mwarp, __shfl_xor_sync(0xffffffffu, mwarp, o));
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * 256);
      float sum = 0.f;
      for (int c0 = 0; c0 < mwarp; c0 += 16) {
        float v[16];
        tmem_ld16(taddr + c0, v);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c0 + c < mfull) sum += fmaxf(v[c], 0.f);
      }
      tc_fence_before();
      mbar_arrive(&accempty[acc]);
      if (valid) {
        const int M = (P + g.B - 1) / g.B;
        if (M > mfull) {   // the partial last block of this prefix
          const uint4* qv = reinterpret_cast<const uint4*>(q + (qrow * g.H + j) * kHeadDim);
          const float4* kv = reinterpret_cast<const float4*>(kpart + qrow * kHeadDim);
          float dt = 0.f;
#pragma unroll 4
          for (int c = 0; c < kHeadDim / 8; ++c) {
            const uint4 x = qv[c];
            const float4 a = kv[2 * c], b = kv[2 * c + 1];
            dt = fmaf(bf16lo(x.x), a.x, dt); dt = fmaf(bf16hi(x.x), a.y, dt);
            dt = fmaf(bf16lo(x.y), a.z, dt); dt = fmaf(bf16hi(x.y), a.w, dt);
            dt = fmaf(bf16lo(x.z), b.x, dt); dt = fmaf(bf16hi(x.z), b.y, dt);
            dt = fmaf(bf16lo(x.w), b.z, dt); dt = fmaf(bf16hi(x.w), b.w, dt);
          }
          sum += fmaxf(dt, 0.f);
        }
        E[qrow * g.H + j] = fabsf(w[qrow * g.H + j]) * sum / (float)M;
      }
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
  }
}

// Pooled keys fp32 -> bf16 hi + lo, [nseq, 256, 128] each, zero rows past the sequence's
// blocks; grid = nseq * 256 blocks of 128 threads.
__global__ void route_tc_split_kernel(const float* __restrict__ k_pool, int Mpool,
                                      uint16_t* __restrict__ hi, uint16_t* __restrict__ lo) {
  const int n = blockIdx.x / kMaxBlocks, b = blockIdx.x % kMaxBlocks, d = threadIdx.x;
  const float x = b < Mpool ? k_pool[((int64_t)n * Mpool + b) * kHeadDim + d] : 0.f;
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(h));
  const int64_t o = ((int64_t)n * kMaxBlocks + b) * kHeadDim + d;
  hi[o] = __bfloat16_as_ushort(h);
  lo[o] = __bfloat16_as_ushort(l);
}

// Mean of each query's partial last block (keys Mfull*B .. P-1); grid = rows, 128 threads.
__global__ void route_tc_partial_kernel(const uint16_t* __restrict__ k, const int32_t* __restrict__ pos,
                                        int T, int64_t L, int B, float* __restrict__ kpart,
                                        int* status) {
  const int64_t row = blockIdx.x;
  const int d = threadIdx.x;
  const int P = prefix_len(pos, row, L, d == 0 ? status : nullptr);
  const int s0 = (P / B) * B, cnt = P - s0;
  float a = 0.f;
  if (cnt > 0) {
    const uint16_t* kr = k + ((row / T) * L + s0) * kHeadDim + d;
    for (int s = 0; s < cnt; ++s) a += bf16_to_f32(kr[(int64_t)s * kHeadDim]);
    a /= (float)cnt;
  }
  kpart[row * kHeadDim + d] = a;
}

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Top-h of E per query (one warp per query): descending E, ties to the lower head.
__global__ void route_tc_select_kernel(const float* __restrict__ E, int rows, int H, int h,
                                       int32_t* __restrict__ heads) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  constexpr int kPer = MISA_MAX_HEADS / 32;
  float e[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = lane + 32 * i;
    e[i] = j < H ? E[row * H + j] : -1.f;
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

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, uint64_t nrows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)nrows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool route_tc_supported(int nseq, int T, int H, int64_t L, int B) {
  if (H < 1 || H > 128 || (128 % H) != 0 || encode_fn() == nullptr) return false;
  const int QT = 128 / H;
  const int64_t Mpool = (L + B - 1) / B;
  if (Mpool > kMaxBlocks || T < 4 * QT) return false;
  if (nseq > 1 && T % QT != 0) return false;   // tiles must not straddle sequences
  return (int64_t)nseq * T * H < INT32_MAX;
}

size_t route_tc_ws_bytes(int nseq, int T, int H) {
  const size_t rows = (size_t)nseq * T;
  return 2 * align256((size_t)nseq * kMaxBlocks * kHeadDim * 2) +
         align256(rows * kHeadDim * 4) + align256(rows * H * 4);
}

cudaError_t launch_route_tc(const uint16_t* q, const float* w, const uint16_t* k,
                            const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                            int64_t L, int B, int h, int32_t* heads, float* E, void* scratch,
                            int* status, cudaStream_t st) {
  const int rows = nseq * T;
  const int Mpool = (int)((L + B - 1) / B);
  char* c = reinterpret_cast<char*>(scratch);
  uint16_t* hi = reinterpret_cast<uint16_t*>(c);
  c += align256((size_t)nseq * kMaxBlocks * kHeadDim * 2);
  uint16_t* lo = reinterpret_cast<uint16_t*>(c);
  c += align256((size_t)nseq * kMaxBlocks * kHeadDim * 2);
  float* kpart = reinterpret_cast<float*>(c);
  c += align256((size_t)rows * kHeadDim * 4);
  float* Ebuf = E ? E : reinterpret_cast<float*>(c);

  route_tc_split_kernel<<<nseq * kMaxBlocks, kHeadDim, 0, st>>>(k_pool, Mpool, hi, lo);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_tc_partial_kernel<<<rows, kHeadDim, 0, st>>>(k, pos, T, L, B, kpart, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, thi, tlo;
  if (!make_map(&tq, q, (uint64_t)rows * H, kRows) ||
      !make_map(&thi, hi, (uint64_t)nseq * kMaxBlocks, kMaxBlocks) ||
      !make_map(&tlo, lo, (uint64_t)nseq * kMaxBlocks, kMaxBlocks))
    return cudaErrorInvalidValue;
  RouteGeo g;
  g.T = T;
  g.H = H;
  g.B = B;
  g.QT = 128 / H;
  g.L = L;
  g.tiles_per_seq = (T + g.QT - 1) / g.QT;
  const int total_tiles = nseq * g.tiles_per_seq;
  e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  route_tc_kernel<<<sms, kThreads, kSmemBytes, st>>>(tq, thi, tlo, q, w, kpart, pos, g, total_tiles,
                                                     Ebuf, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_tc_select_kernel<<<(rows * 32 + 255) / 256, 256, 0, st>>>(Ebuf, rows, H, h, heads);
  return cudaGetLastError();
}

}  // namespace misa
