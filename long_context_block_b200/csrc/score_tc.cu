// K4 (tensor-core form): indexer token scores on tcgen05 for rows that each stream their
// own prefix of keys (decode: one query per sequence).
//
//   routed (Eq. 9):  Ihat[t,s] = sum_{r < h} w[t,H_t[r]] * ReLU(q[t,H_t[r]] . k[s])
//   dense  (Eq. 1):  I[t,s]    = sum_{j < H} w[t,j]      * ReLU(q[t,j] . k[s])
//
// Per 128-key tile the contraction S[s, r] = k[s] . q_r is one tcgen05 MMA chain
// (M = 128 keys, N = the row's head count padded to a multiple of 16, K = 128 in
// eight K = 16 steps) with both operands in shared memory and the fp32 result in TMEM.
// The operation is HBM-bound (256 bytes of keys per token against 2*N*128 flops), so
// the kernel is built around the key stream:
//
//   warp 0     TMA producer: a ring of kStages 32 KB key tiles (two 64-column boxes,
//              128-byte swizzle) plus a double-buffered tile of the row's gathered q;
//   warp 1     MMA issuer (one thread) and TMEM owner;
//   warps 2-5  epilogue: tcgen05.ld of the thread's key row (TMEM lane), then the fused
//              ReLU, w-weighting and head sum, and one coalesced fp32 store per key.
//
// The grid is persistent (one CTA per SM); the rows' key tiles are laid end to end and
// every CTA takes a contiguous range of them, so long and short rows balance.  Every
// wait is bounded: on expiry the kernel records MISA_ERR_DEVICE_TIMEOUT, lets its
// in-flight copies and MMAs finish, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace misa {
namespace {

using namespace sm100;

constexpr int kTileKeys = 128;
constexpr int kKeyTileBytes = kTileKeys * kHeadDim * 2;   // 32 KB
constexpr int kKeyHalfBytes = kKeyTileBytes / 2;           // [128 rows][64 cols] bf16
constexpr int kThreads = 192;
constexpr long long kWaitCycles = 4000000000LL;            // ~2 s at the top SM clock

template <int N>
struct DecodeCfg {
  static constexpr int kStages = N <= 16 ? 6 : (N <= 64 ? 5 : 4);
  static constexpr int kAcc = N <= 32 ? 8 : (N <= 64 ? 4 : 2);
  // accumulator buffers start on power-of-two column offsets
  static constexpr int kAccStride = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : 128;
  static constexpr int kCols = (kAcc * kAccStride) <= 32 ? 32 : (kAcc * kAccStride) <= 64 ? 64
                               : (kAcc * kAccStride) <= 128 ? 128 : 256;
  static constexpr int kQBytes = N * kHeadDim * 2;
  static constexpr int kQHalf = kQBytes / 2;
  static constexpr int kStageBase = 0;
  static constexpr int kQBase = kStages * kKeyTileBytes;
  static constexpr int kBarBase = kQBase + 2 * kQBytes;
  // full[S], empty[S], qfull[2], qempty[2], accfull[A], accempty[A], drain
  static constexpr int kNumBars = 2 * kStages + 4 + 2 * kAcc + 1;
  static constexpr int kMiscBase = kBarBase + kNumBars * 8;
  static constexpr int kHistBase = kMiscBase + 16;            // [kScoreHistBins] u32
  static constexpr int kSmemBytes = kHistBase + kScoreHistBins * 4 + 1024;   // + alignment slack
  static_assert(N % 16 == 0 && N >= 16 && N <= 128, "N");
  static_assert(kQHalf % 1024 == 0, "q half tile must keep the 1 KB swizzle alignment");
};

// Row segment of a CTA's tile range: row r contributes its local tiles [a, b).
struct Seg {
  int r, a, b;
};

__device__ __forceinline__ int find_row(const int32_t* off, int rows, int t) {
  int lo = 0, hi = rows - 1;   // largest r with off[r] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool next_seg(const int32_t* off, int rows, int t0, int t1, int& r,
                                         Seg& s) {
  if (r >= rows) return false;
  const int o0 = off[r], o1 = off[r + 1];
  if (o0 >= t1) return false;
  s.r = r;
  s.a = max(t0, o0) - o0;
  s.b = min(t1, o1) - o0;
  ++r;
  return true;
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, status, kWaitCycles);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Bounded wait used while shutting down: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  volatile int never = 0;
  mbar_wait(bar, parity, &never, status, kWaitCycles);
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1) score_tc_decode_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
    const float* __restrict__ wsel, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ tile_off, int rows, int T, int64_t L, float* __restrict__ out,
    int64_t out_stride, int* status, uint32_t* __restrict__ hist) {
  using C = DecodeCfg<N>;
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int total = tile_off[rows];
  const int t0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
  const int t1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
  if (t0 >= t1) return;

  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::kBarBase);
  uint64_t* full = bars;
  uint64_t* empty = full + C::kStages;
  uint64_t* qfull = empty + C::kStages;
  uint64_t* qempty = qfull + 2;
  uint64_t* accfull = qempty + 2;
  uint64_t* accempty = accfull + C::kAcc;
  uint64_t* drain = accempty + C::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::kMiscBase);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + C::kMiscBase + 4);
  uint32_t* shist = reinterpret_cast<uint32_t*>(base + C::kHistBase);
  if (hist)
    for (int b = tid; b < kScoreHistBins; b += kThreads) shist[b] = 0;

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&qfull[s], 1); mbar_init(&qempty[s], 1); }
    for (int a = 0; a < C::kAcc; ++a) { mbar_init(&accfull[a], 1); mbar_init(&accempty[a], 128); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int r_first = find_row(tile_off, rows, t0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0, qissued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_q);
      int r = r_first;
      Seg sg;
      bool ok = true;
      while (ok && next_seg(tile_off, rows, t0, t1, r, sg)) {
        const int slot = qissued & 1;
        if (!mbar_wait(&qempty[slot], ((qissued >> 1) & 1) ^ 1, abort_flag, status, kWaitCycles))
          break;
        uint8_t* qb = base + C::kQBase + slot * C::kQBytes;
        mbar_arrive_expect_tx(&qfull[slot], C::kQBytes);
        tma_load_2d(qb, &tm_q, &qfull[slot], 0, sg.r * N);
        tma_load_2d(qb + C::kQHalf, &tm_q, &qfull[slot], 64, sg.r * N);
        ++qissued;
        const int64_t y0 = (int64_t)(sg.r / T) * L;
        for (int j = sg.a; j < sg.b; ++j) {
          const int s = issued % C::kStages;
          if (!mbar_wait(&empty[s], ((issued / C::kStages) & 1) ^ 1, abort_flag, status,
                         kWaitCycles)) {
            ok = false;
            break;
          }
          uint8_t* kb = base + C::kStageBase + s * kKeyTileBytes;
          mbar_arrive_expect_tx(&full[s], kKeyTileBytes);
          const int32_t y = (int32_t)(y0 + (int64_t)j * kTileKeys);
          tma_load_2d(kb, &tm_k, &full[s], 0, y);
          tma_load_2d(kb + kKeyHalfBytes, &tm_k, &full[s], 64, y);
          ++issued;
        }
      }
    }
    __syncthreads();   // (A) every role has left its loop
    if (lane == 0) {   // let this CTA's own copies land before the CTA exits
      for (int i = max(0, issued - C::kStages); i < issued; ++i)
        drain_wait(&full[i % C::kStages], (i / C::kStages) & 1, status);
      for (int i = max(0, qissued - 2); i < qissued; ++i) drain_wait(&qfull[i & 1], (i >> 1) & 1, status);
    }
    __syncthreads();   // (B)
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, N);
      const uint32_t smem0 = smem_u32(base);
      int it = 0, acc_it = 0, seg = 0;
      int r = r_first;
      Seg sg;
      bool ok = true;
      while (ok && next_seg(tile_off, rows, t0, t1, r, sg)) {
        const int slot = seg & 1;
        if (!mbar_wait(&qfull[slot], (seg >> 1) & 1, abort_flag, status, kWaitCycles)) break;
        const uint32_t qaddr = smem0 + C::kQBase + slot * C::kQBytes;
        for (int j = sg.a; j < sg.b; ++j) {
          const int s = it % C::kStages;
          const int acc = acc_it % C::kAcc;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1, abort_flag, status, kWaitCycles) ||
              !mbar_wait(&accempty[acc], ((acc_it / C::kAcc) & 1) ^ 1, abort_flag, status,
                         kWaitCycles)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kaddr = smem0 + C::kStageBase + s * kKeyTileBytes;
          const uint32_t d = tmem_base + (uint32_t)(acc * C::kAccStride);
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk) {
            const uint32_t ao = (kk >> 2) * kKeyHalfBytes + (kk & 3) * 32;
            const uint32_t bo = (kk >> 2) * C::kQHalf + (kk & 3) * 32;
            mma_bf16(d, desc_kmajor_sw128(kaddr + ao), desc_kmajor_sw128(qaddr + bo), idesc,
                     kk > 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          mma_commit(&accfull[acc]);
          ++it;
          ++acc_it;
        }
        if (ok) mma_commit(&qempty[slot]);
        ++seg;
      }
      mma_commit(drain);   // completes once every MMA issued above has completed
      drain_wait(drain, 0, status);
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kCols);
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;   // TMEM lanes this warp may read
    const int key_in_tile = quarter * 32 + lane;
    const int etid = tid - 64;      // 0..127 over the four epilogue warps
    int acc_it = 0;
    int r = r_first;
    Seg sg;
    bool ok = true;
    while (ok && next_seg(tile_off, rows, t0, t1, r, sg)) {
      const int P = prefix_len(pos, sg.r, L, nullptr);
      float wv[N];
#pragma unroll
      for (int c = 0; c < N; ++c) wv[c] = __ldg(wsel + (int64_t)sg.r * N + c);
      float* orow = out + (int64_t)sg.r * out_stride;
      for (int j = sg.a; j < sg.b; ++j) {
        const int acc = acc_it % C::kAcc;
        if (!warp_wait(&accfull[acc], (acc_it / C::kAcc) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * C::kAccStride);
        float sc = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < N; c0 += 16) {
          float v[16];
          tmem_ld16(taddr + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) sc = fmaf(wv[c0 + i], fmaxf(v[i], 0.f), sc);
        }
        tc_fence_before();
        mbar_arrive(&accempty[acc]);
        const int s = j * kTileKeys + key_in_tile;
        if (s < P) {
          orow[s] = sc;
          if (hist) atomicAdd(&shist[score_key(sc) >> (32 - kScoreHistBits)], 1u);
        }
        ++acc_it;
      }
      if (hist) {
        // flush this row's histogram; the four epilogue warps are always in the same
        // segment here, and leave together (the abort flag is read after the barrier)
        asm volatile("bar.sync 1, 128;" ::: "memory");
        uint32_t* gh = hist + (int64_t)sg.r * kScoreHistBins;
        for (int b = etid; b < kScoreHistBins; b += 128) {
          const uint32_t v = shist[b];
          if (v) { atomicAdd(gh + b, v); shist[b] = 0; }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        ok = *abort_flag == 0;
      }
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
  }
}

// Gather the row's head vectors (routed heads, or all heads) into a zero-padded
// [rows, N, 128] bf16 operand and their weights into [rows, N]; block 0 also lays the
// rows' key tiles end to end (tile_off[r] = tiles of rows < r).
__global__ void __launch_bounds__(1024) score_tc_prep_kernel(
    const uint16_t* __restrict__ q, const float* __restrict__ w, const int32_t* __restrict__ heads,
    int hsel, int H, int N, const int32_t* __restrict__ pos, int rows, int64_t L,
    uint4* __restrict__ qg, float* __restrict__ wg, int32_t* __restrict__ tile_off, int* status) {
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nh = heads ? hsel : H;
  for (int e = tid; e < N * 16; e += blockDim.x) {
    const int r = e >> 4, c = e & 15;
    int j = -1;
    if (r < nh) {
      j = heads ? heads[row * hsel + r] : r;
      if (j < 0 || j >= H) {
        if (c == 0) set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
        j = -1;
      }
    }
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j >= 0) v = reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim)[c];
    qg[(row * N + r) * 16 + c] = v;
    if (c == 0) wg[row * N + r] = j >= 0 ? w[row * H + j] : 0.f;
  }
  if (blockIdx.x == 0) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < rows; base += blockDim.x) {
      const int rr = base + tid;
      int v = 0;
      if (rr < rows) {
        const int P = prefix_len(pos, rr, L, status);
        v = (P + kTileKeys - 1) / kTileKeys;
      }
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if ((tid & 31) >= o) incl += t;
      }
      if ((tid & 31) == 31) warp_tot[tid >> 5] = incl;
      __syncthreads();
      if (tid < 32) {
        int x = warp_tot[tid];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, x, o);
          if (tid >= o) x += t;
        }
        warp_tot[tid] = x;
      }
      __syncthreads();
      const int excl = carry + (tid >= 32 ? warp_tot[(tid >> 5) - 1] : 0) + incl - v;
      if (rr < rows) tile_off[rr] = excl;
      __syncthreads();
      if (tid == blockDim.x - 1) carry = excl + v;
      __syncthreads();
    }
    if (tid == 0) tile_off[rows] = carry;
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
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// 2-D bf16 map over a [rows, 128] row-major matrix, box = 64 columns x box_rows rows,
// 128-byte swizzle.
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

template <int N>
cudaError_t launch_n(const CUtensorMap& tk, const CUtensorMap& tq, const float* wg,
                     const int32_t* pos, const int32_t* tile_off, int rows, int T, int64_t L,
                     float* out, int64_t out_stride, int* status, uint32_t* hist,
                     cudaStream_t st) {
  using C = DecodeCfg<N>;
  cudaError_t e = cudaFuncSetAttribute(score_tc_decode_kernel<N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  score_tc_decode_kernel<N><<<sms, kThreads, C::kSmemBytes, st>>>(
      tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist);
  return cudaGetLastError();
}

}  // namespace

int score_tc_padded_heads(int nh) { return ((nh + 15) / 16) * 16; }

size_t score_tc_ws_bytes(int64_t rows, int nh) {
  const int64_t N = score_tc_padded_heads(nh);
  return align256((size_t)rows * N * kHeadDim * 2) + align256((size_t)rows * N * 4) +
         align256((size_t)(rows + 1) * 4);
}

bool score_tc_supported(int nseq, int T, int nh, int64_t L) {
  const int64_t rows = (int64_t)nseq * T;
  const int64_t tiles = rows * ((L + kTileKeys - 1) / kTileKeys);
  return nh >= 1 && nh <= 128 && (int64_t)nseq * L < INT32_MAX && tiles < INT32_MAX &&
         rows * score_tc_padded_heads(nh) < INT32_MAX && encode_fn() != nullptr;
}

cudaError_t launch_score_tc(const uint16_t* q, const float* w, const uint16_t* k,
                            const int32_t* heads, int hsel, const int32_t* pos, int nseq, int T,
                            int H, int64_t L, float* out, int64_t out_stride, void* scratch,
                            int* status, uint32_t* hist, cudaStream_t st) {
  const int rows = nseq * T;
  const int nh = heads ? hsel : H;
  const int N = score_tc_padded_heads(nh);
  char* p = reinterpret_cast<char*>(scratch);
  uint4* qg = reinterpret_cast<uint4*>(p);
  p += align256((size_t)rows * N * kHeadDim * 2);
  float* wg = reinterpret_cast<float*>(p);
  p += align256((size_t)rows * N * 4);
  int32_t* tile_off = reinterpret_cast<int32_t*>(p);

  score_tc_prep_kernel<<<rows, 1024, 0, st>>>(q, w, heads, hsel, H, N, pos, rows, L, qg, wg,
                                              tile_off, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tk, tq;
  if (!make_map(&tk, k, (uint64_t)nseq * L, kTileKeys) ||
      !make_map(&tq, qg, (uint64_t)rows * N, (uint32_t)N))
    return cudaErrorInvalidValue;
  switch (N) {
    case 16: return launch_n<16>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 32: return launch_n<32>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 48: return launch_n<48>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 64: return launch_n<64>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 80: return launch_n<80>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 96: return launch_n<96>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 112: return launch_n<112>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    case 128: return launch_n<128>(tk, tq, wg, pos, tile_off, rows, T, L, out, out_stride, status, hist, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace misa
