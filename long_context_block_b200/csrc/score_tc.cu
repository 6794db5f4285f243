// K4 (tensor-core form): indexer token scores on tcgen05.
//
//   routed (Eq. 9):  Ihat[t,s] = sum_{r < h} w[t,H_t[r]] * ReLU(q[t,H_t[r]] . k[s])
//   dense  (Eq. 1):  I[t,s]    = sum_{j < H} w[t,j]      * ReLU(q[t,j] . k[s])
//
// Work unit: QB consecutive query rows of one sequence, each with HS head slots (the
// routed heads, or all heads, zero-padded).  Their q vectors form the MMA's B operand
// (N = QB * HS rows of 128 bf16, resident in shared memory for the unit), and the
// unit's causal prefix of keys streams through as the A operand in 128-key tiles
// (M = 128), K = 128 in eight K = 16 steps, fp32 accumulators in TMEM:
//   S[s, q*HS + r] = k[s] . q_{t0+q, slot r}.
// The epilogue applies ReLU, the slot weights and the sum over a query's slots, so each
// (query, key) score leaves the SM once, as fp32.
//   * decode form (QB = 1): every row streams its own prefix; the contraction is
//     HBM-bound (256 bytes of keys per token), N = HS <= 128.
//   * block form (QB > 1): QB queries of a sequence share every key tile.  With
//     QB = 256 / HS (prefill) N = 256 and the contraction is tensor-bound, 2 * 128 *
//     256 * 128 flops per tile; a few queries (multi-token decode) take a narrower
//     block (N >= 32) and read each key once per sequence instead of once per query.
//
// Warp roles: warp 0 TMA producer (ring of 32 KB key tiles, each two 64-column boxes with
// the 128-byte swizzle; per unit the q tile and its weights); warp 1 MMA issuer (one
// thread) and TMEM owner; the epilogue warps (4 in decode form, 8 or 16 in block form) read
// their TMEM lane quarter with tcgen05.ld.  The grid is persistent (one CTA per SM); the
// units' key tiles are laid end to end and every CTA takes a contiguous range of them,
// so long and short units balance.  Every wait is bounded: on expiry the kernel records
// MISA_ERR_DEVICE_TIMEOUT, lets its in-flight copies and MMAs finish, frees TMEM and
// returns.  In decode form the epilogue can also build a per-row histogram of the score
// keys for the top-k that follows.
//
// Gather mode (MISA-dagger fine stage, Eq. 12): a row scores its own list of candidate
// tokens instead of its prefix.  Its key rows are scattered, so the producer warp copies
// them with cp.async, 16 bytes per lane and two rows per warp step, straight into the
// swizzled tile layout; each lane's arrival on the stage barrier fires when its copies
// have landed, and the MMA thread fences the async proxy before reading the tile.  (A
// TMA row gather, four rows per instruction, measured at about half this rate.)
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
constexpr long long kWaitCycles = 4000000000LL;            // ~2 s at the top SM clock
constexpr int kSmemLimit = 227 * 1024;
constexpr int kIdAhead = 4;                                 // gather ids loaded ahead (tiles)

template <int HS, int QB>
struct Cfg {
  static constexpr int N = HS * QB;
  // full-width blocks (N = 256) whose warps still cover whole queries take 16 epilogue warps
  // (64 columns each), so the epilogue keeps up with the MMA; narrower blocks take 8
  static constexpr int kEpiWarps = QB == 1 ? 4 : (HS * QB == 256 && HS <= 64 ? 16 : 8);
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kAcc = N <= 32 ? 8 : (N <= 64 ? 4 : 2);
  static constexpr int kAccStride = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  static constexpr int kCols = kAcc * kAccStride <= 32 ? 32 : kAcc * kAccStride <= 64 ? 64
                               : kAcc * kAccStride <= 128 ? 128 : kAcc * kAccStride <= 256 ? 256 : 512;
  static constexpr int kQBytes = N * kHeadDim * 2;
  static constexpr int kQHalf = kQBytes / 2;
  static constexpr int kWBytes = N * 4;
  // units are short in decode form (double-buffer the q tile), long in block form; the
  // slot weights are always double-buffered (the epilogue reads them after the MMAs)
  static constexpr int kQBufs = QB == 1 ? 2 : 1;
  static constexpr int kWBufs = 2;
  static constexpr int kHistBytes = QB == 1 ? kScoreHistBins * 4 : 0;
  static constexpr int kFixed = kQBufs * kQBytes + kWBufs * kWBytes + kHistBytes +
                                1024 /*bars, misc*/ + 1024 /*alignment*/;
  static constexpr int kStages0 = (kSmemLimit - kFixed) / kKeyTileBytes;
  static constexpr int kStages = kStages0 > 6 ? 6 : kStages0;
  static constexpr int kStageBase = 0;
  static constexpr int kQBase = kStages * kKeyTileBytes;
  static constexpr int kWBase = kQBase + kQBufs * kQBytes;
  static constexpr int kHistBase = kWBase + kWBufs * kWBytes;
  static constexpr int kBarBase = kHistBase + kHistBytes;
  // full[S], empty[S], qfull[2], qempty[2], wfull[2], wempty[2], accfull[A], accempty[A], drain
  static constexpr int kNumBars = 2 * kStages + 8 + 2 * kAcc + 1;
  static constexpr int kMiscBase = kBarBase + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscBase + 16 + 1024;
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N");
  static_assert(kQHalf % 1024 == 0, "q half tile must keep the 1 KB swizzle alignment");
  static_assert(kStages >= 3, "key ring too shallow");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

// Unit segment of a CTA's tile range: unit u contributes its local tiles [a, b); its
// first tile has the global index o.
struct Seg {
  int u, a, b, o;
};

__device__ __forceinline__ int find_unit(const int32_t* off, int units, int t) {
  int lo = 0, hi = units - 1;   // largest u with off[u] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool next_seg(const int32_t* off, int units, int t0, int t1, int& u,
                                         Seg& s) {
  if (u >= units) return false;
  const int o0 = off[u], o1 = off[u + 1];
  if (o0 >= t1) return false;
  s.u = u;
  s.o = o0;
  s.a = max(t0, o0) - o0;
  s.b = min(t1, o1) - o0;
  ++u;
  return true;
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, long long limit) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, status, limit);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Bounded wait used while shutting down: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status,
                                           long long limit) {
  volatile int never = 0;
  mbar_wait(bar, parity, &never, status, limit);
}

__device__ __forceinline__ void epi_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Geometry of the units: sequence n holds ublk = ceil(T / QB) units; unit u covers rows
// t = (u % ublk) * QB + q, q < QB, t < T.
struct Units {
  int T, QB, ublk;
  __device__ __forceinline__ int seq(int u) const { return u / ublk; }
  __device__ __forceinline__ int t0(int u) const { return (u % ublk) * QB; }
};

template <int HS, int QB, bool kGather>
__global__ void __launch_bounds__(Cfg<HS, QB>::kThreads, 1) score_tc_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
    const float* __restrict__ wsel, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ tile_off, int units, Units geo, int64_t L,
    float* __restrict__ out, int64_t out_stride, int* status, uint32_t* __restrict__ hist,
    const int32_t* __restrict__ gidx, const int32_t* __restrict__ glen,
    const uint16_t* __restrict__ kraw, WaitProbe probe) {
  pdl_prologue();
  using C = Cfg<HS, QB>;
  // bound of every wait (about 2 s normally; a test passes a short one together with a
  // key tile that is never loaded, probe.skip_tile, to make a wait run out)
  const long long kWait = probe.wait_cycles;
  constexpr int N = C::N;
  constexpr int kEpiThreads = 32 * C::kEpiWarps;
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int total = tile_off[units];
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
  uint64_t* wfull = qempty + 2;
  uint64_t* wempty = wfull + 2;
  uint64_t* accfull = wempty + 2;
  uint64_t* accempty = accfull + C::kAcc;
  uint64_t* drain = accempty + C::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::kMiscBase);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + C::kMiscBase + 4);
  uint32_t* shist = reinterpret_cast<uint32_t*>(base + C::kHistBase);
  if (QB == 1 && hist)
    for (int b = tid; b < kScoreHistBins; b += C::kThreads) shist[b] = 0;

  if (tid == 0) {
    // a gathered tile completes with one cp.async arrival per producer lane
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], kGather ? 32 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::kQBufs; ++s) { mbar_init(&qfull[s], 1); mbar_init(&qempty[s], 1); }
    for (int s = 0; s < C::kWBufs; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], C::kEpiWarps);   // one arrival per epilogue warp
    }
    for (int a = 0; a < C::kAcc; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], kEpiThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int u_first = find_unit(tile_off, units, t0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0, qissued = 0, wissued = 0;
    if constexpr (!kGather) {
      // lane 0 streams each unit's q tile, weights and prefix key tiles by TMA
      if (lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
        int u = u_first;
        Seg sg;
        bool ok = true;
        while (ok && next_seg(tile_off, units, t0, t1, u, sg)) {
          const int slot = qissued % C::kQBufs;
          if (!mbar_wait(&qempty[slot], ((qissued / C::kQBufs) & 1) ^ 1, abort_flag, status,
                         kWait))
            break;
          uint8_t* qb = base + C::kQBase + slot * C::kQBytes;
          mbar_arrive_expect_tx(&qfull[slot], C::kQBytes);
          tma_load_2d(qb, &tm_q, &qfull[slot], 0, sg.u * N);
          tma_load_2d(qb + C::kQHalf, &tm_q, &qfull[slot], 64, sg.u * N);
          const int wslot = qissued % C::kWBufs;
          if (!mbar_wait(&wempty[wslot], ((qissued / C::kWBufs) & 1) ^ 1, abort_flag, status,
                         kWait)) {
            ++qissued;
            break;
          }
          mbar_arrive_expect_tx(&wfull[wslot], C::kWBytes);
          bulk_load(base + C::kWBase + wslot * C::kWBytes, wsel + (int64_t)sg.u * N, C::kWBytes,
                    &wfull[wslot]);
          ++qissued;
          ++wissued;
          const int64_t y0 = (int64_t)geo.seq(sg.u) * L;
          for (int j = sg.a; j < sg.b; ++j) {
            const int s = issued % C::kStages;
            if (!mbar_wait(&empty[s], ((issued / C::kStages) & 1) ^ 1, abort_flag, status,
                           kWait)) {
              ok = false;
              break;
            }
            if (sg.o + j == probe.skip_tile) {   // test only: this tile is never loaded
              ++issued;
              continue;
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
    } else {
      // gather mode: the whole warp walks the loop (waits are polled by lane 0 and
      // broadcast); lane 0 loads q and the weights, every lane copies key rows
      if (lane == 0) tma_prefetch_desc(&tm_q);
      int u = u_first;
      Seg sg;
      bool ok = true;
      while (ok && next_seg(tile_off, units, t0, t1, u, sg)) {
        const int slot = qissued % C::kQBufs;
        if (!warp_wait(&qempty[slot], ((qissued / C::kQBufs) & 1) ^ 1, abort_flag, status, kWait)) break;
        uint8_t* qb = base + C::kQBase + slot * C::kQBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&qfull[slot], C::kQBytes);
          tma_load_2d(qb, &tm_q, &qfull[slot], 0, sg.u * N);
          tma_load_2d(qb + C::kQHalf, &tm_q, &qfull[slot], 64, sg.u * N);
        }
        const int wslot = qissued % C::kWBufs;
        if (!warp_wait(&wempty[wslot], ((qissued / C::kWBufs) & 1) ^ 1, abort_flag, status, kWait)) {
          ++qissued;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&wfull[wslot], C::kWBytes);
          bulk_load(base + C::kWBase + wslot * C::kWBytes, wsel + (int64_t)sg.u * N, C::kWBytes,
                    &wfull[wslot]);
        }
        ++qissued;
        ++wissued;
        const int64_t y0 = (int64_t)geo.seq(sg.u) * L;
        // unit = row: its token list and length; lane l gathers keys 4l .. 4l+3 of a tile,
        // whose ids it loads kIdAhead tiles early
        const int32_t* ids = gidx + (int64_t)sg.u * out_stride;
        const int cnt = min(max(glen[sg.u], 0), (int)out_stride);
        int32_t rq[kIdAhead][4];
        auto fetch_ids = [&](int jj, int32_t(&r)[4]) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = jj * kTileKeys + 4 * lane + i;
            int32_t id = c < cnt ? ids[c] : 0;   // padding keys are masked by the epilogue
            if (id < 0 || id >= L) id = 0;
            r[i] = (int32_t)(y0 + id);
          }
        };
#pragma unroll
        for (int d = 0; d < kIdAhead; ++d)
          if (sg.a + d < sg.b) fetch_ids(sg.a + d, rq[d]);
        for (int j = sg.a; j < sg.b; ++j) {
          const int s = issued % C::kStages;
          int32_t r[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) r[i] = rq[0][i];
#pragma unroll
          for (int d = 0; d + 1 < kIdAhead; ++d)
#pragma unroll
            for (int i = 0; i < 4; ++i) rq[d][i] = rq[d + 1][i];
          if (j + kIdAhead < sg.b) fetch_ids(j + kIdAhead, rq[kIdAhead - 1]);
          if (!warp_wait(&empty[s], ((issued / C::kStages) & 1) ^ 1, abort_flag, status, kWait)) {
            ok = false;
            break;
          }
          // 64 warp-wide steps, two key rows each: lanes 0-15 copy row 2i, lanes 16-31 row
          // 2i+1, 16 bytes per lane, into the 128-byte-swizzled halves of the tile.  Row
          // 4m+e's id sits in lane m's r[e].
          const int c = lane & 15, odd = lane >> 4;
          const uint32_t kb_s = smem_u32(base + C::kStageBase + s * kKeyTileBytes) +
                                (uint32_t)((c >> 3) * kKeyHalfBytes);
#pragma unroll
          for (int i = 0; i < kTileKeys / 2; ++i) {
            const int32_t ya = __shfl_sync(0xffffffffu, r[2 * (i & 1)], i >> 1);
            const int32_t yb = __shfl_sync(0xffffffffu, r[2 * (i & 1) + 1], i >> 1);
            const int row = 2 * i + odd;
            const uint32_t dst = kb_s + (uint32_t)(row * 128) + (uint32_t)(((c & 7) ^ (row & 7)) << 4);
            cp_async16(dst, kraw + (int64_t)(odd ? yb : ya) * kHeadDim + c * 8);
          }
          cp_async_mbar_arrive(&full[s]);
          ++issued;
        }
      }
    }
    __syncthreads();   // (A) every role has left its loop
    if (lane == 0) {   // let this CTA's own copies land before the CTA exits
      for (int i = max(0, issued - C::kStages); i < issued; ++i)
        drain_wait(&full[i % C::kStages], (i / C::kStages) & 1, status, kWait);
      for (int i = max(0, qissued - C::kQBufs); i < qissued; ++i)
        drain_wait(&qfull[i % C::kQBufs], (i / C::kQBufs) & 1, status, kWait);
      for (int i = max(0, wissued - C::kWBufs); i < wissued; ++i)
        drain_wait(&wfull[i % C::kWBufs], (i / C::kWBufs) & 1, status, kWait);
    }
    __syncthreads();   // (B)
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, N);
      const uint32_t smem0 = smem_u32(base);
      int it = 0, acc_it = 0, seg = 0;
      int u = u_first;
      Seg sg;
      bool ok = true;
      while (ok && next_seg(tile_off, units, t0, t1, u, sg)) {
        const int slot = seg % C::kQBufs;
        if (!mbar_wait(&qfull[slot], (seg / C::kQBufs) & 1, abort_flag, status, kWait)) break;
        const uint32_t qaddr = smem0 + C::kQBase + slot * C::kQBytes;
        for (int j = sg.a; j < sg.b; ++j) {
          const int s = it % C::kStages;
          const int acc = acc_it % C::kAcc;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1, abort_flag, status, kWait) ||
              !mbar_wait(&accempty[acc], ((acc_it / C::kAcc) & 1) ^ 1, abort_flag, status,
                         kWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if constexpr (kGather) fence_proxy_async_smem();   // tile written by cp.async
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
      drain_wait(drain, 0, status, kWait);
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kCols);
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int kColsPerWarp = N / (C::kEpiWarps / 4);   // column share of a warp
    constexpr int kQPerWarp = QB == 1 ? 1 : kColsPerWarp / HS;
    const int e = warp - 2;
    const int quarter = warp & 3;                 // TMEM lanes this warp may read
    const int col0 = (e / 4) * kColsPerWarp;      // first accumulator column of this warp
    const int q0 = QB == 1 ? 0 : col0 / HS;       // first query of this warp in the unit
    const int key_in_tile = quarter * 32 + lane;
    const int etid = tid - 64;
    // Every epilogue warp walks the same segments and tiles whatever happens, so the
    // named barriers of the histogram flush always match; after a failed (bounded) wait a
    // warp only skips the work.
    int acc_it = 0, seg = 0;
    int u = u_first;
    Seg sg;
    bool ok = true;
    while (next_seg(tile_off, units, t0, t1, u, sg)) {
      const int n = geo.seq(sg.u);
      const int tq0 = geo.t0(sg.u);
      int P[kQPerWarp];   // prefix length of each of this warp's queries (0: no query)
#pragma unroll
      for (int q = 0; q < kQPerWarp; ++q) {
        const int t = tq0 + q0 + q;
        if constexpr (kGather)
          P[q] = t >= geo.T ? 0 : min(max(glen[sg.u], 0), (int)out_stride);
        else
          P[q] = t < geo.T ? prefix_len(pos, (int64_t)n * geo.T + t, L, nullptr) : 0;
      }
      // this warp's queries are consecutive rows of the output
      float* obase = out + ((int64_t)n * geo.T + min(tq0 + q0, geo.T - 1)) * out_stride;
      const int wslot = seg % C::kWBufs;
      if (ok && !warp_wait(&wfull[wslot], (seg / C::kWBufs) & 1, abort_flag, status, kWait)) ok = false;
      const float* wsm = reinterpret_cast<const float*>(base + C::kWBase + wslot * C::kWBytes);
      for (int j = sg.a; j < sg.b && ok; ++j) {
        const int acc = acc_it % C::kAcc;
        if (!warp_wait(&accfull[acc], (acc_it / C::kAcc) & 1, abort_flag, status, kWait)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                               (uint32_t)(acc * C::kAccStride + col0);
        float sc[kQPerWarp];
#pragma unroll
        for (int q = 0; q < kQPerWarp; ++q) sc[q] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < kColsPerWarp; c0 += 16) {
          float v[16];
          tmem_ld16(taddr + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int col = c0 + i;
            const int q = QB == 1 ? 0 : col / HS;
            sc[q] = fmaf(wsm[col0 + col], fmaxf(v[i], 0.f), sc[q]);
          }
        }
        tc_fence_before();
        mbar_arrive(&accempty[acc]);
        const int s = j * kTileKeys + key_in_tile;
#pragma unroll
        for (int q = 0; q < kQPerWarp; ++q) {
          if (s < P[q]) {
            obase[(int64_t)q * out_stride + s] = sc[q];
            if (QB == 1 && hist) atomicAdd(&shist[score_key(sc[q]) >> (32 - kScoreHistBits)], 1u);
          }
        }
        ++acc_it;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[wslot]);   // this warp is done with the weights
      if (QB == 1 && hist) {
        // flush this row's histogram (all epilogue warps are in this segment)
        epi_bar(kEpiThreads);
        uint32_t* gh = hist + (int64_t)sg.u * kScoreHistBins;
        for (int b = etid; b < kScoreHistBins; b += kEpiThreads) {
          const uint32_t v = shist[b];
          if (v) {
            if (ok) atomicAdd(gh + b, v);
            shist[b] = 0;
          }
        }
        epi_bar(kEpiThreads);
      }
      ++seg;
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
  }
}

// Gather each unit's head vectors (routed heads, or all heads) into a zero-padded
// [units, QB * HS, 128] bf16 operand and their weights into [units, QB * HS]; block 0
// also lays the units' key tiles end to end (tile_off[u] = tiles of units < u), sized by
// the causal prefix or, in gather mode, by the row's token-list length.
__global__ void __launch_bounds__(1024) score_tc_prep_kernel(
    const uint16_t* __restrict__ q, const float* __restrict__ w, const int32_t* __restrict__ heads,
    int hsel, int H, int HS, Units geo, const int32_t* __restrict__ pos, int units, int64_t L,
    const int32_t* __restrict__ glen, int gmax, uint4* __restrict__ qg, float* __restrict__ wg,
    int32_t* __restrict__ tile_off, int* status, uint4* __restrict__ zero, int64_t zero16) {
  pdl_prologue();
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  // zero the scorer's histogram scratch (zero16 16-byte words), spread over all blocks
  for (int64_t i = (int64_t)u * blockDim.x + tid; i < zero16; i += (int64_t)gridDim.x * blockDim.x)
    zero[i] = make_uint4(0, 0, 0, 0);
  const int nh = heads ? hsel : H;
  const int N = HS * geo.QB;
  const int n = geo.seq(u), tq0 = geo.t0(u);
  for (int e = tid; e < N * 16; e += blockDim.x) {
    const int col = e >> 4, c = e & 15;
    const int qq = col / HS, r = col % HS;
    const int t = tq0 + qq;
    const int64_t row = (int64_t)n * geo.T + t;
    int j = -1;
    if (t < geo.T && r < nh) {
      j = heads ? heads[row * hsel + r] : r;
      if (j < 0 || j >= H) {
        if (c == 0) set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
        j = -1;
      }
    }
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j >= 0) v = reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim)[c];
    qg[((int64_t)u * N + col) * 16 + c] = v;
    if (c == 0) wg[(int64_t)u * N + col] = j >= 0 ? w[row * H + j] : 0.f;
  }
  if (blockIdx.x == 0) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < units; base += blockDim.x) {
      const int uu = base + tid;
      int v = 0;
      if (uu < units) {
        const int nn = geo.seq(uu), ta = geo.t0(uu);
        int Pmax = 0;
        if (glen)   // gather mode: one row per unit, its token-list length
          Pmax = min(max(glen[uu], 0), gmax);
        else   // eight independent loads per step
          for (int q0 = 0; q0 < geo.QB && ta + q0 < geo.T; q0 += 8) {
            int p8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int qq = q0 + j;
              p8[j] = (qq < geo.QB && ta + qq < geo.T)
                          ? prefix_len(pos, (int64_t)nn * geo.T + ta + qq, L, status) : 0;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) Pmax = max(Pmax, p8[j]);
          }
        v = (Pmax + kTileKeys - 1) / kTileKeys;
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
      if (uu < units) tile_off[uu] = excl;
      __syncthreads();
      if (tid == blockDim.x - 1) carry = excl + v;
      __syncthreads();
    }
    if (tid == 0) tile_off[units] = carry;
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

template <int HS, int QB, bool kGather>
cudaError_t launch_cfg(const CUtensorMap& tk, const CUtensorMap& tq, const float* wg,
                       const int32_t* pos, const int32_t* tile_off, int units, Units geo,
                       int64_t L, float* out, int64_t out_stride, int* status, uint32_t* hist,
                       const int32_t* gidx, const int32_t* glen, const uint16_t* kraw,
                       const WaitProbe& probe, const KernelTimer* timer, cudaStream_t st) {
  using C = Cfg<HS, QB>;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<HS, QB, kGather>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (timer && (e = cudaEventRecord(timer->begin, st)) != cudaSuccess) return e;
  e = launch_pdl(score_tc_kernel<HS, QB, kGather>, dim3(sms), dim3(C::kThreads),
                 (size_t)C::kSmemBytes, st, tk, tq, wg, pos, tile_off, units, geo, L, out,
                 out_stride, status, hist, gidx, glen, kraw, probe);
  if (e == cudaSuccess && timer) e = cudaEventRecord(timer->end, st);
  return e;
}

// Shape of the work units for nh heads and T queries per sequence.
struct Plan {
  int HS, QB, N;
};

Plan plan_for(int nh, int T, bool gather = false) {
  Plan p;
  // Block form whenever a sequence has several queries: QB of them share every key tile.
  // Full width (N = 256) from 256 / HS queries on (prefill); a few queries (multi-token
  // decode) take the next power of two >= T, at least 32 columns, so each unit still reads
  // the sequence's keys once.  Rows with their own token lists take the decode form.
  const int hs_pow2 = nh <= 8 ? 8 : nh <= 16 ? 16 : nh <= 32 ? 32 : nh <= 64 ? 64 : 128;
  const int qb = 256 / hs_pow2;
  if (!gather && T >= 2) {
    int q = 2;
    while (q < T && q < qb) q <<= 1;
    while (q * hs_pow2 < 32) q <<= 1;
    p.HS = hs_pow2;
    p.QB = q;
  } else {
    p.HS = ((nh + 15) / 16) * 16;
    p.QB = 1;
  }
  p.N = p.HS * p.QB;
  return p;
}

}  // namespace

size_t score_tc_ws_bytes(int nseq, int T, int nh, bool gather) {
  const Plan p = plan_for(nh, T, gather);
  const int64_t units = (int64_t)nseq * ((T + p.QB - 1) / p.QB);
  return align256((size_t)units * p.N * kHeadDim * 2) + align256((size_t)units * p.N * 4) +
         align256((size_t)(units + 1) * 4);
}

bool score_tc_block_form(int nh, int T) { return plan_for(nh, T).QB > 1; }

bool score_tc_supported(int nseq, int T, int nh, int64_t L, int64_t span) {
  const Plan p = plan_for(nh, T, span > 0);
  const int64_t units = (int64_t)nseq * ((T + p.QB - 1) / p.QB);
  const int64_t tiles = units * (((span > 0 ? span : L) + kTileKeys - 1) / kTileKeys);
  return nh >= 1 && nh <= 128 && (int64_t)nseq * L < INT32_MAX && tiles < INT32_MAX &&
         units * p.N < INT32_MAX && encode_fn() != nullptr;
}

cudaError_t launch_score_tc(const uint16_t* q, const float* w, const uint16_t* k,
                            const int32_t* heads, int hsel, const int32_t* pos, int nseq, int T,
                            int H, int64_t L, float* out, int64_t out_stride, void* scratch,
                            int* status, uint32_t* hist, cudaStream_t st, const int32_t* gidx,
                            const int32_t* glen, const WaitProbe* test_probe,
                            size_t hist_zero_bytes, const KernelTimer* timer) {
  const bool gather = gidx != nullptr;
  WaitProbe probe;
  probe.wait_cycles = kWaitCycles;
  probe.skip_tile = -1;
  if (test_probe) probe = *test_probe;
  const int nh = heads ? hsel : H;
  const Plan p = plan_for(nh, T, gather);
  Units geo;
  geo.T = T;
  geo.QB = p.QB;
  geo.ublk = (T + p.QB - 1) / p.QB;
  const int units = nseq * geo.ublk;
  char* c = reinterpret_cast<char*>(scratch);
  uint4* qg = reinterpret_cast<uint4*>(c);
  c += align256((size_t)units * p.N * kHeadDim * 2);
  float* wg = reinterpret_cast<float*>(c);
  c += align256((size_t)units * p.N * 4);
  int32_t* tile_off = reinterpret_cast<int32_t*>(c);
  uint4* zero = reinterpret_cast<uint4*>(hist);   // zeroed by the prep kernel in every form
  if (p.QB > 1 || gather) hist = nullptr;         // built by the epilogue in decode form only

  cudaError_t e = launch_pdl(score_tc_prep_kernel, dim3(units), dim3(1024), 0, st, q, w, heads,
                             hsel, H, p.HS, geo, pos, units, L, glen, (int)out_stride, qg, wg,
                             tile_off, status, zero,
                             zero ? (int64_t)(hist_zero_bytes / 16) : (int64_t)0);
  if (e != cudaSuccess) return e;
  CUtensorMap tk, tq;   // (the gather copies key rows with cp.async: tk goes unused)
  if (!make_map(&tk, k, (uint64_t)nseq * L, (uint32_t)kTileKeys) ||
      !make_map(&tq, qg, (uint64_t)units * p.N, (uint32_t)p.N))
    return cudaErrorInvalidValue;
#define MISA_TC_CASE(HS_, QB_)                                                                  \
  if (p.HS == HS_ && p.QB == QB_)                                                               \
    return launch_cfg<HS_, QB_, false>(tk, tq, wg, pos, tile_off, units, geo, L, out, out_stride, \
                                       status, hist, nullptr, nullptr, k, probe, timer, st);
#define MISA_TC_GATHER_CASE(HS_)                                                                \
  if (p.HS == HS_)                                                                              \
    return launch_cfg<HS_, 1, true>(tk, tq, wg, pos, tile_off, units, geo, L, out, out_stride,    \
                                    status, nullptr, gidx, glen, k, probe, timer, st);
  if (gather) {
    MISA_TC_GATHER_CASE(16)
    MISA_TC_GATHER_CASE(32)
    MISA_TC_GATHER_CASE(48)
    MISA_TC_GATHER_CASE(64)
    MISA_TC_GATHER_CASE(80)
    MISA_TC_GATHER_CASE(96)
    MISA_TC_GATHER_CASE(112)
    MISA_TC_GATHER_CASE(128)
    return cudaErrorInvalidValue;
  }
  MISA_TC_CASE(16, 1)
  MISA_TC_CASE(32, 1)
  MISA_TC_CASE(48, 1)
  MISA_TC_CASE(64, 1)
  MISA_TC_CASE(80, 1)
  MISA_TC_CASE(96, 1)
  MISA_TC_CASE(112, 1)
  MISA_TC_CASE(128, 1)
  MISA_TC_CASE(8, 4)
  MISA_TC_CASE(8, 8)
  MISA_TC_CASE(8, 16)
  MISA_TC_CASE(8, 32)
  MISA_TC_CASE(16, 2)
  MISA_TC_CASE(16, 4)
  MISA_TC_CASE(16, 8)
  MISA_TC_CASE(16, 16)
  MISA_TC_CASE(32, 2)
  MISA_TC_CASE(32, 4)
  MISA_TC_CASE(32, 8)
  MISA_TC_CASE(64, 2)
  MISA_TC_CASE(64, 4)
  MISA_TC_CASE(128, 2)
#undef MISA_TC_CASE
#undef MISA_TC_GATHER_CASE
  return cudaErrorInvalidValue;
}

}  // namespace misa
