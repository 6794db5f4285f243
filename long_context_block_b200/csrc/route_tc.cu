// K2 (tensor-core form): the block-pooled router, Eqs. (7)-(8) of the MISA paper summary
// (Methodology section 1), for sequences with many queries (prefill):
//
//   E[t,j] = |w[t,j]| / M_t * ( sum_{b < Mfull_t} ReLU(q[t,j] . kp_b) + ReLU(q[t,j] . kpart_t) )
//   heads_t = the h largest E[t,j]  (ties: lower j)
//
// where Mfull_t = floor(P_t / B) full blocks come from the pooled keys and kpart_t, the
// mean of the keys of query t's partial last block (present when P_t mod B != 0), is
// added on CUDA cores.  The full-block part is a GEMM: A = the (query, head) rows of q
// (128 rows = 128 / H queries per tile, streamed by TMA), B = the sequence's pooled keys
// in chunks of 256 blocks (one chunk resident in shared memory at a time).  A tile makes
// one MMA item per chunk its queries reach (even tiles walk their chunks upward, odd tiles
// downward, so consecutive items mostly share the resident chunk).  Pooled keys are fp32;
// they are split into bf16 hi + lo (hi = bf16(kp), lo = bf16(kp - hi)) so that two bf16
// MMAs reproduce the fp32 products to about 2^-16 relative.  Accumulators live in TMEM
// (N = the item's largest full-block count within its chunk, rounded up to 16).
//
// Epilogue: four groups of 4 warps (one per TMEM lane quarter); group g serves the tiles
// t0 + g, t0 + g + 4, ... with its own 128-column accumulator, so four tiles' per-tile
// latency chains overlap (and the MMAs of one group's item run while the others read theirs).  Each warp owns 32 (query, head) rows of its tile: the partial-block dot
// product reads the query row from the tile's A stage (released by the epilogue, not by the
// MMA) and the tile's partial pooled keys from a shared-memory copy loaded with the A tile;
// then the row's ReLU sum over its causal block count, E (written when asked for), and a
// rank of the row's head among its query's H energies for the top-h heads.  The tile's
// per-row inputs (prefix lengths, |w|) are loaded one group tile ahead.
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
constexpr int kMaxBlocks = 256;                     // pooled keys per chunk (one resident)
constexpr int kItemBlocks = 128;                    // accumulator columns of one MMA item
constexpr int kBBytes = kMaxBlocks * kHeadDim * 2;  // 64 KB per part (hi or lo)
constexpr int kBHalf = kBBytes / 2;
constexpr int kMaxQT = 16;                          // queries per tile (H >= 8)
constexpr int kKpBytes = kMaxQT * kHeadDim * 4;     // partial pooled keys of a tile (fp32)
constexpr int kGroups = 4;                          // epilogue groups
constexpr int kStages = 2;
constexpr int kAccPerGroup = 1;
constexpr int kAcc = kGroups * kAccPerGroup;
constexpr int kCols = kAcc * kItemBlocks;           // 512
constexpr int kGroupThreads = 128;
constexpr int kEpiWarps = kGroups * 4;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;
constexpr long long kWaitCycles = 4000000000LL;

constexpr int kStageBase = 0;
constexpr int kBBase = kStages * kATileBytes;         // hi then lo
constexpr int kKpBase = kBBase + 2 * kBBytes;
constexpr int kEsBase = kKpBase + kStages * kKpBytes;  // E of a tile's rows: [group][2][kRows]
constexpr int kBarBase = kEsBase + kGroups * 2 * kRows * 4;
// full[G] (per epilogue group: a group's tiles complete its phases one by one, so its
// parity waits never alias a stage's later tile), empty[S], bfull, bempty, accfull[A],
// accempty[A], drain
constexpr int kNumBars = kGroups + kStages + 2 + 2 * kAcc + 1;
constexpr int kMiscBase = kBarBase + kNumBars * 8;
constexpr int kMetaTiles = 1024;                       // tiles whose block counts are staged
constexpr int kMetaBase = kMiscBase + 16;              // per-tile full-block counts [kMetaTiles]
constexpr int kSmemBytes = kMetaBase + kMetaTiles * 4 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kGroups % kStages == 0 && kMaxBlocks == 2 * kItemBlocks, "tile-to-group map");

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

__device__ __forceinline__ void group_bar(int grp) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(kGroupThreads) : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes: two loads, one wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "r"(taddr + 16u)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct RouteGeo {
  int T, H, B, QT;   // queries per sequence, heads, block size, queries per tile
  int64_t L;
  int tiles_per_seq;
  int mpad;          // pooled-key rows per sequence in the hi / lo copies (chunks of 256)
};

// Largest full-block count among the queries of tile i.
__device__ __forceinline__ int tile_blocks(const int32_t* pos, const RouteGeo& g, int i) {
  const int n = i / g.tiles_per_seq;
  const int ta = (i % g.tiles_per_seq) * g.QT;
  int mf = 0;
  for (int qq = 0; qq < g.QT && ta + qq < g.T; ++qq)
    mf = max(mf, prefix_len(pos, (int64_t)n * g.T + ta + qq, g.L, nullptr) / g.B);
  return mf;
}
// Chunks of pooled keys a tile whose queries reach mf full blocks visits, and the chunk of
// its k-th visit.  Inside chunk c the tile makes one MMA item per 128-block half that holds
// full blocks (item_present(c, sub, mf)); a tile without full blocks makes one empty item.
__device__ __forceinline__ int tile_items(int mf) { return max(1, (mf + kMaxBlocks - 1) / kMaxBlocks); }
__device__ __forceinline__ int item_chunk(int i, int k, int nc) { return (i & 1) ? nc - 1 - k : k; }
__device__ __forceinline__ bool item_present(int c, int sub, int mf) {
  const int b0 = c * kMaxBlocks + sub * kItemBlocks;
  return b0 < mf || (mf == 0 && b0 == 0);
}

__global__ void __launch_bounds__(kThreads, 1) route_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_hi,
    const __grid_constant__ CUtensorMap tm_lo, const float* __restrict__ w,
    const float* __restrict__ kpart, const int32_t* __restrict__ pos, RouteGeo g, int total_tiles,
    int h, int32_t* __restrict__ heads, float* __restrict__ E, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = (int)((int64_t)total_tiles * blockIdx.x / gridDim.x);
  const int t1 = (int)((int64_t)total_tiles * (blockIdx.x + 1) / gridDim.x);
  if (t0 >= t1) return;
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kBarBase);
  uint64_t* empty = full + kGroups;
  uint64_t* bfull = empty + kStages;
  uint64_t* bempty = bfull + 1;
  uint64_t* accfull = bempty + 1;
  uint64_t* accempty = accfull + kAcc;
  uint64_t* drain = accempty + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kMiscBase);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kMiscBase + 4);
  if (tid == 0) {
    for (int g2 = 0; g2 < kGroups; ++g2) mbar_init(&full[g2], 1);
    for (int s = 0; s < kStages; ++s)
      mbar_init(&empty[s], 1 + 4);   // the MMAs' commit and the serving group's warps
    mbar_init(bfull, 1);
    mbar_init(bempty, 1);
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], kGroupThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kCols);
  // Every tile's largest full-block count, loaded once by all threads (its queries' prefix
  // lengths) so that the producer and the MMA issuer do not wait on them tile by tile.
  int* meta = reinterpret_cast<int*>(base + kMetaBase);
  const bool staged = t1 - t0 <= kMetaTiles;
  if (staged)
    for (int j = tid; j < t1 - t0; j += kThreads) meta[j] = tile_blocks(pos, g, t0 + j);
  auto blocks_of = [&](int i) { return staged ? meta[i - t0] : tile_blocks(pos, g, i); };
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t kp_bytes = (uint32_t)g.QT * kHeadDim * 4;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0, bissued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int64_t cur_key = -1;   // resident chunk: sequence * 65536 + chunk
      bool ok = true;
      for (int i = t0; i < t1 && ok; ++i) {
        const int n = i / g.tiles_per_seq;
        const int s = issued % kStages;
        if (!mbar_wait(&empty[s], ((issued / kStages) & 1) ^ 1, abort_flag, status, kWaitCycles))
          break;
        uint8_t* ab = base + kStageBase + s * kATileBytes;
        const int64_t qrow0 = (int64_t)n * g.T + (int64_t)(i % g.tiles_per_seq) * g.QT;
        uint64_t* fb = &full[issued % kGroups];   // the serving group's barrier
        mbar_arrive_expect_tx(fb, kATileBytes + kp_bytes);
        tma_load_2d(ab, &tm_q, fb, 0, i * kRows);
        tma_load_2d(ab + kAHalf, &tm_q, fb, 64, i * kRows);
        bulk_load(base + kKpBase + s * kKpBytes, kpart + qrow0 * kHeadDim, kp_bytes, fb);
        ++issued;
        const int nc = tile_items(blocks_of(i));
        for (int k = 0; k < nc; ++k) {
          const int c = item_chunk(i, k, nc);
          const int64_t key = (int64_t)n * 65536 + c;
          if (key == cur_key) continue;
          // a new chunk of pooled keys, after the last MMAs on the resident one
          if (!mbar_wait(bempty, (bissued & 1) ^ 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bfull, 2 * kBBytes);
          uint8_t* hb = base + kBBase;
          const int row = n * g.mpad + c * kMaxBlocks;
          tma_load_2d(hb, &tm_hi, bfull, 0, row);
          tma_load_2d(hb + kBHalf, &tm_hi, bfull, 64, row);
          tma_load_2d(hb + kBBytes, &tm_lo, bfull, 0, row);
          tma_load_2d(hb + kBBytes + kBHalf, &tm_lo, bfull, 64, row);
          ++bissued;
          cur_key = key;
        }
      }
    }
    __syncthreads();   // (A)
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i)
        drain_wait(&full[i % kGroups], (i / kGroups) & 1, status);
      if (bissued) drain_wait(bfull, (bissued - 1) & 1, status);
    }
    __syncthreads();   // (B)
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t smem0 = smem_u32(base);
      int it = 0, bseen = 0;
      int uses[kGroups] = {};   // items issued for each group's accumulators
      int64_t cur_key = -1;
      bool ok = true;
      for (int i = t0; i < t1 && ok; ++i) {
        const int n = i / g.tiles_per_seq;
        const int s = it % kStages, grp = it % kGroups;
        if (!mbar_wait(&full[grp], (it / kGroups) & 1, abort_flag, status, kWaitCycles)) break;
        const int mf = blocks_of(i);
        const int nc = tile_items(mf);
        for (int k = 0; k < nc && ok; ++k) {
          const int c = item_chunk(i, k, nc);
          const int64_t key = (int64_t)n * 65536 + c;
          if (key != cur_key) {
            if (cur_key >= 0) mma_commit(bempty);   // the resident chunk may be replaced
            if (!mbar_wait(bfull, bseen & 1, abort_flag, status, kWaitCycles)) {
              ok = false;
              break;
            }
            ++bseen;
            cur_key = key;
          }
          for (int sub = 0; sub < kMaxBlocks / kItemBlocks && ok; ++sub) {
            if (!item_present(c, sub, mf)) continue;
            const int u = uses[grp]++;
            const int acc = grp * kAccPerGroup + (u % kAccPerGroup);
            if (!mbar_wait(&accempty[acc], ((u / kAccPerGroup) & 1) ^ 1, abort_flag, status,
                           kWaitCycles)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int b0 = c * kMaxBlocks + sub * kItemBlocks;
            const int nb = min(max(mf - b0, 0), kItemBlocks);
            const int N = (nb + 15) & ~15;
            if (N > 0) {
              const uint32_t idesc = idesc_bf16_f32(128, N);
              const uint32_t aaddr = smem0 + kStageBase + s * kATileBytes;
              const uint32_t d = tmem_base + (uint32_t)(acc * kItemBlocks);
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                // rows sub * 128 .. of the resident chunk (whole 1 KB swizzle atoms)
                const uint32_t baddr =
                    smem0 + kBBase + part * kBBytes + sub * kItemBlocks * 128;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                  const uint32_t ao = (kk >> 2) * kAHalf + (kk & 3) * 32;
                  const uint32_t bo = (kk >> 2) * kBHalf + (kk & 3) * 32;
                  mma_bf16(d, desc_kmajor_sw128(aaddr + ao), desc_kmajor_sw128(baddr + bo),
                           idesc, (part | kk) ? 1u : 0u);
                }
              }
            }
            mma_commit(&accfull[acc]);
          }
        }
        if (!ok) break;
        mma_commit(&empty[s]);   // the tile's A stage, once all its items' MMAs are done
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
    // ------------------------------------------------------------ epilogue (warps 2 ..)
    const int grp = (warp - 2) >> 2;     // group: tiles t0 + grp, t0 + grp + kGroups, ...
    const int quarter = warp & 3;        // TMEM lanes this warp may read
    const int r = quarter * 32 + lane;   // row of the tile
    const int qq = r / g.H, j = r % g.H;
    float* Es2 = reinterpret_cast<float*>(base + kEsBase) + grp * 2 * kRows;
    // Per-row inputs of tile i: lane l < QT reads query l's prefix length (the tile's
    // largest full-block count is their maximum), every lane its own |w|.
    auto load_meta = [&](int i, int& Pl, float& wabs) {
      const int n = i / g.tiles_per_seq;
      const int ta = (i % g.tiles_per_seq) * g.QT;
      Pl = (lane < g.QT && ta + lane < g.T)
               ? prefix_len(pos, (int64_t)n * g.T + ta + lane, g.L, nullptr) : 0;
      const int tq = ta + qq;
      wabs = fabsf(w[((int64_t)n * g.T + (tq < g.T ? tq : 0)) * g.H + j]);
    };
    // Every epilogue warp of a group walks every tile of the group and meets the group
    // barrier of each, whatever happens; after a failed (bounded) wait a warp only skips
    // the work.
    bool ok = true;
    int uses = 0, gt = 0;
    int Pl_next = 0;
    float w_next = 0.f;
    if (t0 + grp < t1) load_meta(t0 + grp, Pl_next, w_next);
    for (int i = t0 + grp, it = grp; i < t1; i += kGroups, it += kGroups, ++gt) {
      const int s = it % kStages;
      const int n = i / g.tiles_per_seq;
      const int ta = (i % g.tiles_per_seq) * g.QT;
      const int tq = ta + qq;
      const bool valid = tq < g.T;
      const int64_t qrow = (int64_t)n * g.T + (valid ? tq : 0);
      const int Pl = Pl_next;
      const float wabs = w_next;
      if (i + kGroups < t1) load_meta(i + kGroups, Pl_next, w_next);   // one group tile ahead
      int mf = Pl / g.B;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mf = max(mf, __shfl_xor_sync(0xffffffffu, mf, o));
      const int P = __shfl_sync(0xffffffffu, Pl, valid ? qq : 0);   // qq < QT <= 16
      const int mfull = P / g.B;
      const int M = (P + g.B - 1) / g.B;
      const int nc = tile_items(mf);
      // the partial last block: q . kpart over 128 dimensions, reading the query row from
      // the tile's A stage and the partial keys copied with it, then releasing the stage
      float dot = 0.f;
      if (ok && !warp_wait(&full[grp], (it / kGroups) & 1, abort_flag, status)) ok = false;
      if (ok && M > mfull) {
        float d4[4] = {0.f, 0.f, 0.f, 0.f};   // four chains, so the FMAs overlap
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint8_t* arow = base + kStageBase + s * kATileBytes + hf * kAHalf + r * 128;
          const float4* kv = reinterpret_cast<const float4*>(base + kKpBase + s * kKpBytes +
                                                             (qq * kHeadDim + hf * 64) * 4);
#pragma unroll
          for (int c = 0; c < 8; ++c) {   // 16-byte chunk c of the row (128-byte swizzle)
            const uint4 x = *reinterpret_cast<const uint4*>(arow + ((c ^ (r & 7)) << 4));
            const float4 a = kv[2 * c], b = kv[2 * c + 1];
            d4[0] = fmaf(bf16lo(x.x), a.x, d4[0]); d4[1] = fmaf(bf16hi(x.x), a.y, d4[1]);
            d4[2] = fmaf(bf16lo(x.y), a.z, d4[2]); d4[3] = fmaf(bf16hi(x.y), a.w, d4[3]);
            d4[0] = fmaf(bf16lo(x.z), b.x, d4[0]); d4[1] = fmaf(bf16hi(x.z), b.y, d4[1]);
            d4[2] = fmaf(bf16lo(x.w), b.z, d4[2]); d4[3] = fmaf(bf16hi(x.w), b.w, d4[3]);
          }
        }
        dot = (d4[0] + d4[1]) + (d4[2] + d4[3]);
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&empty[s]);   // this warp is done with the stage
      float sum = 0.f;
      for (int k = 0; k < nc; ++k) {   // the tile's items, in the MMA warp's order
        const int c = item_chunk(i, k, nc);
#pragma unroll 1
        for (int sub = 0; sub < kMaxBlocks / kItemBlocks; ++sub) {
          if (!item_present(c, sub, mf)) continue;
          const int acc = grp * kAccPerGroup + (uses % kAccPerGroup);
          const uint32_t par = (uses / kAccPerGroup) & 1;
          ++uses;
          // this row's full blocks inside the item, and the warp's largest count
          const int mrow = min(max(mfull - (c * kMaxBlocks + sub * kItemBlocks), 0), kItemBlocks);
          int mwarp = mrow;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
            mwarp = max(mwarp, __shfl_xor_sync(0xffffffffu, mwarp, o));
          if (ok && !warp_wait(&accfull[acc], par, abort_flag, status)) ok = false;
          if (ok) {
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                   (uint32_t)(acc * kItemBlocks);
            float s4[4] = {0.f, 0.f, 0.f, 0.f};   // four chains, so the adds overlap
            for (int c0 = 0; c0 < mwarp; c0 += 32) {
              float v[32];
              tmem_ld32(taddr + c0, v);
              if (c0 + 32 <= mrow) {
#pragma unroll
                for (int cc = 0; cc < 32; ++cc) s4[cc & 3] += fmaxf(v[cc], 0.f);
              } else {
#pragma unroll
                for (int cc = 0; cc < 32; ++cc)
                  if (c0 + cc < mrow) s4[cc & 3] += fmaxf(v[cc], 0.f);
              }
            }
            sum += (s4[0] + s4[1]) + (s4[2] + s4[3]);
            tc_fence_before();
            mbar_arrive(&accempty[acc]);
          }
        }
      }
      float* Es = Es2 + (gt & 1) * kRows;   // alternate buffers: one group barrier per tile
      const float tot = sum + (M > mfull ? fmaxf(dot, 0.f) : 0.f);
      const float ev = wabs * tot / (float)M;
      Es[r] = ev;
      if (ok && valid && E) E[qrow * g.H + j] = ev;
      group_bar(grp);
      // top-h heads: each row (one head of one query) counts the heads of its query that
      // come before it (larger E, or equal E and a lower index) and writes its own index at
      // that rank when the rank is below h
      if (ok && valid) {   // H is a multiple of 8: four energies per load
        const float4* eq = reinterpret_cast<const float4*>(Es + qq * g.H);
        int rk0 = 0, rk1 = 0;   // two counts, loads four steps ahead
#pragma unroll 4
        for (int j4 = 0; j4 < g.H / 4; ++j4) {
          const float4 o = eq[j4];
          const int jb = 4 * j4;
          rk0 += (o.x > ev || (o.x == ev && jb < j)) ? 1 : 0;
          rk1 += (o.y > ev || (o.y == ev && jb + 1 < j)) ? 1 : 0;
          rk0 += (o.z > ev || (o.z == ev && jb + 2 < j)) ? 1 : 0;
          rk1 += (o.w > ev || (o.w == ev && jb + 3 < j)) ? 1 : 0;
        }
        const int rank = rk0 + rk1;
        if (rank < h) heads[qrow * h + rank] = j;
      }
    }
    __syncthreads();   // (A)
    __syncthreads();   // (B)
  }
}

// Pooled keys fp32 -> bf16 hi + lo, [nseq, mpad, 128] each (mpad = Mpool rounded up to
// whole chunks), zero rows past the sequence's blocks; grid = nseq * mpad blocks of 128
// threads.
__global__ void route_tc_split_kernel(const float* __restrict__ k_pool, int Mpool, int mpad,
                                      uint16_t* __restrict__ hi, uint16_t* __restrict__ lo) {
  const int n = blockIdx.x / mpad, b = blockIdx.x % mpad, d = threadIdx.x;
  const float x = b < Mpool ? k_pool[((int64_t)n * Mpool + b) * kHeadDim + d] : 0.f;
  const __nv_bfloat16 hh = __float2bfloat16_rn(x);
  const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(hh));
  const int64_t o = ((int64_t)n * mpad + b) * kHeadDim + d;
  hi[o] = __bfloat16_as_ushort(hh);
  lo[o] = __bfloat16_as_ushort(l);
}

// Mean of each query's partial last block (keys Mfull*B .. P-1), zero when there is none:
// one warp per query, lane l sums dimensions 4l .. 4l+3 (the warp reads whole key rows).
constexpr int kPartWarps = 8;
__global__ void __launch_bounds__(32 * kPartWarps) route_tc_partial_kernel(
    const uint16_t* __restrict__ k, const int32_t* __restrict__ pos, int rows, int T, int64_t L,
    int B, float* __restrict__ kpart, int* status) {
  const int64_t row = (int64_t)blockIdx.x * kPartWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int P = prefix_len(pos, row, L, lane == 0 ? status : nullptr);
  const int s0 = (P / B) * B, cnt = P - s0;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  const uint2* kr = reinterpret_cast<const uint2*>(k + ((row / T) * L + s0) * kHeadDim) + lane;
  int s = 0;
  for (; s + 4 <= cnt; s += 4) {
    uint2 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = kr[(int64_t)(s + u) * (kHeadDim / 4)];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a0 += bf16lo(v[u].x); a1 += bf16hi(v[u].x); a2 += bf16lo(v[u].y); a3 += bf16hi(v[u].y);
    }
  }
  for (; s < cnt; ++s) {
    const uint2 v = kr[(int64_t)s * (kHeadDim / 4)];
    a0 += bf16lo(v.x); a1 += bf16hi(v.x); a2 += bf16lo(v.y); a3 += bf16hi(v.y);
  }
  const float inv = cnt > 0 ? 1.f / (float)cnt : 0.f;
  reinterpret_cast<float4*>(kpart + row * kHeadDim)[lane] =
      make_float4(a0 * inv, a1 * inv, a2 * inv, a3 * inv);
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

// Rows per sequence of the hi / lo pooled-key copies: whole chunks of kMaxBlocks.
static int64_t route_tc_mpad(int64_t L, int B) {
  const int64_t Mpool = (L + B - 1) / B;
  return (Mpool + kMaxBlocks - 1) / kMaxBlocks * kMaxBlocks;
}

bool route_tc_supported(int nseq, int T, int H, int64_t L, int B) {
  if (H < 8 || H > 128 || (128 % H) != 0 || encode_fn() == nullptr) return false;
  const int QT = 128 / H;
  const int64_t mpad = route_tc_mpad(L, B);
  if (mpad > 65536 || T < 4 * QT) return false;
  if (nseq > 1 && T % QT != 0) return false;   // tiles must not straddle sequences
  return (int64_t)nseq * T * H < INT32_MAX && (int64_t)nseq * mpad < INT32_MAX;
}

size_t route_tc_ws_bytes(int nseq, int T, int H, int64_t L, int B) {
  (void)H;
  const size_t rows = (size_t)nseq * T;
  // pooled keys hi + lo; the partial keys, padded by a tile's queries (the last tile's copy)
  return 2 * align256((size_t)nseq * route_tc_mpad(L, B) * kHeadDim * 2) +
         align256((rows + kMaxQT) * kHeadDim * 4);
}

cudaError_t launch_route_tc(const uint16_t* q, const float* w, const uint16_t* k,
                            const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                            int64_t L, int B, int h, int32_t* heads, float* E, void* scratch,
                            int* status, cudaStream_t st) {
  const int rows = nseq * T;
  const int Mpool = (int)((L + B - 1) / B);
  const int mpad = (int)route_tc_mpad(L, B);
  char* c = reinterpret_cast<char*>(scratch);
  uint16_t* hi = reinterpret_cast<uint16_t*>(c);
  c += align256((size_t)nseq * mpad * kHeadDim * 2);
  uint16_t* lo = reinterpret_cast<uint16_t*>(c);
  c += align256((size_t)nseq * mpad * kHeadDim * 2);
  float* kpart = reinterpret_cast<float*>(c);

  route_tc_split_kernel<<<nseq * mpad, kHeadDim, 0, st>>>(k_pool, Mpool, mpad, hi, lo);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_tc_partial_kernel<<<(rows + kPartWarps - 1) / kPartWarps, 32 * kPartWarps, 0, st>>>(
      k, pos, rows, T, L, B, kpart, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, thi, tlo;
  if (!make_map(&tq, q, (uint64_t)rows * H, kRows) ||
      !make_map(&thi, hi, (uint64_t)nseq * mpad, kMaxBlocks) ||
      !make_map(&tlo, lo, (uint64_t)nseq * mpad, kMaxBlocks))
    return cudaErrorInvalidValue;
  RouteGeo g;
  g.T = T;
  g.H = H;
  g.B = B;
  g.QT = 128 / H;
  g.L = L;
  g.tiles_per_seq = (T + g.QT - 1) / g.QT;
  g.mpad = mpad;
  const int total_tiles = nseq * g.tiles_per_seq;
  e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  route_tc_kernel<<<sms, kThreads, kSmemBytes, st>>>(tq, thi, tlo, w, kpart, pos, g, total_tiles,
                                                     h, heads, E, status);
  return cudaGetLastError();
}

}  // namespace misa
