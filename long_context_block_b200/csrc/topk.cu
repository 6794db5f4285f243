// K5: per-row top-k token selection -- TopK of Eqs. (2), (10), (11), (12) of the MISA
// paper summary.  Output order: descending score, equal scores by ascending token
// index; rows shorter than k are padded with index -1 and value -inf.
//
// Scores are mapped to order-preserving uint32 keys (composite 64-bit pairs with the
// complemented index, so equal keys order by ascending index).  The forms, by row shape:
//
// topk_row_kernel (rows up to 16384 scores, or 40960 with the scorer's histogram): one CTA
// per row stages the row in shared memory with one bulk copy, finds the cutoff bin of a
// 12-bit key histogram (refined by the next 12 bits when the bin is crowded), compacts the
// candidates while counting them into sub-buckets of the bins above the cutoff, and places
// every pair by a scan, a scatter and a rank inside its bucket.
//
// topk_scatter_kernel + topk_group_kernel (longer decode rows with the scorer's histogram):
// many CTAs per row append the candidates to groups of output positions, one CTA per group
// sorts them; topk_hist_overflow_kernel takes rows whose candidates do not fit the groups.
//
// topk_cluster_kernel (other long rows): a row is split over a thread-block cluster of G
// CTAs (G = 1, 2, 4 or 8).  Each CTA keeps its slice of the row in shared memory as keys;
// the k-th largest key is found exactly by a three-pass radix select (11, 11 and 10 bits)
// whose per-pass histograms are summed across the cluster through distributed shared
// memory; the selected pairs (every key above the threshold plus the lowest-index keys
// equal to it) go to the leader CTA, which sorts them.
// topk_kernel (fallback for rows too long for a cluster's shared memory): one CTA per
// row, every radix pass re-reads the row from global memory.
#include <cooperative_groups.h>

#include "blocksort.cuh"
#include "common.cuh"
#include "groupsort.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace misa {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;

__device__ __forceinline__ uint64_t compose(uint32_t key, int32_t id) {
  return ((uint64_t)key << 32) | (uint64_t)(~(uint32_t)id);
}

// Shared-histogram increment by a whole warp: lanes holding the same bin add once.  Used by
// the row kernel's exact (crowded-cutoff) passes, where a row's keys may all fall in one bin
// (exact zeros from the ReLU, ties) and plain atomics would serialise on one address.  Every lane of the
// warp must call it; `ok` = this lane has a key to count.
__device__ __forceinline__ void warp_hist_add(uint32_t* h, uint32_t bin, bool ok) {
  const uint32_t key = ok ? bin : 0xffffffffu;
  const uint32_t m = __match_any_sync(0xffffffffu, key);
  if (ok && (threadIdx.x & 31) == (uint32_t)(__ffs(m) - 1)) atomicAdd(&h[bin], (uint32_t)__popc(m));
}

// Block-wide exclusive prefix sum over one value per thread (all threads must call).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums,
                                                    uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t ws = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, ws, off);
      if (lane >= off) ws += o;
    }
    warp_sums[lane] = ws;
  }
  __syncthreads();
  const uint32_t base = warp > 0 ? warp_sums[warp - 1] : 0u;
  total = warp_sums[31];
  __syncthreads();
  return base + incl - v;
}

// Block-wide exclusive prefix sum for NT threads (all threads must call).
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan_nt(uint32_t v, uint32_t* warp_sums,
                                                       uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = NT / 32;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t x = warp_sums[w];
    if (w < warp) base += x;
    tot += x;
  }
  total = tot;
  __syncthreads();
  return base + incl - v;
}

// Write the first min(n, topk) sorted pairs of `sel` as (index, value), pad the rest.
__device__ __forceinline__ void write_row(const uint64_t* sel, int n, int topk, int64_t row,
                                          int32_t* idx, float* vals) {
  const int nvalid = n < topk ? n : topk;
  for (int i = threadIdx.x; i < topk; i += kThreads) {
    const int64_t o = row * topk + i;
    if (i < nvalid) {
      const uint64_t v = sel[i];
      idx[o] = (int32_t)(~(uint32_t)(v & 0xffffffffu));
      if (vals) vals[o] = key_score((uint32_t)(v >> 32));
    } else {
      idx[o] = -1;
      if (vals) vals[o] = __int_as_float(0xff800000);
    }
  }
}

// Exact selection over a row in global memory (three radix passes that re-read the row):
// fills sel[0 .. sortn) with the min(n, topk) selected (key, index) pairs and zero padding.
// All threads of the block must call it.
// Exact selection over a row in global memory (three radix passes that re-read the row):
// fills sel[0 .. sortn) with the min(n, topk) selected (key, index) pairs and zero padding.
// All NT threads of the block must call it.
template <int NT>
__device__ void select_row_global_nt(const float* __restrict__ x, const int32_t* __restrict__ imap,
                                     int n, int topk, int sortn, uint64_t* sel, uint32_t* hist,
                                     uint32_t* warp_sums, uint32_t& s_digit, uint32_t& s_above,
                                     uint32_t& s_cnt) {
  const int tid = threadIdx.x;
  constexpr int kPerT = kBins / NT;   // histogram bins per thread in the digit search
  if (n <= topk) {
    for (int i = tid; i < sortn; i += NT)
      sel[i] = i < n ? compose(score_key(x[i]), imap ? imap[i] : i) : 0ull;
  } else {
    uint32_t prefix = 0, mask = 0, kneed = (uint32_t)topk;
    for (int p = 0; p < 3; ++p) {
      const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
      const int nb = p == 2 ? 1024 : 2048;
      for (int b = tid; b < kBins; b += NT) hist[b] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += NT) {
        const uint32_t key = score_key(x[i]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
      }
      __syncthreads();
      // suffix scan: thread t covers bins nb-1-kPerT*t-i, i < kPerT
      uint32_t cb[kPerT], local = 0;
#pragma unroll
      for (int i = 0; i < kPerT; ++i) {
        const int b = nb - 1 - kPerT * tid - i;
        cb[i] = b >= 0 ? hist[b] : 0u;
        local += cb[i];
      }
      uint32_t total;
      const uint32_t excl = block_excl_scan_nt<NT>(local, warp_sums, total);
      uint32_t run = excl;
#pragma unroll
      for (int i = 0; i < kPerT; ++i) {
        if (run < kneed && kneed <= run + cb[i]) {
          s_digit = nb - 1 - kPerT * tid - i;
          s_above = run;
        }
        run += cb[i];
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= (uint32_t)(nb - 1) << shift;
      kneed -= s_above;
      __syncthreads();
    }
    const uint32_t thr = prefix;
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    uint32_t eq_taken = 0;
    for (int base = 0; base < n; base += NT) {
      const int i = base + tid;
      const uint32_t key = i < n ? score_key(x[i]) : 0u;
      const bool gt = i < n && key > thr;
      const bool eq = i < n && key == thr;
      if (gt) sel[atomicAdd(&s_cnt, 1u)] = compose(key, imap ? imap[i] : i);
      uint32_t total;
      const uint32_t rank = block_excl_scan_nt<NT>(eq ? 1u : 0u, warp_sums, total);
      if (eq && eq_taken + rank < kneed) sel[atomicAdd(&s_cnt, 1u)] = compose(key, imap ? imap[i] : i);
      eq_taken += total;
    }
    __syncthreads();
    for (int i = topk + tid; i < sortn; i += NT) sel[i] = 0ull;
  }
  __syncthreads();
}

__device__ __forceinline__ void select_row_global(const float* __restrict__ x,
                                                  const int32_t* __restrict__ imap, int n, int topk,
                                                  int sortn, uint64_t* sel, uint32_t* hist,
                                                  uint32_t* warp_sums, uint32_t& s_digit,
                                                  uint32_t& s_above, uint32_t& s_cnt) {
  select_row_global_nt<kThreads>(x, imap, n, topk, sortn, sel, hist, warp_sums, s_digit, s_above,
                                 s_cnt);
}

__global__ void __launch_bounds__(kThreads) topk_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const int32_t* __restrict__ gather_len, const int32_t* __restrict__ index_map, int topk,
    int sortn, int32_t* __restrict__ idx, float* __restrict__ vals, int64_t row0) {
  extern __shared__ uint64_t sel[];   // [sortn]
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_digit, s_above, s_cnt;
  const int64_t row = row0 + blockIdx.x;
  const int n = gather_len ? gather_len[row] : prefix_len(pos, row, L, nullptr);
  select_row_global(scores + row * stride, index_map ? index_map + row * stride : nullptr, n, topk,
                    sortn, sel, hist, warp_sums, s_digit, s_above, s_cnt);
  sort_buf_desc(sel, sortn);
  write_row(sel, n, topk, row, idx, vals);
}

// Shared-memory budget of the cluster form (per CTA): the row slice (4 bytes per score)
// plus the leader's sort buffer (8 bytes per slot); the histogram is static.
constexpr int kClusterSmemBudget = 200 * 1024;
constexpr int kSliceTarget = 8192;   // scores per CTA the cluster size aims for

__global__ void __launch_bounds__(kThreads, 1) topk_cluster_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const int32_t* __restrict__ gather_len, const int32_t* __restrict__ index_map, int topk,
    int sortn, int slice_cap, int32_t* __restrict__ idx, float* __restrict__ vals) {
  extern __shared__ uint8_t dyn[];
  uint64_t* sel = reinterpret_cast<uint64_t*>(dyn);                     // [sortn] (leader)
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn + (size_t)sortn * 8);  // [slice_cap]
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_digit, s_above, s_cnt, s_eq;
  cg::cluster_group cluster = cg::this_cluster();
  const int G = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t row = blockIdx.x / G;
  const int n = gather_len ? gather_len[row] : prefix_len(pos, row, L, nullptr);
  const float* x = scores + row * stride;
  const int32_t* imap = index_map ? index_map + row * stride : nullptr;
  int slice = (n + G - 1) / G;
  slice = (slice + 3) & ~3;
  const int lo = min(n, crank * slice);
  const int cnt = min(n, lo + slice) - lo;
  uint64_t* lsel = cluster.map_shared_rank(sel, 0);

  for (int i = tid; i < cnt; i += kThreads) keys[i] = score_key(x[lo + i]);
  if (tid == 0) { s_cnt = 0; s_eq = 0; }
  __syncthreads();

  if (n <= topk) {
    for (int i = tid; i < cnt; i += kThreads)
      lsel[lo + i] = compose(keys[i], imap ? imap[lo + i] : lo + i);
    if (crank == 0)
      for (int i = n + tid; i < sortn; i += kThreads) sel[i] = 0ull;
    cluster.sync();
  } else {
    uint32_t prefix = 0, mask = 0, kneed = (uint32_t)topk;
    for (int p = 0; p < 3; ++p) {
      const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
      const int nb = p == 2 ? 1024 : 2048;
      for (int b = tid; b < kBins; b += kThreads) hist[b] = 0;
      __syncthreads();
      for (int base = 0; base < cnt; base += kThreads) {
        const int i = base + tid;
        const uint32_t key = i < cnt ? keys[i] : 0u;
        const bool act = i < cnt && (key & mask) == prefix;
        const uint32_t d = act ? (key >> shift) & (uint32_t)(nb - 1) : 0xffffffffu;
        // lanes with the same digit add once (scores crowd into few top-level bins)
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
        if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (uint32_t)__popc(peers));
      }
      cluster.sync();   // every CTA's histogram is complete
      const bool on = 2 * tid < nb;
      uint32_t c_hi = 0, c_lo = 0;
      if (on) {
        for (int c = 0; c < G; ++c) {
          const uint32_t* h = cluster.map_shared_rank(hist, c);
          c_hi += h[nb - 1 - 2 * tid];
          c_lo += h[nb - 2 - 2 * tid];
        }
      }
      uint32_t total;
      const uint32_t excl = block_excl_scan(c_hi + c_lo, warp_sums, total);
      if (on) {
        if (excl < kneed && kneed <= excl + c_hi) {
          s_digit = nb - 1 - 2 * tid;
          s_above = excl;
        } else if (excl + c_hi < kneed && kneed <= excl + c_hi + c_lo) {
          s_digit = nb - 2 - 2 * tid;
          s_above = excl + c_hi;
        }
      }
      cluster.sync();   // digit known here; no CTA still reads another's histogram
      prefix |= s_digit << shift;
      mask |= (uint32_t)(nb - 1) << shift;
      kneed -= s_above;
    }
    const uint32_t thr = prefix;
    // Output slots are fixed without remote atomics: the pairs above the threshold go
    // first, slice by slice in cluster-rank order; then the equal-to-threshold pairs in
    // index order, as many as are needed.
    uint32_t gt_local = 0, eq_local = 0;
    for (int i = tid; i < cnt; i += kThreads) {
      gt_local += keys[i] > thr ? 1u : 0u;
      eq_local += keys[i] == thr ? 1u : 0u;
    }
    gt_local = __reduce_add_sync(0xffffffffu, gt_local);
    eq_local = __reduce_add_sync(0xffffffffu, eq_local);
    if (lane == 0 && gt_local) atomicAdd(&s_cnt, gt_local);
    if (lane == 0 && eq_local) atomicAdd(&s_eq, eq_local);
    cluster.sync();
    uint32_t gt_base = 0, gt_total = 0, eq_before = 0;
    for (int c = 0; c < G; ++c) {
      const uint32_t g = *cluster.map_shared_rank(&s_cnt, c);
      const uint32_t e = *cluster.map_shared_rank(&s_eq, c);
      gt_total += g;
      if (c < crank) { gt_base += g; eq_before += e; }
    }
    const uint32_t my_eq = *cluster.map_shared_rank(&s_eq, crank);
    const uint32_t take_eq = kneed > eq_before ? min(kneed - eq_before, my_eq) : 0u;
    uint32_t gt_done = 0, eq_done = 0;
    for (int base = 0; base < cnt; base += kThreads) {
      const int i = base + tid;
      const uint32_t key = i < cnt ? keys[i] : 0u;
      const bool gt = i < cnt && key > thr;
      const bool eq = i < cnt && key == thr;
      uint32_t tot;
      const uint32_t ex = block_excl_scan((gt ? 1u << 16 : 0u) | (eq ? 1u : 0u), warp_sums, tot);
      if (gt) lsel[gt_base + gt_done + (ex >> 16)] = compose(key, imap ? imap[lo + i] : lo + i);
      const uint32_t re = eq_done + (ex & 0xffffu);
      if (eq && re < take_eq)
        lsel[gt_total + eq_before + re] = compose(key, imap ? imap[lo + i] : lo + i);
      gt_done += tot >> 16;
      eq_done += tot & 0xffffu;
    }
    if (crank == 0)
      for (int i = topk + tid; i < sortn; i += kThreads) sel[i] = 0ull;
    cluster.sync();   // the leader's buffer holds exactly topk pairs
  }
  if (crank != 0) return;
  sort_buf_desc(sel, sortn);
  write_row(sel, n, topk, row, idx, vals);
}

// ---------------------------------------------------------------- histogram-split form
// The score histogram (top kScoreHistBits key bits, one bin = 1/8 octave) gives, for every
// bin at or above the cutoff bin (the bin of the row's k-th largest score), the output
// position of its first score.  Those bins are cut into groups by start position
// (kGroupSpan positions per group); CTA g of a row gathers the scores of group g's bins
// from the row (a compare-and-compact pass over L2-resident scores), sorts them with a
// counting sort on the next key bits (groupsort.cuh) and writes them at their positions.
// Group key ranges are disjoint, so no merge is needed; only the cutoff bin is cut short.
// Rows whose candidates do not fit (more than kMaxGroups groups, or a bin too large for
// one group) are done by topk_hist_overflow_kernel with an exact radix select.
constexpr int kSelThreads = 256;
constexpr int kGroupSpan = 1024;                          // output positions per group
constexpr int kMaxGroups = kTopkCandCap / kGroupSpan;     // at most 16 CTAs per row
constexpr int kGroupBuf = 8192;                           // pairs one group CTA holds
constexpr uint32_t kBigBin = kGroupBuf - kGroupSpan;      // larger bins: overflow path
constexpr int kGroupExactMax = 4096;   // overflow rows up to this k: CTA 0 of the group kernel

// Groups of a row: a bin at or above the cutoff starts before output position k, so its
// group is below ceil(k / kGroupSpan).
__host__ __device__ constexpr int hist_groups(int topk) {
  return (topk + kGroupSpan - 1) / kGroupSpan;
}
constexpr int kScatterPer = 16;                           // scores per thread in pass 1
constexpr int kScatterChunk = kSelThreads * kScatterPer;  // 4096 scores per CTA

// Cutoff bin and candidate statistics of a row from its histogram, identical in every
// kernel that calls it (NT threads, NT dividing kScoreHistBins).  Thread t owns the
// bins [hi - kPer, hi), hi = kScoreHistBins - kPer * t; `before` = scores above them.
template <int NT>
struct HistView {
  static constexpr int kPer = kScoreHistBins / NT;
  uint32_t c[kPer];
  uint32_t before;
  int hi;
};

template <int NT>
__device__ __forceinline__ uint32_t hist_cutoff(const uint32_t* __restrict__ h, uint32_t target,
                                                HistView<NT>& v, uint32_t* warp_sums,
                                                uint32_t& s_cut, uint32_t& s_total,
                                                uint32_t& s_big) {
  constexpr int kPer = HistView<NT>::kPer;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  v.hi = kScoreHistBins - kPer * t;
  uint32_t local = 0;
  const uint4* h4 = reinterpret_cast<const uint4*>(h + v.hi - kPer);   // 16-byte aligned
#pragma unroll
  for (int i = 0; i < kPer / 4; ++i) {
    const uint4 q = h4[kPer / 4 - 1 - i];
    v.c[4 * i + 0] = q.w;
    v.c[4 * i + 1] = q.z;
    v.c[4 * i + 2] = q.y;
    v.c[4 * i + 3] = q.x;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) local += v.c[i];
  if (t == 0) { s_cut = 0; s_total = 0; s_big = 0; }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t pre = 0;
  for (int w = 0; w < warp; ++w) pre += warp_sums[w];
  v.before = pre + incl - local;
  uint32_t run = v.before;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    if (run < target && target <= run + v.c[i]) s_cut = v.hi - 1 - i;
    run += v.c[i];
  }
  __syncthreads();
  const uint32_t cut = s_cut;
  uint32_t cand = 0, big = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if ((uint32_t)(v.hi - 1 - i) >= cut) {
      cand += v.c[i];
      big |= v.c[i] > kBigBin;
    }
  if (cand) atomicAdd(&s_total, cand);
  if (big) s_big = 1;
  __syncthreads();
  return cut;
}

__device__ __forceinline__ bool hist_overflow(uint32_t total, uint32_t big) {
  return total > (uint32_t)(kMaxGroups * kGroupSpan) || big != 0;
}

// Output start of every bin at or above the cutoff and the group it belongs to.
template <int NT>
__device__ __forceinline__ void bin_groups(const HistView<NT>& hv, uint32_t cut, uint8_t* gid) {
  uint32_t run = hv.before;
#pragma unroll
  for (int i = 0; i < HistView<NT>::kPer; ++i) {
    const uint32_t b = hv.hi - 1 - i;
    gid[b] = (b >= cut && hv.c[i]) ? (uint8_t)(run / kGroupSpan) : (uint8_t)0xff;
    run += hv.c[i];
  }
}

// Pass 1: many CTAs per row each read one chunk of the row once and append its
// candidates (scores in bins at or above the cutoff) to their group's buffer.
__global__ void __launch_bounds__(kSelThreads) topk_scatter_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const uint32_t* __restrict__ hist, int topk, uint64_t* __restrict__ cand,
    uint32_t* __restrict__ gcount) {
  pdl_prologue();
  __shared__ uint8_t gid[kScoreHistBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t lcount[kMaxGroups], lbase[kMaxGroups];
  __shared__ uint32_t s_cut, s_total, s_big;
  const int t = threadIdx.x;
  const int64_t row = blockIdx.y;
  const int n = prefix_len(pos, row, L, nullptr);
  const int start = blockIdx.x * kScatterChunk;
  if (start >= n) return;
  if (t < kMaxGroups) lcount[t] = 0;
  HistView<kSelThreads> hv;
  const uint32_t cut = hist_cutoff<kSelThreads>(hist + row * kScoreHistBins, (uint32_t)min(n, topk),
                                                hv, warp_sums, s_cut, s_total, s_big);
  if (hist_overflow(s_total, s_big)) return;
  bin_groups<kSelThreads>(hv, cut, gid);
  const float* x = scores + row * stride;
  uint32_t key[kScatterPer];
#pragma unroll
  for (int j = 0; j < kScatterPer; ++j) {
    const int e = start + j * kSelThreads + t;
    key[j] = e < n ? score_key(x[e]) : 0u;
  }
  __syncthreads();   // gid complete
  uint32_t slot[kScatterPer];
#pragma unroll
  for (int j = 0; j < kScatterPer; ++j) {
    const int e = start + j * kSelThreads + t;
    const uint32_t grp = e < n ? gid[key[j] >> (32 - kScoreHistBits)] : 0xffu;
    slot[j] = grp != 0xffu ? (grp << 16) | atomicAdd(&lcount[grp], 1u) : 0xffffffffu;
  }
  __syncthreads();
  if (t < kMaxGroups && lcount[t]) lbase[t] = atomicAdd(&gcount[row * kMaxGroups + t], lcount[t]);
  __syncthreads();
  uint64_t* crow = cand + row * (int64_t)hist_groups(topk) * kGroupBuf;
#pragma unroll
  for (int j = 0; j < kScatterPer; ++j) {
    if (slot[j] == 0xffffffffu) continue;
    const uint32_t grp = slot[j] >> 16;
    const uint32_t p = lbase[grp] + (slot[j] & 0xffffu);
    if (p < (uint32_t)kGroupBuf)
      crow[grp * kGroupBuf + p] = compose(key[j], start + j * kSelThreads + t);
  }
}

// Pass 2: CTA g of a row sorts group g's candidates and writes them at their positions.
__global__ void __launch_bounds__(kSelThreads, 1) topk_group_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const uint32_t* __restrict__ hist, int topk, const uint64_t* __restrict__ cand,
    int32_t* __restrict__ idx, float* __restrict__ vals) {
  pdl_prologue();
  extern __shared__ uint64_t gbuf[];   // [2 * kGroupBuf]: gathered, then sorted
  __shared__ uint32_t buckets[kSubBucketWords];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_cut, s_total, s_big, s_lo, s_hi, s_start, s_cnt, s_flag;
  __shared__ uint32_t s_digit, s_above, s_sel;
  uint64_t* gathered = gbuf;
  uint64_t* sorted = gbuf + kGroupBuf;
  const int t = threadIdx.x;
  const int64_t row = blockIdx.y;
  const uint32_t g = blockIdx.x;
  const int n = prefix_len(pos, row, L, nullptr);
  const uint32_t target = (uint32_t)min(n, topk);
  if (t == 0) { s_lo = 0xffffffffu; s_hi = 0; s_start = 0xffffffffu; s_cnt = 0; }
  HistView<kSelThreads> hv;
  const uint32_t cut = hist_cutoff<kSelThreads>(hist + row * kScoreHistBins, target, hv, warp_sums,
                                                s_cut, s_total, s_big);
  if (hist_overflow(s_total, s_big)) {
    // crowded cutoff (e.g. many equal scores): an exact selection over the whole row, here
    // by CTA 0 when the selected pairs fit its buffer, else by topk_hist_overflow_kernel
    if (g != 0 || topk > kGroupExactMax) return;
    int sortn = kSelThreads;
    while (sortn < topk) sortn <<= 1;
    select_row_global_nt<kSelThreads>(scores + row * stride, nullptr, n, topk, sortn, gbuf, buckets,
                                      warp_sums, s_digit, s_above, s_sel);
    switch (sortn / kSelThreads) {
      case 1: sort_buf_desc_e<1, kSelThreads>(gbuf); break;
      case 2: sort_buf_desc_e<2, kSelThreads>(gbuf); break;
      case 4: sort_buf_desc_e<4, kSelThreads>(gbuf); break;
      case 8: sort_buf_desc_e<8, kSelThreads>(gbuf); break;
      default: sort_buf_desc_e<16, kSelThreads>(gbuf); break;
    }
    for (int i = t; i < topk; i += kSelThreads) {
      const int64_t o = row * topk + i;
      if ((uint32_t)i < target) {
        const uint64_t v = gbuf[i];
        idx[o] = (int32_t)(~(uint32_t)(v & 0xffffffffu));
        if (vals) vals[o] = key_score((uint32_t)(v >> 32));
      } else {
        idx[o] = -1;
        if (vals) vals[o] = __int_as_float(0xff800000);
      }
    }
    return;
  }
  {
    uint32_t run = hv.before, lo = 0xffffffffu, hb = 0, cnt = 0, st = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < HistView<kSelThreads>::kPer; ++i) {
      const uint32_t b = hv.hi - 1 - i;
      if (b >= cut && hv.c[i] && run / kGroupSpan == g) {
        lo = min(lo, b);
        hb = max(hb, b);
        cnt += hv.c[i];
        st = min(st, run);
      }
      run += hv.c[i];
    }
    if (cnt) {
      atomicMin(&s_lo, lo);
      atomicMax(&s_hi, hb);
      atomicAdd(&s_cnt, cnt);
      atomicMin(&s_start, st);
    }
  }
  __syncthreads();
  if (g == 0)
    for (int i = target + t; i < topk; i += kSelThreads) {
      idx[row * topk + i] = -1;
      if (vals) vals[row * topk + i] = __int_as_float(0xff800000);
    }
  const uint32_t cnt = min(s_cnt, (uint32_t)kGroupBuf);
  if (cnt == 0) return;
  const uint32_t blo = s_lo, bhi = s_hi, start = s_start;
  const uint64_t* src = cand + row * (int64_t)hist_groups(topk) * kGroupBuf + g * kGroupBuf;
  for (uint32_t i = t; i < cnt; i += kSelThreads) gathered[i] = src[i];
  __syncthreads();
  const uint64_t* res = gathered;   // the counting sort leaves its result in place
  if (!group_sort_desc<kSelThreads>(gathered, cnt, sorted, buckets, blo, bhi, warp_sums, s_flag)) {
    // crowded buckets (many equal scores): bitonic sort of the group instead
    res = sorted;
    int sortn = kSelThreads;
    while ((uint32_t)sortn < cnt) sortn <<= 1;
    for (int i = t; i < sortn; i += kSelThreads) sorted[i] = (uint32_t)i < cnt ? gathered[i] : 0ull;
    __syncthreads();
    switch (sortn / kSelThreads) {   // cnt <= kGroupBuf = 32 * kSelThreads
      case 1: sort_buf_desc_e<1, kSelThreads>(sorted); break;
      case 2: sort_buf_desc_e<2, kSelThreads>(sorted); break;
      case 4: sort_buf_desc_e<4, kSelThreads>(sorted); break;
      case 8: sort_buf_desc_e<8, kSelThreads>(sorted); break;
      case 16: sort_buf_desc_e<16, kSelThreads>(sorted); break;
      default: sort_buf_desc_e<32, kSelThreads>(sorted); break;
    }
  }
  for (uint32_t i = t; i < cnt && start + i < target; i += kSelThreads) {
    const uint64_t v = res[i];
    const int64_t o = row * topk + start + i;
    idx[o] = (int32_t)(~(uint32_t)(v & 0xffffffffu));
    if (vals) vals[o] = key_score((uint32_t)(v >> 32));
  }
}

// The score histogram of rows the scorer did not histogram (rows of several queries per
// sequence): grid (chunks of kScatterChunk scores, rows); each CTA counts its chunk's keys
// in shared memory and adds the occupied bins to the row's histogram (zeroed beforehand).
__global__ void __launch_bounds__(kSelThreads) topk_build_hist_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    uint32_t* __restrict__ hist) {
  pdl_prologue();
  __shared__ uint32_t sh[kScoreHistBins];
  const int t = threadIdx.x;
  const int64_t row = blockIdx.y;
  const int n = prefix_len(pos, row, L, nullptr);
  const int start = blockIdx.x * kScatterChunk;
  if (start >= n) return;
  for (int b = t; b < kScoreHistBins; b += kSelThreads) sh[b] = 0;
  __syncthreads();
  const float* x = scores + row * stride;
#pragma unroll
  for (int j = 0; j < kScatterPer; ++j) {
    const int e = start + j * kSelThreads + t;
    if (e < n) atomicAdd(&sh[score_key(x[e]) >> (32 - kScoreHistBits)], 1u);
  }
  __syncthreads();
  uint32_t* gh = hist + row * kScoreHistBins;
  for (int b = t; b < kScoreHistBins; b += kSelThreads)
    if (sh[b]) atomicAdd(gh + b, sh[b]);
}

// Exact selection for the rows topk_group_kernel leaves out (same overflow test, k > 4096).
__global__ void __launch_bounds__(kThreads) topk_hist_overflow_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const uint32_t* __restrict__ hist, int topk, int sortn, int32_t* __restrict__ idx,
    float* __restrict__ vals) {
  pdl_prologue();
  extern __shared__ uint64_t sel[];   // [sortn]
  __shared__ uint32_t hbuf[kBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_cut, s_total, s_big, s_digit, s_above, s_cnt;
  const int64_t row = blockIdx.x;
  const int n = prefix_len(pos, row, L, nullptr);
  HistView<kThreads> hv;
  hist_cutoff<kThreads>(hist + row * kScoreHistBins, (uint32_t)min(n, topk), hv, warp_sums, s_cut,
                        s_total, s_big);
  if (!hist_overflow(s_total, s_big)) return;
  select_row_global(scores + row * stride, nullptr, n, topk, sortn, sel, hbuf, warp_sums, s_digit,
                    s_above, s_cnt);
  sort_buf_desc(sel, sortn);
  write_row(sel, n, topk, row, idx, vals);
}

// ---------------------------------------------------------------- row-resident form
// Rows of up to ROWCAP scores and k <= CAP: one CTA of NT threads per row copies the row
// into shared memory with one bulk asynchronous copy (plain loads for the at most three
// scores on either side of its 16-byte-aligned interior), turns the scores into keys in
// place, finds the cutoff bin with a histogram of the top kScoreHistBits key bits (or
// takes the one the scorer built), compacts the candidates (bins at or above it) counting
// them into sub-buckets, and writes each at the output position that a scan of the bucket
// counts, a scatter into bucket order and a rank inside the bucket give it.  A crowded
// cutoff (more than CAP candidates) takes an exact radix select over the resident keys
// and the adaptive counting sort (groupsort.cuh) instead.  Shapes: 512 threads, 3072
// candidates, 16K rows (two CTAs per SM: many rows, k <= 3072); 512 or 1024 threads, 8192
// candidates, 16K rows (one CTA per SM; 1024 threads when rows are too few to fill the
// SMs); 1024 threads, 3072 candidates, 40K rows (long decode rows).
constexpr int kRowCap = 16384;
constexpr int kLongRowCap = 40960;
constexpr long long kRowWaitCycles = 4000000000LL;
constexpr uint32_t kRowSuspendNs = 20000;   // longest single suspension in the copy wait

template <int NT, int CAP, int ROWCAP>
struct RowCfg {
  // keys [ROWCAP] u32 (+16 bytes to align the bulk copy), later the sorted pairs [<= CAP]
  // u64, then the candidates [CAP] u64
  static constexpr int kKeyPairs = (ROWCAP * 4 + 16) / 8 > CAP ? (ROWCAP * 4 + 16) / 8 : CAP;
  // the adaptive sort's bin tables sit in the key space the sorted pairs leave free, or
  // after the candidates
  static constexpr bool kAuxInKeys = (kKeyPairs - CAP) * 8 >= kAdaptiveAuxBytes;
  static constexpr size_t kAuxOff = kAuxInKeys ? (size_t)CAP * 8 : (size_t)(kKeyPairs + CAP) * 8;
  static constexpr size_t kSmem =
      (size_t)(kKeyPairs + CAP) * sizeof(uint64_t) + (kAuxInKeys ? 0 : kAdaptiveAuxBytes);
  static constexpr int kEMax = CAP <= NT ? 1 : CAP <= 2 * NT ? 2 : CAP <= 4 * NT ? 4
                               : CAP <= 8 * NT ? 8 : 16;
  static constexpr int kBinsPer = 2048 / NT;   // radix-select bins per thread
  static_assert(CAP <= 16 * NT && 2048 % NT == 0 && ROWCAP < 65536, "row kernel shape");
};

template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t& lo, uint32_t& hi, uint32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&red[0], lo);
    atomicMax(&red[1], hi);
  }
  __syncthreads();
  lo = red[0];
  hi = red[1];
}

// Bitonic fallback of the counting sort: sorted[0 .. sortn) descending, sortn = NT * 2^i.
template <int NT, int EMAX>
__device__ __forceinline__ void row_bitonic(uint64_t* sorted, int sortn) {
  const int e = sortn / NT;
  if (e <= 1) sort_buf_desc_e<1, NT>(sorted);
  else if constexpr (EMAX >= 2) {
    if (e == 2) sort_buf_desc_e<2, NT>(sorted);
    else if constexpr (EMAX >= 4) {
      if (e == 4) sort_buf_desc_e<4, NT>(sorted);
      else if constexpr (EMAX >= 8) {
        if (e == 8) sort_buf_desc_e<8, NT>(sorted);
        else if constexpr (EMAX >= 16) sort_buf_desc_e<16, NT>(sorted);
      }
    }
  }
}

template <int NT, int CAP, int ROWCAP, int MINB>
__global__ void __launch_bounds__(NT, MINB) topk_row_kernel(
    const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ pos, int64_t L,
    const int32_t* __restrict__ gather_len, const int32_t* __restrict__ index_map,
    const uint32_t* __restrict__ ghist, int topk, int32_t* __restrict__ idx,
    float* __restrict__ vals, int* status, int64_t row0) {
  pdl_prologue();
  using RC = RowCfg<NT, CAP, ROWCAP>;
  extern __shared__ __align__(128) uint64_t rbuf[];
  uint64_t* sorted = rbuf;                                     // [CAP] sorted pairs (later)
  uint64_t* cand = rbuf + RC::kKeyPairs;                       // [CAP] candidates
  __shared__ __align__(16) uint32_t hist[kSubBucketWords];     // histogram, then buckets
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t red[2];
  __shared__ uint32_t s_cut, s_total, s_big, s_flag, s_digit, s_above, s_top, s_nsub, s_spill;
  __shared__ __align__(8) uint64_t lbar;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t row = row0 + blockIdx.x;
  const int n = gather_len ? gather_len[row] : prefix_len(pos, row, L, nullptr);
  const uint32_t target = (uint32_t)min(n, topk);
  const float* x = scores + row * stride;
  const int32_t* imap = index_map ? index_map + row * stride : nullptr;

  // keys[e] holds score e: the 16-byte-aligned interior of the row arrives by one bulk
  // copy, to a shared address that is 16-byte aligned too (keys starts `hb` bytes in)
  const uint32_t hb = (uint32_t)(reinterpret_cast<uintptr_t>(x) & 15u);
  uint32_t* keys = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(rbuf) + hb);
  const int h0 = min((int)(((16u - hb) & 15u) >> 2), n);   // scores before the interior
  const int nbulk = ((n - h0) >> 2) << 2;                   // interior scores
  if (t == 0) {
    sm100::mbar_init(&lbar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (t == 0 && nbulk > 0) {
    sm100::mbar_arrive_expect_tx(&lbar, (uint32_t)nbulk * 4u);
    sm100::bulk_load(keys + h0, x + h0, (uint32_t)nbulk * 4u, &lbar);
  }
  if (t < h0) keys[t] = __float_as_uint(x[t]);
  if (t < 4 && h0 + nbulk + t < n) keys[h0 + nbulk + t] = __float_as_uint(x[h0 + nbulk + t]);
  for (int b = t; b < kScoreHistBins; b += NT) hist[b] = (ghist && n > (int)target)
                                                    ? ghist[row * kScoreHistBins + b] : 0u;
  if (t == 0) { red[0] = 0xffffffffu; red[1] = 0; s_top = 0; }
  // Warp w owns the contiguous slice [w0, w1) of the row, walked in 32-key steps, in every
  // pass below; the candidates carry their position e in the row, and the index map (if
  // any) is applied to the k outputs only.
  constexpr int kWarps = NT / 32;
  const int wper = (((n + kWarps - 1) / kWarps) + 31) & ~31;
  const int w0 = min(warp * wper, n), w1 = min(w0 + wper, n);
  const uint32_t below = (1u << lane) - 1u;
  uint32_t cut = 0, btop = 0, C = 0;
  const bool select = (uint32_t)n > target;      // else every score is selected
  const bool given = ghist != nullptr && select;   // cutoff known before the keys arrive
  if (given) {   // runs while the bulk copy is in flight
    __syncthreads();
    HistView<NT> hv;
    cut = hist_cutoff<NT>(hist, target, hv, warp_sums, s_cut, s_total, s_big);
    uint32_t top = 0;
#pragma unroll
    for (int i = HistView<NT>::kPer - 1; i >= 0; --i)
      if (hv.c[i]) top = max(top, (uint32_t)(hv.hi - 1 - i));
    if (top) atomicMax(&s_top, top);
    __syncthreads();
    btop = s_top;
    C = s_total;
  }
  bool landed = true;
  if (nbulk > 0) {   // bounded wait for the copy (threads sleep in the wait, not spin)
    long long t0 = clock64();
    while (!sm100::mbar_try_wait_suspend(&lbar, 0, kRowSuspendNs)) {
      if (clock64() - t0 > kRowWaitCycles) {
        landed = false;
        break;
      }
    }
    if (!landed) {   // record it, then give the copy one more bounded wait
      if (t == 0) set_status(status, MISA_ERR_DEVICE_TIMEOUT);
      t0 = clock64();
      landed = true;
      while (!sm100::mbar_try_wait_suspend(&lbar, 0, kRowSuspendNs)) {
        if (clock64() - t0 > kRowWaitCycles) {
          landed = false;
          break;
        }
      }
    }
  }
  // the threads poll on their own: the row goes on only if every thread saw the copy land;
  // otherwise its result is void (never read from a row still being written)
  if (__syncthreads_or(landed ? 0 : 1)) {
    for (int i = t; i < topk; i += NT) {
      idx[row * topk + i] = -1;
      if (vals) vals[row * topk + i] = __int_as_float(0xff800000);
    }
    return;
  }
  // scores -> keys, and in the same pass: the histogram (none given), the bin range (all
  // selected) or this warp's candidate count (cutoff given)
  const uint32_t kgiven = cut << (32 - kScoreHistBits);
  uint32_t lo = 0xffffffffu, hi = 0, cnt = 0;
  auto note = [&](uint32_t kk) {
    const uint32_t b = kk >> (32 - kScoreHistBits);
    if (!select) {
      lo = min(lo, b);
      hi = max(hi, b);
    } else if (given) {
      cnt += kk >= kgiven ? 1u : 0u;
    } else {
      atomicAdd(&hist[b], 1u);
    }
  };
  if (hb == 0) {   // the keys start 16-byte aligned: lane l takes keys e .. e + 3, e = w0 + 4 l + 128 i
#pragma unroll 2
    for (int e = w0 + 4 * lane; e < w1; e += 128) {
      if (e + 4 <= w1) {
        uint4 v = *reinterpret_cast<const uint4*>(keys + e);
        v.x = score_key(__uint_as_float(v.x));
        v.y = score_key(__uint_as_float(v.y));
        v.z = score_key(__uint_as_float(v.z));
        v.w = score_key(__uint_as_float(v.w));
        *reinterpret_cast<uint4*>(keys + e) = v;
        note(v.x);
        note(v.y);
        note(v.z);
        note(v.w);
      } else {
        for (int u = e; u < w1; ++u) {
          const uint32_t kk = score_key(__uint_as_float(keys[u]));
          keys[u] = kk;
          note(kk);
        }
      }
    }
  } else {
#pragma unroll 4
    for (int e = w0 + lane; e < w1; e += 32) {
      const uint32_t kk = score_key(__uint_as_float(keys[e]));
      keys[e] = kk;
      note(kk);
    }
  }
  __syncthreads();
  if (!select) {
    block_minmax<NT>(lo, hi, red);
    cut = lo;
    btop = hi;
    C = (uint32_t)n;
    cnt = (uint32_t)(w1 - w0) / 32u + ((uint32_t)lane < (uint32_t)((w1 - w0) & 31) ? 1u : 0u);
  } else if (!given) {
    HistView<NT> hv;
    cut = hist_cutoff<NT>(hist, target, hv, warp_sums, s_cut, s_total, s_big);
    // highest occupied bin
    uint32_t top = 0;
#pragma unroll
    for (int i = HistView<NT>::kPer - 1; i >= 0; --i)
      if (hv.c[i]) top = max(top, (uint32_t)(hv.hi - 1 - i));
    if (top) atomicMax(&s_top, top);
    __syncthreads();
    btop = s_top;
    C = s_total;
  }
  __syncthreads();
  // A crowded cutoff bin (more candidates than CAP): refine the threshold with a histogram
  // of the next 12 key bits of the keys in that bin, one more pass over the row; only rows
  // with massive ties (exact zeros from the ReLU, equal keys) still overflow.
  uint32_t kcut = cut << (32 - kScoreHistBits);   // keys >= kcut are candidates
  bool refined = false;
  if (select && C > (uint32_t)CAP) {
    const uint32_t above = C - hist[cut];   // keys in the bins above the cutoff bin
    __syncthreads();
    for (int b = t; b < kScoreHistBins; b += NT) hist[b] = 0;
    __syncthreads();
#pragma unroll 4
    for (int e = w0 + lane; e < w1; e += 32) {
      const uint32_t kk = keys[e];
      if ((kk >> (32 - kScoreHistBits)) == cut)
        atomicAdd(&hist[(kk >> (32 - 2 * kScoreHistBits)) & (kScoreHistBins - 1)], 1u);
    }
    __syncthreads();
    HistView<NT> hv2;
    const uint32_t sc = hist_cutoff<NT>(hist, target - above, hv2, warp_sums, s_cut, s_total, s_big);
    if (above + s_total <= (uint32_t)CAP) {
      kcut |= sc << (32 - 2 * kScoreHistBits);
      C = above + s_total;
      refined = true;
    }
    __syncthreads();
  }
  const bool fits = C <= (uint32_t)CAP;
  const uint64_t* res = sorted;   // the sorted pairs, for the output loop at the end
  if (fits) {
    // The candidates are counted into sub-buckets while they are compacted -- bins
    // [cut, btop], each split into 2^sb sub-buckets on the key bits below the bin, sb as
    // large as kSubBuckets allows, numbered so that larger keys get smaller buckets -- then
    // one scan, one scatter into bucket order and a rank inside each bucket (a pair counts
    // the larger pairs of its bucket, mostly none) give every pair its output position,
    // which is written to idx / vals directly.
    const uint32_t nbins = btop - cut + 1;
    int sb = 0;
    while (sb < 20 && (nbins << (sb + 1)) <= (uint32_t)kSubBuckets) ++sb;
    auto bucket_of = [&](uint32_t key) -> uint32_t {   // key >= kcut, so its bin >= cut
      const uint32_t low = sb ? (key >> (32 - kScoreHistBits - sb)) & ((1u << sb) - 1u) : 0u;
      const uint32_t bin = min(key >> (32 - kScoreHistBits), btop);   // (a given histogram
      return ((btop - bin) << sb) | ((1u << sb) - 1u - low);           //  that disagrees)
    };
    uint32_t* sub = hist;   // the histogram is not read again on this path
    // Candidate slots: a region of kReg per warp, then a shared pool of the rest of cand,
    // then (when the key space holds CAP pairs past the row's keys and past the CAP pairs
    // the scatter writes at its start) a spill area there.  A pair that finds no slot
    // sends the row through the two-pass compaction.
    constexpr uint32_t kReg = (uint32_t)CAP * 7u / 10u / kWarps;
    constexpr uint32_t kPool = (uint32_t)CAP - kReg * kWarps;
    uint64_t* pool = cand + kReg * kWarps;
    const uint32_t kfree = (uint32_t)((hb + 4u * (uint32_t)n + 7u) / 8u);   // first free pair
    const uint32_t spill_cap =
        (hb == 0 && kfree >= (uint32_t)CAP && kfree + (uint32_t)CAP <= (uint32_t)RC::kKeyPairs)
            ? (uint32_t)CAP : 0u;
    uint64_t* spill = rbuf + kfree;
    for (uint32_t b = t; b < (uint32_t)kSubBuckets; b += NT) sub[bpad(b)] = 0;
    if (t == 0) s_spill = 0;
    __syncthreads();
    // one-pass compaction: warp w takes the row's key steps w, w + kWarps, ... (an even
    // sample of the row) and appends its candidates to its own region, then to the pool
    // and the spill area; every candidate is counted in its sub-bucket, stored or not
    // candidate of rank r in this warp's region: store it there, or at overflow slot o
    // (pool, then spill area) when r >= kReg
    auto put = [&](uint32_t r, uint32_t o, uint32_t key, int ee) {
      atomicAdd(&sub[bpad(bucket_of(key))], 1u);
      if (r < kReg)
        cand[warp * kReg + r] = compose(key, ee);
      else if (o < kPool)
        pool[o] = compose(key, ee);
      else if (o - kPool < spill_cap)
        spill[o - kPool] = compose(key, ee);
    };
    uint32_t wc = 0;
    if (hb == 0) {   // 128-key steps: lane l takes keys e .. e + 3
#pragma unroll 2
      for (int e0 = warp * 128; e0 < n; e0 += 128 * kWarps) {
        const int e = e0 + 4 * lane;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (e + 4 <= n) {
          v = *reinterpret_cast<const uint4*>(keys + e);
        } else {
          if (e < n) v.x = keys[e];
          if (e + 1 < n) v.y = keys[e + 1];
          if (e + 2 < n) v.z = keys[e + 2];
        }
        const bool t0 = e < n && v.x >= kcut, t1 = e + 1 < n && v.y >= kcut;
        const bool t2 = e + 2 < n && v.z >= kcut, t3 = e + 3 < n && v.w >= kcut;
        const uint32_t c = (uint32_t)t0 + (uint32_t)t1 + (uint32_t)t2 + (uint32_t)t3;
        // lane prefix of the counts from ballots of their bits
        const uint32_t b0 = __ballot_sync(0xffffffffu, c & 1u);
        const uint32_t b1 = __ballot_sync(0xffffffffu, c & 2u);
        const uint32_t b2 = __ballot_sync(0xffffffffu, c & 4u);
        uint32_t r = wc + __popc(b0 & below) + 2u * __popc(b1 & below) + 4u * __popc(b2 & below);
        const uint32_t step = __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
        // ranks at or past kReg overflow: one shared-counter add per warp step, each lane's
        // overflowing pairs in rank order after the lower lanes' ones
        uint32_t o = 0u;
        if (wc + step > kReg) {
          const uint32_t first = max(r, kReg), last = max(r + c, kReg);
          const uint32_t mine = last - first;   // 0 .. 4
          const uint32_t o0 = __ballot_sync(0xffffffffu, mine & 1u);
          const uint32_t o1 = __ballot_sync(0xffffffffu, mine & 2u);
          const uint32_t o2 = __ballot_sync(0xffffffffu, mine & 4u);
          const uint32_t tot = __popc(o0) + 2u * __popc(o1) + 4u * __popc(o2);
          uint32_t base = 0u;
          if (lane == 0) base = atomicAdd(&s_spill, tot);
          base = __shfl_sync(0xffffffffu, base, 0);
          o = base + __popc(o0 & below) + 2u * __popc(o1 & below) + 4u * __popc(o2 & below);
          o -= first - r;   // so that the pair of rank q >= kReg gets o + (q - r)
        }
        if (t0) { put(r, o, v.x, e); ++r; ++o; }
        if (t1) { put(r, o, v.y, e + 1); ++r; ++o; }
        if (t2) { put(r, o, v.z, e + 2); ++r; ++o; }
        if (t3) { put(r, o, v.w, e + 3); ++r; ++o; }
        wc += step;
      }
    } else {   // 32-key steps
#pragma unroll 4
      for (int e0 = warp * 32; e0 < n; e0 += 32 * kWarps) {
        const int e = e0 + lane;
        const uint32_t key = e < n ? keys[e] : 0u;
        const bool take = e < n && key >= kcut;
        const uint32_t m = __ballot_sync(0xffffffffu, take);
        const uint32_t r = wc + __popc(m & below);
        uint32_t o = 0u;
        if (take && r >= kReg) o = atomicAdd(&s_spill, 1u);
        if (take) put(r, o, key, e);
        wc += __popc(m);
      }
    }
    __syncthreads();
    const uint32_t novf = s_spill;                    // pairs past the regions
    const bool regions = novf <= kPool + spill_cap;
    const uint32_t npool = regions ? min(novf, kPool) : 0u;
    const uint32_t nspill = regions ? novf - npool : 0u;
    const uint32_t wreg = min(wc, kReg);              // pairs in this warp's region
    if (!regions) {
      // a region overflowed: the two-pass compaction (count per warp slice, block scan,
      // ballot ranks) into cand[0 .. C)
      if ((select && !given) || refined) {   // count this lane's candidates (else counted above)
        cnt = 0;
#pragma unroll 4
        for (int e = w0 + lane; e < w1; e += 32) cnt += keys[e] >= kcut ? 1u : 0u;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      uint32_t tot;
      uint32_t p = __shfl_sync(0xffffffffu,
                               block_excl_scan_nt<NT>(lane == 0 ? cnt : 0u, warp_sums, tot), 0);
      C = min(tot, (uint32_t)CAP);
#pragma unroll 4
      for (int e0 = w0; e0 < w1; e0 += 32) {
        const int e = e0 + lane;
        const uint32_t key = e < w1 ? keys[e] : 0u;
        const bool take = e < w1 && key >= kcut;
        const uint32_t m = __ballot_sync(0xffffffffu, take);
        const uint32_t r = p + __popc(m & below);
        if (take && r < (uint32_t)CAP) cand[r] = compose(key, e);   // (a histogram that
        p += __popc(m);                                            //  disagrees cannot overflow)
      }
    }
    // exclusive scan of the bucket counts (thread t owns a run of kSubBuckets / NT buckets);
    // the total is the number of candidates
    constexpr int kPer = kSubBuckets / NT;
    uint32_t c[kPer], local = 0, big = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      c[i] = sub[bpad(t * kPer + i)];
      local += c[i];
      big |= c[i] > kMaxBucket ? 1u : 0u;
    }
    uint32_t tot;
    uint32_t run = block_excl_scan_nt<NT>(local, warp_sums, tot);
    const bool crowded = __syncthreads_or(big ? 1 : 0);
    if (regions) C = tot;
    if (!crowded && tot == C) {
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        sub[bpad(t * kPer + i)] = run;   // bucket start, advanced to its end by the scatter
        run += c[i];
      }
      __syncthreads();
      // scatter into bucket order (the key space is dead: `sorted` takes the pairs)
      if (regions) {
        for (uint32_t i = lane; i < wreg; i += 32) {
          const uint64_t v = cand[warp * kReg + i];
          sorted[atomicAdd(&sub[bpad(bucket_of((uint32_t)(v >> 32)))], 1u)] = v;
        }
        for (uint32_t i = t; i < npool + nspill; i += NT) {
          const uint64_t v = i < npool ? pool[i] : spill[i - npool];
          sorted[atomicAdd(&sub[bpad(bucket_of((uint32_t)(v >> 32)))], 1u)] = v;
        }
      } else {
        for (uint32_t i = t; i < C; i += NT) {
          const uint64_t v = cand[i];
          sorted[atomicAdd(&sub[bpad(bucket_of((uint32_t)(v >> 32)))], 1u)] = v;
        }
      }
      __syncthreads();
      // rank inside the bucket -> output position; bucket b spans [end(b - 1), end(b)).
      // Four pairs per thread per step, so that their shared-memory chains overlap.
      for (uint32_t i0 = t; i0 < C; i0 += 4 * NT) {
        uint64_t v[4];
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = i0 + u * NT < C ? sorted[i0 + u * NT] : 0ull;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          o[u] = 0xffffffffu;
          if (i0 + u * NT < C) {
            const uint32_t b = bucket_of((uint32_t)(v[u] >> 32));
            const uint32_t s0 = b ? sub[bpad(b - 1)] : 0u, s1 = sub[bpad(b)];
            uint32_t r = 0;
            if (s1 - s0 > 1u)
              for (uint32_t j = s0; j < s1; ++j) r += sorted[j] > v[u] ? 1u : 0u;
            o[u] = s0 + r;
          }
        }
        int32_t id[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int32_t e = (int32_t)(~(uint32_t)(v[u] & 0xffffffffu));   // position in the row
          id[u] = (imap && o[u] < target) ? imap[e] : e;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (o[u] < target) {
            idx[row * topk + o[u]] = id[u];
            if (vals) vals[row * topk + o[u]] = key_score((uint32_t)(v[u] >> 32));
          }
      }
      for (int i = (int)target + t; i < topk; i += NT) {
        idx[row * topk + i] = -1;
        if (vals) vals[row * topk + i] = __int_as_float(0xff800000);
      }
      return;
    }
    // crowded buckets (many equal keys), or a count that disagrees with the compaction:
    // bitonic sort of the candidates instead
    if (regions) {
      if (lane == 0) warp_sums[warp] = wreg;
      __syncthreads();
      uint32_t pre = 0, all = 0;
      for (int w2 = 0; w2 < kWarps; ++w2) {
        if (w2 < warp) pre += warp_sums[w2];
        all += warp_sums[w2];
      }
      for (uint32_t i = lane; i < wreg && pre + i < (uint32_t)CAP; i += 32)
        sorted[pre + i] = cand[warp * kReg + i];
      for (uint32_t i = t; i < npool + nspill && all + i < (uint32_t)CAP; i += NT)
        sorted[all + i] = i < npool ? pool[i] : spill[i - npool];
    } else {
      for (uint32_t i = t; i < C; i += NT) sorted[i] = cand[i];
    }
    int sortn = NT;
    while ((uint32_t)sortn < C) sortn <<= 1;
    for (int i = (int)C + t; i < sortn; i += NT) sorted[i] = 0ull;
    __syncthreads();
    row_bitonic<NT, RC::kEMax>(sorted, sortn);
  } else {
    // crowded cutoff bin: exact threshold by a radix select over the resident keys, then
    // exactly `target` pairs (above the threshold, then equal ones in index order)
    uint32_t prefix = 0, mask = 0, kneed = target;
    for (int p = 0; p < 3; ++p) {
      const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
      const int nb = p == 2 ? 1024 : 2048;
      for (int b = t; b < 2048; b += NT) hist[b] = 0;
      __syncthreads();
      for (int e0 = 0; e0 < n; e0 += NT) {   // block-wide steps (warp-wide histogram adds)
        const int e = e0 + t;
        const uint32_t key = e < n ? keys[e] : 0u;
        warp_hist_add(hist, (key >> shift) & (nb - 1), e < n && (key & mask) == prefix);
      }
      __syncthreads();
      // suffix scan: thread t covers bins nb-1-kBinsPer*t-i, i < kBinsPer
      uint32_t cb[RC::kBinsPer], local = 0;
#pragma unroll
      for (int i = 0; i < RC::kBinsPer; ++i) {
        const int b = nb - 1 - RC::kBinsPer * t - i;
        cb[i] = b >= 0 ? hist[b] : 0u;
        local += cb[i];
      }
      uint32_t tot;
      const uint32_t excl = block_excl_scan_nt<NT>(local, warp_sums, tot);
      uint32_t run = excl;
#pragma unroll
      for (int i = 0; i < RC::kBinsPer; ++i) {
        if (run < kneed && kneed <= run + cb[i]) {
          s_digit = nb - 1 - RC::kBinsPer * t - i;
          s_above = run;
        }
        run += cb[i];
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= (uint32_t)(nb - 1) << shift;
      kneed -= s_above;
      __syncthreads();
    }
    const uint32_t thr = prefix;
    // Ranks in (warp, step, lane) order are ranks in index order: one block scan places
    // every warp's keys above the threshold and its equal ones.
    uint32_t ngt = 0, neq = 0;
    for (int e = w0 + lane; e < w1; e += 32) {
      const uint32_t key = keys[e];
      ngt += key > thr;
      neq += key == thr;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
      neq += __shfl_xor_sync(0xffffffffu, neq, o);
    }
    uint32_t tot;   // n <= kRowCap < 2^16: both counts fit 16 bits
    const uint32_t ex = block_excl_scan_nt<NT>(lane == 0 ? (ngt << 16) | neq : 0u, warp_sums, tot);
    const uint32_t wex = __shfl_sync(0xffffffffu, ex, 0);
    const uint32_t G = tot >> 16;   // keys above the threshold = target - kneed
    uint32_t gpos = wex >> 16, epos = wex & 0xffffu;
    for (int e0 = w0; e0 < w1; e0 += 32) {
      const int e = e0 + lane;
      const uint32_t key = e < w1 ? keys[e] : 0u;
      const bool gt = e < w1 && key > thr;
      const bool eq = e < w1 && key == thr;
      const uint32_t mg = __ballot_sync(0xffffffffu, gt);
      const uint32_t me = __ballot_sync(0xffffffffu, eq);
      if (gt) cand[gpos + __popc(mg & below)] = compose(key, e);
      if (eq) {
        const uint32_t r = epos + __popc(me & below);
        if (r < kneed) cand[G + r] = compose(key, e);
      }
      gpos += __popc(mg);
      epos += __popc(me);
    }
    C = target;
    cut = thr >> (32 - kScoreHistBits);
    btop = 0;
    for (int e = t; e < n; e += NT) btop = max(btop, keys[e] >> (32 - kScoreHistBits));
    uint32_t lo_dummy = 0xffffffffu;
    if (t == 0) { red[0] = 0xffffffffu; red[1] = 0; }
    __syncthreads();
    block_minmax<NT>(lo_dummy, btop, red);
    __syncthreads();
    // keys are dead from here on: their space is the sort's scratch
    res = cand;   // the counting sort leaves its result in place
    if (!group_sort_adaptive<NT>(cand, C, sorted, hist,
                                 reinterpret_cast<uint8_t*>(rbuf) + RC::kAuxOff, cut, btop,
                                 warp_sums, s_flag, s_nsub, nullptr)) {
      res = sorted;
      int sortn = NT;
      while ((uint32_t)sortn < C) sortn <<= 1;
      for (int i = t; i < sortn; i += NT) sorted[i] = (uint32_t)i < C ? cand[i] : 0ull;
      __syncthreads();
      row_bitonic<NT, RC::kEMax>(sorted, sortn);
    }
  }
  // outputs, four per thread per step so that the index-map loads overlap
  for (int i0 = t; i0 < topk; i0 += 4 * NT) {
    int32_t id[4];
    uint32_t key[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * NT;
      id[u] = -1;
      key[u] = 0u;
      if (i < topk && (uint32_t)i < target) {
        const uint64_t v = res[i];
        const int32_t e = (int32_t)(~(uint32_t)(v & 0xffffffffu));   // position in the row
        id[u] = imap ? imap[e] : e;
        key[u] = (uint32_t)(v >> 32);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * NT;
      if (i < topk) {
        const int64_t o = row * topk + i;
        const bool ok = (uint32_t)i < target;
        idx[o] = ok ? id[u] : -1;
        if (vals) vals[o] = ok ? key_score(key[u]) : __int_as_float(0xff800000);
      }
    }
  }
}

template <int NT, int CAP, int ROWCAP, int MINB>
cudaError_t launch_row(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                       const int32_t* gather_len, const int32_t* index_map, const uint32_t* ghist,
                       int rows, int topk, int32_t* idx, float* vals, int* status,
                       cudaStream_t st) {
  using RC = RowCfg<NT, CAP, ROWCAP>;
  cudaError_t e = cudaFuncSetAttribute(topk_row_kernel<NT, CAP, ROWCAP, MINB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RC::kSmem);
  if (e != cudaSuccess) return e;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    e = launch_pdl(topk_row_kernel<NT, CAP, ROWCAP, MINB>, dim3((unsigned)nr), dim3(NT),
                   RC::kSmem, st, scores, stride, pos, L, gather_len, index_map, ghist, topk, idx,
                   vals, status, row0);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

int topk_sort_size(int topk) {
  int s = kThreads;
  while (s < topk) s <<= 1;
  return s;
}

cudaError_t launch_topk_hist(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                             const uint32_t* hist, uint64_t* cand, uint32_t* gcount, int rows,
                             int topk, int32_t* idx, float* vals, int* status, cudaStream_t st) {
  if (L <= kLongRowCap && topk <= 3072)
    return launch_row<1024, 3072, kLongRowCap, 1>(scores, stride, pos, L, nullptr, nullptr, hist,
                                                  rows, topk, idx, vals, status, st);
  dim3 sgrid((unsigned)((L + kScatterChunk - 1) / kScatterChunk), (unsigned)rows);
  cudaError_t e = launch_pdl(topk_scatter_kernel, sgrid, dim3(kSelThreads), 0, st, scores, stride,
                             pos, L, hist, topk, cand, gcount);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)2 * kGroupBuf * sizeof(uint64_t);
  e = cudaFuncSetAttribute(topk_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(topk_group_kernel, dim3(hist_groups(topk), (unsigned)rows), dim3(kSelThreads), smem, st,
                 scores, stride, pos, L, hist, topk, (const uint64_t*)cand, idx, vals);
  if (e != cudaSuccess || topk <= kGroupExactMax) return e;   // the group kernel covers overflow rows
  const int sortn = topk_sort_size(topk);
  const size_t ov_smem = (size_t)sortn * sizeof(uint64_t);
  e = cudaFuncSetAttribute(topk_hist_overflow_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ov_smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_hist_overflow_kernel, dim3(rows), dim3(kThreads), ov_smem, st, scores,
                    stride, pos, L, hist, topk, sortn, idx, vals);
}

cudaError_t launch_build_hist(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                              int rows, uint32_t* hist, cudaStream_t st) {
  const dim3 grid((unsigned)((L + kScatterChunk - 1) / kScatterChunk), (unsigned)rows);
  return launch_pdl(topk_build_hist_kernel, grid, dim3(kSelThreads), 0, st, scores, stride, pos, L,
                    hist);
}

size_t topk_hist_zero_bytes(int64_t rows) {
  return align256((size_t)rows * kScoreHistBins * 4) + align256((size_t)rows * kMaxGroups * 4);
}

size_t topk_hist_ws_bytes(int64_t rows, int topk) {
  return align256((size_t)rows * kScoreHistBins * 4) + align256((size_t)rows * kMaxGroups * 4) +
         align256((size_t)rows * hist_groups(topk) * kGroupBuf * 8);
}

// Cluster size for rows of up to `len` scores, or 0 when the cluster form does not fit.
static int cluster_size_for(int64_t len, int sortn) {
  for (int G = 1; G <= 8; G <<= 1) {
    const int64_t slice = (((len + G - 1) / G) + 3) & ~int64_t(3);
    const int64_t smem = (int64_t)sortn * 8 + slice * 4;
    if ((slice <= kSliceTarget || G == 8) && smem <= kClusterSmemBudget) return G;
    if (G == 8) break;
  }
  return 0;
}

cudaError_t launch_topk(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                        const int32_t* gather_len, const int32_t* index_map, int rows,
                        int topk, int32_t* idx, float* vals, int* status, cudaStream_t st) {
  const int sortn = topk_sort_size(topk);
  const int64_t maxlen = gather_len ? stride : L;
  if (maxlen <= kRowCap && topk <= 8192) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (topk <= 3072 && rows >= 2 * sms)
      return launch_row<512, 3072, kRowCap, 2>(scores, stride, pos, L, gather_len, index_map,
                                               nullptr, rows, topk, idx, vals, status, st);
    if (rows >= sms)
      return launch_row<512, 8192, kRowCap, 1>(scores, stride, pos, L, gather_len, index_map,
                                               nullptr, rows, topk, idx, vals, status, st);
    return launch_row<1024, 8192, kRowCap, 1>(scores, stride, pos, L, gather_len, index_map,
                                              nullptr, rows, topk, idx, vals, status, st);
  }
  if (maxlen <= kLongRowCap && topk <= 3072)
    return launch_row<1024, 3072, kLongRowCap, 1>(scores, stride, pos, L, gather_len, index_map,
                                                  nullptr, rows, topk, idx, vals, status, st);
  const int G = cluster_size_for(maxlen, sortn);
  if (G > 0) {
    const int64_t slice = (((maxlen + G - 1) / G) + 3) & ~int64_t(3);
    const size_t smem = (size_t)sortn * 8 + (size_t)slice * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
      const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(nr * G), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = G;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const int64_t off_rows = row0;
      e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores + off_rows * stride, stride,
                             pos ? pos + off_rows : nullptr, L,
                             gather_len ? gather_len + off_rows : nullptr,
                             index_map ? index_map + off_rows * stride : nullptr, topk, sortn,
                             (int)slice, idx + off_rows * topk, vals ? vals + off_rows * topk : nullptr);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const size_t smem = (size_t)sortn * sizeof(uint64_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    topk_kernel<<<(unsigned)nr, kThreads, smem, st>>>(scores, stride, pos, L, gather_len,
                                                      index_map, topk, sortn, idx, vals, row0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace misa
