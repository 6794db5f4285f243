// Descending sort of a small group of (key, index) pairs whose keys lie in a known range
// of histogram bins: a counting sort on the top bits of the key, then every pair finds
// its place inside its bucket by counting the larger pairs there (all threads at once,
// so a crowded bucket does not serialise on one thread).  Scores are continuous, so after
// 12 + sb key bits almost every bucket holds one or two pairs; a group whose largest
// bucket is too big is left to the caller's bitonic fallback.
#pragma once

#include <cstdint>

#include "internal.h"

namespace misa {

constexpr int kSubBuckets = 4096;     // counting-sort buckets per group
constexpr int kSubBucketWords = kSubBuckets + kSubBuckets / 32;   // padded: see bpad()
constexpr uint32_t kMaxBucket = 256;   // larger buckets -> bitonic fallback

// One padding word per 32 buckets, so that threads reading runs of 16 consecutive
// buckets hit distinct shared-memory banks.
__device__ __forceinline__ uint32_t bpad(uint32_t b) { return b + (b >> 5); }

// After a counting-sort scatter: in[0 .. cnt) holds the pairs grouped by bucket (bucket b
// occupies [end[b-1], end[b]), `ends` read through bpad), unordered inside a bucket.  Every
// pair counts the larger pairs of its bucket and is written to out[start + rank]: out is
// sorted descending (pairs are unique).  bucket_of(v) recomputes the bucket of pair v.
template <int NT, typename BucketOf>
__device__ __forceinline__ void rank_in_buckets(const uint64_t* in, uint32_t cnt, uint64_t* out,
                                                const uint32_t* ends, BucketOf bucket_of) {
  for (uint32_t i = threadIdx.x; i < cnt; i += NT) {
    const uint64_t v = in[i];
    const uint32_t b = bucket_of(v);
    const uint32_t s = b ? ends[bpad(b - 1)] : 0u, e = ends[bpad(b)];
    uint32_t r = 0;
    for (uint32_t j = s; j < e; ++j) r += in[j] > v ? 1u : 0u;
    out[s + r] = v;
  }
}

// Bucket of pair `v` (key in the high 32 bits) for a group spanning bins [blo, blo+nb),
// numbered so that larger keys get smaller bucket numbers.
__device__ __forceinline__ uint32_t sub_bucket(uint64_t v, uint32_t blo, uint32_t nb, int sb) {
  const uint32_t key = (uint32_t)(v >> 32);
  const uint32_t bin = key >> (32 - kScoreHistBits);
  const uint32_t below = sb ? (key >> (32 - kScoreHistBits - sb)) & ((1u << sb) - 1u) : 0u;
  const uint32_t sub = ((bin - blo) << sb) | below;
  return (nb << sb) - 1u - sub;
}

// Sort in[0 .. cnt) (shared memory, unique pairs, keys in bins [blo, bhi]) descending;
// the result is in `in` (`out` is scratch of cnt pairs).  buckets: kSubBucketWords words of
// shared memory.  All NT threads must call it.  Returns false (both buffers unchanged)
// when a bucket holds more than kMaxBucket pairs.
template <int NT>
__device__ bool group_sort_desc(uint64_t* in, uint32_t cnt, uint64_t* out,
                                uint32_t* buckets, uint32_t blo, uint32_t bhi,
                                uint32_t* warp_sums, uint32_t& s_flag) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint32_t nb = bhi - blo + 1;
  int sb = 0;
  while (sb < 20 && (nb << (sb + 1)) <= (uint32_t)kSubBuckets) ++sb;
  const uint32_t nsub = nb << sb;
  for (uint32_t i = t; i < nsub; i += NT) buckets[bpad(i)] = 0;
  if (t == 0) s_flag = 0;
  __syncthreads();
  for (uint32_t i = t; i < cnt; i += NT) atomicAdd(&buckets[bpad(sub_bucket(in[i], blo, nb, sb))], 1u);
  __syncthreads();
  // exclusive scan of the bucket sizes; thread t owns a contiguous run of buckets
  constexpr int kPer = kSubBuckets / NT;
  uint32_t c[kPer], local = 0, big = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const uint32_t b = t * kPer + i;
    c[i] = b < nsub ? buckets[bpad(b)] : 0u;
    local += c[i];
    big |= c[i] > kMaxBucket;
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  if (big) s_flag = 1;
  __syncthreads();
  uint32_t run = 0;
  for (int w = 0; w < warp; ++w) run += warp_sums[w];
  run += incl - local;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const uint32_t b = t * kPer + i;
    if (b < nsub) buckets[bpad(b)] = run;   // bucket start, advanced to its end by the scatter
    run += c[i];
  }
  __syncthreads();
  if (s_flag) return false;
  for (uint32_t i = t; i < cnt; i += NT) {
    const uint64_t v = in[i];
    out[atomicAdd(&buckets[bpad(sub_bucket(v, blo, nb, sb))], 1u)] = v;
  }
  __syncthreads();
  rank_in_buckets<NT>(out, cnt, in, buckets,
                      [&](uint64_t v) { return sub_bucket(v, blo, nb, sb); });
  __syncthreads();
  return true;
}

}  // namespace misa

namespace misa {

// Bytes of shared memory group_sort_adaptive needs besides its bucket array: a word per
// histogram bin (candidate counts, then bucket offsets) and a byte per bin (sub-bucket
// bits).
constexpr int kAdaptiveAuxBytes = kScoreHistBins * 4 + kScoreHistBins;

// Descending sort like group_sort_desc, for candidates whose keys spread over many bins
// unevenly (rows whose cutoff reaches far down, or short rows taken whole): bin b of
// [blo, bhi] gets 2^s_b sub-buckets on the key bits below the bin, s_b chosen from the
// bin's own candidate count (about two pairs per sub-bucket) and lowered uniformly until
// the sub-buckets fit kSubBuckets.  `aux`: kAdaptiveAuxBytes of shared memory.
// bin_counts (nullable): the number of pairs in each histogram bin, indexed by bin, when
// the caller knows it exactly (every pair of bins [blo, bhi] is in `in`); it may be the
// same array as `buckets`.  Same contract (result in `in`) and fallback signal as
// group_sort_desc.
template <int NT>
__device__ bool group_sort_adaptive(uint64_t* in, uint32_t cnt, uint64_t* out,
                                    uint32_t* buckets, uint8_t* aux, uint32_t blo, uint32_t bhi,
                                    uint32_t* warp_sums, uint32_t& s_flag, uint32_t& s_tot,
                                    const uint32_t* bin_counts) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  constexpr int kWarps = NT / 32;
  constexpr int kPerB = kScoreHistBins / NT;   // bins per thread, highest bins first
  uint32_t* binw = reinterpret_cast<uint32_t*>(aux);   // counts, then bucket offsets
  uint8_t* bshift = aux + kScoreHistBins * 4;
  const uint32_t nb = bhi - blo + 1;
  if (bin_counts) {
    for (uint32_t i = t; i < nb; i += NT) binw[i] = bin_counts[blo + i];
    if (t == 0) s_flag = 0;
    __syncthreads();
  } else {
    for (uint32_t i = t; i < nb; i += NT) binw[i] = 0;
    if (t == 0) s_flag = 0;
    __syncthreads();
    for (uint32_t i = t; i < cnt; i += NT)
      atomicAdd(&binw[(uint32_t)(in[i] >> (64 - kScoreHistBits)) - blo], 1u);
    __syncthreads();
  }
  // Common case, at most one bin per thread: thread t sizes bin bhi - t (descending order)
  // and one block scan gives the offsets; when the wanted sub-buckets exceed kSubBuckets the
  // general path below lowers them uniformly.
  bool sized = false;
  if (nb <= (uint32_t)NT) {
    const uint32_t c = (uint32_t)t < nb ? binw[bhi - blo - t] : 0u;
    const int lg = c <= 2 ? 0 : 32 - __clz(c - 1);   // ceil(log2 c)
    const int sb = min(max(lg - 1, 0), 32 - kScoreHistBits);
    const uint32_t sz = (uint32_t)t < nb ? 1u << sb : 0u;
    uint32_t incl = sz;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    uint32_t run = incl - sz, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t x = warp_sums[w];
      if (w < warp) run += x;
      total += x;
    }
    __syncthreads();
    if (total <= (uint32_t)kSubBuckets) {
      if ((uint32_t)t < nb) {
        binw[bhi - blo - t] = run;
        bshift[bhi - blo - t] = (uint8_t)sb;
      }
      if (t == 0) s_tot = total;
      __syncthreads();
      sized = true;
    }
  }
  if (!sized) {
  // desired sub-bucket bits per bin: 2^s >= count / 2
  int s0[kPerB];
#pragma unroll
  for (int j = 0; j < kPerB; ++j) {
    const uint32_t p = t * kPerB + j;   // position in descending bin order
    const uint32_t c = p < nb ? binw[bhi - blo - p] : 0u;
    const int lg = c <= 2 ? 0 : 32 - __clz(c - 1);   // ceil(log2 c)
    s0[j] = min(max(lg - 1, 0), 32 - kScoreHistBits);
  }
  int delta = 0;
  for (;; ++delta) {
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < kPerB; ++j)
      if ((uint32_t)(t * kPerB + j) < nb) local += 1u << max(s0[j] - delta, 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    if (lane == 0) warp_sums[warp] = local;
    __syncthreads();
    uint32_t tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += warp_sums[w];
    __syncthreads();
    if (tot <= (uint32_t)kSubBuckets) break;   // nb <= kSubBuckets: ends by delta = 20
  }
  // bucket offsets in descending bin order
  uint32_t sz[kPerB], local = 0;
#pragma unroll
  for (int j = 0; j < kPerB; ++j) {
    const bool in_range = (uint32_t)(t * kPerB + j) < nb;
    s0[j] = max(s0[j] - delta, 0);
    sz[j] = in_range ? 1u << s0[j] : 0u;
    local += sz[j];
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t run = incl - local, total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t x = warp_sums[w];
    if (w < warp) run += x;
    total += x;
  }
  if (t == 0) s_tot = total;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPerB; ++j) {
    const uint32_t p = t * kPerB + j;
    if (p < nb) {
      binw[bhi - blo - p] = run;
      bshift[bhi - blo - p] = (uint8_t)s0[j];
    }
    run += sz[j];
  }
  __syncthreads();
  }   // !sized
  const uint32_t nsub = s_tot;
  auto bucket_of = [&](uint64_t v) -> uint32_t {
    const uint32_t key = (uint32_t)(v >> 32);
    const uint32_t b = (key >> (32 - kScoreHistBits)) - blo;
    const uint32_t s = bshift[b];
    const uint32_t sub = s ? (key >> (32 - kScoreHistBits - s)) & ((1u << s) - 1u) : 0u;
    return binw[b] + ((1u << s) - 1u - sub);   // larger keys -> smaller bucket numbers
  };
  for (uint32_t i = t; i < nsub; i += NT) buckets[bpad(i)] = 0;
  __syncthreads();
  for (uint32_t i = t; i < cnt; i += NT) atomicAdd(&buckets[bpad(bucket_of(in[i]))], 1u);
  __syncthreads();
  constexpr int kPer = kSubBuckets / NT;
  uint32_t c[kPer], lsum = 0, big = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const uint32_t b = t * kPer + i;
    c[i] = b < nsub ? buckets[bpad(b)] : 0u;
    lsum += c[i];
    big |= c[i] > kMaxBucket;
  }
  uint32_t incl2 = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl2, o);
    if (lane >= o) incl2 += v;
  }
  if (lane == 31) warp_sums[warp] = incl2;
  if (big) s_flag = 1;
  __syncthreads();
  uint32_t r2 = 0;
  for (int w = 0; w < warp; ++w) r2 += warp_sums[w];
  r2 += incl2 - lsum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const uint32_t b = t * kPer + i;
    if (b < nsub) buckets[bpad(b)] = r2;
    r2 += c[i];
  }
  __syncthreads();
  if (s_flag) return false;
  for (uint32_t i = t; i < cnt; i += NT) {
    const uint64_t v = in[i];
    out[atomicAdd(&buckets[bpad(bucket_of(v))], 1u)] = v;
  }
  __syncthreads();
  rank_in_buckets<NT>(out, cnt, in, buckets, bucket_of);
  __syncthreads();
  return true;
}

}  // namespace misa
