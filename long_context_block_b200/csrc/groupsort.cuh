// Descending sort of a small group of (key, index) pairs whose keys lie in a known range
// of histogram bins: a counting sort on the top bits of the key followed by insertion
// sorts of the (tiny) buckets.  Scores are continuous, so after 12 + sb key bits almost
// every bucket holds one or two pairs; a group whose largest bucket is too big is left
// to the caller's bitonic fallback.
#pragma once

#include <cstdint>

#include "internal.h"

namespace misa {

constexpr int kSubBuckets = 4096;     // counting-sort buckets per group
constexpr int kSubBucketWords = kSubBuckets + kSubBuckets / 32;   // padded: see bpad()
constexpr uint32_t kMaxBucket = 48;   // larger buckets -> bitonic fallback

// One padding word per 32 buckets, so that threads reading runs of 16 consecutive
// buckets hit distinct shared-memory banks.
__device__ __forceinline__ uint32_t bpad(uint32_t b) { return b + (b >> 5); }

// Bucket of pair `v` (key in the high 32 bits) for a group spanning bins [blo, blo+nb),
// numbered so that larger keys get smaller bucket numbers.
__device__ __forceinline__ uint32_t sub_bucket(uint64_t v, uint32_t blo, uint32_t nb, int sb) {
  const uint32_t key = (uint32_t)(v >> 32);
  const uint32_t bin = key >> (32 - kScoreHistBits);
  const uint32_t below = sb ? (key >> (32 - kScoreHistBits - sb)) & ((1u << sb) - 1u) : 0u;
  const uint32_t sub = ((bin - blo) << sb) | below;
  return (nb << sb) - 1u - sub;
}

// Sort in[0 .. cnt) (shared memory, unique pairs, keys in bins [blo, bhi]) into
// out[0 .. cnt) descending.  buckets: kSubBucketWords words of shared memory.  All NT
// threads must call it.  Returns false (leaving `out` unspecified) when a bucket holds
// more than kMaxBucket pairs.
template <int NT>
__device__ bool group_sort_desc(const uint64_t* in, uint32_t cnt, uint64_t* out,
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
  // insertion sort inside every bucket [end of previous bucket, end of this bucket)
  for (uint32_t b = t; b < nsub; b += NT) {
    const uint32_t e = buckets[bpad(b)];
    const uint32_t s = b ? buckets[bpad(b - 1)] : 0u;
    for (uint32_t i = s + 1; i < e; ++i) {
      const uint64_t v = out[i];
      uint32_t j = i;
      while (j > s && out[j - 1] < v) {
        out[j] = out[j - 1];
        --j;
      }
      out[j] = v;
    }
  }
  __syncthreads();
  return true;
}

}  // namespace misa
