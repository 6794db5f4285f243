// K7 (preparation): MISA-dagger candidate lists -- Eq. (12) of the MISA paper summary
// (Methodology section 2) re-scores the coarse candidates Omega_t with all heads and
// keeps the top k.  To make that final TopK resolve equal scores by token index with
// the ordinary index-order pass, each row's candidates are first put in ascending token
// order.  Empty slots (-1) and ids outside the query's prefix are dropped (the latter are
// recorded as bad device input); `count` receives the number of valid candidates.
//
// Omega_t is a set of token ids inside the prefix [0, P), so the ordering is a bitmap
// compaction: one bit per prefix token in shared memory, set by the candidates, then a
// block-wide scan of the words' popcounts writes the ids in ascending order (a repeated
// id counts once).  With few rows a row's prefix is split over a cluster of CTAs, each
// holding the bitmap of one slice of the prefix: every CTA reads all the row's candidates
// and keeps its slice's, and takes its output offset from the lower slices' counts over
// distributed shared memory.  Prefixes too long for a shared-memory bitmap take a bitonic
// sort.
#include <cooperative_groups.h>

#include "blocksort.cuh"
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = kSortThreads;
constexpr int kBitmapThreads = 512;
constexpr int kBitmapMaxBytes = 200 * 1024;

__global__ void __launch_bounds__(kBitmapThreads) bitmap_candidates_kernel(
    const int32_t* __restrict__ cand, const int32_t* __restrict__ pos, int64_t L, int kprime,
    int32_t* __restrict__ sorted, int32_t* __restrict__ count, int* status, int64_t row0) {
  pdl_prologue();
  extern __shared__ uint32_t bm[];   // [ceil(P / 32)] words
  __shared__ uint32_t warp_sums[kBitmapThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = row0 + blockIdx.x;
  const int P = prefix_len(pos, row, L, tid == 0 ? status : nullptr);
  const int nwords = (P + 31) >> 5;
  for (int i = tid; i < nwords; i += kBitmapThreads) bm[i] = 0u;
  __syncthreads();
  const int32_t* c_row = cand + row * kprime;
  for (int i = tid; i < kprime; i += kBitmapThreads) {
    const int32_t c = c_row[i];
    if (c >= 0 && c < P)
      atomicOr(&bm[c >> 5], 1u << (c & 31));
    else if (c != -1)
      set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
  }
  __syncthreads();
  // thread t owns words [t * per, (t + 1) * per)
  const int per = (nwords + kBitmapThreads - 1) / kBitmapThreads;
  const int w0 = min(tid * per, nwords), w1 = min(w0 + per, nwords);
  uint32_t local = 0;
  for (int i = w0; i < w1; ++i) local += __popc(bm[i]);
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t off = incl - local, total = 0;
  for (int w = 0; w < kBitmapThreads / 32; ++w) {
    const uint32_t s = warp_sums[w];
    if (w < warp) off += s;
    total += s;
  }
  int32_t* out = sorted + row * kprime;
  for (int i = w0; i < w1; ++i) {
    uint32_t b = bm[i];
    while (b) {
      const int bit = __ffs(b) - 1;
      out[off++] = i * 32 + bit;
      b &= b - 1u;
    }
  }
  for (int i = (int)total + tid; i < kprime; i += kBitmapThreads) out[i] = -1;
  if (tid == 0) count[row] = (int32_t)total;
}

// The cluster form: grid (slices, rows), a cluster of `gridDim.x` CTAs per row; CTA x holds
// the bitmap of prefix words [x * wps, (x + 1) * wps).
constexpr int kSliceMaxWords = 4096;   // 16 KB of bitmap per CTA
__global__ void __launch_bounds__(kBitmapThreads) bitmap_candidates_split_kernel(
    const int32_t* __restrict__ cand, const int32_t* __restrict__ pos, int64_t L, int kprime,
    int32_t* __restrict__ sorted, int32_t* __restrict__ count, int* status, int64_t row0) {
  pdl_prologue();
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ uint32_t bm[kSliceMaxWords];
  __shared__ uint32_t warp_sums[kBitmapThreads / 32];
  __shared__ uint32_t s_total;   // this slice's distinct candidates
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slices = (int)gridDim.x, slice = (int)blockIdx.x;
  const int64_t row = row0 + blockIdx.y;
  const int P = prefix_len(pos, row, L, tid == 0 && slice == 0 ? status : nullptr);
  const int nwords = (P + 31) >> 5;
  const int wps = (nwords + slices - 1) / slices;
  const int sw0 = min(slice * wps, nwords), sw1 = min(sw0 + wps, nwords);
  const int lo = sw0 * 32, hi = min(sw1 * 32, P);   // this slice's tokens [lo, hi)
  for (int i = tid; i < sw1 - sw0; i += kBitmapThreads) bm[i] = 0u;
  __syncthreads();
  const int32_t* c_row = cand + row * kprime;
  for (int i = tid; i < kprime; i += kBitmapThreads) {
    const int32_t c = c_row[i];
    if (c >= lo && c < hi)
      atomicOr(&bm[(c >> 5) - sw0], 1u << (c & 31));
    else if (slice == 0 && c != -1 && (c < 0 || c >= P))
      set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
  }
  __syncthreads();
  const int nw = sw1 - sw0;
  const int per = (nw + kBitmapThreads - 1) / kBitmapThreads;
  const int w0 = min(tid * per, nw), w1 = min(w0 + per, nw);
  uint32_t local = 0;
  for (int i = w0; i < w1; ++i) local += __popc(bm[i]);
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t off = incl - local, total = 0;
  for (int w = 0; w < kBitmapThreads / 32; ++w) {
    const uint32_t v = warp_sums[w];
    if (w < warp) off += v;
    total += v;
  }
  if (tid == 0) s_total = total;
  cluster.sync();   // every slice's count is set
  uint32_t below = 0, all = 0;   // distinct candidates in the lower slices, in all slices
  for (int r = 0; r < slices; ++r) {
    const uint32_t v = *cluster.map_shared_rank(&s_total, r);
    if (r < slice) below += v;
    all += v;
  }
  int32_t* out = sorted + row * kprime;
  off += below;
  for (int i = w0; i < w1; ++i) {
    uint32_t b = bm[i];
    while (b) {
      const int bit = __ffs(b) - 1;
      out[off++] = (sw0 + i) * 32 + bit;
      b &= b - 1u;
    }
  }
  if (slice == slices - 1) {
    for (int i = (int)all + tid; i < kprime; i += kBitmapThreads) out[i] = -1;
    if (tid == 0) count[row] = (int32_t)all;
  }
  cluster.sync();   // no CTA leaves while others may still read its count
}

__global__ void __launch_bounds__(kThreads) sort_candidates_kernel(
    const int32_t* __restrict__ cand, const int32_t* __restrict__ pos, int64_t L, int kprime,
    int sortn, int32_t* __restrict__ sorted, int32_t* __restrict__ count, int* status,
    int64_t row0) {
  extern __shared__ uint64_t buf[];   // [sortn]
  const int tid = threadIdx.x;
  const int64_t row = row0 + blockIdx.x;
  const int P = prefix_len(pos, row, L, tid == 0 ? status : nullptr);
  __shared__ int s_count;
  if (tid == 0) s_count = 0;
  __syncthreads();
  int valid_local = 0;
  // ascending token order = descending order of the complemented id; empty slots are 0
  for (int i = tid; i < sortn; i += kThreads) {
    uint64_t v = 0;
    if (i < kprime) {
      const int32_t c = cand[row * kprime + i];
      if (c >= 0 && c < P) {
        v = (uint64_t)(~(uint32_t)c) << 32;
        ++valid_local;
      } else if (c != -1) {
        set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
      }
    }
    buf[i] = v;
  }
  if (valid_local) atomicAdd(&s_count, valid_local);
  sort_buf_desc(buf, sortn);
  for (int i = tid; i < kprime; i += kThreads) {
    const uint64_t v = buf[i];
    sorted[row * kprime + i] = v ? (int32_t)(~(uint32_t)(v >> 32)) : -1;
  }
  if (tid == 0) count[row] = s_count;
}

}  // namespace

cudaError_t launch_sort_candidates(const int32_t* cand, const int32_t* pos, int rows,
                                   int64_t L, int kprime, int32_t* sorted, int32_t* count,
                                   int* status, cudaStream_t st) {
  const size_t bm_bytes = (size_t)((L + 31) / 32) * sizeof(uint32_t);
  const bool bitmap = bm_bytes <= (size_t)kBitmapMaxBytes;
  const int sortn = topk_sort_size(kprime);
  const size_t smem = bitmap ? bm_bytes : (size_t)sortn * sizeof(uint64_t);
  cudaError_t e = bitmap ? cudaFuncSetAttribute(bitmap_candidates_kernel,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem)
                         : cudaFuncSetAttribute(sort_candidates_kernel,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
  if (e != cudaSuccess) return e;
  // few rows: split each row's prefix over a cluster of up to 8 CTAs
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t words = (L + 31) / 32;
  int slices = 1;
  while (slices < 8 && (int64_t)rows * slices * 2 <= sms && words / (slices * 2) >= 256) slices *= 2;
  if (bitmap && slices > 1 && (words + slices - 1) / slices <= kSliceMaxWords) {
    for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
      const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)slices, (unsigned)nr, 1);
      cfg.blockDim = dim3(kBitmapThreads, 1, 1);
      cfg.dynamicSmemBytes = 0;
      cfg.stream = st;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)slices;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      e = cudaLaunchKernelEx(&cfg, bitmap_candidates_split_kernel, cand, pos, L, kprime, sorted,
                             count, status, row0);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    if (bitmap)
      e = launch_pdl(bitmap_candidates_kernel, dim3((unsigned)nr), dim3(kBitmapThreads), smem, st,
                     cand, pos, L, kprime, sorted, count, status, row0);
    else {
      sort_candidates_kernel<<<(unsigned)nr, kThreads, smem, st>>>(cand, pos, L, kprime, sortn,
                                                                   sorted, count, status, row0);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace misa
