// Host-side launchers shared between the kernel files and the C ABI layer.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace misa {

// Launch with programmatic dependent launch allowed: the kernel may be scheduled while the
// previous kernel in the stream finishes.  Every kernel launched this way starts with
// pdl_prologue() (common.cuh), which waits for the previous kernel's completion and writes
// before anything else, so stream order is kept.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Host checks of a caller's device buffer (validate.cu): non-null, `align`-aligned, on the
// current device, and at least `bytes` long when its allocation range can be queried.
// Return MISA_OK or MISA_ERR_INVALID_ARG.  check_opt accepts a null pointer.
int check_dev(const void* p, size_t bytes, size_t align);
int check_opt(const void* p, size_t bytes, size_t align);

// Workspace layout helpers: every region starts on a 256-byte boundary.
constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace header holding the sticky device status word.
constexpr size_t kStatusBytes = 256;

// Histogram of the top kScoreHistBits bits of the order-preserving score keys, used to
// cut long rows down to a small candidate set before the exact top-k.
constexpr int kScoreHistBits = 12;
constexpr int kScoreHistBins = 1 << kScoreHistBits;
// Candidate capacity per row of the histogram-filtered top-k.
constexpr int kTopkCandCap = 16384;

// Router: blocks of the prefix handled by one CTA of the partial-energy pass.
constexpr int kRouteChunk = 32;

// K1 -- mean pooling (pool.cu): every block, or only the blocks that meet the token range
// [s_begin, s_end) (s_end < 0: up to L).
cudaError_t launch_pool_mean(const uint16_t* k, int nseq, int64_t L, int B, float* k_pool,
                             cudaStream_t st, int64_t s_begin = 0, int64_t s_end = -1);

// K2 -- router (route.cu): a thread-block cluster per query row sums the head energies
// over chunks of the prefix's pooled blocks, then E and the top-h.  No scratch.
cudaError_t launch_route(const uint16_t* q, const float* w, const uint16_t* k,
                         const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                         int64_t L, int B, int h, int32_t* heads, float* E, int* status,
                         cudaStream_t st);

// K2 in block-score mode (route.cu), for the HISA-style filter: G[row, b] = sum_j
// w[row,j] * ReLU(q[row,j] . kp_b) for the blocks b < M_t of each query's prefix (row stride
// ceil(L/B)), and last_block[row] = M_t - 1.
cudaError_t launch_block_scores(const uint16_t* q, const float* w, const uint16_t* k,
                                const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                                int64_t L, int B, float* G, int32_t* last_block, int* status,
                                cudaStream_t st);

// K8 -- the HISA-style token-axis block filter (hisa.cu): block scores, top-m blocks, their
// tokens re-scored with all H heads, top-k.  Scratch: hisa_ws_bytes(...), 256-aligned.
size_t hisa_ws_bytes(int nseq, int T, int H, int64_t L, int B, int m);
cudaError_t launch_hisa(const uint16_t* q, const float* w, const uint16_t* k, const float* k_pool,
                        const int32_t* pos, int nseq, int T, int H, int64_t L, int B, int m,
                        int topk, int32_t* idx, float* vals, int32_t* blocks, void* scratch,
                        int* status, cudaStream_t st);

// K2 -- router on tcgen05 for sequences with many queries (route_tc.cu): the full-block
// part of Eq. (7) as a GEMM against the sequence's pooled keys (bf16 hi + lo, chunks of 256
// blocks), the partial block on CUDA cores, then the top-h.  needs route_tc_ws_bytes(...)
// of scratch.
bool route_tc_supported(int nseq, int T, int H, int64_t L, int B);
size_t route_tc_ws_bytes(int nseq, int T, int H, int64_t L, int B);
cudaError_t launch_route_tc(const uint16_t* q, const float* w, const uint16_t* k,
                            const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                            int64_t L, int B, int h, int32_t* heads, float* E, void* scratch,
                            int* status, cudaStream_t st);

// K4 -- token scoring on CUDA cores, any head subset (score_simt.cu).
//   heads == nullptr: all H heads (dense, Eq. 1); otherwise hsel heads per row (Eq. 9).
//   gather_ids != nullptr: score the tokens gather_ids[row, 0 .. gather_len[row]) instead
//   of the prefix 0 .. pos[row]; output row stride is `out_stride`.
cudaError_t launch_score_simt(const uint16_t* q, const float* w, const uint16_t* k,
                              const int32_t* heads, int hsel, const int32_t* pos,
                              const int32_t* gather_ids, const int32_t* gather_len,
                              int nseq, int T, int H, int64_t L, float* out,
                              int64_t out_stride, int* status, cudaStream_t st);

// K4 -- token scoring on tcgen05 tensor cores (score_tc.cu): rows streaming their own key
// prefix (decode form), or blocks of queries sharing key tiles (block form, when a
// sequence has enough queries).  Same contract as launch_score_simt; needs
// score_tc_ws_bytes(nseq, T, nh, gather) bytes of 256-aligned scratch.
//   span: 0 for prefix scoring, else the gather list stride (kprime).
bool score_tc_supported(int nseq, int T, int nh, int64_t L, int64_t span = 0);
bool score_tc_block_form(int nh, int T);
size_t score_tc_ws_bytes(int nseq, int T, int nh, bool gather = false);
//   hist (nullable): per-row kScoreHistBins-bin histogram of the written scores' keys,
//   accumulated in the epilogue (prefix decode form only; in the other forms it is left for
//   launch_build_hist); the scorer's prep kernel first zeroes hist_zero_bytes bytes (a
//   multiple of 16) from hist in every form.
//   gather_ids / gather_len (both or neither): row r scores the gather_len[r] tokens
//   gather_ids[r * out_stride + i] (each in [0, L)) into out[r * out_stride + i]; every
//   row takes the decode form and its keys are fetched four rows per TMA gather.
//   test_probe (nullable; tests only): a shorter bound for every wait of the scorer and
//   one key tile (global index in the CTAs' end-to-end tile order) that is never loaded,
//   so that a wait runs out and the expiry path (record MISA_ERR_DEVICE_TIMEOUT, let the
//   copies and MMAs in flight finish, free TMEM, return) runs.
struct WaitProbe {
  long long wait_cycles;
  int skip_tile;
};
//   timer (nullable; benchmark only): events recorded on st directly before and after the
//   scoring kernel's launch (after the prep kernel).
struct KernelTimer {
  cudaEvent_t begin;
  cudaEvent_t end;
};
cudaError_t launch_score_tc(const uint16_t* q, const float* w, const uint16_t* k,
                            const int32_t* heads, int hsel, const int32_t* pos, int nseq, int T,
                            int H, int64_t L, float* out, int64_t out_stride, void* scratch,
                            int* status, uint32_t* hist, cudaStream_t st,
                            const int32_t* gather_ids = nullptr,
                            const int32_t* gather_len = nullptr,
                            const WaitProbe* test_probe = nullptr,
                            size_t hist_zero_bytes = 0, const KernelTimer* timer = nullptr);

// K5 -- per-row top-k selection (topk.cu).
//   Row r has len = gather_len ? gather_len[r] : pos[r] + 1 scores at scores + r * stride.
//   index_map (nullable, same stride) gives the token id of each entry; the entries of a
//   row must then be in ascending token order (ties resolve by array order).
cudaError_t launch_topk(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                        const int32_t* gather_len, const int32_t* index_map, int rows,
                        int topk, int32_t* idx, float* vals, int* status, cudaStream_t st);

// K5 for long rows with a histogram of their scores (topk.cu).  Rows that fit one SM's
// shared memory (up to 40960 scores, k <= 3072) are selected by one CTA per row that takes
// the cutoff bin from the histogram; longer rows split the bins at or above the cutoff
// into groups of output positions: a scatter pass appends every candidate to its group's
// buffer and one CTA per group sorts and writes it.  hist: rows x kScoreHistBins;
// gcount: rows x 16 (zeroed, directly after hist); cand: topk_hist_ws_bytes layout.
cudaError_t launch_topk_hist(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                             const uint32_t* hist, uint64_t* cand, uint32_t* gcount, int rows,
                             int topk, int32_t* idx, float* vals, int* status, cudaStream_t st);
// The score histogram (kScoreHistBins bins per row, zeroed by the caller) of rows that the
// scorer did not histogram (topk.cu).  rows <= 65535.
cudaError_t launch_build_hist(const float* scores, int64_t stride, const int32_t* pos, int64_t L,
                              int rows, uint32_t* hist, cudaStream_t st);
// Scratch of the histogram path: histogram, group counts, group buffers (ceil(topk / 1024)
// groups of 8192 pairs per row), each region 256-aligned.
size_t topk_hist_ws_bytes(int64_t rows, int topk);
// Bytes at the start of that scratch which must be zero before the scores are histogrammed
// (the histogram and the group counts).
size_t topk_hist_zero_bytes(int64_t rows);

// Power-of-two length of the shared-memory sort buffer for `topk` entries (topk.cu).
int topk_sort_size(int topk);

// K7 -- MISA-dagger candidate preparation: sort each row's candidates ascending,
// drop empty / out-of-prefix slots, count the valid ones (rerank.cu).
cudaError_t launch_sort_candidates(const int32_t* cand, const int32_t* pos, int rows,
                                   int64_t L, int kprime, int32_t* sorted, int32_t* count,
                                   int* status, cudaStream_t st);

}  // namespace misa
