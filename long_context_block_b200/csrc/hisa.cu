// K8: the HISA-style token-axis block filter, the variant the MISA page sets MISA against
// ("Key distinction from HISA", Methodology section 1): the router's affinities
// A[t,j,b] = w[t,j] * ReLU(q[t,j] . kp_b) are reduced across heads instead of across
// blocks, G[t,b] = sum_j A[t,j,b]; the m blocks with the largest G are kept, and the
// original all-head indexer (Eq. 1) scores only the tokens of those blocks, whose top k
// is the selection (the two-stage search of the HISA abstract).
//
// Launch sequence (every step on the GPU, no host synchronisation):
//   1. route_kernel in block-score mode: G [rows, Mpool] and each row's last block index;
//   2. top-m of G per row (the top-k kernels over rows of M_t block scores);
//   3. the kept blocks in ascending order (the candidate bitmap kernel of MISA-dagger);
//   4. hisa_expand_kernel: the kept blocks' tokens, ascending, and their count;
//   5. the all-head re-score of those tokens (the scorer's gather mode);
//   6. the top k over them, through the token index map.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

// Row r: the tokens of its kept blocks sb[r, 0 .. nb) (ascending block ids, nb =
// bcount[r]) laid end to end, B slots per block, into tok[r, :]; count[r] = the number of
// tokens inside the prefix.  Only the prefix's last block can be partial, and it is the
// last kept block when kept, so the valid tokens are a prefix of the row.
__global__ void __launch_bounds__(256) hisa_expand_kernel(
    const int32_t* __restrict__ sb, const int32_t* __restrict__ bcount, int m,
    const int32_t* __restrict__ pos, int64_t L, int B, int64_t span, int32_t* __restrict__ tok,
    int32_t* __restrict__ count, int64_t row0) {
  pdl_prologue();
  const int64_t row = row0 + blockIdx.x;
  const int P = prefix_len(pos, row, L, nullptr);
  const int nb = min(max(bcount[row], 0), m);
  const int32_t* blocks = sb + row * m;
  int32_t* out = tok + row * span;
  const int64_t nslots = (int64_t)nb * B;
  for (int64_t e = threadIdx.x; e < nslots; e += blockDim.x) {
    const int r = (int)(e / B), i = (int)(e - (int64_t)r * B);
    const int64_t s = (int64_t)blocks[r] * B + i;
    out[e] = s < P ? (int32_t)s : 0;   // slots past the prefix lie beyond `count`
  }
  if (threadIdx.x == 0) {
    int c = 0;
    if (nb > 0) {
      const int64_t last0 = (int64_t)blocks[nb - 1] * B;
      c = (nb - 1) * B + (int)min((int64_t)B, max((int64_t)0, (int64_t)P - last0));
    }
    count[row] = c;
  }
}

}  // namespace

size_t hisa_ws_bytes(int nseq, int T, int H, int64_t L, int B, int m) {
  const size_t rows = (size_t)nseq * T;
  const int64_t Mpool = (L + B - 1) / B;
  const size_t span = (size_t)m * B;
  return align256(rows * Mpool * 4) + 3 * align256(rows * 4) + 2 * align256(rows * m * 4) +
         2 * align256(rows * span * 4) + score_tc_ws_bytes(nseq, T, H, true);
}

cudaError_t launch_hisa(const uint16_t* q, const float* w, const uint16_t* k, const float* k_pool,
                        const int32_t* pos, int nseq, int T, int H, int64_t L, int B, int m,
                        int topk, int32_t* idx, float* vals, int32_t* blocks, void* scratch,
                        int* status, cudaStream_t st) {
  const int rows = nseq * T;
  const int64_t Mpool = (L + B - 1) / B;
  const int64_t span = (int64_t)m * B;
  char* c = reinterpret_cast<char*>(scratch);
  auto take = [&](size_t bytes) {
    char* p = c;
    c += align256(bytes);
    return p;
  };
  float* G = reinterpret_cast<float*>(take((size_t)rows * Mpool * 4));
  int32_t* last_block = reinterpret_cast<int32_t*>(take((size_t)rows * 4));
  int32_t* bcount = reinterpret_cast<int32_t*>(take((size_t)rows * 4));
  int32_t* count = reinterpret_cast<int32_t*>(take((size_t)rows * 4));
  int32_t* blk_ws = reinterpret_cast<int32_t*>(take((size_t)rows * m * 4));
  int32_t* sorted_blk = reinterpret_cast<int32_t*>(take((size_t)rows * m * 4));
  int32_t* tok = reinterpret_cast<int32_t*>(take((size_t)rows * span * 4));
  float* cscore = reinterpret_cast<float*>(take((size_t)rows * span * 4));
  void* tc_scratch = c;
  int32_t* blk = blocks ? blocks : blk_ws;

  cudaError_t e = launch_block_scores(q, w, k, k_pool, pos, nseq, T, H, L, B, G, last_block,
                                      status, st);
  if (e != cudaSuccess) return e;
  // row r holds M_t = last_block[r] + 1 block scores
  e = launch_topk(G, Mpool, last_block, Mpool, nullptr, nullptr, rows, m, blk, nullptr, status,
                  st);
  if (e != cudaSuccess) return e;
  e = launch_sort_candidates(blk, last_block, rows, Mpool, m, sorted_blk, bcount, status, st);
  if (e != cudaSuccess) return e;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    e = launch_pdl(hisa_expand_kernel, dim3((unsigned)nr), dim3(256), 0, st, sorted_blk, bcount,
                   m, pos, L, B, span, tok, count, row0);
    if (e != cudaSuccess) return e;
  }
  if (score_tc_supported(nseq, T, H, L, span))
    e = launch_score_tc(q, w, k, nullptr, H, pos, nseq, T, H, L, cscore, span, tc_scratch, status,
                        nullptr, st, tok, count);
  else
    e = launch_score_simt(q, w, k, nullptr, H, pos, tok, count, nseq, T, H, L, cscore, span,
                          status, st);
  if (e != cudaSuccess) return e;
  return launch_topk(cscore, span, pos, L, count, tok, rows, topk, idx, vals, status, st);
}

}  // namespace misa
