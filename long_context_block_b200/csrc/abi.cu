// C ABI of the MISA indexer library: argument validation, workspace layout and the
// launch sequence of each entry point.  Declarations and contracts: include/misa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "misa.h"
#include "misa_testing.h"

using namespace misa;

namespace {

#define MISA_TRY(expr)            \
  do {                            \
    const int _s = (expr);        \
    if (_s != MISA_OK) return _s; \
  } while (0)

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MISA_OK : MISA_ERR_CUDA; }

// Shape checks shared by all query-side entry points (host-only, no CUDA calls).
int check_shape(int nseq, int T, int H, int d, int64_t L) {
  if (nseq < 1 || T < 1 || H < 1 || d < 1 || L < 1) return MISA_ERR_INVALID_ARG;
  if (L >= INT32_MAX || (int64_t)nseq * T >= INT32_MAX) return MISA_ERR_INVALID_ARG;
  if (d != MISA_HEAD_DIM || H > MISA_MAX_HEADS) return MISA_ERR_UNSUPPORTED;
  return MISA_OK;
}
int check_topk(int topk) {
  if (topk < 1) return MISA_ERR_INVALID_ARG;
  if (topk > MISA_MAX_TOPK) return MISA_ERR_UNSUPPORTED;
  return MISA_OK;
}

size_t route_ws(int nseq, int T, int H, int64_t L, int B) {
  if (route_tc_supported(nseq, T, H, L, B))
    return kStatusBytes + route_tc_ws_bytes(nseq, T, H, L, B);
  return kStatusBytes;   // the cluster router needs no scratch
}
// Rows up to this count whose length reaches kHistPathMinLen use the histogram-filtered
// top-k, fed by a score histogram built in the tensor-core scorer's epilogue.
constexpr int kHistPathMaxRows = 1024;
constexpr int64_t kHistPathMinLen = 8192;

bool hist_path(int nseq, int T, int64_t L, int nh) {
  return (int64_t)nseq * T <= kHistPathMaxRows && L >= kHistPathMinLen &&
         !score_tc_block_form(nh, T);
}
// Rows of several queries per sequence longer than the row top-k holds (16384 scores): the
// histogram comes from a separate pass over the scores instead of the scorer's epilogue.
constexpr int64_t kHistKernelMinLen = 16385;
bool hist_kernel_path(int nseq, int T, int64_t L, int nh) {
  return (int64_t)nseq * T <= kHistPathMaxRows && L >= kHistKernelMinLen &&
         score_tc_block_form(nh, T);
}

size_t score_ws(int nseq, int T, int64_t L, int nh, int topk) {
  const int64_t rows = (int64_t)nseq * T;
  return kStatusBytes + align256((size_t)rows * L * sizeof(float)) +
         score_tc_ws_bytes(nseq, T, nh) +
         (hist_path(nseq, T, L, nh) || hist_kernel_path(nseq, T, L, nh)
              ? topk_hist_ws_bytes(rows, topk) : 0);
}
size_t dagger_ws(int nseq, int T, int H, int kprime) {
  const size_t rows = (size_t)nseq * T;
  return kStatusBytes + 2 * align256(rows * kprime * sizeof(int32_t)) +
         align256(rows * sizeof(int32_t)) + score_tc_ws_bytes(nseq, T, H, true);
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws_bytes < need) return MISA_ERR_WORKSPACE_TOO_SMALL;
  return check_dev(ws, need, 256);
}

int* status_word(void* ws) { return reinterpret_cast<int*>(ws); }
char* ws_region(void* ws, size_t off) { return reinterpret_cast<char*>(ws) + kStatusBytes + off; }

}  // namespace

extern "C" {

size_t misa_workspace_size(int op, int nseq, int T, int H, int d, int64_t L, int B, int h,
                           int topk, int kprime) {
  if (check_shape(nseq, T, H, d, L) != MISA_OK) return 0;
  switch (op) {
    case MISA_OP_ROUTE_HEADS:
      if (B < 1 || h < 1 || h > H) return 0;
      return route_ws(nseq, T, H, L, B);
    case MISA_OP_SCORE_TOPK:
      if (h < 1 || h > H || check_topk(topk) != MISA_OK) return 0;
      return score_ws(nseq, T, L, h, topk);
    case MISA_OP_DSA_TOPK:
      if (check_topk(topk) != MISA_OK) return 0;
      return score_ws(nseq, T, L, H, topk);
    case MISA_OP_SCORE_ROWS:
      if (h < 1 || h > H) return 0;
      return kStatusBytes + score_tc_ws_bytes(nseq, T, h);
    case MISA_OP_DAGGER_RERANK:
      if (check_topk(topk) != MISA_OK || kprime < topk || kprime > MISA_MAX_TOPK) return 0;
      return dagger_ws(nseq, T, H, kprime);
    case MISA_OP_HISA_TOPK:   // h carries m
      if (B < 1 || h < 1 || (int64_t)h * B > MISA_MAX_TOPK || check_topk(topk) != MISA_OK)
        return 0;
      return kStatusBytes + hisa_ws_bytes(nseq, T, H, L, B, h);
    default:
      return 0;
  }
}

int misa_pool_keys(const uint16_t* k, int nseq, int64_t L, int d, int B, float* k_pool,
                   void* stream) {
  MISA_TRY(check_shape(nseq, 1, 1, d, L));
  if (B < 1) return MISA_ERR_INVALID_ARG;
  const int64_t M = (L + B - 1) / B;
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(k_pool, (size_t)nseq * M * d * 4, 16));
  return cuda_status(launch_pool_mean(k, nseq, L, B, k_pool, (cudaStream_t)stream));
}

int misa_pool_keys_range(const uint16_t* k, int nseq, int64_t L, int d, int B,
                         int64_t s_begin, int64_t s_end, float* k_pool, void* stream) {
  MISA_TRY(check_shape(nseq, 1, 1, d, L));
  if (B < 1 || s_begin < 0 || s_end < s_begin || s_end > L) return MISA_ERR_INVALID_ARG;
  const int64_t M = (L + B - 1) / B;
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(k_pool, (size_t)nseq * M * d * 4, 16));
  if (s_end == s_begin) return MISA_OK;
  return cuda_status(
      launch_pool_mean(k, nseq, L, B, k_pool, (cudaStream_t)stream, s_begin, s_end));
}

int misa_route_heads(const uint16_t* q, const float* w, const uint16_t* k, const float* k_pool,
                     const int32_t* pos, int nseq, int T, int H, int d, int64_t L, int B, int h,
                     int32_t* heads, float* E, void* ws, size_t ws_bytes, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  if (B < 1 || h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  const size_t rows = (size_t)nseq * T;
  const int64_t M = (L + B - 1) / B;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(k_pool, (size_t)nseq * M * d * 4, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  MISA_TRY(check_dev(heads, rows * h * 4, 4));
  MISA_TRY(check_opt(E, rows * H * 4, 4));
  MISA_TRY(check_ws(ws, ws_bytes, route_ws(nseq, T, H, L, B)));
  if (route_tc_supported(nseq, T, H, L, B))
    return cuda_status(launch_route_tc(q, w, k, k_pool, pos, nseq, T, H, L, B, h, heads, E,
                                       ws_region(ws, 0), status_word(ws), (cudaStream_t)stream));
  return cuda_status(launch_route(q, w, k, k_pool, pos, nseq, T, H, L, B, h, heads, E,
                                  status_word(ws), (cudaStream_t)stream));
}

static int score_topk_common(const uint16_t* q, const float* w, const uint16_t* k,
                             const int32_t* heads, int h, const int32_t* pos, int nseq, int T,
                             int H, int d, int64_t L, int topk, int32_t* idx, float* vals,
                             float* scores, void* ws, size_t ws_bytes, void* stream) {
  const size_t rows = (size_t)nseq * T;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  if (heads) MISA_TRY(check_dev(heads, rows * h * 4, 4));
  MISA_TRY(check_dev(idx, rows * topk * 4, 4));
  MISA_TRY(check_opt(vals, rows * topk * 4, 4));
  MISA_TRY(check_opt(scores, rows * L * 4, 4));
  const int nh = heads ? h : H;
  MISA_TRY(check_ws(ws, ws_bytes, score_ws(nseq, T, L, nh, topk)));
  cudaStream_t st = (cudaStream_t)stream;
  float* sc = scores ? scores : reinterpret_cast<float*>(ws_region(ws, 0));
  int* status = status_word(ws);
  if (score_tc_supported(nseq, T, nh, L)) {
    const size_t sc_bytes = align256(rows * L * sizeof(float));
    void* tc_scratch = ws_region(ws, sc_bytes);
    if (hist_path(nseq, T, L, nh) || hist_kernel_path(nseq, T, L, nh)) {
      char* hp = ws_region(ws, sc_bytes + score_tc_ws_bytes(nseq, T, nh));
      const size_t hb = align256(rows * kScoreHistBins * 4);
      uint32_t* hist = reinterpret_cast<uint32_t*>(hp);
      uint32_t* gcount = reinterpret_cast<uint32_t*>(hp + hb);
      uint64_t* cand = reinterpret_cast<uint64_t*>(hp + topk_hist_zero_bytes(rows));
      // the scorer's prep kernel zeroes the histogram and the group counts
      MISA_TRY(cuda_status(launch_score_tc(q, w, k, heads, h, pos, nseq, T, H, L, sc, L,
                                           tc_scratch, status, hist, st, nullptr, nullptr,
                                           nullptr, topk_hist_zero_bytes(rows))));
      if (!hist_path(nseq, T, L, nh))
        MISA_TRY(cuda_status(launch_build_hist(sc, L, pos, L, (int)rows, hist, st)));
      return cuda_status(launch_topk_hist(sc, L, pos, L, hist, cand, gcount, (int)rows, topk, idx,
                                          vals, status, st));
    }
    MISA_TRY(cuda_status(launch_score_tc(q, w, k, heads, h, pos, nseq, T, H, L, sc, L, tc_scratch,
                                         status, nullptr, st)));
  } else {
    MISA_TRY(cuda_status(launch_score_simt(q, w, k, heads, h, pos, nullptr, nullptr, nseq, T, H,
                                           L, sc, L, status, st)));
  }
  return cuda_status(launch_topk(sc, L, pos, L, nullptr, nullptr, (int)rows, topk, idx, vals,
                                 status, st));
}

int misa_score_topk(const uint16_t* q, const float* w, const uint16_t* k, const int32_t* heads,
                    const int32_t* pos, int nseq, int T, int H, int d, int64_t L, int h,
                    int topk, int32_t* idx, float* vals, float* scores, void* ws,
                    size_t ws_bytes, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  if (h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  if (h > MISA_MAX_ROUTED) return MISA_ERR_UNSUPPORTED;
  MISA_TRY(check_topk(topk));
  if (heads == nullptr) return MISA_ERR_INVALID_ARG;
  return score_topk_common(q, w, k, heads, h, pos, nseq, T, H, d, L, topk, idx, vals, scores,
                           ws, ws_bytes, stream);
}

int dsa_score_topk(const uint16_t* q, const float* w, const uint16_t* k, const int32_t* pos,
                   int nseq, int T, int H, int d, int64_t L, int topk, int32_t* idx,
                   float* vals, float* scores, void* ws, size_t ws_bytes, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  MISA_TRY(check_topk(topk));
  return score_topk_common(q, w, k, nullptr, H, pos, nseq, T, H, d, L, topk, idx, vals, scores,
                           ws, ws_bytes, stream);
}

int misa_score_rows(const uint16_t* q, const float* w, const uint16_t* k, const int32_t* heads,
                    const int32_t* pos, int nseq, int T, int H, int d, int64_t L, int h,
                    float* scores, void* ws, size_t ws_bytes, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  if (h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  if (heads && h > MISA_MAX_ROUTED) return MISA_ERR_UNSUPPORTED;
  const int nh = heads ? h : H;
  const size_t rows = (size_t)nseq * T;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  if (heads) MISA_TRY(check_dev(heads, rows * h * 4, 4));
  MISA_TRY(check_dev(scores, rows * L * 4, 4));
  const size_t need = kStatusBytes + score_tc_ws_bytes(nseq, T, nh);
  MISA_TRY(check_ws(ws, ws_bytes, need));
  cudaStream_t st = (cudaStream_t)stream;
  if (score_tc_supported(nseq, T, nh, L))
    return cuda_status(launch_score_tc(q, w, k, heads, h, pos, nseq, T, H, L, scores, L,
                                       ws_region(ws, 0), status_word(ws), nullptr, st));
  return cuda_status(launch_score_simt(q, w, k, heads, h, pos, nullptr, nullptr, nseq, T, H, L,
                                       scores, L, status_word(ws), st));
}

int misa_dagger_rerank(const uint16_t* q, const float* w, const uint16_t* k, const int32_t* pos,
                       const int32_t* cand, int nseq, int T, int H, int d, int64_t L, int kprime,
                       int topk, int32_t* idx, float* vals, void* ws, size_t ws_bytes,
                       void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  MISA_TRY(check_topk(topk));
  if (kprime < topk) return MISA_ERR_INVALID_ARG;
  if (kprime > MISA_MAX_TOPK) return MISA_ERR_UNSUPPORTED;
  const size_t rows = (size_t)nseq * T;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  MISA_TRY(check_dev(cand, rows * kprime * 4, 4));
  MISA_TRY(check_dev(idx, rows * topk * 4, 4));
  MISA_TRY(check_opt(vals, rows * topk * 4, 4));
  MISA_TRY(check_ws(ws, ws_bytes, dagger_ws(nseq, T, H, kprime)));
  cudaStream_t st = (cudaStream_t)stream;
  int* status = status_word(ws);
  const size_t ids_bytes = align256(rows * kprime * sizeof(int32_t));
  int32_t* sorted = reinterpret_cast<int32_t*>(ws_region(ws, 0));
  float* cscore = reinterpret_cast<float*>(ws_region(ws, ids_bytes));
  int32_t* count = reinterpret_cast<int32_t*>(ws_region(ws, 2 * ids_bytes));
  void* tc_scratch = ws_region(ws, 2 * ids_bytes + align256(rows * sizeof(int32_t)));
  MISA_TRY(cuda_status(
      launch_sort_candidates(cand, pos, (int)rows, L, kprime, sorted, count, status, st)));
  if (score_tc_supported(nseq, T, H, L, kprime))
    MISA_TRY(cuda_status(launch_score_tc(q, w, k, nullptr, H, pos, nseq, T, H, L, cscore, kprime,
                                         tc_scratch, status, nullptr, st, sorted, count)));
  else
    MISA_TRY(cuda_status(launch_score_simt(q, w, k, nullptr, H, pos, sorted, count, nseq, T, H,
                                           L, cscore, kprime, status, st)));
  return cuda_status(launch_topk(cscore, kprime, pos, L, count, sorted, (int)rows, topk, idx,
                                 vals, status, st));
}

int hisa_block_filter_topk(const uint16_t* q, const float* w, const uint16_t* k,
                           const float* k_pool, const int32_t* pos, int nseq, int T, int H, int d,
                           int64_t L, int B, int m, int topk, int32_t* idx, float* vals,
                           int32_t* blocks, void* ws, size_t ws_bytes, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  MISA_TRY(check_topk(topk));
  if (B < 1 || m < 1) return MISA_ERR_INVALID_ARG;
  if ((int64_t)m * B > MISA_MAX_TOPK) return MISA_ERR_UNSUPPORTED;
  const size_t rows = (size_t)nseq * T;
  const int64_t M = (L + B - 1) / B;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(k_pool, (size_t)nseq * M * d * 4, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  MISA_TRY(check_dev(idx, rows * topk * 4, 4));
  MISA_TRY(check_opt(vals, rows * topk * 4, 4));
  MISA_TRY(check_opt(blocks, rows * m * 4, 4));
  MISA_TRY(check_ws(ws, ws_bytes, kStatusBytes + hisa_ws_bytes(nseq, T, H, L, B, m)));
  return cuda_status(launch_hisa(q, w, k, k_pool, pos, nseq, T, H, L, B, m, topk, idx, vals,
                                 blocks, ws_region(ws, 0), status_word(ws), (cudaStream_t)stream));
}

const char* misa_status_string(int status) {
  switch (status) {
    case MISA_OK: return "ok";
    case MISA_ERR_INVALID_ARG: return "invalid argument";
    case MISA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MISA_ERR_CUDA: return "CUDA error";
    case MISA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MISA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MISA_ERR_BAD_DEVICE_INPUT: return "device input out of range (pos, head id or candidate)";
    case MISA_ERR_STATIC_SCRATCH_TOO_SMALL:
      return "call exceeds the fixed scratch of misa_score_topk_noalloc (nseq*T*L > 4194304)";
    default: return "unknown status";
  }
}

int misa_check_device_status(void* ws, void* stream) {
  if (ws == nullptr) return MISA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MISA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MISA_ERR_CUDA;
  if (v != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return MISA_ERR_CUDA;
  return v;
}

// ---------------------------------------------------------------- test-only entry points
// (declared in include/misa_testing.h)

int misa_testing_score_simt(const uint16_t* q, const float* w, const uint16_t* k,
                            const int32_t* heads, const int32_t* pos, const int32_t* gather_ids,
                            const int32_t* gather_len, int nseq, int T, int H, int d, int64_t L,
                            int h, int64_t out_stride, float* scores, void* ws, size_t ws_bytes,
                            void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  if (h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  const bool gather = gather_ids != nullptr;
  if (gather != (gather_len != nullptr)) return MISA_ERR_INVALID_ARG;
  if (out_stride < 1 || (!gather && out_stride < L) || out_stride >= INT32_MAX)
    return MISA_ERR_INVALID_ARG;
  const size_t rows = (size_t)nseq * T;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  if (heads) MISA_TRY(check_dev(heads, rows * h * 4, 4));
  if (gather) {
    MISA_TRY(check_dev(gather_ids, rows * out_stride * 4, 4));
    MISA_TRY(check_dev(gather_len, rows * 4, 4));
  }
  MISA_TRY(check_dev(scores, rows * out_stride * 4, 4));
  MISA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  return cuda_status(launch_score_simt(q, w, k, heads, h, pos, gather_ids, gather_len, nseq, T,
                                       H, L, scores, out_stride, status_word(ws),
                                       (cudaStream_t)stream));
}

int misa_testing_score_rows_wait_expiry(const uint16_t* q, const float* w, const uint16_t* k,
                                        const int32_t* heads, const int32_t* pos, int nseq,
                                        int T, int H, int d, int64_t L, int h, float* scores,
                                        void* ws, size_t ws_bytes, long long wait_cycles,
                                        int skip_tile, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  if (h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  if (wait_cycles < 1000 || wait_cycles > 4000000000LL || skip_tile < -1)
    return MISA_ERR_INVALID_ARG;
  const int nh = heads ? h : H;
  if (!score_tc_supported(nseq, T, nh, L)) return MISA_ERR_UNSUPPORTED;
  const size_t rows = (size_t)nseq * T;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  if (heads) MISA_TRY(check_dev(heads, rows * h * 4, 4));
  MISA_TRY(check_dev(scores, rows * L * 4, 4));
  MISA_TRY(check_ws(ws, ws_bytes, kStatusBytes + score_tc_ws_bytes(nseq, T, nh)));
  WaitProbe probe;
  probe.wait_cycles = wait_cycles;
  probe.skip_tile = skip_tile;
  return cuda_status(launch_score_tc(q, w, k, heads, h, pos, nseq, T, H, L, scores, L,
                                     ws_region(ws, 0), status_word(ws), nullptr,
                                     (cudaStream_t)stream, nullptr, nullptr, &probe));
}

int misa_testing_score_rows_timed(const uint16_t* q, const float* w, const uint16_t* k,
                                  const int32_t* heads, const int32_t* pos, int nseq, int T,
                                  int H, int d, int64_t L, int h, float* scores, void* ws,
                                  size_t ws_bytes, float* kernel_ms, void* stream) {
  MISA_TRY(check_shape(nseq, T, H, d, L));
  if (h < 1 || h > H || kernel_ms == nullptr) return MISA_ERR_INVALID_ARG;
  if (heads && h > MISA_MAX_ROUTED) return MISA_ERR_UNSUPPORTED;
  const int nh = heads ? h : H;
  if (!score_tc_supported(nseq, T, nh, L)) return MISA_ERR_UNSUPPORTED;
  const size_t rows = (size_t)nseq * T;
  MISA_TRY(check_dev(q, rows * H * d * 2, 16));
  MISA_TRY(check_dev(w, rows * H * 4, 4));
  MISA_TRY(check_dev(k, (size_t)nseq * L * d * 2, 16));
  MISA_TRY(check_dev(pos, rows * 4, 4));
  if (heads) MISA_TRY(check_dev(heads, rows * h * 4, 4));
  MISA_TRY(check_dev(scores, rows * L * 4, 4));
  MISA_TRY(check_ws(ws, ws_bytes, kStatusBytes + score_tc_ws_bytes(nseq, T, nh)));
  KernelTimer timer;
  MISA_TRY(cuda_status(cudaEventCreate(&timer.begin)));
  cudaError_t e = cudaEventCreate(&timer.end);
  if (e == cudaSuccess) {
    e = launch_score_tc(q, w, k, heads, h, pos, nseq, T, H, L, scores, L, ws_region(ws, 0),
                        status_word(ws), nullptr, (cudaStream_t)stream, nullptr, nullptr,
                        nullptr, 0, &timer);
    if (e == cudaSuccess) e = cudaEventSynchronize(timer.end);
    if (e == cudaSuccess) e = cudaEventElapsedTime(kernel_ms, timer.begin, timer.end);
    cudaEventDestroy(timer.end);
  }
  cudaEventDestroy(timer.begin);
  return cuda_status(e);
}

}  // extern "C"
