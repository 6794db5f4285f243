/*
 * misa.h -- C ABI of the B200 (sm_100a) MISA indexer library.
 *
 * The operations are those of "MISA: Mixture of Indexer Sparse Attention for
 * Long-Context LLM Inference" (picx.dev summary page, Methodology sections 1-2):
 * block pooling of indexer keys (Eq. 4), the block-pooled head router
 * (Eqs. 7-8), routed token scoring with top-k selection (Eqs. 9-10), the dense
 * DSA indexer the method replaces (Introduction, Eqs. 1-2), and the
 * hierarchical MISA-dagger re-rank (Eqs. 11-12).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every tensor pointer is a DEVICE pointer on the current CUDA
 *   device.  bf16 tensors are passed as their 16-bit patterns (uint16_t).
 *   q, k and k_pool must be 16-byte aligned; all tensors are dense, row-major
 *   (last index fastest), with no padding.
 * Shapes.  nseq independent sequences; T query rows per sequence; L keys per
 *   sequence; H = H^I indexer heads; d = head dim (only d = 128 is built);
 *   B = router block size; h = routed heads; topk = k; kprime = k'.
 *     q      bf16  [nseq, T, H, d]    indexer queries q^I
 *     w      fp32  [nseq, T, H]       head weights w^I
 *     k      bf16  [nseq, L, d]       indexer keys k^I (one key stream per sequence)
 *     pos    int32 [nseq, T]          absolute position of each query; query (n, t)
 *                                     sees keys s = 0 .. pos[n,t] (prefix P = pos+1)
 *     k_pool fp32  [nseq, ceil(L/B), d]
 *     heads  int32 [nseq, T, h]
 *     E      fp32  [nseq, T, H]
 *     idx    int32 [nseq, T, topk]    selected token indices
 *     vals   fp32  [nseq, T, topk]    their scores
 * Ownership.  The caller owns every buffer.  The library never allocates or
 *   frees device memory and keeps no state between calls.  Scratch space is a
 *   caller-provided workspace of at least misa_workspace_size(...) bytes; it must
 *   be zero-filled once after allocation (its first 256 bytes hold a sticky
 *   device status word) and must not be used by two calls that overlap on the GPU.
 * Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *   enqueue work; none of them synchronises, except misa_check_device_status.
 * Errors.  Every call returns a status (MISA_OK = 0).  Arguments are validated on
 *   the host before anything is enqueued; an invalid call enqueues nothing.
 *   Conditions only the GPU can see (a pos[] entry >= L, a candidate outside its
 *   query's prefix, a bounded wait that expired) are recorded in the workspace
 *   status word; the affected values are clamped or skipped, never read out of
 *   bounds.  misa_check_device_status() reports and clears that word.
 * Ordering.  idx rows list tokens by descending score, equal scores by ascending
 *   token index, and are padded with -1 (vals -inf) when fewer than topk tokens
 *   exist.  heads rows list heads by descending E, equal E by ascending head index.
 */
#ifndef MISA_B200_MISA_H
#define MISA_B200_MISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define MISA_OK                      0
#define MISA_ERR_INVALID_ARG         1  /* bad pointer, alignment, shape or parameter   */
#define MISA_ERR_UNSUPPORTED         2  /* valid but not built (e.g. d != 128)          */
#define MISA_ERR_CUDA                3  /* a CUDA runtime call or launch failed          */
#define MISA_ERR_DEVICE_TIMEOUT      4  /* a bounded device-side wait expired            */
#define MISA_ERR_WORKSPACE_TOO_SMALL 5  /* ws_bytes < misa_workspace_size(...)            */
#define MISA_ERR_BAD_DEVICE_INPUT    6  /* device data out of range (pos >= L, cand)     */
#define MISA_ERR_STATIC_SCRATCH_TOO_SMALL 7  /* call larger than the fixed scratch of
                                                misa_score_topk_noalloc                 */

/* Operation ids for misa_workspace_size. */
#define MISA_OP_ROUTE_HEADS   1
#define MISA_OP_SCORE_TOPK    2
#define MISA_OP_DSA_TOPK      3
#define MISA_OP_DAGGER_RERANK 4
#define MISA_OP_SCORE_ROWS    5
#define MISA_OP_HISA_TOPK     6

/* Limits of this build (larger values return MISA_ERR_UNSUPPORTED). */
#define MISA_HEAD_DIM        128
#define MISA_MAX_HEADS       128
#define MISA_MAX_ROUTED      128  /* h <= H <= MISA_MAX_HEADS */
#define MISA_MAX_TOPK        16384

/*
 * Bytes of workspace the operation `op` needs for these sizes (0 on invalid
 * arguments).  Arguments an operation does not use are ignored.  Host-only.
 */
size_t misa_workspace_size(int op, int nseq, int T, int H, int d, int64_t L, int B,
                           int h, int topk, int kprime);

/*
 * Block pooling of the indexer keys, Eq. (4) (Methodology section 1), with Pool
 * read as the arithmetic mean: k_pool[n, b, :] = mean of k[n, s, :] over
 * s in [b*B, min((b+1)*B, L)).  The last block may be partial and is then the
 * mean of its valid keys.  Output fp32 [nseq, ceil(L/B), d].  No workspace.
 */
int misa_pool_keys(const uint16_t* k, int nseq, int64_t L, int d, int B, float* k_pool,
                   void* stream);

/*
 * Refresh of the pooled keys after keys changed: recomputes, for every sequence,
 * exactly the blocks of Eq. (4) that meet the token range [s_begin, s_end) and
 * leaves every other block of k_pool as it is.  The pages count the router as
 * O(H * M) per query, which presumes the pooled keys are kept rather than rebuilt;
 * in decode a step appends one key, so the caller refreshes [pos, pos + 1) and only
 * that key's block is re-read (B keys instead of L).  Same layout as
 * misa_pool_keys; 0 <= s_begin <= s_end <= L, else MISA_ERR_INVALID_ARG; an empty
 * range launches nothing.  No workspace.
 */
int misa_pool_keys_range(const uint16_t* k, int nseq, int64_t L, int d, int B,
                         int64_t s_begin, int64_t s_end, float* k_pool, void* stream);

/*
 * Block-pooled head router, Eqs. (7)-(8) (Methodology section 1).  For query
 * (n, t) with prefix P = pos+1 and M = ceil(P/B) blocks of that prefix:
 *   A[j, b] = w[j] * ReLU(q[j] . kp_b),   E[j] = (1/M) * sum_b |A[j, b]|,
 *   heads   = the h largest E[j].
 * kp_b is k_pool[n, b] for blocks that lie wholly inside the prefix; when P is
 * not a multiple of B the last block is the mean of keys (M-1)*B .. P-1, read
 * from k.  E may be NULL.  Needs misa_workspace_size(MISA_OP_ROUTE_HEADS, ...).
 */
int misa_route_heads(const uint16_t* q, const float* w, const uint16_t* k,
                     const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                     int d, int64_t L, int B, int h, int32_t* heads, float* E, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * Routed token scoring and selection, Eqs. (9)-(10) (Methodology section 1):
 *   Ihat[s] = sum_{r < h} w[heads[r]] * ReLU(q[heads[r]] . k[s]),  s = 0 .. pos,
 *   idx = TopK_s(Ihat, topk).
 * With topk = k' this is also the MISA-dagger coarse stage, Eq. (11).  vals and
 * scores may be NULL; scores, when given, is fp32 [nseq, T, L] and receives Ihat
 * for s <= pos (later entries are left untouched).  Head ids outside [0, H) are
 * recorded as bad device input and skipped.
 * Needs misa_workspace_size(MISA_OP_SCORE_TOPK, ...).
 */
int misa_score_topk(const uint16_t* q, const float* w, const uint16_t* k,
                    const int32_t* heads, const int32_t* pos, int nseq, int T, int H,
                    int d, int64_t L, int h, int topk, int32_t* idx, float* vals,
                    float* scores, void* ws, size_t ws_bytes, void* stream);

/*
 * Dense DSA indexer, Eqs. (1)-(2) (Introduction): the same as misa_score_topk
 * with all H heads.  Needs misa_workspace_size(MISA_OP_DSA_TOPK, ...).
 */
int dsa_score_topk(const uint16_t* q, const float* w, const uint16_t* k,
                   const int32_t* pos, int nseq, int T, int H, int d, int64_t L, int topk,
                   int32_t* idx, float* vals, float* scores, void* ws, size_t ws_bytes,
                   void* stream);

/*
 * Token scores without selection: Eq. (9) over each query's prefix when heads is given
 * (h heads per query), Eq. (1) with all H heads when heads is NULL.  scores is fp32
 * [nseq, T, L]; entries s > pos are left untouched.  This is the scoring kernel of
 * misa_score_topk / dsa_score_topk on its own (same launch configuration), for callers
 * that select tokens themselves or inspect the scores.
 * Needs misa_workspace_size(MISA_OP_SCORE_ROWS, ...) (h = H when heads is NULL).
 */
int misa_score_rows(const uint16_t* q, const float* w, const uint16_t* k, const int32_t* heads,
                    const int32_t* pos, int nseq, int T, int H, int d, int64_t L, int h,
                    float* scores, void* ws, size_t ws_bytes, void* stream);

/*
 * MISA-dagger fine stage, Eq. (12) (Methodology section 2): for each query,
 * re-score the candidate tokens cand[n, t, 0 .. kprime-1] (int32, any order;
 * -1 = empty slot; a repeated id counts once) with all H heads,
 * I[s] = sum_j w[j] * ReLU(q[j] . k[s]), and return the topk best (ties: lower
 * token index).  Candidates outside [0, pos] are recorded as bad device input and
 * skipped.
 * Needs misa_workspace_size(MISA_OP_DAGGER_RERANK, ...).
 */
int misa_dagger_rerank(const uint16_t* q, const float* w, const uint16_t* k,
                       const int32_t* pos, const int32_t* cand, int nseq, int T, int H,
                       int d, int64_t L, int kprime, int topk, int32_t* idx, float* vals,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * HISA-style token-axis block filter, the variant the pages contrast MISA with
 * ("Key distinction from HISA", Methodology section 1; the HISA abstract's
 * block-level coarse filter followed by token-level refinement).  Both use the
 * router's affinities A[j, b] = w[j] * ReLU(q[j] . kp_b) over the blocks of the
 * query's prefix (partial last block as in misa_route_heads); this one reduces
 * them across heads, G[b] = sum_j A[j, b], keeps the m blocks with the largest G
 * (ties: lower b), scores the tokens of the kept blocks with all H heads (Eq. 1),
 * and returns their topk best in idx / vals (order and padding as elsewhere).
 * k_pool must hold the pooled keys for this B (misa_pool_keys).  blocks (nullable,
 * int32 [nseq, T, m]) receives the kept blocks by descending G, -1 padded.
 * 1 <= m, m * B <= MISA_MAX_TOPK.
 * Needs misa_workspace_size(MISA_OP_HISA_TOPK, ..., B, m (as h), topk, 0).
 */
int hisa_block_filter_topk(const uint16_t* q, const float* w, const uint16_t* k,
                           const float* k_pool, const int32_t* pos, int nseq, int T, int H,
                           int d, int64_t L, int B, int m, int topk, int32_t* idx, float* vals,
                           int32_t* blocks, void* ws, size_t ws_bytes, void* stream);

/*
 * misa_score_topk without any allocation or workspace.  The paper has no
 * counterpart of this entry point; it serves callers that cannot allocate device
 * memory or pass a workspace (code running inside an allocator-free region of a
 * serving engine, or a plugin whose host framework owns every allocation).
 *
 * Computes exactly what misa_score_topk computes (Ihat and its top-k; vals may be
 * NULL).  Its scratch is a fixed array inside the library's device image: 16 MiB
 * on every GPU that loads the library, held until the process exits, enough for
 * nseq * T * L <= 4,194,304 scores; larger calls return
 * MISA_ERR_STATIC_SCRATCH_TOO_SMALL and enqueue nothing.  All calls on a device
 * share that array and it keeps the last call's contents, so calls whose GPU work
 * overlaps (other streams, other host threads) race and must be serialised by the
 * caller.  Every call looks up the array's address with the caller's device
 * current; the first call on a device also loads the library there, so make it
 * before any stream capture.  Pointers are checked like misa_score_topk's (on the
 * current device, aligned, long enough); a bad one returns MISA_ERR_INVALID_ARG.  device_status (nullable,
 * device int32) receives this call's device-side status word (MISA_OK or
 * MISA_ERR_BAD_DEVICE_INPUT), as misa_check_device_status would report it.
 * Calls no cudaMalloc, cudaFree or allocating library routine.
 */
int misa_score_topk_noalloc(const uint16_t* q, const float* w, const uint16_t* k,
                            const int32_t* heads, const int32_t* pos, int nseq, int T, int H,
                            int d, int64_t L, int h, int topk, int32_t* idx, float* vals,
                            int32_t* device_status, void* stream);

/* Static text for a status code.  Host-only. */
const char* misa_status_string(int status);

/*
 * Synchronise `stream`, read the workspace status word, clear it, and return it
 * (MISA_OK when no device-side condition was recorded).
 */
int misa_check_device_status(void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MISA_B200_MISA_H */
