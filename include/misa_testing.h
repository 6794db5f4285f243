/*
 * misa_testing.h -- test-only entry points of the B200 MISA indexer library.
 *
 * These are not part of the indexer's API (include/misa.h).  Two of them exist so that a
 * test can reach code paths the ordinary entry points only take in rare conditions,
 * and compare them with an independent CPU reference:
 *   - the CUDA-core scorer, which misa_score_topk / dsa_score_topk / the MISA-dagger
 *     re-rank fall back to when the tensor-core scorer cannot take a shape (nseq * L
 *     at or above 2^31, or no driver entry point for tensor maps);
 *   - the expiry path of the tensor-core scorer's bounded waits: record
 *     MISA_ERR_DEVICE_TIMEOUT, let the copies and MMAs already in flight finish,
 *     free the tensor memory, and return, leaving the context usable.
 * The third times the tensor-core scoring kernel on its own, for the roofline of the
 * benchmark.
 * Conventions (pointers, layouts, ownership, workspace, status codes) are those of
 * include/misa.h.
 */
#ifndef MISA_B200_MISA_TESTING_H
#define MISA_B200_MISA_TESTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * The CUDA-core token scorer on its own.  Prefix mode (gather_ids NULL): for every
 * query row, scores[row * out_stride + s] = Eq. (9) under heads (h per row) or, with
 * heads NULL, Eq. (1) with all H heads, for s = 0 .. pos; out_stride >= L.  Gather mode
 * (gather_ids and gather_len both given): row r scores the tokens
 * gather_ids[r * out_stride + i], i < gather_len[r] (each in [0, L); others are
 * reported as bad device input and scored as token 0), into scores[r * out_stride + i].
 * ws: at least 256 bytes (the status word only), zero-filled.
 */
int misa_testing_score_simt(const uint16_t* q, const float* w, const uint16_t* k,
                            const int32_t* heads, const int32_t* pos,
                            const int32_t* gather_ids, const int32_t* gather_len, int nseq,
                            int T, int H, int d, int64_t L, int h, int64_t out_stride,
                            float* scores, void* ws, size_t ws_bytes, void* stream);

/*
 * misa_score_rows on the tensor-core scorer with every bounded wait shortened to
 * wait_cycles SM clock cycles (1000 .. 4e9) and, when skip_tile >= 0, the key tile
 * with that index (tiles of 128 keys, counted over the rows' prefixes laid end to
 * end) never loaded, so that the waits for it run out.  The scorer then records
 * MISA_ERR_DEVICE_TIMEOUT in the workspace status word (read it with
 * misa_check_device_status) and returns; the scores of the CTA that held the tile
 * are incomplete.  With skip_tile = -1 it computes exactly what misa_score_rows
 * computes.  Returns MISA_ERR_UNSUPPORTED where misa_score_rows would not use the
 * tensor-core scorer.  Workspace: misa_workspace_size(MISA_OP_SCORE_ROWS, ...).
 */
int misa_testing_score_rows_wait_expiry(const uint16_t* q, const float* w, const uint16_t* k,
                                        const int32_t* heads, const int32_t* pos, int nseq,
                                        int T, int H, int d, int64_t L, int h, float* scores,
                                        void* ws, size_t ws_bytes, long long wait_cycles,
                                        int skip_tile, void* stream);

/*
 * misa_score_rows on the tensor-core scorer, and the device time of its scoring kernel
 * alone: two CUDA events recorded on `stream` around that kernel's launch (after the
 * gather kernel that precedes it, which they leave out).  Blocks until the kernel has
 * finished, then writes the elapsed milliseconds to *kernel_ms (host memory).  Returns
 * MISA_ERR_UNSUPPORTED where misa_score_rows would not use the tensor-core scorer,
 * MISA_ERR_INVALID_ARG when kernel_ms is NULL.  Workspace: misa_workspace_size(
 * MISA_OP_SCORE_ROWS, ...).
 */
int misa_testing_score_rows_timed(const uint16_t* q, const float* w, const uint16_t* k,
                                  const int32_t* heads, const int32_t* pos, int nseq, int T,
                                  int H, int d, int64_t L, int h, float* scores, void* ws,
                                  size_t ws_bytes, float* kernel_ms, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MISA_B200_MISA_TESTING_H */
