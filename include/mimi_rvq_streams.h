/*
 * mimi_rvq_streams.h -- the token streams between the Mimi codec and the
 * Moshi language model, on the GPU: delay-pattern packing of the multi-stream
 * frame, its inverse, and the sum of per-stream embeddings that is the
 * Temporal Transformer's input.
 *
 * Sources (page title, section):
 *  - "Moshi: a Speech-Text Foundation Model for Real-Time Dialogue" (notes),
 *    section 3c "Moshi - multi-stream generation": K = 17 sub-streams per
 *    12.5 Hz frame (k1 text; k2 semantic + k3..k9 acoustic of Moshi; k10
 *    semantic + k11..k17 acoustic of the user), acoustic tokens delayed by
 *    tau = 1-2 steps behind the semantic one, text before its audio.
 *  - Chinese annotated translation of the Moshi technical report: section
 *    "RQ-Transformer" (at step s the Temporal Transformer's input is the sum of
 *    K learned embedding tables of the tokens of step s - 1), "acoustic delay"
 *    and "multi-stream modeling" (the delay applies to both audio streams,
 *    which are concatenated), and the delay-pattern ablation ([0,1,...,7],
 *    [0,2,...,2], [0,0,...,0]).
 *
 * Readings (the delay equation is lost in the pages' extraction): with 0-based
 * steps, packed[s][k] = stream_k[s - delay_k] when 0 <= s - delay_k < T and the
 * stream's pad token otherwise; text and the semantic level have delay 0 (the
 * caller passes delays[0] = 0 for the standard patterns, but any delays >= 0
 * are accepted); columns are [text, stream 0 levels 0..7, stream 1 levels
 * 0..7]; pad tokens are one past each vocabulary (32000 text, 2048 audio) and
 * have their own embedding rows.
 *
 * All pointers are device pointers except where marked host; all arrays are
 * row-major and caller-owned, 16-byte aligned. Calls are asynchronous on
 * `stream` and allocate nothing. Status codes are those of mimi_rvq.h;
 * argument errors return at once, nothing is launched.
 */
#ifndef MIMI_RVQ_STREAMS_H
#define MIMI_RVQ_STREAMS_H

#include <stdint.h>

#include "mimi_rvq.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MIMI_RVQ_TEXT_CARD 32000  /* text vocabulary (SentencePiece, 32k) */
#define MIMI_RVQ_TEXT_PAD 32000   /* pad id of the text stream */
#define MIMI_RVQ_AUDIO_PAD 2048   /* pad id of an audio stream */
#define MIMI_RVQ_MAX_STREAMS 64   /* largest K for mimi_rvq_embed_sum */

/*
 * Pack T frames into the multi-stream sequence packed [S][K], K = 1 + 8 *
 * n_audio (17 for Moshi + user). text [T] int32 (NULL: every text slot is
 * text_pad); audio [n_audio][T][8] int16 codes (n_audio 0..7); delays: host
 * [8], delays[q] >= 0 steps for level q (the same pattern for every audio
 * stream). S >= 0 steps are written (T + max delay holds every token).
 * Returns MIMI_RVQ_EINVAL on a bad argument.
 */
int mimi_rvq_delay_pack(const int32_t *text, const int16_t *audio, int n_audio, int64_t T,
                        const int32_t *delays, int64_t S, int32_t text_pad, int32_t audio_pad,
                        int32_t *packed, struct CUstream_st *stream);

/*
 * Inverse shift of one audio stream: audio [T][8] int16 with audio[t][q] =
 * packed[t + delays[q]][col0 + q], from packed [S][K] (col0 + 8 <= K, T +
 * max delay <= S, else MIMI_RVQ_EINVAL). Values are copied as they are (a pad
 * token stays 2048, which mimi_rvq_decode then reports as out of range).
 */
int mimi_rvq_delay_unpack(const int32_t *packed, int64_t S, int K, int col0,
                          const int32_t *delays, int64_t T, int16_t *audio,
                          struct CUstream_st *stream);

/*
 * out[s] = sum over k = 0..K-1 of row tokens[s][k] of table k, for s < S.
 * tables: the K tables' rows stacked, [sum rows][d], MIMI_RVQ_F32 or
 * MIMI_RVQ_BF16 (table_dtype); rows: host [K] row counts; tokens [S][K] int32;
 * out [S][d], MIMI_RVQ_F32 or MIMI_RVQ_BF16 (out_dtype). d must be a multiple
 * of 8, K in 1..MIMI_RVQ_MAX_STREAMS. The sum is taken in float32, k in order.
 * A negative token is an absent stream and adds nothing; a token >= rows[k]
 * adds nothing and is counted into *n_bad (device uint64, caller-zeroed; may
 * be NULL).
 * Failure: the bf16, d = 4096 form waits on its copies with bounded waits
 * (about 2 s). If one runs out, the kernel stops, lets the copies it issued
 * land, and returns early (the output is then undefined); it records the
 * timeout in the library's token-stream status word, which
 * mimi_rvq_streams_get_error() reports, and also sets *n_bad to UINT64_MAX
 * when n_bad is not NULL.
 */
int mimi_rvq_embed_sum(const void *tables, int table_dtype, int K, const int64_t *rows, int d,
                       const int32_t *tokens, int64_t S, void *out, int out_dtype,
                       uint64_t *n_bad, struct CUstream_st *stream);

/*
 * Status of the token-stream kernels since the last call: synchronises
 * `stream`, then returns and clears the status word that a timed-out wait of
 * mimi_rvq_embed_sum sets (MIMI_RVQ_ETIMEOUT; MIMI_RVQ_OK if none; ECUDA if a
 * CUDA call fails). The word is shared by every caller in the process.
 */
int mimi_rvq_streams_get_error(struct CUstream_st *stream);

/*
 * Failure-path self-test of mimi_rvq_embed_sum's bounded waits, without
 * hanging or faulting the GPU: launches the embedding-sum kernel in a form
 * whose producers issue no copy, so its consumers' wait runs out a short
 * budget (about 50 ms); the kernel records the timeout and returns, and the
 * next mimi_rvq_streams_get_error returns MIMI_RVQ_ETIMEOUT. Needs no buffers.
 */
int mimi_rvq_streams_wait_selftest(struct CUstream_st *stream);

#ifdef __cplusplus
}
#endif

#endif /* MIMI_RVQ_STREAMS_H */
