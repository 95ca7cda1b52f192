/*
 * moshi_streams.c -- float64 CPU oracle for the token streams between the
 * Mimi codec and the Moshi language model: the delay-pattern packing of the
 * multi-stream frame, its inverse, and the Temporal Transformer's input (the
 * sum of one learned embedding per sub-stream).
 *
 * TEST INFRASTRUCTURE, like oracle.c: only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark use it; it shares nothing with the CUDA
 * library. Plain loops in index order; sums in float64.
 *
 * Sources (page title, section):
 *  [P2] "Moshi: a Speech-Text Foundation Model for Real-Time Dialogue"
 *       (notes), section 3c "Moshi - multi-stream generation": K = 17
 *       sub-streams per 12.5 Hz frame -- k1 text, k2 semantic and k3..k9
 *       acoustic of Moshi, k10 semantic and k11..k17 acoustic of the user --
 *       with the acoustic tokens delayed by tau = 1-2 steps behind the
 *       semantic one; the text token of a frame comes before its audio.
 *  [P3] Chinese annotated translation of the Moshi technical report:
 *       section "RQ-Transformer" (at step s the Temporal Transformer takes the
 *       sum of K learned embedding tables of the values of V_{s-1});
 *       section "Audio modeling", "acoustic delay" (a delay of 1 to 2 steps
 *       between semantic and acoustic features; the equation itself is lost
 *       in the page's extraction); section "Multi-stream modeling" (the delay
 *       is applied to both audio streams, which are then concatenated into V);
 *       the delay-pattern ablation (pattern [0,1,...,7]: every RVQ level one
 *       step after the previous, 8 steps = 640 ms; [0,2,...,2]: 240 ms;
 *       [0,0,...,0]: 80 ms, the least at 12.5 Hz; acoustic delay 1 in the
 *       final model: 160 ms theoretical latency).
 *
 * Readings taken where the pages are silent or garbled (stated, not hidden):
 *  - a delay shifts a stream later: with 0-based steps, V[s][k] = A[s - d_k][k]
 *    when 0 <= s - d_k < T, and the stream's pad token otherwise (before the
 *    stream starts and after it ends);
 *  - the text stream and the semantic stream have delay 0;
 *  - column order [text, Moshi q = 0..Q-1, user q = 0..Q-1] (K = 1 + 2Q);
 *  - the pad token of a stream is the id one past its vocabulary (32000 for
 *    text, 2048 for audio) and has its own embedding row;
 *  - a pattern's theoretical latency is (1 + max delay) frames;
 *  - embedding input: out[s] = sum over k, in order, of row V[s][k] of table k;
 *    a negative id is an absent sub-stream and adds nothing; an id past the
 *    table adds nothing and is counted.
 *
 * Layouts: row-major. text [T] int32; audio [n_audio][T][Q] int16; V [S][K]
 * int32; tables: the K tables' rows stacked, [sum rows_k][d], float32 or
 * bf16 bit patterns.
 */
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/*
 * Multi-stream frame: V [S][1 + n_audio * Q]. Column 0 is text[s] (delay 0)
 * or text_pad when s >= T or text is NULL; column 1 + a*Q + q is audio stream
 * a's level q shifted by delays[q], or audio_pad where no token exists.
 */
int oracle_delay_pack(const int32_t *text, const int16_t *audio, int n_audio, int64_t T, int Q,
                      const int32_t *delays, int64_t S, int32_t text_pad, int32_t audio_pad,
                      int32_t *V)
{
    if (T < 0 || S < 0 || Q <= 0 || n_audio < 0 || !delays || (S > 0 && !V) ||
        (n_audio > 0 && T > 0 && !audio))
        return ORACLE_EINVAL;
    for (int q = 0; q < Q; ++q)
        if (delays[q] < 0) return ORACLE_EINVAL;
    const int K = 1 + n_audio * Q;
    for (int64_t s = 0; s < S; ++s) {
        int32_t *row = V + s * K;
        row[0] = (text && s < T) ? text[s] : text_pad;
        for (int a = 0; a < n_audio; ++a)
            for (int q = 0; q < Q; ++q) {
                const int64_t t = s - delays[q];
                row[1 + a * Q + q] =
                    (t >= 0 && t < T) ? (int32_t)audio[((int64_t)a * T + t) * Q + q] : audio_pad;
            }
    }
    return ORACLE_OK;
}

/*
 * Inverse shift of one audio stream: audio [T][Q] from the Q columns of V
 * that start at col0: audio[t][q] = V[t + delays[q]][col0 + q]. Needs
 * T + max delay <= S.
 */
int oracle_delay_unpack(const int32_t *V, int64_t S, int K, int col0, int Q,
                        const int32_t *delays, int64_t T, int16_t *audio)
{
    if (S < 0 || T < 0 || K <= 0 || Q <= 0 || col0 < 0 || col0 + Q > K || !delays ||
        (T > 0 && (!V || !audio)))
        return ORACLE_EINVAL;
    for (int q = 0; q < Q; ++q)
        if (delays[q] < 0 || T + delays[q] > S) return ORACLE_EINVAL;
    for (int64_t t = 0; t < T; ++t)
        for (int q = 0; q < Q; ++q)
            audio[t * Q + q] = (int16_t)V[(t + delays[q]) * K + col0 + q];
    return ORACLE_OK;
}

/* Theoretical latency of a delay pattern: (1 + max delay) frames of frame_ms. */
double oracle_delay_latency_ms(const int32_t *delays, int Q, double frame_ms)
{
    int m = 0;
    for (int q = 0; q < Q; ++q)
        if (delays[q] > m) m = delays[q];
    return (1.0 + m) * frame_ms;
}

static double table_value(const void *tables, int dtype, int64_t idx)
{
    if (dtype == ORACLE_BF16) {
        uint32_t u = (uint32_t)((const uint16_t *)tables)[idx] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)tables)[idx];
}

/*
 * Temporal Transformer input: out[s][i] = sum_{k=0..K-1} E_k[V[s][k]][i] in
 * float64, k in order. rows [K] are the tables' row counts (stacked in that
 * order). Absent (negative) ids add nothing; ids >= rows[k] add nothing and
 * are counted in *n_bad (may be NULL).
 */
int oracle_embed_sum(const void *tables, int dtype, int K, const int64_t *rows, int d,
                     const int32_t *V, int64_t S, int nthreads, double *out, int64_t *n_bad)
{
    if (K <= 0 || d <= 0 || S < 0 || !rows || (dtype != ORACLE_F32 && dtype != ORACLE_BF16) ||
        (S > 0 && (!tables || !V || !out)))
        return ORACLE_EINVAL;
    int64_t offset[64];
    if (K > 64) return ORACLE_EINVAL;
    offset[0] = 0;
    for (int k = 1; k < K; ++k) offset[k] = offset[k - 1] + rows[k - 1];
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t s = 0; s < S; ++s) {
        double *o = out + s * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        for (int k = 0; k < K; ++k) {
            const int64_t id = V[s * K + k];
            if (id < 0) continue;
            if (id >= rows[k]) {
                ++bad;
                continue;
            }
            const int64_t base = (offset[k] + id) * (int64_t)d;
            for (int i = 0; i < d; ++i) o[i] += table_value(tables, dtype, base + i);
        }
    }
    if (n_bad) *n_bad = bad;
    return ORACLE_OK;
}
