/*
 * oracle.c -- float64 CPU oracle for the split residual vector quantiser
 * (split RVQ) at the bottleneck of the Mimi audio codec.
 *
 * TEST INFRASTRUCTURE. This file exists only so that tests, the smoke check
 * and the CPU-baseline leg of the benchmark can check the CUDA library
 * against a plain definition. The product path never links, loads or calls
 * it, and it shares no code, header, table or helper with the CUDA library.
 *
 * It is written to be read against the pages, not to be fast: every input is
 * widened exactly to IEEE float64, every distance is a direct sum of squared
 * differences in index order, and the only parallelism is one frame per
 * OpenMP iteration (frames are independent). Built with -ffp-contract=off so
 * that no multiply-add is fused behind the reader's back.
 *
 * Sources (page title, section):
 *  [P1] "Voice multimodal: Moshi, 200 ms, can interrupt" (mizuki-eaf blog),
 *       section 3 "Mimi: compressing 24 kHz sound to 12.5 Hz tokens":
 *       24 kHz in, 12.5 Hz tokens, 1.1 kbps; codebook 1 semantic, the 7 after
 *       it acoustic.
 *  [P2] "Moshi: a Speech-Text Foundation Model for Real-Time Dialogue"
 *       (notes), section 2 "Building blocks" (each RVQ codebook quantises the
 *       previous one's residual) and section 3a "Mimi - the audio codec"
 *       (latent 512 projected to 256 before the RVQ; split RVQ, 8 codebooks
 *       of 2048; outputs summed; strides 4,5,6,8 and a final 2).
 *  [P3] Chinese annotated translation of the Moshi technical report,
 *       section "Architecture" (the RVQ applies VQ iteratively to the residual
 *       of the previous quantiser, N_A centroids per codebook, codes in
 *       {1..N_A}), section "Quantization rate" (Q = 8, N_A = 2048, 1.1 kbps,
 *       the "Lin" projection 512->256 before the RVQ and back to 512 before
 *       decoding, quantizer dropout), section "Learning semantic-acoustic
 *       tokens with split RVQ" (a plain VQ for semantics and a 7-level RVQ
 *       applied in parallel, outputs added), intro table of codec bit-rates.
 *
 * Readings taken where the pages are silent (stated, not hidden):
 *  - distance is squared Euclidean (nearest centroid);
 *  - ties go to the lowest index (the first minimum in index order);
 *  - one shared W_in and one W_out, no bias;
 *  - codes are 0-based, i.e. the report's {1..N_A} minus one;
 *  - code column 0 is the semantic codebook, columns 1..7 the acoustic levels;
 *  - by default the acoustic RVQ quantises y itself, side by side with the
 *    semantic VQ ([P3] split RVQ); variant 1 lets it quantise y - S_s, what
 *    the semantic VQ leaves over (the other reading of [P2] 3a).
 *
 * Layouts: row-major. z [N][D_in] (fp32 or bf16 bit patterns), W_in [D][D_in],
 * C [Q][K][D] (codebook 0 semantic, 1..Q-1 acoustic), W_out [D_out][D],
 * codes [N][n_q] int16.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ERANGE 2

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double latent_at(const void *z, int dtype, int64_t idx)
{
    if (dtype == ORACLE_BF16)
        return widen_bf16(((const uint16_t *)z)[idx]);
    return (double)((const float *)z)[idx];
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Threads an OpenMP parallel region would use with the given request. */
int oracle_threads(int nthreads)
{
#ifdef _OPENMP
    set_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/*
 * y = W_in . z for one frame: the "Lin" 512 -> 256 of [P3] "Quantization
 * rate" and [P2] 3a (the 512-d latent is mapped to 256-d ahead of the RVQ).
 * Sum over j in index order.
 */
static void project_one(const void *z, int dtype, int64_t frame, int D_in, int D,
                        const float *W_in, double *y)
{
    for (int i = 0; i < D; ++i) {
        double acc = 0.0;
        const float *w = W_in + (size_t)i * D_in;
        for (int j = 0; j < D_in; ++j)
            acc += (double)w[j] * latent_at(z, dtype, frame * D_in + j);
        y[i] = acc;
    }
}

/*
 * Nearest codeword of one codebook to r: the VQ step of [P3] "Architecture"
 * (nearest of N_A centroids). d_k = sum_i (r_i - c_k,i)^2, the first k with
 * the smallest d_k wins. Also reports the best distance and the second
 * smallest distance over the other indices (equal to the best on an exact
 * tie; +inf when K == 1).
 */
static int nearest_one(const double *r, const float *book, int K, int D,
                       double *d_best, double *d_second)
{
    int best = 0;
    double db = INFINITY, ds = INFINITY;
    for (int k = 0; k < K; ++k) {
        const float *c = book + (size_t)k * D;
        double d = 0.0;
        for (int i = 0; i < D; ++i) {
            double t = r[i] - (double)c[i];
            d += t * t;
        }
        if (d < db) {
            ds = db;
            db = d;
            best = k;
        } else if (d < ds) {
            ds = d;
        }
    }
    *d_best = db;
    *d_second = ds;
    return best;
}

/*
 * Split RVQ of one projected latent y [D]:
 *  codebook 0 (semantic, a plain VQ on y)           -- [P3] split RVQ, [P1] 3
 *  codebooks 1..n_q-1 (acoustic RVQ, greedy):        -- [P2] 2, [P3] Architecture
 *      r_0 = y        (variant 0: side by side with the semantic VQ, [P3])
 *      r_0 = y - S_s  (variant 1: on what the semantic VQ leaves, [P2] 3a)
 *      a_l = nearest(r_{l-1}, codebook l);  r_l = r_{l-1} - codebook l [a_l]
 * n_q < Q keeps only the first n_q codebooks (quantizer dropout at inference,
 * [P3] "Quantization rate"). codes, d_best, d_second point at this frame's
 * n_q entries; the distance pointers may be NULL. r is caller scratch [D].
 */
static void split_rvq_one(const double *y, int D, int K, const float *C, int n_q,
                          int variant, double *r, int16_t *codes, double *d_best,
                          double *d_second)
{
    double db, ds;
    int s = nearest_one(y, C, K, D, &db, &ds);
    codes[0] = (int16_t)s;
    if (d_best) d_best[0] = db;
    if (d_second) d_second[0] = ds;

    const float *S_s = C + (size_t)s * D;
    for (int i = 0; i < D; ++i)
        r[i] = variant == 1 ? y[i] - (double)S_s[i] : y[i];

    for (int l = 1; l < n_q; ++l) {
        const float *book = C + (size_t)l * K * D;
        int a = nearest_one(r, book, K, D, &db, &ds);
        codes[l] = (int16_t)a;
        if (d_best) d_best[l] = db;
        if (d_second) d_second[l] = ds;
        const float *A_a = book + (size_t)a * D;
        for (int i = 0; i < D; ++i)
            r[i] -= (double)A_a[i];
    }
}

/* Split RVQ on projected latents y [N][D] -> codes [N][n_q] (and distances). */
int oracle_encode_projected(const double *y, int64_t N, int D, int K, int Q,
                            const float *C, int n_q, int variant, int nthreads,
                            int16_t *codes, double *d_best, double *d_second)
{
    if (N < 0 || D <= 0 || D > 4096 || K <= 0 || K > 32768 || Q <= 0 || n_q <= 0 ||
        n_q > Q || (variant != 0 && variant != 1) || (N > 0 && (!y || !C || !codes)))
        return ORACLE_EINVAL;
    set_threads(nthreads);
#pragma omp parallel
    {
        double r[4096];
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < N; ++n)
            split_rvq_one(y + (size_t)n * D, D, K, C, n_q, variant, r, codes + n * n_q,
                          d_best ? d_best + n * n_q : NULL,
                          d_second ? d_second + n * n_q : NULL);
    }
    return ORACLE_OK;
}

/* y = W_in . z for every frame; y [N][D]. */
int oracle_project(const void *z, int dtype, int64_t N, int D_in, int D,
                   const float *W_in, int nthreads, double *y)
{
    if (N < 0 || D_in <= 0 || D <= 0 || (dtype != ORACLE_F32 && dtype != ORACLE_BF16) ||
        (N > 0 && (!z || !W_in || !y)))
        return ORACLE_EINVAL;
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        project_one(z, dtype, n, D_in, D, W_in, y + (size_t)n * D);
    return ORACLE_OK;
}

/*
 * Full encode: latents z [N][D_in] -> codes [N][n_q]. The projection and the
 * split RVQ above, one frame at a time. y_out [N][D] may be NULL.
 */
int oracle_encode(const void *z, int dtype, int64_t N, int D_in, int D, int K, int Q,
                  const float *W_in, const float *C, int n_q, int variant, int nthreads,
                  int16_t *codes, double *d_best, double *d_second, double *y_out)
{
    if (N < 0 || D_in <= 0 || D <= 0 || D > 4096 || K <= 0 || K > 32768 || Q <= 0 ||
        n_q <= 0 || n_q > Q || (variant != 0 && variant != 1) ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16) ||
        (N > 0 && (!z || !W_in || !C || !codes)))
        return ORACLE_EINVAL;
    set_threads(nthreads);
#pragma omp parallel
    {
        double y[4096], r[4096];
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < N; ++n) {
            project_one(z, dtype, n, D_in, D, W_in, y);
            if (y_out)
                memcpy(y_out + (size_t)n * D, y, sizeof(double) * (size_t)D);
            split_rvq_one(y, D, K, C, n_q, variant, r, codes + n * n_q,
                          d_best ? d_best + n * n_q : NULL,
                          d_second ? d_second + n * n_q : NULL);
        }
    }
    return ORACLE_OK;
}

/*
 * Decode: q = S_s + sum_{l=1..n_q-1} A_{l,a_l} (the two quantisers' outputs
 * summed, [P2] 3a / [P3] split RVQ; the RVQ output is the sum of its levels),
 * then x = W_out . q (projected back to 512 before decoding, [P3]
 * "Quantization rate"). codes [N][n_q]; out [N][D_out]; q_out [N][D] may be
 * NULL. A code outside [0, K) makes the call return ORACLE_ERANGE (nothing is
 * clamped here: the oracle refuses what it cannot define).
 */
int oracle_decode(const int16_t *codes, int64_t N, int D, int K, int Q, int n_q, int D_out,
                  const float *C, const float *W_out, int nthreads, double *out, double *q_out)
{
    if (N < 0 || D <= 0 || D > 4096 || K <= 0 || Q <= 0 || n_q <= 0 || n_q > Q || D_out <= 0 ||
        (N > 0 && (!codes || !C || !W_out || !out)))
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < N * n_q; ++e)
        if (codes[e] < 0 || codes[e] >= K)
            return ORACLE_ERANGE;
    set_threads(nthreads);
#pragma omp parallel
    {
        double q[4096];
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int i = 0; i < D; ++i)
                q[i] = 0.0;
            for (int l = 0; l < n_q; ++l) {
                const float *c = C + ((size_t)l * K + (size_t)codes[n * n_q + l]) * D;
                for (int i = 0; i < D; ++i)
                    q[i] += (double)c[i];
            }
            if (q_out)
                memcpy(q_out + (size_t)n * D, q, sizeof(double) * (size_t)D);
            for (int o = 0; o < D_out; ++o) {
                const float *w = W_out + (size_t)o * D;
                double acc = 0.0;
                for (int i = 0; i < D; ++i)
                    acc += (double)w[i] * q[i];
                out[(size_t)n * D_out + o] = acc;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Rates the pages fix ([P1] 3, [P2] 3a, [P3] "Quantization rate"):
 * frame rate = sample rate / product of the encoder strides; one code per
 * codebook per frame, each of ceil(log2 K) bits.
 */
double oracle_frame_rate(double sample_rate, const int *strides, int n_strides)
{
    double hop = 1.0;
    for (int i = 0; i < n_strides; ++i)
        hop *= (double)strides[i];
    return sample_rate / hop;
}

int oracle_bits_per_code(int64_t K)
{
    int bits = 0;
    while (((int64_t)1 << bits) < K)
        ++bits;
    return bits;
}

double oracle_bitrate(double frame_rate, int Q, int64_t K)
{
    return frame_rate * (double)Q * (double)oracle_bits_per_code(K);
}
