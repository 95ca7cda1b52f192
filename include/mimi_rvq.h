/*
 * mimi_rvq.h -- C ABI of the B200 (sm_100a) split residual vector quantiser
 * of the Mimi codec: the tokenizer bottleneck behind Moshi.
 *
 * What the library computes (per 80 ms frame, 12.5 Hz):
 *   encode:  y = W_in . z                                  512 -> 256 "Lin"
 *            s   = argmin_k ||y - S_k||^2                  semantic plain VQ (codebook 0)
 *            a_l = argmin_k ||r_{l-1} - A_{l,k}||^2,  r_0 = y,  r_l = r_{l-1} - A_{l,a_l}
 *                                                          acoustic RVQ, levels l = 1..7
 *            codes = (s, a_1, ..., a_7)                    8 codes of 11 bits: 1.1 kbps
 *   decode:  x = W_out . (S_s + sum_l A_{l,a_l})           outputs summed, 256 -> 512
 *
 * Passages (page title, section):
 *   "Moshi: a Speech-Text Foundation Model for Real-Time Dialogue" (notes),
 *     section 2 (RVQ levels quantise the previous level's residual) and
 *     section 3a "Mimi" (512 -> 256 before the RVQ, split RVQ of 8 codebooks of
 *     2048, semantic codebook 1 and a 7-level acoustic RVQ, outputs summed);
 *   annotated translation of the Moshi technical report, sections
 *     "Architecture" (VQ applied iteratively to the previous quantiser's
 *     residual, N_A centroids), "Quantization rate" (Q = 8, N_A = 2048,
 *     1.1 kbps at 12.5 Hz, "Lin" to 256 before the RVQ and back to 512 before
 *     decoding, quantizer dropout) and "split RVQ" (a plain semantic VQ and a
 *     7-level RVQ applied side by side, outputs added).
 * Readings where the pages are silent: squared Euclidean distance; ties go
 * to the lowest index; codes are 0-based; code column 0 is semantic; by
 * default the acoustic RVQ quantises y itself; no bias in either projection.
 *
 * Conventions shared by every call:
 *   - Pointers are DEVICE pointers (cudaMalloc'd or managed) unless a call says
 *     otherwise; the caller owns every input and output buffer. Row-major,
 *     rows contiguous. Every pointer must be 16-byte aligned.
 *   - Asynchronous on `stream` (NULL = legacy default stream) unless stated;
 *     no host synchronisation, no allocation, no exceptions.
 *   - Argument errors are returned at once (negative status) and nothing is
 *     enqueued. Errors that only the device sees (an out-of-range code in
 *     decode, a wait that timed out) set a flag in the handle that
 *     mimi_rvq_get_error() returns.
 *   - A handle is immutable after create; one handle may be used from several
 *     host threads and streams at once, except that concurrent encode calls on
 *     the same handle must be on the same stream (they share the re-score
 *     work list).
 *   - N = 0 is a no-op that returns MIMI_RVQ_OK.
 */
#ifndef MIMI_RVQ_H
#define MIMI_RVQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                      /* = cudaStream_t */
typedef struct mimi_rvq *mimi_rvq_t;     /* opaque handle */

#define MIMI_RVQ_LATENT_DIM    512       /* encoder latent width (512-d @ 12.5 Hz) */
#define MIMI_RVQ_DIM           256       /* projected width the quantisers see */
#define MIMI_RVQ_CODEBOOK_SIZE 2048      /* N_A: codewords per codebook (11 bits) */
#define MIMI_RVQ_NUM_CODEBOOKS 8         /* Q: 1 semantic + 7 acoustic levels */

enum { MIMI_RVQ_F32 = 0, MIMI_RVQ_BF16 = 1 };   /* latent element types */

enum {
    MIMI_RVQ_OK      =  0,
    MIMI_RVQ_EINVAL  = -1,   /* bad argument: NULL, misaligned, host pointer, size, dtype */
    MIMI_RVQ_ENOMEM  = -2,   /* device allocation failed in create */
    MIMI_RVQ_ECUDA   = -3,   /* a CUDA runtime or driver call failed */
    MIMI_RVQ_ERANGE  = -4,   /* decode met a code outside [0, 2048) (device-detected) */
    MIMI_RVQ_EDEVICE = -5,   /* current device is not an sm_100 part */
    MIMI_RVQ_ETIMEOUT = -6   /* a kernel wait ran out its bound and the kernel returned early */
};

/*
 * Create a handle on the current device.
 *   codebooks [8][2048][256] fp32: codebook 0 is the semantic VQ, 1..7 the
 *             acoustic RVQ levels in order.
 *   W_in      [256][512] fp32, y = W_in . z.
 *   W_out     [512][256] fp32, x = W_out . q.
 * Synchronous. The inputs are copied (the caller keeps ownership) and the
 * derived tables are built once: bf16 codebooks, squared codeword norms,
 * the split W_in, the decode tables W_out . C_l. Returns EINVAL on a NULL or
 * host pointer, ENOMEM if device memory runs out, EDEVICE off sm_100.
 */
int mimi_rvq_create(const float *codebooks, const float *W_in, const float *W_out,
                    mimi_rvq_t *out);

/* Free every device buffer of the handle. NULL is ignored. Synchronous. */
void mimi_rvq_destroy(mimi_rvq_t h);

/*
 * Encode N frames: latents [N][512] of type dtype (MIMI_RVQ_F32 or
 * MIMI_RVQ_BF16) -> codes [N][8] int16 (column 0 semantic, 1..7 acoustic
 * levels). Codes equal the float64 definition above wherever the best and
 * second-best squared distances of every level differ by more than the float32
 * re-score error (about 1e-6 of d_best); closer calls may go either way.
 */
int mimi_rvq_encode(mimi_rvq_t h, const void *latents, int dtype, int64_t N,
                    int16_t *codes, struct CUstream_st *stream);

/*
 * Streaming step: one 512-d frame for each of B concurrent streams (B >= 0),
 * frames [B][512] -> codes [B][8]. The quantiser keeps no state between
 * frames, so a step is an encode of B frames tuned for latency: up to 32
 * frames per thread-block cluster the device runs at once (480 on B200:
 * 15 clusters of 8 CTAs) run a float32 kernel on clusters that split the
 * codebooks (its codes equal mimi_rvq_encode_scan's; it keeps no state, so
 * such steps may run on several streams at once); larger steps up to 2304
 * frames (while 8 CTAs per 128-frame group fit the device) run a
 * codebook-sliced form of the tensor-core encoder (one launch; codes as the
 * batch encoder's); larger steps run the batch encoder. On a device without
 * clusters, steps of up to 256 frames run a float32 kernel over groups of CTAs
 * (also the full scan's codes). Allocates nothing, never synchronises the
 * host, and may be captured in a CUDA graph. Steps other than the cluster
 * form share the handle's scratch: issue them in stream order.
 */
int mimi_rvq_encode_step(mimi_rvq_t h, const void *frames, int dtype, int B,
                         int16_t *codes, struct CUstream_st *stream);

/*
 * Streaming step with options: n_q and variant as for mimi_rvq_encode_ex
 * (codes [B][n_q]); otherwise as mimi_rvq_encode_step.
 */
int mimi_rvq_encode_step_ex(mimi_rvq_t h, const void *frames, int dtype, int B, int n_q,
                            int variant, int16_t *codes, struct CUstream_st *stream);

/*
 * Encode with options. n_q in 1..8 keeps only the first n_q codebooks (the
 * semantic one and n_q - 1 acoustic levels: quantizer dropout at inference,
 * for a lower bit-rate); codes are then [N][n_q]. variant 0 is the split RVQ
 * above (acoustic RVQ on y); variant 1 runs the acoustic RVQ on y - S_s
 * instead, the other reading of the notes' section 3a. mimi_rvq_encode is
 * n_q = 8, variant = 0.
 */
int mimi_rvq_encode_ex(mimi_rvq_t h, const void *latents, int dtype, int64_t N, int n_q,
                       int variant, int16_t *codes, struct CUstream_st *stream);

/*
 * Diagnostic: mimi_rvq_encode (n_q = 8, variant 0, N <= 1 048 576) that also
 * adds, into cycles[0..23] (device, caller-zeroed, uint64), the SM clock
 * cycles each role of the tensor-core kernel spent, summed over CTAs:
 *   0 TMA producer waiting for a free stage      1 MMA waiting for operand tiles
 *   2 MMA waiting for a drained score buffer     3 MMA waiting for a level's A operand
 *   4 MMA waiting for staged latents             5 epilogue waiting for a score tile
 *   6 epilogue scanning scores                   7 epilogue merge / window / re-score
 *   8 epilogue residual update                   9 epilogue latent staging, y read-out
 *  10 epilogue barrier waits                    11 whole CTA
 * (counters 5..10 are one epilogue thread per CTA), and event counts summed over the
 * epilogue warps (not cycles): 12 32-column chunks scanned; 13 256-column tiles in
 * which some lane put a displaced best into the candidate list; chunks in which some
 * lane 14 had a runner-up near the window, 15 had three or more keys near it; then
 * cycles again, as parts of 7: 16 list
 * exchange (its barrier included) and merge, 17 float32 re-score, 18 dot exchange and
 * the pick; as part of 6: 19 copying a score tile to registers, writing the next
 * tile's norms and releasing the buffer; as parts of 8: 20 waiting for the MMA to
 * finish with the A operand, 21 gather, subtract and stores, 22 combining the
 * halves' norms; 23 unused. Codes are the same as mimi_rvq_encode's.
 */
int mimi_rvq_encode_profile(mimi_rvq_t h, const void *latents, int dtype, int64_t N,
                            int16_t *codes, uint64_t *cycles, struct CUstream_st *stream);

/*
 * The projection step alone: latents [N][512] -> y = W_in . z [N][256] fp32,
 * computed exactly as encode computes it (split-precision bf16 products on
 * the tensor cores, float32 accumulation).
 */
int mimi_rvq_project(mimi_rvq_t h, const void *latents, int dtype, int64_t N, float *y,
                     struct CUstream_st *stream);

/*
 * Plain float32 encoder on CUDA cores, for comparison and diagnosis: the
 * result contract of mimi_rvq_encode_ex, but every one of the 2048 codewords
 * of each codebook is scored in float32 (no tensor cores, no candidate
 * pruning). About 4.2 M FMA per frame, so it is slow.
 */
int mimi_rvq_encode_scan(mimi_rvq_t h, const void *latents, int dtype, int64_t N, int n_q,
                         int variant, int16_t *codes, struct CUstream_st *stream);

/*
 * Decode N frames: codes [N][8] int16 -> latents [N][512] fp32. A code
 * outside [0, 2048) is clamped into range for the gather (the output stays
 * defined) and sets MIMI_RVQ_ERANGE in the handle's error flag.
 */
int mimi_rvq_decode(mimi_rvq_t h, const int16_t *codes, int64_t N, float *latents,
                    struct CUstream_st *stream);

/* Decode codes [N][n_q] of an n_q-codebook encode (n_q in 1..8): the sum runs
 * over the first n_q codebooks only. mimi_rvq_decode is n_q = 8. */
int mimi_rvq_decode_ex(mimi_rvq_t h, const int16_t *codes, int64_t N, int n_q, float *latents,
                       struct CUstream_st *stream);

/*
 * Synchronises `stream`, then returns and clears the handle's device error
 * flag: MIMI_RVQ_OK, MIMI_RVQ_ERANGE or MIMI_RVQ_ETIMEOUT (ECUDA if the
 * synchronisation itself failed).
 */
int mimi_rvq_get_error(mimi_rvq_t h, struct CUstream_st *stream);

/*
 * Self-test of the failure path: launches one small kernel on `stream` whose
 * wait can never complete -- which = 0: an mbarrier phase nothing completes
 * (the tensor-core encoder's kind of wait); which = 1: a group barrier that
 * only one of its two members reaches (the wide encoder's kind of wait). The
 * kernel gives up after about 50 ms, records the timeout and returns, so the
 * next mimi_rvq_get_error returns MIMI_RVQ_ETIMEOUT (and resets the state a
 * timeout can leave behind); the handle stays usable. Returns MIMI_RVQ_EINVAL
 * for another `which`.
 */
int mimi_rvq_wait_selftest(mimi_rvq_t h, int which, struct CUstream_st *stream);

/*
 * Turn the thread-block-cluster form of the float32 latency encoder on (enabled = 1,
 * the default where the device runs clusters) or off (0). Off, streaming steps of
 * up to 256 frames and the float32 re-encode after a batch encode run the group form
 * instead (CTAs of a cooperative launch meeting at barriers in global memory: slower,
 * same codes), as on a device without clusters. Host-side setting of the handle, read
 * by the calls issued after it; not to be changed while another thread issues calls
 * on the handle. Returns MIMI_RVQ_OK, or MIMI_RVQ_EINVAL for a NULL handle or an
 * enabled value other than 0 or 1. Turning it on where the device runs no clusters
 * changes nothing.
 */
int mimi_rvq_set_cluster_form(mimi_rvq_t h, int enabled);

/*
 * Counters since create (synchronises `stream`): frames encoded, and frames
 * whose bf16 candidate pass could not certify its candidate set at some level
 * and were resolved in float32 instead (re-encoded by the full scan after a
 * batch encode; the row scanned exactly inside the kernel in a sliced
 * streaming step). Either pointer may be NULL.
 */
int mimi_rvq_stats(mimi_rvq_t h, struct CUstream_st *stream, int64_t *frames_encoded,
                   int64_t *frames_rescanned);

/*
 * Encode without a handle and without allocating device memory, for callers
 * that cannot call cudaMalloc: a host that lets libraries use only the device
 * buffers it hands them, or a real-time audio thread, where cudaMalloc and
 * cudaFree may synchronise the device. The pages have no counterpart to this
 * call; it is part of this library's interface, not of the method.
 *   codebooks [8][2048][256] fp32 (only the first n_q are read), W_in
 *   [256][512] fp32, latents [N][512] (MIMI_RVQ_F32 or MIMI_RVQ_BF16),
 *   codes [N][n_q] int16 out; all device pointers owned by the caller.
 * Same arithmetic and codes as mimi_rvq_encode_scan (the float32 full scan:
 * exact float32 scores, slow). Its one piece of scratch, the squared codeword
 * norms, lives in a 64 KiB static device array (at most 8 codebooks of 2048;
 * n_q outside 1..8 returns MIMI_RVQ_EINVAL) that every GPU loading the
 * library holds until exit. The first call in a CUDA context on a device
 * looks up that array's address (again after a device reset, which loads the
 * library's module into a new context); make that first call before any
 * stream capture. Every call shares the array and rewrites it, so calls that
 * overlap on the GPU (other streams, other host threads) race: serialise them.
 * Alignment (this call only; the 16-byte rule of the other calls does not
 * apply): codebooks 16 bytes (read as float4), W_in 4 bytes, latents 4 bytes
 * for MIMI_RVQ_F32 and 2 bytes for MIMI_RVQ_BF16, codes 2 bytes; otherwise
 * MIMI_RVQ_EINVAL.
 */
int mimi_rvq_encode_noalloc(const float *codebooks, const float *W_in, const void *latents,
                            int dtype, int64_t N, int n_q, int16_t *codes,
                            struct CUstream_st *stream);

/* Static English text for a status code. */
const char *mimi_rvq_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* MIMI_RVQ_H */
