// encode_tc.cu -- fused projection + split-RVQ encode on tcgen05 tensor cores.
//
// Per tile of 128 frames (one persistent CTA per SM, tiles strided over CTAs):
//
//   1. projection y = W_in . z on the tensor cores, in split precision so that
//      y is float32-accurate: z = z_hi + z_lo and W_in = W_hi + W_lo (bf16
//      halves; bf16 latents are exact, so z_lo = 0) and
//      y = z_hi W_hi^T + z_lo W_hi^T + z_hi W_lo^T, accumulated in TMEM
//      columns [0, 256). Those columns then hold the residual r (float32) for
//      the whole level chain: it never leaves the SM.
//   2. for each codebook l = 0 (semantic, on y) and 1..7 (acoustic, on r):
//      candidate half-scores ||c||^2 / 2 - bf16(r) . bf16(c) for all 2048
//      codewords as 8 tcgen05 GEMM tiles [128 x 256] x [256 x 256] with A =
//      -bf16(r). Each tile ends with one K = 16 step that adds ||c||^2 / 2 into
//      the accumulator (A = ones, B = the norm's three exact bf16 parts), so the
//      epilogue reads the half-score directly (codebook tiles
//      streamed by TMA into a shared-memory ring, one 256-row box per stage;
//      the accumulator is TMEM columns [256, 512), which the epilogue copies
//      into registers at once so that the next tile's MMAs overlap its scan).
//      The epilogue keeps a sorted list of the best 8 candidate keys per row.
//   3. certified pick: with E a rigorous bound on |bf16 score - exact score|
//      (from ||r||, this row's bf16 rounding residual ||bf16(r) - r||, and the
//      codebook's max ||c|| and max ||bf16(c) - c||), every codeword outside
//      the top-8 is ruled out when
//      s_8 > s_1 + 2E; the candidates within s_1 + 2E are re-scored in float32
//      (||c||^2 - 2 r.c with r read from TMEM and c from the float32
//      codebook); a single candidate needs no re-score. If the top-8 cannot be
//      certified the frame is queued for a float32 re-encode (the wide encoder,
//      in list mode, after this kernel); the sliced streaming form instead scans
//      that row exactly in float32 inside the kernel.
//   4. acoustic levels: r -= c_win in TMEM, and bf16(r) is written into the
//      shared-memory A operand of the next level.
//
// Warp roles (384 threads, three warpgroups): warp 0 issues TMA loads, warp 1
// allocates TMEM and issues the MMAs (one thread each), warps 2 and 3 idle;
// warps 4..11 are the epilogue: the two warps of a TMEM lane quarter (frame rows
// 32q .. 32q + 31) split each score tile's columns and the residual's
// dimensions between them. The semantic level (0)
// and acoustic level 1 share the A operand bf16(y), so the tensor core runs
// from level 0 into level 1 while the epilogue re-scores level 0.
#include <cuda.h>

#include "handle.cuh"
#include "ptx.cuh"

namespace mimi {
namespace {

constexpr int BM = 128;                 // frames per tile = TMEM lanes
constexpr int BN = 256;                 // codewords per score tile (one N = 256 MMA)
constexpr int BK = 64;                  // K elements per stage (128 B of bf16)
constexpr int NT = kK / BN;             // 8 score tiles per codebook
constexpr int KCH = kD / BK;            // 4 K chunks per score tile
constexpr int PKCH = kDin / BK;         // 8 K chunks of the projection
// A bulk tensor copy costs the SM about the same time whatever its size (up to
// a 32 KiB box), so each stage is one 256-row box: a whole score tile's 64-wide
// K chunk, or every output row of the projection's.
constexpr int STAGES = 4;
constexpr int TOPK = 8;                 // candidate list length per row and half
constexpr int STAGE_BYTES = BN * BK * 2;        // 32 KiB
constexpr int A_CHUNK_BYTES = BM * BK * 2;      // 16 KiB
constexpr int RING_OFF = 0;
constexpr int A_OFF = STAGES * STAGE_BYTES;             // 128 KiB
constexpr int X_OFF = A_OFF + KCH * A_CHUNK_BYTES;      // 192 KiB: epilogue exchange area
constexpr int XKEYS_OFF = X_OFF;                        // [2][BM][TOPK + 2] keys, best, evicted
constexpr int XDOT_OFF = XKEYS_OFF + 2 * BM * 10 * 4;   // [2][BM][TOPK] partial re-score dots
constexpr int XNORM_OFF = XDOT_OFF + 2 * BM * TOPK * 4; // [2][BM][2] partial norms
// The norm step's operands (16 K elements, no swizzle): B holds the three bf16
// parts of ||c||^2 / 2 of the score tile's codewords, A holds ones.
constexpr int NORMB_OFF = XNORM_OFF + 2 * BM * 2 * 4;  // [BN][16] bf16
constexpr int ONESA_OFF = NORMB_OFF + BN * 32;         // [BM][16] bf16
constexpr int BAR_OFF = ONESA_OFF + BM * 32;
// The rows of a level whose candidate set could not be certified: one bit per
// row, a 32-bit word per TMEM lane quarter.
constexpr int UMASK_OFF = BAR_OFF + 512;
constexpr int SMEM_BYTES = UMASK_OFF + 64 + 1024;  // slack for 1 KiB alignment
constexpr int kEpiWarps = 8;            // two per TMEM lane quarter: column halves
constexpr int kCtrlWarps = 4;           // warpgroup 0: TMA (warp 0), MMA (warp 1), two idle
constexpr int kThreads = 32 * (kCtrlWarps + kEpiWarps);   // 384: three warpgroups
// Registers. The CTA is launched with kLaunchRegs per thread (the most 384
// threads may have); warpgroup 0 then gives registers back and the two epilogue
// warpgroups take them (setmaxnreg), since the epilogue holds a whole score
// tile's half-rows in registers. The split must fit what the CTA was launched
// with, or the increase would wait forever; the host checks the compiled
// register count against it before every launch.
constexpr int kLaunchRegs = 168;
constexpr int kCtrlRegs = 64;
constexpr int kEpiRegs = 216;
static_assert(32 * (kCtrlWarps * kCtrlRegs + kEpiWarps * kEpiRegs) <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_SCORE = 256;    // the score buffer: columns [256, 512)

// Candidate bound. With e_r = bf16(r) - r and e_c = bf16(c) - c,
//   bf16(r).bf16(c) - r.c = r.e_c + e_r.c + e_r.e_c,
// so by Cauchy-Schwarz |error of the product sum| <= ||r|| ||e_c|| + ||e_r|| ||c||
// + ||e_r|| ||e_c||, using the exact ||e_r|| of this row and the codebook's
// max ||c||, max ||e_c||. The tensor core's float32 accumulation of 256
// products adds at most 256 * 2^-23 of the absolute sum (taken as 2^-14 of
// ||bf16(r)|| ||bf16(c)||, twice the need), and the float32 score
// ||c||^2 - 2 acc rounds once more (2^-21 of its magnitude, with slack).
// E bounds |bf16 score - exact score| for every codeword.

constexpr float kAccRel = 6.103515625e-05f;         // 2^-14
constexpr float kScoreRel = 4.76837158203125e-07f;  // 2^-21

// Candidate keys: a float32 score whose low 11 mantissa bits are replaced by
// the codeword index, so that one min/max orders (score, index) pairs and the
// index travels with the score. The replacement moves the value by less than
// 2^-12 of its magnitude; every comparison that must be rigorous widens by
// key_slack(x) = 2^-11 |x|, which covers it. Keys are built in two steps
// (local_key, then globalize) below.
__device__ __forceinline__ int key_index(float k) { return __float_as_int(k) & 0x7FF; }
__device__ __forceinline__ float key_slack(float k) { return fabsf(k) * 4.8828125e-4f; }
// Smallest raw score a key can stand for (an empty slot, +inf, stays +inf).
__device__ __forceinline__ float key_lower(float k) {
    return k < __int_as_float(0x7f800000) ? k - key_slack(k) : k;
}

// Optional self-profile: cycles each role spends waiting or working, summed
// over CTAs into prof[kProfSlots], and counts of the scan's slower branches
// (diagnostic entry point only; the production instantiation has none of it).
enum ProfSlot {
    P_PROD_EMPTY = 0,   // producer waiting for a free ring stage
    P_MMA_FULL,         // MMA waiting for codebook / weight tiles
    P_MMA_TEMPTY,       // MMA waiting for a drained TMEM score buffer
    P_MMA_AFULL,        // MMA waiting for the next level's A operand
    P_MMA_ZFULL,        // MMA waiting for staged latents
    P_EPI_TFULL,        // epilogue (one thread) waiting for a score tile
    P_EPI_SCAN,         // epilogue scanning score tiles
    P_EPI_PICK,         // epilogue merge, window, re-score
    P_EPI_UPDATE,       // epilogue residual update (including its waits)
    P_EPI_STAGE,        // epilogue latent staging and y read-out
    P_EPI_ESYNC,        // epilogue barrier waits
    P_CTA_TOTAL,        // whole CTA
    P_N_CHUNK,          // event counts, summed over epilogue warps: 32-column chunks scanned,
    P_N_DEM,            //   256-column tiles where some lane put a displaced best in the list,
    P_N_SECOND,         //   chunks where some lane had a runner-up near the window,
    P_N_MORE,           //   chunks where some lane had three or more keys near it
    P_PICK_XCHG,        // parts of P_EPI_PICK: list exchange (barrier included) and merge,
    P_PICK_RESCORE,     //   float32 re-score of the window,
    P_PICK_SELECT,      //   dot exchange (barrier included) and the pick
    P_SCAN_DRAIN,       // part of P_EPI_SCAN: score tile to registers, next norms, release
    P_UPD_AWAIT,        // parts of P_EPI_UPDATE: waiting for the MMA to finish with the A operand,
    P_UPD_WORK,         //   gather, subtract, TMEM and A-operand stores,
    P_UPD_SYNC,         //   combining the halves' norms (barrier included)
    P_UNUSED,
    kProfSlots = 24
};

struct Bars {
    uint64_t full[STAGES], empty[STAGES];
    uint64_t zfull[2], zempty[2];
    uint64_t yfull, afull, aempty, drain;
    uint64_t tfull, tempty;     // the TMEM score buffer
    uint64_t nready;            // the norm step's B tile holds the next score tile's norms
    uint64_t ebar;          // epilogue-wide barrier (all epilogue threads arrive)
    uint32_t tmem_base;
    int abort;
};

// Per-row candidate state for one level: the best key seen, an ascending list
// of the best other keys that were inside the window when they appeared, and
// the smallest key that has fallen off the end of the list. Inserting +inf is
// a no-op, so callers insert unconditionally (no divergent branches).
struct Cands {
    float ts[TOPK];
    float best, evicted;
};

__device__ __forceinline__ void cands_reset(Cands& c) {
#pragma unroll
    for (int p = 0; p < TOPK; ++p) c.ts[p] = __int_as_float(0x7f800000);
    c.best = c.evicted = __int_as_float(0x7f800000);
}

__device__ __forceinline__ void cands_insert(Cands& c, float k) {
#pragma unroll
    for (int p = 0; p < TOPK; ++p) {
        const float lo = fminf(c.ts[p], k);
        k = fmaxf(c.ts[p], k);
        c.ts[p] = lo;
    }
    c.evicted = fminf(c.evicted, k);
}

// Insert five keys at once: sort them (a 9-comparator network), keep the 8
// smallest of the list and the five (elementwise minima of the ascending list
// and the reversed five form a bitonic sequence of the 8 smallest; three
// half-cleaner stages sort it), and the smallest of the rest joins evicted.
// Same list and evicted as five cands_insert calls, with a 9-step dependency
// chain instead of 40.
__device__ __forceinline__ void cx(float& a, float& b) {
    const float lo = fminf(a, b);
    b = fmaxf(a, b);
    a = lo;
}
// Merge an ascending list of 8 keys into c: the same list and evicted as 8
// cands_insert calls.
__device__ __forceinline__ void cands_merge8(Cands& c, const float (&s)[TOPK]) {
    float m[8], d[8];
#pragma unroll
    for (int i = 0; i < TOPK; ++i) {
        m[i] = fminf(c.ts[i], s[TOPK - 1 - i]);
        d[i] = fmaxf(c.ts[i], s[TOPK - 1 - i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) cx(m[i], m[i + 4]);
    cx(m[0], m[2]); cx(m[1], m[3]); cx(m[4], m[6]); cx(m[5], m[7]);
    cx(m[0], m[1]); cx(m[2], m[3]); cx(m[4], m[5]); cx(m[6], m[7]);
#pragma unroll
    for (int i = 0; i < TOPK; ++i) c.ts[i] = m[i];
    c.evicted = fminf(c.evicted, fminf(fminf(fmin3(d[0], d[1], d[2]), fmin3(d[3], d[4], d[5])),
                                       fminf(d[6], d[7])));
}
__device__ __forceinline__ void cands_insert5(Cands& c, const float (&k)[5]) {
    const float inf = __int_as_float(0x7f800000);
    float s[8] = {k[0], k[1], k[2], k[3], k[4], inf, inf, inf};
    cx(s[0], s[1]); cx(s[3], s[4]); cx(s[2], s[4]);
    cx(s[2], s[3]); cx(s[0], s[3]); cx(s[0], s[2]);
    cx(s[1], s[4]); cx(s[1], s[3]); cx(s[1], s[2]);
    cands_merge8(c, s);
}
// Sort 8 keys ascending (a 19-comparator network).
__device__ __forceinline__ void sort8(float (&s)[8]) {
    cx(s[0], s[2]); cx(s[1], s[3]); cx(s[4], s[6]); cx(s[5], s[7]);
    cx(s[0], s[4]); cx(s[1], s[5]); cx(s[2], s[6]); cx(s[3], s[7]);
    cx(s[0], s[1]); cx(s[2], s[3]); cx(s[4], s[5]); cx(s[6], s[7]);
    cx(s[2], s[4]); cx(s[3], s[5]);
    cx(s[1], s[4]); cx(s[3], s[6]);
    cx(s[1], s[2]); cx(s[3], s[4]); cx(s[5], s[6]);
}

// Chunk-local keys carry the element's position 0..31 in their 5 low bits;
// globalize swaps that for the 11-bit codeword index k0 + position.
__device__ __forceinline__ float local_key(float s, int j) {
    return __int_as_float((__float_as_int(s) & ~31) | j);
}
__device__ __forceinline__ float globalize(float k, int k0) {
    const int b = __float_as_int(k);
    return __int_as_float((b & ~0x7FF) | (k0 + (b & 31)));
}

// min(1, max(0, a * b + c)) in one FMA-pipe instruction.
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
    float r;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Smallest of 32 keys with a tree of 3-input minima (16 instructions).
__device__ __forceinline__ float min_of_32(const float (&k)[32]) {
    float m8[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) m8[q] = fminf(fmin3(k[4 * q], k[4 * q + 1], k[4 * q + 2]), k[4 * q + 3]);
    return fminf(fmin3(m8[0], m8[1], m8[2]), fmin3(m8[3], m8[4], fmin3(m8[5], m8[6], m8[7])));
}

// Best two of 32 keys: pairwise min/max, then a tree of top-2 merges.
__device__ __forceinline__ void top2_of_32(const float (&k)[32], float& c1, float& c2) {
    float L[16], H[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        L[i] = fminf(k[2 * i], k[2 * i + 1]);
        H[i] = fmaxf(k[2 * i], k[2 * i + 1]);
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float a = L[2 * i], b = L[2 * i + 1];
            L[i] = fminf(a, b);
            H[i] = fmin3(fmaxf(a, b), H[2 * i], H[2 * i + 1]);
        }
    }
    c1 = L[0];
    c2 = H[0];
}

// Cycle counter of the self-profile; without it the counters fold away, so
// the production kernel carries no profiling registers.
template <bool kProf>
__device__ __forceinline__ long long pclock() {
    if constexpr (kProf) return clock64();
    return 0;
}

// One CTA per SM (its shared memory and TMEM take the whole SM).
// kSliced: the codebook-sliced form for streaming steps. CTA b serves frame
// tile b / kSlices and, at every level, only score tile b % kSlices; after the
// two halves have merged their lists, half 0 publishes the CTA's per-row list to
// slice_lists, the group's CTAs meet at a bounded group barrier, and every CTA
// merges the kSlices lists in slice order, so all of them certify, re-score and
// pick the same codeword and keep the same residual. Slice 0 writes the codes.
template <bool kProf, bool kSliced = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_encode_tc(const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_Whi,
                const __grid_constant__ CUtensorMap tm_Wlo, const float* __restrict__ C32,
                const float* __restrict__ cnorm, const uint2* __restrict__ cnorm3,
                const float* __restrict__ cbound,
                const void* __restrict__ z, int dtype, int64_t n, int n_q, int variant,
                int16_t* __restrict__ codes, float* __restrict__ y_out, int* err,
                int* rescan_count, int* rescan_list, unsigned long long* stats,
                unsigned long long* prof, float* __restrict__ slice_lists, unsigned* slice_bars,
                float2* __restrict__ slice_exact) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1 KiB alignment (128-byte swizzle atoms) as an offset into the shared
    // array, so that the compiler keeps the shared address space (LDS / STS)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + BAR_OFF);
    volatile int* abort = &bars->abort;
    const uint32_t ring = smem_u32(smem + RING_OFF);
    const uint32_t abase = smem_u32(smem + A_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_tiles = (n + BM - 1) / BM;
    // frame tiles of this CTA: blockIdx.x, + gridDim.x, ... (sliced: exactly one)
    const int64_t tile_first = kSliced ? blockIdx.x / kSlices : blockIdx.x;
    const int64_t tile_step = kSliced ? n_tiles : gridDim.x;
    // score tiles of every level: all of them (sliced: this CTA's slice)
    const int slice = kSliced ? (int)(blockIdx.x % kSlices) : 0;
    const int nt_begin = kSliced ? slice : 0, nt_end = kSliced ? slice + 1 : NT;
    const bool f32_in = (dtype == 0);
    // Level l rewrites the A operand (r -= c_win, then bf16(r)) for level l + 1
    // when the next level quantises a different vector: always for acoustic
    // levels, and after the semantic level too when the acoustic RVQ runs on
    // y - S_s (variant 1).
    auto updates_after = [&](int l) { return l < n_q - 1 && (l >= 1 || variant == 1); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->zfull[b], kEpiWarps);
            mbar_init(&bars->zempty[b], 1);
        }
        mbar_init(&bars->tfull, 1);
        mbar_init(&bars->tempty, kEpiWarps);
        mbar_init(&bars->nready, kEpiWarps);
        mbar_init(&bars->yfull, 1);
        mbar_init(&bars->afull, kEpiWarps);
        mbar_init(&bars->aempty, 1);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->ebar, 32 * kEpiWarps);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_C);
        prefetch_tmap(&tm_Whi);
        prefetch_tmap(&tm_Wlo);
    }
    // the norm step's operands: ones (A, constant) and, for the first score tile
    // (codebook 0, codewords 0..255), the norms (B); the B tile's second K half is zero
    for (int i = threadIdx.x; i < BN; i += kThreads) {
        if (i < BM) {
            *reinterpret_cast<uint4*>(smem + ONESA_OFF + k16_offset(i, 0)) =
                make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);  // bf16 1, 1, 1, 0, ...
            *reinterpret_cast<uint4*>(smem + ONESA_OFF + k16_offset(i, 1)) = make_uint4(0u, 0u, 0u, 0u);
        }
        const uint2 nv = __ldg(cnorm3 + nt_begin * BN + i);
        *reinterpret_cast<uint4*>(smem + NORMB_OFF + k16_offset(i, 0)) = make_uint4(nv.x, nv.y, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + NORMB_OFF + k16_offset(i, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const long long t_cta0 = pclock<kProf>();

    if (warp < kCtrlWarps) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
      // warps 2 and 3 are idle and wait at the final barrier
      if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            long long p_empty = 0;
            auto load = [&](const CUtensorMap* tm, int x, int y) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                const long long t0 = pclock<kProf>();
                const bool r = mbar_wait(&bars->empty[s], ph ^ 1, abort, err);
                p_empty += pclock<kProf>() - t0;
                if (!r) return false;
                mbar_arrive_expect_tx(&bars->full[s], STAGE_BYTES);
                tma_load_2d(smem + RING_OFF + s * STAGE_BYTES, tm, &bars->full[s], x, y);
                ++it;
                return true;
            };
            for (int64_t tile = tile_first; tile < n_tiles && ok; tile += tile_step) {
                for (int kc = 0; kc < PKCH && ok; ++kc)
                    ok = ok && load(&tm_Whi, kc * BK, 0) && load(&tm_Wlo, kc * BK, 0);
                for (int l = 0; l < n_q && ok; ++l)
                    for (int nt = nt_begin; nt < nt_end && ok; ++nt)
                        for (int kc = 0; kc < KCH && ok; ++kc)
                            ok = load(&tm_C, kc * BK, l * kK + nt * BN);
            }
            // drain: every issued copy must land before the CTA exits
            const uint32_t first = it > STAGES ? it - STAGES : 0;
            for (uint32_t j = first; j < it; ++j)
                mbar_wait(&bars->full[j % STAGES], (j / STAGES) & 1, abort, err);
            if (kProf && prof) atomicAdd(prof + P_PROD_EMPTY, (unsigned long long)p_empty);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(BM, BN);
            uint32_t it = 0, zuse[2] = {0, 0}, acnt = 0, tcnt = 0;
            bool ok = true;
            long long p_full = 0, p_tempty = 0, p_afull = 0, p_zfull = 0;
            auto twait = [&](uint64_t* bar, uint32_t parity, long long& acc) {
                const long long t0 = pclock<kProf>();
                const bool r = mbar_wait(bar, parity, abort, err);
                acc += pclock<kProf>() - t0;
                return r;
            };
            for (int64_t tile = tile_first; tile < n_tiles && ok; tile += tile_step) {
                // projection: y = z_hi W_hi + z_lo W_hi + z_hi W_lo into columns [0, 256)
                for (int kc = 0; kc < PKCH && ok; ++kc) {
                    const int zb = kc & 1;
                    ok = twait(&bars->zfull[zb], zuse[zb] & 1, p_zfull);
                    ++zuse[zb];
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a_hi = abase + zb * 2 * A_CHUNK_BYTES;
                    const uint32_t a_lo = a_hi + A_CHUNK_BYTES;
                    // g = 0: W_hi (z_hi and z_lo), g = 1: W_lo (z_hi); all 256 outputs at once
                    for (int g = 0; g < 2 && ok; ++g) {
                        const int s = it % STAGES;
                        ok = twait(&bars->full[s], (it / STAGES) & 1, p_full);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t b = ring + s * STAGE_BYTES;
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            const uint32_t acc = (kc > 0 || k > 0 || g >= 1) ? 1u : 0u;
                            umma_bf16(tmem, sw128_desc(a_hi + 32 * k), sw128_desc(b + 32 * k), idesc,
                                      acc);
                            if (g == 0 && f32_in)
                                umma_bf16(tmem, sw128_desc(a_lo + 32 * k), sw128_desc(b + 32 * k),
                                          idesc, 1u);
                        }
                        umma_commit(&bars->empty[s]);
                        ++it;
                    }
                    umma_commit(&bars->zempty[zb]);
                }
                if (!ok) break;
                umma_commit(&bars->yfull);
                // the eight codebooks
                for (int l = 0; l < n_q && ok; ++l) {
                    if (l == 0 || updates_after(l - 1)) {
                        ok = twait(&bars->afull, acnt & 1, p_afull);
                        ++acnt;
                        if (!ok) break;
                        tc_fence_after();
                    }
                    for (int nt = nt_begin; nt < nt_end && ok; ++nt) {
                        ok = twait(&bars->tempty, (tcnt & 1) ^ 1, p_tempty);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t d = tmem + TMEM_SCORE;
                        // A = -bf16(r) over the 256 dimensions, then ||c||^2 / 2 added by the
                        // norm step once the epilogue has written this tile's norms
                        for (int kc = 0; kc < KCH && ok; ++kc) {
                            const int s = it % STAGES;
                            ok = twait(&bars->full[s], (it / STAGES) & 1, p_full);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t b = ring + s * STAGE_BYTES;
                            const uint32_t a = abase + kc * A_CHUNK_BYTES;
#pragma unroll
                            for (int k = 0; k < BK / 16; ++k)
                                umma_bf16(d, sw128_desc(a + 32 * k), sw128_desc(b + 32 * k), idesc,
                                          (kc > 0 || k > 0) ? 1u : 0u);
                            umma_commit(&bars->empty[s]);
                            ++it;
                        }
                        if (!ok) break;
                        ok = twait(&bars->nready, tcnt & 1, p_tempty);
                        if (!ok) break;
                        tc_fence_after();
                        umma_bf16(d, k16_desc(smem_u32(smem + ONESA_OFF)),
                                  k16_desc(smem_u32(smem + NORMB_OFF)), idesc, 1u);
                        umma_commit(&bars->tfull);
                        ++tcnt;
                    }
                    if (updates_after(l) || l == n_q - 1) umma_commit(&bars->aempty);
                }
            }
            // drain: every issued MMA must complete before TMEM is freed
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, abort, err);
            if (kProf && prof) {
                atomicAdd(prof + P_MMA_FULL, (unsigned long long)p_full);
                atomicAdd(prof + P_MMA_TEMPTY, (unsigned long long)p_tempty);
                atomicAdd(prof + P_MMA_AFULL, (unsigned long long)p_afull);
                atomicAdd(prof + P_MMA_ZFULL, (unsigned long long)p_zfull);
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
        // ------------------------------------------------------------ epilogue
        // Eight warps. Warp w reads TMEM lanes 32 (w % 4) .. + 31 (its rows);
        // the two warps of a lane quarter split every 256-column score tile
        // (half h takes columns 128 h .. + 127) and the 256 dimensions of r
        // (half h owns dimensions 128 h .. + 127). Each thread keeps a sorted
        // list of its half's 8 best keys; the halves merge at the end of a level.
        const int quarter = warp & 3;
        const int half = (warp - kCtrlWarps) >> 2;
        const int row = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        const int etid = threadIdx.x - 32 * kCtrlWarps;  // 0..255 within the epilogue: norm-tile row
        // The score tiles run in the order (frame tile, codebook l, tile nt); after
        // draining one, thread etid writes its codeword's norm parts for the next into the
        // norm step's B tile. Each value is loaded one tile ahead of its write.
        auto next_tile = [&](int& l, int& nt) {
            if (++nt == nt_end) {
                nt = nt_begin;
                if (++l == n_q) l = 0;
            }
        };
        int pf_l = 0, pf_nt = nt_begin;
        next_tile(pf_l, pf_nt);  // the setup wrote tile (0, 0); this is the one after it
        if (lane == 0) mbar_arrive(&bars->nready);  // tile (0, 0)'s norms are in place
        uint2 pf_norm = __ldg(cnorm3 + (size_t)pf_l * kK + pf_nt * BN + etid);
        float* xkeys = reinterpret_cast<float*>(smem + XKEYS_OFF);
        float* xdot = reinterpret_cast<float*>(smem + XDOT_OFF);
        float* xnorm = reinterpret_cast<float*>(smem + XNORM_OFF);
        volatile unsigned* s_umask = reinterpret_cast<volatile unsigned*>(smem + UMASK_OFF);
        // the exact scan of an uncertified row: the row's r (256 floats) and each warp's
        // best, in the list-exchange area (free from the re-score on; see below)
        float* s_r = xkeys;
        float* s_bs = xkeys + kD;
        int* s_bk = reinterpret_cast<int*>(xkeys + kD + kEpiWarps);
        uint32_t zuse[2] = {0, 0}, aecnt = 0, tcnt = 0, tile_iter = 0;
        bool ok = true;
        unsigned long long done = 0;
        long long p_tfull = 0, p_scan = 0, p_pick = 0, p_update = 0, p_stage = 0, p_esync = 0;
        long long p_xchg = 0, p_rescore = 0, p_select = 0, p_drain = 0, t_sub = 0;
        long long p_uawait = 0, p_uwork = 0, p_usync = 0;
        // attribute the cycles since t_sub to one of the finer counters
        auto sub = [&](long long& acc) {
            const long long t = pclock<kProf>();
            acc += t - t_sub;
            t_sub = t;
        };
        unsigned long long n_chunk = 0, n_dem = 0, n_sec = 0, n_more = 0;
        long long t_mark = pclock<kProf>();
        // attribute the cycles since the last mark to one counter
        auto mark = [&](long long& acc) {
            const long long t = pclock<kProf>();
            acc += t - t_mark;
            t_mark = t;
        };
        // every lane of the warp takes the same branch after a wait, so the
        // .sync.aligned TMEM loads below are never reached divergently
        auto ewait = [&](uint64_t* bar, uint32_t parity) {
            const bool r = mbar_wait(bar, parity, abort, err);
            return __all_sync(0xffffffffu, r) != 0;
        };
        // Pack this half's 128 dimensions of r (TMEM chunks 4h..4h+3, held in
        // v by the caller one chunk at a time) into the A operand and its norms.
        auto write_a_chunk = [&](int ch, const uint32_t (&v)[32], float& nr2, float& ner2) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = __uint_as_float(v[2 * i]), b = __uint_as_float(v[2 * i + 1]);
                nr2 = fmaf(a, a, nr2);
                nr2 = fmaf(b, b, nr2);
                pk[i] = pack_bf16x2(-a, -b);  // the operand is -bf16(r) (rounding is symmetric)
                const float ea = bf16_lo_to_f32(pk[i]) + a, eb = bf16_hi_to_f32(pk[i]) + b;
                ner2 = fmaf(ea, ea, ner2);
                ner2 = fmaf(eb, eb, ner2);
            }
            uint8_t* dst = smem + A_OFF + (ch >> 1) * A_CHUNK_BYTES;
#pragma unroll
            for (int p = 0; p < 4; ++p)
                *reinterpret_cast<uint4*>(dst + sw128_offset(row, (ch & 1) * 4 + p)) =
                    make_uint4(pk[4 * p], pk[4 * p + 1], pk[4 * p + 2], pk[4 * p + 3]);
        };
        // Barrier over the epilogue threads on an mbarrier, so that the wait is
        // bounded and gives way when another warp has aborted.
        uint32_t ephase = 0;
        auto esync = [&]() {
            mbar_arrive(&bars->ebar);
            const long long t0 = pclock<kProf>();
            const bool r = mbar_wait(&bars->ebar, ephase & 1, abort, err);
            p_esync += pclock<kProf>() - t0;
            ++ephase;
            return __all_sync(0xffffffffu, r) != 0;
        };
        // Barrier of the group's CTAs (sliced form), among the epilogue threads only:
        // every thread's list writes are fenced, the epilogue meets, one thread adds
        // this CTA's arrival and (if wait) spins, bounded, until the count reaches
        // target, and the epilogue meets again.
        unsigned episode = 0;
        auto group_sync = [&](unsigned* bar, unsigned target, bool wait) {
            // the CTA meets first; then one thread fences (which orders every write the
            // CTA barrier ordered before it) and arrives, as a grid-wide barrier does
            if (!esync()) return false;
            if (etid == 0) {
                __threadfence();
                asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
                if (wait) {
                    const long long t0 = clock64();
                    while (true) {
                        unsigned v;
                        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
                        if (v >= target) break;
                        if (clock64() - t0 > kWaitBudgetCycles) {
                            atomicOr(err, MIMI_DEV_ERR_TIMEOUT);
                            *abort = 1;
                            break;
                        }
                    }
                    __threadfence();
                }
            }
            if (!wait) return true;
            return esync() && !*abort;
        };
        // Both halves publish their partial norms; both read back the same sum.
        auto combine_norms = [&](float& nr2, float& ner2) {
            xnorm[(half * BM + row) * 2 + 0] = nr2;
            xnorm[(half * BM + row) * 2 + 1] = ner2;
            if (!esync()) return false;
            nr2 = xnorm[row * 2 + 0] + xnorm[(BM + row) * 2 + 0];
            ner2 = xnorm[row * 2 + 1] + xnorm[(BM + row) * 2 + 1];
            return true;
        };

        for (int64_t tile = tile_first; tile < n_tiles && ok; tile += tile_step, ++tile_iter) {
            const int64_t frame = tile * BM + row;
            const bool valid = frame < n;
            // the A region is z staging now: wait for the previous tile's last MMAs
            if (tile_iter > 0 && n_q > 0) {
                ok = ewait(&bars->aempty, aecnt & 1);
                ++aecnt;
                if (!ok) break;
            }
            // ---- stage z (bf16 hi / lo split) for the projection; this half
            //      writes pieces 4h..4h+3 (32 elements) of each 64-wide K chunk
            for (int kc = 0; kc < PKCH && ok; ++kc) {
                const int zb = kc & 1;
                if (zuse[zb] > 0) {
                    ok = ewait(&bars->zempty[zb], (zuse[zb] - 1) & 1);
                    if (!ok) break;
                }
                ++zuse[zb];
                uint8_t* zhi = smem + A_OFF + zb * 2 * A_CHUNK_BYTES;
                uint8_t* zlo = zhi + A_CHUNK_BYTES;
                const int e0 = kc * BK + half * 32;
                if (f32_in) {
                    const float4* src = reinterpret_cast<const float4*>(
                        static_cast<const float*>(z) + (valid ? frame : 0) * kDin + e0);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float4 u = valid ? __ldg(src + 2 * p) : make_float4(0.f, 0.f, 0.f, 0.f);
                        const float4 w = valid ? __ldg(src + 2 * p + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
                        uint4 h, lo;
                        h.x = pack_bf16x2(u.x, u.y);
                        h.y = pack_bf16x2(u.z, u.w);
                        h.z = pack_bf16x2(w.x, w.y);
                        h.w = pack_bf16x2(w.z, w.w);
                        lo.x = pack_bf16x2(u.x - bf16_lo_to_f32(h.x), u.y - bf16_hi_to_f32(h.x));
                        lo.y = pack_bf16x2(u.z - bf16_lo_to_f32(h.y), u.w - bf16_hi_to_f32(h.y));
                        lo.z = pack_bf16x2(w.x - bf16_lo_to_f32(h.z), w.y - bf16_hi_to_f32(h.z));
                        lo.w = pack_bf16x2(w.z - bf16_lo_to_f32(h.w), w.w - bf16_hi_to_f32(h.w));
                        *reinterpret_cast<uint4*>(zhi + sw128_offset(row, half * 4 + p)) = h;
                        *reinterpret_cast<uint4*>(zlo + sw128_offset(row, half * 4 + p)) = lo;
                    }
                } else {
                    const uint4* src = reinterpret_cast<const uint4*>(
                        static_cast<const uint16_t*>(z) + (valid ? frame : 0) * kDin + e0);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint4 h = valid ? __ldg(src + p) : make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4*>(zhi + sw128_offset(row, half * 4 + p)) = h;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->zfull[zb]);
            }
            if (!ok) break;
            // ---- y from TMEM: this half's 128 dimensions -> A operand (levels 0, 1), norms
            ok = ewait(&bars->yfull, tile_iter & 1);
            if (!ok) break;
            tc_fence_after();
            float nr2 = 0.f, ner2 = 0.f;  // ||r||^2 and ||bf16(r) - r||^2 of this row
            for (int c4 = 0; c4 < 4; ++c4) {
                const int ch = half * 4 + c4;
                uint32_t v[32];
                tmem_ld32(trow + ch * 32, v);
                tmem_wait_ld();
                if (y_out && valid) {
                    float4* dst = reinterpret_cast<float4*>(y_out + frame * kD + ch * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                              __uint_as_float(v[4 * q4 + 2]),
                                              __uint_as_float(v[4 * q4 + 3]));
                }
                if (n_q > 0) write_a_chunk(ch, v, nr2, ner2);
            }
            tc_fence_before();
            if (n_q == 0) continue;  // projection only: y has been written out
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->afull);
            ok = combine_norms(nr2, ner2);
            if (!ok) break;

            mark(p_stage);
            int win_codes[kQ];
            bool flagged = false;
            for (int l = 0; l < n_q && ok; ++l) {
                const float* book = C32 + (size_t)l * kK * kD;
                const float4 cb = __ldg(reinterpret_cast<const float4*>(cbound) + l);
                const float cmax = cb.x, cnmax = cb.y, ecmax = cb.z;
                const float nr = sqrtf(nr2) * 1.0001f, ner = sqrtf(ner2) * 1.0001f;
                // E bounds |accumulated half-score - exact half-score|: the product error,
                // the float32 accumulation of the products and of ||c||^2 / 2, and rounding
                // slack; two keys can each be off by E, hence the window 2 E.
                const float dot_err = nr * ecmax + ner * cmax + ner * ecmax +
                                      kAccRel * ((nr + ner) * (cmax + ecmax) + 0.5f * cnmax);
                const float E = dot_err * 1.0001f +
                                kScoreRel * (0.5f * cnmax + (nr + ner) * (cmax + ecmax));
                const float twoE = 2.f * E;
                Cands cs;
                cands_reset(cs);
                // ---- scan this half of the 8 score tiles of the codebook
                for (int nt = nt_begin; nt < nt_end; ++nt) {
                    mark(p_scan);
                    ok = ewait(&bars->tfull, tcnt & 1);
                    mark(p_tfull);
                    ++tcnt;
                    if (!ok) break;
                    tc_fence_after();
                    t_sub = pclock<kProf>();
                    // this half's 128 columns of the tile, all in registers: the buffer is
                    // released before the scan so that the next tile's MMAs run meanwhile
                    uint32_t v[4][32];
                    {
                        uint32_t w[2][64];
                        tmem_ld64(trow + TMEM_SCORE + half * 128, w[0]);
                        tmem_ld64(trow + TMEM_SCORE + half * 128 + 64, w[1]);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 128; ++j) v[j >> 5][j & 31] = w[j >> 6][j & 63];
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->tempty);
                    // this tile's norm step has completed (it precedes the tile's commit):
                    // write the next tile's norms; the MMA waits for them only at that
                    // tile's norm step, after its 16 score MMAs
                    *reinterpret_cast<uint4*>(smem + NORMB_OFF + k16_offset(etid, 0)) =
                        make_uint4(pf_norm.x, pf_norm.y, 0u, 0u);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->nready);
                    next_tile(pf_l, pf_nt);
                    pf_norm = __ldg(cnorm3 + (size_t)pf_l * kK + pf_nt * BN + etid);
                    sub(p_drain);
                    // ---- the tile: first, without branches, every chunk's minimum, the
                    //      tile's new best and window, and each chunk's count of other keys
                    //      near the window; then the list insertions (one vote per tile) and,
                    //      for the chunks that need them, the runner-up and further keys.
                    //      Keys outside the window of a later (lower) best can never be
                    //      candidates, so judging the whole tile against its final best is
                    //      as rigorous as going chunk by chunk.
                    const float inf = __int_as_float(0x7f800000);
                    float kk[4][32];
                    float c1k[4], g1[4];
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) kk[c2][j] = local_key(__uint_as_float(v[c2][j]), j);
                        c1k[c2] = min_of_32(kk[c2]);
                        g1[c2] = globalize(c1k[c2], nt * BN + half * 128 + c2 * 32);
                    }
                    const float old_best = cs.best;
                    cs.best = fminf(old_best, fminf(fminf(g1[0], g1[1]), fminf(g1[2], g1[3])));
                    const float thr = cs.best + key_slack(cs.best) + twoE;
                    // Any other key of a chunk inside the window? On the FMA pipe:
                    // sum_j sat(kd (Td - key_j)), minus the minimum's own term. Td widens thr
                    // by more than the key perturbations, and every key below Td adds at
                    // least 2^-16, far above the rounding of the sum (<= 2^-18).
                    const float Td = thr + 1.953125e-3f * (fabsf(thr) + twoE);
                    const float kd = __fdividef(16.f, fabsf(Td) + twoE + 1e-30f);
                    const float K = fmaf(kd, Td, 1.52587890625e-05f);
                    float other[4];
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {
                        float a[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) a[i] = fma_sat(-kd, kk[c2][i], K);
#pragma unroll
                        for (int j = 8; j < 32; j += 8)
#pragma unroll
                            for (int i = 0; i < 8; ++i) a[i] += fma_sat(-kd, kk[c2][j + i], K);
                        other[c2] = (((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]))) -
                                    fma_sat(-kd, c1k[c2], K);
                    }
                    // the old best and the chunk minima, except the new best, join the list
                    // when they are inside the window
                    float ins[5];
                    ins[0] = (old_best != cs.best && key_lower(old_best) <= thr) ? old_best : inf;
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2)
                        ins[1 + c2] = (g1[c2] != cs.best && key_lower(g1[c2]) <= thr) ? g1[c2] : inf;
                    const bool any_in = fminf(fminf(ins[0], ins[1]), fminf(fminf(ins[2], ins[3]), ins[4])) < inf;
                    if (kProf) n_chunk += 4;
                    if (__any_sync(0xffffffffu, any_in)) {
                        if (kProf) ++n_dem;
                        cands_insert5(cs, ins);
                    }
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {
                        const int k0 = nt * BN + half * 128 + c2 * 32;
                        const bool second_cand = other[c2] > 9.5367431640625e-07f;  // 2^-20
                        if (__any_sync(0xffffffffu, second_cand)) {
                            if (kProf) ++n_sec;
                            // some lane has another key near the window: its runner-up goes
                            // in, and a third key is looked for only if the sum says so
                            float c1b, c2k;
                            top2_of_32(kk[c2], c1b, c2k);
                            const float g2 = globalize(c2k, k0);
                            const bool second_in = second_cand && key_lower(g2) <= thr;
                            cands_insert(cs, second_in ? g2 : inf);
                            const bool more = second_cand &&
                                              (other[c2] - fma_sat(-kd, c2k, K)) > 9.5367431640625e-07f;
                            if (__any_sync(0xffffffffu, more)) {
                                if (kProf) ++n_more;
                                // further keys in ascending order (the keys are distinct: they
                                // carry their position), while they are inside the window
                                float last = c2k;
                                bool go = more;
#pragma unroll 1
                                for (int t = 0; t < TOPK - 2 && __any_sync(0xffffffffu, go); ++t) {
                                    float nk[32];
#pragma unroll
                                    for (int j = 0; j < 32; ++j) nk[j] = kk[c2][j] > last ? kk[c2][j] : inf;
                                    const float mn = min_of_32(nk);
                                    const float gn = globalize(mn, k0);
                                    const bool in = go && mn < inf && key_lower(gn) <= thr;
                                    cands_insert(cs, in ? gn : inf);
                                    go = in;
                                    last = mn;
                                }
                                // a chunk with more window keys than the list holds: what was
                                // not taken counts as evicted, so the row is not certified
                                if (go) cs.evicted = fminf(cs.evicted, globalize(last, k0));
                            }
                        }
                    }
                }
                if (!ok) break;
                mark(p_scan);
                t_sub = pclock<kProf>();
                // ---- exchange both halves' lists; both merge them the same way
                {
                    float* mine = xkeys + (half * BM + row) * 10;
#pragma unroll
                    for (int p = 0; p < TOPK; ++p) mine[p] = cs.ts[p];
                    mine[8] = cs.best;
                    mine[9] = cs.evicted;
                }
                ok = esync();
                if (!ok) break;
                {
                    const float* k0 = xkeys + row * 10;
                    const float* k1 = xkeys + (BM + row) * 10;
#pragma unroll
                    for (int p = 0; p < TOPK; ++p) cs.ts[p] = k0[p];
                    cs.best = k0[8];
                    cs.evicted = fminf(k0[9], k1[9]);
                    const float best1 = k1[8];
                    cands_insert(cs, fmaxf(cs.best, best1));
                    cs.best = fminf(cs.best, best1);
                    {
                        float k1l[TOPK];
#pragma unroll
                        for (int p = 0; p < TOPK; ++p) k1l[p] = k1[p];
                        cands_merge8(cs, k1l);  // the other half's ascending list
                    }
                    if constexpr (kSliced) {
                        // publish this CTA's list of the row, meet the group's other slices,
                        // then merge every slice's list (in slice order, so all slices get
                        // the same list); after the last level only slice 0 goes on
                        // two buffers by level parity: a slice that has raced ahead to the next
                        // level's publication never overwrites lists a slower slice still reads
                        // (no group barrier need separate the two when no row needs the exact scan)
                        float* lists = slice_lists +
                                       ((size_t)(l & 1) * kSliceMaxGroups + tile) * kSlices * BM * kSliceListFloats;
                        if (half == 0) {
                            float* mine = lists + ((size_t)slice * BM + row) * kSliceListFloats;
#pragma unroll
                            for (int p = 0; p < TOPK; ++p) __stcg(mine + p, cs.ts[p]);
                            __stcg(mine + 8, cs.best);
                            __stcg(mine + 9, cs.evicted);
                        }
                        ++episode;
                        ok = group_sync(slice_bars + tile * kWideBarStride, kSlices * episode, true);
                        if (!ok) break;
                        // all slices' lists in one round trip, then merged in slice order
                        float e[kSlices][kSliceListFloats];
#pragma unroll
                        for (int t = 0; t < kSlices; ++t) {
                            const float* o = lists + ((size_t)t * BM + row) * kSliceListFloats;
#pragma unroll
                            for (int p = 0; p < kSliceListFloats; ++p) e[t][p] = __ldcg(o + p);
                        }
                        // a tree of pairwise merges of the ascending lists, then the
                        // slices' bests (the smallest is the group's; the other seven,
                        // sorted, join the list): the list and evicted of inserting every
                        // key in turn
                        static_assert(kSlices == 8, "the merge tree assumes 8 slices");
                        Cands q[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
#pragma unroll
                            for (int p = 0; p < TOPK; ++p) q[i].ts[p] = e[2 * i][p];
                            q[i].evicted = fminf(e[2 * i][9], e[2 * i + 1][9]);
                            float b[TOPK];
#pragma unroll
                            for (int p = 0; p < TOPK; ++p) b[p] = e[2 * i + 1][p];
                            cands_merge8(q[i], b);
                        }
                        cands_merge8(q[0], q[1].ts);
                        q[0].evicted = fminf(q[0].evicted, q[1].evicted);
                        cands_merge8(q[2], q[3].ts);
                        q[2].evicted = fminf(q[2].evicted, q[3].evicted);
                        cands_merge8(q[0], q[2].ts);
                        q[0].evicted = fminf(q[0].evicted, q[2].evicted);
                        float bb[kSlices];
                        float gbest = __int_as_float(0x7f800000);
#pragma unroll
                        for (int t = 0; t < kSlices; ++t) gbest = fminf(gbest, e[t][8]);
#pragma unroll
                        for (int t = 0; t < kSlices; ++t) bb[t] = e[t][8] == gbest ? __int_as_float(0x7f800000) : e[t][8];
                        sort8(bb);
                        cands_merge8(q[0], bb);
#pragma unroll
                        for (int p = 0; p < TOPK; ++p) cs.ts[p] = q[0].ts[p];
                        cs.evicted = q[0].evicted;
                        cs.best = gbest;
                    }
                    cands_insert(cs, cs.best);  // the best heads the candidate list
                    const float wthr = cs.best + key_slack(cs.best) + twoE;
                    int m = 0;
#pragma unroll
                    for (int p = 0; p < TOPK; ++p) m += (key_lower(cs.ts[p]) <= wthr) ? 1 : 0;
                    const bool certified = key_lower(cs.evicted) > wthr;
                    if constexpr (kSliced) {
                        // uncertified rows are marked for the exact scan below (every word is
                        // rewritten at every level); the statistic counts each such frame once
                        if (half == 0) {
                            const unsigned um = __ballot_sync(0xffffffffu, valid && !certified);
                            if (lane == 0) s_umask[quarter] = um;
                            if (valid && !certified && !flagged && slice == 0) atomicAdd(&stats[1], 1ull);
                        }
                        flagged = flagged || !certified;
                    } else {
                        // the frame is queued for the float32 re-encode after this kernel (an
                        // exact scan here would read the whole float32 codebook per row)
                        if (half == 0 && valid && !certified && !flagged) {
                            flagged = true;
                            const int slot = atomicAdd(rescan_count, 1);
                            if (slot < (int)kRescanCapacity) rescan_list[slot] = (int)frame;
                        }
                    }
                    sub(p_xchg);
                    // ||c||^2 of the window's candidates for the pick, fetched now so that
                    // the loads overlap the re-score
                    float cnp[TOPK];
#pragma unroll
                    for (int p = 0; p < TOPK; ++p)
                        cnp[p] = (m > 1 && p < m) ? __ldg(cnorm + (size_t)l * kK + key_index(cs.ts[p])) : 0.f;
                    // ---- float32 re-score of the window: each half dots its own 128
                    //      dimensions of r with every candidate. The window entries are a
                    //      prefix of the sorted list (m of them). r is read from TMEM 32
                    //      dimensions at a time (one wait), and those dimensions of four
                    //      candidates are fetched together (one L2 round trip per group).
                    float dot[TOPK];
#pragma unroll
                    for (int p = 0; p < TOPK; ++p) dot[p] = 0.f;
                    int mw = m > 1 ? m : 0;  // candidates to re-score, warp maximum
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mw = max(mw, __shfl_xor_sync(0xffffffffu, mw, o));
                    if (mw > 0) {
                        // row offsets of the candidates (lanes without a p-th read the best's row)
                        uint32_t crow[TOPK];
#pragma unroll
                        for (int p = 0; p < TOPK; ++p)
                            crow[p] = (uint32_t)key_index(m > 1 && p < m ? cs.ts[p] : cs.ts[0]) * kD +
                                      half * 128;
#pragma unroll 1
                        for (int q = 0; q < 4; ++q) {
                            uint32_t v[32];
#pragma unroll
                            for (int pb = 0; pb < TOPK; pb += 4) {
                                if (pb < mw) {
                                    // only lanes with a (pb + j)-th candidate load it: the
                                    // rows are scattered, so each lane's loads are separate
                                    // L2 transactions; the first group's are issued before
                                    // r's TMEM read, so the two latencies overlap
                                    float4 c[4][8];
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        const bool act = pb + j < m && m > 1;
                                        const float* cp = book + crow[pb + j] + q * 32;
#pragma unroll
                                        for (int q8 = 0; q8 < 4; ++q8) {
                                            if (act) {
                                                ldg_v8(cp + 8 * q8, c[j][2 * q8], c[j][2 * q8 + 1]);
                                            } else {
                                                c[j][2 * q8] = make_float4(0.f, 0.f, 0.f, 0.f);
                                                c[j][2 * q8 + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
                                            }
                                        }
                                    }
                                    if (pb == 0) {
                                        tmem_ld32(trow + half * 128 + q * 32, v);
                                        tmem_wait_ld();
                                    }
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        float a0 = 0.f, a1 = 0.f;
#pragma unroll
                                        for (int q4 = 0; q4 < 8; ++q4) {
                                            a0 = fmaf(__uint_as_float(v[4 * q4 + 0]), c[j][q4].x, a0);
                                            a1 = fmaf(__uint_as_float(v[4 * q4 + 1]), c[j][q4].y, a1);
                                            a0 = fmaf(__uint_as_float(v[4 * q4 + 2]), c[j][q4].z, a0);
                                            a1 = fmaf(__uint_as_float(v[4 * q4 + 3]), c[j][q4].w, a1);
                                        }
                                        dot[pb + j] += a0 + a1;
                                    }
                                }
                            }
                        }
                    }
                    sub(p_rescore);
                    float* xd = xdot + (half * BM + row) * TOPK;
#pragma unroll
                    for (int p = 0; p < TOPK; ++p) xd[p] = dot[p];
                    ok = esync();
                    if (!ok) break;
                    int win = key_index(cs.best);
                    if (m > 1) {
                        const float* d0 = xdot + row * TOPK;
                        const float* d1 = xdot + (BM + row) * TOPK;
                        float bs = __int_as_float(0x7f800000);
                        int bw = 0x7fffffff;
#pragma unroll
                        for (int p = 0; p < TOPK; ++p) {
                            if (p < m) {
                                const int k = key_index(cs.ts[p]);
                                const float e = fmaf(-2.f, d0[p] + d1[p], cnp[p]);
                                if (e < bs || (e == bs && k < bw)) {
                                    bs = e;
                                    bw = k;
                                }
                            }
                        }
                        if (bw < kK) win = bw;
                    }
                    // ---- sliced: rows whose candidate set could not be certified (more window
                    //      keys than the list holds) take an exact float32 scan of the slice's
                    //      256 codewords, row by row, instead of a re-encode after the kernel.
                    //      The row's r goes through shared memory; each warp takes 32
                    //      codewords (lane j: dimensions 8 j .. 8 j + 7 of a row, a coalesced
                    //      1 KiB load, then a butterfly sum); the lowest score wins, ties to the
                    //      lowest index, over the warps and then over the group's slices. Rows
                    //      go in ascending order, the same in every slice of a group.
                    unsigned um[4] = {0u, 0u, 0u, 0u};
                    int nu = 0;
                    if constexpr (kSliced) {
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            um[w] = s_umask[w];
                            nu += __popc(um[w]);
                        }
                    }
                    for (int i = 0; i < nu; ++i) {
                        int u = 0;
#pragma unroll
                        for (int w = 3; w >= 0; --w)  // the lowest marked row left
                            if (um[w]) u = w * 32 + __ffs(um[w]) - 1;
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            if (w == (u >> 5)) um[w] &= um[w] - 1;
                        if (quarter == (u >> 5)) {  // both warps of u's lane quarter (warp-uniform)
#pragma unroll 1
                            for (int c4 = 0; c4 < 4; ++c4) {
                                uint32_t v[32];
                                tmem_ld32(trow + (half * 4 + c4) * 32, v);
                                tmem_wait_ld();
                                if (lane == (u & 31)) {
                                    float4* dst = reinterpret_cast<float4*>(s_r + (half * 4 + c4) * 32);
#pragma unroll
                                    for (int q4 = 0; q4 < 8; ++q4)
                                        dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                                              __uint_as_float(v[4 * q4 + 2]),
                                                              __uint_as_float(v[4 * q4 + 3]));
                                }
                            }
                        }
                        ok = esync();
                        if (!ok) break;
                        const int ew = etid >> 5;
                        constexpr int kn = BN / kEpiWarps;   // codewords per warp
                        const int kb = nt_begin * BN + ew * kn;
                        const float4 ra = reinterpret_cast<const float4*>(s_r)[2 * lane];
                        const float4 rb = reinterpret_cast<const float4*>(s_r)[2 * lane + 1];
                        float bs = __int_as_float(0x7f800000);
                        int bk = 0x7fffffff;
                        // 16 codeword rows per step in flight (one at a time would be bound by
                        // the latency of each load)
                        constexpr int kRows = 16;
#pragma unroll 1
                        for (int j0 = 0; j0 < kn; j0 += kRows) {
                            float4 ca[kRows], cb[kRows];
                            float cn[kRows];
#pragma unroll
                            for (int t = 0; t < kRows; ++t) {
                                ldg_v8(book + (size_t)(kb + j0 + t) * kD + 8 * lane, ca[t], cb[t]);
                                cn[t] = __ldg(cnorm + (size_t)l * kK + kb + j0 + t);
                            }
#pragma unroll
                            for (int t = 0; t < kRows; ++t) {
                                float d = ra.x * ca[t].x;
                                d = fmaf(ra.y, ca[t].y, d);
                                d = fmaf(ra.z, ca[t].z, d);
                                d = fmaf(ra.w, ca[t].w, d);
                                d = fmaf(rb.x, cb[t].x, d);
                                d = fmaf(rb.y, cb[t].y, d);
                                d = fmaf(rb.z, cb[t].z, d);
                                d = fmaf(rb.w, cb[t].w, d);
#pragma unroll
                                for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                                const float e = fmaf(-2.f, d, cn[t]);
                                if (e < bs) {  // codewords ascending: a tie keeps the lower index
                                    bs = e;
                                    bk = kb + j0 + t;
                                }
                            }
                        }
                        if (lane == 0) {
                            s_bs[ew] = bs;
                            s_bk[ew] = bk;
                        }
                        ok = esync();
                        if (!ok) break;
                        float gb = __int_as_float(0x7f800000);
                        int gk = 0x7fffffff;
#pragma unroll
                        for (int w = 0; w < kEpiWarps; ++w) {
                            const float e = s_bs[w];
                            const int k = s_bk[w];
                            if (e < gb || (e == gb && k < gk)) {
                                gb = e;
                                gk = k;
                            }
                        }
                        if constexpr (kSliced) {
                            float2* ex = slice_exact + ((size_t)tile * BM + u) * kSlices;
                            if (etid == 0) __stcg(ex + slice, make_float2(gb, __int_as_float(gk)));
                            ++episode;
                            ok = group_sync(slice_bars + tile * kWideBarStride, kSlices * episode, true);
                            if (!ok) break;
                            gb = __int_as_float(0x7f800000);
                            gk = 0x7fffffff;
#pragma unroll
                            for (int t = 0; t < kSlices; ++t) {
                                const float2 x = __ldcg(ex + t);
                                const int k = __float_as_int(x.y);
                                if (x.x < gb || (x.x == gb && k < gk)) {
                                    gb = x.x;
                                    gk = k;
                                }
                            }
                        }
                        if (row == u && gk < kK) win = gk;
                        ok = esync();  // s_r and the warp bests are rewritten for the next row
                        if (!ok) break;
                    }
                    if (!ok) break;
                    if constexpr (kSliced) {
                        // the group's last arrival: slice 0 waits for all of them, then resets
                        // the counter for the next launch
                        if (l == n_q - 1) {
                            ++episode;
                            ok = group_sync(slice_bars + tile * kWideBarStride, kSlices * episode,
                                            slice == 0);
                            if (!ok) break;
                            if (slice == 0 && etid == 0) atomicExch(slice_bars + tile * kWideBarStride, 0u);
                        }
                    }
                    win_codes[l] = win;
                    sub(p_select);
                    mark(p_pick);
                    // ---- residual update r -= c_win for the next level, split by halves
                    if (updates_after(l)) {
                        t_sub = pclock<kProf>();
                        ok = ewait(&bars->aempty, aecnt & 1);
                        ++aecnt;
                        if (!ok) break;
                        sub(p_uawait);
                        nr2 = 0.f;
                        ner2 = 0.f;
                        // the winner's half-row with all 32 loads in flight (one round trip);
                        // r read from TMEM 64 dimensions at a time
                        const float* cw = book + (size_t)win * kD + half * 128;
                        float4 c[32];
#pragma unroll
                        for (int q8 = 0; q8 < 16; ++q8) ldg_v8(cw + 8 * q8, c[2 * q8], c[2 * q8 + 1]);
#pragma unroll
                        for (int b2 = 0; b2 < 2; ++b2) {
                            uint32_t v[2][32];
                            tmem_ld32(trow + (half * 4 + 2 * b2) * 32, v[0]);
                            tmem_ld32(trow + (half * 4 + 2 * b2 + 1) * 32, v[1]);
                            tmem_wait_ld();
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2) {
                                const int c4i = 2 * b2 + h2;
                                const int ch = half * 4 + c4i;
#pragma unroll
                                for (int q4 = 0; q4 < 8; ++q4) {
                                    const float4 cc = c[c4i * 8 + q4];
                                    v[h2][4 * q4 + 0] = __float_as_uint(__uint_as_float(v[h2][4 * q4 + 0]) - cc.x);
                                    v[h2][4 * q4 + 1] = __float_as_uint(__uint_as_float(v[h2][4 * q4 + 1]) - cc.y);
                                    v[h2][4 * q4 + 2] = __float_as_uint(__uint_as_float(v[h2][4 * q4 + 2]) - cc.z);
                                    v[h2][4 * q4 + 3] = __float_as_uint(__uint_as_float(v[h2][4 * q4 + 3]) - cc.w);
                                }
                                tmem_st32(trow + ch * 32, v[h2]);
                                write_a_chunk(ch, v[h2], nr2, ner2);
                            }
                        }
                        tmem_wait_st();
                        fence_proxy_async_smem();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars->afull);
                        sub(p_uwork);
                        ok = combine_norms(nr2, ner2);
                        if (!ok) break;
                        sub(p_usync);
                        mark(p_update);
                    }
                }
            }
            if (!ok) break;
            tc_fence_before();
            if (half == 0 && valid && (!kSliced || slice == 0)) {
                if (n_q == kQ) {
                    uint4 pk;
                    pk.x = (uint32_t)(uint16_t)win_codes[0] | ((uint32_t)(uint16_t)win_codes[1] << 16);
                    pk.y = (uint32_t)(uint16_t)win_codes[2] | ((uint32_t)(uint16_t)win_codes[3] << 16);
                    pk.z = (uint32_t)(uint16_t)win_codes[4] | ((uint32_t)(uint16_t)win_codes[5] << 16);
                    pk.w = (uint32_t)(uint16_t)win_codes[6] | ((uint32_t)(uint16_t)win_codes[7] << 16);
                    *reinterpret_cast<uint4*>(codes + frame * kQ) = pk;
                } else {
                    for (int l = 0; l < n_q; ++l) codes[frame * n_q + l] = (int16_t)win_codes[l];
                }
                ++done;
            }
        }
        mark(p_stage);
        if (kProf && prof && warp == kCtrlWarps && lane == 0) {
            atomicAdd(prof + P_EPI_TFULL, (unsigned long long)p_tfull);
            atomicAdd(prof + P_EPI_SCAN, (unsigned long long)p_scan);
            atomicAdd(prof + P_EPI_PICK, (unsigned long long)p_pick);
            atomicAdd(prof + P_EPI_UPDATE, (unsigned long long)p_update);
            atomicAdd(prof + P_EPI_STAGE, (unsigned long long)p_stage);
            atomicAdd(prof + P_EPI_ESYNC, (unsigned long long)p_esync);
            atomicAdd(prof + P_PICK_XCHG, (unsigned long long)p_xchg);
            atomicAdd(prof + P_PICK_RESCORE, (unsigned long long)p_rescore);
            atomicAdd(prof + P_PICK_SELECT, (unsigned long long)p_select);
            atomicAdd(prof + P_SCAN_DRAIN, (unsigned long long)p_drain);
            atomicAdd(prof + P_UPD_AWAIT, (unsigned long long)p_uawait);
            atomicAdd(prof + P_UPD_WORK, (unsigned long long)p_uwork);
            atomicAdd(prof + P_UPD_SYNC, (unsigned long long)p_usync);
        }
        if (kProf && prof && lane == 0) {
            atomicAdd(prof + P_N_CHUNK, n_chunk);
            atomicAdd(prof + P_N_DEM, n_dem);
            atomicAdd(prof + P_N_SECOND, n_sec);
            atomicAdd(prof + P_N_MORE, n_more);
        }
        // count frames (one atomic per warp)
        for (int o = 16; o > 0; o >>= 1) done += __shfl_xor_sync(0xffffffffu, done, o);
        if (lane == 0 && done) atomicAdd(&stats[0], done);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
    if (kProf && prof && threadIdx.x == 0)
        atomicAdd(prof + P_CTA_TOTAL, (unsigned long long)(pclock<kProf>() - t_cta0));
}

}  // namespace

cudaError_t encode_tc_configure() {
    for (auto* k : {k_encode_tc<false>, k_encode_tc<true>, k_encode_tc<false, true>}) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        // the register split needs the launch allocation it was sized for
        cudaFuncAttributes a;
        e = cudaFuncGetAttributes(&a, k);
        if (e != cudaSuccess) return e;
        if (a.numRegs < kLaunchRegs || a.maxThreadsPerBlock < kThreads)
            return cudaErrorLaunchOutOfResources;
    }
    return cudaSuccess;
}

cudaError_t launch_encode_tc(const Tables& t, const void* z, int dtype, int64_t n, int n_q,
                             int variant, int16_t* codes, float* y_out, cudaStream_t s,
                             int max_ctas, unsigned long long* prof) {
    if (n <= 0) return cudaSuccess;
    const int64_t tiles = (n + BM - 1) / BM;
    const int grid = (int)(tiles < max_ctas ? tiles : max_ctas);
    auto* kernel = prof ? k_encode_tc<true> : k_encode_tc<false>;
    kernel<<<grid, kThreads, SMEM_BYTES, s>>>(t.tm_C, t.tm_Whi, t.tm_Wlo, t.C32, t.cnorm,
                                              reinterpret_cast<const uint2*>(t.cnorm3), t.cbound,
                                              z, dtype, n, n_q, variant, codes, y_out, t.err,
                                              t.rescan_count, t.rescan_list, t.stats, prof,
                                              nullptr, nullptr, nullptr);
    return cudaGetLastError();
}

bool sliced_fits(int B, int num_sms) {
    if (B <= 0 || B > BM * kSliceMaxGroups) return false;
    return ((B + BM - 1) / BM) * kSlices <= num_sms;
}

cudaError_t launch_encode_tc_sliced(const Tables& t, const void* z, int dtype, int B, int n_q,
                                    int variant, int16_t* codes, cudaStream_t s) {
    if (!sliced_fits(B, t.num_sms)) return cudaErrorInvalidValue;
    const int groups = (B + BM - 1) / BM;
    CUtensorMap tm_C = t.tm_C, tm_Whi = t.tm_Whi, tm_Wlo = t.tm_Wlo;
    const float* C32 = t.C32;
    const float* cnorm = t.cnorm;
    const uint2* cnorm3 = reinterpret_cast<const uint2*>(t.cnorm3);
    const float* cbound = t.cbound;
    int64_t n = B;
    float* y_out = nullptr;
    int* err = t.err;
    int* rescan_count = t.rescan_count;
    int* rescan_list = t.rescan_list;
    unsigned long long* stats = t.stats;
    unsigned long long* prof = nullptr;
    float* lists = t.slice_lists;
    unsigned* bars = t.wide_bars + kSliceBarBase * kWideBarStride;
    float2* exact = t.slice_exact;
    void* args[] = {&tm_C, &tm_Whi, &tm_Wlo, &C32, &cnorm, &cnorm3, &cbound, &z, &dtype, &n,
                    &n_q, &variant, &codes, &y_out, &err, &rescan_count, &rescan_list, &stats,
                    &prof, &lists, &bars, &exact};
    // every CTA of a group waits for the others: all must be resident at once
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k_encode_tc<false, true>),
                                       dim3(groups * kSlices), dim3(kThreads), args, SMEM_BYTES, s);
}

}  // namespace mimi
