// encode_cluster.cu -- latency encode of a streaming step on thread-block clusters.
//
// The frames of a step are cut into blocks of at most 32, one per cluster of CS
// CTAs (16 where the device co-schedules at least as many CTAs that way, else
// 8). CTA `rank` of a cluster owns codewords [rank * K / CS, (rank + 1) * K / CS)
// of every codebook and scores them against all frames of its block on the CUDA
// cores, in float32 and in the full scan's order:
//
//   score(f, k) = ||c_k||^2 - 2 r_f . c_k      (4 partial sums, as the full scan)
//
// Per level each CTA reduces its keys (order-preserving score bits, codeword
// index) per frame into its own shared memory; one cluster barrier closes the
// level, and every CTA then reads the CS minima of each frame through
// distributed shared memory, so all pick the same winner (lowest score, ties to
// the lowest index) and apply the same update to their own copy of r. The
// projection y = W_in . z is split over the cluster's CTAs by output dimension
// and gathered the same way. The codes are the ones mimi_rvq_encode_scan
// returns.
//
// Against the group form of encode_wide.cu (groups of CTAs meeting at barriers
// in global memory): a cluster barrier is a hardware barrier, the minima cross
// no L2 round trips, and a CTA updates r for the few frames of its cluster
// only. Clusters never wait on one another, so the launch needs no
// co-residency guarantee and leaves no state behind (graph replays and
// concurrent streams need no reset).
//
// Scoring is bound by shared-memory operand traffic, so the thread tile is
// chosen for it: the four lanes w = 0..3 of a lane quad each keep one of the
// four partial sums (dimensions i + w, i stepping by 4) of U frames x V
// codewords, reading their operands with 32-bit loads that hit 32 distinct
// banks (a warp's 8 quads take 8 consecutive codewords); the partials are
// combined at the end of the level by two shuffles, (p0 + p1) + (p2 + p3),
// the scan's order. The CTA's codewords arrive by TMA as slabs of 32
// dimensions (one 128-byte row per codeword, 128-byte swizzle) in two 64 KiB
// stages, each filled by one 3-D box of 2 or 4 slabs; one thread refills a
// stage once every warp is done with it.
#include "latency_common.cuh"

namespace mimi {
namespace {

using lat::kThreads;
using lat::load_latent4;
using lat::pack_key;
using lat::RSTRIDE;
using lat::umin64;

constexpr int kSlabDims = 32;                        // dimensions per slab (128 bytes per codeword)
constexpr int kSlabsPerLevel = kD / kSlabDims;       // 8
constexpr int NST = 2;                               // stages
constexpr int STAGE_BYTES = 64 * 1024;               // a stage: 64 KiB of slabs (2 or 4)
constexpr int YSTRIDE = 32;                          // row stride (floats) of the projection block
constexpr int R_OFF = NST * STAGE_BYTES;             // bytes: r rows
constexpr int Y_OFF = R_OFF + kClusterMaxBlock * RSTRIDE * 4;      // projection block
constexpr int MK_OFF = Y_OFF + kClusterMaxBlock * YSTRIDE * 4;     // [2][block] minimum keys
constexpr int WIN_OFF = MK_OFF + 2 * kClusterMaxBlock * 8;         // [block] winners
constexpr int BAR_OFF = WIN_OFF + kClusterMaxBlock * 4;            // [NST] slab barriers
constexpr int ABORT_OFF = BAR_OFF + NST * 8;
constexpr int RED_OFF = ABORT_OFF + 16;                            // [8 warps][16] per-warp minima
constexpr int FRAME_OFF = RED_OFF + 8 * 16 * 8;                    // [block] frame indices
constexpr int SMEM_BYTES = FRAME_OFF + kClusterMaxBlock * 4 + 1024;  // + alignment of the stages
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(BAR_OFF % 8 == 0 && MK_OFF % 8 == 0 && RED_OFF % 8 == 0, "alignment");
// the projection stages F + kD / CS rows of all kDin + 1 columns over the slab stages and the
// r rows, before either is in use
static_assert((kClusterMaxBlock + kD / 8) * (kDin + 1) * 4 <= Y_OFF, "projection staging fits");

// y = W_in . z for a tile of PF frames (rows pf.., clamped to F - 1: computed,
// never stored) x PD outputs (rows pd..) of the staged latents and W_in rows (row
// stride kDin + 1): every output a sequential FMA chain over all kDin columns (the
// full scan's order), each staged value read once for the tile's chains.
template <int PF, int PD>
__device__ __forceinline__ void proj_tile(const float* z_s, const float* w_s, int pf, int pd, int F,
                                          float* y_s) {
    constexpr int JS = kDin + 1;
    float acc[PF][PD];
#pragma unroll
    for (int i = 0; i < PF; ++i)
#pragma unroll
        for (int k = 0; k < PD; ++k) acc[i][k] = 0.f;
    const float* zr[PF];
#pragma unroll
    for (int i = 0; i < PF; ++i) zr[i] = z_s + min(pf + i, F - 1) * JS;
    const float* wr = w_s + pd * JS;
#pragma unroll 8
    for (int j = 0; j < kDin; ++j) {
        float zv[PF], wv[PD];
#pragma unroll
        for (int i = 0; i < PF; ++i) zv[i] = zr[i][j];
#pragma unroll
        for (int k = 0; k < PD; ++k) wv[k] = wr[k * JS + j];
#pragma unroll
        for (int i = 0; i < PF; ++i)
#pragma unroll
            for (int k = 0; k < PD; ++k) acc[i][k] = fmaf(wv[k], zv[i], acc[i][k]);
    }
#pragma unroll
    for (int i = 0; i < PF; ++i)
        if (pf + i < F)
#pragma unroll
            for (int k = 0; k < PD; ++k) y_s[(pf + i) * YSTRIDE + pd + k] = acc[i][k];
}

struct ClusterArgs {
    const float* C32;
    const float* Win32;
    const float* cnorm;
    int* err;
    unsigned long long* stats;
    const void* z;
    int dtype, B, n_q, variant;
    int cs;   // CTAs per cluster
    int fc;   // frames per cluster (the last cluster may have fewer)
    int16_t* codes;
    // list mode (re-encode of the frames the tensor-core encoder could not certify):
    // frames list[0 .. min(*list_count, list_cap)), nc x fc per pass; nullptr: frames 0..B-1
    const int* list;
    const int* list_count;
    int list_cap;
};

// Thread tile U frames x V codewords per lane quad; warps split as WF (frame
// blocks of U) x WC (codeword blocks of 8V), WC = (K / CS) / (8V). kList: the
// list mode (passes over the listed frames); otherwise one block of frames.
template <int U, int V, bool kList>
__global__ void __launch_bounds__(kThreads, 1)
    k_encode_cluster(const __grid_constant__ CUtensorMap tm_C32, ClusterArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* r_s = reinterpret_cast<float*>(sm + R_OFF);
    float* y_s = reinterpret_cast<float*>(sm + Y_OFF);
    unsigned long long* mk_s = reinterpret_cast<unsigned long long*>(sm + MK_OFF);
    int* win_s = reinterpret_cast<int*>(sm + WIN_OFF);
    int* frame_s = reinterpret_cast<int*>(sm + FRAME_OFF);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + BAR_OFF);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + ABORT_OFF);
    unsigned long long* red_s = reinterpret_cast<unsigned long long*>(sm + RED_OFF);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int g = lane >> 2, w = lane & 3;
    const int cs = a.cs;
    const int rank = (int)cluster_ctarank();
    const int nc = gridDim.x / cs, cl = blockIdx.x / cs;
    int n_frames = a.B;
    if constexpr (kList) {
        n_frames = min(__ldcg(a.list_count), a.list_cap);
        if (blockIdx.x == 0 && tid == 0 && n_frames > 0)
            atomicAdd(&a.stats[1], (unsigned long long)n_frames);
    }
    const int slice = kK / cs;
    const int WC = slice / (8 * V);
    const int wf = wid / WC, wc = wid % WC;
    const int k_base = rank * slice;
    const int DO = kD / cs;             // projection outputs of this CTA: [rank * DO, rank * DO + DO)
    const int slab_bytes = slice * 128;
    const int nb = STAGE_BYTES / slab_bytes;   // slabs per stage: 2 (clusters of 8) or 4 (of 16)
    const int spl = kSlabsPerLevel / nb;       // stages per level
    const int total = a.n_q * spl;

    // stage t of a pass (sg of the launch): slabs [nb (t % spl), + nb) of this CTA's
    // codewords of level t / spl, one box (the slab index is the map's outer dimension)
    auto issue = [&](int sg, int t) {
        uint64_t* bar = &full[sg % NST];
        mbar_arrive_expect_tx(bar, (uint32_t)STAGE_BYTES);
        tma_load_3d(sm + (sg % NST) * STAGE_BYTES, &tm_C32, bar, 0, (t / spl) * kK + k_base,
                    (t % spl) * nb);
    };
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) mbar_init(&full[i], 1);
        *abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    int s = 0;  // stage index over the launch (barrier parity)
    // frames f0 .. f0 + F - 1 of the step, or of the list (all CTAs of a cluster agree)
    auto pass = [&](const int f0, const int F) {
        if constexpr (kList) {
            if (tid < F) frame_s[tid] = __ldcg(a.list + f0 + tid);
            __syncthreads();
        }
        auto frame_of = [&](int f) {
            if constexpr (kList) return frame_s[f];
            else return f0 + f;
        };

        // ---- y = W_in . z for the cluster's F frames x this CTA's DO outputs, each a
        //      sequential FMA chain over j (the full scan's order); latents and W_in rows
        //      staged whole (every load in flight at once) over the slab stages and r rows.
        //      Shared-memory reads bound the chains, so for more than six frames a
        //      thread keeps 2 or 4 frames x 2 outputs in registers and each value it
        //      reads feeds several chains; for a few frames, one chain per thread.
        {
            const int d0 = rank * DO;
            constexpr int JS = kDin + 1, J4 = kDin / 4;
            float* z_s = reinterpret_cast<float*>(sm);   // [F][JS]
            float* w_s = z_s + F * JS;                   // [DO][JS]
            const int nz = F * J4, nt = (F + DO) * J4;
            for (int e0 = tid; e0 < nt; e0 += 16 * kThreads) {
                float4 v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int e = e0 + u * kThreads;
                    if (e < nz)
                        v[u] = load_latent4(a.z, a.dtype, (int64_t)frame_of(e / J4) * kDin + 4 * (e % J4));
                    else if (e < nt)
                        v[u] = __ldg(reinterpret_cast<const float4*>(
                            a.Win32 + (size_t)(d0 + (e - nz) / J4) * kDin + 4 * ((e - nz) % J4)));
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int e = e0 + u * kThreads;
                    if (e < nt) {
                        float* d = z_s + (e / J4) * JS + 4 * (e % J4);  // w_s follows z_s
                        d[0] = v[u].x;
                        d[1] = v[u].y;
                        d[2] = v[u].z;
                        d[3] = v[u].w;
                    }
                }
            }
            __syncthreads();
            const int pf_n = F <= 6 ? 1 : F <= 12 ? 2 : 4, pd_n = F <= 6 ? 1 : 2;
            const int nob = DO / pd_n, nfb = (F + pf_n - 1) / pf_n;
            if (tid < nfb * nob) {
                const int pf = (tid / nob) * pf_n, pd = (tid % nob) * pd_n;
                if (pf_n == 1) proj_tile<1, 1>(z_s, w_s, pf, pd, F, y_s);
                else if (pf_n == 2) proj_tile<2, 2>(z_s, w_s, pf, pd, F, y_s);
                else proj_tile<4, 2>(z_s, w_s, pf, pd, F, y_s);
            }
        }
        __syncthreads();  // the staging is read: the stages take the first slabs
        if (tid == 0)
            for (int t = 0; t < NST && t < total; ++t) issue(s + t, t);
        cluster_sync();  // every CTA's projection block is written

        // r = y, gathered from the cluster's CTAs; the rows past F up to the thread
        // tile's end are zero (scored, never published)
        const int rows = (8 / WC) * U;
        for (int e = tid; e < rows * (kD / 4); e += kThreads) {
            const int f = e >> 6, d = 4 * (e & 63);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (f < F) v = ld_cluster_f4(cluster_map(smem_u32(y_s + f * YSTRIDE + d % DO), (uint32_t)(d / DO)));
            *reinterpret_cast<float4*>(r_s + f * RSTRIDE + d) = v;
        }
        __syncthreads();

        // this lane's codewords (row within the CTA's slice: cw0 + 8v) and frames (fr0 + u)
        const int cw0 = wc * 8 * V + g;
        const int fr0 = wf * U;
        int tl = 0;  // stage index within the pass
        for (int l = 0; l < a.n_q; ++l) {
            // minima by level parity: a slot is rewritten two levels later, after the
            // barrier that every CTA reaches only once it has read it
            unsigned long long* mk = mk_s + (l & 1) * kClusterMaxBlock;
            // after the level's scores this lane holds the dots of codewords vq + k, k < V / 4
            // (see below): their ||c||^2 now, so the loads overlap the scoring
            const int vq = (w & 1) * (V / 2) + (w >> 1) * (V / 4);
            float cnv[V / 4];
#pragma unroll
            for (int k = 0; k < V / 4; ++k)
                cnv[k] = __ldg(a.cnorm + (size_t)l * kK + k_base + cw0 + 8 * (vq + k));
            float acc[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int v = 0; v < V; ++v) acc[u][v] = 0.f;
            for (int tt = 0; tt < spl; ++tt, ++s, ++tl) {
                mbar_wait(&full[s % NST], (uint32_t)(s / NST) & 1u, abort, a.err);
#pragma unroll 1
                for (int jj = 0; jj < nb; ++jj) {
                    // codeword row cw0 + 8v of slab jj: 128 bytes, 16-byte unit x at x ^ (row & 7),
                    // and row & 7 = g
                    const uint8_t* cb = sm + (s % NST) * STAGE_BYTES + jj * slab_bytes + cw0 * 128 + 4 * w;
                    const float* rb = r_s + fr0 * RSTRIDE + (tt * nb + jj) * kSlabDims + w;
#pragma unroll
                    for (int i = 0; i < kSlabDims; i += 4) {
                        const int off = ((i >> 2) ^ g) << 4;
                        float cv[V], rv[U];
#pragma unroll
                        for (int v = 0; v < V; ++v) cv[v] = *reinterpret_cast<const float*>(cb + v * 1024 + off);
#pragma unroll
                        for (int u = 0; u < U; ++u) rv[u] = rb[u * RSTRIDE + i];
#pragma unroll
                        for (int u = 0; u < U; ++u)
#pragma unroll
                            for (int v = 0; v < V; ++v) acc[u][v] = fmaf(rv[u], cv[v], acc[u][v]);
                    }
                }
                __syncthreads();  // every warp is done with the stage
                if (tid == 0 && tl + NST < total) issue(s + NST, tl + NST);
            }
            // dot = (p0 + p1) + (p2 + p3) across the quad as a reduce-scatter: lanes w and
            // w ^ 1 add their partials of the codeword half each keeps (w & 1 picks it), then
            // lanes w and w ^ 2 those of the quarter each keeps (w & 2), so lane w ends with
            // the dots of codewords vq + k, k < V / 4 (3 UV / 4 shuffles instead of 2 UV; the
            // sums are the same, each addition being commutative). Then the minimum key per
            // frame over the warp and one slot per warp and frame.
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float h[V / 2];
#pragma unroll
                for (int k = 0; k < V / 2; ++k) {
                    const float lo = acc[u][k], hi = acc[u][k + V / 2];
                    const float send = (w & 1) ? lo : hi, keep = (w & 1) ? hi : lo;
                    h[k] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                }
                unsigned long long best = ~0ull;
#pragma unroll
                for (int k = 0; k < V / 4; ++k) {
                    const float a0 = h[k], a1 = h[k + V / 4];
                    const float send = (w & 2) ? a0 : a1, keep = (w & 2) ? a1 : a0;
                    const float dot = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    best = umin64(best, pack_key(fmaf(-2.f, dot, cnv[k]), k_base + cw0 + 8 * (vq + k)));
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) best = umin64(best, __shfl_xor_sync(0xffffffffu, best, o));
                if (lane == 0) red_s[wid * 16 + u] = best;
            }
            __syncthreads();
            // frame f: the minimum over the WC warps that scored its codewords
            if (tid < F) {
                const int fw = (tid / U) * WC, fu = tid % U;
                unsigned long long m = red_s[fw * 16 + fu];
                for (int c = 1; c < WC; ++c) m = umin64(m, red_s[(fw + c) * 16 + fu]);
                mk[tid] = m;
            }
            cluster_sync();  // every CTA's minima of this level are in its shared memory
            // winners: the minimum over the cluster's CTAs of each frame
            if (tid < F) {
                const uint32_t addr = smem_u32(mk + tid);
                unsigned long long m[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) m[r] = r < cs ? ld_cluster_u64(cluster_map(addr, (uint32_t)r)) : ~0ull;
#pragma unroll
                for (int r = 1; r < 16; ++r) m[0] = umin64(m[0], m[r]);
                int wn = (int)(uint32_t)m[0];
                if (wn < 0 || wn >= kK) wn = 0;  // only reachable with NaN / Inf inputs
                win_s[tid] = wn;
                if (rank == 0) a.codes[(size_t)frame_of(tid) * a.n_q + l] = (int16_t)wn;
            }
            if (l == a.n_q - 1) break;
            __syncthreads();
            // acoustic levels chain on r; variant 1 also starts the chain at y - S_s
            if (l >= 1 || a.variant == 1) {
                const float* book = a.C32 + (size_t)l * kK * kD;
                const int ne = F * (kD / 4);
                for (int e0 = tid; e0 < ne; e0 += 8 * kThreads) {
                    float4 cw[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int e = e0 + u * kThreads;
                        if (e < ne) cw[u] = __ldg(reinterpret_cast<const float4*>(book + (size_t)win_s[e >> 6] * kD) + (e & 63));
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int e = e0 + u * kThreads;
                        if (e < ne) {
                            float4* r = reinterpret_cast<float4*>(r_s + (e >> 6) * RSTRIDE + 4 * (e & 63));
                            float4 v = *r;
                            v.x -= cw[u].x;
                            v.y -= cw[u].y;
                            v.z -= cw[u].z;
                            v.w -= cw[u].w;
                            *r = v;
                        }
                    }
                }
            }
            __syncthreads();  // r updated before the next level's scores
        }
    };
    if constexpr (kList) {
        for (int base = 0; base < n_frames; base += nc * a.fc) {
            const int F = min(a.fc, n_frames - (base + cl * a.fc));
            if (F > 0) pass(base + cl * a.fc, F);
        }
    } else {
        pass(cl * a.fc, min(a.fc, n_frames - cl * a.fc));  // >= 1 frame: no empty cluster launched
    }
    // a wait that ran out (the error flag is set) may have left its stage's copy in flight:
    // wait for the last stages' copies (bounded) so that none lands after the CTA exits
    if (*abort && tid == 0) {
        for (int k = s > NST ? s - NST : 0; k < s; ++k) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&full[k % NST], (uint32_t)(k / NST) & 1u) &&
                   clock64() - t0 < kWaitBudgetCycles) {
            }
        }
    }
    if (!kList && blockIdx.x == 0 && tid == 0) atomicAdd(&a.stats[0], (unsigned long long)a.B);
    cluster_sync();  // no CTA leaves while another may still read its shared memory
}

// The thread tiles built, as (U, V): V = 4 (one warp per frame block: rows = U
// with clusters of 8) for small blocks, V = 8 (two or four warps per frame
// block) for large ones, so that every frame count from 1 to 32 has a tile with
// little padding. A plan takes the cheapest by the cost model below.
struct Tile {
    int U, V;
    const void* kernel;
};
template <int U, int V>
Tile tile() {
    return {U, V, reinterpret_cast<const void*>(k_encode_cluster<U, V, false>)};
}
const Tile kTiles[] = {tile<1, 4>(), tile<2, 4>(), tile<3, 4>(),  tile<4, 4>(),  tile<6, 4>(),
                       tile<8, 4>(), tile<5, 8>(), tile<6, 8>(),  tile<8, 8>(),  tile<9, 8>(),
                       tile<10, 8>(), tile<12, 8>(), tile<14, 8>(), tile<16, 8>()};
// The list mode's one tile: 32 frames per cluster of 8 (a pass of 32 x clusters frames).
const void* const kListKernel = reinterpret_cast<const void*>(k_encode_cluster<16, 8, true>);

cudaError_t configure_kernel(const void* k) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

cudaLaunchConfig_t launch_config(int grid, int cs, cudaStream_t s, cudaLaunchAttribute* at) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cfg;
}

// Clusters of `cs` CTAs the device can run at once (0 if it cannot run one).
int max_clusters(int cs) {
    cudaLaunchAttribute at[1];
    const cudaLaunchConfig_t cfg = launch_config(cs * 16, cs, nullptr, at);
    int n = 0;
    for (const Tile& tl : kTiles) {
        int m = 0;
        if (cudaOccupancyMaxActiveClusters(&m, tl.kernel, &cfg) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        n = (tl.kernel == kTiles[0].kernel || m < n) ? m : n;
    }
    return n;
}

// Modelled cycles of one level of a CTA: the slabs' bytes at the L2-to-shared-memory
// rate measured for one SM (~41 B/clk), against the scoring of 64 steps of 4
// dimensions (per step the larger of 8 warps x (U + V) shared-memory loads and 2
// warps per scheduler x U V FMAs; measured ~1.7x this), plus the fixed work of
// reducing, exchanging and updating (~3 000 cycles).
long long level_cycles(int cs, const Tile& tl) {
    const long long stream = (long long)(kK / cs) * 1024 / 41;
    const long long lds = 8 * (tl.U + tl.V), fma = 2 * tl.U * tl.V;
    const long long score = 64 * (lds > fma ? lds : fma) * 17 / 10;
    return (stream > score ? stream : score) + 3000;
}

}  // namespace

cudaError_t encode_cluster_configure(Tables& t) {
    t.cl_max8 = 0;
    t.cl_max16 = 0;
    for (const Tile& tl : kTiles)
        if (configure_kernel(tl.kernel) != cudaSuccess) {
            // no cluster form on this device: streaming steps take the other encoders
            cudaGetLastError();
            return cudaSuccess;
        }
    if (configure_kernel(kListKernel) != cudaSuccess) {
        cudaGetLastError();
        return cudaSuccess;
    }
    t.cl_max8 = max_clusters(8);
    t.cl_max16 = max_clusters(16);
    return cudaSuccess;
}

ClusterPlan plan_encode_cluster(const Tables& t, int B) {
    ClusterPlan p{};
    if (B <= 0) return p;
    long long best = -1;
    for (int cs = 8; cs <= 16; cs *= 2) {
        const int nmax = cs == 8 ? t.cl_max8 : t.cl_max16;
        if (nmax <= 0) continue;
        const int fc = (B + nmax - 1) / nmax;
        if (fc > kClusterMaxBlock) continue;
        const int slice = kK / cs;
        for (int i = 0; i < (int)(sizeof(kTiles) / sizeof(kTiles[0])); ++i) {
            const Tile& tl = kTiles[i];
            const int wc = slice / (8 * tl.V);
            if (wc < 1 || 8 % wc != 0) continue;
            const int rows = (8 / wc) * tl.U;
            if (rows < fc || rows > kClusterMaxBlock) continue;
            const long long c = level_cycles(cs, tl);
            if (best < 0 || c < best) {
                best = c;
                p.cs = cs;
                p.fc = fc;
                p.nc = (B + fc - 1) / fc;
                p.tile = i;
                p.U = tl.U;
                p.V = tl.V;
            }
        }
    }
    p.ok = best >= 0;
    return p;
}

cudaError_t launch_encode_cluster(const Tables& t, const ClusterPlan& p, const void* z, int dtype,
                                  int B, int n_q, int variant, int16_t* codes, cudaStream_t s,
                                  bool rescan_list) {
    if (!p.ok) return cudaErrorInvalidValue;
    ClusterArgs a;
    a.C32 = t.C32;
    a.Win32 = t.Win32;
    a.cnorm = t.cnorm;
    a.err = t.err;
    a.stats = t.stats;
    a.z = z;
    a.dtype = dtype;
    a.B = B;
    a.n_q = n_q;
    a.variant = variant;
    a.cs = p.cs;
    a.fc = p.fc;
    a.codes = codes;
    a.list = rescan_list ? t.rescan_list : nullptr;
    a.list_count = rescan_list ? t.rescan_count : nullptr;
    a.list_cap = (int)kRescanCapacity;
    cudaLaunchAttribute at[1];
    const cudaLaunchConfig_t cfg = launch_config(p.nc * p.cs, p.cs, s, at);
    const CUtensorMap* tm = p.cs == 8 ? &t.tm_C32_8 : &t.tm_C32_16;
    void* args[] = {const_cast<CUtensorMap*>(tm), &a};
    if (rescan_list && !(p.cs == 8 && p.U == 16 && p.V == 8)) return cudaErrorInvalidConfiguration;
    return cudaLaunchKernelExC(&cfg, rescan_list ? kListKernel : kTiles[p.tile].kernel, args);
}

}  // namespace mimi
