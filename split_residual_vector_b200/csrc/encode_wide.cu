// encode_wide.cu -- latency encode for small batches, group form: the float32
// re-encode of the frames the batch tensor-core encoder could not certify, and
// streaming steps on a device without the cluster form (encode_cluster.cu).
//
// The tensor-core encoder gives each 128-frame tile to one SM, which then
// walks the 8 codebooks in series: a batch of a few frames occupies one SM and
// waits out the whole chain. Here the work of a small batch is spread over the
// whole GPU instead. Frames are cut into groups of at most 64; each group gets
// S CTAs, and each CTA scores a slice of every codebook against all frames of
// its group on the CUDA cores, in float32:
//
//   score(f, k) = ||c_k||^2 - 2 r_f . c_k      (4 partial sums, as the full scan)
//
// Each CTA writes, per frame, the minimum over its slice of the key
// (order-preserving score bits, codeword index) to its own slot; a barrier
// among the group's CTAs (bounded spin) closes the level, and every CTA then
// reduces the S slots of each frame -- so the lowest score wins and ties go to
// the lowest index -- and applies the same residual update to its own copy of
// r in shared memory: one barrier per level. The projection y = W_in . z is
// split over the group's CTAs as frame blocks x output blocks and exchanged
// through global memory behind one more barrier. Every sum is taken in the
// float32 full scan's order, so the codes are the ones mimi_rvq_encode_scan
// returns.
//
// Codeword chunks are double-buffered with cp.async; the next level's first
// chunk does not depend on the winners, so its copy overlaps the barrier.
//
// All CTAs of a launch must be resident at once (they wait on one another):
// the launch is cooperative and the grid never exceeds the SM count.
#include "latency_common.cuh"

namespace mimi {
namespace {

using lat::cp_async16;
using lat::cp_async_commit;
using lat::cp_async_wait_all;
using lat::kProjItems;
using lat::kThreads;
using lat::load_latent4;
using lat::pack_key;
using lat::RSTRIDE;
using lat::umin64;
constexpr int FG = kWideGroupFrames;    // frames per group

struct WideArgs {
    const float* C32;
    const float* Win32;
    const float* cnorm;
    int* err;
    unsigned long long* stats;
    const void* z;
    int dtype, B, n_q, variant;
    int groups, S, per_k, jc, fb;
    int16_t* codes;
    float* y;                       // [B][256] projection exchange
    unsigned* bars;                 // [kWideMaxGroups][kWideBarStride] barrier words
    unsigned long long* partial;    // [n_q][groups][FG][S] per-CTA minimum keys
    // list mode (re-scan of the frames the tensor-core encoder could not certify):
    // frames list[0 .. min(*list_count, list_cap)), taken B at a time; nullptr: frames 0..B-1
    const int* list;
    const int* list_count;
    int list_cap;
};

// Copy the codeword rows of chunk c (level c / nch) into buf.
template <int KS>
__device__ __forceinline__ void issue_chunk(const WideArgs& a, float* buf, int c, int nch, int k_lo,
                                            int k_hi) {
    const int l = c / nch;
    const int kc = k_lo + (c - l * nch) * KS;
    const int nk = min(KS, k_hi - kc);
    const float* src = a.C32 + ((size_t)l * kK + kc) * kD;
    for (int e = threadIdx.x; e < nk * (kD / 4); e += kThreads) {
        const int k = e / (kD / 4), i4 = e % (kD / 4);
        cp_async16(buf + k * RSTRIDE + 4 * i4, src + (size_t)k * kD + 4 * i4);
    }
    cp_async_commit();
}

// Thread tile: U frames (tf + 16u) x V codewords (tk + 16v) of the current
// chunk of 16V codewords; 4 partial sums each, as the full scan.
template <int U, int V>
__global__ void __launch_bounds__(kThreads, 1) k_encode_wide(WideArgs a) {
    constexpr int KS = 16 * V;
    // global loads per thread issued together: many for groups of more than 16
    // frames (fewer for the largest thread tile, whose scoring registers leave less
    // room); 4 for the smallest steps, which have few loads to batch and are
    // measured faster with the smaller register footprint
    constexpr int kBatch = U == 1 ? 4 : (U * V >= 16 ? 8 : 16);
    extern __shared__ __align__(16) float smem_w[];
    // c_buf0 | r_s | c_buf1 ; the projection stages its operands over r_s .. c_buf1
    auto cbuf = [&](int c) { return smem_w + ((c & 1) ? (KS + FG) * RSTRIDE : 0); };
    float* r_s = smem_w + KS * RSTRIDE;
    __shared__ int win_s[FG];
    const int tid = threadIdx.x;
    const int S = a.S;
    __shared__ int frame_s[FG];
    const int group = blockIdx.x / S, member = blockIdx.x % S;
    const int f0 = group * FG;
    unsigned* bar = a.bars + group * kWideBarStride;

    const int k_lo = member * a.per_k, k_hi = min(kK, k_lo + a.per_k);
    const int nch = (k_hi - k_lo + KS - 1) / KS;
    const int total = a.n_q * nch;
    const int tf = tid >> 4, tk = tid & 15;
    int n_frames = a.B;
    if (a.list != nullptr) {
        n_frames = min(__ldcg(a.list_count), a.list_cap);
        if (blockIdx.x == 0 && tid == 0 && n_frames > 0)
            atomicAdd(&a.stats[1], (unsigned long long)n_frames);
    }
    unsigned episode = 0;
    int frames_done = 0;

    for (int base = 0; base < n_frames; base += a.B) {
        // this group's frames of the batch (all members agree, so a group with none skips it)
        const int F = min(FG, min(a.B, n_frames - base) - f0);
        if (F <= 0) continue;
        const int next_base = base + a.B;
        const bool final_batch = next_base >= n_frames || n_frames - next_base <= f0;
        if (tid < F) frame_s[tid] = a.list != nullptr ? __ldg(a.list + base + f0 + tid) : base + f0 + tid;
        __syncthreads();
        issue_chunk<KS>(a, cbuf(0), 0, nch, k_lo, k_hi);

        // ---- y = W_in . z, the group's frames x 256 outputs split over its S CTAs as
        //      fb frame blocks x S / fb output blocks: this CTA computes frames
        //      [fb0, fb1) x outputs [d0, d1), each output a sequential FMA chain over j
        //      (the full scan's order). The latents and W_in rows are staged in passes of
        //      JC columns (row stride JC + 1: conflict-free column reads), with batched
        //      vector loads.
        {
            const int OB = S / a.fb;
            const int fpb = (F + a.fb - 1) / a.fb, opb = (kD + OB - 1) / OB;
            const int fb0 = min(F, (member / OB) * fpb), fb1 = min(F, fb0 + fpb), nf = fb1 - fb0;
            const int d0 = min(kD, (member % OB) * opb), d1 = min(kD, d0 + opb), nd = d1 - d0;
            const int items = nf * nd;
            const int JC = a.jc, JS = JC + 1, J4 = JC / 4;
            float* z_s = r_s;             // [nf][JS]
            float* w_s = r_s + nf * JS;   // [nd][JS]
            const int nq_items = (items + kThreads - 1) / kThreads;  // uniform over the CTA
            int zo[kProjItems], wo[kProjItems];
            bool act[kProjItems];
            float acc[kProjItems];
#pragma unroll
            for (int q = 0; q < kProjItems; ++q) {
                const int it = tid + q * kThreads;
                act[q] = it < items;
                zo[q] = act[q] ? (it / nd) * JS : 0;
                wo[q] = act[q] ? (it % nd) * JS : 0;
                acc[q] = 0.f;
            }
            for (int j0 = 0; j0 < kDin; j0 += JC) {
                __syncthreads();
                const int nz = nf * J4, nt = (nf + nd) * J4;
                for (int e0 = tid; e0 < nt; e0 += kBatch * kThreads) {
                    float4 v[kBatch];
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int e = e0 + u * kThreads;
                        if (e < nz)
                            v[u] = load_latent4(a.z, a.dtype, (int64_t)frame_s[fb0 + e / J4] * kDin + j0 + 4 * (e % J4));
                        else if (e < nt)
                            v[u] = __ldg(reinterpret_cast<const float4*>(
                                a.Win32 + (size_t)(d0 + (e - nz) / J4) * kDin + j0 + 4 * ((e - nz) % J4)));
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
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
                lat::proj_chain_any(nq_items, z_s, w_s, zo, wo, acc, JC);
            }
#pragma unroll
            for (int q = 0; q < kProjItems; ++q)
                if (act[q]) {
                    const int it = tid + q * kThreads;
                    a.y[(size_t)(f0 + fb0 + it / nd) * kD + d0 + it % nd] = acc[q];
                }
        }
        ++episode;
        group_arrive(bar);
        if (!group_wait(bar, S * episode, a.err)) {
            cp_async_wait_all();
            return;
        }
        for (int e = tid; e < FG * (kD / 4); e += kThreads) {
            const int f = e / (kD / 4), i4 = e % (kD / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (f < F) v = __ldcg(reinterpret_cast<const float4*>(a.y + (size_t)(f0 + f) * kD) + i4);
            *reinterpret_cast<float4*>(r_s + f * RSTRIDE + 4 * i4) = v;
        }

        // partial-key reduction: TPF threads per frame (a power of two, <= 32)
        int tpf = 32;
        while (tpf * F > kThreads) tpf >>= 1;
        const int rf = tid / tpf, rsub = tid % tpf;

        int c = 0;
        for (int l = 0; l < a.n_q; ++l) {
            const float* cn = a.cnorm + (size_t)l * kK;
            unsigned long long mk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) mk[u] = ~0ull;
            for (int kc = k_lo; kc < k_hi; kc += KS, ++c) {
                const int nk = min(KS, k_hi - kc);
                cp_async_wait_all();
                __syncthreads();  // chunk c landed; chunk c - 1 consumed; r_s up to date
                if (c + 1 < total) issue_chunk<KS>(a, cbuf(c + 1), c + 1, nch, k_lo, k_hi);
                const float* c_s = cbuf(c);
                // the chunk's ||c||^2, loaded before the dot products so that their latency
                // is hidden (for the widest codeword tile after them: it was measured
                // slower there, its accumulators leave no registers to spare)
                float cnv[V];
                if constexpr (V <= 2) {
#pragma unroll
                    for (int v = 0; v < V; ++v) cnv[v] = tk + 16 * v < nk ? __ldg(cn + kc + tk + 16 * v) : 0.f;
                }
                float acc[U][V][4];
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int v = 0; v < V; ++v)
#pragma unroll
                        for (int w = 0; w < 4; ++w) acc[u][v][w] = 0.f;
#pragma unroll 4
                for (int i = 0; i < kD; i += 4) {
                    float4 rv[U], cv[V];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        rv[u] = *reinterpret_cast<const float4*>(r_s + (tf + 16 * u) * RSTRIDE + i);
#pragma unroll
                    for (int v = 0; v < V; ++v)
                        cv[v] = *reinterpret_cast<const float4*>(c_s + (tk + 16 * v) * RSTRIDE + i);
#pragma unroll
                    for (int u = 0; u < U; ++u)
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            acc[u][v][0] = fmaf(rv[u].x, cv[v].x, acc[u][v][0]);
                            acc[u][v][1] = fmaf(rv[u].y, cv[v].y, acc[u][v][1]);
                            acc[u][v][2] = fmaf(rv[u].z, cv[v].z, acc[u][v][2]);
                            acc[u][v][3] = fmaf(rv[u].w, cv[v].w, acc[u][v][3]);
                        }
                }
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int k = tk + 16 * v;
                    if (k < nk) {
                        if constexpr (V > 2) cnv[v] = __ldg(cn + kc + k);
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const float dot = (acc[u][v][0] + acc[u][v][1]) + (acc[u][v][2] + acc[u][v][3]);
                            mk[u] = umin64(mk[u], pack_key(fmaf(-2.f, dot, cnv[v]), kc + k));
                        }
                    }
                }
            }
            // this CTA's minimum per frame -> its slot
            unsigned long long* part = a.partial + ((size_t)l * a.groups + group) * FG * S;
#pragma unroll
            for (int u = 0; u < U; ++u) {
#pragma unroll
                for (int o = 8; o > 0; o >>= 1)
                    mk[u] = umin64(mk[u], __shfl_xor_sync(0xffffffffu, mk[u], o));
                const int f = tf + 16 * u;
                if (tk == 0 && f < F) __stcg(part + (size_t)f * S + member, mk[u]);
            }
            // after the last level only member 0 (which writes the codes) needs the
            // winners; the others move on once they have arrived
            ++episode;
            group_arrive(bar);
            const bool last = l == a.n_q - 1;
            if (last && member != 0) break;
            if (!group_wait(bar, S * episode, a.err)) {
                cp_async_wait_all();
                return;
            }
            // winners: minimum over the group's S slots of each frame (loads in batches of
            // kBatch, all in flight together)
            {
                unsigned long long m = ~0ull;
                if (rf < F)
                    for (int s0 = rsub; s0 < S; s0 += kBatch * tpf) {
                        unsigned long long v[kBatch];
#pragma unroll
                        for (int u = 0; u < kBatch; ++u) {
                            const int sl = s0 + u * tpf;
                            v[u] = sl < S ? __ldcg(part + (size_t)rf * S + sl) : ~0ull;
                        }
#pragma unroll
                        for (int u = 0; u < kBatch; ++u) m = umin64(m, v[u]);
                    }
                for (int o = tpf >> 1; o > 0; o >>= 1) m = umin64(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (rsub == 0 && rf < F) {
                    int w = (int)(uint32_t)m;
                    if (w < 0 || w >= kK) w = 0;  // only reachable with NaN / Inf inputs
                    win_s[rf] = w;
                    if (member == 0) a.codes[(size_t)frame_s[rf] * a.n_q + l] = (int16_t)w;
                }
            }
            if (last) {
                // after the group's last batch every member has arrived for the last
                // time: reset the count for the next launch (or graph replay)
                if (final_batch && tid == 0) atomicExch(bar, 0u);
                break;
            }
            __syncthreads();
            // acoustic levels chain on r; variant 1 also starts the chain at y - S_s
            if (l < a.n_q - 1 && (l >= 1 || a.variant == 1)) {
                // the winners' rows in batches of kBatch loads per thread, all in flight
                // before the subtractions
                const float* book = a.C32 + (size_t)l * kK * kD;
                const int ne = F * (kD / 4);
                for (int e0 = tid; e0 < ne; e0 += kBatch * kThreads) {
                    float4 cw[kBatch];
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int e = e0 + u * kThreads;
                        if (e < ne)
                            cw[u] = __ldg(reinterpret_cast<const float4*>(book + (size_t)win_s[e / (kD / 4)] * kD) +
                                          e % (kD / 4));
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int e = e0 + u * kThreads;
                        if (e < ne) {
                            float4* r = reinterpret_cast<float4*>(r_s + (e / (kD / 4)) * RSTRIDE + 4 * (e % (kD / 4)));
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
        }
        frames_done += F;
        __syncthreads();  // frame_s and the buffers are rewritten by the next batch
    }  // batches
    if (a.list == nullptr && member == 0 && tid == 0 && frames_done > 0)
        atomicAdd(&a.stats[0], (unsigned long long)frames_done);
}

int smem_bytes(int V) { return (2 * 16 * V + FG) * RSTRIDE * 4; }

template <int U, int V>
cudaError_t configure_one() {
    return cudaFuncSetAttribute(k_encode_wide<U, V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_bytes(V));
}

template <int U>
const void* pick_v(int V) {
    if (V == 1) return reinterpret_cast<const void*>(k_encode_wide<U, 1>);
    if (V == 2) return reinterpret_cast<const void*>(k_encode_wide<U, 2>);
    return reinterpret_cast<const void*>(k_encode_wide<U, 4>);
}

const void* pick_kernel(int U, int V) {
    if (U == 1) return pick_v<1>(V);
    if (U == 2) return pick_v<2>(V);
    return pick_v<4>(V);
}

}  // namespace

WidePlan plan_encode_wide(int B, int num_sms) {
    WidePlan p{};
    if (B <= 0 || B > kWideMaxFrames) return p;
    p.groups = (B + FG - 1) / FG;
    if (p.groups > num_sms || p.groups > kWideMaxGroups) return p;
    const int s_max = num_sms / p.groups;
    // codewords per CTA: a multiple of 16, at least 16
    int per_k = (kK + s_max - 1) / s_max;
    per_k = (per_k + 15) / 16 * 16;
    p.per_k = per_k;
    p.S = (kK + per_k - 1) / per_k;
    p.grid = p.groups * p.S;
    const int fmax = B < FG ? B : FG;
    p.U = fmax <= 16 ? 1 : fmax <= 32 ? 2 : 4;
    p.V = per_k <= 16 ? 1 : per_k <= 32 ? 2 : 4;
    // projection: the frames x outputs of a group split into fb frame blocks x
    // S / fb output blocks (fb a power of two dividing S, at most the frames),
    // chosen to stage the fewest rows (latents + W_in) per CTA; at most kProjItems
    // outputs per thread, operands staged in chunks of jc latent columns over the r
    // tile and the second codeword buffer
    int best_rows = 1 << 30;
    for (int fb = 1; fb <= fmax && p.S % fb == 0; fb *= 2) {
        const int rows = (fmax + fb - 1) / fb + (kD + p.S / fb - 1) / (p.S / fb);
        if (rows < best_rows) {
            best_rows = rows;
            p.fb = fb;
        }
    }
    const int fpb = (fmax + p.fb - 1) / p.fb, opb = (kD + p.S / p.fb - 1) / (p.S / p.fb);
    if (fpb * opb > kProjItems * kThreads) return p;
    const int region = (FG + 16 * p.V) * RSTRIDE;
    for (int jc = kDin; jc >= 16; jc >>= 1)
        if ((fpb + opb) * (jc + 1) <= region) {
            p.jc = jc;
            break;
        }
    if (p.jc == 0) return p;
    p.smem = smem_bytes(p.V);
    p.ok = true;
    return p;
}

size_t wide_partial_bytes(int num_sms) {
    return sizeof(unsigned long long) * (size_t)kQ * num_sms * FG;
}

cudaError_t encode_wide_configure() {
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = configure_one<1, 1>();
    if (e == cudaSuccess) e = configure_one<1, 2>();
    if (e == cudaSuccess) e = configure_one<1, 4>();
    if (e == cudaSuccess) e = configure_one<2, 1>();
    if (e == cudaSuccess) e = configure_one<2, 2>();
    if (e == cudaSuccess) e = configure_one<2, 4>();
    if (e == cudaSuccess) e = configure_one<4, 1>();
    if (e == cudaSuccess) e = configure_one<4, 2>();
    if (e == cudaSuccess) e = configure_one<4, 4>();
    return e;
}

cudaError_t launch_encode_wide(const Tables& t, const WidePlan& p, const void* z, int dtype, int B,
                               int n_q, int variant, int16_t* codes, cudaStream_t s,
                               bool rescan_list) {
    if (!p.ok) return cudaErrorInvalidValue;
    WideArgs a;
    a.list = rescan_list ? t.rescan_list : nullptr;
    a.list_count = rescan_list ? t.rescan_count : nullptr;
    a.list_cap = (int)kRescanCapacity;
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
    a.groups = p.groups;
    a.S = p.S;
    a.per_k = p.per_k;
    a.jc = p.jc;
    a.fb = p.fb;
    a.codes = codes;
    a.y = t.wide_y;
    a.bars = t.wide_bars;
    a.partial = t.wide_partial;
    void* args[] = {&a};
    return cudaLaunchCooperativeKernel(pick_kernel(p.U, p.V), dim3(p.grid), dim3(kThreads), args,
                                       p.smem, s);
}

}  // namespace mimi
