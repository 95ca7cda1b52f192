// streams.cu -- the token streams between the codec and the language model:
// delay-pattern packing of the multi-stream frame, its inverse, and the sum of
// per-stream embeddings (the Temporal Transformer's input). Declared in
// include/mimi_rvq_streams.h.
//
// Packing and unpacking are index shifts: one thread per output token, the
// delays passed by value. The embedding sum is a gather bound by memory: for
// each step, K table rows of d elements are read (K = 17, d = 4096: 139 KB in
// bf16) and one row of d is written. Three forms, chosen by shape:
//   - bf16 tables of d = 4096 (the Temporal Transformer's width), K <= 32: a
//     producer/consumer kernel that copies whole table rows into a shared-
//     memory ring with bulk copies (k_embed_sum_tma);
//   - other bf16 shapes with K <= 28: each thread copies its own 16-byte
//     pieces of several stages ahead with cp.async (k_embed_sum_async);
//   - otherwise (float32 tables, more tables): one CTA per step, each thread
//     issuing the loads of up to 8 tables' rows before adding them.
// The sum is float32, table k in order; outputs are stored with evict-first
// hints so the hot table rows keep the L2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/mimi_rvq.h"
#include "../../include/mimi_rvq_streams.h"
#include "ptx.cuh"

namespace mimi {

// Error bits (MIMI_DEV_ERR_*) of the handle-free token-stream calls: a kernel
// whose bounded wait ran out sets MIMI_DEV_ERR_TIMEOUT here, whether or not the
// caller passed an n_bad counter; mimi_rvq_streams_get_error reads and clears it.
static __device__ int g_stream_err;

namespace {

constexpr int kQ = 8;
constexpr int kThreads = 256;
constexpr int kMaxK = MIMI_RVQ_MAX_STREAMS;
constexpr int kBatch = 8;  // table rows loaded before they are added

struct Delays {
    int d[kQ];
};

// dl.d[q] without a dynamically indexed (local-memory) copy of the struct.
__device__ __forceinline__ int delay_of(const Delays& dl, int q) {
    int v = dl.d[0];
#pragma unroll
    for (int j = 1; j < kQ; ++j)
        if (q == j) v = dl.d[j];
    return v;
}

__global__ void k_delay_pack(const int32_t* __restrict__ text, const int16_t* __restrict__ audio,
                             int n_audio, int64_t T, Delays dl, int64_t S, int32_t text_pad,
                             int32_t audio_pad, int32_t* __restrict__ packed) {
    const int K = 1 + kQ * n_audio;
    const int64_t n = S * K;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t s = e / K;
        const int k = (int)(e - s * K);
        int32_t v;
        if (k == 0) {
            v = (text != nullptr && s < T) ? __ldg(text + s) : text_pad;
        } else {
            const int a = (k - 1) / kQ, q = (k - 1) % kQ;
            const int64_t t = s - delay_of(dl, q);
            v = (t >= 0 && t < T) ? (int32_t)__ldg(audio + ((int64_t)a * T + t) * kQ + q) : audio_pad;
        }
        packed[e] = v;
    }
}

__global__ void k_delay_unpack(const int32_t* __restrict__ packed, int K, int col0, Delays dl,
                               int64_t T, int16_t* __restrict__ audio) {
    const int64_t n = T * kQ;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = e / kQ;
        const int q = (int)(e - t * kQ);
        audio[e] = (int16_t)__ldg(packed + (t + delay_of(dl, q)) * K + col0 + q);
    }
}

struct Tables {
    int64_t off[kMaxK];   // first row of table k in the stacked tables
    int64_t rows[kMaxK];
};

// 8 consecutive table elements as float32.
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
}

template <typename TT, typename OT>
__global__ void __launch_bounds__(kThreads)
    k_embed_sum(const TT* __restrict__ tables, Tables tb, int K, int d,
                const int32_t* __restrict__ tokens, int64_t S, OT* __restrict__ out,
                unsigned long long* __restrict__ n_bad) {
    const int units = d / 8;
    for (int64_t s = blockIdx.x; s < S; s += gridDim.x) {
        const int32_t* tok = tokens + s * K;
        if (threadIdx.x == 0 && n_bad != nullptr) {
            unsigned bad = 0;
            for (int k = 0; k < K; ++k) {
                const int32_t id = __ldg(tok + k);
                bad += id >= 0 && id >= tb.rows[k];
            }
            if (bad) atomicAdd(n_bad, (unsigned long long)bad);
        }
        for (int u = threadIdx.x; u < units; u += kThreads) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int k0 = 0; k0 < K; k0 += kBatch) {
                float v[kBatch][8];
                bool ok[kBatch];
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    const int k = k0 + b;
                    const int32_t id = k < K ? __ldg(tok + k) : -1;
                    ok[b] = id >= 0 && id < tb.rows[k < K ? k : 0];
                    if (ok[b]) load8(tables + (tb.off[k] + id) * d + 8 * u, v[b]);
                }
#pragma unroll
                for (int b = 0; b < kBatch; ++b)
                    if (ok[b])
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[j] += v[b][j];
            }
            store8(out + s * d + 8 * u, acc);
        }
    }
}

// bf16 tables, the pipelined form: a stage is 256 consecutive 8-element units
// of one step's output (half a row at d = 4096); thread t owns unit t of every
// stage. For NST stages ahead, each thread copies its own 16-byte piece of each
// of the step's K table rows into its own shared-memory slots with cp.async
// (no registers held, no block-wide synchronisation: a thread only reads what
// it copied), then adds the K pieces of the oldest stage in table order and
// stores the unit. At K = 17 and NST = 3 that keeps 204 KB of loads in flight
// per SM.
constexpr int kStageUnits = kThreads;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int NST, typename OT>
__global__ void __launch_bounds__(kThreads, 1)
    k_embed_sum_async(const __nv_bfloat16* __restrict__ tables, Tables tb, int K, int d,
                      const int32_t* __restrict__ tokens, int64_t S, OT* __restrict__ out,
                      unsigned long long* __restrict__ n_bad) {
    extern __shared__ __align__(16) uint4 slots[];  // [NST][K][kStageUnits]
    const int t = threadIdx.x;
    const int units = d / 8;
    const int sps = (units + kStageUnits - 1) / kStageUnits;  // stages per step
    const int64_t steps_here = S > blockIdx.x ? (S - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t n_stages = steps_here * sps;
    uint32_t valid[NST];

    // copy stage j (this CTA's (j / sps)-th step, part j % sps) into buffer j % NST
    auto issue = [&](int64_t j, uint32_t& mask) {
        mask = 0;
        if (j < n_stages) {
            const int64_t s = blockIdx.x + (j / sps) * gridDim.x;
            const int u = (int)(j % sps) * kStageUnits + t;
            const int32_t* tok = tokens + s * K;
            uint4* buf = slots + (size_t)(j % NST) * K * kStageUnits;
            if (u < units)
                for (int k = 0; k < K; ++k) {
                    const int32_t id = __ldg(tok + k);
                    if (id >= 0 && id < tb.rows[k]) {
                        cp_async16(buf + k * kStageUnits + t, tables + (tb.off[k] + id) * d + 8 * u);
                        mask |= 1u << k;
                    }
                }
            if (n_bad != nullptr && t == 0 && j % sps == 0) {
                unsigned bad = 0;
                for (int k = 0; k < K; ++k) {
                    const int32_t id = __ldg(tok + k);
                    bad += id >= 0 && id >= tb.rows[k];
                }
                if (bad) atomicAdd(n_bad, (unsigned long long)bad);
            }
        }
        cp_async_commit();
    };

#pragma unroll
    for (int b = 0; b < NST; ++b) issue(b, valid[b]);
    for (int64_t j = 0; j < n_stages; ++j) {
        cp_async_wait<NST - 1>();  // this thread's copies of stage j have landed
        const int b = (int)(j % NST);
        uint32_t mask = 0;
#pragma unroll
        for (int q = 0; q < NST; ++q)
            if (q == b) mask = valid[q];
        const int64_t s = blockIdx.x + (j / sps) * gridDim.x;
        const int u = (int)(j % sps) * kStageUnits + t;
        const uint4* buf = slots + (size_t)b * K * kStageUnits;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int k = 0; k < K; ++k)
            if (mask & (1u << k)) {
                const uint4 w = buf[k * kStageUnits + t];
                const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[2 * e] += __uint_as_float(x[e] << 16);
                    acc[2 * e + 1] += __uint_as_float(x[e] & 0xFFFF0000u);
                }
            }
        if (u < units) store8(out + s * d + 8 * u, acc);
        uint32_t nm;
        issue(j + NST, nm);  // refills buffer b: this thread's reads of it are done
#pragma unroll
        for (int q = 0; q < NST; ++q)
            if (q == b) valid[q] = nm;
    }
    cp_async_wait<0>();
}

// bf16 tables, bulk-copy form (d = 4096, the Temporal Transformer's width;
// compiled for that width so every shared-memory offset is a constant). A
// stage is a group of up to G = 6 whole table rows of one step (48 KB). Producer warps
// (two, taking alternate stages) copy the group's rows into a shared-memory
// ring with one bulk copy per row (lane i issues row g*G + i; completion is
// counted on the stage's mbarrier in bytes), so neither token reads nor
// address arithmetic fall on the 16 consumer warps, which wait on a stage's
// mbarrier each at its own pace. Each consumer thread owns 8 columns, keeps
// their float32 sums across the step's row groups (table order is kept), adds
// with mixed-precision adds (bf16 operand widened exactly), and stores after
// the last group. A bulk copy costs about the
// same to issue whatever its size, so whole-row copies keep the copy count per
// byte low; at K = 17 four stages (192 KB) are in flight per SM.
constexpr int kConsumerWarps = 16;
constexpr int kProducerWarps = 2;
constexpr int kTmaThreads = 32 * (kConsumerWarps + kProducerWarps);
constexpr int kGroupBytes = 48 * 1024;   // rows per stage: as many as fit 48 KB
constexpr long long kSpinBudget = 4000000000LL;  // ~2 s: no legitimate wait comes near it

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void bar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void bar_arrive_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
// Bounded wait for the phase of the given parity; false if the budget ran out
// or another thread of the CTA already gave up (*stop != 0, unless stop is
// null; the caller then records the failure in *stop).
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, volatile int* stop,
                                         long long budget) {
    const long long t0 = clock64();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if ((stop != nullptr && *stop) || clock64() - t0 > budget) return false;
    }
}
__device__ __forceinline__ void bulk_copy(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(smem_dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
// a += float32(low bf16 of x), b += float32(high bf16 of x): mixed-precision
// adds (the bf16 operand widens exactly; one rounding each).
__device__ __forceinline__ void add_bf16x2(float& a, float& b, uint32_t x) {
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\t"
        "add.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(a), "+f"(b)
        : "r"(x));
}

// kSelfTest: the instantiation of the wait self-test. Its producers issue no
// copy and never arrive, so the consumers' first wait runs out its (short)
// budget and the failure path below runs; it reads no tokens or tables and
// stores nothing.
template <int NST, typename OT, int D, bool kSelfTest = false>
__global__ void __launch_bounds__(kTmaThreads, 1)
    k_embed_sum_tma(const __nv_bfloat16* __restrict__ tables, Tables tb, int K,
                    const int32_t* __restrict__ tokens, int64_t S, OT* __restrict__ out,
                    unsigned long long* __restrict__ n_bad, long long budget) {
    constexpr int d = D;
    constexpr int G = kGroupBytes / (2 * D) < 32 ? kGroupBytes / (2 * D) : 32;  // rows per stage
    static_assert(G >= 1 && D % 8 == 0 && D <= kConsumerWarps * 32 * 8, "shape");
    extern __shared__ __align__(128) uint8_t ring[];  // [NST][G][D] bf16
    __shared__ __align__(8) uint64_t full[NST], empty[NST];
    __shared__ uint32_t valid[NST];
    __shared__ int64_t last_issued[kProducerWarps];   // last stage each producer copied
    __shared__ volatile int failed;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = (K + G - 1) / G;
    const int64_t steps_here = S > blockIdx.x ? (S - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t n_stages = steps_here * groups;
    constexpr uint32_t row_bytes = 2u * D, stage_bytes = G * row_bytes;
    if (threadIdx.x == 0) {
        for (int b = 0; b < NST; ++b) {
            bar_init(&full[b], 1);
            bar_init(&empty[b], kConsumerWarps);
            valid[b] = 0;
        }
        for (int p = 0; p < kProducerWarps; ++p) last_issued[p] = -1;
        failed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp >= kConsumerWarps) {
        // ---- producer warps: warp p takes stages j = p, p + P, ...; none once a wait failed
        const int p = warp - kConsumerWarps;
        for (int64_t j = p; j < n_stages && !kSelfTest; j += kProducerWarps) {
            if (failed) break;
            const int b = (int)(j % NST);
            const int g = (int)(j % groups);
            const int64_t s = blockIdx.x + (j / groups) * gridDim.x;
            const int k = g * G + lane;
            const bool in = lane < G && k < K;
            const int32_t id = in ? __ldg(tokens + s * K + k) : -1;  // before the wait
            const bool ok = in && id >= 0 && id < tb.rows[in ? k : 0];
            if (n_bad != nullptr) {
                const uint32_t bad = __ballot_sync(0xffffffffu, in && id >= 0 && !ok);
                if (lane == 0 && bad) atomicAdd(n_bad, (unsigned long long)__popc(bad));
            }
            const uint32_t mask = __ballot_sync(0xffffffffu, ok);
            if (j >= NST) {  // wait until the consumers released this buffer
                int w = 1;
                if (lane == 0) w = bar_wait(&empty[b], (uint32_t)((j / NST - 1) & 1), &failed, budget);
                if (!__shfl_sync(0xffffffffu, w, 0)) {
                    if (lane == 0) failed = 1;
                    break;
                }
            }
            if (lane == 0) {
                valid[b] = mask;
                last_issued[p] = j;
                bar_arrive_tx(&full[b], (uint32_t)__popc(mask) * row_bytes);
            }
            __syncwarp();
            if (ok)
                bulk_copy(ring + b * stage_bytes + lane * row_bytes,
                          tables + (tb.off[k] + id) * d, row_bytes, &full[b]);
        }
    } else {
        // ---- consumer warps: columns [8t, 8t + 8)
        const int c8 = threadIdx.x * 8;
        float acc[8];
        for (int64_t j = 0; j < n_stages; ++j) {
            const int b = (int)(j % NST);
            const int g = (int)(j % groups);
            if (g == 0)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
            // after a failed wait the thread stops waiting but the loop runs on
            const bool have = !failed && bar_wait(&full[b], (uint32_t)((j / NST) & 1), &failed, budget);
            if (!have) failed = 1;
            const uint32_t mask = valid[b];
            if (c8 < d) {
                const uint8_t* buf = ring + b * stage_bytes + c8 * 2;
                uint4 w[G];
#pragma unroll
                for (int i = 0; i < G; ++i)
                    if ((mask >> i) & 1u) w[i] = *reinterpret_cast<const uint4*>(buf + i * row_bytes);
#pragma unroll
                for (int i = 0; i < G; ++i)
                    if ((mask >> i) & 1u) {
                        add_bf16x2(acc[0], acc[1], w[i].x);
                        add_bf16x2(acc[2], acc[3], w[i].y);
                        add_bf16x2(acc[4], acc[5], w[i].z);
                        add_bf16x2(acc[6], acc[7], w[i].w);
                    }
            }
            // a buffer is released only by warps whose every lane saw its copies land, so
            // after a failure no copy is issued into a buffer that may still be filling
            if (__all_sync(0xffffffffu, have) && lane == 0) bar_arrive(&empty[b]);
            if (!kSelfTest && g == groups - 1 && c8 < d) {
                const int64_t s = blockIdx.x + (j / groups) * gridDim.x;
                store8(out + s * d + c8, acc);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && failed) {
        atomicOr(&g_stream_err, MIMI_DEV_ERR_TIMEOUT);
        if (n_bad != nullptr) atomicExch(n_bad, ~0ull);
        // Copies already issued may still be landing in the ring; each buffer has at most
        // one (a buffer is refilled only after its previous copies landed), the last stage
        // issued into it. Wait for each of those (bounded) before the CTA exits.
        for (int b = 0; b < NST; ++b) {
            int64_t jl = -1;
            for (int p = 0; p < kProducerWarps; ++p)
                for (int64_t j = last_issued[p]; j >= 0 && j > last_issued[p] - (int64_t)kProducerWarps * NST;
                     j -= kProducerWarps)
                    if (j % NST == b && j > jl) jl = j;
            if (jl >= 0) bar_wait(&full[b], (uint32_t)((jl / NST) & 1), nullptr, budget);
        }
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool device_pointer(const void* p) {
    if (!p || !aligned16(p)) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

int grid_for(int64_t work, int per_block) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (work + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sms * 8;
    return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

int status(cudaError_t e) {
    if (e == cudaSuccess) return MIMI_RVQ_OK;
    cudaGetLastError();
    return MIMI_RVQ_ECUDA;
}

// Dynamic shared memory the ring may use (the static barriers take the rest).
constexpr int kRingLimit = 226 * 1024;

// The bulk-copy form is compiled for one row width: the Temporal Transformer's
// d = 4096 (rows of 8 KB, 6 per stage).
constexpr int kTmaWidth = 4096;

// Rows per bulk-copy stage: as many whole rows as fit kGroupBytes (at most 32).
constexpr int tma_group(int d) {
    return kGroupBytes / (d * 2) < 1 ? 1 : (kGroupBytes / (d * 2) > 32 ? 32 : kGroupBytes / (d * 2));
}

// Bulk-copy stages that fit the ring (0 or 1: the form does not apply; at most 8
// are used).
int tma_stages(int d, int K) {
    if (d != kTmaWidth || K > 32) return 0;
    const int n = kRingLimit / (tma_group(d) * d * 2);
    return n >= 8 ? 8 : n;
}

// Stages of copies in flight that fit the shared memory for K tables (0: none).
int async_stages(int K) {
    const int per_stage = K * kStageUnits * 16;
    const int n = (227 * 1024) / per_stage;
    return n >= 4 ? 4 : n;  // 2 .. 4 are instantiated
}

template <int NST, typename OT>
cudaError_t launch_embed_async_n(const void* tables, const Tables& tb, int K, int d,
                                 const int32_t* tokens, int64_t S, void* out,
                                 unsigned long long* n_bad, cudaStream_t s) {
    const int smem = NST * K * kStageUnits * 16;
    // raise the kernel's shared-memory limit once per device
    static unsigned long long configured = 0;  // bit per device
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev >= 64 || !(configured & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_embed_sum_async<NST, OT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev < 64) __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELAXED);
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)(S < sms ? S : sms);
    k_embed_sum_async<NST, OT><<<grid, kThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(tables), tb, K, d, tokens, S, static_cast<OT*>(out),
        n_bad);
    return cudaGetLastError();
}

template <int NST, typename OT>
cudaError_t launch_embed_tma_n(const void* tables, const Tables& tb, int K, int d,
                               const int32_t* tokens, int64_t S, void* out,
                               unsigned long long* n_bad, cudaStream_t s) {
    constexpr int D = kTmaWidth;
    const int smem = NST * tma_group(D) * D * 2;
    static unsigned long long configured = 0;  // bit per device
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev >= 64 || !(configured & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_embed_sum_tma<NST, OT, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingLimit);
        if (e != cudaSuccess) return e;
        if (dev < 64) __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELAXED);
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)(S < sms ? S : sms);
    (void)d;
    k_embed_sum_tma<NST, OT, D><<<grid, kTmaThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(tables), tb, K, tokens, S, static_cast<OT*>(out), n_bad,
        kSpinBudget);
    return cudaGetLastError();
}

template <typename OT>
cudaError_t launch_embed_tma(int nst, const void* tables, const Tables& tb, int K, int d,
                             const int32_t* tokens, int64_t S, void* out,
                             unsigned long long* n_bad, cudaStream_t s) {
    switch (nst >= 8 ? 8 : nst) {
        case 8: return launch_embed_tma_n<8, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
        case 7: return launch_embed_tma_n<7, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
        case 6: return launch_embed_tma_n<6, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
        case 5: return launch_embed_tma_n<5, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
        case 4: return launch_embed_tma_n<4, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
        case 3: return launch_embed_tma_n<3, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
        default: return launch_embed_tma_n<2, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
    }
}

template <typename OT>
cudaError_t launch_embed_async(int nst, const void* tables, const Tables& tb, int K, int d,
                               const int32_t* tokens, int64_t S, void* out,
                               unsigned long long* n_bad, cudaStream_t s) {
    if (nst >= 4) return launch_embed_async_n<4, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
    if (nst == 3) return launch_embed_async_n<3, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
    return launch_embed_async_n<2, OT>(tables, tb, K, d, tokens, S, out, n_bad, s);
}

template <typename TT, typename OT>
cudaError_t launch_embed(const void* tables, const Tables& tb, int K, int d, const int32_t* tokens,
                         int64_t S, void* out, unsigned long long* n_bad, cudaStream_t s) {
    k_embed_sum<TT, OT><<<grid_for(S, 1), kThreads, 0, s>>>(
        static_cast<const TT*>(tables), tb, K, d, tokens, S, static_cast<OT*>(out), n_bad);
    return cudaGetLastError();
}

// ~50 ms at 2 GHz: long enough to be a real wait, short for a test.
constexpr long long kSelftestBudget = 100000000LL;

cudaError_t launch_embed_selftest(cudaStream_t s) {
    auto* k = k_embed_sum_tma<2, __nv_bfloat16, kTmaWidth, true>;
    const int smem = 2 * tma_group(kTmaWidth) * kTmaWidth * 2;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    Tables tb{};
    k<<<1, kTmaThreads, smem, s>>>(nullptr, tb, MIMI_RVQ_MAX_STREAMS / 4, nullptr, 1, nullptr,
                                   nullptr, kSelftestBudget);
    return cudaGetLastError();
}

}  // namespace
}  // namespace mimi

extern "C" int mimi_rvq_streams_get_error(struct CUstream_st* stream) {
    using namespace mimi;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return status(cudaErrorUnknown);
    int bits = 0;
    if (cudaMemcpyFromSymbol(&bits, g_stream_err, sizeof(int)) != cudaSuccess)
        return status(cudaErrorUnknown);
    if (bits) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_stream_err, &zero, sizeof(int)) != cudaSuccess)
            return status(cudaErrorUnknown);
    }
    return (bits & MIMI_DEV_ERR_TIMEOUT) ? MIMI_RVQ_ETIMEOUT : MIMI_RVQ_OK;
}

extern "C" int mimi_rvq_streams_wait_selftest(struct CUstream_st* stream) {
    return mimi::status(mimi::launch_embed_selftest(stream));
}

extern "C" int mimi_rvq_delay_pack(const int32_t* text, const int16_t* audio, int n_audio,
                                   int64_t T, const int32_t* delays, int64_t S, int32_t text_pad,
                                   int32_t audio_pad, int32_t* packed,
                                   struct CUstream_st* stream) {
    using namespace mimi;
    if (T < 0 || S < 0 || n_audio < 0 || n_audio > 7 || !delays) return MIMI_RVQ_EINVAL;
    Delays dl;
    for (int q = 0; q < kQ; ++q) {
        if (delays[q] < 0) return MIMI_RVQ_EINVAL;
        dl.d[q] = delays[q];
    }
    if (S == 0) return MIMI_RVQ_OK;
    if (!device_pointer(packed) || (text && !device_pointer(text)) ||
        (n_audio > 0 && T > 0 && !device_pointer(audio)))
        return MIMI_RVQ_EINVAL;
    const int64_t n = S * (1 + kQ * (int64_t)n_audio);
    k_delay_pack<<<grid_for(n, kThreads), kThreads, 0, stream>>>(text, audio, n_audio, T, dl, S,
                                                                 text_pad, audio_pad, packed);
    return status(cudaGetLastError());
}

extern "C" int mimi_rvq_delay_unpack(const int32_t* packed, int64_t S, int K, int col0,
                                     const int32_t* delays, int64_t T, int16_t* audio,
                                     struct CUstream_st* stream) {
    using namespace mimi;
    if (S < 0 || T < 0 || K <= 0 || col0 < 0 || col0 + kQ > K || !delays) return MIMI_RVQ_EINVAL;
    Delays dl;
    for (int q = 0; q < kQ; ++q) {
        if (delays[q] < 0 || T + delays[q] > S) return MIMI_RVQ_EINVAL;
        dl.d[q] = delays[q];
    }
    if (T == 0) return MIMI_RVQ_OK;
    if (!device_pointer(packed) || !device_pointer(audio)) return MIMI_RVQ_EINVAL;
    k_delay_unpack<<<grid_for(T * kQ, kThreads), kThreads, 0, stream>>>(packed, K, col0, dl, T,
                                                                        audio);
    return status(cudaGetLastError());
}

extern "C" int mimi_rvq_embed_sum(const void* tables, int table_dtype, int K, const int64_t* rows,
                                  int d, const int32_t* tokens, int64_t S, void* out,
                                  int out_dtype, uint64_t* n_bad, struct CUstream_st* stream) {
    using namespace mimi;
    if (K <= 0 || K > kMaxK || d <= 0 || d % 8 != 0 || S < 0 || !rows) return MIMI_RVQ_EINVAL;
    if ((table_dtype != MIMI_RVQ_F32 && table_dtype != MIMI_RVQ_BF16) ||
        (out_dtype != MIMI_RVQ_F32 && out_dtype != MIMI_RVQ_BF16))
        return MIMI_RVQ_EINVAL;
    Tables tb;
    int64_t total = 0;
    for (int k = 0; k < K; ++k) {
        if (rows[k] <= 0) return MIMI_RVQ_EINVAL;
        tb.off[k] = total;
        tb.rows[k] = rows[k];
        total += rows[k];
    }
    for (int k = K; k < kMaxK; ++k) tb.off[k] = tb.rows[k] = 0;
    if (S == 0) return MIMI_RVQ_OK;
    if (!device_pointer(tables) || !device_pointer(tokens) || !device_pointer(out) ||
        (n_bad && (reinterpret_cast<uintptr_t>(n_bad) & 7u)))
        return MIMI_RVQ_EINVAL;
    auto* bad = reinterpret_cast<unsigned long long*>(n_bad);
    cudaError_t e;
    const int nst = async_stages(K), tst = tma_stages(d, K);
    if (table_dtype == MIMI_RVQ_BF16 && tst >= 2 && K <= 32)
        e = out_dtype == MIMI_RVQ_BF16
                ? launch_embed_tma<__nv_bfloat16>(tst, tables, tb, K, d, tokens, S, out, bad, stream)
                : launch_embed_tma<float>(tst, tables, tb, K, d, tokens, S, out, bad, stream);
    else if (table_dtype == MIMI_RVQ_BF16 && nst >= 2 && K <= 32)
        e = out_dtype == MIMI_RVQ_BF16
                ? launch_embed_async<__nv_bfloat16>(nst, tables, tb, K, d, tokens, S, out, bad, stream)
                : launch_embed_async<float>(nst, tables, tb, K, d, tokens, S, out, bad, stream);
    else if (table_dtype == MIMI_RVQ_BF16)
        e = out_dtype == MIMI_RVQ_BF16
                ? launch_embed<__nv_bfloat16, __nv_bfloat16>(tables, tb, K, d, tokens, S, out, bad, stream)
                : launch_embed<__nv_bfloat16, float>(tables, tb, K, d, tokens, S, out, bad, stream);
    else
        e = out_dtype == MIMI_RVQ_BF16
                ? launch_embed<float, __nv_bfloat16>(tables, tb, K, d, tokens, S, out, bad, stream)
                : launch_embed<float, float>(tables, tb, K, d, tokens, S, out, bad, stream);
    return status(e);
}
