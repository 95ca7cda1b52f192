// scan_body.cuh -- the float32 full-scan encode of one frame, shared by the
// handle's full-scan kernel (encode_scan.cu) and the allocation-free entry
// point (noalloc.cu), so that both compute the same sums in the same order.
//
// One 256-thread block per frame: y = W_in . z in float32 (one output per
// thread, a sequential FMA chain over the 512 latent columns), then for each of
// the first n_q codebooks every codeword's score ||c||^2 - 2 r.c in float32
// (four partial dot products, summed pairwise), a block argmin (lowest index on
// ties), and r -= chosen codeword for the levels that feed the next one.
#pragma once
#include "handle.cuh"

namespace mimi {
namespace scan {

constexpr int kThreads = 256;

__device__ __forceinline__ float load_latent(const void* z, int dtype, int64_t idx) {
    if (dtype == 1) {
        const unsigned short b = static_cast<const unsigned short*>(z)[idx];
        return __uint_as_float((uint32_t)b << 16);
    }
    return static_cast<const float*>(z)[idx];
}

// Lexicographic (score, index) minimum.
__device__ __forceinline__ void take_min(float& s, int& k, float s2, int k2) {
    if (s2 < s || (s2 == s && k2 < k)) {
        s = s2;
        k = k2;
    }
}

struct Smem {
    float z[kDin], y[kD], r[kD], red_s[kThreads / 32];
    int red_k[kThreads / 32];
};

// W(i, j) returns W_in[i][j]; callers differ only in the layout they read it from.
// variant 1 starts the acoustic chain at y - S_s (the semantic codeword removed).
template <class W>
__device__ void encode_frame(W w_in, const float* __restrict__ C, const float* __restrict__ cnorm,
                             const void* z, int dtype, int64_t frame, int n_q, int variant,
                             int16_t* codes, Smem& sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int j = tid; j < kDin; j += kThreads) sm.z[j] = load_latent(z, dtype, frame * kDin + j);
    __syncthreads();
    {
        float acc = 0.f;
        for (int j = 0; j < kDin; ++j) acc = fmaf(w_in(tid, j), sm.z[j], acc);
        sm.y[tid] = acc;
        sm.r[tid] = acc;
    }
    __syncthreads();
    for (int l = 0; l < n_q; ++l) {
        const float* target = (l == 0) ? sm.y : sm.r;
        const float* book = C + (size_t)l * kK * kD;
        float best_s = __int_as_float(0x7f800000);
        int best_k = 0x7fffffff;
        for (int k = tid; k < kK; k += kThreads) {
            const float4* c = reinterpret_cast<const float4*>(book + (size_t)k * kD);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
            for (int i = 0; i < kD / 4; ++i) {
                const float4 v = __ldg(c + i);
                a0 = fmaf(target[4 * i + 0], v.x, a0);
                a1 = fmaf(target[4 * i + 1], v.y, a1);
                a2 = fmaf(target[4 * i + 2], v.z, a2);
                a3 = fmaf(target[4 * i + 3], v.w, a3);
            }
            const float dot = (a0 + a1) + (a2 + a3);
            take_min(best_s, best_k, fmaf(-2.f, dot, cnorm[(size_t)l * kK + k]), k);
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float s2 = __shfl_xor_sync(0xffffffffu, best_s, o);
            const int k2 = __shfl_xor_sync(0xffffffffu, best_k, o);
            take_min(best_s, best_k, s2, k2);
        }
        if (lane == 0) {
            sm.red_s[warp] = best_s;
            sm.red_k[warp] = best_k;
        }
        __syncthreads();
        if (warp == 0) {
            best_s = lane < kThreads / 32 ? sm.red_s[lane] : __int_as_float(0x7f800000);
            best_k = lane < kThreads / 32 ? sm.red_k[lane] : 0x7fffffff;
            for (int o = 16; o > 0; o >>= 1) {
                const float s2 = __shfl_xor_sync(0xffffffffu, best_s, o);
                const int k2 = __shfl_xor_sync(0xffffffffu, best_k, o);
                take_min(best_s, best_k, s2, k2);
            }
            if (lane == 0) sm.red_k[0] = best_k;
        }
        __syncthreads();
        int win = sm.red_k[0];
        if (win < 0 || win >= kK) win = 0;  // only reachable with NaN / Inf inputs
        if (tid == 0) codes[frame * n_q + l] = (int16_t)win;
        if (l >= 1 || variant == 1) sm.r[tid] -= book[(size_t)win * kD + tid];
        __syncthreads();
    }
}

}  // namespace scan
}  // namespace mimi
