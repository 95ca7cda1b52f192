// encode_scan.cu -- float32 full-scan encode on CUDA cores.
//
// One 256-thread block per frame: y = W_in . z in float32 (one output per
// thread, index order), then for each codebook every codeword's score
// ||c||^2 - 2 r.c in float32, a block argmin (lowest index on ties), and for
// the acoustic levels r -= chosen codeword. It scans all 2048 x 8 codewords,
// so it is slow (about 4.2 M FMA per frame) but has no candidate pruning.
// It is the plain float32 encoder for comparison; the latency encoder
// (encode_wide.cu) computes the same scores in the same order.
#include "handle.cuh"

namespace mimi {
namespace {

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

__device__ void scan_one_frame(const Tables& t, const void* z, int dtype, int64_t frame,
                               int n_q, int variant, int16_t* codes, float* sz, float* sy,
                               float* sr, float* red_s, int* red_k) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int j = tid; j < kDin; j += kThreads) sz[j] = load_latent(z, dtype, frame * kDin + j);
    __syncthreads();
    {
        float acc = 0.f;
        for (int j = 0; j < kDin; ++j) acc = fmaf(t.WinT32[(size_t)j * kD + tid], sz[j], acc);
        sy[tid] = acc;
        sr[tid] = acc;
    }
    __syncthreads();
    for (int l = 0; l < n_q; ++l) {
        const float* target = (l == 0) ? sy : sr;
        const float* book = t.C32 + (size_t)l * kK * kD;
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
            const float s = fmaf(-2.f, dot, t.cnorm[(size_t)l * kK + k]);
            take_min(best_s, best_k, s, k);
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float s2 = __shfl_xor_sync(0xffffffffu, best_s, o);
            const int k2 = __shfl_xor_sync(0xffffffffu, best_k, o);
            take_min(best_s, best_k, s2, k2);
        }
        if (lane == 0) {
            red_s[warp] = best_s;
            red_k[warp] = best_k;
        }
        __syncthreads();
        if (warp == 0) {
            best_s = lane < kThreads / 32 ? red_s[lane] : __int_as_float(0x7f800000);
            best_k = lane < kThreads / 32 ? red_k[lane] : 0x7fffffff;
            for (int o = 16; o > 0; o >>= 1) {
                const float s2 = __shfl_xor_sync(0xffffffffu, best_s, o);
                const int k2 = __shfl_xor_sync(0xffffffffu, best_k, o);
                take_min(best_s, best_k, s2, k2);
            }
            if (lane == 0) red_k[0] = best_k;
        }
        __syncthreads();
        int win = red_k[0];
        if (win < 0 || win >= kK) win = 0;  // only reachable with NaN / Inf inputs
        if (tid == 0) codes[frame * n_q + l] = (int16_t)win;
        // acoustic levels chain on r; variant 1 also starts the chain at y - S_s
        if (l >= 1 || variant == 1) sr[tid] -= book[(size_t)win * kD + tid];
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads) k_encode_scan(Tables t, const void* z, int dtype,
                                                          int64_t n, int n_q, int variant,
                                                          int16_t* codes) {
    __shared__ float sz[kDin], sy[kD], sr[kD], red_s[kThreads / 32];
    __shared__ int red_k[kThreads / 32];
    for (int64_t f = blockIdx.x; f < n; f += gridDim.x)
        scan_one_frame(t, z, dtype, f, n_q, variant, codes, sz, sy, sr, red_s, red_k);
}

}  // namespace

cudaError_t launch_encode_scan(const Tables& t, const void* z, int dtype, int64_t n, int n_q,
                               int variant, int16_t* codes, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int grid = (int)(n < 148 * 8 ? n : 148 * 8);
    k_encode_scan<<<grid, kThreads, 0, s>>>(t, z, dtype, n, n_q, variant, codes);
    return cudaGetLastError();
}

}  // namespace mimi
