// noalloc.cu -- an encode entry point that allocates no device memory.
//
// mimi_rvq_create allocates the handle's tables with cudaMalloc. Some callers
// cannot call cudaMalloc at all: a host that lets libraries use only the
// device buffers it hands them (its own pool), or a real-time audio thread,
// where cudaMalloc / cudaFree may synchronise the device and miss the 80 ms
// frame deadline. mimi_rvq_encode_noalloc serves them without a handle: the
// caller passes the codebooks, W_in, the latents and the codes buffer, and the
// only scratch the computation needs -- the squared codeword norms that
// create would have put in the handle -- lives in the file-scope device array
// below (64 KiB on every GPU that loads the library, held until exit).
//
// It is a variant of the float32 full-scan encoder: the same arithmetic in
// the same order (so the same codes), reading W_in row-major from the caller
// and the norms from the static array instead of the handle's tables.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/mimi_rvq.h"
#include "handle.cuh"

namespace mimi {

// Squared norms of at most kQ codebooks of kK codewords (64 KiB), rewritten in
// full by every call, so nothing in it has to start at zero. Every call shares
// it: calls that overlap on the GPU race.
static __device__ __align__(256) float g_noalloc_norms[kQ * kK];

namespace {

constexpr int kThreads = 256;
constexpr int kMaxDevices = 64;

float* g_norms_addr[kMaxDevices] = {};
std::mutex g_setup_mutex;

// Device address of the static array for `dev` (the current device), looked
// up once per device. Returns nullptr if the lookup fails.
float* norms_address(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_norms_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_norms) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_norms_addr[dev] = static_cast<float*>(p);
    }
    return g_norms_addr[dev];
}

// ||c||^2 in float64, rounded to float32 (as create computes it): one warp per codeword.
__global__ void k_noalloc_norms(const float* __restrict__ C, int n_q, float* __restrict__ norms) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= n_q * kK) return;
    const float* c = C + (size_t)warp * kD;
    double s = 0.0;
    for (int i = lane; i < kD; i += 32) s += (double)c[i] * (double)c[i];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) norms[warp] = (float)s;
}

__device__ __forceinline__ float load_latent(const void* z, int dtype, int64_t idx) {
    if (dtype == 1) {
        const unsigned short b = static_cast<const unsigned short*>(z)[idx];
        return __uint_as_float((uint32_t)b << 16);
    }
    return static_cast<const float*>(z)[idx];
}

__device__ __forceinline__ void take_min(float& s, int& k, float s2, int k2) {
    if (s2 < s || (s2 == s && k2 < k)) {
        s = s2;
        k = k2;
    }
}

// One 256-thread block per frame (grid-strided): y = W_in . z, then for each
// of the first n_q codebooks the float32 score ||c||^2 - 2 r.c of all 2048
// codewords, a block argmin (lowest index on ties), and r -= chosen codeword
// for the acoustic levels.
__global__ void __launch_bounds__(kThreads) k_noalloc_scan(const float* __restrict__ C,
                                                           const float* __restrict__ W_in,
                                                           const float* __restrict__ norms,
                                                           const void* __restrict__ z, int dtype,
                                                           int64_t n, int n_q,
                                                           int16_t* __restrict__ codes) {
    __shared__ float sz[kDin], sy[kD], sr[kD], red_s[kThreads / 32];
    __shared__ int red_k[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int64_t frame = blockIdx.x; frame < n; frame += gridDim.x) {
        for (int j = tid; j < kDin; j += kThreads) sz[j] = load_latent(z, dtype, frame * kDin + j);
        __syncthreads();
        {
            const float* w = W_in + (size_t)tid * kDin;
            float acc = 0.f;
            for (int j = 0; j < kDin; ++j) acc = fmaf(w[j], sz[j], acc);
            sy[tid] = acc;
            sr[tid] = acc;
        }
        __syncthreads();
        for (int l = 0; l < n_q; ++l) {
            const float* target = (l == 0) ? sy : sr;
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
                take_min(best_s, best_k, fmaf(-2.f, dot, norms[(size_t)l * kK + k]), k);
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
            if (l >= 1) sr[tid] -= book[(size_t)win * kD + tid];
            __syncthreads();
        }
    }
}

bool is_device_buffer(const void* p) {
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u)) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace
}  // namespace mimi

extern "C" int mimi_rvq_encode_noalloc(const float* codebooks, const float* W_in,
                                       const void* latents, int dtype, int64_t N, int n_q,
                                       int16_t* codes, struct CUstream_st* stream) {
    using namespace mimi;
    if (dtype != MIMI_RVQ_F32 && dtype != MIMI_RVQ_BF16) return MIMI_RVQ_EINVAL;
    // the static scratch holds the norms of at most kQ codebooks
    if (n_q < 1 || n_q > kQ || N < 0) return MIMI_RVQ_EINVAL;
    if (N == 0) return MIMI_RVQ_OK;
    if (!is_device_buffer(codebooks) || !is_device_buffer(W_in) || !is_device_buffer(latents) ||
        !is_device_buffer(codes))
        return MIMI_RVQ_EINVAL;
    int dev = -1, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return MIMI_RVQ_ECUDA;
    if (major != 10) return MIMI_RVQ_EDEVICE;
    float* norms = norms_address(dev);
    if (!norms) return MIMI_RVQ_ECUDA;
    k_noalloc_norms<<<(n_q * kK * 32 + 255) / 256, 256, 0, stream>>>(codebooks, n_q, norms);
    const int grid = (int)(N < 148 * 8 ? N : 148 * 8);
    k_noalloc_scan<<<grid, kThreads, 0, stream>>>(codebooks, W_in, norms, latents, dtype, N, n_q,
                                                  codes);
    return cudaGetLastError() == cudaSuccess ? MIMI_RVQ_OK : MIMI_RVQ_ECUDA;
}
