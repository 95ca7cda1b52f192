// encode_scan.cu -- float32 full-scan encode on CUDA cores.
//
// One 256-thread block per frame (scan_body.cuh): float32 projection, all
// 8 x 2048 scores in float32, block argmin (lowest index on ties), and for the
// acoustic levels r -= chosen codeword. It scans every codeword, so it is slow
// (about 4.2 M FMA per frame) but has no candidate pruning. It is the plain
// float32 encoder for comparison; the latency encoder (encode_wide.cu) computes
// the same scores in the same order.
#include "handle.cuh"
#include "scan_body.cuh"

namespace mimi {
namespace {

// W_in read from its transpose [Din][D]: consecutive threads read consecutive words.
struct WinTransposed {
    const float* WT;
    __device__ __forceinline__ float operator()(int i, int j) const {
        return WT[(size_t)j * kD + i];
    }
};

__global__ void __launch_bounds__(scan::kThreads) k_encode_scan(Tables t, const void* z, int dtype,
                                                                int64_t n, int n_q, int variant,
                                                                int16_t* codes) {
    __shared__ scan::Smem sm;
    for (int64_t f = blockIdx.x; f < n; f += gridDim.x)
        scan::encode_frame(WinTransposed{t.WinT32}, t.C32, t.cnorm, z, dtype, f, n_q, variant,
                           codes, sm);
}

}  // namespace

cudaError_t launch_encode_scan(const Tables& t, const void* z, int dtype, int64_t n, int n_q,
                               int variant, int16_t* codes, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int64_t cap = (int64_t)t.num_sms * 8;  // 8 resident blocks of 256 threads per SM
    const int grid = (int)(n < cap ? n : cap);
    k_encode_scan<<<grid, scan::kThreads, 0, s>>>(t, z, dtype, n, n_q, variant, codes);
    return cudaGetLastError();
}

}  // namespace mimi
