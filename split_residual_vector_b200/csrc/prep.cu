// prep.cu -- create-time kernels: derive every table the encode and decode
// kernels read from the float32 codebooks and projections, once per handle.
#include <cuda_bf16.h>

#include "handle.cuh"

namespace mimi {
namespace {

// bf16 copy of the codebooks (round to nearest even).
__global__ void k_to_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                          int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

// One warp per codeword: ||c||^2 in float64, rounded to float32; and the
// per-codebook maxima, rounded up, that the candidate bound needs:
// cbound[4q + 0] = max ||c||, [4q + 1] = max ||c||^2, [4q + 2] = max ||bf16(c) - c||.
__global__ void k_norms(const float* __restrict__ C, float* __restrict__ cnorm,
                        float* __restrict__ cbound) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= kQ * kK) return;
    const float* c = C + (size_t)warp * kD;
    double s = 0.0, e = 0.0;
    for (int i = lane; i < kD; i += 32) {
        const double v = (double)c[i];
        const double d = (double)__bfloat162float(__float2bfloat16_rn(c[i])) - v;
        s += v * v;
        e += d * d;
    }
    for (int o = 16; o > 0; o >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, o);
        e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (lane == 0) {
        cnorm[warp] = (float)s;
        const int q = warp / kK;
        // non-negative floats order like their bit patterns
        atomicMax(reinterpret_cast<int*>(&cbound[4 * q + 0]), __float_as_int(__double2float_ru(sqrt(s))));
        atomicMax(reinterpret_cast<int*>(&cbound[4 * q + 1]), __float_as_int(__double2float_ru(s)));
        atomicMax(reinterpret_cast<int*>(&cbound[4 * q + 2]), __float_as_int(__double2float_ru(sqrt(e))));
    }
}

// ||c||^2 / 2 as three bf16 parts whose sum is exact (a float32 has 24
// significant bits, each part takes the next 8): the B operand of the encode
// kernel's norm step, which adds ||c||^2 / 2 to every score in the tensor core.
__global__ void k_norm_split(const float* __restrict__ cnorm, __nv_bfloat16* __restrict__ out,
                             int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float x = cnorm[i] * 0.5f;
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
    out[4 * i + 0] = h;
    out[4 * i + 1] = m;
    out[4 * i + 2] = l;
    out[4 * i + 3] = __float2bfloat16_rn(0.f);
}

// W_in -> (hi, lo) bf16 split and a float32 transpose [Din][D].
__global__ void k_split_win(const float* __restrict__ W, __nv_bfloat16* __restrict__ hi,
                            __nv_bfloat16* __restrict__ lo, float* __restrict__ WT) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= kD * kDin) return;
    const int i = idx / kDin, j = idx % kDin;
    const float w = W[idx];
    const __nv_bfloat16 h = __float2bfloat16_rn(w);
    hi[idx] = h;
    lo[idx] = __float2bfloat16_rn(w - __bfloat162float(h));
    WT[(size_t)j * kD + i] = w;
}

// P[r][o] = sum_i C[r][i] * W_out[o][i] for every codeword row r of every
// codebook: the decode table (the 256 -> 512 projection of each codeword).
// float64 accumulation, 64 x 64 output tile per block, 4 x 4 per thread.
__global__ void __launch_bounds__(256) k_decode_table(const float* __restrict__ C,
                                                      const float* __restrict__ Wout,
                                                      float* __restrict__ P) {
    __shared__ double sc[16][65];
    __shared__ double sw[16][65];
    const int r0 = blockIdx.y * 64, o0 = blockIdx.x * 64;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int k0 = 0; k0 < kD; k0 += 16) {
        for (int e = threadIdx.x; e < 64 * 16; e += 256) {
            const int rr = e / 16, kk = e % 16;
            sc[kk][rr] = C[(size_t)(r0 + rr) * kD + k0 + kk];
            sw[kk][rr] = Wout[(size_t)(o0 + rr) * kD + k0 + kk];
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            double a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = sc[kk][ty + 16 * u];
                b[u] = sw[kk][tx + 16 * u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v)
            P[(size_t)(r0 + ty + 16 * u) * kDin + o0 + tx + 16 * v] = (float)acc[u][v];
}

}  // namespace

cudaError_t prep_tables(Tables& t, const float* W_out, cudaStream_t s) {
    const int64_t nC = (int64_t)kQ * kK * kD;
    k_to_bf16<<<592, 256, 0, s>>>(t.C32, t.Cbf, nC);
    cudaError_t e = cudaMemsetAsync(t.cbound, 0, sizeof(float) * 4 * kQ, s);
    if (e != cudaSuccess) return e;
    k_norms<<<(kQ * kK * 32 + 255) / 256, 256, 0, s>>>(t.C32, t.cnorm, t.cbound);
    k_norm_split<<<(kQ * kK + 255) / 256, 256, 0, s>>>(t.cnorm, t.cnorm3, kQ * kK);
    k_split_win<<<(kD * kDin + 255) / 256, 256, 0, s>>>(t.Win32, t.Win_hi, t.Win_lo, t.WinT32);
    dim3 grid(kDin / 64, kQ * kK / 64);
    k_decode_table<<<grid, 256, 0, s>>>(t.C32, W_out, t.P);
    return cudaGetLastError();
}

}  // namespace mimi
