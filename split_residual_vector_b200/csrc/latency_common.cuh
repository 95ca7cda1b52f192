// latency_common.cuh -- pieces shared by the two float32 latency encoders
// (encode_wide.cu: groups of CTAs behind global-memory barriers; encode_cluster.cu:
// thread-block clusters behind hardware cluster barriers). Both score in the
// float32 full scan's order, so both return the codes mimi_rvq_encode_scan does.
#pragma once
#include "handle.cuh"
#include "ptx.cuh"

namespace mimi {
namespace lat {

constexpr int kThreads = 256;
constexpr int RSTRIDE = kD + 4;   // padded row stride (floats) of the shared r and codeword tiles
constexpr int kProjItems = 8;     // projection outputs per thread (at most)

// Latents idx .. idx + 3 (idx a multiple of 4) as float32.
__device__ __forceinline__ float4 load_latent4(const void* z, int dtype, int64_t idx) {
    if (dtype == 1) {
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(static_cast<const unsigned short*>(z) + idx));
        return make_float4(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u),
                           __uint_as_float(b.y << 16), __uint_as_float(b.y & 0xFFFF0000u));
    }
    return __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(z) + idx));
}

// (score, index) -> one unsigned 64-bit key with the same order: score bits
// mapped to an unsigned with the float order (-0 taken as +0, so equal scores
// compare equal as in a float comparison), index in the low word.
__device__ __forceinline__ unsigned long long pack_key(float s, int k) {
    uint32_t b = __float_as_uint(s);
    if (b == 0x80000000u) b = 0u;
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)b << 32) | (uint32_t)k;
}

__device__ __forceinline__ unsigned long long umin64(unsigned long long a, unsigned long long b) {
    return a < b ? a : b;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// y = W_in . z outputs of this thread: NQ items (tid + q * 256) with offsets
// zo / wo into the staged latents and W_in rows, each a sequential FMA chain
// over the JC staged columns (inactive items compute on clamped offsets and
// are never stored). Operands are read into registers JB columns at a time
// before the chain steps that use them, so shared-memory latency is paid once
// per batch rather than once per step.
template <int NQ>
__device__ __forceinline__ void proj_chain(const float* z_s, const float* w_s, const int* zo,
                                           const int* wo, float* acc, int JC) {
    constexpr int JB = NQ >= 8 ? 4 : (NQ >= 4 ? 8 : 16);  // divides JC (a multiple of 16)
    for (int j0 = 0; j0 < JC; j0 += JB) {
        float wv[NQ][JB], zv[NQ][JB];
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
            for (int j = 0; j < JB; ++j) {
                wv[q][j] = w_s[wo[q] + j0 + j];
                zv[q][j] = z_s[zo[q] + j0 + j];
            }
#pragma unroll
        for (int j = 0; j < JB; ++j)
#pragma unroll
            for (int q = 0; q < NQ; ++q) acc[q] = fmaf(wv[q][j], zv[q][j], acc[q]);
    }
}

// proj_chain with the item count chosen at run time (nq_items uniform over the CTA).
__device__ __forceinline__ void proj_chain_any(int nq_items, const float* z_s, const float* w_s,
                                               const int* zo, const int* wo, float* acc, int JC) {
    if (nq_items <= 1) proj_chain<1>(z_s, w_s, zo, wo, acc, JC);
    else if (nq_items <= 2) proj_chain<2>(z_s, w_s, zo, wo, acc, JC);
    else if (nq_items <= 4) proj_chain<4>(z_s, w_s, zo, wo, acc, JC);
    else proj_chain<8>(z_s, w_s, zo, wo, acc, JC);
}

}  // namespace lat
}  // namespace mimi
