// handle.cuh -- the device-resident tables behind a mimi_rvq_t handle and the
// launch entry points of each kernel file.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mimi {

constexpr int kDin = 512;     // latent width
constexpr int kD = 256;       // projected width
constexpr int kK = 2048;      // codewords per codebook
constexpr int kQ = 8;         // codebooks: 0 semantic, 1..7 acoustic

// Frames whose candidate set could not be certified are re-encoded by the
// float32 full scan; the work list holds at most this many frames per launch
// of the tensor-core kernel (encode is split into chunks of this size, so the
// list cannot overflow).
constexpr int64_t kRescanCapacity = 1 << 20;

struct Tables {
    // float32 originals
    float* C32 = nullptr;         // [Q][K][D] codebooks (0 semantic)
    float* Win32 = nullptr;       // [D][Din] W_in
    float* WinT32 = nullptr;      // [Din][D] W_in transposed (the full-scan kernel's layout)
    // derived at create
    __nv_bfloat16* Cbf = nullptr;     // [Q][K][D] bf16(C), candidate-pass B operand
    __nv_bfloat16* Win_hi = nullptr;  // [D][Din] bf16(W_in)
    __nv_bfloat16* Win_lo = nullptr;  // [D][Din] bf16(W_in - Win_hi)
    float* cnorm = nullptr;           // [Q][K] ||c||^2 (float64 sum, rounded)
    float* cbound = nullptr;          // [Q][4]: max ||c||, max ||c||^2, max ||bf16(c) - c||, 0 (rounded up)
    float* P = nullptr;               // [Q][K][Din] W_out . c (float64 sum, rounded): decode rows
    // device state
    int* err = nullptr;               // error bits (MIMI_DEV_ERR_*)
    int* rescan_count = nullptr;      // frames queued for the full scan in this launch
    int* rescan_list = nullptr;       // [kRescanCapacity] frame indices
    unsigned long long* stats = nullptr;  // [0] frames encoded, [1] frames re-scanned
    // TMA descriptors (bf16, 64 x 128 boxes, 128-byte swizzle)
    CUtensorMap tm_C;             // Cbf as [Q*K rows][D cols]
    CUtensorMap tm_Whi;           // Win_hi as [D rows][Din cols]
    CUtensorMap tm_Wlo;           // Win_lo
};

// prep.cu
cudaError_t prep_tables(Tables& t, const float* W_out, cudaStream_t s);
// encode_tc.cu
cudaError_t encode_tc_configure();  // once per device, before the first launch
// n_q codebooks (0 = projection only, writing y_out [n][256]); codes [n][n_q];
// variant 1 runs the acoustic RVQ on y - S_s.
// prof (nullable, device, 16 counters): per-role cycle counters, see ProfSlot.
cudaError_t launch_encode_tc(const Tables& t, const void* z, int dtype, int64_t n, int n_q,
                             int variant, int16_t* codes, float* y_out, cudaStream_t s,
                             int max_ctas, unsigned long long* prof = nullptr);
// encode_scan.cu
cudaError_t launch_encode_scan(const Tables& t, const void* z, int dtype, int64_t n, int n_q,
                               int variant, int16_t* codes, cudaStream_t s);
cudaError_t launch_rescan(const Tables& t, const void* z, int dtype, int n_q, int variant,
                          int16_t* codes, cudaStream_t s);
// decode.cu
cudaError_t launch_decode(const Tables& t, const int16_t* codes, int64_t n, int n_q, float* out,
                          cudaStream_t s);

}  // namespace mimi
