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

// Frames whose candidate set could not be certified are re-encoded in float32
// by the wide encoder; the work list holds at most this many frames per launch
// of the tensor-core kernel (encode is split into chunks of this size, so the
// list cannot overflow).
constexpr int64_t kRescanCapacity = 1 << 20;

// Largest batch the group form of the latency encoder takes: the float32
// re-encode of the frames the batch tensor-core encoder could not certify, 1024
// at a time, and (on a device without the cluster form) streaming steps up to
// kSlicedMinFrames - 1 frames.
constexpr int kWideMaxFrames = 1024;
constexpr int kWideGroupFrames = 64;  // frames per group of the latency encoder
constexpr int kWideMaxGroups = 64;    // group barriers (the last one is the wait self-test's)
constexpr int kWideBarStride = 32;    // words per group barrier (count, generation; own 128 B line)

// Codebook-sliced form of the tensor-core encoder (streaming steps): each group
// of up to 128 frames gets kSlices CTAs, one per 256-codeword score tile of a
// level; the CTAs of a group exchange their candidate lists through global
// memory behind a group barrier (group barriers kSliceBarBase .. + groups - 1 of
// wide_bars, which the latency encoder and the wait self-test do not use).
constexpr int kSlices = 8;
constexpr int kSliceMaxGroups = 18;   // 18 x 8 CTAs fit on 148 SMs, one CTA each
constexpr int kSliceBarBase = 32;
constexpr int kSliceListFloats = 10;  // per row: 8 candidate keys, best, evicted
// Streaming steps the cluster form cannot take (more than 32 frames per cluster)
// run the sliced tensor-core encoder when its CTAs fit the device. On a device
// without the cluster form, steps of fewer than kSlicedMinFrames frames run the
// group form of the latency encoder instead. Measured per step on B200: the group
// form 52 us at 1 frame, 105 us at 128, 136 us at 256, 211-219 us from 320 to 511
// frames; the sliced encoder 207-209 us from 256 to 511 frames, 215 us at 1024.
constexpr int kSlicedMinFrames = 257;

// Cluster form of the latency encoder (streaming steps): blocks of at most
// kClusterMaxBlock frames, one per cluster of 8 or 16 CTAs, all clusters resident
// at once (so steps of at most kClusterMaxBlock x the clusters the device runs).
constexpr int kClusterMaxBlock = 32;

struct Tables {
    int num_sms = 148;            // SMs of the handle's device (grid sizes)
    int cl_max8 = 0;              // cluster form: clusters of 8 CTAs the device runs at once
    int cl_max16 = 0;             //   and of 16 (0: that size is not available)
    // float32 originals
    float* C32 = nullptr;         // [Q][K][D] codebooks (0 semantic)
    float* Win32 = nullptr;       // [D][Din] W_in
    float* WinT32 = nullptr;      // [Din][D] W_in transposed (the full-scan kernel's layout)
    // derived at create
    __nv_bfloat16* Cbf = nullptr;     // [Q][K][D] bf16(C), candidate-pass B operand
    __nv_bfloat16* Win_hi = nullptr;  // [D][Din] bf16(W_in)
    __nv_bfloat16* Win_lo = nullptr;  // [D][Din] bf16(W_in - Win_hi)
    float* cnorm = nullptr;           // [Q][K] ||c||^2 (float64 sum, rounded)
    __nv_bfloat16* cnorm3 = nullptr;  // [Q][K][4] (h, m, l, 0): h + m + l = cnorm / 2 exactly
    float* cbound = nullptr;          // [Q][4]: max ||c||, max ||c||^2, max ||bf16(c) - c||, 0 (rounded up)
    float* P = nullptr;               // [Q][K][Din] W_out . c (float64 sum, rounded): decode rows
    // device state
    int* err = nullptr;               // error bits (MIMI_DEV_ERR_*)
    int* rescan_count = nullptr;      // frames queued for the full scan in this launch
    int* rescan_list = nullptr;       // [kRescanCapacity] frame indices
    unsigned long long* stats = nullptr;  // [0] frames encoded, [1] frames re-scanned
    float* wide_y = nullptr;          // [kWideMaxFrames][D] latency encoder: projection exchange
    unsigned* wide_bars = nullptr;                // [kWideMaxGroups][kWideBarStride] group barriers
    unsigned long long* wide_partial = nullptr;   // per-CTA minimum keys, wide_partial_bytes()
    float* slice_lists = nullptr;   // [2][kSliceMaxGroups][kSlices][128][kSliceListFloats] sliced encoder
    float2* slice_exact = nullptr;  // [kSliceMaxGroups][128][kSlices] sliced encoder: exact-scan bests
    // TMA descriptors (bf16, 64 x 256 boxes, 128-byte swizzle)
    CUtensorMap tm_C;             // Cbf as [Q*K rows][D cols]
    CUtensorMap tm_Whi;           // Win_hi as [D rows][Din cols]
    CUtensorMap tm_Wlo;           // Win_lo
    CUtensorMap tm_C32_8;         // C32 as [Q*K rows][D cols] fp32, boxes of 32 columns x K / 8
                                  // rows (the cluster form's slabs), 128-byte swizzle
    CUtensorMap tm_C32_16;        // the same with K / 16 rows
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
// Codebook-sliced tensor-core encode of B frames (one cooperative launch of
// ceil(B / 128) * kSlices CTAs); false from sliced_fits if B is outside
// (0, 128 * kSliceMaxGroups] or the CTAs do not fit on the device at once.
bool sliced_fits(int B, int num_sms);
cudaError_t launch_encode_tc_sliced(const Tables& t, const void* z, int dtype, int B, int n_q,
                                    int variant, int16_t* codes, cudaStream_t s);
// encode_scan.cu
cudaError_t launch_encode_scan(const Tables& t, const void* z, int dtype, int64_t n, int n_q,
                               int variant, int16_t* codes, cudaStream_t s);
// encode_wide.cu
struct WidePlan {
    bool ok = false;   // false: B is outside (0, kWideMaxFrames] or needs more CTAs than SMs
    int groups = 0;    // frame groups of at most 64
    int S = 0;         // CTAs per group (codebook slices)
    int per_k = 0;     // codewords per slice
    int grid = 0;      // groups * S (<= SM count: every CTA resident at once)
    int U = 0, V = 0;  // thread tile: 16U frames x 16V codewords
    int jc = 0;        // projection: latent columns staged per pass
    int fb = 1;        // projection: frame blocks per group (S / fb output blocks)
    int smem = 0;      // dynamic shared memory bytes
};
WidePlan plan_encode_wide(int B, int num_sms);

size_t wide_partial_bytes(int num_sms);
cudaError_t encode_wide_configure();  // once per device, before the first launch
// Launches on one set of tables must be stream-ordered (they share the scratch).
// rescan_list: encode the frames of t.rescan_list (count on the device), B at a
// time with plan p, instead of frames 0..B-1.
cudaError_t launch_encode_wide(const Tables& t, const WidePlan& p, const void* z, int dtype, int B,
                               int n_q, int variant, int16_t* codes, cudaStream_t s,
                               bool rescan_list = false);
// encode_cluster.cu
struct ClusterPlan {
    bool ok = false;  // false: no cluster form, or more than kClusterMaxBlock frames per cluster
    int cs = 0;       // CTAs per cluster (8 or 16)
    int nc = 0;       // clusters (one frame block each)
    int fc = 0;       // frames per cluster (the last may have fewer)
    int tile = 0;     // thread tile (index of the built tiles)
    int U = 0, V = 0; //   U frames x V codewords per lane quad
};
// once per handle, after encode_wide_configure: sets t.cl_max8 and t.cl_max16 (0
// for a cluster size the device cannot run; not an error)
cudaError_t encode_cluster_configure(Tables& t);
ClusterPlan plan_encode_cluster(const Tables& t, int B);
// Frames 0..B-1 read only the tables: launches on several streams may overlap.
// rescan_list: encode the frames of t.rescan_list (count on the device) instead, nc x fc
// per pass of the launch (plan for B = kClusterMaxBlock x clusters; B itself unused).
cudaError_t launch_encode_cluster(const Tables& t, const ClusterPlan& p, const void* z, int dtype,
                                  int B, int n_q, int variant, int16_t* codes, cudaStream_t s,
                                  bool rescan_list = false);
// selftest.cu: a kernel whose wait can never complete (which 0: an mbarrier,
// as the tensor-core encoder waits; 1: a group barrier, as the wide encoder
// waits); it times out after ~50 ms and records MIMI_DEV_ERR_TIMEOUT.
cudaError_t launch_wait_selftest(const Tables& t, int which, cudaStream_t s);
// decode.cu
cudaError_t launch_decode(const Tables& t, const int16_t* codes, int64_t n, int n_q, float* out,
                          cudaStream_t s);

}  // namespace mimi
