// api.cu -- the extern "C" boundary declared in include/mimi_rvq.h.
//
// Host side only: argument checks, the handle's device tables, TMA descriptor
// encoding, and launches. Every step of the computation runs in the kernels of
// prep.cu, encode_tc.cu, encode_wide.cu, encode_scan.cu and decode.cu.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <new>

#include "../../include/mimi_rvq.h"
#include "handle.cuh"
#include "ptx.cuh"

struct mimi_rvq {
    int device = 0;
    int num_sms = 148;
    mimi::Tables t;
    int cl_max8 = 0, cl_max16 = 0;  // the device's cluster counts (t's are 0 while the form is off)
};

namespace {

using mimi::kD;
using mimi::kDin;
using mimi::kK;
using mimi::kQ;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A pointer the device can dereference: device or managed memory.
bool device_pointer(const void* p) {
    if (!p || !aligned16(p)) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MIMI_RVQ_OK;
    if (e == cudaErrorMemoryAllocation) return MIMI_RVQ_ENOMEM;
    return MIMI_RVQ_ECUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 tensor [rows][cols] (row-major), boxes of 64 columns x 256 rows
// (32 KiB: one stage of the tensor-core encoder's ring), 128-byte swizzle: the
// layout the UMMA shared-memory descriptors expect.
// fp32 tensor [rows][256] (row-major) seen as slabs: dimension 0 the 32 columns of
// a slab, 1 the rows (1024-byte stride), 2 the 8 slabs of a row (128-byte stride);
// boxes of 32 columns x box_rows rows x box_slabs slabs (64 KiB), 128-byte swizzle:
// the cluster encoder's stages, each slab's rows contiguous in shared memory.
bool make_tmap_slabs(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {32, rows, 8};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 4, 128};
    const cuuint32_t box[3] = {32, box_rows, 65536 / (box_rows * 128)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, 256};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void free_tables(mimi::Tables& t) {
    void* ptrs[] = {t.C32, t.Win32, t.WinT32, t.Cbf, t.Win_hi, t.Win_lo, t.cnorm, t.cnorm3, t.cbound,
                    t.P, t.err, t.rescan_count, t.rescan_list, t.stats, t.wide_y,
                    t.wide_bars, t.wide_partial, t.slice_lists, t.slice_exact};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    const int sms = t.num_sms;
    t = mimi::Tables{};
    t.num_sms = sms;
}

template <class T>
cudaError_t dalloc(T** p, size_t count) {
    return cudaMalloc(reinterpret_cast<void**>(p), sizeof(T) * count);
}

// Re-encode the frames the batch tensor-core kernel queued (count on the device)
// with the float32 wide encoder, 1024 at a time (16 groups of 64 share the GPU).
cudaError_t rescan(mimi_rvq_t h, const void* z, int dtype, int n_q, int variant, int16_t* codes,
                   cudaStream_t s) {
    // the cluster form, 32 frames per cluster per pass, where the device runs it
    const int per_pass = mimi::kClusterMaxBlock * h->t.cl_max8;
    if (per_pass > 0) {
        const mimi::ClusterPlan cp = mimi::plan_encode_cluster(h->t, per_pass);
        if (cp.ok && cp.cs == 8 && cp.U == 16 && cp.V == 8)  // the list mode's tile
            return mimi::launch_encode_cluster(h->t, cp, z, dtype, per_pass, n_q, variant, codes, s,
                                               true);
    }
    const int batch = mimi::kWideMaxFrames;
    const mimi::WidePlan p = mimi::plan_encode_wide(batch, h->num_sms);
    if (!p.ok) return cudaErrorInvalidConfiguration;
    return mimi::launch_encode_wide(h->t, p, z, dtype, batch, n_q, variant, codes, s, true);
}

int check_common(mimi_rvq_t h, const void* in, const void* out, int64_t n) {
    if (!h || n < 0) return MIMI_RVQ_EINVAL;
    if (n == 0) return MIMI_RVQ_OK;
    if (!device_pointer(in) || !device_pointer(out)) return MIMI_RVQ_EINVAL;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MIMI_RVQ_EINVAL;
    return 1;  // proceed
}

}  // namespace

extern "C" {

const char* mimi_rvq_strerror(int status) {
    switch (status) {
        case MIMI_RVQ_OK: return "ok";
        case MIMI_RVQ_EINVAL: return "invalid argument";
        case MIMI_RVQ_ENOMEM: return "out of device memory";
        case MIMI_RVQ_ECUDA: return "CUDA error";
        case MIMI_RVQ_ERANGE: return "code outside [0, 2048) in decode input";
        case MIMI_RVQ_EDEVICE: return "device is not sm_100 (B200)";
        case MIMI_RVQ_ETIMEOUT: return "a kernel wait ran out its bound";
        default: return "unknown status";
    }
}

int mimi_rvq_create(const float* codebooks, const float* W_in, const float* W_out,
                    mimi_rvq_t* out) {
    if (!out) return MIMI_RVQ_EINVAL;
    *out = nullptr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MIMI_RVQ_ECUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MIMI_RVQ_ECUDA;
    if (prop.major != 10) return MIMI_RVQ_EDEVICE;
    if (!device_pointer(codebooks) || !device_pointer(W_in) || !device_pointer(W_out))
        return MIMI_RVQ_EINVAL;

    mimi_rvq* h = new (std::nothrow) mimi_rvq;
    if (!h) return MIMI_RVQ_ENOMEM;
    h->device = dev;
    h->num_sms = prop.multiProcessorCount;
    mimi::Tables& t = h->t;
    t.num_sms = h->num_sms;
    const size_t nC = (size_t)kQ * kK * kD;
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = dalloc(&t.C32, nC);
    if (e == cudaSuccess) e = dalloc(&t.Win32, (size_t)kD * kDin);
    if (e == cudaSuccess) e = dalloc(&t.WinT32, (size_t)kD * kDin);
    if (e == cudaSuccess) e = dalloc(&t.Cbf, nC);
    if (e == cudaSuccess) e = dalloc(&t.Win_hi, (size_t)kD * kDin);
    if (e == cudaSuccess) e = dalloc(&t.Win_lo, (size_t)kD * kDin);
    if (e == cudaSuccess) e = dalloc(&t.cnorm, (size_t)kQ * kK);
    if (e == cudaSuccess) e = dalloc(&t.cnorm3, (size_t)kQ * kK * 4);
    if (e == cudaSuccess) e = dalloc(&t.cbound, (size_t)4 * kQ);
    if (e == cudaSuccess) e = dalloc(&t.P, (size_t)kQ * kK * kDin);
    if (e == cudaSuccess) e = dalloc(&t.err, 1);
    if (e == cudaSuccess) e = dalloc(&t.rescan_count, 1);
    if (e == cudaSuccess) e = dalloc(&t.rescan_list, (size_t)mimi::kRescanCapacity);
    if (e == cudaSuccess) e = dalloc(&t.stats, 2);
    if (e == cudaSuccess) e = dalloc(&t.wide_y, (size_t)mimi::kWideMaxFrames * kD);
    if (e == cudaSuccess)
        e = dalloc(&t.wide_bars, (size_t)mimi::kWideMaxGroups * mimi::kWideBarStride);
    if (e == cudaSuccess)
        e = cudaMalloc(reinterpret_cast<void**>(&t.wide_partial),
                       mimi::wide_partial_bytes(h->num_sms));
    if (e == cudaSuccess)
        e = dalloc(&t.slice_lists, (size_t)2 * mimi::kSliceMaxGroups * mimi::kSlices * 128 *
                                       mimi::kSliceListFloats);
    if (e == cudaSuccess)
        e = dalloc(&t.slice_exact, (size_t)mimi::kSliceMaxGroups * 128 * mimi::kSlices);
    cudaStream_t s = nullptr;
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(t.C32, codebooks, sizeof(float) * nC, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(t.Win32, W_in, sizeof(float) * kD * kDin, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t.err, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t.rescan_count, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t.stats, 0, 2 * sizeof(unsigned long long), s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(t.wide_bars, 0,
                            sizeof(unsigned) * mimi::kWideMaxGroups * mimi::kWideBarStride, s);
    if (e == cudaSuccess) e = mimi::prep_tables(t, W_out, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (s) cudaStreamDestroy(s);
    if (e == cudaSuccess) e = mimi::encode_tc_configure();
    if (e == cudaSuccess) e = mimi::encode_wide_configure();
    if (e == cudaSuccess) e = mimi::encode_cluster_configure(t);
    if (e != cudaSuccess) {
        free_tables(t);
        delete h;
        cudaGetLastError();
        return from_cuda(e);
    }
    if (!make_tmap(&t.tm_C, t.Cbf, (uint64_t)kQ * kK, kD) ||
        !make_tmap(&t.tm_Whi, t.Win_hi, kD, kDin) || !make_tmap(&t.tm_Wlo, t.Win_lo, kD, kDin)) {
        free_tables(t);
        delete h;
        return MIMI_RVQ_ECUDA;
    }
    // the cluster form needs its slab maps; a size without one stays off
    if (!make_tmap_slabs(&t.tm_C32_8, t.C32, (uint64_t)kQ * kK, kK / 8)) t.cl_max8 = 0;
    if (!make_tmap_slabs(&t.tm_C32_16, t.C32, (uint64_t)kQ * kK, kK / 16)) t.cl_max16 = 0;
    h->cl_max8 = t.cl_max8;
    h->cl_max16 = t.cl_max16;
    *out = h;
    return MIMI_RVQ_OK;
}

void mimi_rvq_destroy(mimi_rvq_t h) {
    if (!h) return;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != h->device) cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    free_tables(h->t);
    if (prev >= 0 && prev != h->device) cudaSetDevice(prev);
    delete h;
}

int mimi_rvq_encode_ex(mimi_rvq_t h, const void* latents, int dtype, int64_t N, int n_q,
                       int variant, int16_t* codes, struct CUstream_st* stream) {
    if (dtype != MIMI_RVQ_F32 && dtype != MIMI_RVQ_BF16) return MIMI_RVQ_EINVAL;
    if (n_q < 1 || n_q > kQ || (variant != 0 && variant != 1)) return MIMI_RVQ_EINVAL;
    const int c = check_common(h, latents, codes, N);
    if (c <= 0) return c;
    const size_t elt = dtype == MIMI_RVQ_F32 ? 4 : 2;
    for (int64_t f0 = 0; f0 < N; f0 += mimi::kRescanCapacity) {
        const int64_t n = N - f0 < mimi::kRescanCapacity ? N - f0 : mimi::kRescanCapacity;
        const void* z = static_cast<const uint8_t*>(latents) + (size_t)f0 * kDin * elt;
        int16_t* out = codes + f0 * n_q;
        cudaError_t e = cudaMemsetAsync(h->t.rescan_count, 0, sizeof(int), stream);
        if (e == cudaSuccess)
            e = mimi::launch_encode_tc(h->t, z, dtype, n, n_q, variant, out, nullptr, stream,
                                       h->num_sms);
        if (e == cudaSuccess) e = rescan(h, z, dtype, n_q, variant, out, stream);
        if (e != cudaSuccess) return from_cuda(e);
    }
    return MIMI_RVQ_OK;
}

int mimi_rvq_encode(mimi_rvq_t h, const void* latents, int dtype, int64_t N, int16_t* codes,
                    struct CUstream_st* stream) {
    return mimi_rvq_encode_ex(h, latents, dtype, N, kQ, 0, codes, stream);
}

int mimi_rvq_encode_step_ex(mimi_rvq_t h, const void* frames, int dtype, int B, int n_q,
                            int variant, int16_t* codes, struct CUstream_st* stream) {
    if (!h || B < 0) return MIMI_RVQ_EINVAL;
    if (dtype != MIMI_RVQ_F32 && dtype != MIMI_RVQ_BF16) return MIMI_RVQ_EINVAL;
    if (n_q < 1 || n_q > kQ || (variant != 0 && variant != 1)) return MIMI_RVQ_EINVAL;
    const mimi::ClusterPlan cp = mimi::plan_encode_cluster(h->t, B);
    if (cp.ok) {
        // float32 latency encode on thread-block clusters
        const int c = check_common(h, frames, codes, B);
        if (c <= 0) return c;
        return from_cuda(
            mimi::launch_encode_cluster(h->t, cp, frames, dtype, B, n_q, variant, codes, stream));
    }
    if (B >= mimi::kSlicedMinFrames && mimi::sliced_fits(B, h->num_sms)) {
        // codebook-sliced tensor-core encode (rows it cannot certify take an exact
        // float32 scan inside the kernel: one launch)
        const int c = check_common(h, frames, codes, B);
        if (c <= 0) return c;
        return from_cuda(
            mimi::launch_encode_tc_sliced(h->t, frames, dtype, B, n_q, variant, codes, stream));
    }
    const mimi::WidePlan p = mimi::plan_encode_wide(B, h->num_sms);
    if (!p.ok) return mimi_rvq_encode_ex(h, frames, dtype, (int64_t)B, n_q, variant, codes, stream);
    const int c = check_common(h, frames, codes, B);
    if (c <= 0) return c;
    return from_cuda(
        mimi::launch_encode_wide(h->t, p, frames, dtype, B, n_q, variant, codes, stream));
}

int mimi_rvq_encode_step(mimi_rvq_t h, const void* frames, int dtype, int B, int16_t* codes,
                         struct CUstream_st* stream) {
    return mimi_rvq_encode_step_ex(h, frames, dtype, B, kQ, 0, codes, stream);
}

int mimi_rvq_encode_profile(mimi_rvq_t h, const void* latents, int dtype, int64_t N,
                            int16_t* codes, uint64_t* cycles, struct CUstream_st* stream) {
    if (dtype != MIMI_RVQ_F32 && dtype != MIMI_RVQ_BF16) return MIMI_RVQ_EINVAL;
    if (N > mimi::kRescanCapacity) return MIMI_RVQ_EINVAL;
    const int c = check_common(h, latents, codes, N);
    if (c <= 0) return c;
    if (!device_pointer(cycles)) return MIMI_RVQ_EINVAL;
    cudaError_t e = cudaMemsetAsync(h->t.rescan_count, 0, sizeof(int), stream);
    if (e == cudaSuccess)
        e = mimi::launch_encode_tc(h->t, latents, dtype, N, kQ, 0, codes, nullptr, stream,
                                   h->num_sms, reinterpret_cast<unsigned long long*>(cycles));
    if (e == cudaSuccess) e = rescan(h, latents, dtype, kQ, 0, codes, stream);
    return from_cuda(e);
}

int mimi_rvq_project(mimi_rvq_t h, const void* latents, int dtype, int64_t N, float* y,
                     struct CUstream_st* stream) {
    if (dtype != MIMI_RVQ_F32 && dtype != MIMI_RVQ_BF16) return MIMI_RVQ_EINVAL;
    const int c = check_common(h, latents, y, N);
    if (c <= 0) return c;
    return from_cuda(mimi::launch_encode_tc(h->t, latents, dtype, N, 0, 0, nullptr, y, stream,
                                            h->num_sms));
}

int mimi_rvq_encode_scan(mimi_rvq_t h, const void* latents, int dtype, int64_t N, int n_q,
                         int variant, int16_t* codes, struct CUstream_st* stream) {
    if (dtype != MIMI_RVQ_F32 && dtype != MIMI_RVQ_BF16) return MIMI_RVQ_EINVAL;
    if (n_q < 1 || n_q > kQ || (variant != 0 && variant != 1)) return MIMI_RVQ_EINVAL;
    const int c = check_common(h, latents, codes, N);
    if (c <= 0) return c;
    return from_cuda(mimi::launch_encode_scan(h->t, latents, dtype, N, n_q, variant, codes, stream));
}

int mimi_rvq_decode_ex(mimi_rvq_t h, const int16_t* codes, int64_t N, int n_q, float* latents,
                       struct CUstream_st* stream) {
    if (n_q < 1 || n_q > kQ) return MIMI_RVQ_EINVAL;
    const int c = check_common(h, codes, latents, N);
    if (c <= 0) return c;
    return from_cuda(mimi::launch_decode(h->t, codes, N, n_q, latents, stream));
}

int mimi_rvq_decode(mimi_rvq_t h, const int16_t* codes, int64_t N, float* latents,
                    struct CUstream_st* stream) {
    return mimi_rvq_decode_ex(h, codes, N, kQ, latents, stream);
}

int mimi_rvq_wait_selftest(mimi_rvq_t h, int which, struct CUstream_st* stream) {
    if (!h || (which != 0 && which != 1)) return MIMI_RVQ_EINVAL;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MIMI_RVQ_EINVAL;
    return from_cuda(mimi::launch_wait_selftest(h->t, which, stream));
}

int mimi_rvq_set_cluster_form(mimi_rvq_t h, int enabled) {
    if (!h || (enabled != 0 && enabled != 1)) return MIMI_RVQ_EINVAL;
    h->t.cl_max8 = enabled ? h->cl_max8 : 0;
    h->t.cl_max16 = enabled ? h->cl_max16 : 0;
    return MIMI_RVQ_OK;
}

int mimi_rvq_get_error(mimi_rvq_t h, struct CUstream_st* stream) {
    if (!h) return MIMI_RVQ_EINVAL;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MIMI_RVQ_ECUDA;
    int bits = 0;
    if (cudaMemcpy(&bits, h->t.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MIMI_RVQ_ECUDA;
    if (bits && cudaMemset(h->t.err, 0, sizeof(int)) != cudaSuccess) return MIMI_RVQ_ECUDA;
    // a wait that ran out may have left a group barrier mid-count
    if ((bits & mimi::MIMI_DEV_ERR_TIMEOUT) &&
        cudaMemset(h->t.wide_bars, 0,
                   sizeof(unsigned) * mimi::kWideMaxGroups * mimi::kWideBarStride) != cudaSuccess)
        return MIMI_RVQ_ECUDA;
    if (bits & mimi::MIMI_DEV_ERR_TIMEOUT) return MIMI_RVQ_ETIMEOUT;
    if (bits & mimi::MIMI_DEV_ERR_RANGE) return MIMI_RVQ_ERANGE;
    return MIMI_RVQ_OK;
}

int mimi_rvq_stats(mimi_rvq_t h, struct CUstream_st* stream, int64_t* frames_encoded,
                   int64_t* frames_rescanned) {
    if (!h) return MIMI_RVQ_EINVAL;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MIMI_RVQ_ECUDA;
    unsigned long long v[2] = {0, 0};
    if (cudaMemcpy(v, h->t.stats, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MIMI_RVQ_ECUDA;
    if (frames_encoded) *frames_encoded = (int64_t)v[0];
    if (frames_rescanned) *frames_rescanned = (int64_t)v[1];
    return MIMI_RVQ_OK;
}

}  // extern "C"
