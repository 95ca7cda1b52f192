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
// It runs the float32 full-scan encode of scan_body.cuh (the same arithmetic in
// the same order as mimi_rvq_encode_scan, so the same codes), reading W_in
// row-major from the caller and the norms from the static array.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "../../include/mimi_rvq.h"
#include "handle.cuh"
#include "scan_body.cuh"

namespace mimi {

// Squared norms of at most kQ codebooks of kK codewords (64 KiB), rewritten in
// full by every call, so nothing in it has to start at zero. Every call shares
// it: calls that overlap on the GPU race.
static __device__ __align__(256) float g_noalloc_norms[kQ * kK];

namespace {

constexpr int kMaxDevices = 64;

// The array's device address is a property of the module loaded into one CUDA
// context: after a device reset (or any new primary context) the module is
// loaded again and the array may live elsewhere. The address is therefore
// cached per device together with the id of the context it was looked up in,
// and looked up again whenever the current context's id differs.
struct Slot {
    unsigned long long ctx_id = 0;
    float* norms = nullptr;
    int sms = 0;
};
Slot g_slots[kMaxDevices];
std::mutex g_setup_mutex;

bool current_context_id(unsigned long long* id) {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the static array in the current context of device `dev`
// (and the device's SM count). The first call in a context looks the address
// up; later calls in that context only compare the context id.
bool setup(int dev, float** norms, int* sms) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    Slot& s = g_slots[dev];
    if (!have_id || s.norms == nullptr || s.ctx_id != id) {
        // the lookup loads the module into the device's primary context (and makes that
        // context current) if nothing has yet
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_norms) != cudaSuccess || !current_context_id(&id)) {
            cudaGetLastError();
            s = Slot{};
            return false;
        }
        int n_sm = 0;
        if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            n_sm <= 0) {
            cudaGetLastError();
            s = Slot{};
            return false;
        }
        s.norms = static_cast<float*>(p);
        s.sms = n_sm;
        s.ctx_id = id;
    }
    *norms = s.norms;
    *sms = s.sms;
    return true;
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

// W_in read row-major [D][Din], as the caller holds it.
struct WinRowMajor {
    const float* W;
    __device__ __forceinline__ float operator()(int i, int j) const {
        return W[(size_t)i * kDin + j];
    }
};

__global__ void __launch_bounds__(scan::kThreads) k_noalloc_scan(const float* __restrict__ C,
                                                                 const float* __restrict__ W_in,
                                                                 const float* __restrict__ norms,
                                                                 const void* __restrict__ z,
                                                                 int dtype, int64_t n, int n_q,
                                                                 int16_t* __restrict__ codes) {
    __shared__ scan::Smem sm;
    for (int64_t frame = blockIdx.x; frame < n; frame += gridDim.x)
        scan::encode_frame(WinRowMajor{W_in}, C, norms, z, dtype, frame, n_q, 0, codes, sm);
}

// Device (or managed) memory whose address is a multiple of `align` bytes.
bool is_device_buffer(const void* p, uintptr_t align) {
    if (!p || (reinterpret_cast<uintptr_t>(p) & (align - 1))) return false;
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
    // codewords are read as float4; W_in and latents element by element; codes are int16
    if (!is_device_buffer(codebooks, 16) || !is_device_buffer(W_in, 4) ||
        !is_device_buffer(latents, dtype == MIMI_RVQ_F32 ? 4 : 2) || !is_device_buffer(codes, 2))
        return MIMI_RVQ_EINVAL;
    int dev = -1, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return MIMI_RVQ_ECUDA;
    if (major != 10) return MIMI_RVQ_EDEVICE;
    float* norms = nullptr;
    int sms = 0;
    if (!setup(dev, &norms, &sms)) return MIMI_RVQ_ECUDA;
    k_noalloc_norms<<<(n_q * kK * 32 + 255) / 256, 256, 0, stream>>>(codebooks, n_q, norms);
    const int64_t cap = (int64_t)sms * 8;  // 8 resident blocks of 256 threads per SM
    const int grid = (int)(N < cap ? N : cap);
    k_noalloc_scan<<<grid, scan::kThreads, 0, stream>>>(codebooks, W_in, norms, latents, dtype, N,
                                                        n_q, codes);
    return cudaGetLastError() == cudaSuccess ? MIMI_RVQ_OK : MIMI_RVQ_ECUDA;
}
