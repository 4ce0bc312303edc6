// noalloc.cu -- nvfp4_gemm_noalloc: the block-scaled GEMM for callers that cannot allocate
// device memory, with its split-K scratch in a fixed array that lives in the library.
//
// nvfp4_gemm needs a caller-provided workspace for split-K (the per-tile arrival counters
// and fp32 partial tiles). Some callers cannot provide one: code that runs inside a host
// framework which has already reserved all device memory for its own pool (a cudaMalloc
// there fails, or would fragment memory the framework manages), plugin-style interfaces
// whose call signature offers no workspace argument, and latency-critical paths where
// cudaMalloc / cudaFree are not acceptable because they can synchronise the device. This
// entry point gives them the same kernel with the scratch taken from a file-scope
// __device__ array of kNoallocScratchBytes; it calls no allocating routine.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/nvfp4.h"
#include "internal.h"

namespace {

// The scratch array. Every GPU that loads this library holds these bytes until the process
// exits. All calls on a device share it and it keeps the last call's contents.
constexpr size_t kNoallocScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_nvfp4_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device address of the array per device, and the CUDA context it was looked up in. The
// module (and with it the array) is loaded once per context: after the primary context is
// released and created again it may sit at another address, so a change of context repeats
// the look-up.
void* g_scratch_ptr[kMaxDevices];
void* g_scratch_ctx[kMaxDevices];

using CtxGetCurrentFn = int (*)(void**);   // cuCtxGetCurrent(CUcontext*) -> CUresult

CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// In host code `g_nvfp4_noalloc_scratch` names a host-side stand-in, not device memory;
// the device address must come from cudaGetSymbolAddress, taken with the device current.
// Set-up: the first call on a device (and the first after its context changed) looks it up.
// A host thread that has made no CUDA call yet has no context bound; the look-up binds the
// device's primary context to it, and the context is read again afterwards.
nvfp4_status scratch_address(int dev, void** out)
{
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return NVFP4_ERR_CUDA;
    void* ctx = nullptr;
    if (get(&ctx) != 0) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_mu);
    if (ctx == nullptr || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_nvfp4_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        if (get(&ctx) != 0 || ctx == nullptr) return NVFP4_ERR_CUDA;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return NVFP4_OK;
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm_noalloc(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                const uint8_t* sfB, const float* alpha, void* out,
                                int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NVFP4_OK;
    constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
    if (M > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // the same pointer, shape and alignment checks as nvfp4_gemm
    const int chk = nvfp4::check_gemm_args(A, sfA, B, sfB, alpha, out, N, K);
    if (chk != NVFP4_OK) return static_cast<nvfp4_status>(chk);

    int num_sms = 0;
    unsigned* err_word = nullptr;
    const int st = nvfp4::query_current_device(&num_sms, &err_word);
    if (st != NVFP4_OK) return static_cast<nvfp4_status>(st);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    void* scratch = nullptr;
    nvfp4_status s = scratch_address(dev, &scratch);
    if (s != NVFP4_OK) return s;

    // Same tiling as nvfp4_gemm with a workspace available; a plan whose split-K scratch
    // would not fit in the fixed array is rejected, not silently changed.
    nvfp4::GemmPlan plan = nvfp4::plan_gemm(M, N, K, true, num_sms);
    if (plan.ws_bytes > 0) {
        if (plan.ws_bytes > kNoallocScratchBytes) return NVFP4_ERR_WORKSPACE;
        // The tile counters must start at zero; a previous call may have been cut short.
        if (cudaMemsetAsync(scratch, 0, plan.ws_counter_bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
    }
    nvfp4::GemmLaunch L{A, sfA, B, sfB, alpha, out, M, N, K, nullptr, 0, 0,
                        plan.ws_bytes > 0 ? scratch : nullptr, err_word};
    bool enc_failed = false;
    cudaError_t e = nvfp4::launch_gemm(plan, L, stream, &enc_failed);
    if (enc_failed) return NVFP4_ERR_CUDA;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

}  // extern "C"
