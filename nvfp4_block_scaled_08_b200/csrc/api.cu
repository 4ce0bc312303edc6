// api.cu -- the extern "C" boundary of libnvfp4 (declared in include/nvfp4.h): argument
// checks, device checks, the device error word, and dispatch to the kernels.
//
// Interface lessons carried over from the reference pages: alpha and out are explicit,
// required arguments ("The Moment the Zeros Disappeared", section "What This Means": a
// call without them failed with a TypeError); block_size is fixed at 16 ("The Art of
// Reading the Manual", section "Assumptions and Their Consequences"); B is N x K/2
// ("The Moment the Zeros Disappeared", section "The Subject Message", item 3); bad shapes
// are rejected with a clear status (the same page's "K dimension mismatch"); and there is
// no automatic fallback to another backend ("The Moment the Zeros Disappeared", section
// "What This Means": the auto backend's fallback chain failed).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/nvfp4.h"
#include "internal.h"
#include "ptx.cuh"

namespace {

__device__ unsigned g_nvfp4_error_word;

// Code the bounded-wait check records in the device error word.
constexpr unsigned kErrWaitCheck = 0x1FF;

// One CTA waits, with the kernels' bounded-wait routine and the given limit, on an mbarrier
// that nothing ever arrives at: the wait gives up, raises the CTA's abort flag, records
// kErrWaitCheck in the device error word, and the kernel returns normally.
__global__ void bounded_wait_check_kernel(unsigned* err_word, uint64_t timeout_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        nvfp4::mbar_init(&bar, 1);
        abort_flag = 0;
        nvfp4::fence_mbarrier_init();
    }
    __syncthreads();
    const nvfp4::AbortState ab{&abort_flag, err_word};
    if (threadIdx.x == 0) nvfp4::mbar_wait(&bar, 0, ab, kErrWaitCheck, timeout_ns);
    __syncthreads();
}

struct DeviceInfo {
    bool init = false;
    bool arch_ok = false;
    int num_sms = 0;
    unsigned* err_word = nullptr;
};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

nvfp4_status current_device(DeviceInfo* out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.init) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        d.arch_ok = (major == 10 && minor == 0);
        d.num_sms = sms;
        void* p = nullptr;
        if (d.arch_ok) {
            if (cudaGetSymbolAddress(&p, g_nvfp4_error_word) != cudaSuccess) {
                cudaGetLastError();
                return NVFP4_ERR_CUDA;
            }
        }
        d.err_word = static_cast<unsigned*>(p);
        d.init = true;
    }
    *out = d;
    return d.arch_ok ? NVFP4_OK : NVFP4_ERR_ARCH;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

nvfp4_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return NVFP4_OK;
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
}

nvfp4_status check_gemm_common(const void* A, const void* sfA, const void* B, const void* sfB,
                               const void* alpha, const void* out, int64_t N, int64_t K)
{
    return static_cast<nvfp4_status>(nvfp4::check_gemm_args(A, sfA, B, sfB, alpha, out, N, K));
}

}  // namespace

namespace nvfp4 {

// Shape and pointer checks shared by every GEMM entry point (also nvfp4_gemm_noalloc); no
// CUDA call.
int check_gemm_args(const void* A, const void* sfA, const void* B, const void* sfB,
                    const void* alpha, const void* out, int64_t N, int64_t K)
{
    if (!A || !sfA || !B || !sfB || !alpha || !out) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 256 != 0 || K > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (N % 8 != 0 || N > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(A) || !aligned16(sfA) || !aligned16(B) || !aligned16(sfB) || !aligned16(out))
        return NVFP4_ERR_MISALIGNED;
    if (!aligned4(alpha)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

}  // namespace nvfp4

namespace nvfp4 {

// Device checks for entry points defined in other translation units: arch, SM count and
// the device error word of the current device (same rules as every call in this file).
int query_current_device(int* num_sms, unsigned** err_word)
{
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st == NVFP4_OK) {
        *num_sms = d.num_sms;
        *err_word = d.err_word;
    }
    return static_cast<int>(st);
}

}  // namespace nvfp4

extern "C" {

const char* nvfp4_status_string(nvfp4_status s)
{
    switch (s) {
        case NVFP4_OK: return "NVFP4_OK";
        case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG: null pointer, negative size or bad enum value";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "NVFP4_ERR_UNSUPPORTED_SHAPE: need K % 256 == 0, N % 8 == 0, dims < 2^31";
        case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED: pointers and row strides must be 16-byte aligned";
        case NVFP4_ERR_ARCH: return "NVFP4_ERR_ARCH: device is not compute capability 10.0 (sm_100a)";
        case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA: a CUDA runtime or driver call failed";
        case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT: a kernel gave up on a bounded wait";
        case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE: workspace smaller than nvfp4_gemm_workspace_size()";
    }
    return "NVFP4_ERR_UNKNOWN";
}

nvfp4_status nvfp4_global_scale(const void* x, nvfp4_in_dtype dtype, int64_t numel, float* gs_out,
                                cudaStream_t stream)
{
    if (!gs_out || numel < 0 || (numel > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_F32 && dtype != NVFP4_IN_BF16) return NVFP4_ERR_INVALID_ARG;
    if ((numel > 0 && !aligned16(x)) || !aligned4(gs_out)) return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_global_scale(x, dtype == NVFP4_IN_BF16, numel, gs_out, stream,
                                                d.num_sms));
}

nvfp4_status nvfp4_quantize(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                            int64_t ld_x, const float* gs, uint8_t* q, uint8_t* sf,
                            cudaStream_t stream)
{
    if (rows < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_F32 && dtype != NVFP4_IN_BF16) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || K == 0) return NVFP4_OK;
    if (!x || !gs || !q || !sf) return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0 || K > kMaxDim || rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld_x < K) return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = dtype == NVFP4_IN_BF16 ? 2 : 4;
    if (!aligned16(x) || (ld_x * esz) % 16 != 0 || !aligned16(q) || !aligned4(gs))
        return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_quantize(x, dtype == NVFP4_IN_BF16, rows, K, ld_x, gs, q, sf,
                                            stream, d.num_sms));
}

nvfp4_status nvfp4_quantize_dynamic_ex(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                                       int64_t ld_x, float* gs_out, uint8_t* q, uint8_t* sf,
                                       const float* gs_other, int32_t n_alpha, float* alpha_out,
                                       nvfp4_sf_layout sf_layout, cudaStream_t stream)
{
    if (rows < 0 || K < 0 || n_alpha < 0) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_F32 && dtype != NVFP4_IN_BF16) return NVFP4_ERR_INVALID_ARG;
    if (sf_layout != NVFP4_SF_LINEAR && sf_layout != NVFP4_SF_TILED && sf_layout != NVFP4_SF_8X4)
        return NVFP4_ERR_INVALID_ARG;
    if (!gs_out) return NVFP4_ERR_INVALID_ARG;
    if (n_alpha > 0 && (!gs_other || !alpha_out)) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || K == 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;   // no tensor to take a scale of
    if (!x || !q || !sf) return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0 || K > kMaxDim || rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (sf_layout != NVFP4_SF_LINEAR && K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld_x < K) return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = dtype == NVFP4_IN_BF16 ? 2 : 4;
    if (rows * (K * esz / 16) >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || (ld_x * esz) % 16 != 0 || !aligned16(q) || !aligned4(gs_out) ||
        (n_alpha > 0 && (!aligned4(gs_other) || !aligned4(alpha_out))))
        return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_quantize_dynamic(x, dtype == NVFP4_IN_BF16, rows, K, ld_x, gs_out, q, sf,
                                                    static_cast<int>(sf_layout), gs_other, n_alpha,
                                                    alpha_out, d.err_word, stream, d.num_sms));
}

nvfp4_status nvfp4_quantize_dynamic(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                                    int64_t ld_x, float* gs_out, uint8_t* q, uint8_t* sf,
                                    const float* gs_other, int32_t n_alpha, float* alpha_out,
                                    cudaStream_t stream)
{
    return nvfp4_quantize_dynamic_ex(x, dtype, rows, K, ld_x, gs_out, q, sf, gs_other, n_alpha, alpha_out,
                                     NVFP4_SF_LINEAR, stream);
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t K, nvfp4_sf_layout sf_layout)
{
    if (rows < 0 || K <= 0 || K % 16 != 0) return 0;
    if (sf_layout == NVFP4_SF_LINEAR) return static_cast<size_t>(rows) * static_cast<size_t>(K / 16);
    if (sf_layout == NVFP4_SF_TILED && K % 64 == 0)
        return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(K / 16);
    if (sf_layout == NVFP4_SF_8X4 && K % 64 == 0)
        return static_cast<size_t>((rows + 7) / 8 * 8) * static_cast<size_t>(K / 16);
    return 0;
}

nvfp4_status nvfp4_sf_tile(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* sf_tiled, cudaStream_t stream)
{
    if (rows < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || K == 0) return NVFP4_OK;
    if (!sf || !sf_tiled) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0 || K > kMaxDim || rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_sf_tile(sf, rows, K, sf_tiled, stream, d.num_sms));
}

nvfp4_status nvfp4_sf_8x4(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* sf_8x4, cudaStream_t stream)
{
    if (rows < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || K == 0) return NVFP4_OK;
    if (!sf || !sf_8x4) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0 || K > kMaxDim || rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_sf_8x4(sf, rows, K, sf_8x4, stream, d.num_sms));
}

nvfp4_status nvfp4_alpha(const float* gs_a, const float* gs_b, int32_t n, float* alpha,
                         cudaStream_t stream)
{
    if (n < 0) return NVFP4_ERR_INVALID_ARG;
    if (n == 0) return NVFP4_OK;
    if (!gs_a || !gs_b || !alpha) return NVFP4_ERR_INVALID_ARG;
    if (!aligned4(gs_a) || !aligned4(gs_b) || !aligned4(alpha)) return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_alpha(gs_a, gs_b, n, alpha, stream));
}

size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0 || K % 256 != 0) return 0;
    DeviceInfo d;
    if (current_device(&d) != NVFP4_OK) return 0;
    return nvfp4::plan_gemm(M, N, K, true, d.num_sms).ws_bytes;
}

nvfp4_status nvfp4_gemm_ex3(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                            const float* alpha, void* out, int64_t M, int64_t N, int64_t K, void* ws,
                            size_t ws_bytes, nvfp4_sf_layout sf_layout, nvfp4_out_dtype out_dtype,
                            uint32_t flags, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~static_cast<uint32_t>(NVFP4_GEMM_B_READY)) != 0) return NVFP4_ERR_INVALID_ARG;
    if (sf_layout != NVFP4_SF_LINEAR && sf_layout != NVFP4_SF_TILED && sf_layout != NVFP4_SF_8X4)
        return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32)
        return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (M > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4_status st = check_gemm_common(A, sfA, B, sfB, alpha, out, N, K);
    if (st != NVFP4_OK) return st;
    if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    st = current_device(&d);
    if (st != NVFP4_OK) return st;
    nvfp4::GemmPlan plan = nvfp4::plan_gemm(M, N, K, ws != nullptr, d.num_sms);
    if (plan.ws_bytes > 0 && ws_bytes < plan.ws_bytes) return NVFP4_ERR_WORKSPACE;
    const bool tiled = sf_layout == NVFP4_SF_TILED;
    // tiled scales: Q tiles start on 128-row tile boundaries (tuning overrides can break it)
    if (tiled && (plan.swap ? plan.q_tiles != 1 : (plan.bn % 128 != 0)))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4::GemmLaunch L{A, sfA, B, sfB, alpha, out, M, N, K, nullptr, 0, 0, ws, d.err_word, tiled,
                        static_cast<int32_t>(out_dtype)};
    L.sf_8x4 = sf_layout == NVFP4_SF_8X4;
    L.b_ready = (flags & NVFP4_GEMM_B_READY) != 0;
    bool enc_failed = false;
    cudaError_t e = nvfp4::launch_gemm(plan, L, stream, &enc_failed);
    if (enc_failed) return NVFP4_ERR_CUDA;
    return from_cuda(e);
}

nvfp4_status nvfp4_gemm_ex2(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                            const float* alpha, void* out, int64_t M, int64_t N, int64_t K, void* ws,
                            size_t ws_bytes, nvfp4_sf_layout sf_layout, nvfp4_out_dtype out_dtype,
                            cudaStream_t stream)
{
    return nvfp4_gemm_ex3(A, sfA, B, sfB, alpha, out, M, N, K, ws, ws_bytes, sf_layout, out_dtype, 0u, stream);
}

nvfp4_status nvfp4_mx_quantize(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K, int64_t ld_x,
                               uint8_t* q, uint8_t* sf, nvfp4_sf_layout sf_layout, cudaStream_t stream)
{
    if (rows < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_F32 && dtype != NVFP4_IN_BF16) return NVFP4_ERR_INVALID_ARG;
    if (sf_layout != NVFP4_SF_LINEAR && sf_layout != NVFP4_SF_TILED) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || K == 0) return NVFP4_OK;
    if (!x || !q || !sf) return NVFP4_ERR_INVALID_ARG;
    if (K % 32 != 0 || K > kMaxDim || rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (sf_layout == NVFP4_SF_TILED && K % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld_x < K) return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = dtype == NVFP4_IN_BF16 ? 2 : 4;
    if (rows * (K / 8) >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || (ld_x * esz) % 16 != 0 || !aligned16(q)) return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_mx_quantize(x, dtype == NVFP4_IN_BF16, rows, K, ld_x, q, sf,
                                               sf_layout == NVFP4_SF_TILED, stream, d.num_sms));
}

size_t nvfp4_mx_sf_bytes(int64_t rows, int64_t K, nvfp4_sf_layout sf_layout)
{
    if (rows < 0 || K <= 0 || K % 32 != 0) return 0;
    if (sf_layout == NVFP4_SF_LINEAR) return static_cast<size_t>(rows) * static_cast<size_t>(K / 32);
    if (sf_layout == NVFP4_SF_TILED && K % 128 == 0)
        return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(K / 32);
    return 0;
}

nvfp4_status nvfp4_mx_sf_tile(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* sf_tiled, cudaStream_t stream)
{
    if (rows < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || K == 0) return NVFP4_OK;
    if (!sf || !sf_tiled) return NVFP4_ERR_INVALID_ARG;
    if (K % 128 != 0 || K > kMaxDim || rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_sf_tile(sf, rows, K, sf_tiled, stream, d.num_sms, 32));
}

nvfp4_status nvfp4_mx_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                           const float* alpha, void* out, int64_t M, int64_t N, int64_t K, void* ws,
                           size_t ws_bytes, nvfp4_out_dtype out_dtype, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32)
        return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (M > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4_status st = check_gemm_common(A, sfA, B, sfB, alpha, out, N, K);
    if (st != NVFP4_OK) return st;
    if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    st = current_device(&d);
    if (st != NVFP4_OK) return st;
    nvfp4::GemmPlan plan = nvfp4::plan_gemm(M, N, K, ws != nullptr, d.num_sms);
    if (plan.ws_bytes > 0 && ws_bytes < plan.ws_bytes) return NVFP4_ERR_WORKSPACE;
    // tiled scales: Q tiles start on 128-row tile boundaries (tuning overrides can break it)
    if (plan.swap ? plan.q_tiles != 1 : (plan.bn % 128 != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4::GemmLaunch L{A, sfA, B, sfB, alpha, out, M, N, K, nullptr, 0, 0, ws, d.err_word, true,
                        static_cast<int32_t>(out_dtype)};
    L.mx = true;
    bool enc_failed = false;
    cudaError_t e = nvfp4::launch_gemm(plan, L, stream, &enc_failed);
    if (enc_failed) return NVFP4_ERR_CUDA;
    return from_cuda(e);
}

nvfp4_status nvfp4_gemm_act(const void* x, nvfp4_in_dtype dtype, int64_t ld_x, const float* gs_b,
                            const uint8_t* B, const uint8_t* sfB, void* out, int64_t M, int64_t N, int64_t K,
                            float* gs_out, float* alpha_out, nvfp4_out_dtype out_dtype, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_F32 && dtype != NVFP4_IN_BF16) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32)
        return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!gs_b) return NVFP4_ERR_INVALID_ARG;
    // the shared checks with x in A's place (its scales come from the kernel: sfA is not read)
    nvfp4_status st = check_gemm_common(x, B, B, sfB, gs_b, out, N, K);
    if (st != NVFP4_OK) return st;
    if (M > 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld_x < K) return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = dtype == NVFP4_IN_BF16 ? 2 : 4;
    if ((ld_x * esz) % 16 != 0 || (gs_out && !aligned4(gs_out)) || (alpha_out && !aligned4(alpha_out)))
        return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    st = current_device(&d);
    if (st != NVFP4_OK) return st;
    nvfp4::GemmPlan plan = nvfp4::plan_gemm(M, N, K, false, d.num_sms);
    // every CTA's K slice must fit its stage ring; the cluster's slices together cover K
    const int nk = static_cast<int>(K / 256);
    const int stages = nvfp4::act_gemm_stages(plan.bn);
    if (!plan.swap || plan.q_tiles != 1 || plan.groups != 1 || stages == 0 ||
        (nk + plan.splits - 1) / plan.splits > stages)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4::GemmLaunch L{nullptr, nullptr, B, sfB, gs_b, out, M, N, K, nullptr, 0, 0, nullptr, d.err_word, true,
                        static_cast<int32_t>(out_dtype)};
    L.A = static_cast<const uint8_t*>(x);
    L.sfA = B;
    L.act = x;
    L.act_ld = ld_x;
    L.act_bf16 = dtype == NVFP4_IN_BF16;
    L.gs_b = gs_b;
    L.gs_out = gs_out;
    L.alpha_out = alpha_out;
    bool enc_failed = false;
    cudaError_t e = nvfp4::launch_gemm(plan, L, stream, &enc_failed);
    if (enc_failed) return NVFP4_ERR_CUDA;
    return from_cuda(e);
}

nvfp4_status nvfp4_gemm_ex(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                           const float* alpha, void* out, int64_t M, int64_t N, int64_t K, void* ws,
                           size_t ws_bytes, nvfp4_sf_layout sf_layout, cudaStream_t stream)
{
    return nvfp4_gemm_ex2(A, sfA, B, sfB, alpha, out, M, N, K, ws, ws_bytes, sf_layout, NVFP4_OUT_BF16,
                          stream);
}

nvfp4_status nvfp4_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                        const float* alpha, void* out, int64_t M, int64_t N, int64_t K, void* ws,
                        size_t ws_bytes, cudaStream_t stream)
{
    return nvfp4_gemm_ex2(A, sfA, B, sfB, alpha, out, M, N, K, ws, ws_bytes, NVFP4_SF_LINEAR, NVFP4_OUT_BF16,
                          stream);
}

size_t nvfp4_grouped_gemm_workspace_size(int32_t E, int64_t total_rows, int64_t N, int64_t K)
{
    (void)E; (void)total_rows; (void)N; (void)K;
    return 0;
}

nvfp4_status nvfp4_grouped_gemm_ex(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                   const uint8_t* sfB, const float* alpha,
                                   const int32_t* expert_offsets, int32_t E, int64_t total_rows,
                                   int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                                   cudaStream_t stream)
{
    if (E < 0 || total_rows < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32)
        return NVFP4_ERR_INVALID_ARG;
    if (E == 0 || total_rows == 0 || N == 0) return NVFP4_OK;
    if (E > nvfp4::kMaxExperts) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (total_rows > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!expert_offsets) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_gemm_common(A, sfA, B, sfB, alpha, out, N, K);
    if (st != NVFP4_OK) return st;
    if (!aligned4(expert_offsets)) return NVFP4_ERR_MISALIGNED;
    if (static_cast<int64_t>(E) * N > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo d;
    st = current_device(&d);
    if (st != NVFP4_OK) return st;
    nvfp4::GemmPlan plan = nvfp4::plan_grouped(E, total_rows, N, K, d.num_sms);
    nvfp4::GemmLaunch L{A, sfA, B, sfB, alpha, out, 0, N, K, expert_offsets, E, total_rows,
                        nullptr, d.err_word, false, static_cast<int32_t>(out_dtype)};
    bool enc_failed = false;
    cudaError_t e = nvfp4::launch_gemm(plan, L, stream, &enc_failed);
    if (enc_failed) return NVFP4_ERR_CUDA;
    return from_cuda(e);
}

nvfp4_status nvfp4_grouped_gemm_swiglu(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                       const uint8_t* sfB, const float* alpha,
                                       const int32_t* expert_offsets, int32_t E, int64_t total_rows,
                                       int64_t I, int64_t K, const float* gs_h, uint8_t* h_q,
                                       uint8_t* h_sf, cudaStream_t stream)
{
    if (E < 0 || total_rows < 0 || I < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    if (E == 0 || total_rows == 0 || I == 0) return NVFP4_OK;
    if (!expert_offsets || !gs_h || !h_sf) return NVFP4_ERR_INVALID_ARG;
    if (E > nvfp4::kMaxExperts || total_rows > kMaxDim || I % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    nvfp4_status st = check_gemm_common(A, sfA, B, sfB, alpha, h_q, 2 * I, K);
    if (st != NVFP4_OK) return st;
    if (!aligned4(expert_offsets) || !aligned4(gs_h)) return NVFP4_ERR_MISALIGNED;
    if (static_cast<int64_t>(E) * 2 * I > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo d;
    st = current_device(&d);
    if (st != NVFP4_OK) return st;
    nvfp4::GemmPlan plan = nvfp4::plan_grouped(E, total_rows, 2 * I, K, d.num_sms);
    nvfp4::GemmLaunch L{A, sfA, B, sfB, alpha, nullptr, 0, 2 * I, K, expert_offsets, E, total_rows,
                        nullptr, d.err_word, false, 0, h_q, h_sf, gs_h};
    bool enc_failed = false;
    cudaError_t e = nvfp4::launch_gemm(plan, L, stream, &enc_failed);
    if (enc_failed) return NVFP4_ERR_CUDA;
    return from_cuda(e);
}

nvfp4_status nvfp4_grouped_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                const uint8_t* sfB, const float* alpha,
                                const int32_t* expert_offsets, int32_t E, int64_t total_rows,
                                int64_t N, int64_t K, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t stream)
{
    (void)ws; (void)ws_bytes;
    return nvfp4_grouped_gemm_ex(A, sfA, B, sfB, alpha, expert_offsets, E, total_rows, N, K, out,
                                 NVFP4_OUT_BF16, stream);
}

nvfp4_status nvfp4_moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* experts,
                             float* weights, int32_t* expert_offsets, int32_t* row_of, int32_t* token_of_row,
                             cudaStream_t stream)
{
    if (T < 0 || E <= 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if (E > 1024 || k > 32 || k > E) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!expert_offsets) return NVFP4_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !experts || !weights || !row_of || !token_of_row)) return NVFP4_ERR_INVALID_ARG;
    if (static_cast<int64_t>(T) * k > kMaxDim || static_cast<int64_t>(T) * E > (int64_t(1) << 40))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned4(logits) || !aligned4(experts) || !aligned4(weights) || !aligned4(expert_offsets) ||
        !aligned4(row_of) || !aligned4(token_of_row))
        return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_moe_route(logits, T, E, k, experts, weights, expert_offsets, row_of,
                                             token_of_row, stream));
}

nvfp4_status nvfp4_moe_gather_quantize(const void* x, nvfp4_in_dtype dtype, int32_t T, int64_t H, int64_t ld_x,
                                       int32_t k, const int32_t* row_of, float* gs_out, uint8_t* q, uint8_t* sf,
                                       const float* gs_other, int32_t n_alpha, float* alpha_out,
                                       cudaStream_t stream)
{
    if (T < 0 || H < 0 || k <= 0 || n_alpha < 0) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_F32 && dtype != NVFP4_IN_BF16) return NVFP4_ERR_INVALID_ARG;
    if (!gs_out || (n_alpha > 0 && (!gs_other || !alpha_out))) return NVFP4_ERR_INVALID_ARG;
    if (T == 0 || H == 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;     // no tensor to take a scale of
    if (!x || !row_of || !q || !sf) return NVFP4_ERR_INVALID_ARG;
    if (H % 16 != 0 || H > kMaxDim || k > 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld_x < H) return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = dtype == NVFP4_IN_BF16 ? 2 : 4;
    if (static_cast<int64_t>(T) * (H * esz / 16) >= (int64_t(1) << 31) ||
        static_cast<int64_t>(T) * k * (H / 2) >= (int64_t(1) << 40))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || (ld_x * esz) % 16 != 0 || !aligned16(q) || !aligned4(gs_out) || !aligned4(row_of) ||
        (n_alpha > 0 && (!aligned4(gs_other) || !aligned4(alpha_out))))
        return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_gather_quantize(x, dtype == NVFP4_IN_BF16, T, H, ld_x, k, row_of, gs_out, q,
                                                   sf, gs_other, n_alpha, alpha_out, d.err_word, stream,
                                                   d.num_sms));
}

nvfp4_status nvfp4_moe_combine(const void* y, nvfp4_out_dtype y_dtype, const float* weights,
                               const int32_t* row_of, int32_t T, int64_t H, int32_t k, void* out,
                               nvfp4_out_dtype out_dtype, cudaStream_t stream)
{
    if (T < 0 || H < 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if ((y_dtype != NVFP4_OUT_BF16 && y_dtype != NVFP4_OUT_F16 && y_dtype != NVFP4_OUT_F32) ||
        (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32))
        return NVFP4_ERR_INVALID_ARG;
    if (T == 0 || H == 0) return NVFP4_OK;
    if (!y || !weights || !row_of || !out) return NVFP4_ERR_INVALID_ARG;
    if (H % 8 != 0 || H > kMaxDim || k > 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(y) || !aligned16(out) || !aligned4(weights) || !aligned4(row_of)) return NVFP4_ERR_MISALIGNED;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_moe_combine(y, static_cast<int32_t>(y_dtype), weights, row_of, T, H, k, out,
                                               static_cast<int32_t>(out_dtype), stream, d.num_sms));
}

nvfp4_status nvfp4_set_plan_override(int32_t bn, int32_t cluster, int32_t groups, int32_t band,
                                     int32_t grouped_bn, int32_t pair)
{
    if (bn < 0 || cluster < 0 || groups < 0 || band < 0 || grouped_bn < 0 || pair < 0 || pair > 3)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4::set_plan_override(bn, cluster, groups, band, grouped_bn, pair);
    return NVFP4_OK;
}

nvfp4_status nvfp4_round_e4m3(const float* x, int64_t n, uint8_t* out, cudaStream_t stream)
{
    if (n < 0) return NVFP4_ERR_INVALID_ARG;
    if (n == 0) return NVFP4_OK;
    if (!x || !out) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_round(x, n, out, false, stream, d.num_sms));
}

nvfp4_status nvfp4_round_e2m1(const float* x, int64_t n, uint8_t* out, cudaStream_t stream)
{
    if (n < 0) return NVFP4_ERR_INVALID_ARG;
    if (n == 0) return NVFP4_OK;
    if (!x || !out) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_round(x, n, out, true, stream, d.num_sms));
}

nvfp4_status nvfp4_check_bounded_wait(uint32_t timeout_us, cudaStream_t stream)
{
    if (timeout_us == 0 || timeout_us > 1000000u) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    bounded_wait_check_kernel<<<1, 32, 0, stream>>>(d.err_word, 1000ull * timeout_us);
    return from_cuda(cudaGetLastError());
}

nvfp4_status nvfp4_last_device_error(cudaStream_t stream, uint32_t* where_out)
{
    DeviceInfo d;
    nvfp4_status st = current_device(&d);
    if (st != NVFP4_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_nvfp4_error_word, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    if (where_out) *where_out = v;
    if (v == 0) return NVFP4_OK;
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_nvfp4_error_word, &zero, sizeof(zero)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_ERR_TIMEOUT;
}

}  // extern "C"
