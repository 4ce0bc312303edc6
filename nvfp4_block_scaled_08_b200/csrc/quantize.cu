// quantize.cu -- NVFP4 two-level quantisation kernels for sm_100a: per-tensor global scale
// (amax reduction), per-16-element block scale (e4m3) and element codes (e2m1), plus the
// GEMM alpha and the elementwise conversions exposed for exhaustive checking. The
// arithmetic itself lives in quant_core.cuh.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cooperative_groups.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "quant_core.cuh"

namespace nvfp4 {

// ------------------------------------------------------------------ global scale

template <typename T>
__global__ void __launch_bounds__(512) amax_kernel(const T* __restrict__ x, const VecIndex ix, uint32_t nv,
                                                   unsigned* __restrict__ acc_bits)
{
    __shared__ float red[32];
    float m = amax_sweep<T>(GlobalVecs<T>{x, ix}, blockIdx.x * blockDim.x + threadIdx.x, nv,
                            gridDim.x * blockDim.x);
    m = block_max(m, red);
    // non-negative floats order like their bit patterns
    if (threadIdx.x == 0) atomicMax(acc_bits, __float_as_uint(m));
}

template <typename T>
__global__ void amax_tail_kernel(const T* __restrict__ x, int n, unsigned* __restrict__ acc_bits)
{
    float m = 0.0f;
    if (static_cast<int>(threadIdx.x) < n) {
        if constexpr (sizeof(T) == 4) m = fabsf(x[threadIdx.x]);
        else m = fabsf(__bfloat162float(x[threadIdx.x]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) atomicMax(acc_bits, __float_as_uint(m));
}

// gs = 2688 / amax (448 * 6), or 1 if the tensor is all zero; in place over the amax bits.
__global__ void global_scale_finalize_kernel(float* gs)
{
    const float amax = __uint_as_float(*reinterpret_cast<unsigned*>(gs));
    *gs = (amax == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, amax);
}

__global__ void alpha_kernel(const float* __restrict__ gs_a, const float* __restrict__ gs_b,
                             int32_t n, float* __restrict__ alpha)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) alpha[i] = __fdiv_rn(1.0f, __fmul_rn(gs_a[0], gs_b[i]));
}

// ------------------------------------------------------------------ quantisation

template <typename T>
__global__ void __launch_bounds__(512) quantize_kernel(const T* __restrict__ x, const VecIndex ix, uint32_t nv,
                                                       const float* __restrict__ gs_ptr,
                                                       uint8_t* __restrict__ q, const SfOut sfo)
{
    __shared__ float rcp_tab[256];
    const float gs = __ldg(gs_ptr);
    build_rcp_table(gs, rcp_tab);
    quantize_sweep<T>(GlobalVecs<T>{x, ix}, blockIdx.x * blockDim.x + (threadIdx.x & ~31u), nv,
                      gridDim.x * blockDim.x, gs, rcp_tab, DenseDst{q, sfo});
}

// One cooperative launch: amax of the whole tensor -> grid barrier -> global scale (and the
// GEMM alpha against other tensors' global scales) -> quantisation.
// RESIDENT: block b reads its contiguous share [b * chunk, ...) of the vectors once, keeps it
// in shared memory during the barrier and quantises it from there; otherwise the blocks sweep
// the tensor grid-strided twice (the second time mostly from L2).
// The per-block maxima are parked in the first 4 * gridDim.x bytes of q, followed by one
// "read" flag per block (cleared before the barrier, set once the block has read every
// maximum). Only the blocks whose codes overwrite that area wait for all flags (every block,
// when the codes are scattered); the launcher keeps gridDim.x * 8 <= the bytes of q. The wait
// is bounded; on a timeout the kernel records kErrQuantFlags in err_word and goes on (the
// codes of that call are then undefined).
constexpr uint32_t kFlagRead = 0x52454144u;
constexpr uint32_t kErrQuantFlags = 0x201;

template <typename T, bool RESIDENT, int THREADS, class Dst>
__global__ void __launch_bounds__(THREADS) quantize_dynamic_kernel(
    const T* __restrict__ x, const VecIndex ix, uint32_t nv, uint32_t chunk,
    float* __restrict__ gs_out, uint8_t* __restrict__ q, const Dst dst,
    const float* __restrict__ gs_other, int32_t n_alpha, float* __restrict__ alpha_out,
    unsigned* __restrict__ err_word)
{
    namespace cg = cooperative_groups;
    constexpr int V = InTraits<T>::kPerThread;
    cg::grid_group grid = cg::this_grid();
    extern __shared__ uint4 stash_raw[];
    typename InTraits<T>::Raw* stash = reinterpret_cast<typename InTraits<T>::Raw*>(stash_raw);
    __shared__ float red[32];
    float* partial = reinterpret_cast<float*>(q);
    volatile uint32_t* read_flag = reinterpret_cast<volatile uint32_t*>(q) + gridDim.x;
    const uint32_t nblocks = gridDim.x;
    const uint32_t bid = blockIdx.x;
    grid_dependency_wait();      // launched early behind the previous kernel: wait for its data

    uint32_t v0 = 0, v1 = 0;
    float m;
    if constexpr (RESIDENT) {
        block_range(nv, chunk, bid, v0, v1);
        m = amax_sweep<T>(GlobalVecs<T>{x, ix}, v0 + threadIdx.x, v1, blockDim.x, stash, v0);
    } else {
        m = amax_sweep<T>(GlobalVecs<T>{x, ix}, bid * blockDim.x + threadIdx.x, nv, nblocks * blockDim.x);
    }
    m = block_max(m, red);
    if (threadIdx.x == 0) {
        partial[bid] = m;
        read_flag[bid] = 0u;
    }
    grid.sync();

    float a = 0.0f;
    for (uint32_t i = threadIdx.x; i < nblocks; i += blockDim.x) a = fmaxf(a, __ldcg(partial + i));
    a = block_max(a, red);       // ends with __syncthreads: every read of the maxima is done
    const float gs = (a == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, a);
    if (threadIdx.x == 0) {
        __threadfence();
        read_flag[bid] = kFlagRead;
    }
    if (bid == 0) {
        if (threadIdx.x == 0) *gs_out = gs;
        for (int32_t i = threadIdx.x; i < n_alpha; i += blockDim.x)
            alpha_out[i] = __fdiv_rn(1.0f, __fmul_rn(gs, gs_other[i]));
    }
    // a dependent GEMM may start its prologue now (it waits for this grid before reading)
    cudaTriggerProgrammaticLaunchCompletion();

    // this block's first code byte; the parked area is q[0, 8 * nblocks)
    const uint32_t first_vec = RESIDENT ? v0 : bid * blockDim.x;
    if (!Dst::kContiguous || static_cast<uint64_t>(first_vec) * (V / 2) < 8ull * nblocks) {
        // every thread watches its own flags (one L2 round trip, not one per block)
        const uint64_t t0 = globaltimer_ns();
        bool late = false;
        for (uint32_t b = threadIdx.x; b < nblocks && !late; b += blockDim.x) {
            while (read_flag[b] != kFlagRead) {
                if (globaltimer_ns() - t0 > kWaitTimeoutNs) { late = true; break; }
            }
        }
        if (late) atomicCAS(err_word, 0u, kErrQuantFlags);
        __threadfence();
        __syncthreads();
    }

    __shared__ float rcp_tab[256];
    build_rcp_table(gs, rcp_tab);
    if constexpr (RESIDENT) {
        quantize_sweep<T>(StashVecs<T>{stash, v0}, v0 + (threadIdx.x & ~31u), v1, blockDim.x, gs, rcp_tab, dst);
    } else {
        quantize_sweep<T>(GlobalVecs<T>{x, ix}, bid * blockDim.x + (threadIdx.x & ~31u), nv,
                          nblocks * blockDim.x, gs, rcp_tab, dst, true);
    }
}

// The same operation for small tensors in one thread-block cluster (no cooperative launch,
// no grid barrier): CTA r reads its contiguous share [r * chunk, ...) once into shared
// memory and reduces its maximum, the cluster exchanges the per-CTA maxima through
// distributed shared memory, and every CTA quantises its share from shared memory.
// gridDim = (1, cluster size, 1).
template <typename T, class Dst>
__global__ void __launch_bounds__(512) quantize_dynamic_cluster_kernel(
    const T* __restrict__ x, const VecIndex ix, uint32_t nv, uint32_t chunk,
    float* __restrict__ gs_out, const Dst dst,
    const float* __restrict__ gs_other, int32_t n_alpha, float* __restrict__ alpha_out)
{
    extern __shared__ uint4 stash_raw[];
    typename InTraits<T>::Raw* stash = reinterpret_cast<typename InTraits<T>::Raw*>(stash_raw);
    __shared__ float red[32];
    __shared__ float cta_max;
    grid_dependency_wait();      // launched early behind the previous kernel: wait for its data
    uint32_t v0, v1;
    block_range(nv, chunk, blockIdx.y, v0, v1);
    float m = amax_sweep<T>(GlobalVecs<T>{x, ix}, v0 + threadIdx.x, v1, blockDim.x, stash, v0);
    m = block_max(m, red);
    if (threadIdx.x == 0) cta_max = m;
    cluster_sync();                                   // every CTA's maximum is in place
    const uint32_t cs = gridDim.y;
    float a = 0.0f;
    if (threadIdx.x < 32) {
        if (threadIdx.x < cs)
            a = ld_shared_cluster_f32(mapa_shared(smem_u32(&cta_max), threadIdx.x));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (threadIdx.x == 0) red[0] = a;
    }
    cluster_arrive();                                 // done reading the peers' maxima
    __syncthreads();
    a = red[0];
    const float gs = (a == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, a);
    if (blockIdx.y == 0) {
        if (threadIdx.x == 0) *gs_out = gs;
        for (int32_t i = threadIdx.x; i < n_alpha; i += blockDim.x)
            alpha_out[i] = __fdiv_rn(1.0f, __fmul_rn(gs, gs_other[i]));
    }
    cudaTriggerProgrammaticLaunchCompletion();
    __shared__ float rcp_tab[256];
    build_rcp_table(gs, rcp_tab);
    quantize_sweep<T>(StashVecs<T>{stash, v0}, v0 + (threadIdx.x & ~31u), v1, blockDim.x, gs, rcp_tab, dst);
    cluster_wait();                                   // no CTA leaves while a peer may read it
}

// ------------------------------------------------------------------ MXFP4

template <typename T>
__global__ void __launch_bounds__(512) mx_quantize_kernel(const T* __restrict__ x, const VecIndex ix, uint32_t nv,
                                                          uint8_t* __restrict__ q, const SfOut sfo)
{
    grid_dependency_wait();      // launched early behind the previous kernel: wait for its data
    mx_quantize_sweep<T>(GlobalVecs<T>{x, ix}, blockIdx.x * blockDim.x + (threadIdx.x & ~31u), nv,
                         gridDim.x * blockDim.x, q, sfo);
}

// ------------------------------------------------------------------ elementwise conversions

__global__ void round_e4m3_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ out)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
        out[i] = static_cast<uint8_t>(f32_to_e4m3(x[i]));
}

__global__ void round_e2m1_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ out)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
        out[i] = static_cast<uint8_t>(f32x2_to_e2m1x2(x[i], 0.0f) & 0xFu);
}

// ------------------------------------------------------------------ launchers

// Blocks of 512 threads for a sweep over nv vectors (kUnroll per thread per pass), at most
// `cap`.
static int grid_1d(int64_t nv, int64_t cap)
{
    int64_t g = (nv + 512 * kUnroll - 1) / (512 * kUnroll);
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

static int grid_for(int64_t threads, int num_sms)
{
    int64_t blocks = (threads + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return static_cast<int>(blocks);
}

cudaError_t launch_global_scale(const void* x, bool bf16, int64_t numel, float* gs,
                                cudaStream_t stream, int num_sms)
{
    cudaError_t e = cudaMemsetAsync(gs, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    if (numel > 0) {
        // numel elements viewed as one row of 16-byte vectors, plus a scalar tail
        const int V = 8;                       // elements per vector (quant_core.cuh)
        const int64_t nvec = numel / V;
        if (nvec > 0) {
            // pieces of fewer than 2^31 vectors; the maxima meet in one atomicMax word
            const int64_t piece = int64_t(1) << 30;
            for (int64_t v0 = 0; v0 < nvec; v0 += piece) {
                const int64_t n = std::min(piece, nvec - v0);
                const VecIndex ix = make_vec_index(n, n * V, n * V);
                const int grid = grid_1d(n, static_cast<int64_t>(num_sms) * 4);
                if (bf16)
                    amax_kernel<__nv_bfloat16><<<grid, 512, 0, stream>>>(
                        static_cast<const __nv_bfloat16*>(x) + v0 * V, ix, static_cast<uint32_t>(n),
                        reinterpret_cast<unsigned*>(gs));
                else
                    amax_kernel<float><<<grid, 512, 0, stream>>>(
                        static_cast<const float*>(x) + v0 * V, ix, static_cast<uint32_t>(n),
                        reinterpret_cast<unsigned*>(gs));
                e = cudaGetLastError();
                if (e != cudaSuccess) return e;
            }
        }
        const int64_t tail = numel - nvec * V;
        if (tail > 0) {
            if (bf16)
                amax_tail_kernel<__nv_bfloat16><<<1, 32, 0, stream>>>(
                    static_cast<const __nv_bfloat16*>(x) + nvec * V, static_cast<int>(tail),
                    reinterpret_cast<unsigned*>(gs));
            else
                amax_tail_kernel<float><<<1, 32, 0, stream>>>(
                    static_cast<const float*>(x) + nvec * V, static_cast<int>(tail),
                    reinterpret_cast<unsigned*>(gs));
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    global_scale_finalize_kernel<<<1, 1, 0, stream>>>(gs);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx,
                            const float* gs, uint8_t* q, uint8_t* sf, cudaStream_t stream,
                            int num_sms)
{
    const int V = 8;                       // elements per vector (quant_core.cuh)
    const int64_t vpr = K / V;
    if (rows == 0 || vpr == 0) return cudaSuccess;
    const VecIndex ix = make_vec_index(vpr, ldx, K);
    // row pieces of fewer than 2^31 vectors (rows are independent once gs is known)
    const int64_t piece_rows = std::max<int64_t>(1, (int64_t(1) << 30) / vpr);
    const size_t esz = bf16 ? 2 : 4;
    for (int64_t r0 = 0; r0 < rows; r0 += piece_rows) {
        const int64_t n_rows = std::min(piece_rows, rows - r0);
        const int64_t nv = n_rows * vpr;
        const int grid = grid_1d(nv, static_cast<int64_t>(num_sms) * 4);
        const void* xp = static_cast<const uint8_t*>(x) + static_cast<size_t>(r0 * ldx) * esz;
        uint8_t* qp = q + r0 * (K / 2);
        const SfOut sp = make_sf_out(sf + r0 * (K / 16), kSfLinear, ix, K);
        if (bf16)
            quantize_kernel<__nv_bfloat16><<<grid, 512, 0, stream>>>(
                static_cast<const __nv_bfloat16*>(xp), ix, static_cast<uint32_t>(nv), gs, qp, sp);
        else
            quantize_kernel<float><<<grid, 512, 0, stream>>>(
                static_cast<const float*>(xp), ix, static_cast<uint32_t>(nv), gs, qp, sp);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Largest cluster (16, else 8) of 512-thread quantiser CTAs the device runs; cached.
template <typename T, class Dst>
static int quantize_cluster_size()
{
    static int cached[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { cudaGetLastError(); return 0; }
    std::lock_guard<std::mutex> g(mu);
    if (cached[dev] == 0) {
        auto kern = quantize_dynamic_cluster_kernel<T, Dst>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        int best = -1;
        for (int cs : {16, 8}) {
            cudaLaunchConfig_t cfg;
            std::memset(&cfg, 0, sizeof(cfg));
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = 1;
            attr.val.clusterDim.y = cs;
            attr.val.clusterDim.z = 1;
            cfg.gridDim = dim3(1, cs, 1);
            cfg.blockDim = dim3(512, 1, 1);
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) { best = cs; break; }
            cudaGetLastError();
        }
        cached[dev] = best;
    }
    return cached[dev] > 0 ? cached[dev] : 0;
}

// Tensors up to this size are quantised by one cluster; larger ones by a cooperative grid
// (measured on B200: one 16-CTA cluster wins at 393 KB, loses from 1.5 MB up).
constexpr int64_t kClusterQuantizeMaxBytes = int64_t(512) << 10;
// Shared-memory share per cluster CTA the launcher allows (the input is kept on chip).
constexpr int64_t kClusterStashMaxBytes = int64_t(200) << 10;
// Tensors up to this size use one 1024-thread block per SM (half the grid-barrier
// participants), larger ones two 512-thread blocks (measured on B200: 1024 wins at 1.5 and
// 6.3 MB, loses at 25 MB).
constexpr int64_t kCoopSmallBytes = int64_t(8) << 20;

static inline int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// Cooperative grid: BPS blocks of THREADS per SM at most (co-resident), at least two vectors
// per thread, and room for the parked maxima and flags (8 bytes per block) in q. Each block
// keeps its share in shared memory when it fits (about 200 KB per SM); otherwise the tensor
// is swept twice.
template <typename T, int THREADS, int BPS, class Dst>
static cudaError_t launch_coop(const T* x, const VecIndex& ix, int64_t nv, float* gs_out, uint8_t* q,
                               const Dst& sf, const float* gs_other, int32_t n_alpha, float* alpha_out,
                               int64_t q_bytes, unsigned* err_word, cudaStream_t stream, int num_sms)
{
    constexpr int64_t kResidentMaxBytes = (int64_t(200) << 10) / BPS;
    // at least 32 bytes of input per thread
    const int64_t per_block = 32 * static_cast<int64_t>(THREADS) / static_cast<int64_t>(sizeof(typename InTraits<T>::Raw));
    int64_t blocks = std::min<int64_t>(BPS * static_cast<int64_t>(num_sms), (nv + per_block - 1) / per_block);
    blocks = std::max<int64_t>(1, std::min<int64_t>(blocks, q_bytes / 8));
    int64_t chunk = round_up((nv + blocks - 1) / blocks, 32);
    constexpr int64_t kVecBytes = sizeof(typename InTraits<T>::Raw);
    const bool resident = chunk * kVecBytes <= kResidentMaxBytes;
    void (*kern)(const T*, const VecIndex, uint32_t, uint32_t, float*, uint8_t*, const Dst, const float*,
                 int32_t, float*, unsigned*) =
        resident ? quantize_dynamic_kernel<T, true, THREADS, Dst> : quantize_dynamic_kernel<T, false, THREADS, Dst>;
    size_t smem = 0;
    if (resident) {
        static std::once_flag once;
        std::call_once(once, [] {
            cudaFuncSetAttribute(quantize_dynamic_kernel<T, true, THREADS, Dst>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kResidentMaxBytes));
        });
        smem = static_cast<size_t>(chunk) * kVecBytes;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t fit = static_cast<int64_t>(std::min(per_sm, BPS)) * num_sms;   // co-resident blocks
    if (resident) {
        if (blocks > fit) {        // fewer blocks than planned: larger shares (same smem bound)
            blocks = fit;
            chunk = round_up((nv + blocks - 1) / blocks, 32);
            if (chunk * kVecBytes > static_cast<int64_t>(smem)) return cudaErrorInvalidConfiguration;
        }
        blocks = (nv + chunk - 1) / chunk;       // no empty block
    } else {
        blocks = std::min(blocks, fit);
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const uint32_t nv32 = static_cast<uint32_t>(nv), chunk32 = static_cast<uint32_t>(chunk);
    cudaError_t le = cudaLaunchKernelEx(&cfg, kern, x, ix, nv32, chunk32, gs_out, q, sf, gs_other, n_alpha,
                                        alpha_out, err_word);
    if (le == cudaErrorNotSupported || le == cudaErrorInvalidValue) {
        // a runtime that refuses the early-launch attribute on a cooperative launch: without it
        cudaGetLastError();
        cfg.numAttrs = 1;
        le = cudaLaunchKernelEx(&cfg, kern, x, ix, nv32, chunk32, gs_out, q, sf, gs_other, n_alpha, alpha_out,
                                err_word);
    }
    return le;
}

template <typename T, class Dst>
static cudaError_t launch_dynamic_t(const T* x, int64_t rows, int64_t vpr, const VecIndex& ix, int64_t K,
                                    float* gs_out, uint8_t* q, const Dst& sf,
                                    const float* gs_other, int32_t n_alpha, float* alpha_out,
                                    int64_t q_bytes, unsigned* err_word, cudaStream_t stream, int num_sms)
{
    const int64_t bytes = rows * K * static_cast<int64_t>(sizeof(T));
    const int64_t nv = rows * vpr;                       // < 2^31 (checked by the caller)
    const int ccs = bytes <= kClusterQuantizeMaxBytes ? quantize_cluster_size<T, Dst>() : 0;
    if (ccs > 0) {
        const int cs = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ccs, (nv + 511) / 512)));
        const int64_t chunk = round_up((nv + cs - 1) / cs, 32);
        if (chunk * static_cast<int64_t>(sizeof(typename InTraits<T>::Raw)) > kClusterStashMaxBytes)
            return cudaErrorInvalidValue;
        auto kern = quantize_dynamic_cluster_kernel<T, Dst>;
        static std::once_flag once;
        std::call_once(once, [&] {
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kClusterStashMaxBytes));
        });
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3(1, static_cast<unsigned>(cs), 1);
        cfg.blockDim = dim3(512, 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(chunk) * sizeof(typename InTraits<T>::Raw);
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = static_cast<unsigned>(cs);
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, kern, x, ix, static_cast<uint32_t>(nv), static_cast<uint32_t>(chunk),
                                  gs_out, sf, gs_other, n_alpha, alpha_out);
    }

    if (bytes <= kCoopSmallBytes)
        return launch_coop<T, 1024, 1>(x, ix, nv, gs_out, q, sf, gs_other, n_alpha, alpha_out, q_bytes, err_word,
                                       stream, num_sms);
    return launch_coop<T, 512, 2>(x, ix, nv, gs_out, q, sf, gs_other, n_alpha, alpha_out, q_bytes, err_word,
                                  stream, num_sms);
}

cudaError_t launch_quantize_dynamic(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx,
                                    float* gs_out, uint8_t* q, uint8_t* sf, int sf_layout,
                                    const float* gs_other, int32_t n_alpha, float* alpha_out,
                                    unsigned* err_word, cudaStream_t stream, int num_sms)
{
    const int V = 8;                       // elements per vector (quant_core.cuh)
    const int64_t vpr = K / V;
    const int64_t q_bytes = rows * (K / 2);
    const VecIndex ix = make_vec_index(vpr, ldx, K);
    const DenseDst dst{q, make_sf_out(sf, sf_layout, ix, K)};
    if (bf16)
        return launch_dynamic_t(static_cast<const __nv_bfloat16*>(x), rows, vpr, ix, K, gs_out, q, dst,
                                gs_other, n_alpha, alpha_out, q_bytes, err_word, stream, num_sms);
    return launch_dynamic_t(static_cast<const float*>(x), rows, vpr, ix, K, gs_out, q, dst, gs_other,
                            n_alpha, alpha_out, q_bytes, err_word, stream, num_sms);
}

cudaError_t launch_gather_quantize(const void* x, bool bf16, int64_t T, int64_t H, int64_t ldx, int32_t k,
                                   const int32_t* row_of, float* gs_out, uint8_t* q, uint8_t* sf,
                                   const float* gs_other, int32_t n_alpha, float* alpha_out,
                                   unsigned* err_word, cudaStream_t stream, int num_sms)
{
    const int V = 8;                       // elements per vector (quant_core.cuh)
    const int64_t vpr = H / V;
    const int64_t q_bytes = T * k * (H / 2);
    const VecIndex ix = make_vec_index(vpr, ldx, H);
    const ScatterDst dst{q, sf, row_of, k, ix.vpr, ix.mul, ix.shift};
    if (bf16)
        return launch_dynamic_t(static_cast<const __nv_bfloat16*>(x), T, vpr, ix, H, gs_out, q, dst,
                                gs_other, n_alpha, alpha_out, q_bytes, err_word, stream, num_sms);
    return launch_dynamic_t(static_cast<const float*>(x), T, vpr, ix, H, gs_out, q, dst, gs_other,
                            n_alpha, alpha_out, q_bytes, err_word, stream, num_sms);
}

cudaError_t launch_mx_quantize(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx, uint8_t* q,
                               uint8_t* sf, bool sf_tiled, cudaStream_t stream, int num_sms)
{
    const int V = 8;                       // elements per vector (quant_core.cuh)
    const int64_t vpr = K / V;
    if (rows == 0 || vpr == 0) return cudaSuccess;
    const VecIndex ix = make_vec_index(vpr, ldx, K);
    const int64_t nv = rows * vpr;         // < 2^31 (checked by the caller)
    const SfOut sfo = make_sf_out(sf, sf_tiled ? kSfTiled : kSfLinear, ix, K, 32);
    // one vector per thread per pass: enough warps to cover the tensor, at most 8 per SM
    int64_t grid = (nv + 511) / 512;
    if (grid > static_cast<int64_t>(num_sms) * 4) grid = static_cast<int64_t>(num_sms) * 4;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(512, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (bf16)
        return cudaLaunchKernelEx(&cfg, mx_quantize_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(x),
                                  ix, static_cast<uint32_t>(nv), q, sfo);
    return cudaLaunchKernelEx(&cfg, mx_quantize_kernel<float>, static_cast<const float*>(x), ix,
                              static_cast<uint32_t>(nv), q, sfo);
}

cudaError_t launch_alpha(const float* gs_a, const float* gs_b, int32_t n, float* alpha,
                         cudaStream_t stream)
{
    if (n <= 0) return cudaSuccess;
    alpha_kernel<<<(n + 255) / 256, 256, 0, stream>>>(gs_a, gs_b, n, alpha);
    return cudaGetLastError();
}

cudaError_t launch_round(const float* x, int64_t n, uint8_t* out, bool e2m1, cudaStream_t stream,
                         int num_sms)
{
    if (n <= 0) return cudaSuccess;
    const int grid = grid_for(n, num_sms);
    if (e2m1) round_e2m1_kernel<<<grid, 256, 0, stream>>>(x, n, out);
    else round_e4m3_kernel<<<grid, 256, 0, stream>>>(x, n, out);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ scale layout

// Row-major scales [rows][kb] -> the 8 x 4 layout (quant_core.cuh, SfOut), one output byte per
// thread; rows past `rows` in the last 8-row group are zero.
__global__ void sf_8x4_kernel(const uint8_t* __restrict__ sf, int64_t rows, int64_t kb, int64_t kb4,
                              uint8_t* __restrict__ out, int64_t out_bytes)
{
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < out_bytes;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t block = o >> 5, within = o & 31;
        const int64_t rg = block / kb4, cg = block - rg * kb4;
        const int64_t r = rg * 8 + (within >> 2);
        const int64_t c = cg * 4 + (within & 3);
        out[o] = r < rows ? sf[r * kb + c] : 0;
    }
}

cudaError_t launch_sf_8x4(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* out, cudaStream_t stream,
                          int num_sms)
{
    const int64_t kb = K / 16;
    const int64_t out_bytes = (rows + 7) / 8 * 8 * kb;
    if (out_bytes == 0) return cudaSuccess;
    const int grid = grid_for(out_bytes, num_sms);
    sf_8x4_kernel<<<grid, 256, 0, stream>>>(sf, rows, kb, kb / 4, out, out_bytes);
    return cudaGetLastError();
}

// Row-major scales [rows][K/16] -> the tiled layout (quant_core.cuh, SfOut), one output byte
// per thread; rows past `rows` in the last 128-row tile are zero.
__global__ void sf_tile_kernel(const uint8_t* __restrict__ sf, int64_t rows, int64_t kb, int64_t kb4,
                               uint8_t* __restrict__ out, int64_t out_bytes)
{
    for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < out_bytes;
         o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t block = o >> 9, within = o & 511;
        const int64_t rt = block / kb4, kt = block - rt * kb4;
        const int64_t r = rt * 128 + ((within >> 2) & 3) * 32 + (within >> 4);
        const int64_t c = kt * 4 + (within & 3);
        out[o] = r < rows ? sf[r * kb + c] : 0;
    }
}

cudaError_t launch_sf_tile(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* out, cudaStream_t stream,
                           int num_sms, int block)
{
    const int64_t kb = K / block;          // scale columns per row
    const int64_t out_bytes = (rows + 127) / 128 * 128 * kb;
    if (out_bytes == 0) return cudaSuccess;
    const int grid = grid_for(out_bytes, num_sms);
    sf_tile_kernel<<<grid, 256, 0, stream>>>(sf, rows, kb, kb / 4, out, out_bytes);
    return cudaGetLastError();
}

}  // namespace nvfp4
