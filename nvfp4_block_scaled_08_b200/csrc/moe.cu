// moe.cu -- the mixture-of-experts layer around the grouped GEMM ("When a Benchmark Crashes",
// section "Why This Message Was Written": every token goes to 8 of 256 experts): top-k routing
// of the router logits, the expert-sorted permutation (a stable counting sort), and the weighted
// combine of the down projection's rows. The quantisation of the tokens into expert-sorted rows
// (gather + quantise in one launch) is quantize.cu's launch_gather_quantize.
//
// Readings (the pages name the layer only): probabilities are a softmax over the expert
// logits; a token takes its k largest, ties going to the lower expert index, in descending
// order; its k weights are those probabilities renormalised to sum to 1; the expert-sorted
// order lists each expert's (token, slot) pairs in ascending token order; the combine sums
// each token's k output rows weighted by its k weights.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace nvfp4 {

// ------------------------------------------------------------------ top-k routing

// One warp per token. Lane l holds logits l, l + 32, ... of its token (PER of them, E <= 32
// PER; entries past E count as taken) and keeps its best untaken entry (larger logit first,
// then the lower expert index). k rounds of a warp arg-max over the lanes' bests (ties to the
// lower expert index; the softmax is monotonic, so this is the order of the probabilities);
// only the winning lane marks its entry taken and looks for its next best.
// Weights: w_s = exp(l_s - l_0) / sum_j exp(l_j - l_0) over the k winners (l_0 the largest):
// the softmax probabilities renormalised over the winners (the full softmax's denominator
// cancels), in fp32 with CUDA's expf, summed in slot order.
template <int PER>
__device__ __forceinline__ void lane_best(const float (&v)[PER], uint32_t taken, int lane, float& bv, int& bi)
{
    bv = -INFINITY;
    bi = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (!(taken & (1u << i)) && (v[i] > bv || bi == 0x7FFFFFFF)) {
            bv = v[i];
            bi = lane + 32 * i;
        }
    }
}

template <int PER>
__global__ void __launch_bounds__(256) moe_topk_kernel(const float* __restrict__ logits, int32_t T, int32_t E,
                                                       int32_t k, int32_t* __restrict__ experts,
                                                       float* __restrict__ weights)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;                                   // warp-uniform
    const float* row = logits + t * E;
    float v[PER];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldg(row + e) : -INFINITY;
        if (e >= E) taken |= 1u << i;
    }
    float bv;
    int bi;
    lane_best<PER>(v, taken, lane, bv, bi);
    float my_val = 0.0f, top = 0.0f;
    int my_idx = 0;
    for (int s = 0; s < k; ++s) {
        // warp arg-max of the lanes' bests: larger value, then lower index
        float wv = bv;
        int wi = bi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
            if (ov > wv || (ov == wv && oi < wi)) {
                wv = ov;
                wi = oi;
            }
        }
        if ((wi & 31) == lane) {
            taken |= 1u << (wi >> 5);
            lane_best<PER>(v, taken, lane, bv, bi);
        }
        if (s == 0) top = wv;
        if (lane == s) {
            my_val = wv;
            my_idx = wi;
        }
    }
    // weights of the k winners: lane s holds winner s
    const float ex = lane < k ? expf(my_val - top) : 0.0f;
    float sum = 0.0f;
    for (int s = 0; s < k; ++s) sum += __shfl_sync(0xffffffffu, ex, s);
    if (lane < k) {
        experts[t * k + lane] = my_idx;
        weights[t * k + lane] = ex / sum;
    }
}

// ------------------------------------------------------------------ expert-sorted permutation

// Block e (1024 threads): the (token, slot) pairs routed to expert e, in ascending token
// order; pair p = t k + s, and ascending p is ascending token order (a token's k experts are
// distinct). The pairs are read in rounds of 16 per thread: load j of thread i is the 16-byte
// vector 4 (i + 1024 j) .. + 3 (four 4-byte loads if `experts` is not 16-byte aligned), so every
// load instruction is coalesced. The four loads' hit
// counts (each 0..4) travel packed in 16-bit fields of one 64-bit value through one block
// scan, which gives every hit its rank among expert e's pairs (all of load j's pairs precede
// load j + 1's); the rank is written to rank_out[p] (each pair has one expert, so exactly one
// block writes it). The expert's count goes to count_out[e].
constexpr int kRankThreads = 1024;
constexpr int kRankLoads = 4;                          // 16-byte loads per thread and round

__device__ __forceinline__ unsigned long long warp_incl_scan_u64(unsigned long long v, int lane)
{
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += y;
    }
    return v;
}

__global__ void __launch_bounds__(kRankThreads) moe_rank_kernel(const int32_t* __restrict__ experts, int64_t pairs,
                                                                int32_t* __restrict__ rank_out,
                                                                int32_t* __restrict__ count_out)
{
    __shared__ unsigned long long warp_tot[kRankThreads / 32];
    __shared__ unsigned long long s_total;
    const int e = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int64_t kVec = 4;
    constexpr int64_t kRound = kVec * kRankThreads * kRankLoads;
    const bool vec_ok = (reinterpret_cast<uintptr_t>(experts) & 15u) == 0;   // else 4-byte loads
    int32_t run = 0;                                   // expert e's pairs before this round
    for (int64_t p0 = 0; p0 < pairs; p0 += kRound) {
        int4 v[kRankLoads];
        uint32_t hits[kRankLoads];
        unsigned long long packed = 0;
#pragma unroll
        for (int j = 0; j < kRankLoads; ++j) {
            const int64_t p = p0 + kVec * (tid + static_cast<int64_t>(kRankThreads) * j);
            if (vec_ok && p + kVec <= pairs) {
                v[j] = __ldg(reinterpret_cast<const int4*>(experts + p));
            } else {
                v[j].x = p < pairs ? __ldg(experts + p) : -1;
                v[j].y = p + 1 < pairs ? __ldg(experts + p + 1) : -1;
                v[j].z = p + 2 < pairs ? __ldg(experts + p + 2) : -1;
                v[j].w = p + 3 < pairs ? __ldg(experts + p + 3) : -1;
            }
            hits[j] = (v[j].x == e ? 1u : 0u) | (v[j].y == e ? 2u : 0u) | (v[j].z == e ? 4u : 0u) |
                      (v[j].w == e ? 8u : 0u);
            packed |= static_cast<unsigned long long>(__popc(hits[j])) << (16 * j);
        }
        // exclusive scan of the packed counts over the block (thread order within each load j;
        // a field never exceeds 4 * 1024, so the fields do not carry into one another)
        const unsigned long long incl = warp_incl_scan_u64(packed, lane);
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const unsigned long long t = warp_tot[lane];
            const unsigned long long ti = warp_incl_scan_u64(t, lane);
            warp_tot[lane] = ti - t;                   // the warps before this one
            if (lane == 31) s_total = ti;              // the round's count per load
        }
        __syncthreads();
        const unsigned long long excl = warp_tot[warp] + incl - packed;
        const unsigned long long total = s_total;
        int32_t base = run;
#pragma unroll
        for (int j = 0; j < kRankLoads; ++j) {
            int32_t r = base + static_cast<int32_t>((excl >> (16 * j)) & 0xFFFFu);
            if (hits[j]) {
                const int64_t p = p0 + kVec * (tid + static_cast<int64_t>(kRankThreads) * j);
                if (hits[j] & 1u) rank_out[p] = r++;
                if (hits[j] & 2u) rank_out[p + 1] = r++;
                if (hits[j] & 4u) rank_out[p + 2] = r++;
                if (hits[j] & 8u) rank_out[p + 3] = r++;
            }
            base += static_cast<int32_t>((total >> (16 * j)) & 0xFFFFu);
        }
        run = base;
        __syncthreads();                               // warp_tot and s_total are reused
    }
    if (tid == 0) count_out[e] = run;
}

// One block: offsets[0] = 0, offsets[e + 1] = offsets[e] + count[e], in place (the counts are
// read from offsets[1 .. E], where moe_rank_kernel left them; E <= 1024, one per thread).
__global__ void __launch_bounds__(1024) moe_scan_kernel(int32_t E, int32_t* __restrict__ offsets)
{
    __shared__ int32_t warp_tot[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = tid < E ? offsets[tid + 1] : 0;
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();                                   // every count has been read
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    if (tid < E) offsets[tid + 1] = base + incl;
    if (tid == 0) offsets[0] = 0;
}

// Every pair p = t k + s: row_of[p] = offsets[expert] + rank (the rank is read from row_of[p],
// in place) and token_of_row[row_of[p]] = t. Grid-stride; each block keeps the offsets in
// shared memory.
__global__ void __launch_bounds__(256) moe_fill_kernel(const int32_t* __restrict__ experts, int64_t pairs,
                                                       int32_t E, int32_t k, const int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ row_of,
                                                       int32_t* __restrict__ token_of_row)
{
    __shared__ int32_t s_off[1025];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    for (int64_t p = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; p < pairs;
         p += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t row = s_off[__ldg(experts + p)] + row_of[p];
        row_of[p] = row;
        token_of_row[row] = static_cast<int32_t>(p / k);
    }
}

cudaError_t launch_moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* experts,
                             float* weights, int32_t* offsets, int32_t* row_of, int32_t* token_of_row,
                             cudaStream_t stream)
{
    cudaError_t e;
    if (T > 0) {
        // entries per lane: the power of two at or above ceil(E / 32)
        const int per = (E + 31) / 32;
        const unsigned grid = static_cast<unsigned>((T + 7) / 8);
        if (per <= 1) moe_topk_kernel<1><<<grid, 256, 0, stream>>>(logits, T, E, k, experts, weights);
        else if (per <= 2) moe_topk_kernel<2><<<grid, 256, 0, stream>>>(logits, T, E, k, experts, weights);
        else if (per <= 4) moe_topk_kernel<4><<<grid, 256, 0, stream>>>(logits, T, E, k, experts, weights);
        else if (per <= 8) moe_topk_kernel<8><<<grid, 256, 0, stream>>>(logits, T, E, k, experts, weights);
        else if (per <= 16) moe_topk_kernel<16><<<grid, 256, 0, stream>>>(logits, T, E, k, experts, weights);
        else moe_topk_kernel<32><<<grid, 256, 0, stream>>>(logits, T, E, k, experts, weights);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    moe_rank_kernel<<<E, kRankThreads, 0, stream>>>(experts, static_cast<int64_t>(T) * k, row_of, offsets + 1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    moe_scan_kernel<<<1, 1024, 0, stream>>>(E, offsets);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t pairs = static_cast<int64_t>(T) * k;
    if (pairs > 0) {
        int64_t blocks = (pairs + 255) / 256;
        if (blocks > 1024) blocks = 1024;
        moe_fill_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(experts, pairs, E, k, offsets, row_of,
                                                                          token_of_row);
        e = cudaGetLastError();
    }
    return e;
}

// ------------------------------------------------------------------ combine

template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&v)[8])
{
    if constexpr (DT == 2) {            // fp32
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (DT == 0) {    // bf16: the upper half of an fp32
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            } else {                    // fp16
                v[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
                v[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
            }
        }
    }
}

__device__ __forceinline__ void store8(void* base, int64_t idx, int32_t dt, const float (&v)[8])
{
    if (dt == 2) {
        float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + idx);
        p[0] = make_float4(v[0], v[1], v[2], v[3]);
        p[1] = make_float4(v[4], v[5], v[6], v[7]);
        return;
    }
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (dt == 1) {
            w[i] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[2 * i]))) |
                   (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[2 * i + 1]))) << 16);
        } else {
            w[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i]))) |
                   (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1]))) << 16);
        }
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(base) + idx) = make_uint4(w[0], w[1], w[2], w[3]);
}

// out[t, :] = sum_s weights[t, s] * y[row_of[t, s], :] in fp32, slots in ascending order (fixed,
// deterministic); one thread per 8 consecutive columns of a token (16- or 32-byte loads and
// stores, consecutive threads on consecutive addresses), grid-stride.
template <int YDT>
__global__ void __launch_bounds__(256) moe_combine_kernel(const void* __restrict__ y, const float* __restrict__ w,
                                                          const int32_t* __restrict__ row_of, int32_t T, int64_t H,
                                                          int32_t k, void* __restrict__ out, int32_t out_dt)
{
    const int64_t per_row = H / 8;
    const int64_t items = static_cast<int64_t>(T) * per_row;
    for (int64_t it = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; it < items;
         it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = it / per_row;
        const int64_t c = (it - t * per_row) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int s = 0; s < k; ++s) {
            const int64_t row = __ldg(row_of + t * k + s);
            const float ws = __ldg(w + t * k + s);
            float v[8];
            load8<YDT>(y, row * H + c, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = fmaf(ws, v[j], acc[j]);
        }
        store8(out, t * H + c, out_dt, acc);
    }
}

cudaError_t launch_moe_combine(const void* y, int32_t y_dt, const float* weights, const int32_t* row_of,
                               int32_t T, int64_t H, int32_t k, void* out, int32_t out_dt, cudaStream_t stream,
                               int num_sms)
{
    const int64_t items = static_cast<int64_t>(T) * (H / 8);
    int64_t blocks = (items + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const dim3 g(static_cast<unsigned>(blocks));
    if (y_dt == 0) moe_combine_kernel<0><<<g, 256, 0, stream>>>(y, weights, row_of, T, H, k, out, out_dt);
    else if (y_dt == 1) moe_combine_kernel<1><<<g, 256, 0, stream>>>(y, weights, row_of, T, H, k, out, out_dt);
    else moe_combine_kernel<2><<<g, 256, 0, stream>>>(y, weights, row_of, T, H, k, out, out_dt);
    return cudaGetLastError();
}

}  // namespace nvfp4
