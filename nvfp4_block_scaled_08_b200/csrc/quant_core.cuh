// quant_core.cuh -- the NVFP4 quantisation arithmetic of the quantiser kernels: format
// conversions, the flat vector view of a [rows, K] tensor, the amax and quantisation sweeps
// and the block reductions.
//
// Format: packed e2m1 values two per byte with one float8_e4m3fn scale per 16 K-elements
// ("When a Benchmark Crashes", section "Input Knowledge Required", item 3; block_size=16
// from "The Art of Reading the Manual", section "The Message"). The pages give no recipe;
// this library uses the two-level NVFP4 recipe with the fixed fp32 operation order stated
// in include/nvfp4.h. Every fp32 operation uses an explicitly rounded intrinsic
// (__fdiv_rn, __fmul_rn), so no contraction or reassociation can change a result.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// fp32 -> e4m3fn byte, round to nearest even, finite values saturate to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float v)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(v), "f"(v));
    return r & 0xFFu;
}

// e4m3fn byte -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte)
{
    const uint16_t pair = static_cast<uint16_t>(byte | (byte << 8));
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Two fp32 values -> one byte of e2m1 codes (round to nearest even, saturating at +-6),
// `lo` in the low nibble.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "mov.b32 %0, {t, 0, 0, 0};\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// Eight fp32 values times r, each product rounded to nearest even (four packed two-lane
// multiplies, mul.rn.f32x2), then e2m1-coded and packed into 32 bits: value 2i in the low
// nibble of byte i, as f32x2_to_e2m1x2 does for one pair.
__device__ __forceinline__ uint32_t scale_to_e2m1x8(const float (&v)[8], float r)
{
    uint32_t out;
    asm("{\n\t"
        ".reg .b64 s, p0, p1, p2, p3;\n\t"
        ".reg .f32 y0, y1, y2, y3, y4, y5, y6, y7;\n\t"
        ".reg .b8 c0, c1, c2, c3;\n\t"
        "mov.b64 s, {%9, %9};\n\t"
        "mov.b64 p0, {%1, %2};\n\t"
        "mov.b64 p1, {%3, %4};\n\t"
        "mov.b64 p2, {%5, %6};\n\t"
        "mov.b64 p3, {%7, %8};\n\t"
        "mul.rn.f32x2 p0, p0, s;\n\t"
        "mul.rn.f32x2 p1, p1, s;\n\t"
        "mul.rn.f32x2 p2, p2, s;\n\t"
        "mul.rn.f32x2 p3, p3, s;\n\t"
        "mov.b64 {y0, y1}, p0;\n\t"
        "mov.b64 {y2, y3}, p1;\n\t"
        "mov.b64 {y4, y5}, p2;\n\t"
        "mov.b64 {y6, y7}, p3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c0, y1, y0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c1, y3, y2;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c2, y5, y4;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c3, y7, y6;\n\t"
        "mov.b32 %0, {c0, c1, c2, c3};\n\t"
        "}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(r));
    return out;
}

// Every lane handles a "vector" of 8 consecutive elements (two lanes per 16-element block):
// 32 bytes of fp32 (two 16-byte loads) or 16 bytes of bf16.
struct Raw32 {
    uint4 lo, hi;
};

template <typename T> struct InTraits;
template <> struct InTraits<float> {
    static constexpr int kPerThread = 8;
    using Raw = Raw32;
    __device__ static Raw load(const float* p)
    {
        return Raw32{__ldg(reinterpret_cast<const uint4*>(p)), __ldg(reinterpret_cast<const uint4*>(p + 4))};
    }
    __device__ static Raw zero() { return Raw32{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)}; }
    __device__ static void decode(const Raw& u, float (&v)[8])
    {
        v[0] = __uint_as_float(u.lo.x); v[1] = __uint_as_float(u.lo.y);
        v[2] = __uint_as_float(u.lo.z); v[3] = __uint_as_float(u.lo.w);
        v[4] = __uint_as_float(u.hi.x); v[5] = __uint_as_float(u.hi.y);
        v[6] = __uint_as_float(u.hi.z); v[7] = __uint_as_float(u.hi.w);
    }
};
template <> struct InTraits<__nv_bfloat16> {
    static constexpr int kPerThread = 8;
    using Raw = uint4;
    __device__ static Raw load(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ static Raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
    __device__ static void decode(const Raw& u, float (&v)[8])
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

// ------------------------------------------------------------------ indexing

// A [rows, K] tensor of T (row stride ld elements) is read as nv = rows * vpr 16-byte
// vectors (V elements each, vpr = K / V per row), numbered row-major: vector i is row
// i / vpr, column i % vpr. Every launch keeps nv < 2^31, so indices are 32-bit. With
// contiguous rows (ld == K) vector i sits at x + i * V and no division is needed;
// otherwise the row comes from a multiply-high by a precomputed reciprocal ("round-up"
// method of Granlund and Montgomery, PLDI 1994: with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (mulhi(n, m) + n) >> l for every n < 2^32).
// The codes and scales are written contiguously: vector i's codes at q + i * V / 2, the
// scale of the 16-element block holding it at sf + i / (16 / V).
struct VecIndex {
    uint32_t vpr;      // vectors per row
    uint32_t mul;      // m above (d = vpr)
    uint32_t shift;    // l above
    uint32_t contiguous;
    int64_t ld;        // row stride in elements
};

inline VecIndex make_vec_index(int64_t vpr, int64_t ld, int64_t K)
{
    VecIndex ix;
    ix.vpr = static_cast<uint32_t>(vpr);
    uint32_t l = 0;
    while ((uint64_t(1) << l) < static_cast<uint64_t>(vpr)) ++l;
    ix.shift = l;
    ix.mul = static_cast<uint32_t>(((uint64_t(1) << 32) * ((uint64_t(1) << l) - static_cast<uint64_t>(vpr)))
                                   / static_cast<uint64_t>(vpr) + 1);
    ix.contiguous = (ld == K) ? 1u : 0u;
    ix.ld = ld;
    return ix;
}

template <int V>
__device__ __forceinline__ int64_t vec_offset(const VecIndex& ix, uint32_t i)
{
    if (ix.contiguous) return static_cast<int64_t>(i) * V;
    const uint32_t r = static_cast<uint32_t>((static_cast<uint64_t>(__umulhi(i, ix.mul)) + i) >> ix.shift);
    const uint32_t c = i - r * ix.vpr;
    return static_cast<int64_t>(r) * ix.ld + static_cast<int64_t>(c) * V;
}

// Where the block scales go: row-major [rows][K/16] bytes, or the tiled layout of
// include/nvfp4.h (NVFP4_SF_TILED): for row r and scale column c (16-element block),
//     ((r / 128) * (K / 64) + c / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4,
// i.e. 512-byte blocks of 128 rows x 4 scales, each holding, in its 16-byte row i, the scales
// of rows i, i + 32, i + 64, i + 96: the source layout of tcgen05.cp ... 32x128b.warpx4.
// Or the 8 x 4 layout (NVFP4_SF_8X4): 32-byte blocks of 8 rows x 4 scales, row-major inside
// the block, the blocks of a row group consecutive along K:
//     ((r / 8) * (K / 64) + c / 4) * 32 + (r % 8) * 4 + c % 4.
enum : int32_t { kSfLinear = 0, kSfTiled = 1, kSf8x4 = 2 };

struct SfOut {
    uint8_t* sf;
    int32_t layout;          // kSfLinear, kSfTiled or kSf8x4
    uint32_t kb4;            // 4-scale column groups per row: K / 64 (NVFP4), K / 128 (MXFP4)
    uint32_t vpr, mul, shift;  // vector -> row, as in VecIndex

    // Scale of vector i's block. Offsets fit in 32 bits: there are fewer than 2^31 vectors,
    // so fewer than 2^30 scales, and the non-linear layouts pad the rows to 128 at most.
    template <int TPB>
    __device__ __forceinline__ uint8_t* at(uint32_t i) const
    {
        if (layout == kSfLinear) return sf + i / TPB;
        const uint32_t r = static_cast<uint32_t>((static_cast<uint64_t>(__umulhi(i, mul)) + i) >> shift);
        const uint32_t c = (i - r * vpr) / TPB;
        if (layout == kSf8x4) return sf + (((r >> 3) * kb4 + (c >> 2)) * 32u + (r & 7u) * 4u + (c & 3u));
        return sf + (((r >> 7) * kb4 + (c >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u));
    }
};

// block: elements per scale (16 for NVFP4, 32 for MXFP4); the non-linear layouts hold 4 scale
// columns per block, so a row group spans K / (4 block) blocks.
inline SfOut make_sf_out(uint8_t* sf, int layout, const VecIndex& ix, int64_t K, int block = 16)
{
    SfOut o;
    o.sf = sf;
    o.layout = layout;
    o.kb4 = static_cast<uint32_t>(K / (4 * block));
    o.vpr = ix.vpr;
    o.mul = ix.mul;
    o.shift = ix.shift;
    return o;
}

// Loads in flight per thread in the sweeps below.
constexpr int kUnroll = 4;

__device__ __forceinline__ float block_max(float m, float* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
    if (threadIdx.x < 32) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (threadIdx.x == 0) red[0] = m;
    }
    __syncthreads();
    m = red[0];
    __syncthreads();
    return m;
}

// Where a sweep's 16-byte vectors come from: global memory (vector i of the tensor), or this
// block's shared-memory copy of vectors [v0, v1) (stash[i - v0]).
template <typename T>
struct GlobalVecs {
    const T* x;
    VecIndex ix;
    __device__ typename InTraits<T>::Raw operator()(uint32_t i) const
    {
        return InTraits<T>::load(x + vec_offset<InTraits<T>::kPerThread>(ix, i));
    }
};
template <typename T>
struct StashVecs {
    const typename InTraits<T>::Raw* stash;
    uint32_t v0;
    __device__ typename InTraits<T>::Raw operator()(uint32_t i) const { return stash[i - v0]; }
};

// max |x| over vectors i0, i0 + step, ... < end of this thread, kUnroll loads in flight. With
// `keep`, every loaded vector is also copied to stash[i - v0] (the block's own range).
template <typename T, typename Src>
__device__ __forceinline__ float amax_sweep(const Src& src, uint32_t i0, uint32_t end, uint32_t step,
                                            typename InTraits<T>::Raw* keep = nullptr, uint32_t v0 = 0)
{
    constexpr int V = InTraits<T>::kPerThread;
    constexpr int U = kUnroll;
    float m = 0.0f;
    for (; i0 < end; i0 += U * step) {
        typename InTraits<T>::Raw w[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t i = i0 + u * step;
            w[u] = i < end ? src(i) : InTraits<T>::zero();
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t i = i0 + u * step;
            if (keep != nullptr && i < end) keep[i - v0] = w[u];
            float v[V];
            InTraits<T>::decode(w[u], v);
#pragma unroll
            for (int k = 0; k < V; ++k) m = fmaxf(m, fabsf(v[k]));
        }
    }
    return m;
}

// Quantise vectors [.., end): this warp takes the 32 consecutive vectors w0 + lane, then
// w0 + step + lane, ... (w0 warp-uniform and a multiple of 32). The TPB lanes that share a
// 16-element block are consecutive lanes of the warp (a block never straddles a row since
// vpr % TPB == 0); after a butterfly exchange each of them holds the block maximum and
// computes the same scale (no divergent branch), and the first of them stores it.
// Per block, in fp32 with explicit rounding and in this order:
//   amax -> s = e4m3(amax / 6 * gs) -> r = s ? gs / s : 0 -> codes e2m1(x * r).
// rcp_tab[c] = gs / e4m3(c) (0 where e4m3(c) is zero) for all 256 scale codes: every block
// scale of the tensor shares gs, so the division is done once per code (by the first 256
// threads), not once per 16-element block. Same operands, same rounding: the same values.
__device__ __forceinline__ void build_rcp_table(float gs, float* rcp_tab)
{
    if (threadIdx.x < 256) {
        const float sfd = e4m3_to_f32(threadIdx.x);
        rcp_tab[threadIdx.x] = (sfd == 0.0f) ? 0.0f : __fdiv_rn(gs, sfd);
    }
    __syncthreads();
}

// Where the codes and scale of vector i go.
// DenseDst: the codes of vector i at q + 4 i, its block scale through SfOut (row-major order).
struct DenseDst {
    uint8_t* q;
    SfOut sfo;
    static constexpr bool kContiguous = true;   // codes of vector i at q + 4 i
    template <int TPB>
    __device__ __forceinline__ void store(uint32_t i, uint32_t packed, uint32_t sfq, bool leader) const
    {
        *reinterpret_cast<uint32_t*>(q + static_cast<int64_t>(i) * 4) = packed;
        if (leader) *sfo.at<TPB>(i) = static_cast<uint8_t>(sfq);
    }
};

// ScatterDst: row t of the input goes to the k rows row_of[t k + s] (s < k) of the output
// (codes [rows_out][vpr * 4] bytes, linear scales [rows_out][vpr / 2]): the expert-sorted
// activations of a mixture-of-experts layer, quantised once per token.
struct ScatterDst {
    uint8_t* q;
    uint8_t* sf;
    const int32_t* row_of;
    int32_t k;
    uint32_t vpr, mul, shift;    // vector -> input row, as in VecIndex
    static constexpr bool kContiguous = false;
    template <int TPB>
    __device__ __forceinline__ void store(uint32_t i, uint32_t packed, uint32_t sfq, bool leader) const
    {
        const uint32_t t = static_cast<uint32_t>((static_cast<uint64_t>(__umulhi(i, mul)) + i) >> shift);
        const uint32_t c = i - t * vpr;
        for (int s = 0; s < k; ++s) {
            const int64_t row = __ldg(row_of + static_cast<int64_t>(t) * k + s);
            *reinterpret_cast<uint32_t*>(q + row * (static_cast<int64_t>(vpr) * 4) + c * 4) = packed;
            if (leader) sf[row * (static_cast<int64_t>(vpr) / TPB) + c / TPB] = static_cast<uint8_t>(sfq);
        }
    }
};

// reverse: walk the warp's chunks last to first (a second sweep over a tensor larger than
// the first sweep could leave in L2 then starts on what the first sweep read last). Each
// vector is quantised on its own, so the order does not change any output.
template <typename T, typename Src, typename Dst>
__device__ __forceinline__ void quantize_sweep(const Src& src, uint32_t w_first, uint32_t end, uint32_t step,
                                               float gs, const float* rcp_tab, const Dst& dst,
                                               bool reverse = false)
{
    constexpr int V = InTraits<T>::kPerThread;   // elements per thread (8)
    static_assert(V == 8, "8 elements per lane: 4 bytes of codes");
    constexpr int TPB = 16 / V;                  // threads per 16-element block
    constexpr int U = kUnroll;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t stride = U * step;
    const uint32_t chunks = w_first < end ? (end - w_first + stride - 1) / stride : 0u;
    for (uint32_t n = 0; n < chunks; ++n) {      // warp-uniform
        const uint32_t w0 = w_first + (reverse ? chunks - 1u - n : n) * stride;
        float v[U][V];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t i = w0 + u * step + lane;
            InTraits<T>::decode(i < end ? src(i) : InTraits<T>::zero(), v[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t ibase = w0 + u * step;
            if (ibase >= end) break;                 // warp-uniform
            const uint32_t i = ibase + lane;
            float amax = 0.0f;
#pragma unroll
            for (int k = 0; k < V; ++k) amax = fmaxf(amax, fabsf(v[u][k]));
#pragma unroll
            for (int o = 1; o < TPB; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));

            const float sf32 = __fmul_rn(__fdiv_rn(amax, 6.0f), gs);
            const uint32_t sfq = f32_to_e4m3(sf32);
            const float rcp = rcp_tab[sfq];
            const uint32_t packed = scale_to_e2m1x8(v[u], rcp);
            if (i < end) dst.template store<TPB>(i, packed, sfq, (lane & (TPB - 1)) == 0);
        }
    }
}

// MXFP4 (OCP MX v1.0 FP4: e2m1 elements, one E8M0 scale 2^(byte - 127) per 32 elements, no
// per-tensor scale; "The Art of Reading the Manual", section "The Message": use_nvfp4=False).
// Per block: shared_exp = floor(log2(amax)) - 2, clamped to [-127, 127] (an all-zero block:
// -127); byte = shared_exp + 127; codes e2m1_rn_satfinite(x * 2^-shared_exp). For finite
// amax >= 0 with biased exponent field E (0 for zero and subnormals), floor(log2(amax)) =
// E - 127 when E > 0, so byte = max(E - 2, 0) (E = 1 and subnormals clamp to byte 0), and
// 2^-shared_exp is the normal float with biased exponent 254 - byte (byte <= 252). x times a
// power of two is exact unless the product is below 2^-126, where no e2m1 code depends on
// the rounding (only the sign, which the product keeps).
// Four lanes (32 elements, 8 each) per block, warp-aligned vectors [w0 + lane, ...).
template <typename T, typename Src>
__device__ __forceinline__ void mx_quantize_sweep(const Src& src, uint32_t w0, uint32_t end, uint32_t step,
                                                  uint8_t* __restrict__ q, const SfOut& sfo)
{
    constexpr int V = InTraits<T>::kPerThread;
    static_assert(V == 8, "8 elements per lane");
    constexpr int TPB = 32 / V;                  // lanes per 32-element block
    const uint32_t lane = threadIdx.x & 31;
    for (; w0 < end; w0 += step) {               // warp-uniform
        const uint32_t i = w0 + lane;
        float v[V];
        InTraits<T>::decode(i < end ? src(i) : InTraits<T>::zero(), v);
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < V; ++k) amax = fmaxf(amax, fabsf(v[k]));
#pragma unroll
        for (int o = 1; o < TPB; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int e = static_cast<int>(__float_as_uint(amax) >> 23);   // amax >= 0: no sign bit
        const uint32_t byte = static_cast<uint32_t>(e > 2 ? e - 2 : 0);
        const float scale = __uint_as_float((254u - byte) << 23);
        const uint32_t packed = scale_to_e2m1x8(v, scale);
        if (i < end) {
            *reinterpret_cast<uint32_t*>(q + static_cast<int64_t>(i) * 4) = packed;
            if ((lane & (TPB - 1)) == 0) *sfo.at<TPB>(i) = static_cast<uint8_t>(byte);
        }
    }
}

// This block's contiguous share of nv vectors when they are split into blocks of `chunk`
// (a multiple of 32): [v0, v1).
__device__ __forceinline__ void block_range(uint32_t nv, uint32_t chunk, uint32_t bid, uint32_t& v0,
                                            uint32_t& v1)
{
    const uint64_t a = static_cast<uint64_t>(bid) * chunk;
    v0 = static_cast<uint32_t>(a < nv ? a : nv);
    v1 = static_cast<uint32_t>(a + chunk < nv ? a + chunk : nv);
}

}  // namespace nvfp4
