// gemm_kernel.cuh -- persistent, warp-specialised NVFP4 block-scaled GEMM for sm_100a.
//
// Computes out[m, n] = bf16(alpha * sum_k deq(A)[m, k] * deq(B)[n, k]) where both operands
// are packed e2m1 (two per byte, K-contiguous) with one e4m3 scale per 16 K-elements
// ("The Art of Reading the Manual", section "The Message": mm_fp4 with block_size=16,
// alpha and out; "When a Benchmark Crashes", section "Input Knowledge Required", item 3).
//
// The tensor cores see the problem as D[P, Q] = P x Q^T with a 128-row P tile (the MMA's
// M) and a BN-row Q tile (the MMA's N):
//   * SWAP = false: P = A (tokens), Q = B (weights); out[p][q].
//   * SWAP = true : P = B (weights), Q = A (tokens); out[q][p]. Used when there are few
//     tokens (decode shapes, MoE experts), so that the 128-row MMA dimension is filled by
//     weight rows and the tokens become a narrow MMA N.
//   * GROUPED     : SWAP with per-expert weights B[e] and token rows [off[e], off[e+1]).
//
// Roles (384 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: A/B tiles (128-byte swizzle) and the scales: with tiled
//               scales (SFT) one 2 KB bulk copy per 128 rows and stage, already in the form
//               tcgen05.cp reads; with linear scales, linear [rows][16 B] tiles.
//   warp 1      TMEM allocator and single-thread MMA issuer (tcgen05.cp of scales, then
//               four 128 x BN x 64 block-scaled MMAs per 256-element K stage).
//   warps 2-3   linear scales only: re-layout, alternate stages: turn the TMA'd [rows][16 B]
//               scale tile into the 32-row x 16-byte blocks that tcgen05.cp ... 32x128b.warpx4
//               replicates into the TMEM layout the MMA reads (row r at column base + r/32,
//               byte = k-block). Warp 3 first builds the per-expert tile prefix (grouped).
//   warps 4-11  epilogue, two warpgroups (one per half of the tile's columns; warp w reads
//               TMEM lane quadrant w % 4): TMEM -> registers -> alpha -> bf16 (or fp16, fp32)
//               -> global; with split-K,
//               the cluster's fp32 partials meet in shared memory (st.async over DSMEM)
//               and are summed in a fixed rank order (deterministic); with several
//               clusters per tile, through the workspace in a fixed group order.
// Every wait is bounded (kWaitTimeoutNs); on a timeout the CTA records an error code,
// stops all roles, lets in-flight copies and MMAs land, frees TMEM and exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_core.cuh"

namespace nvfp4 {

// Error codes recorded in the device error word (which wait gave up).
enum : uint32_t {
    kErrProducerEmpty = 0x101,
    kErrSfFull = 0x102,
    kErrMmaAccEmpty = 0x103,
    kErrMmaFull = 0x104,
    kErrMmaSf = 0x105,
    kErrEpiAccFull = 0x106,
    kErrSplitRx = 0x107,
    kErrMmaSfFree = 0x108,
    kErrActqMax = 0x10B,
    kErrMmaActq = 0x10C,
};

// Threads per CTA: warps 0-3 (producer, MMA, scale re-layout) and two epilogue warpgroups.
constexpr int kEpilogueWarps = 8;
constexpr int kGemmThreads = 32 * (4 + kEpilogueWarps);

// Output element types (include/nvfp4.h, nvfp4_out_dtype).
enum : int32_t { kOutBF16 = 0, kOutF16 = 1, kOutF32 = 2 };

struct GemmArgs {
    int32_t M, N;             // output is out[M][N] (row-major, leading dimension N)
    int32_t p_rows, q_rows;   // rows of the P and Q operands (non-grouped)
    int32_t num_kstages;      // K / 256
    int32_t num_p_tiles;      // ceil(p_rows / 128)
    int32_t num_q_tiles;      // ceil(q_rows / BN) (non-grouped)
    int32_t splits;           // split-K factor (non-grouped; 1 = none) = cluster_size * groups
    int32_t cluster_size;     // split-K CTAs per thread-block cluster (reduced over DSMEM)
    int32_t groups;           // clusters per output tile (reduced through the workspace)
    int32_t num_tiles;        // non-grouped: p_tiles * q_tiles * splits
    int32_t band;             // non-grouped: P tiles per rasterisation band (>= 1)
    int32_t narrow_from;      // PAIR, BN = 256: work items from here on are half tiles (see decode_tile)
    void* out;                // out_dtype elements
    int32_t out_dtype;        // kOutBF16, kOutF16 or kOutF32
    const float* alpha;       // [1] or [E]
    float* ws_partial;        // split-K fp32 partial tiles
    uint32_t* ws_counters;    // split-K per-tile arrival counters
    unsigned* err_word;
    const uint8_t* sf_p;      // SFT: tiled scales of the P / Q operands
    const uint8_t* sf_q;
    int32_t sf_kb4;           // SFT: 512-byte scale blocks per 128-row tile (K / 64)
    int32_t sf_8x4;           // linear-path scales in the 8 x 4 layout (1) or row-major (0)
    int32_t b_ready;          // B and its scales are not written by a kernel that may still run
    const int32_t* expert_offsets;  // grouped: [E + 1]
    int32_t num_experts;
    int32_t total_rows;       // grouped: rows of A / out
    const void* act;          // ACTQ: activations A [M, K] (fp32 or bf16), row stride act_ld elements
    int64_t act_ld;
    int32_t act_bf16;
    const float* gs_b;        // ACTQ: the weights' global scale (device, 1)
    float* gs_out;            // ACTQ: optional outputs: A's global scale and alpha (device, 1 each)
    float* alpha_out;
    uint8_t* h_q;             // SWIGLU: NVFP4 codes of h [total_rows, I/2]
    uint8_t* h_sf;            // SWIGLU: e4m3 scales of h [total_rows, I/16]
    const float* gs_h;        // SWIGLU: global scale of h (device, 1)
    int32_t inter;            // SWIGLU: I (gate rows = up rows), N = 2 I
};

template <int BN_, bool SWAP_, bool GROUPED_, bool SFT_ = false, bool SWIGLU_ = false, bool MX_ = false,
          bool PAIR_ = false, bool ACTQ_ = false>
struct GemmCfg {
    static constexpr int BN = BN_;
    static constexpr bool SWAP = SWAP_;
    static constexpr bool GROUPED = GROUPED_;
    // SWIGLU (grouped gate_up only): a P tile holds 64 gate rows and the 64 matching up rows,
    // as four groups of [16 gate rows, 16 up rows] (one 5-D TMA view of the weights), and the
    // epilogue writes h = silu(gate) * up quantised to NVFP4 instead of the product itself.
    static constexpr bool SWIGLU = SWIGLU_;
    static_assert(!SWIGLU || GROUPED, "the fused SwiGLU epilogue serves the grouped gate_up GEMM");
    // MX: MXFP4 operands (one E8M0 scale per 32 K elements, "use_nvfp4=False"), scales in the
    // tiled layout: a stage's 8 scale bytes per row are two 512-byte blocks per 128 rows, each
    // covering 128 K elements; the MMA is the block32 form with UE8M0 scales, and the two
    // 64-wide MMAs of a block read its scale column at byte 0 and byte 2.
    static constexpr bool MX = MX_;
    static constexpr int SF_BLOCKS = MX ? 2 : 4;   // 512-byte scale blocks per stage and 128 rows
    // SFT: both operands' scales in the tiled layout (include/nvfp4.h, NVFP4_SF_TILED): a
    // stage's scales of 128 rows are one contiguous 2 KB run already in the tcgen05.cp source
    // layout, fetched by a bulk copy (no re-layout step). Q tiles then start on a 128-row
    // tile boundary: BN >= 128 a multiple of 128, or a single Q tile (few-token swap).
    static constexpr bool SFT = SFT_;
    static_assert(!SFT || !GROUPED, "tiled scales serve the dense GEMM");
    static_assert(!MX || (SFT && !GROUPED), "MXFP4 serves the dense GEMM with tiled scales");
    // PAIR: the two CTAs of a 2-CTA cluster compute one 256 x BN tile with the 2-SM MMA
    // (cta_group::2, M = 256): CTA r loads P rows [p0 + 128 r, + 128), Q rows
    // [q0 + BN/2 r, + BN/2) and the scales of its P rows and of all BN Q rows; the even CTA
    // issues the MMAs, which read both CTAs' stages, and each CTA's TMEM receives its own 128
    // rows of the tile. For BN = 256 a stage is 38 KB per SM instead of 54 KB for the same MMA
    // work (5 deep); BN = 128 gives 28 KB stages (7 deep) and twice the work items. Every
    // copy's completion is counted on the even CTA's full barrier; its commits release both
    // CTAs' stages and accumulators.
    static constexpr bool PAIR = PAIR_;
    // Grouped pairs (GPAIR): the two CTAs hold 128 weight rows each of a 256-row weight tile
    // pair of one expert and half of its token tile (each CTA loads all the tile's token
    // scales); their linear scales are re-laid out in each CTA, which then signals the even
    // CTA's sfready barrier before the MMA may copy them.
    static constexpr bool GPAIR = PAIR && GROUPED;
    static_assert(!PAIR || (SFT && !SWAP && !GROUPED && (BN == 256 || BN == 128)) ||
                  (GROUPED && SWAP && !SFT && (BN == 128 || BN == 176)),
                  "CTA pairs compute 256 x 256 or 256 x 128 dense tiles, or grouped 256 x 128 / 176 tiles");
    // ACTQ (few-token launches with tiled weight scales): the activations come in as fp32 or
    // bf16 and are quantised inside the kernel. Every CTA of a split-K cluster reads its own K
    // slice of them, the slices' maxima meet over distributed shared memory (the cluster's
    // slices cover all of A: the tensor's global scale without a grid barrier), and each CTA
    // quantises its slice straight into the Q stages in the MMA's swizzled operand layout,
    // with its scales in the tcgen05.cp block layout; the epilogue warps do this before they
    // wait for the accumulator. The CTA's whole K slice fits in the stage ring (kcnt <=
    // STAGES): Q stage ks holds K stage ks for the whole launch.
    static constexpr bool ACTQ = ACTQ_;
    static_assert(!ACTQ || (SWAP && !GROUPED && SFT && !MX && !PAIR && BN <= 64),
                  "in-kernel activation quantisation serves the few-token NVFP4 launches");
    static constexpr int ACTQ_BYTES = ACTQ ? 1024 + 64 + 64 : 0;   // gs / e4m3 table, maxima slots, reduction
    static_assert(!SFT || BN % 128 == 0 || (SWAP && BN <= 64), "Q tiles on 128-row tile boundaries");
    static_assert(!GROUPED || SWAP, "grouped GEMM runs with weights as the MMA M operand");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be 16..256, step 16");

    static constexpr int BM = 128;                 // MMA M
    static constexpr int BK_BYTES = 128;           // 256 fp4 values per K stage
    static constexpr int P_BYTES = BM * BK_BYTES;  // 16 KB
    static constexpr int Q_BYTES = (PAIR ? BN / 2 : BN) * BK_BYTES;   // this CTA's rows of the Q tile
    static constexpr int QG = (BN + 127) / 128;    // 128-row scale groups of the Q tile
    static constexpr int SFP_BYTES = 512 * SF_BLOCKS;   // 128 rows x 16 B (NVFP4) or 8 B (MX)
    static constexpr int SFQ_BYTES = SFP_BYTES * QG;
    static constexpr int SF_TMA_P = BM * 16;       // bytes the scale TMA writes
    static constexpr int SF_TMA_Q = BN * 16;
    static constexpr uint32_t TX_BYTES = P_BYTES + Q_BYTES + SF_TMA_P + SF_TMA_Q;
    static constexpr uint32_t PAIR_TX_BYTES = 2u * (P_BYTES + Q_BYTES + SFP_BYTES + SFP_BYTES * QG);  // both CTAs'
    // PAIR, BN = 256: a half tile (256 x 128) loads half the Q rows and one Q scale group
    static constexpr bool NARROW = PAIR && BN == 256 && !GROUPED;
    static constexpr uint32_t PAIR_TX_NARROW = 2u * (P_BYTES + Q_BYTES / 2 + SFP_BYTES + SFP_BYTES);
    static constexpr int SF_ROWS256 = SFP_BYTES / 256;   // PAIR: a stage's scale run as rows of 256 bytes
    // Grouped: the token tile is loaded in boxes of QBOX rows, only as many as the expert's
    // rows in the tile need (a tile of a 256-wide plan often holds ~128 rows of one expert).
    // (176-row tiles: two boxes of 88, which end exactly at the tile)
    static constexpr int QBOX = BN < 64 ? BN : (BN == 176 ? 88 : 64);
    static_assert(!GROUPED || BN % QBOX == 0, "token boxes tile the token buffer");
    static constexpr int STAGE_BYTES = P_BYTES + Q_BYTES + SFP_BYTES + SFQ_BYTES;

    // TMEM columns: two accumulators, then the scale factors: SFA (4 k-blocks x 4 columns),
    // then SFB (4 k-blocks x 4 columns per 128 Q rows). When two BN = 256 accumulators fill
    // all 512 columns (SF_IN_ACC), a tile's scale factors live in the top SF_COLS columns of
    // the other accumulator instead: the epilogue drains those columns of the previous tile
    // first and signals sf_free, and the MMA warp waits for that before the tile's first
    // tcgen05.cp (by then the previous tile's MMAs have completed, so the copies cannot
    // overwrite scales still being read, and the epilogue overlaps the next tile's MMAs).
    static constexpr int SF_COLS = 4 * SF_BLOCKS * (1 + QG);
    static constexpr int ACC_STAGES = 2;
    static constexpr bool SF_IN_ACC = 2 * BN + SF_COLS > 512;
    static_assert(!SF_IN_ACC || SF_COLS <= 64, "scale columns fit the last 64-column chunk");
    // column of SFA: absolute, or (SF_IN_ACC) relative to the other accumulator
    static constexpr int TMEM_SFA = SF_IN_ACC ? BN - SF_COLS : ACC_STAGES * BN;
    static constexpr int TMEM_USED = SF_IN_ACC ? ACC_STAGES * BN : ACC_STAGES * BN + SF_COLS;
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                   : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");

    static constexpr int SMEM_LIMIT = 232448;      // max dynamic shared memory per block
    // SWIGLU: gs_h / e4m3 table (256 floats), per epilogue warp a 16-token x 8-byte code stage
    // and a 16-byte scale stage
    static constexpr int SWIGLU_BYTES = SWIGLU ? 1024 + kEpilogueWarps * (128 + 16) : 0;
    // split-K receive buffer: this rank's chunk (at most ceil(16 / cs) * 8 rows) from each of
    // cs <= 8 ranks, cs * ceil(16 / cs) * 8 <= 168 rows of [BN + 4] floats. Few-token (swap)
    // launches give it a region of its own (RX_OWN), so that the cluster barrier before the
    // exchange moves into the prologue; other split-K launches reuse the drained stage ring.
    static constexpr int PSTRIDE = BN + 4;
    static constexpr bool RX_OWN = SWAP && !GROUPED;
    static constexpr int RX_BYTES = RX_OWN ? ((168 * PSTRIDE * 4 + 1023) & ~1023) : 0;
    static constexpr int MISC_BYTES = 1024 + (GROUPED ? 4 * (kMaxExperts + 1) : 0) + SWIGLU_BYTES + RX_BYTES +
                                      ACTQ_BYTES;
    static constexpr int ALIGN_SLACK = 1024;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - MISC_BYTES - ALIGN_SLACK) / STAGE_BYTES;
    // Few-token (swap, non-grouped) launches split K finely and run a handful of stages per
    // CTA: four buffers suffice and leave room on the SM for the neighbouring kernels' blocks.
    static constexpr int STAGE_CAP = (SWAP && !GROUPED) ? 4 : 12;
    static constexpr int STAGES = STAGES_FIT > STAGE_CAP ? STAGE_CAP : STAGES_FIT;
    static_assert(STAGES >= 2, "pipeline depth");

    // Shared memory layout (offsets from a 1024-byte aligned base).
    static constexpr int OFF_P = 0;
    static constexpr int OFF_Q = OFF_P + STAGES * P_BYTES;
    static constexpr int OFF_SFP = OFF_Q + STAGES * Q_BYTES;
    static constexpr int OFF_SFQ = OFF_SFP + STAGES * SFP_BYTES;
    static constexpr int OFF_BAR = OFF_SFQ + STAGES * SFQ_BYTES;
    // barriers: full, sfready, empty [STAGES]; acc_full, acc_empty [2]; mma_done; split-K rx;
    // sf_free [2]; activations quantised, slice maxima received (ACTQ); GPAIR: this CTA's
    // scales landed [STAGES]
    static constexpr int NUM_BARS = 4 * STAGES + 10;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;     // tmem base, flags
    static constexpr int OFF_PREFIX = OFF_MISC + 64;
    static constexpr int OFF_SWIGLU = OFF_PREFIX + (GROUPED ? ((4 * (kMaxExperts + 1) + 15) & ~15) : 0);
    static constexpr int OFF_RX = (OFF_SWIGLU + SWIGLU_BYTES + 1023) & ~1023;
    static constexpr int OFF_ACTQ = OFF_RX + RX_BYTES;
    static constexpr int SMEM_BYTES = OFF_ACTQ + ACTQ_BYTES + ALIGN_SLACK;
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
    static_assert(RX_OWN || 168 * PSTRIDE * 4 <= STAGES * STAGE_BYTES, "split-K receive buffer fits the pipeline buffers");
    static_assert(OFF_Q % 1024 == 0 && OFF_SFP % 1024 == 0, "swizzle atoms need 1 KB alignment");
};

// One unit of work: a 128-row P tile x a BN-row Q tile over a range of K stages.
struct Tile {
    int32_t p0;        // first P row (within the expert for grouped)
    int32_t q0;        // first Q row (global row of A for grouped)
    int32_t k0;        // first K stage
    int32_t kcnt;      // number of K stages
    int32_t pq;        // index of the output tile (split-K counter slot)
    int32_t split;     // split index
    int32_t expert;    // grouped: expert id
    int32_t q_valid;   // grouped: valid Q rows in this tile (<= BN)
    int32_t q_span;    // Q rows (MMA N) of the tile: BN, or BN / 2 for a half tile
};

// Row range of expert e, clamped to [0, total_rows] and made non-decreasing, so that
// malformed offsets can only shrink the work, never index outside A or out.
__device__ __forceinline__ void expert_rows(const GemmArgs& a, int e, int32_t& r0, int32_t& rows)
{
    const int32_t lo = min(max(a.expert_offsets[e], 0), a.total_rows);
    const int32_t hi = min(max(a.expert_offsets[e + 1], lo), a.total_rows);
    r0 = lo;
    rows = hi - lo;
}

template <class Cfg>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, int32_t t, const int32_t* prefix)
{
    Tile ti;
    if constexpr (Cfg::GROUPED) {
        // expert e: largest e with prefix[e] <= t (empty experts have prefix[e] == prefix[e+1])
        int lo = 0, hi = a.num_experts;       // invariant: prefix[lo] <= t < prefix[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix[mid] <= t) lo = mid; else hi = mid;
        }
        const int e = lo;
        int32_t r0, rows;
        expert_rows(a, e, r0, rows);
        const int32_t qt_count = (rows + Cfg::BN - 1) / Cfg::BN;
        const int32_t local = t - prefix[e];
        const int32_t pt = local / qt_count;
        const int32_t qt = local - pt * qt_count;
        // GPAIR: pt counts 256-row weight tile pairs; this CTA's half
        if constexpr (Cfg::PAIR) ti.p0 = (2 * pt + static_cast<int32_t>(cluster_ctarank())) * Cfg::BM;
        else ti.p0 = pt * Cfg::BM;
        ti.q0 = r0 + qt * Cfg::BN;
        ti.q_valid = min(Cfg::BN, rows - qt * Cfg::BN);
        ti.q_span = Cfg::BN;
        ti.k0 = 0;
        ti.kcnt = a.num_kstages;
        ti.pq = 0;
        ti.split = 0;
        ti.expert = e;
    } else {
        // PAIR, BN = 256: items from narrow_from on split the last output tiles in two halves
        // of 128 columns each (a last wave of tiles shorter than a full one fills twice as
        // many SMs for half as long): item narrow_from + 2 j + h is half h of tile narrow_from + j.
        int32_t half = -1;
        if constexpr (Cfg::NARROW) {
            if (t >= a.narrow_from) {
                half = (t - a.narrow_from) & 1;
                t = a.narrow_from + ((t - a.narrow_from) >> 1);
            }
        }
        const int32_t split = t % a.splits;
        const int32_t pq = t / a.splits;
        // Output tiles in bands of `band` P tiles: column by column (Q tile) within a band, P
        // tile fastest, so that the tiles in flight at once share a few A and B panels in L2.
        const int32_t per_band = a.band * a.num_q_tiles;
        const int32_t b = pq / per_band;
        const int32_t in_band = pq - b * per_band;
        const int32_t width = min(a.band, a.num_p_tiles - b * a.band);
        const int32_t qt = in_band / width;
        const int32_t pt = b * a.band + (in_band - qt * width);
        const int32_t base = a.num_kstages / a.splits;
        const int32_t rem = a.num_kstages % a.splits;
        if constexpr (Cfg::PAIR) ti.p0 = (2 * pt + static_cast<int32_t>(cluster_ctarank())) * Cfg::BM;
        else ti.p0 = pt * Cfg::BM;
        ti.q0 = qt * Cfg::BN + (half > 0 ? Cfg::BN / 2 : 0);
        ti.q_span = half >= 0 ? Cfg::BN / 2 : Cfg::BN;
        ti.k0 = split * base + min(split, rem);
        ti.kcnt = base + (split < rem ? 1 : 0);
        ti.pq = pq;
        ti.split = split;
        ti.expert = 0;
        ti.q_valid = min(ti.q_span, a.q_rows - ti.q0);
    }
    return ti;
}

__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t nthreads, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Two fp32 values -> one 32-bit word of the 16-bit output type (round to nearest even),
// `lo` in the low half.
__device__ __forceinline__ uint32_t pack_out16x2(float lo, float hi, int32_t dt)
{
    return dt == kOutF16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

// out[idx] = alpha * v in the output type (one element).
__device__ __forceinline__ void store_out1(const GemmArgs& a, size_t idx, float v)
{
    if (a.out_dtype == kOutF32) static_cast<float*>(a.out)[idx] = v;
    else if (a.out_dtype == kOutF16) static_cast<__half*>(a.out)[idx] = __float2half_rn(v);
    else static_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(v);
}

// Eight consecutive output elements out[idx .. idx + 7] = v[0..7] (idx % 8 == 0): one 16-byte
// store for 16-bit types, two for fp32.
__device__ __forceinline__ void store_out8(const GemmArgs& a, size_t idx, const float (&v)[8])
{
    if (a.out_dtype == kOutF32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + idx);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        const int32_t dt = a.out_dtype;
        uint4 w;
        w.x = pack_out16x2(v[0], v[1], dt);
        w.y = pack_out16x2(v[2], v[3], dt);
        w.z = pack_out16x2(v[4], v[5], dt);
        w.w = pack_out16x2(v[6], v[7], dt);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + idx) = w;
    }
}

// Store 16 consecutive accumulator columns (c .. c + 15) of P row `p` as alpha * v in the
// output type.
template <class Cfg>
__device__ __forceinline__ void store_out16(const GemmArgs& a, const Tile& ti, int p, int c,
                                            const uint32_t (&r)[16], float alpha)
{
    if constexpr (!Cfg::SWAP) {
        // thread owns output row m = p, columns n = q0 + c .. + 15 (N % 8 == 0)
        const int n0 = ti.q0 + c;
        if (p < a.M) {
            const size_t idx = static_cast<size_t>(p) * a.N + n0;
            float v[2][8];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j >> 3][j & 7] = alpha * __uint_as_float(r[j]);
            if (n0 < a.N) store_out8(a, idx, v[0]);
            if (n0 + 8 < a.N) store_out8(a, idx + 8, v[1]);
        }
    } else {
        // thread owns output column n = p; accumulator columns are output rows
        const int n = p;
        if (n < a.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int qi = c + j;
                bool valid;
                if constexpr (Cfg::GROUPED) valid = qi < ti.q_valid;
                else valid = ti.q0 + qi < a.M;
                if (valid)
                    store_out1(a, static_cast<size_t>(ti.q0 + qi) * a.N + n, alpha * __uint_as_float(r[j]));
            }
        }
    }
}

// An 8 x 8 transpose of 16-bit elements within each group of 8 lanes: lane 8 g + j enters
// with elements 0..7 of row j (w[k] = elements 2k, 2k+1, the lower one in the low half) and
// leaves with element j of rows 0..7 in the same packing. Three butterfly stages (lane bit m =
// 4, 2, 1): each lane hands its partner (lane ^ m) the four elements it is about to replace
// and puts the four it receives at their index ^ m.
__device__ __forceinline__ void transpose8x8_b16(uint32_t (&w)[4], int lane)
{
    const int j = lane & 7;
    {   // m = 4: whole words 2, 3 <-> 0, 1
        const bool hb = (j & 4) != 0;
        const uint32_t s0 = hb ? w[0] : w[2], s1 = hb ? w[1] : w[3];
        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 4), r1 = __shfl_xor_sync(0xffffffffu, s1, 4);
        if (hb) { w[0] = r0; w[1] = r1; } else { w[2] = r0; w[3] = r1; }
    }
    {   // m = 2: words 1, 3 <-> 0, 2
        const bool hb = (j & 2) != 0;
        const uint32_t s0 = hb ? w[0] : w[1], s1 = hb ? w[2] : w[3];
        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 2), r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
        if (hb) { w[0] = r0; w[2] = r1; } else { w[1] = r0; w[3] = r1; }
    }
    {   // m = 1: high halves (odd elements) <-> low halves (even elements)
        const bool hb = (j & 1) != 0;
        const uint32_t sel = hb ? 0x5410u : 0x7632u;
        const uint32_t s0 = __byte_perm(w[0], w[1], sel), s1 = __byte_perm(w[2], w[3], sel);
        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
        if (hb) {
            w[0] = __byte_perm(w[0], r0, 0x3254u);
            w[1] = __byte_perm(w[1], r0, 0x3276u);
            w[2] = __byte_perm(w[2], r1, 0x3254u);
            w[3] = __byte_perm(w[3], r1, 0x3276u);
        } else {
            w[0] = __byte_perm(w[0], r0, 0x5410u);
            w[1] = __byte_perm(w[1], r0, 0x7610u);
            w[2] = __byte_perm(w[2], r1, 0x5410u);
            w[3] = __byte_perm(w[3], r1, 0x7610u);
        }
    }
}

// Weights-as-M (swap, grouped) epilogue for 16-bit outputs: the warp holds 32 P rows (its lanes:
// output columns p0 + 32 quad + lane) x 16 accumulator columns c .. c + 15 (output rows, one per
// token). Scaled, rounded and packed, each 8 x 8 block is transposed within its group of 8
// lanes, so that lane 8 g + i holds token c + 8 b + i's output columns p0 + 32 quad + 8 g .. + 7:
// one 16-byte store per lane and block, 64 contiguous bytes per token row and warp.
template <class Cfg>
__device__ __forceinline__ void store_tok16(const GemmArgs& a, const Tile& ti, int quad, int lane, int c,
                                            const uint32_t (&r)[16], float alpha)
{
    const int32_t dt = a.out_dtype;
    uint32_t w[2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[b][k] = pack_out16x2(alpha * __uint_as_float(r[8 * b + 2 * k]),
                                   alpha * __uint_as_float(r[8 * b + 2 * k + 1]), dt);
    transpose8x8_b16(w[0], lane);
    transpose8x8_b16(w[1], lane);
    const int n = ti.p0 + 32 * quad + 8 * (lane >> 3);      // 8 output columns; N % 8 == 0
    if (n >= a.N) return;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const int qi = c + 8 * b + (lane & 7);
        bool valid;
        if constexpr (Cfg::GROUPED) valid = qi < ti.q_valid;
        else valid = ti.q0 + qi < a.M;
        if (valid)
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + static_cast<size_t>(ti.q0 + qi) * a.N + n) =
                make_uint4(w[b][0], w[b][1], w[b][2], w[b][3]);
    }
}

// An 8 x 8 transpose of 16-byte chunks within each group of 8 lanes (three butterfly stages of
// shuffles: at stage m the lanes whose bit m differs from the chunk index's swap those
// chunks): lane 8 g + j enters with chunks 0..7 of its own row and leaves with chunk j of
// rows 8 g .. 8 g + 7 (w[t] = row 8 g + t).
__device__ __forceinline__ void transpose_chunks8(uint32_t (&w)[8][4], int lane)
{
    const int j = lane & 7;
#pragma unroll
    for (int m = 4; m >= 1; m >>= 1) {
        const bool hi = (j & m) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (e & m) continue;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t send = hi ? w[e][k] : w[e ^ m][k];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
                if (hi) w[e][k] = recv;
                else w[e ^ m][k] = recv;
            }
        }
    }
}

// Stores 64 accumulator columns (c0 .. c0 + 63) of the 32 rows a warp holds (lane = row,
// non-swap tiles) as alpha * v in the output type, each store instruction writing 4 rows x 128
// contiguous bytes. A lane's row is cut into 16-byte chunks (8 columns of a 16-bit type, 4 of
// fp32); after transpose_chunks8, lanes 8 g .. 8 g + 7 write one 128-byte row segment together.
// (Stores straight from the row-per-lane layout would touch 32 lines per instruction.)
template <class Cfg>
__device__ __forceinline__ void store_rows64(const GemmArgs& a, const Tile& ti, int quad, int lane, int c0,
                                             const uint32_t (&r)[4][16], float alpha)
{
    const int j = lane & 7;
    const int m0 = ti.p0 + 32 * quad + (lane & ~7);
    uint32_t w[8][4];
    if (a.out_dtype == kOutF32) {
        // two halves of 32 columns, 8 chunks of 4 fp32 each
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    w[e][k] = __float_as_uint(alpha * __uint_as_float(r[2 * h + (e >> 2)][(e & 3) * 4 + k]));
            transpose_chunks8(w, lane);
            const int n = ti.q0 + c0 + 32 * h + 4 * j;
            if (n < a.N) {
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const int m = m0 + t;
                    if (m < a.M)
                        *reinterpret_cast<uint4*>(static_cast<float*>(a.out) + static_cast<size_t>(m) * a.N + n) =
                            make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
                }
            }
        }
        return;
    }
    const int32_t dt = a.out_dtype;
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[e][k] = pack_out16x2(alpha * __uint_as_float(r[e >> 1][(e & 1) * 8 + 2 * k]),
                                   alpha * __uint_as_float(r[e >> 1][(e & 1) * 8 + 2 * k + 1]), dt);
    transpose_chunks8(w, lane);
    const int n = ti.q0 + c0 + 8 * j;
    if (n < a.N) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int m = m0 + t;
            if (m < a.M)
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + static_cast<size_t>(m) * a.N + n) =
                    make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
        }
    }
}

// Rows [chunk_begin(k), chunk_begin(k + 1)) of a 128-row tile belong to cluster rank k:
// whole 8-row groups, as evenly as possible (at most ceil(16 / cs) * 8 rows per rank).
__device__ __forceinline__ int chunk_begin(int k, int cs) { return ((k * 16 + cs - 1) / cs) * 8; }
// The rank whose chunk holds `row`.
__device__ __forceinline__ int chunk_owner(int row, int cs) { return ((row >> 3) * cs) >> 4; }

// Writes a reduced chunk of a tile: rows [r0, r0 + rows) of the 128 x BN accumulator tile,
// each the in-order sum of `nsrc` fp32 copies in shared memory (copy j, chunk row lr, column
// c at src[(j * rows + lr) * PSTRIDE + c]), times alpha, in the output type. All 128 epilogue
// threads (tid) take part; each writes 8 consecutive outputs (16 bytes, or 32 for fp32) and
// consecutive threads write consecutive addresses.
template <class Cfg>
__device__ __forceinline__ void store_chunk(const GemmArgs& a, const Tile& ti, const float* src, int nsrc,
                                            int r0, int rows, int tid, float alpha)
{
    constexpr int BN = Cfg::BN;
    constexpr int PS = Cfg::PSTRIDE;
    if constexpr (!Cfg::SWAP) {
        // item = (chunk row lr, 8-column group c8); output row p0 + r0 + lr, columns q0 + 8 c8
        constexpr int G = BN / 8;
        for (int item = tid; item < rows * G; item += 128) {
            const int lr = item / G;
            const int c = (item % G) * 8;
            float v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) v[t] = 0.0f;
            for (int j = 0; j < nsrc; ++j) {
                const float* s = src + (j * rows + lr) * PS + c;
                const float4 x0 = *reinterpret_cast<const float4*>(s);
                const float4 x1 = *reinterpret_cast<const float4*>(s + 4);
                v[0] += x0.x; v[1] += x0.y; v[2] += x0.z; v[3] += x0.w;
                v[4] += x1.x; v[5] += x1.y; v[6] += x1.z; v[7] += x1.w;
            }
            const int m = ti.p0 + r0 + lr;
            const int n0 = ti.q0 + c;
            if (m < a.M && n0 < a.N) {
#pragma unroll
                for (int t = 0; t < 8; ++t) v[t] *= alpha;
                store_out8(a, static_cast<size_t>(m) * a.N + n0, v);
            }
        }
    } else {
        // item = (accumulator column c, 8-row group g); output row q0 + c, columns
        // p0 + r0 + 8 g .. + 7 (chunk rows are weight rows, i.e. output columns)
        const int G = rows >> 3;
        for (int item = tid; item < BN * G; item += 128) {
            const int c = item / G;
            const int lr = (item - c * G) * 8;
            float v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) v[t] = 0.0f;
            for (int j = 0; j < nsrc; ++j) {
                const float* s = src + (j * rows + lr) * PS + c;
#pragma unroll
                for (int t = 0; t < 8; ++t) v[t] += s[t * PS];
            }
            const int m = ti.q0 + c;
            const int n0 = ti.p0 + r0 + lr;
            if (m < a.M && n0 < a.N) {
#pragma unroll
                for (int t = 0; t < 8; ++t) v[t] *= alpha;
                store_out8(a, static_cast<size_t>(m) * a.N + n0, v);
            }
        }
    }
}

// SwiGLU + NVFP4 epilogue of 16 accumulator columns (tokens c .. c + 15 of the tile) in one
// warp of TMEM lane quadrant `quad`: P rows 32 quad + i (i < 16) are gate row j0 + 16 quad + i
// and P rows 32 quad + 16 + i the up row of the same index (j0 = p0 / 2), so that lane i and
// lane 16 + i hold g and u of intermediate index j = j0 + 16 quad + i, and each half-warp's 16
// indices are one NVFP4 block of h. After one exchange lane i (i < 16) holds (g, u) of tokens
// c .. c + 7 and lane 16 + i those of tokens c + 8 .. c + 15:
//     g, u = alpha * acc;   h = (g / (1 + exp(-g))) * u     (fp32, CUDA's expf)
// then the quantiser's steps for the 16 values of a token (a half-warp), with the fixed
// global scale gs_h, in fp32 with explicit rounding and in this order:
//     amax -> s = e4m3(amax / 6 * gs_h) -> r = s ? gs_h / s : 0 -> codes e2m1(h * r)
// (rcp_tab[s] = gs_h / e4m3(s), as the quantiser builds it). Codes go through the warp's
// stage (16 tokens x 8 bytes) and leave as one 8-byte store per token; the scale as one byte.
template <class Cfg>
__device__ __forceinline__ void swiglu_chunk16(const GemmArgs& a, const Tile& ti, int quad, int lane, int c,
                                               const uint32_t (&r)[16], float alpha, float gsh,
                                               const float* rcp_tab, uint8_t* stage, uint8_t* sstage)
{
    const bool up = lane >= 16;
    const int i = lane & 15;
    float h[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        const float lo = alpha * __uint_as_float(r[cc]);        // token c + cc
        const float hi = alpha * __uint_as_float(r[cc + 8]);    // token c + 8 + cc
        const float other = __shfl_xor_sync(0xffffffffu, up ? lo : hi, 16);
        const float g = up ? other : lo;
        const float u = up ? hi : other;
        h[cc] = (g / (1.0f + expf(-g))) * u;
    }
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        float amax = fabsf(h[cc]);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const uint32_t sfq = f32_to_e4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gsh));
        const uint32_t code = f32x2_to_e2m1x2(__fmul_rn(h[cc], rcp_tab[sfq]), 0.0f) & 0xFu;
        const uint32_t hi_code = __shfl_xor_sync(0xffffffffu, code, 1);
        const int tok = cc + (up ? 8 : 0);
        if ((i & 1) == 0) stage[tok * 8 + (i >> 1)] = static_cast<uint8_t>(code | (hi_code << 4));
        if (i == 0) sstage[tok] = static_cast<uint8_t>(sfq);
    }
    __syncwarp();
    if (lane < 16) {
        const int tok = c + lane;
        if (tok < ti.q_valid) {
            const size_t row = static_cast<size_t>(ti.q0 + tok);
            const int blk = (ti.p0 >> 5) + quad;          // 16-element block of h: j0 / 16 + quad
            *reinterpret_cast<uint2*>(a.h_q + row * (a.inter >> 1) + blk * 8) =
                *reinterpret_cast<const uint2*>(stage + lane * 8);
            a.h_sf[row * (a.inter >> 4) + blk] = sstage[lane];
        }
    }
    __syncwarp();
}

// 32-bit asynchronous store into a cluster peer's shared memory, completion counted (bytes) on
// the peer's mbarrier; both addresses from mapa.
__device__ __forceinline__ void st_async_u32(uint32_t remote_addr, uint32_t v, uint32_t remote_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                 ::"r"(remote_addr), "r"(v), "r"(remote_bar)
                 : "memory");
}

// ACTQ: quantises this CTA's K slice of the activations into its Q stages (run by the 256
// epilogue threads, e = 0 .. 255, before the epilogue proper). Returns alpha = 1 / (gs_A gs_B),
// or a negative value if a wait gave up. The steps and fp32 operations are the quantiser's
// (nvfp4_quantize_dynamic): the global scale from the maximum over all of A, then per 16-element
// block amax -> s = e4m3(amax / 6 * gs) -> r = gs / e4m3(s) (table) -> codes e2m1(x * r).
// Vector v (8 elements) of the slice: token row v / (kcnt 32), K stage (v / 32) % kcnt, element
// 8 (v % 32) of the stage; lanes 2j, 2j + 1 hold one 16-element block.
template <class Cfg, typename T>
__device__ __forceinline__ float actq_quantize_t(const GemmArgs& a, uint8_t* smem, int k0, int kcnt, int e,
                                                 uint64_t* amax_bar, const AbortState& ab)
{
    using Raw = typename InTraits<T>::Raw;
    constexpr int U = 4;                                       // loads in flight per thread
    const T* x = static_cast<const T*>(a.act);
    const int M = a.M;
    const uint32_t per_row = static_cast<uint32_t>(kcnt) * 32u;
    const uint32_t nvec = static_cast<uint32_t>(M) * per_row;
    float* rcp_tab = reinterpret_cast<float*>(smem + Cfg::OFF_ACTQ);
    float* slots = reinterpret_cast<float*>(smem + Cfg::OFF_ACTQ + 1024);
    float* red = reinterpret_cast<float*>(smem + Cfg::OFF_ACTQ + 1024 + 64);
    auto load = [&](uint32_t v) -> Raw {
        if (v >= nvec) return InTraits<T>::zero();
        const uint32_t r = v / per_row, w = v - r * per_row;
        const int64_t k = (static_cast<int64_t>(k0) + (w >> 5)) * 256 + (w & 31) * 8;
        return InTraits<T>::load(x + static_cast<int64_t>(r) * a.act_ld + k);
    };

    // zero the slice's Q stages (padding token rows stay zero) while the first loads fly
    {
        uint4* q = reinterpret_cast<uint4*>(smem + Cfg::OFF_Q);
        for (int i = e; i < kcnt * Cfg::Q_BYTES / 16; i += 256) q[i] = make_uint4(0u, 0u, 0u, 0u);
        uint4* sq = reinterpret_cast<uint4*>(smem + Cfg::OFF_SFQ);
        for (int i = e; i < kcnt * Cfg::SFQ_BYTES / 16; i += 256) sq[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    // 1. the slice's maximum
    float m = 0.0f;
    for (uint32_t v0 = e; v0 < nvec; v0 += 256 * U) {
        Raw raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) raw[u] = load(v0 + 256 * u);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float vals[8];
            InTraits<T>::decode(raw[u], vals);
#pragma unroll
            for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(vals[k]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((e & 31) == 0) red[e >> 5] = m;
    named_bar_sync(1, 256);
    // 2. the cluster's maxima: every CTA's slice together is all of A
    const int cs = a.cluster_size;
    bool ok = true;
    if (e == 0) {
        float cm = 0.0f;
        for (int w = 0; w < 8; ++w) cm = fmaxf(cm, red[w]);
        const uint32_t rank = cs > 1 ? cluster_ctarank() : 0u;
        slots[rank] = cm;
        if (cs > 1) {
            for (int pr = 0; pr < cs; ++pr) {
                if (pr == static_cast<int>(rank)) continue;
                st_async_u32(mapa_shared(smem_u32(&slots[rank]), static_cast<uint32_t>(pr)), __float_as_uint(cm),
                             mapa_shared(smem_u32(amax_bar), static_cast<uint32_t>(pr)));
            }
            mbar_arrive_expect_tx(amax_bar, static_cast<uint32_t>((cs - 1) * 4));
            ok = mbar_wait(amax_bar, 0, ab, kErrActqMax);
        }
    }
    ok = named_bar_and(1, 256, ok);
    if (!ok) return -1.0f;
    float amax = 0.0f;
    for (int r = 0; r < cs; ++r) amax = fmaxf(amax, slots[r]);
    const float gs = (amax == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, amax);
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(gs, __ldg(a.gs_b)));
    {
        const float sfd = e4m3_to_f32(static_cast<uint32_t>(e));
        rcp_tab[e] = (sfd == 0.0f) ? 0.0f : __fdiv_rn(gs, sfd);
    }
    if (blockIdx.x == 0 && e == 0) {
        if (a.gs_out) *a.gs_out = gs;
        if (a.alpha_out) *a.alpha_out = alpha;
    }
    named_bar_sync(1, 256);
    // 3. codes and block scales into the Q stages: the warp takes 32 consecutive vectors
    //    (lanes 2j, 2j + 1 share a 16-element block), U groups of them per round
    const int lane = e & 31;
    for (uint32_t w0 = static_cast<uint32_t>(e & ~31); w0 < nvec; w0 += 256 * U) {   // warp-uniform
        Raw raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) raw[u] = load(w0 + 256 * u + lane);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t vb = w0 + 256 * u;
            if (vb >= nvec) break;                             // warp-uniform (nvec % 32 == 0)
            const uint32_t v = vb + lane;
            float vals[8];
            InTraits<T>::decode(raw[u], vals);
            float bm = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) bm = fmaxf(bm, fabsf(vals[k]));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
            const uint32_t sfq = f32_to_e4m3(__fmul_rn(__fdiv_rn(bm, 6.0f), gs));
            const uint32_t packed = scale_to_e2m1x8(vals, rcp_tab[sfq]);
            const uint32_t r = v / per_row, w = v - r * per_row;
            const uint32_t st = w >> 5, uu = w & 31;
            const uint32_t kbyte = uu * 4;                     // 4 code bytes per vector
            uint8_t* qs = smem + Cfg::OFF_Q + st * Cfg::Q_BYTES + r * 128;
            *reinterpret_cast<uint32_t*>(qs + ((((kbyte >> 4) ^ (r & 7u)) << 4) | (kbyte & 15u))) = packed;
            if ((uu & 1u) == 0) {
                const uint32_t kb = uu >> 1;                   // 16-element block of the stage
                smem[Cfg::OFF_SFQ + st * Cfg::SFQ_BYTES + (kb >> 2) * 512 + (r & 31u) * 16 + ((r >> 5) & 3u) * 4 +
                     (kb & 3u)] = static_cast<uint8_t>(sfq);
            }
        }
    }
    fence_proxy_async_smem();                                  // generic writes -> tensor core reads
    named_bar_sync(1, 256);
    return alpha;
}

// Split-K epilogue of one CTA, run by the 128 threads of the first epilogue warpgroup
// (thread = accumulator row; named barrier 2);
// every CTA of a split-K launch owns exactly one tile. The `cluster_size` CTAs of a cluster
// hold consecutive K slices of the same output tile, and row chunk k is reduced by cluster
// rank k. Once the receive buffers may be written (a region of their own: since the
// prologue's cluster barrier; otherwise after a cluster barrier here, when every CTA of the
// cluster has drained its main loop) each thread copies its accumulator row, straight from
// TMEM through registers, into slot `rank` of the owning rank's receive buffer
// [cs][my_rows][PSTRIDE]: st.async to a peer (completion counted in bytes on the peer's rx
// barrier), a plain store for its own chunk. Once the peers' bytes have landed all 128
// threads sum the chunk over the slots in rank order (fixed, deterministic) and write it as
// bf16. With `groups` > 1 clusters per tile the fp32 chunk goes to the workspace instead,
// and the last of the `groups` CTAs holding the same chunk (arrival counter) sums the
// chunks in group order.
template <class Cfg>
__device__ __forceinline__ void split_k_epilogue(const GemmArgs& a, const Tile& ti, uint8_t* smem,
                                                 uint64_t* rx_bar, volatile int* s_is_last,
                                                 uint32_t tacc, int row, float alpha,
                                                 const AbortState& ab)
{
    constexpr int BN = Cfg::BN;
    constexpr int PS = Cfg::PSTRIDE;
    const int cs = a.cluster_size;
    const int g = a.groups;
    const int rank = cs > 1 ? static_cast<int>(cluster_ctarank()) : 0;
    const int owner = chunk_owner(row, cs);
    float* rx = reinterpret_cast<float*>(smem + (Cfg::RX_OWN ? Cfg::OFF_RX : Cfg::OFF_P));
    // the receive buffer aliases the stage ring: wait until every CTA of the cluster has drained
    // its main loop (with a region of its own, the prologue's cluster barrier covered it)
    if (!Cfg::RX_OWN && cs > 1) { cluster_arrive(); cluster_wait(); }

    const int my0 = chunk_begin(rank, cs);
    const int my_rows = chunk_begin(rank + 1, cs) - my0;
    const int grp = ti.split / cs;
    const bool is_owner = owner == rank;
    const int own0 = chunk_begin(owner, cs);
    const int own_rows = chunk_begin(owner + 1, cs) - own0;

    // 1. every row to slot `rank` of its owner's receive buffer. tcgen05.ld is .sync.aligned:
    //    every lane of the warp executes every load, only the destination depends on the row.
    {
        float* mine = rx + (rank * own_rows + (row - own0)) * PS;        // in the owner's buffer
        const uint32_t dst = cs > 1 ? mapa_shared(smem_u32(mine), static_cast<uint32_t>(owner)) : 0u;
        const uint32_t bar = cs > 1 ? mapa_shared(smem_u32(rx_bar), static_cast<uint32_t>(owner)) : 0u;
        for (int c = 0; c < BN; c += 16) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(tacc + c, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 f = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                             __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                if (is_owner) *reinterpret_cast<float4*>(mine + c + 4 * i) = f;
                else st_async_f4(dst + (c + 4 * i) * 4, f.x, f.y, f.z, f.w, bar);
            }
        }
    }
    // 2. wait (all epilogue threads, bounded) for the other ranks' copies of this CTA's rows;
    //    the named barrier publishes the own-slot rows to all 128 threads
    bool ok = true;
    if (cs > 1) {
        if (row == my0)
            mbar_arrive_expect_tx(rx_bar, static_cast<uint32_t>((cs - 1) * my_rows * BN * 4));
        ok = mbar_wait(rx_bar, 0, ab, kErrSplitRx);
    }
    __syncwarp();
    ok = named_bar_and(2, 128, ok);
    if (!ok) return;

    // 3. reduce over the ranks in order
    if (g == 1) {
        store_chunk<Cfg>(a, ti, rx, cs, my0, my_rows, row, alpha);
        return;
    }
    float* chunk_ws = a.ws_partial + (static_cast<size_t>(ti.pq) * g + grp) * (128 * BN)
                    + static_cast<size_t>(my0) * BN;
    for (int item = row; item < my_rows * (BN / 4); item += 128) {
        const int lr = item / (BN / 4);
        const int c = (item % (BN / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < cs; ++k) {
            const float4 f = *reinterpret_cast<const float4*>(rx + (k * my_rows + lr) * PS + c);
            v.x += f.x; v.y += f.y; v.z += f.z; v.w += f.w;
        }
        __stcg(reinterpret_cast<float4*>(chunk_ws + lr * BN + c), v);
    }

    // groups > 1: the last of the `groups` CTAs that hold chunk `rank` of this tile sums the
    // chunks from the workspace in group order (into receive slot 0), then stores them
    __threadfence();
    __syncwarp();
    named_bar_sync(2, 128);
    uint32_t* counter = a.ws_counters + static_cast<size_t>(ti.pq) * cs + rank;
    if (row == 0) {
        const uint32_t prev = atomicAdd(counter, 1u);
        *s_is_last = (prev == static_cast<uint32_t>(g - 1)) ? 1 : 0;
    }
    __syncwarp();
    named_bar_sync(2, 128);
    if (!*s_is_last) return;
    __threadfence();
    const float* tile_ws = a.ws_partial + static_cast<size_t>(ti.pq) * g * (128 * BN)
                         + static_cast<size_t>(my0) * BN;
    for (int item = row; item < my_rows * (BN / 4); item += 128) {
        const int lr = item / (BN / 4);
        const int c = (item % (BN / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < g; ++j) {
            const float4 f = __ldcg(reinterpret_cast<const float4*>(
                tile_ws + static_cast<size_t>(j) * (128 * BN) + lr * BN + c));
            v.x += f.x; v.y += f.y; v.z += f.z; v.w += f.w;
        }
        *reinterpret_cast<float4*>(rx + lr * PS + c) = v;
    }
    __syncwarp();
    named_bar_sync(2, 128);
    store_chunk<Cfg>(a, ti, rx, 1, my0, my_rows, row, alpha);
    if (row == 0) *counter = 0u;             // re-arm for the next call
}

// Copies of one stage of a dense tiled-scale tile (SFT, single CTA) into ring slot `stage`,
// all completing on that slot's full barrier: part 1 = the weight operand (B: Q, or P when the
// weights are the MMA M operand) and its scales, after arming the barrier for the whole
// stage; part 2 = the activation operand (A) and its scales; part 3 = both. The stage's scale
// blocks of each 128-row tile are one contiguous run (2 KB, MX 1 KB); only the Q row tiles that
// exist are fetched (the last Q tile may end past the rows). ACTQ: the weights only (the
// epilogue warps fill the Q stages).
template <class Cfg>
__device__ __forceinline__ void sft_stage_copies(const GemmArgs& a, const Tile& ti, int32_t ks, uint32_t stage,
                                                 uint8_t* smem, const CUtensorMap* tm_p, const CUtensorMap* tm_q,
                                                 uint64_t* full_bar, int part)
{
    constexpr int QG = Cfg::QG;
    const uint64_t pol_stream = l2_policy_evict_first();  // weights: read once
    const uint64_t pol_keep = l2_policy_evict_last();     // activations: re-read
    const uint64_t pol_p = Cfg::SWAP ? pol_stream : pol_keep;
    const uint64_t pol_q = Cfg::SWAP ? pol_keep : pol_stream;
    uint64_t* fb = &full_bar[stage];
    const int32_t kx = (ti.k0 + ks) * Cfg::BK_BYTES;
    uint8_t* pbuf = smem + Cfg::OFF_P + stage * Cfg::P_BYTES;
    uint8_t* qbuf = smem + Cfg::OFF_Q + stage * Cfg::Q_BYTES;
    uint8_t* sfpb = smem + Cfg::OFF_SFP + stage * Cfg::SFP_BYTES;
    uint8_t* sfqb = smem + Cfg::OFF_SFQ + stage * Cfg::SFQ_BYTES;
    const int64_t kb = Cfg::SF_BLOCKS * static_cast<int64_t>(ti.k0 + ks);
    const int ng = Cfg::ACTQ ? 0 : min(QG, (a.q_rows - ti.q0 + 127) >> 7);
    const bool weights = (part & 1) != 0, acts = (part & 2) != 0;
    const bool do_p = Cfg::SWAP ? weights : acts;          // P is the weights when swapped
    const bool do_q = !Cfg::ACTQ && (Cfg::SWAP ? acts : weights);
    if (weights) {
        const uint32_t q_bytes = Cfg::ACTQ ? 0u : static_cast<uint32_t>(Cfg::Q_BYTES + Cfg::SFP_BYTES * ng);
        mbar_arrive_expect_tx(fb, Cfg::P_BYTES + Cfg::SFP_BYTES + q_bytes);
    }
    if (do_p) {
        tma_load_2d(pbuf, tm_p, fb, kx, ti.p0, pol_p);
        bulk_load(sfpb, a.sf_p + ((ti.p0 >> 7) * static_cast<int64_t>(a.sf_kb4) + kb) * 512, Cfg::SFP_BYTES, fb,
                  pol_p);
    }
    if (do_q) {
        tma_load_2d(qbuf, tm_q, fb, kx, ti.q0, pol_q);
        for (int g = 0; g < ng; ++g)
            bulk_load(sfqb + Cfg::SFP_BYTES * g,
                      a.sf_q + (((ti.q0 >> 7) + g) * static_cast<int64_t>(a.sf_kb4) + kb) * 512, Cfg::SFP_BYTES,
                      fb, pol_q);
    }
}

template <class Cfg>
__global__ void __launch_bounds__(kGemmThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_sfp, const __grid_constant__ CUtensorMap tm_sfq,
                  const __grid_constant__ CUtensorMap tm_q_half, const GemmArgs args)
{
    constexpr int BN = Cfg::BN;
    constexpr int STAGES = Cfg::STAGES;
    constexpr int QG = Cfg::QG;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full_bar = bars;
    uint64_t* sfready_bar = bars + STAGES;
    uint64_t* empty_bar = bars + 2 * STAGES;
    uint64_t* acc_full_bar = bars + 3 * STAGES;
    uint64_t* acc_empty_bar = bars + 3 * STAGES + 2;
    uint64_t* mma_done_bar = bars + 3 * STAGES + 4;
    uint64_t* rx_bar = bars + 3 * STAGES + 5;       // split-K: partial rows received from peers
    uint64_t* sf_free_bar = bars + 3 * STAGES + 6;  // SF_IN_ACC: scale columns drained
    uint64_t* actq_bar = bars + 3 * STAGES + 8;     // ACTQ: the Q stages hold the activations
    uint64_t* amax_bar = bars + 3 * STAGES + 9;     // ACTQ: the peers' slice maxima arrived
    uint64_t* sf_full_bar = bars + 3 * STAGES + 10; // GPAIR: this CTA's scales of stage s landed
    uint32_t* s_tmem_base = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
    volatile int* s_is_last = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 8);
    int32_t* s_prefix = reinterpret_cast<int32_t*>(smem + Cfg::OFF_PREFIX);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const AbortState ab{s_abort, args.err_word};

    // ------------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            // GPAIR: the even CTA's counts one re-layout arrival from each CTA
            mbar_init(&sfready_bar[s], Cfg::GPAIR ? 2 : 1);
            mbar_init(&empty_bar[s], 1);
            mbar_init(&sf_full_bar[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full_bar[s], 1);
            // PAIR: the even CTA's barriers count both CTAs' epilogue warps
            mbar_init(&acc_empty_bar[s], Cfg::PAIR ? 2 * kEpilogueWarps : kEpilogueWarps);
            mbar_init(&sf_free_bar[s], Cfg::PAIR ? 8 : 4);   // the second epilogue warpgroup(s)
        }
        mbar_init(mma_done_bar, 1);
        mbar_init(rx_bar, 1);
        mbar_init(actq_bar, 1);
        mbar_init(amax_bar, 1);
        *s_abort = 0;
        *s_is_last = 0;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_p);
        prefetch_tensormap(&tm_q);
        if constexpr (!Cfg::SFT || Cfg::PAIR) {
            prefetch_tensormap(&tm_sfp);
            prefetch_tensormap(&tm_sfq);
        }
        if constexpr (Cfg::NARROW) prefetch_tensormap(&tm_q_half);
    }
    if (warp == 1) {
        if constexpr (Cfg::PAIR) {
            tmem_alloc_pair(s_tmem_base, Cfg::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(s_tmem_base, Cfg::TMEM_COLS);
            tmem_relinquish();
        }
    }
    // Everything above touches only this CTA's resources and the kernel parameters. Reads of
    // data the previous kernel in the stream may write come after grid_dependency_wait():
    // here for the grouped offsets, in each role below for the rest (the MMA and scale
    // warps read shared and tensor memory only).
    if constexpr (Cfg::GROUPED) {
        if (warp == 3) {
            grid_dependency_wait();
            // Tiles per expert: (N / 128 weight tiles) x ceil(rows_e / BN) token tiles.
            const int E = args.num_experts;
            const int per = (E + 31) / 32;
            const int e0 = lane * per;
            int local = 0;
            for (int i = 0; i < per; ++i) {
                const int e = e0 + i;
                if (e < E) {
                    int32_t r0, rows;
                    expert_rows(args, e, r0, rows);
                    local += args.num_p_tiles * ((rows + BN - 1) / BN);
                }
            }
            int incl = local;
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
            }
            int run = incl - local;
            for (int i = 0; i < per; ++i) {
                const int e = e0 + i;
                if (e < E) {
                    s_prefix[e] = run;
                    int32_t r0, rows;
                    expert_rows(args, e, r0, rows);
                    run += args.num_p_tiles * ((rows + BN - 1) / BN);
                }
            }
            if (lane == 31) s_prefix[E] = incl;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // PAIR: the odd CTA's copies and epilogue arrive on the even CTA's barriers and the even
    // CTA's commits on the odd CTA's; split-K with a receive region of its own: peers send into
    // it as soon as their rows are done. Either way both CTAs' barriers are initialised before
    // either touches the other's.
    if constexpr (Cfg::PAIR) cluster_sync();
    if constexpr (Cfg::RX_OWN) {
        if (args.splits > 1 && args.cluster_size > 1) cluster_sync();
    }
    // Every CTA of this grid is resident: the next kernel in the stream may be scheduled
    // (it waits for this grid's completion before touching memory).
    grid_launch_dependents();

    const uint32_t tmem_base = *s_tmem_base;
    const int32_t num_tiles = Cfg::GROUPED ? s_prefix[args.num_experts] : args.num_tiles;
    // persistent work loop: CTA pairs (PAIR) walk the work items as one
    const int32_t tile_start = static_cast<int32_t>(Cfg::PAIR ? blockIdx.x >> 1 : blockIdx.x);
    const int32_t tile_step = static_cast<int32_t>(Cfg::PAIR ? gridDim.x >> 1 : gridDim.x);

    if (warp == 0) {
        // -------------------------------------------------------------- TMA producer
        // The whole warp walks the loop (uniform control flow and operands); one elected
        // lane issues the copies.
        const uint64_t pol_stream = l2_policy_evict_first();  // weights: read once
        const uint64_t pol_keep = l2_policy_evict_last();     // activations: re-read
        const uint64_t pol_p = Cfg::SWAP ? pol_stream : pol_keep;
        const uint64_t pol_q = Cfg::SWAP ? pol_keep : pol_stream;
        // The first tile's stages whose weight tiles (and scales) were requested before the
        // wait for the previous kernel in the stream (b_ready: the caller guarantees that no
        // kernel that may still run writes B); their full barriers are armed for the whole
        // stage, and the activations follow after the wait.
        int32_t early = 0;
        if constexpr (Cfg::SFT && !Cfg::PAIR && !Cfg::GROUPED) {
            if (args.b_ready && tile_start < num_tiles) {
                const Tile ti = decode_tile<Cfg>(args, tile_start, s_prefix);
                early = ti.kcnt < STAGES ? ti.kcnt : STAGES;
                if (elect_one()) {
                    for (int32_t ks = 0; ks < early; ++ks) sft_stage_copies<Cfg>(args, ti, ks, ks, smem, &tm_p, &tm_q,
                                                                                 full_bar, 1);
                }
                __syncwarp();
            }
        }
        if constexpr (!Cfg::GROUPED) {
            // Warm L2 with this CTA's first weight tiles while the previous kernel finishes
            // (a prefetch only fills L2, the coherence point, so it cannot see stale data).
            if (early == 0 && tile_start < num_tiles && elect_one()) {
                const Tile ti = decode_tile<Cfg>(args, tile_start, s_prefix);
                const int n = ti.kcnt < STAGES ? ti.kcnt : STAGES;
                for (int ks = 0; ks < n; ++ks) {
                    const int32_t kx = (ti.k0 + ks) * Cfg::BK_BYTES;
                    if constexpr (Cfg::SWAP) tma_prefetch_2d(&tm_p, kx, ti.p0);
                    else if constexpr (Cfg::PAIR) tma_prefetch_2d(&tm_q, kx, ti.q0 + (ti.q_span / 2) * static_cast<int32_t>(cluster_ctarank()));
                    else tma_prefetch_2d(&tm_q, kx, ti.q0);
                }
            }
            __syncwarp();
        }
        grid_dependency_wait();
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = true;
        for (int32_t t = tile_start; t < num_tiles && ok; t += tile_step) {
            const Tile ti = decode_tile<Cfg>(args, t, s_prefix);
            for (int32_t ks = 0; ks < ti.kcnt; ++ks) {
                ok = __all_sync(0xffffffffu, mbar_wait(&empty_bar[stage], phase ^ 1u, ab, kErrProducerEmpty));
                if (!ok) break;
                if (elect_one()) {
                    uint64_t* fb = &full_bar[stage];
                    const int32_t kx = (ti.k0 + ks) * Cfg::BK_BYTES;   // byte offset along K
                    const int32_t sx = (ti.k0 + ks) * 16;              // scale byte offset
                    uint8_t* pbuf = smem + Cfg::OFF_P + stage * Cfg::P_BYTES;
                    uint8_t* qbuf = smem + Cfg::OFF_Q + stage * Cfg::Q_BYTES;
                    uint8_t* sfpb = smem + Cfg::OFF_SFP + stage * Cfg::SFP_BYTES;
                    uint8_t* sfqb = smem + Cfg::OFF_SFQ + stage * Cfg::SFQ_BYTES;
                    if constexpr (Cfg::GPAIR) {
                        // this CTA's 128 weight rows and half of the token tile's MMA N (its
                        // rows rounded up to 16), both counted on the even CTA's full barrier,
                        // which the even CTA arms for both CTAs' bytes; the scales of its weight
                        // rows and of all the tile's token rows on its own sf_full barrier (its
                        // re-layout warps wait there)
                        const uint32_t rank = cluster_ctarank();
                        const uint32_t fb0 = mapa_shared(smem_u32(fb), 0);
                        const int n_mma = min(BN, (ti.q_valid + 15) & ~15);
                        const int half = n_mma / 2;
                        const int qb = (half + Cfg::QBOX - 1) / Cfg::QBOX;
                        const int sb = (n_mma + Cfg::QBOX - 1) / Cfg::QBOX;
                        uint64_t* sfb = &sf_full_bar[stage];
                        if (rank == 0)
                            mbar_arrive_expect_tx(fb, 2u * static_cast<uint32_t>(Cfg::P_BYTES + qb * Cfg::QBOX * Cfg::BK_BYTES));
                        mbar_arrive_expect_tx(sfb, static_cast<uint32_t>(Cfg::SF_TMA_P + sb * Cfg::QBOX * 16));
                        if constexpr (Cfg::SWIGLU) {
                            tma_load_5d_pair(pbuf, &tm_p, fb0, kx, 0, 0, ti.p0 >> 5, ti.expert, pol_p);
                            tma_load_5d(sfpb, &tm_sfp, sfb, sx, 0, 0, ti.p0 >> 5, ti.expert, pol_p);
                        } else {
                            tma_load_3d_pair(pbuf, &tm_p, fb0, kx, ti.p0, ti.expert, pol_p);
                            tma_load_3d(sfpb, &tm_sfp, sfb, sx, ti.p0, ti.expert, pol_p);
                        }
                        for (int b = 0; b < qb; ++b)
                            tma_load_2d_pair(qbuf + b * Cfg::QBOX * Cfg::BK_BYTES, &tm_q, fb0, kx,
                                             ti.q0 + half * static_cast<int32_t>(rank) + b * Cfg::QBOX, pol_q);
                        for (int b = 0; b < sb; ++b)
                            tma_load_2d(sfqb + b * Cfg::QBOX * 16, &tm_sfq, sfb, sx, ti.q0 + b * Cfg::QBOX, pol_q);
                    } else if constexpr (Cfg::GROUPED) {
                        // boxes of QBOX token rows covering the tile's MMA N (its rows rounded
                        // up to 16); the 8-row swizzle atoms of the boxes line up as in one box
                        const int n_mma = min(BN, (ti.q_valid + 15) & ~15);
                        const int boxes = (n_mma + Cfg::QBOX - 1) / Cfg::QBOX;
                        mbar_arrive_expect_tx(fb, Cfg::P_BYTES + Cfg::SF_TMA_P +
                                                  static_cast<uint32_t>(boxes * Cfg::QBOX * (Cfg::BK_BYTES + 16)));
                        if constexpr (Cfg::SWIGLU) {
                            // 4 groups x [16 gate rows, 16 up rows] of intermediate indices
                            // [p0 / 2, p0 / 2 + 64): group coordinate (p0 / 2) / 16
                            tma_load_5d(pbuf, &tm_p, fb, kx, 0, 0, ti.p0 >> 5, ti.expert, pol_p);
                            tma_load_5d(sfpb, &tm_sfp, fb, sx, 0, 0, ti.p0 >> 5, ti.expert, pol_p);
                        } else {
                            tma_load_3d(pbuf, &tm_p, fb, kx, ti.p0, ti.expert, pol_p);
                            tma_load_3d(sfpb, &tm_sfp, fb, sx, ti.p0, ti.expert, pol_p);
                        }
                        for (int b = 0; b < boxes; ++b) {
                            tma_load_2d(qbuf + b * Cfg::QBOX * Cfg::BK_BYTES, &tm_q, fb, kx,
                                        ti.q0 + b * Cfg::QBOX, pol_q);
                            tma_load_2d(sfqb + b * Cfg::QBOX * 16, &tm_sfq, fb, sx, ti.q0 + b * Cfg::QBOX,
                                        pol_q);
                        }
                    } else if constexpr (Cfg::PAIR) {
                        // this CTA's P rows and Q rows, the scales of its P rows and of the whole
                        // Q tile; all counted on the even CTA's full barrier, which the even CTA
                        // arms for both CTAs' bytes (rows past the operands read as zero). The
                        // scale runs are read through 2-D views of the tiled layout (rows of
                        // 256 bytes), so that they can complete on the even CTA's barrier too.
                        // (a half tile: 64 Q rows per CTA through the half-height map, and the
                        // scales of its 128 Q rows only)
                        const uint32_t rank = cluster_ctarank();
                        const uint32_t fb0 = mapa_shared(smem_u32(fb), 0);
                        const bool narrow = Cfg::NARROW && ti.q_span < BN;
                        if (rank == 0) mbar_arrive_expect_tx(fb, narrow ? Cfg::PAIR_TX_NARROW : Cfg::PAIR_TX_BYTES);
                        const int32_t kb = Cfg::SF_BLOCKS * (ti.k0 + ks);
                        const int32_t kb4 = args.sf_kb4;
                        tma_load_2d_pair(pbuf, &tm_p, fb0, kx, ti.p0, pol_p);
                        tma_load_2d_pair(qbuf, narrow ? &tm_q_half : &tm_q, fb0, kx,
                                         ti.q0 + (ti.q_span / 2) * static_cast<int32_t>(rank), pol_q);
                        tma_load_2d_pair(sfpb, &tm_sfp, fb0, 0, ((ti.p0 >> 7) * kb4 + kb) * 2, pol_p);
#pragma unroll
                        for (int g = 0; g < QG; ++g)
                            if (g == 0 || !narrow)
                                tma_load_2d_pair(sfqb + Cfg::SFP_BYTES * g, &tm_sfq, fb0, 0,
                                                 (((ti.q0 >> 7) + g) * kb4 + kb) * 2, pol_q);
                    } else if constexpr (Cfg::SFT) {
                        // (the first tile's `early` stages: their weight copies are in flight)
                        const bool first = t == tile_start && ks < early;
                        sft_stage_copies<Cfg>(args, ti, ks, stage, smem, &tm_p, &tm_q, full_bar, first ? 2 : 3);
                    } else {
                        // row-major scales: [rows][16 B] per stage; 8 x 4 scales: the scale map's
                        // rows are 8-row groups, a stage's 4 blocks of one group 128 contiguous
                        // bytes at byte 128 * stage (tiles start on 8-row boundaries)
                        const int32_t sfx = args.sf_8x4 ? kx : sx;
                        const int32_t sfr = args.sf_8x4 ? 3 : 0;
                        mbar_arrive_expect_tx(fb, Cfg::TX_BYTES);
                        tma_load_2d(pbuf, &tm_p, fb, kx, ti.p0, pol_p);
                        tma_load_2d(sfpb, &tm_sfp, fb, sfx, ti.p0 >> sfr, pol_p);
                        tma_load_2d(qbuf, &tm_q, fb, kx, ti.q0, pol_q);
                        tma_load_2d(sfqb, &tm_sfq, fb, sfx, ti.q0 >> sfr, pol_q);
                    }
                }
                __syncwarp();
                ++issued;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // Let every copy still in flight land before shared memory can be released (the odd
        // CTA of a pair cannot wait on the even CTA's full barrier: it waits until the MMAs
        // that read each stage have released it). The `early` weight copies of the first tile
        // are among the issued stages once the loop has reached them; the loop can stop before
        // that only after some role waited 1 s in vain, long after those copies landed.
        const bool on_empty = Cfg::PAIR && cluster_ctarank() != 0;
        const uint32_t inflight = issued < (uint32_t)STAGES ? issued : (uint32_t)STAGES;
        for (uint32_t i = 1; i <= inflight; ++i) {
            const int s = ((int)stage - (int)i + 2 * STAGES) % STAGES;
            const uint32_t ph = ((int)stage - (int)i < 0) ? (phase ^ 1u) : phase;
            mbar_wait_drain(on_empty ? &empty_bar[s] : &full_bar[s], ph);
            if constexpr (Cfg::GPAIR) mbar_wait_drain(&sf_full_bar[s], ph);   // this CTA's scale copies
        }
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA issuer
        // Whole warp in the loop, one elected lane issues tcgen05.cp / tcgen05.mma (PAIR: the
        // even CTA's warp for both CTAs; the odd CTA's only allocates and frees TMEM).
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        uint32_t sf_phases = 0;                    // bit b: parity of the next sf_free[b] wait
        bool ok = !(Cfg::PAIR && cluster_ctarank() != 0);
        if constexpr (Cfg::ACTQ) ok = __all_sync(0xffffffffu, mbar_wait(actq_bar, 0, ab, kErrMmaActq));
        for (int32_t t = tile_start; t < num_tiles && ok; t += tile_step) {
            const Tile ti = decode_tile<Cfg>(args, t, s_prefix);
            ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty_bar[acc], acc_phase ^ 1u, ab, kErrMmaAccEmpty));
            if (!ok) break;
            if constexpr (Cfg::SF_IN_ACC) {
                if (t != tile_start) {                         // the previous tile's scale columns
                    const uint32_t o = acc ^ 1u;
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&sf_free_bar[o], (sf_phases >> o) & 1u, ab, kErrMmaSfFree));
                    if (!ok) break;
                    sf_phases ^= 1u << o;
                }
            }
            tc_fence_after();
            const uint32_t sf_a = tmem_base + Cfg::TMEM_SFA + (Cfg::SF_IN_ACC ? (acc ^ 1u) * BN : 0u);
            const uint32_t sf_b = sf_a + 4 * Cfg::SF_BLOCKS;    // after the SFA columns
            uint32_t n_mma = BN;
            if constexpr (Cfg::GROUPED) n_mma = min(BN, (ti.q_valid + 15) & ~15);
            if constexpr (Cfg::NARROW) n_mma = static_cast<uint32_t>(ti.q_span);
            constexpr uint32_t kMmaM = Cfg::PAIR ? 256 : 128;
            const uint32_t idesc = Cfg::MX ? idesc_mxf4_ue8m0(kMmaM, n_mma) : idesc_mxf4nvf4(kMmaM, n_mma);
            const uint32_t d_tmem = tmem_base + acc * BN;
            for (int32_t ks = 0; ks < ti.kcnt; ++ks) {
                bool got = mbar_wait(&full_bar[stage], phase, ab, kErrMmaFull);
                if constexpr (!Cfg::SFT) got = got && mbar_wait(&sfready_bar[stage], phase, ab, kErrMmaSf);
                ok = __all_sync(0xffffffffu, got);
                if (!ok) break;
                // ACTQ: the activations' K stage ks stays in Q stage ks for the whole launch
                const uint32_t qslot = Cfg::ACTQ ? static_cast<uint32_t>(ks) : stage;
                if (elect_one()) {
                    const uint32_t sfp = smem_u32(smem + Cfg::OFF_SFP + stage * Cfg::SFP_BYTES);
                    const uint32_t sfq = smem_u32(smem + Cfg::OFF_SFQ + qslot * Cfg::SFQ_BYTES);
#pragma unroll
                    for (int j = 0; j < Cfg::SF_BLOCKS; ++j) {
                        if constexpr (Cfg::PAIR) {
                            tmem_cp_32x128b_warpx4_pair(sf_a + 4 * j, sdesc_sf_32x16(sfp + 512 * j));
#pragma unroll
                            for (int g = 0; g < QG; ++g)
                                if (128 * g < static_cast<int>(n_mma))
                                    tmem_cp_32x128b_warpx4_pair(sf_b + 4 * QG * j + 4 * g,
                                                                sdesc_sf_32x16(sfq + Cfg::SFP_BYTES * g + 512 * j));
                        } else {
                            tmem_cp_32x128b_warpx4(sf_a + 4 * j, sdesc_sf_32x16(sfp + 512 * j));
#pragma unroll
                            for (int g = 0; g < QG; ++g)
                                tmem_cp_32x128b_warpx4(sf_b + 4 * QG * j + 4 * g,
                                                       sdesc_sf_32x16(sfq + Cfg::SFP_BYTES * g + 512 * j));
                        }
                    }
                    const uint64_t pdesc =
                        sdesc_kmajor_sw128(smem_u32(smem + Cfg::OFF_P + stage * Cfg::P_BYTES));
                    const uint64_t qdesc =
                        sdesc_kmajor_sw128(smem_u32(smem + Cfg::OFF_Q + qslot * Cfg::Q_BYTES));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // advance 32 bytes (64 fp4 values) along K inside the swizzled rows
                        const uint32_t accum = (ks > 0 || j > 0) ? 1u : 0u;
                        if constexpr (Cfg::MX) {
                            // block j / 2; its scale column holds 4 E8M0 bytes per row (K 128):
                            // bytes 0-1 for the first 64, 2-3 for the second
                            const uint32_t id = idesc_sf_id(idesc, 2u * (j & 1));
                            if constexpr (Cfg::PAIR)
                                mma_mxf4_block32_pair(d_tmem, pdesc + 2u * j, qdesc + 2u * j, id, sf_a + 4 * (j >> 1),
                                                      sf_b + 4 * QG * (j >> 1), accum);
                            else
                                mma_mxf4_block32(d_tmem, pdesc + 2u * j, qdesc + 2u * j, id, sf_a + 4 * (j >> 1),
                                                 sf_b + 4 * QG * (j >> 1), accum);
                        } else {
                            if constexpr (Cfg::PAIR)
                                mma_mxf4nvf4_pair(d_tmem, pdesc + 2u * j, qdesc + 2u * j, idesc, sf_a + 4 * j,
                                                  sf_b + 4 * QG * j, accum);
                            else
                                mma_mxf4nvf4(d_tmem, pdesc + 2u * j, qdesc + 2u * j, idesc, sf_a + 4 * j,
                                             sf_b + 4 * QG * j, accum);
                        }
                    }
                    if constexpr (Cfg::PAIR) mma_commit_both(&empty_bar[stage]);   // both CTAs' stage
                    else mma_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (elect_one()) {
                if constexpr (Cfg::PAIR) mma_commit_both(&acc_full_bar[acc]);
                else mma_commit(&acc_full_bar[acc]);
            }
            __syncwarp();
            if (++acc == Cfg::ACC_STAGES) { acc = 0; acc_phase ^= 1u; }
        }
        // Arrives once every tcgen05 operation issued above has completed (PAIR: in both CTAs,
        // from the even CTA's warp).
        if (elect_one()) {
            if constexpr (Cfg::PAIR) {
                if (cluster_ctarank() == 0) mma_commit_both(mma_done_bar);
            } else {
                mma_commit(mma_done_bar);
            }
        }
        __syncwarp();
    } else if (!Cfg::SFT && (warp == 2 || warp == 3)) {
        // -------------------------------------------------------------- scale re-layout
        // The TMA wrote row r's 16 scale bytes (k-blocks 0..15 of the stage) at r * 16
        // (8 x 4 layout: row r's k-step j word at (r / 8) * 128 + j * 32 + (r % 8) * 4).
        // The MMA for k-step j (k-blocks 4j..4j+3) needs, per 128-row group, a 512-byte
        // block whose 16-byte row i holds the 4 scale bytes of rows i, i+32, i+64, i+96.
        // Each lane owns row i = lane: it reads its 4 rows (16 B each), transposes the
        // 4 x 4 words in registers and writes 4 blocks (one per k-step), in place.
        // Warps 2 and 3 take alternate stages.
        const bool in_8x4 = args.sf_8x4 != 0;
        const uint32_t sf_warp = static_cast<uint32_t>(warp - 2);
        uint32_t stage = 0, phase = 0, seq = 0;
        for (int32_t t = tile_start; t < num_tiles; t += tile_step) {
            const Tile ti = decode_tile<Cfg>(args, t, s_prefix);
            bool ok = true;
            for (int32_t ks = 0; ks < ti.kcnt; ++ks, ++seq) {
                if ((seq & 1u) != sf_warp) {
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    continue;
                }
                ok = mbar_wait(Cfg::GPAIR ? &sf_full_bar[stage] : &full_bar[stage], phase, ab, kErrSfFull);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                uint8_t* sfpb = smem + Cfg::OFF_SFP + stage * Cfg::SFP_BYTES;
                uint8_t* sfqb = smem + Cfg::OFF_SFQ + stage * Cfg::SFQ_BYTES;
#pragma unroll
                for (int grp = 0; grp < 1 + QG; ++grp) {
                    uint8_t* base = grp == 0 ? sfpb : sfqb + 2048 * (grp - 1);
                    const int rows_here = grp == 0 ? 128 : min(128, BN - 128 * (grp - 1));
                    uint4 v[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int r = 32 * q + lane;
                        if (r >= rows_here) {
                            v[q] = make_uint4(0u, 0u, 0u, 0u);
                        } else if (in_8x4) {
                            const uint32_t* w = reinterpret_cast<const uint32_t*>(base + (r >> 3) * 128 + (r & 7) * 4);
                            v[q] = make_uint4(w[0], w[8], w[16], w[24]);
                        } else {
                            v[q] = *reinterpret_cast<const uint4*>(base + 16 * r);
                        }
                    }
                    __syncwarp();
                    uint4 o0 = make_uint4(v[0].x, v[1].x, v[2].x, v[3].x);
                    uint4 o1 = make_uint4(v[0].y, v[1].y, v[2].y, v[3].y);
                    uint4 o2 = make_uint4(v[0].z, v[1].z, v[2].z, v[3].z);
                    uint4 o3 = make_uint4(v[0].w, v[1].w, v[2].w, v[3].w);
                    *reinterpret_cast<uint4*>(base + 0 * 512 + 16 * lane) = o0;
                    *reinterpret_cast<uint4*>(base + 1 * 512 + 16 * lane) = o1;
                    *reinterpret_cast<uint4*>(base + 2 * 512 + 16 * lane) = o2;
                    *reinterpret_cast<uint4*>(base + 3 * 512 + 16 * lane) = o3;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    // GPAIR: the even CTA's MMA warp copies both CTAs' scales, each from the
                    // shared memory of the CTA that wrote them
                    if constexpr (Cfg::GPAIR) mbar_arrive_remote(mapa_shared(smem_u32(&sfready_bar[stage]), 0));
                    else mbar_arrive(&sfready_bar[stage]);
                }
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------- epilogue
        // Two warpgroups: warps 4 + 4h + q read TMEM lane quadrant q and take half h of the
        // tile's columns (split-K: the first warpgroup reduces, the second only keeps pace).
        grid_dependency_wait();                    // alpha, out and the workspace
        const int quad = warp & 3;                 // TMEM lane quadrant this warp may read
        const int half = (warp - 4) >> 2;
        const int row = 32 * quad + lane;          // accumulator row (P row within the tile)
        float gsh = 0.0f;
        float* rcp_tab = reinterpret_cast<float*>(smem + Cfg::OFF_SWIGLU);
        uint8_t* stage_w = smem + Cfg::OFF_SWIGLU + 1024 + (warp - 4) * 128;
        uint8_t* sstage_w = smem + Cfg::OFF_SWIGLU + 1024 + kEpilogueWarps * 128 + (warp - 4) * 16;
        float actq_alpha = 0.0f;
        if constexpr (Cfg::ACTQ) {
            const Tile t0 = decode_tile<Cfg>(args, tile_start, s_prefix);
            actq_alpha = args.act_bf16
                ? actq_quantize_t<Cfg, __nv_bfloat16>(args, smem, t0.k0, t0.kcnt, threadIdx.x - 128, amax_bar, ab)
                : actq_quantize_t<Cfg, float>(args, smem, t0.k0, t0.kcnt, threadIdx.x - 128, amax_bar, ab);
            if (actq_alpha >= 0.0f && threadIdx.x == 128) mbar_arrive(actq_bar);
        }
        if constexpr (Cfg::SWIGLU) {
            // gs_h / e4m3(s) for all 256 scale codes, once per CTA (one entry per epilogue thread)
            gsh = __ldg(args.gs_h);
            const uint32_t code = threadIdx.x - 128;
            const float sfd = e4m3_to_f32(code);
            rcp_tab[code] = (sfd == 0.0f) ? 0.0f : __fdiv_rn(gsh, sfd);
            named_bar_sync(1, 32 * kEpilogueWarps);
        }
        uint32_t acc = 0, acc_phase = 0;
        for (int32_t t = tile_start; t < num_tiles; t += tile_step) {
            const Tile ti = decode_tile<Cfg>(args, t, s_prefix);
            bool ok = mbar_wait(&acc_full_bar[acc], acc_phase, ab, kErrEpiAccFull);
            ok = named_bar_and(1, 32 * kEpilogueWarps, ok);
            if (!ok) {
                if constexpr (!Cfg::GROUPED) {
                    // cluster peers wait for this CTA on the cluster barrier: arrive anyway (the
                    // second warpgroup arrives in the teardown)
                    if (!Cfg::RX_OWN && half == 0 && args.splits > 1 && args.cluster_size > 1) {
                        cluster_arrive();
                        cluster_wait();
                    }
                }
                break;
            }
            tc_fence_after();

            const float alpha = Cfg::ACTQ ? actq_alpha
                              : Cfg::GROUPED ? __ldg(args.alpha + ti.expert) : __ldg(args.alpha);
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(32 * quad) << 16) + acc * BN;
            const int p = ti.p0 + row;             // P row this thread owns
            const bool split_k = !Cfg::GROUPED && args.splits > 1;
            int n_cols = BN;
            if constexpr (Cfg::GROUPED) n_cols = min(BN, (ti.q_valid + 15) & ~15);
            if constexpr (Cfg::NARROW) n_cols = ti.q_span;
            if constexpr (!Cfg::GROUPED) {
                if (split_k && half == 0)
                    split_k_epilogue<Cfg>(args, ti, smem, rx_bar, s_is_last, tacc, row, alpha, ab);
            }
            // this warpgroup's columns [c_lo, c_hi), multiples of 16
            const int mid = ((n_cols / 2 + 15) / 16) * 16;
            const int c_lo = half ? mid : 0;
            int c_hi = split_k ? c_lo : (half ? n_cols : mid);
            if constexpr (Cfg::SF_IN_ACC) {
                // the second warpgroup frees the last 64 columns (the next tile's scale
                // columns) first: into registers, signal, then store them
                if (half == 1 && !split_k) {
                    uint32_t r[4][16];
                    const bool need = n_cols > BN - 64;
                    if (need) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x16(tacc + BN - 64 + 16 * i, r[i]);
                        tmem_ld_wait();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (Cfg::PAIR) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&sf_free_bar[acc]), 0));
                        else mbar_arrive_relaxed(&sf_free_bar[acc]);
                    }
                    if (need) {
                        if constexpr (!Cfg::SWAP && !Cfg::GROUPED) {
                            store_rows64<Cfg>(args, ti, quad, lane, BN - 64, r, alpha);
                        } else if constexpr (Cfg::SWIGLU) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                if (BN - 64 + 16 * i < n_cols)
                                    swiglu_chunk16<Cfg>(args, ti, quad, lane, BN - 64 + 16 * i, r[i], alpha, gsh,
                                                        rcp_tab, stage_w, sstage_w);
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                if (BN - 64 + 16 * i < n_cols) {
                                    if (args.out_dtype != kOutF32)
                                        store_tok16<Cfg>(args, ti, quad, lane, BN - 64 + 16 * i, r[i], alpha);
                                    else
                                        store_out16<Cfg>(args, ti, p, BN - 64 + 16 * i, r[i], alpha);
                                }
                        }
                    }
                    c_hi = min(c_hi, BN - 64);
                }
            }

            if constexpr (!Cfg::SWAP && !Cfg::GROUPED) {
                // 64-column chunks: four 16-column TMEM loads in flight, coalesced row stores
                int c0 = c_lo;
                for (; c0 + 64 <= c_hi; c0 += 64) {
                    uint32_t r[4][16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x16(tacc + c0 + 16 * i, r[i]);
                    tmem_ld_wait();
                    store_rows64<Cfg>(args, ti, quad, lane, c0, r, alpha);
                }
                // the rest (BN = 224, 192: 48, 32 columns per half) the plain way
                for (; c0 < c_hi; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(tacc + c0, r);
                    tmem_ld_wait();
                    store_out16<Cfg>(args, ti, p, c0, r, alpha);
                }
            } else {
                // two 16-column TMEM loads in flight per wait
                for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
                    uint32_t r[2][16];
                    const bool two = c0 + 16 < c_hi;
                    tmem_ld_32x32b_x16(tacc + c0, r[0]);
                    if (two) tmem_ld_32x32b_x16(tacc + c0 + 16, r[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h == 1 && !two) break;
                        const int c = c0 + 16 * h;
                        if constexpr (Cfg::SWIGLU)
                            swiglu_chunk16<Cfg>(args, ti, quad, lane, c, r[h], alpha, gsh, rcp_tab, stage_w, sstage_w);
                        else if (args.out_dtype != kOutF32)
                            store_tok16<Cfg>(args, ti, quad, lane, c, r[h], alpha);
                        else
                            store_out16<Cfg>(args, ti, p, c, r[h], alpha);
                    }
                }
            }
            // Accumulator drained into registers / workspace: hand it back to the MMA warp (PAIR:
            // the even CTA's, which writes both CTAs' accumulators).
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (Cfg::PAIR) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&acc_empty_bar[acc]), 0));
                else mbar_arrive_relaxed(&acc_empty_bar[acc]);
            }
            if (++acc == Cfg::ACC_STAGES) { acc = 0; acc_phase ^= 1u; }

        }
    }

    // ------------------------------------------------------------------ teardown
    __syncwarp();
    if constexpr (!Cfg::GROUPED && !Cfg::RX_OWN) {
        // split-K: the non-epilogue warps (and the second epilogue warpgroup) are done with
        // the pipeline; together with the first epilogue warpgroup's arrival (after its
        // accumulator is complete) this tells the cluster peers that this CTA's shared memory
        // may receive their partial rows
        if ((warp < 4 || warp >= 8) && args.splits > 1 && args.cluster_size > 1) {
            cluster_arrive();
            cluster_wait();
        }
    }
    if constexpr (Cfg::RX_OWN) {
        // split-K with a receive region of its own: no cluster barrier. Every byte a peer sends
        // to this CTA (partial rows; ACTQ: slice maxima) is counted on this CTA's own rx (amax)
        // barrier, which its epilogue has waited for, so nothing is still on its way here when
        // it leaves. After an abort those waits may not have completed: wait for them once more,
        // bounded, so that no peer's rows land in the shared memory of a CTA that has left.
        if (warp == 4 && lane == 0 && args.splits > 1 && args.cluster_size > 1) {
            if (!mbar_test_wait(rx_bar, 0)) mbar_wait_drain(rx_bar, 0);
            if constexpr (Cfg::ACTQ) {
                if (!mbar_test_wait(amax_bar, 0)) mbar_wait_drain(amax_bar, 0);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (lane == 0) mbar_wait_drain(mma_done_bar, 0);
        __syncwarp();
    }
    if constexpr (Cfg::PAIR) {
        // neither CTA frees its TMEM or leaves while the other's copies, arrivals or the even
        // CTA's MMAs may still reach it: every thread of both arrives once, after its own roles
        // are done and both MMA warps have seen the last commit
        __syncthreads();
        cluster_sync();
    }
    if (warp == 1) {
        tc_fence_after();
        if constexpr (Cfg::PAIR) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
        else tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace nvfp4
