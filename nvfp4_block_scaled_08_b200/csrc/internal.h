// internal.h -- declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

// Largest expert count the grouped GEMM accepts (its tile prefix lives in shared memory).
constexpr int kMaxExperts = 1024;

// quantize.cu
cudaError_t launch_global_scale(const void* x, bool bf16, int64_t numel, float* gs,
                                cudaStream_t stream, int num_sms);
cudaError_t launch_quantize(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx,
                            const float* gs, uint8_t* q, uint8_t* sf, cudaStream_t stream,
                            int num_sms);
// sf_layout: 0 linear, 1 tiled (128 x 4), 2 8 x 4 (nvfp4_sf_layout)
cudaError_t launch_quantize_dynamic(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx,
                                    float* gs_out, uint8_t* q, uint8_t* sf, int sf_layout,
                                    const float* gs_other, int32_t n_alpha, float* alpha_out,
                                    unsigned* err_word, cudaStream_t stream, int num_sms);
// Dynamic quantisation of x[T, H] (global scale over all of x) with every row t's codes and
// scales written to the k rows row_of[t k + s] of q[T k, H/2] and sf[T k, H/16] (linear).
cudaError_t launch_gather_quantize(const void* x, bool bf16, int64_t T, int64_t H, int64_t ldx, int32_t k,
                                   const int32_t* row_of, float* gs_out, uint8_t* q, uint8_t* sf,
                                   const float* gs_other, int32_t n_alpha, float* alpha_out,
                                   unsigned* err_word, cudaStream_t stream, int num_sms);
// moe.cu: top-k routing and the expert-sorted permutation (three launches), the combine.
cudaError_t launch_moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* experts,
                             float* weights, int32_t* offsets, int32_t* row_of, int32_t* token_of_row,
                             cudaStream_t stream);
cudaError_t launch_moe_combine(const void* y, int32_t y_dt, const float* weights, const int32_t* row_of,
                               int32_t T, int64_t H, int32_t k, void* out, int32_t out_dt, cudaStream_t stream,
                               int num_sms);
// Row-major NVFP4 scales [rows][K / 16] -> the 8 x 4 layout.
cudaError_t launch_sf_8x4(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* out, cudaStream_t stream,
                          int num_sms);
// Row-major scales [rows][K / block] -> the tiled layout (block = 16: NVFP4, 32: MXFP4).
cudaError_t launch_sf_tile(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* out, cudaStream_t stream,
                           int num_sms, int block = 16);
// MXFP4 quantisation (E8M0 scale per 32 elements, no per-tensor scale), linear or tiled scales.
cudaError_t launch_mx_quantize(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx, uint8_t* q,
                               uint8_t* sf, bool sf_tiled, cudaStream_t stream, int num_sms);
cudaError_t launch_alpha(const float* gs_a, const float* gs_b, int32_t n, float* alpha,
                         cudaStream_t stream);
cudaError_t launch_round(const float* x, int64_t n, uint8_t* out, bool e2m1, cudaStream_t stream,
                         int num_sms);

// Tiling chosen for one GEMM call.
struct GemmPlan {
    int bn = 0;            // Q tile rows (MMA N)
    bool swap = false;     // weights as the 128-row MMA operand
    bool grouped = false;
    int splits = 1;        // split-K factor = cluster * groups
    int cluster = 1;       // split-K CTAs per thread-block cluster (DSMEM reduction)
    int groups = 1;        // clusters per output tile (workspace reduction when > 1)
    int p_tiles = 0, q_tiles = 0;
    int num_tiles = 0;     // work items (non-grouped)
    int band = 1;          // P tiles per rasterisation band (non-grouped)
    int grid = 0;          // persistent CTAs
    bool pair = false;     // 2-CTA clusters sharing 256-row Q tiles (tiled scales, no split-K)
    int pair_grid = 0;     // CTAs of the pair launch (2 per cluster)
    int pair_band = 1;     // rasterisation band of the pair launch, in P tile pairs
    int pair_items = 0;    // work items of the pair launch (tiles, the last ones split in halves)
    int narrow_from = 0;   // first half-tile item of the pair launch (= pair_items: none)
    size_t ws_bytes = 0;   // workspace needed (split-K)
    size_t ws_counter_bytes = 0;
};

// gemm.cu
// allow_workspace: a split-K workspace may be used (groups > 1); cluster-only split-K
// needs none.
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, bool allow_workspace, int num_sms);
GemmPlan plan_grouped(int32_t E, int64_t total_rows, int64_t N, int64_t K, int num_sms);
// Forces planner choices for later calls (0 = the planner's own); nvfp4_set_plan_override.
void set_plan_override(int bn, int cluster, int groups, int band, int grouped_bn, int pair);

struct GemmLaunch {
    const uint8_t* A; const uint8_t* sfA; const uint8_t* B; const uint8_t* sfB;
    const float* alpha; void* out;
    int64_t M, N, K;
    const int32_t* offsets; int32_t E; int64_t total_rows;
    void* ws;
    unsigned* err_word;
    bool sf_tiled = false;      // sfA and sfB in the tiled layout (dense GEMM only)
    int32_t out_dtype = 0;      // nvfp4_out_dtype of out
    // grouped gate_up with the fused SwiGLU + NVFP4 epilogue (h_q != nullptr): B holds gate rows
    // [0, N/2) and up rows [N/2, N) per expert; h = silu(gate) * up is written as codes h_q
    // [total_rows, N/4] and e4m3 scales h_sf [total_rows, N/32] with the global scale gs_h
    uint8_t* h_q = nullptr;
    uint8_t* h_sf = nullptr;
    const float* gs_h = nullptr;
    bool mx = false;            // MXFP4 operands (E8M0 scale per 32 elements, tiled scales)
    // activations quantised inside the GEMM (few tokens): A is act [M, K] (fp32 or bf16)
    const void* act = nullptr;
    int64_t act_ld = 0;
    bool act_bf16 = false;
    const float* gs_b = nullptr;
    float* gs_out = nullptr;
    float* alpha_out = nullptr;
    bool sf_8x4 = false;        // sfA and sfB in the 8 x 4 layout (dense NVFP4 GEMM only)
    bool b_ready = false;       // NVFP4_GEMM_B_READY: B's first stages may load before the
                                // wait for the previous kernel in the stream
};

// api.cu: nvfp4_status of the current device's checks; fills the SM count and the device
// error word on success.
int query_current_device(int* num_sms, unsigned** err_word);

// api.cu: nvfp4_status of the pointer and shape checks every GEMM entry point applies (null
// pointers, K % 256, N % 8, sizes below 2^31, 16-byte alignment, alpha 4-byte aligned).
int check_gemm_args(const void* A, const void* sfA, const void* B, const void* sfB,
                    const void* alpha, const void* out, int64_t N, int64_t K);

// Stage ring depth of the activation-quantising few-token GEMM with token tile width bn (the
// most K stages one CTA can hold); 0 for other widths.
int act_gemm_stages(int bn);

// Returns cudaSuccess or the first CUDA error; *encode_failed is set if a TMA descriptor
// could not be encoded.
cudaError_t launch_gemm(const GemmPlan& plan, const GemmLaunch& L, cudaStream_t stream,
                        bool* encode_failed);

}  // namespace nvfp4
