/*
 * nvfp4.h -- C ABI of libnvfp4: NVFP4 block-scaled quantisation and matrix multiplication
 * for NVIDIA B200 (sm_100a).
 *
 * The operation (reference pages: "The Moment the Zeros Disappeared", section "The Subject
 * Message"; "The Art of Reading the Manual", section "The Message", the mm_fp4 signature):
 *
 *     out[m, n] = bf16( alpha * sum_k deq(A)[m, k] * deq(B)[n, k] )
 *     deq(X)[r, k] = e2m1(X[r, k]) * e4m3(sfX[r, k / 16])
 *
 * Data formats (all row-major, "TN": both operands contiguous along K):
 *   - packed operand X[rows, K/2] uint8: element k of a row sits in byte k/2, even k in the
 *     low nibble; a nibble is an e2m1 code (sign, 2-bit exponent, 1-bit mantissa;
 *     magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).
 *   - scales sfX[rows, K/16] uint8: one float8_e4m3fn per 16 consecutive K elements
 *     (block_size = 16, fixed), linear layout, row stride K/16 bytes.
 *   - B is stored N x K/2 (the pages' "(K//2, N) column-major" view of the same bytes).
 *   - alpha: fp32 on the device (a required argument, never implied), out: bf16 [M, N]
 *     row-major, caller-allocated (also required).
 *
 * Conventions shared by every call:
 *   - The caller owns all memory. Except where a call says otherwise, pointers are device
 *     pointers and must be 16-byte aligned. The library allocates no device memory; it
 *     keeps only a per-process cache of TMA descriptors and device attributes.
 *   - Calls are asynchronous on the given stream (0 = legacy default stream). The returned
 *     status covers argument checks and launch errors only. A kernel that gives up on a
 *     bounded internal wait records NVFP4_ERR_TIMEOUT in a device error word that
 *     nvfp4_last_device_error() reads; the outputs of the call whose kernel recorded it are
 *     undefined (the kernel stops early, or goes on after a wait that did not complete).
 *   - No fallback: on a device other than compute capability 10.0 every compute call
 *     returns NVFP4_ERR_ARCH; there is no CPU or alternative-backend path.
 *   - Shapes: K % 256 == 0, N % 8 == 0, M >= 0 arbitrary (M == 0 is a no-op), all sizes
 *     below 2^31 elements per dimension.
 *   - Thread safety: calls may be made from several host threads.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum value */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 256 != 0, N % 8 != 0, too large, ... */
    NVFP4_ERR_MISALIGNED = 3,         /* a pointer or leading dimension breaks 16-byte alignment */
    NVFP4_ERR_ARCH = 4,               /* device is not sm_100 (B200 / B100 class) */
    NVFP4_ERR_CUDA = 5,               /* a CUDA runtime or driver call failed */
    NVFP4_ERR_TIMEOUT = 6,            /* a kernel gave up on a bounded wait (device error word) */
    NVFP4_ERR_WORKSPACE = 7           /* workspace given but smaller than required */
} nvfp4_status;

typedef enum {
    NVFP4_IN_F32 = 0,
    NVFP4_IN_BF16 = 1
} nvfp4_in_dtype;

/*
 * Layout of a scale matrix (one e4m3 byte per 16 K-elements of each row).
 *   NVFP4_SF_LINEAR: row-major [rows][K/16] bytes.
 *   NVFP4_SF_TILED:  512-byte blocks of 128 rows x 4 scales (64 K-elements): the scale of row r,
 *                    column c (c = k / 16) is at byte
 *                        ((r / 128) * (K / 64) + c / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4,
 *                    rows padded to a multiple of 128 (the padding is never read into an output).
 *                    Each block's 16-byte row i holds the scales of rows i, i + 32, i + 64, i + 96:
 *                    the operand layout of the tensor cores' scale copies, so the GEMM fetches a
 *                    stage's scales with one bulk copy per 128 rows. Requires K % 64 == 0.
 *   NVFP4_SF_8X4:    32-byte blocks of 8 rows x 4 scales, row-major inside the block, a row group's
 *                    blocks consecutive along K: the scale of row r, column c is at byte
 *                        ((r / 8) * (K / 64) + c / 4) * 32 + (r % 8) * 4 + c % 4,
 *                    rows padded to a multiple of 8 (the padding is never read into an output).
 *                    The mm_fp4 signature's use_8x4_sf_layout ("The Art of Reading the Manual",
 *                    section "The Message") names an 8 x 4 scale layout without defining it; this
 *                    is the library's reading: the tiled layout's 4-scale columns with 8-row
 *                    instead of 128-row groups, so that a few-token scale matrix is padded to 8
 *                    rows, not 128. The dense NVFP4 GEMM reads it directly (one 2D copy per stage
 *                    and operand, re-laid in shared memory). Requires K % 64 == 0.
 */
typedef enum {
    NVFP4_SF_LINEAR = 0,
    NVFP4_SF_TILED = 1,
    NVFP4_SF_8X4 = 2
} nvfp4_sf_layout;

/*
 * Element type of a GEMM output (the mm_fp4 signature's out_dtype: "The Art of Reading the
 * Manual", section "The Message"). The value alpha * acc is computed in fp32 from the fp32
 * accumulator and rounded once to the output type, to nearest even; fp16 values beyond its
 * range become +-infinity. NVFP4_OUT_F32 stores alpha * acc itself (4 bytes per element).
 */
typedef enum {
    NVFP4_OUT_BF16 = 0,
    NVFP4_OUT_F16 = 1,
    NVFP4_OUT_F32 = 2
} nvfp4_out_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* nvfp4_status_string(nvfp4_status s);

/*
 * Per-tensor global scale: gs_out[0] = 2688 / max|x| in fp32 (2688 = 448 * 6, so the
 * largest block scale of the tensor lands on e4m3's maximum 448), or 1 if x is all zero.
 * The pages name the NVFP4 format (e2m1 values, one e4m3 scale per 16 elements: "When a
 * Benchmark Crashes", section "Input Knowledge Required", item 3) but give no quantisation
 * recipe; this two-level recipe (a per-tensor fp32 scale, then per-block scales) is the
 * library's reading of them, and nvfp4_quantize below follows it.
 * x: device, numel elements of the given dtype, 16-byte aligned. gs_out: device, one
 * float, used as the reduction accumulator while the call runs (its old value is
 * ignored). Three stream operations (clear, reduce, finalise). numel == 0 gives 1.
 */
nvfp4_status nvfp4_global_scale(const void* x, nvfp4_in_dtype dtype, int64_t numel,
                                float* gs_out, cudaStream_t stream);

/*
 * Two-level NVFP4 quantisation of x[rows, K] (row stride ld_x elements) with the global
 * scale gs (device, one float, normally from nvfp4_global_scale). For every row and every
 * 16-element block j, in fp32 with round-to-nearest-even and no fused operations:
 *     amax = max |x|;  s = e4m3_rn_satfinite((amax / 6) * gs);  r = s ? gs / s : 0
 *     code_k = e2m1_rn_satfinite(x_k * r)    (ties to the even code; sign kept, so a
 *                                             negative value that rounds to 0 gives 0x8)
 * Outputs: q[rows, K/2] (device) and sf[rows, K/16] (device, e4m3 bytes), both
 * caller-allocated. Requires K % 16 == 0 here (the GEMMs require K % 256 == 0),
 * ld_x * sizeof(dtype) % 16 == 0, x, q 16-byte aligned.
 */
nvfp4_status nvfp4_quantize(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                            int64_t ld_x, const float* gs, uint8_t* q, uint8_t* sf,
                            cudaStream_t stream);

/*
 * Activation quantisation in one launch: computes the global scale of x exactly as
 * nvfp4_global_scale does, writes it to gs_out[0], quantises x with it exactly as
 * nvfp4_quantize does, and, for i < n_alpha, writes alpha_out[i] = 1 / (gs_out[0] *
 * gs_other[i]) exactly as nvfp4_alpha does (n_alpha == 0: gs_other / alpha_out unused).
 * Same layouts and requirements as nvfp4_quantize; gs_out, gs_other, alpha_out: device.
 * One launch (tensors up to 512 KB: one thread-block cluster; larger: a cooperative grid
 * with one grid barrier). The first 8 bytes per block of q hold the per-block maxima and
 * "read" flags before they receive the codes. rows * K must be below
 * 2^31 * (16 / sizeof(dtype)).
 */
nvfp4_status nvfp4_quantize_dynamic(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                                    int64_t ld_x, float* gs_out, uint8_t* q, uint8_t* sf,
                                    const float* gs_other, int32_t n_alpha, float* alpha_out,
                                    cudaStream_t stream);

/*
 * nvfp4_quantize_dynamic with the scales written in the given layout (the same values; for
 * NVFP4_SF_TILED and NVFP4_SF_8X4, sf holds nvfp4_sf_bytes(rows, K, sf_layout) bytes and
 * K % 64 == 0; the padding rows' bytes are left as they are).
 * nvfp4_quantize_dynamic is this call with NVFP4_SF_LINEAR.
 */
nvfp4_status nvfp4_quantize_dynamic_ex(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                                       int64_t ld_x, float* gs_out, uint8_t* q, uint8_t* sf,
                                       const float* gs_other, int32_t n_alpha, float* alpha_out,
                                       nvfp4_sf_layout sf_layout, cudaStream_t stream);

/* Bytes of a scale matrix of `rows` rows and K elements per row in the given layout (0 for an
 * invalid layout or K). */
size_t nvfp4_sf_bytes(int64_t rows, int64_t K, nvfp4_sf_layout sf_layout);

/*
 * Re-lays row-major scales sf[rows][K/16] (device) out as NVFP4_SF_TILED into sf_tiled (device,
 * nvfp4_sf_bytes(rows, K, NVFP4_SF_TILED) bytes; padding rows become 0). K % 64 == 0. For
 * weights, once, before the GEMMs that use them.
 */
nvfp4_status nvfp4_sf_tile(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* sf_tiled,
                           cudaStream_t stream);

/*
 * Re-lays row-major scales sf[rows][K/16] (device) out as NVFP4_SF_8X4 into sf_8x4 (device,
 * nvfp4_sf_bytes(rows, K, NVFP4_SF_8X4) bytes; padding rows become 0). K % 64 == 0. One launch.
 */
nvfp4_status nvfp4_sf_8x4(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* sf_8x4,
                          cudaStream_t stream);

/*
 * GEMM scale from the two global scales: alpha[i] = 1 / (gs_a[0] * gs_b[i]) in fp32,
 * for i < n (n = 1 for a single GEMM, n = experts for the grouped GEMM). All device.
 */
nvfp4_status nvfp4_alpha(const float* gs_a, const float* gs_b, int32_t n, float* alpha,
                         cudaStream_t stream);

/*
 * Workspace bytes nvfp4_gemm uses for split-K on this device for this shape (0 when the
 * shape runs without split-K). Returns 0 if no CUDA device is usable.
 */
size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * Block-scaled NVFP4 GEMM: out[M, N] = bf16(alpha[0] * sum_k deq(A)[m, k] deq(B)[n, k]).
 * A[M, K/2], sfA[M, K/16], B[N, K/2], sfB[N, K/16], alpha[1], out[M, N]: device.
 * ws / ws_bytes: optional split-K workspace (device). ws == NULL runs without split-K.
 * A non-NULL ws must be at least nvfp4_gemm_workspace_size(M, N, K) bytes
 * (NVFP4_ERR_WORKSPACE otherwise), 256-byte aligned, and zero-filled before its first
 * use; every completed call leaves its tile counters at zero again, so one zero fill
 * serves any number of calls. Calls that share a workspace must not overlap in time.
 * Split-K partial sums are reduced in a fixed order, so results are deterministic.
 */
nvfp4_status nvfp4_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                        const uint8_t* sfB, const float* alpha, void* out,
                        int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                        cudaStream_t stream);

/*
 * nvfp4_gemm with both scale matrices in the given layout: sfA of nvfp4_sf_bytes(M, K, layout)
 * and sfB of nvfp4_sf_bytes(N, K, layout) bytes (device). The results are bit for bit those of
 * nvfp4_gemm on the same scales in the linear layout. NVFP4_SF_TILED skips the
 * kernel's scale re-layout step (one bulk copy per stage and 128 rows) and is the faster
 * layout. With tuning overrides that place token tiles off 128-row tile boundaries it returns
 * NVFP4_ERR_UNSUPPORTED_SHAPE. NVFP4_SF_8X4 runs every tiling the linear layout runs (tiles
 * start on 8-row boundaries). nvfp4_gemm is this call with NVFP4_SF_LINEAR.
 */
nvfp4_status nvfp4_gemm_ex(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                           const uint8_t* sfB, const float* alpha, void* out,
                           int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                           nvfp4_sf_layout sf_layout, cudaStream_t stream);

/*
 * nvfp4_gemm_ex with the output element type chosen: out[M, N] holds elements of out_dtype
 * (2 or 4 bytes each, row-major, 16-byte aligned). Same operation, checks and split-K rules;
 * nvfp4_gemm_ex is this call with NVFP4_OUT_BF16. A bad out_dtype: NVFP4_ERR_INVALID_ARG.
 */
nvfp4_status nvfp4_gemm_ex2(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                            const uint8_t* sfB, const float* alpha, void* out,
                            int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                            nvfp4_sf_layout sf_layout, nvfp4_out_dtype out_dtype, cudaStream_t stream);

/* Flags of nvfp4_gemm_ex3. */
enum { NVFP4_GEMM_B_READY = 1 };

/*
 * nvfp4_gemm_ex2 with flags (nvfp4_gemm_ex2 is this call with flags = 0); other bits:
 * NVFP4_ERR_INVALID_ARG. Same operation, output bits, checks and split-K rules.
 *   NVFP4_GEMM_B_READY: the caller guarantees that B and sfB are not written by any kernel
 *     that may still be running when this call's kernel starts (for example weights quantised
 *     earlier and not rewritten since). The kernel is launched early behind the previous
 *     kernel in the stream (programmatic dependent launch); with this flag it also loads its
 *     first K stages of B into shared memory before waiting for that kernel, instead of only
 *     requesting them into L2. Applies to NVFP4_SF_TILED launches on one CTA per tile (few-token
 *     and mid-size products); the others ignore it. Without the guarantee the result may read
 *     stale B.
 */
nvfp4_status nvfp4_gemm_ex3(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                            const uint8_t* sfB, const float* alpha, void* out,
                            int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                            nvfp4_sf_layout sf_layout, nvfp4_out_dtype out_dtype, uint32_t flags,
                            cudaStream_t stream);

/*
 * MXFP4: the mm_fp4 variant that use_nvfp4=False selects ("The Art of Reading the Manual",
 * section "The Message"; the pages name it without defining it). The library's reading is
 * OCP Microscaling v1.0 FP4: e2m1 elements as above, one E8M0 scale byte per 32 consecutive K
 * elements (value 2^(byte - 127); 255 is NaN and never written) and no per-tensor scale.
 *
 * nvfp4_mx_quantize: for every row and 32-element block, with amax = max|x| (fp32):
 *     shared_exp = floor(log2(amax)) - 2, clamped to [-127, 127] (all-zero block: -127),
 *     byte = shared_exp + 127,  code_k = e2m1_rn_satfinite(x_k * 2^-shared_exp)
 * (elements in (6, 8) * 2^shared_exp saturate to 6). x[rows, K] fp32 or bf16 (row stride
 * ld_x), q[rows, K/2] as for NVFP4, sf: E8M0 bytes in the given layout: NVFP4_SF_LINEAR
 * [rows][K/32], or NVFP4_SF_TILED: the NVFP4 tiled layout with K/32 scale columns (512-byte
 * blocks of 128 rows x 4 scales; row r, column c = k / 32 at
 * ((r / 128) * (K / 128) + c / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4, rows padded
 * to 128; K % 128 == 0). One launch, no reduction across blocks. K % 32 == 0.
 */
nvfp4_status nvfp4_mx_quantize(const void* x, nvfp4_in_dtype dtype, int64_t rows, int64_t K,
                               int64_t ld_x, uint8_t* q, uint8_t* sf, nvfp4_sf_layout sf_layout,
                               cudaStream_t stream);

/* Bytes of an MXFP4 scale matrix of `rows` rows and K elements per row in the given layout. */
size_t nvfp4_mx_sf_bytes(int64_t rows, int64_t K, nvfp4_sf_layout sf_layout);

/* Re-lays row-major MXFP4 scales [rows][K/32] out as NVFP4_SF_TILED (K % 128 == 0). */
nvfp4_status nvfp4_mx_sf_tile(const uint8_t* sf, int64_t rows, int64_t K, uint8_t* sf_tiled,
                              cudaStream_t stream);

/*
 * MXFP4 GEMM: out[M, N] = alpha[0] * sum_k deq(A)[m, k] deq(B)[n, k] in out_dtype, with
 * deq(X)[r, k] = e2m1(X[r, k]) * 2^(sfX[r, k / 32] - 127). A, B as for nvfp4_gemm; sfA, sfB:
 * E8M0 scales in the tiled layout (nvfp4_mx_sf_bytes(rows, K, NVFP4_SF_TILED) bytes each, from
 * nvfp4_mx_quantize or nvfp4_mx_sf_tile). alpha is a required device scalar (1 for plain MX).
 * Same shape rules, split-K workspace rules and determinism as nvfp4_gemm.
 */
nvfp4_status nvfp4_mx_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                           const float* alpha, void* out, int64_t M, int64_t N, int64_t K, void* ws,
                           size_t ws_bytes, nvfp4_out_dtype out_dtype, cudaStream_t stream);

/*
 * Few-token GEMM on unquantised activations: the quantisation of x and the product in one
 * launch. Computes exactly what nvfp4_quantize_dynamic_ex(x, gs_other = gs_b) followed by
 * nvfp4_gemm_ex2 compute (the same codes, scales, alpha and MMAs, so the same output bits):
 * out[M, N] = alpha * sum_k deq(Q(x))[m, k] deq(B)[n, k], alpha = 1 / (gs_x * gs_b[0]), gs_x =
 * 2688 / max|x| (1 if x is all zero). x[M, K]: fp32 or bf16 (device, row stride ld_x elements,
 * 16-byte aligned rows), gs_b: the weights' global scale (device, 1 float), B[N, K/2] and
 * sfB in NVFP4_SF_TILED (device), out[M, N] of out_dtype. gs_out / alpha_out (device, 1 float
 * each, optional): receive gs_x and alpha. M <= 64 (decode shapes); the planned split-K
 * cluster must give every CTA at most its stage ring's depth of 256-element K stages (K <=
 * 1024 per CTA at 64 tokens), else NVFP4_ERR_UNSUPPORTED_SHAPE (the two-call path serves
 * those shapes). Each CTA of the cluster reads its own K slice of x and the slices' maxima meet
 * in distributed shared memory, so the global scale needs no grid-wide barrier.
 */
nvfp4_status nvfp4_gemm_act(const void* x, nvfp4_in_dtype dtype, int64_t ld_x, const float* gs_b,
                            const uint8_t* B, const uint8_t* sfB, void* out, int64_t M, int64_t N, int64_t K,
                            float* gs_out, float* alpha_out, nvfp4_out_dtype out_dtype, cudaStream_t stream);

/*
 * Grouped (mixture-of-experts) NVFP4 GEMM ("When a Benchmark Crashes", section "Why This
 * Message Was Written": 256 experts, 8 active per token). Rows of A are sorted by expert;
 * expert e owns rows [expert_offsets[e], expert_offsets[e+1]) and computes
 *     out[r, n] = bf16(alpha[e] * sum_k deq(A)[r, k] deq(B[e])[n, k]).
 * A[total_rows, K/2], sfA[total_rows, K/16], B[E, N, K/2], sfB[E, N, K/16], alpha[E],
 * expert_offsets[E + 1] (int32, non-decreasing, offsets[0] == 0, offsets[E] <= total_rows),
 * out[total_rows, N]: all device. The offsets are read on the device (no host sync);
 * empty experts are allowed; output rows past offsets[E] are not written.
 * ws / ws_bytes: reserved, pass NULL / 0 (nvfp4_grouped_gemm_workspace_size returns 0).
 */
size_t nvfp4_grouped_gemm_workspace_size(int32_t E, int64_t total_rows, int64_t N, int64_t K);

nvfp4_status nvfp4_grouped_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                const uint8_t* sfB, const float* alpha,
                                const int32_t* expert_offsets, int32_t E, int64_t total_rows,
                                int64_t N, int64_t K, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t stream);

/*
 * nvfp4_grouped_gemm with the output element type chosen (out[total_rows, N] of out_dtype;
 * no workspace). nvfp4_grouped_gemm is this call with NVFP4_OUT_BF16.
 */
nvfp4_status nvfp4_grouped_gemm_ex(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                   const uint8_t* sfB, const float* alpha,
                                   const int32_t* expert_offsets, int32_t E, int64_t total_rows,
                                   int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                                   cudaStream_t stream);

/*
 * Grouped gate_up GEMM of a mixture-of-experts MLP with the SwiGLU activation and the NVFP4
 * requantisation for the down projection fused into its epilogue (the layer of "When a
 * Benchmark Crashes", section "Why This Message Was Written": 256 experts, MoE intermediate
 * size I = 2048, gate_up N = 2 I). Per expert e and row r in [expert_offsets[e],
 * expert_offsets[e+1]), with v = alpha[e] * sum_k deq(A)[r, k] deq(B[e])[n, k] in fp32:
 *     g = v[n = j], u = v[n = I + j],  h[r, j] = (g / (1 + exp(-g))) * u     (j < I, fp32)
 * and h is quantised exactly as nvfp4_quantize does, with the fixed global scale gs_h
 * (device, one float, chosen in advance: an epilogue cannot know max|h|):
 *     h_q[total_rows, I/2] (e2m1 codes) and h_sf[total_rows, I/16] (e4m3, linear layout),
 * ready to be the A operand of the down projection (nvfp4_grouped_gemm with
 * alpha_down[e] = 1 / (gs_h * gsB_down[e])). B[E, 2I, K/2] holds the gate rows [0, I) then
 * the up rows [I, 2I) of each expert, sfB[E, 2I, K/16] likewise. The gate / up split of the
 * gate_up output and this order are the library's reading (the pages name the layer, not its
 * activation). Requires I % 64 == 0 and the nvfp4_grouped_gemm conditions; h_q 16-byte
 * aligned. Rows past expert_offsets[E] are not written. h is computed in fp32 with CUDA's
 * expf, so a code can differ from a correctly rounded fp64 evaluation where h lies next to a
 * rounding boundary.
 */
nvfp4_status nvfp4_grouped_gemm_swiglu(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                       const uint8_t* sfB, const float* alpha,
                                       const int32_t* expert_offsets, int32_t E, int64_t total_rows,
                                       int64_t I, int64_t K, const float* gs_h, uint8_t* h_q,
                                       uint8_t* h_sf, cudaStream_t stream);

/*
 * The mixture-of-experts layer around the grouped GEMMs ("When a Benchmark Crashes", section
 * "Why This Message Was Written": every token is routed to 8 of 256 experts). The pages name
 * the layer, not its router; the readings: probabilities are a softmax over the expert logits;
 * a token takes its k largest, ties going to the lower expert index, in descending order; its
 * k weights are those probabilities renormalised to sum to 1; the expert-sorted order lists
 * each expert's (token, slot) pairs in ascending token order.
 *
 * nvfp4_moe_route: logits[T, E] (fp32, device) ->
 *   experts[T, k] (int32): slot s = the s-th largest logit (exact: the selection compares the
 *                          logits themselves, which order like the probabilities);
 *   weights[T, k] (fp32):  exp(l_s - l_0) / sum_j exp(l_j - l_0) over the k winners (fp32,
 *                          CUDA's expf; within a few ulp of the exact renormalised softmax);
 *   expert_offsets[E + 1]: expert e owns rows [offsets[e], offsets[e+1]) of the sorted order;
 *   row_of[T, k]:          the sorted row that holds token t's slot s;
 *   token_of_row[T k]:     the token of every sorted row.
 * All device, int32 / fp32, 4-byte aligned. E <= 1024, k <= min(E, 32). Four launches; no
 * scratch (row_of and expert_offsets hold the ranks and counts until the last ones). Results
 * are deterministic (no atomics). T == 0 writes expert_offsets as all zero.
 */
nvfp4_status nvfp4_moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* experts,
                             float* weights, int32_t* expert_offsets, int32_t* row_of,
                             int32_t* token_of_row, cudaStream_t stream);

/*
 * Quantises the tokens x[T, H] (fp32 or bf16, row stride ld_x elements) once, exactly as
 * nvfp4_quantize_dynamic does (global scale of all of x written to gs_out[0], alpha_out[i] =
 * 1 / (gs_out[0] * gs_other[i]) for i < n_alpha, e.g. against every expert's weight scale), and
 * writes token t's codes and scales to each of its k expert-sorted rows row_of[t, s]:
 * q[T k, H/2] and sf[T k, H/16] (linear layout), the A operand of the grouped GEMM. Quantising
 * then gathering equals gathering then quantising, as rows are independent once the global
 * scale is known. One launch. Requires H % 16 == 0, k <= 32; x, q 16-byte aligned; every row
 * index in row_of below T k (as nvfp4_moe_route writes them).
 */
nvfp4_status nvfp4_moe_gather_quantize(const void* x, nvfp4_in_dtype dtype, int32_t T, int64_t H,
                                       int64_t ld_x, int32_t k, const int32_t* row_of, float* gs_out,
                                       uint8_t* q, uint8_t* sf, const float* gs_other, int32_t n_alpha,
                                       float* alpha_out, cudaStream_t stream);

/*
 * The weighted combine after the down projection: out[t, :] = sum_s weights[t, s] *
 * y[row_of[t, s], :] for t < T, accumulated in fp32 in ascending slot order (deterministic) and
 * rounded once to out_dtype. y[T k, H] holds y_dtype elements (the down GEMM's output), out
 * [T, H] out_dtype; both 16-byte aligned, H % 8 == 0, k <= 32. All device.
 */
nvfp4_status nvfp4_moe_combine(const void* y, nvfp4_out_dtype y_dtype, const float* weights,
                               const int32_t* row_of, int32_t T, int64_t H, int32_t k, void* out,
                               nvfp4_out_dtype out_dtype, cudaStream_t stream);

/*
 * nvfp4_gemm without a workspace argument and without any device allocation. The reference
 * pages have no counterpart to this call; it exists for callers that cannot allocate
 * device memory: code running inside a host framework that has reserved all device memory
 * for its own pool (a cudaMalloc there fails or fragments memory the framework manages),
 * plugin-style interfaces whose signature offers no workspace, and latency-critical paths
 * that cannot afford cudaMalloc / cudaFree because they may synchronise the device.
 *
 * Same operation, arguments, layouts and checks as nvfp4_gemm (A, sfA, B, sfB, alpha, out
 * are caller-owned device memory; the caller still passes inputs and outputs). The split-K
 * scratch comes from one fixed array inside the library, NVFP4_NOALLOC_SCRATCH_BYTES large,
 * that every GPU which loads the library holds until the process exits. A shape whose
 * split-K scratch would exceed that size returns NVFP4_ERR_WORKSPACE (nothing launched).
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress
 * with that device current), and so does the first call after the device's CUDA context was
 * created anew or from a host thread with no context bound yet; make that first call before
 * any stream capture. All calls on
 * a device share the array and it keeps the last call's contents: each call clears the part
 * that must start at zero, and calls whose kernels overlap on the GPU (other streams,
 * other host threads) race on it, so serialise them. Calls no cudaMalloc / cudaFree.
 */
#define NVFP4_NOALLOC_SCRATCH_BYTES (16u << 20)

nvfp4_status nvfp4_gemm_noalloc(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                                const uint8_t* sfB, const float* alpha, void* out,
                                int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/*
 * Tuning and test hook: forces parts of the GEMM launch plan for every later call in the
 * process, from any thread (0 = the planner's own choice for that part):
 *   bn          dense tile width along the weights: 128, 192, 224 or 256 (linear scales;
 *               NVFP4_SF_TILED accepts 128 and 256), other values ignored;
 *   cluster     split-K CTAs per thread-block cluster, 1 ... 8;
 *   groups      split-K clusters per output tile, reduced through the workspace (needs one);
 *   band        output P tiles per rasterisation band;
 *   grouped_bn  token tile width of the grouped GEMM: 32, 64, 128, 176 or 256;
 *   pair        CTA pairs computing 256-row tiles with the 2-SM MMA (tiled scales, no split-K):
 *               0 = the planner (pairs for 256-wide tiles with K >= 3072; a last wave of
 *               256 x 256 tiles that fills at most half of the pairs runs as 256 x 128
 *               halves), 1 = never, 2 = for every 256- or 128-wide tile, 3 = as 0 but
 *               without the halves; the grouped GEMM runs pairs for 128- and 176-row token
 *               tiles unless this is 1.
 * The planner's choices need no override; results stay within the GEMM tolerance under any
 * of them, and every override layout is deterministic. Negative values (pair above 3):
 * NVFP4_ERR_INVALID_ARG.
 */
nvfp4_status nvfp4_set_plan_override(int32_t bn, int32_t cluster, int32_t groups, int32_t band,
                                     int32_t grouped_bn, int32_t pair);

/*
 * Elementwise conversions used by the quantiser, exposed so that they can be checked
 * exhaustively: out[i] = e4m3_rn_satfinite(x[i]) (one byte), or e2m1_rn_satfinite(x[i])
 * (one code 0..15 per byte). x, out: device, n elements, no alignment requirement.
 */
nvfp4_status nvfp4_round_e4m3(const float* x, int64_t n, uint8_t* out, cudaStream_t stream);
nvfp4_status nvfp4_round_e2m1(const float* x, int64_t n, uint8_t* out, cudaStream_t stream);

/*
 * Diagnostic of the failure path: launches one CTA that waits, with the same bounded-wait
 * routine every kernel uses, on an mbarrier that nothing ever completes. After timeout_us
 * microseconds (1 ... 1000000) the wait gives up and the kernel records code 0x1FF in the
 * device error word and returns normally: the next nvfp4_last_device_error reports
 * NVFP4_ERR_TIMEOUT with that code, and the CUDA context stays usable. No fault, no hang.
 */
nvfp4_status nvfp4_check_bounded_wait(uint32_t timeout_us, cudaStream_t stream);

/*
 * Reads and clears the current device's error word. Synchronises `stream` first.
 * Returns NVFP4_OK if no kernel recorded an error since the last call, NVFP4_ERR_TIMEOUT
 * if one gave up on a bounded wait, NVFP4_ERR_CUDA if the read itself failed.
 * *where_out (optional, host) receives the raw code: the wait that gave up.
 */
nvfp4_status nvfp4_last_device_error(cudaStream_t stream, uint32_t* where_out);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
