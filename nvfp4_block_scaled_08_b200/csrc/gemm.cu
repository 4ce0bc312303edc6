// gemm.cu -- host side of the NVFP4 GEMMs: tile planning, TMA descriptor encoding (with a
// per-process cache) and the launch of the persistent sm_100a kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>

#include "gemm_kernel.cuh"
#include "internal.h"

namespace nvfp4 {

// ------------------------------------------------------------------ planning

// Process-wide overrides of the planner's choices (nvfp4_set_plan_override; 0 = planner).
// Plain atomics: a GEMM call reads them without a lock or a string look-up.
static std::atomic<int> g_force_bn{0}, g_force_cluster{0}, g_force_groups{0}, g_force_band{0},
    g_force_grouped_bn{0}, g_force_pair{0};

void set_plan_override(int bn, int cluster, int groups, int band, int grouped_bn, int pair)
{
    g_force_bn.store(bn, std::memory_order_relaxed);
    g_force_cluster.store(cluster, std::memory_order_relaxed);
    g_force_groups.store(groups, std::memory_order_relaxed);
    g_force_band.store(band, std::memory_order_relaxed);
    g_force_grouped_bn.store(grouped_bn, std::memory_order_relaxed);
    g_force_pair.store(pair, std::memory_order_relaxed);
}

static int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// Largest number of clusters of `cs` CTAs (one CTA per SM, as every GEMM variant here
// uses over 100 KB of shared memory) that the current device runs at once; cached per
// device. Clusters are placed inside a GPC, so this is below num_sms / cs.
static int max_active_clusters(int cs);

// Tiling for out[M, N] = A[M, K] x B[N, K]^T on `num_sms` SMs.
//  * M <= 64: weights fill the 128-row MMA operand (swap), tokens are an MMA N of 16-64.
//  * otherwise: 128-row token tiles x 128- or 256-row weight tiles, whichever finishes in
//    fewer tile-waves (wider tiles cost ~2x per tile but move less data per FLOP).
//  * split-K when the tiles cannot fill the SMs: the K stages of a tile are shared out
//    over the CTAs of one thread-block cluster (up to 8), which reduce their partial tiles
//    over distributed shared memory; the largest cluster whose clusters all run in one
//    wave is taken. Layouts with `groups` > 1 clusters per tile, which meet in the
//    workspace, are available through the overrides (and nvfp4_gemm_noalloc's scratch).
// nvfp4_set_plan_override can force the tile width, cluster size, groups and band (tuning
// and tests only).
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, bool allow_workspace, int num_sms)
{
    GemmPlan p;
    const int nk = static_cast<int>(K / 256);
    if (M <= 64) {
        p.swap = true;
        p.bn = M <= 16 ? 16 : M <= 32 ? 32 : 64;
        p.p_tiles = ceil_div(N, 128);
        p.q_tiles = ceil_div(M, p.bn);
    } else {
        p.swap = false;
        p.p_tiles = ceil_div(M, 128);
        const int t256 = p.p_tiles * ceil_div(N, 256);
        const int t128 = p.p_tiles * ceil_div(N, 128);
        const double c256 = static_cast<double>(ceil_div(t256, num_sms)) * 2.0;
        const double c128 = static_cast<double>(ceil_div(t128, num_sms)) * 1.15;
        p.bn = (N > 128 && c256 <= c128) ? 256 : 128;
        // too few 256-wide tiles to fill the GPU: split-K follows, and 128-wide tiles halve
        // the partial tile each CTA hands over (and the splits needed)
        if (p.bn == 256 && t256 * 4 < num_sms * 3 && nk >= 2) p.bn = 128;
        const int force = g_force_bn.load(std::memory_order_relaxed);
        if (force == 128 || force == 192 || force == 224 || force == 256) p.bn = force;
        p.q_tiles = ceil_div(N, p.bn);
    }
    const int tiles = p.p_tiles * p.q_tiles;
    int cs = 1, g = 1;
    if (tiles * 4 < num_sms * 3 && nk >= 2) {
        // One cluster per output tile, as many K slices per cluster as fit in one wave
        // (measured: a single cluster reduction beats any workspace round trip).
        const int s_max = std::min({8, nk, num_sms / tiles});
        for (int c = s_max; c >= 2; --c) {
            if (tiles <= max_active_clusters(c)) { cs = c; break; }
        }
    }
    const int fc = g_force_cluster.load(std::memory_order_relaxed);
    const int fg = g_force_groups.load(std::memory_order_relaxed);
    if (fc > 0 || fg > 0) {
        cs = std::max(1, std::min(fc > 0 ? fc : cs, 8));
        g = std::max(1, fg > 0 ? fg : g);
        if (!allow_workspace) g = 1;
        while (cs * g > nk && g > 1) --g;
        while (cs * g > nk && cs > 1) --cs;
    }
    // Rasterisation band. While both packed operands fit in L2 together, P-fastest order
    // over the whole grid (one band); beyond that, bands of 32 P tiles (4096 rows of A): all
    // of B streams through L2 once per band while the band's rows of A stay there. DRAM
    // bytes read by one launch on B200 (ncu), bands of 16 / 32 / 64 P tiles: 16384^3 with
    // CTA pairs 3.31 / 2.23 / 4.65 GB in 1579 / 1509 / 1663 us, single CTAs 1.57 / 1.13 GB
    // (16 / 32); 32768 x 8192 x 8192 1.36 / 0.68 / 0.69 GB in 846 / 798 / 817 us;
    // 65536 x 16384 x 4096 1.54 / 0.91 / 0.61 GB in 1861 / 1815 / 1799 us;
    // 16384 x 16384 x 32768 9.87 / 9.62 / 14.8 GB in 3401 / 3386 / 3698 us.
    const double packed_bytes = static_cast<double>(M + N) * static_cast<double>(K) * 0.5;
    p.band = packed_bytes <= 80e6 ? p.p_tiles : std::max(1, std::min(p.p_tiles, 32));
    {
        const int fb = g_force_band.load(std::memory_order_relaxed);
        if (fb > 0) p.band = std::min(p.p_tiles, fb);
    }
    p.cluster = cs;
    p.groups = g;
    p.splits = cs * g;
    p.num_tiles = tiles * p.splits;
    // split-K launches exactly one CTA per work item (the reduction relies on it)
    p.grid = p.splits > 1 ? p.num_tiles : std::min(p.num_tiles, num_sms);
    if (g > 1) {
        p.ws_counter_bytes = ((static_cast<size_t>(tiles) * cs * 4 + 255) / 256) * 256;
        p.ws_bytes = p.ws_counter_bytes + static_cast<size_t>(tiles) * g * 128 * p.bn * sizeof(float);
    }
    // CTA pairs computing 256 x 256 tiles with the 2-SM MMA (tiled scales): 256-wide Q tiles
    // without split-K, at least one pair of P tiles and at least 12 K stages; the pair's work
    // items are P tile pairs. Each SM then stages 38 KB per K step instead of 54 KB for the
    // same MMA work. Measured on B200: 16384^3 in 1528-1577 us against 1771-1850 us, 8192^3 in
    // 193-194 us against 215-224 us, 4096^3 in 30.3 us against 32.7 us, 8192 x 4096 x 6144 in
    // 77.6 us against 84.5 us; with 8 K stages (4096 x 6144 x 2048) single CTAs win, 28.8
    // against 30.8 us. 256 x 128 pair tiles (the override with bn = 128) lost to 256 x 256
    // ones on every shape measured.
    // 1: off, 2: wherever possible, 3: the planner's pairs without half tiles
    const int fp = g_force_pair.load(std::memory_order_relaxed);
    const bool pair_shape = !p.swap && p.splits == 1 && p.p_tiles >= 2;
    p.pair = pair_shape && (((fp == 0 || fp == 3) && p.bn == 256 && nk >= 12) || (fp == 2 && (p.bn == 256 || p.bn == 128)));
    if (p.pair) {
        const int pairs = ((p.p_tiles + 1) / 2) * p.q_tiles;
        const int clusters = std::max(1, std::min(pairs, max_active_clusters(2)));
        p.pair_grid = 2 * clusters;
        p.pair_band = std::max(1, p.band / 2);
        // A last wave of 256 x 256 tiles that fills at most half of the pairs runs as twice
        // as many 256 x 128 halves, in about half the time (4096^3: 256 tiles on 74 pairs,
        // 3.46 rounds).
        const int tail = pairs % clusters;
        p.pair_items = pairs;
        p.narrow_from = pairs;
        if (p.bn == 256 && tail > 0 && 2 * tail <= clusters && fp != 3) {
            p.narrow_from = pairs - tail;
            p.pair_items = pairs + tail;
        }
    }
    return p;
}

// Grouped: weights always fill the MMA M; the token tile width follows the mean rows per
// expert (the actual per-tile MMA N is rounded up from the rows present, on the device).
GemmPlan plan_grouped(int32_t E, int64_t total_rows, int64_t N, int64_t K, int num_sms)
{
    (void)K;
    GemmPlan p;
    p.grouped = true;
    p.swap = true;
    // 176-row tiles cover experts of up to 176 rows in one tile with a 44 KB stage (5 deep)
    // where 256-row tiles need 54 KB (4 deep): more weight bytes in flight per SM
    const int64_t avg = E > 0 ? total_rows / E : 0;
    p.bn = avg <= 24 ? 32 : avg <= 48 ? 64 : avg <= 96 ? 128 : avg <= 140 ? 176 : 256;
    const int force = g_force_grouped_bn.load(std::memory_order_relaxed);
    if (force == 32 || force == 64 || force == 128 || force == 176 || force == 256) p.bn = force;
    p.p_tiles = ceil_div(N, 128);
    p.splits = 1;
    p.grid = num_sms;
    // CTA pairs for 128- and 176-row token tiles (about 100 or more rows per expert): two CTAs
    // share a token tile, each holding 128 weight rows of a 256-row pair and half of the
    // tokens, so a stage is 33 KB per SM instead of 44 KB (6 deep instead of 5) for the same
    // MMA work. Measured on B200 (T = 4096, 256 experts): down 434 -> 404 us, gate_up 735 ->
    // 673-680 us. Plan override pair = 1 switches them off.
    const int fp = g_force_pair.load(std::memory_order_relaxed);
    p.pair = fp != 1 && (p.bn == 128 || p.bn == 176) && p.p_tiles >= 2;
    if (p.pair) p.pair_grid = 2 * std::max(1, max_active_clusters(2));
    return p;
}

// ------------------------------------------------------------------ TMA descriptors

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

struct MapKey {
    std::array<uint64_t, 18> v;
    bool operator<(const MapKey& o) const { return v < o.v; }
};

static std::mutex g_map_mu;
static std::map<MapKey, CUtensorMap> g_map_cache;

// uint8 tensor of `rank` (2 ... 5) dims (innermost first: dims[0] bytes per row), strides of
// dims 1 .. rank-1 in bytes, box extents per dim; cached per (pointer, geometry, device).
static bool get_map_nd(CUtensorMap* out, const void* ptr, int rank, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box, bool swizzle128)
{
    int dev = 0;
    cudaGetDevice(&dev);
    MapKey key;
    key.v.fill(0);
    key.v[0] = reinterpret_cast<uint64_t>(ptr);
    key.v[1] = static_cast<uint64_t>(rank) | (swizzle128 ? 0x100ull : 0ull) | (static_cast<uint64_t>(dev) << 16);
    for (int i = 0; i < rank; ++i) {
        key.v[2 + i] = dims[i];
        key.v[7 + i] = box[i];
        if (i + 1 < rank) key.v[12 + i] = strides[i];
    }
    {
        std::lock_guard<std::mutex> g(g_map_mu);
        auto it = g_map_cache.find(key);
        if (it != g_map_cache.end()) {
            *out = it->second;
            return true;
        }
    }
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5];
    cuuint64_t st[4];
    cuuint32_t bx[5];
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        if (i + 1 < rank) st[i] = strides[i];
    }
    CUtensorMap m;
    std::memset(&m, 0, sizeof(m));
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<cuuint32_t>(rank), const_cast<void*>(ptr), d,
                    st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    {
        std::lock_guard<std::mutex> g(g_map_mu);
        if (g_map_cache.size() > 8192) g_map_cache.clear();
        g_map_cache[key] = m;
    }
    *out = m;
    return true;
}

// uint8 tensor of `rank` (2 or 3) dims {inner bytes, rows[, depth]} with row stride
// `stride1` and depth stride `stride2` (bytes); box {box0, box1[, 1]}.
static bool get_map(CUtensorMap* out, const void* ptr, int rank, uint64_t d0, uint64_t d1,
                    uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1,
                    bool swizzle128)
{
    const uint64_t dims[3] = {d0, d1, d2};
    const uint64_t strides[2] = {stride1, stride2};
    const uint32_t box[3] = {box0, box1, 1};
    return get_map_nd(out, ptr, rank, dims, strides, box, swizzle128);
}

// The gate_up weights [E, 2I, row_bytes] viewed so that one box of 128 rows holds four groups of
// [16 gate rows j .. j + 15, the 16 up rows I + j .. I + j + 15]: dims (innermost first)
// {row_bytes, 16 rows, gate/up, I / 16 groups, E}, strides {row_bytes, I rows, 16 rows,
// 2I rows}, box {box0, 16, 2, 4, 1}.
static bool get_map_swiglu(CUtensorMap* out, const void* ptr, uint64_t row_bytes, uint64_t I, uint64_t E,
                           uint32_t box0, bool swizzle128)
{
    const uint64_t dims[5] = {row_bytes, 16, 2, I / 16, E};
    const uint64_t strides[4] = {row_bytes, I * row_bytes, 16 * row_bytes, 2 * I * row_bytes};
    const uint32_t box[5] = {box0, 16, 2, 4, 1};
    return get_map_nd(out, ptr, 5, dims, strides, box, swizzle128);
}

// ------------------------------------------------------------------ launch

constexpr int kMaxDevicesForAttr = 64;

static int max_active_clusters(int cs)
{
    static std::mutex mu;
    static int cache[kMaxDevicesForAttr][9];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesForAttr || cs < 1 || cs > 8) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> g(mu);
    if (cache[dev][cs] == 0) {
        // any GEMM variant gives the same answer: all use one CTA per SM
        using Cfg = GemmCfg<128, false, false>;
        auto kern = nvfp4_gemm_kernel<Cfg>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = cs;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3(cs * 64, 1, 1);
        cfg.blockDim = dim3(kGemmThreads, 1, 1);
        cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][cs] = n > 0 ? n : -1;
    }
    return cache[dev][cs] > 0 ? cache[dev][cs] : 0;
}

template <int BN, bool SWAP, bool GROUPED, bool SFT = false, bool SWIGLU = false, bool MX = false,
          bool PAIR = false, bool ACTQ = false>
static cudaError_t run(const GemmPlan& plan, const GemmLaunch& L, cudaStream_t stream,
                       bool* encode_failed)
{
    using Cfg = GemmCfg<BN, SWAP, GROUPED, SFT, SWIGLU, MX, PAIR, ACTQ>;
    auto kern = nvfp4_gemm_kernel<Cfg>;
    // Opt in to the large dynamic shared memory once per device (not a stream operation,
    // so a later launch may be captured into a CUDA graph).
    static std::once_flag attr_once[kMaxDevicesForAttr];
    static cudaError_t attr_err[kMaxDevicesForAttr];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevicesForAttr) return cudaErrorInvalidDevice;
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg::SMEM_BYTES);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];

    const uint64_t kb = static_cast<uint64_t>(L.K / 2);    // packed bytes per row
    const uint64_t ks = static_cast<uint64_t>(L.K / 16);   // scale bytes per row
    CUtensorMap tp, tq, tsp, tsq, tq_half;
    bool ok = true;
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.cluster_size = 1;
    a.groups = 1;
    a.M = static_cast<int32_t>(L.M);
    a.N = static_cast<int32_t>(L.N);
    a.num_kstages = static_cast<int32_t>(L.K / 256);
    a.num_p_tiles = plan.p_tiles;
    a.out = L.out;
    a.out_dtype = L.out_dtype;
    a.alpha = L.alpha;
    a.err_word = L.err_word;
    a.b_ready = L.b_ready ? 1 : 0;
    if constexpr (GROUPED) {
        const uint64_t E = static_cast<uint64_t>(L.E);
        const uint64_t rows = static_cast<uint64_t>(L.total_rows);
        if constexpr (SWIGLU) {
            const uint64_t I = static_cast<uint64_t>(L.N / 2);
            ok &= get_map_swiglu(&tp, L.B, kb, I, E, 128, true);
            ok &= get_map_swiglu(&tsp, L.sfB, ks, I, E, 16, false);
            a.h_q = L.h_q;
            a.h_sf = L.h_sf;
            a.gs_h = L.gs_h;
            a.inter = static_cast<int32_t>(I);
        } else {
            ok &= get_map(&tp, L.B, 3, kb, L.N, E, kb, kb * L.N, 128, 128, true);
            ok &= get_map(&tsp, L.sfB, 3, ks, L.N, E, ks, ks * L.N, 16, 128, false);
        }
        ok &= get_map(&tq, L.A, 2, kb, rows, 1, kb, 0, 128, Cfg::QBOX, true);
        ok &= get_map(&tsq, L.sfA, 2, ks, rows, 1, ks, 0, 16, Cfg::QBOX, false);
        a.p_rows = a.N;
        a.q_rows = static_cast<int32_t>(L.total_rows);
        a.splits = 1;
        if constexpr (PAIR) a.num_p_tiles = static_cast<int32_t>((L.N + 255) / 256);   // weight tile pairs
        a.expert_offsets = L.offsets;
        a.num_experts = L.E;
        a.total_rows = static_cast<int32_t>(L.total_rows);
    } else {
        const uint8_t* P = SWAP ? L.B : L.A;
        const uint8_t* sP = SWAP ? L.sfB : L.sfA;
        const uint8_t* Q = SWAP ? L.A : L.B;
        const uint8_t* sQ = SWAP ? L.sfA : L.sfB;
        const uint64_t p_rows = static_cast<uint64_t>(SWAP ? L.N : L.M);
        const uint64_t q_rows = static_cast<uint64_t>(SWAP ? L.M : L.N);
        ok &= get_map(&tp, P, 2, kb, p_rows, 1, kb, 0, 128, 128, true);
        if constexpr (ACTQ) tq = tp;          // unused: the kernel quantises the activations itself
        else ok &= get_map(&tq, Q, 2, kb, q_rows, 1, kb, 0, 128, PAIR ? BN / 2 : BN, true);   // PAIR: half tiles
        // PAIR, BN = 256: each CTA's 64 rows of a 256 x 128 half tile
        if constexpr (Cfg::NARROW) ok &= get_map(&tq_half, Q, 2, kb, q_rows, 1, kb, 0, 128, BN / 4, true);
        if constexpr (PAIR) {
            // the tiled scales as rows of 256 bytes: a stage's run of one 128-row tile is
            // SFP_BYTES / 256 rows (past the last tile: zero fill)
            const uint64_t sp_rows = (p_rows + 127) / 128 * (L.K / (MX ? 64 : 32));
            const uint64_t sq_rows = (q_rows + 127) / 128 * (L.K / (MX ? 64 : 32));
            ok &= get_map(&tsp, sP, 2, 256, sp_rows, 1, 256, 0, 256, Cfg::SF_ROWS256, false);
            ok &= get_map(&tsq, sQ, 2, 256, sq_rows, 1, 256, 0, 256, Cfg::SF_ROWS256, false);
            a.sf_p = sP;
            a.sf_q = sQ;
            a.sf_kb4 = static_cast<int32_t>(L.K / (MX ? 128 : 64));
        } else if constexpr (SFT) {
            tsp = tp;                       // unused: the scales come by bulk copy
            tsq = tq;
            a.sf_p = sP;
            a.sf_q = sQ;
            a.sf_kb4 = static_cast<int32_t>(L.K / (MX ? 128 : 64));   // 512-byte blocks per 128 rows
        } else if (L.sf_8x4) {
            // rows of the map: 8-row groups of K / 2 bytes; a stage's box: 128 bytes of 128 / 8
            // (P) or BN / 8 (Q) groups, the same bytes as the row-major box
            const uint64_t gb = static_cast<uint64_t>(L.K / 2);
            ok &= get_map(&tsp, sP, 2, gb, (p_rows + 7) / 8, 1, gb, 0, 128, 128 / 8, false);
            ok &= get_map(&tsq, sQ, 2, gb, (q_rows + 7) / 8, 1, gb, 0, 128, BN / 8, false);
            a.sf_8x4 = 1;
        } else {
            ok &= get_map(&tsp, sP, 2, ks, p_rows, 1, ks, 0, 16, 128, false);
            ok &= get_map(&tsq, sQ, 2, ks, q_rows, 1, ks, 0, 16, BN, false);
        }
        a.p_rows = static_cast<int32_t>(p_rows);
        a.q_rows = static_cast<int32_t>(q_rows);
        if constexpr (ACTQ) {
            a.act = L.act;
            a.act_ld = L.act_ld;
            a.act_bf16 = L.act_bf16 ? 1 : 0;
            a.gs_b = L.gs_b;
            a.gs_out = L.gs_out;
            a.alpha_out = L.alpha_out;
        }
        a.num_q_tiles = plan.q_tiles;
        if constexpr (PAIR) a.num_p_tiles = (plan.p_tiles + 1) / 2;   // work items are P tile pairs
        a.splits = plan.splits;
        a.cluster_size = plan.cluster;
        a.groups = plan.groups;
        a.num_tiles = plan.num_tiles;
        a.band = plan.band;
        if (plan.groups > 1) {
            a.ws_counters = static_cast<uint32_t*>(L.ws);
            a.ws_partial = reinterpret_cast<float*>(static_cast<uint8_t*>(L.ws) + plan.ws_counter_bytes);
        }
    }
    if constexpr (!Cfg::NARROW) tq_half = tq;   // unused
    if (!ok) {
        *encode_failed = true;
        return cudaSuccess;
    }
    if constexpr (PAIR) {
        a.band = plan.pair_band;
        a.num_tiles = plan.pair_items;
        a.narrow_from = plan.narrow_from;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(PAIR ? plan.pair_grid : plan.grid), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = stream;
    // programmatic dependent launch: the prologue overlaps the previous kernel's tail
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = static_cast<unsigned>(plan.cluster);
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
    if constexpr (PAIR) attrs[1].val.clusterDim.x = 2;
    cfg.attrs = attrs;
    cfg.numAttrs = (PAIR || (!GROUPED && plan.cluster > 1)) ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, tp, tq, tsp, tsq, tq_half, a);
}

int act_gemm_stages(int bn)
{
    switch (bn) {
        case 16: return GemmCfg<16, true, false, true, false, false, false, true>::STAGES;
        case 32: return GemmCfg<32, true, false, true, false, false, false, true>::STAGES;
        case 64: return GemmCfg<64, true, false, true, false, false, false, true>::STAGES;
        default: return 0;
    }
}

cudaError_t launch_gemm(const GemmPlan& plan, const GemmLaunch& L, cudaStream_t stream,
                        bool* encode_failed)
{
    *encode_failed = false;
    if (plan.grid <= 0) return cudaSuccess;
    if (L.act) {
        if (!plan.swap || plan.q_tiles != 1 || plan.groups != 1 || !L.sf_tiled || L.mx) return cudaErrorInvalidValue;
        switch (plan.bn) {
            case 16: return run<16, true, false, true, false, false, false, true>(plan, L, stream, encode_failed);
            case 32: return run<32, true, false, true, false, false, false, true>(plan, L, stream, encode_failed);
            case 64: return run<64, true, false, true, false, false, false, true>(plan, L, stream, encode_failed);
            default: return cudaErrorInvalidValue;
        }
    }
    if (L.mx) {
        if (plan.grouped || !L.sf_tiled) return cudaErrorInvalidValue;
        if (plan.swap) {
            if (plan.q_tiles != 1) return cudaErrorInvalidValue;   // Q tile at row 0
            switch (plan.bn) {
                case 16: return run<16, true, false, true, false, true>(plan, L, stream, encode_failed);
                case 32: return run<32, true, false, true, false, true>(plan, L, stream, encode_failed);
                case 64: return run<64, true, false, true, false, true>(plan, L, stream, encode_failed);
                default: return cudaErrorInvalidValue;
            }
        }
        if (plan.pair && plan.bn == 256)
            return run<256, false, false, true, false, true, true>(plan, L, stream, encode_failed);
        if (plan.pair && plan.bn == 128)
            return run<128, false, false, true, false, true, true>(plan, L, stream, encode_failed);
        switch (plan.bn) {
            case 128: return run<128, false, false, true, false, true>(plan, L, stream, encode_failed);
            case 256: return run<256, false, false, true, false, true>(plan, L, stream, encode_failed);
            default: return cudaErrorInvalidValue;
        }
    }
    if (L.sf_8x4 && (plan.grouped || L.sf_tiled || L.h_q != nullptr)) return cudaErrorInvalidValue;
    if (L.sf_tiled) {
        if (plan.grouped) return cudaErrorInvalidValue;
        if (plan.swap) {
            if (plan.q_tiles != 1) return cudaErrorInvalidValue;   // Q tile at row 0
            switch (plan.bn) {
                case 16: return run<16, true, false, true>(plan, L, stream, encode_failed);
                case 32: return run<32, true, false, true>(plan, L, stream, encode_failed);
                case 64: return run<64, true, false, true>(plan, L, stream, encode_failed);
                default: return cudaErrorInvalidValue;
            }
        }
        if (plan.pair && plan.bn == 256)
            return run<256, false, false, true, false, false, true>(plan, L, stream, encode_failed);
        if (plan.pair && plan.bn == 128)
            return run<128, false, false, true, false, false, true>(plan, L, stream, encode_failed);
        switch (plan.bn) {
            case 128: return run<128, false, false, true>(plan, L, stream, encode_failed);
            case 256: return run<256, false, false, true>(plan, L, stream, encode_failed);
            default: return cudaErrorInvalidValue;      // 192 / 224 tiles: linear scales only
        }
    }
    if (plan.grouped && L.h_q != nullptr && plan.pair) {
        if (plan.bn == 128) return run<128, true, true, false, true, false, true>(plan, L, stream, encode_failed);
        if (plan.bn == 176) return run<176, true, true, false, true, false, true>(plan, L, stream, encode_failed);
        return cudaErrorInvalidValue;
    }
    if (plan.grouped && L.h_q != nullptr) {
        switch (plan.bn) {
            case 32: return run<32, true, true, false, true>(plan, L, stream, encode_failed);
            case 64: return run<64, true, true, false, true>(plan, L, stream, encode_failed);
            case 128: return run<128, true, true, false, true>(plan, L, stream, encode_failed);
            case 176: return run<176, true, true, false, true>(plan, L, stream, encode_failed);
            case 256: return run<256, true, true, false, true>(plan, L, stream, encode_failed);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.grouped && plan.pair) {
        if (plan.bn == 128) return run<128, true, true, false, false, false, true>(plan, L, stream, encode_failed);
        if (plan.bn == 176) return run<176, true, true, false, false, false, true>(plan, L, stream, encode_failed);
        return cudaErrorInvalidValue;
    }
    if (plan.grouped) {
        switch (plan.bn) {
            case 32: return run<32, true, true>(plan, L, stream, encode_failed);
            case 64: return run<64, true, true>(plan, L, stream, encode_failed);
            case 128: return run<128, true, true>(plan, L, stream, encode_failed);
            case 176: return run<176, true, true>(plan, L, stream, encode_failed);
            case 256: return run<256, true, true>(plan, L, stream, encode_failed);
            default: return cudaErrorInvalidValue;
        }
    }
    if (plan.swap) {
        switch (plan.bn) {
            case 16: return run<16, true, false>(plan, L, stream, encode_failed);
            case 32: return run<32, true, false>(plan, L, stream, encode_failed);
            case 64: return run<64, true, false>(plan, L, stream, encode_failed);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (plan.bn) {
        case 128: return run<128, false, false>(plan, L, stream, encode_failed);
        case 192: return run<192, false, false>(plan, L, stream, encode_failed);
        case 224: return run<224, false, false>(plan, L, stream, encode_failed);
        case 256: return run<256, false, false>(plan, L, stream, encode_failed);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace nvfp4
