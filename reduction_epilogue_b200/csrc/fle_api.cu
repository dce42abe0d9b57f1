// fle_api.cu -- the C ABI of libfle (declared in include/fle.h): argument
// checks, launch planning, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "fle.h"
#include "fle_testing.h"
#include "fle_kernel.cuh"
#include "fle_kernel_pair.cuh"

namespace {

using fle::KParams;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool probed = false;
    bool ok = false;
    int sms = 0;
    int pairs = 0;    // co-resident CTA pairs of the TF32 pair kernel (0: unavailable)
    int pairs3x = 0;  // and of the 3xTF32 pair kernel
};

// Co-resident 2-CTA clusters of a pair kernel on the current device.
template <int PREC>
int max_active_pairs() {
    auto kern = fle::fle_gemm_pair_kernel<PREC, 1, fle::kPairBN, false>;
    const int smem = fle::PairCfg<PREC, 1>::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(fle::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FLE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FLE_ERR_CUDA;
        d.probed = true;
        d.ok = (major == 10 && minor == 0);
        d.sms = sms;
        d.pairs = d.ok ? max_active_pairs<fle::kPrecTF32>() : 0;
        d.pairs3x = d.ok ? max_active_pairs<fle::kPrec3xTF32>() : 0;
    }
    if (!d.ok) return FLE_ERR_ARCH;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return FLE_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = d;
    return FLE_OK;
}

// 2-D fp32 K-major operand [rows, K]: box of 32 fp32 (128 bytes) along K by
// box_rows rows, 128-byte swizzle, out-of-range elements read as zero.
int encode_operand(CUtensorMap* map, const float* base, int64_t rows, int64_t K, int box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * sizeof(float)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(fle::kBK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FLE_OK : FLE_ERR_CUDA;
}

// 2-D fp32 output [rows, cols] for epilogue TMA stores: box of 32 columns
// (128 bytes) by 32 rows, 128-byte swizzle; out-of-range elements are not
// written.
int encode_output(CUtensorMap* map, float* base, int64_t rows, int64_t cols) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * sizeof(float)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FLE_OK : FLE_ERR_CUDA;
}

bool is_pow2_upto32(int k) { return k == 1 || k == 2 || k == 4 || k == 8 || k == 16 || k == 32; }

int check_desc(const fle_epilogue_desc* d) {
    if (!d) return FLE_ERR_NULL;
    if (d->kind < FLE_EPI_SCALE_HARDTANH_GELU || d->kind > FLE_EPI_NONE) return FLE_ERR_DESC;
    if (d->precision != FLE_PREC_3XTF32 && d->precision != FLE_PREC_TF32) return FLE_ERR_DESC;
    if (d->flags & ~(FLE_FLAG_GELU_TANH | FLE_FLAG_FOLD_SCALE)) return FLE_ERR_DESC;
    if (d->kind != FLE_EPI_NONE && !std::isfinite(d->scale)) return FLE_ERR_DESC;
    if (d->kind == FLE_EPI_SCALE_HARDTANH_GELU) {
        if (!std::isfinite(d->clamp_lo) || !std::isfinite(d->clamp_hi) || d->clamp_lo > d->clamp_hi)
            return FLE_ERR_DESC;
    }
    if (d->kind == FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX) {
        if (!is_pow2_upto32(d->pool_k) || d->pool_stride != d->pool_k) return FLE_ERR_DESC;
    }
    return FLE_OK;
}

int check_shape(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d) {
    const int64_t lim = (int64_t(1) << 31);
    if (M < 0 || K < 0 || N < 0 || M >= lim || K >= lim || N >= lim) return FLE_ERR_SHAPE;
    // 2^40 outputs (4 TiB of fp32) is far beyond any device; below it every
    // tile count of every plan fits an int
    if (M * N >= (int64_t(1) << 40)) return FLE_ERR_SHAPE;
    if (d->kind == FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX && N < d->pool_k) return FLE_ERR_SHAPE;
    if (K % 4 != 0) return FLE_ERR_ALIGN;
    return FLE_OK;
}

struct Plan {
    bool swap = false;
    bool pair = false;         // tiles of 256 A rows on CTA pairs (cta_group::2)
    int kps = 1;               // k-blocks per ring stage
    int bk = 32;               // k-block width in fp32
    int bn = 256;
    int prec = fle::kPrecTF32;
    int stages = 0;
    int tiles_a = 0, tiles_b = 0, tiles = 0;
    int num_kb = 0;
    int dp_tiles = 0;          // tiles done whole, one CTA each
    int64_t sk_iters = 0;      // k-blocks of the remaining tiles, spread over sk_grid CTAs
    int sk_tiles = 0;
    int sk_grid = 0;
    int sk_slots = 2;          // partial slots per stream-K CTA: 1 when every CTA holds one shared tile
    int grid = 0;
    size_t partial_bytes = 0;  // workspace: 2 partial tiles per CTA ...
    size_t ws_bytes = 0;       // ... then one arrival counter per stream-K tile
    // mixed widths (512-wide pair kernel): mix_wide 512-wide tiles, then
    // mix_narrow 384-wide ones; per panel, mix_a[r] and mix_b[r] of them
    int mix_wide = 0, mix_narrow = 0;
    unsigned char mix_a[fle::kMaxMixPanels] = {};
    unsigned char mix_b[fle::kMaxMixPanels] = {};
    // 3xTF32: the low parts of x written once into the workspace (at
    // lo_offset, M x K fp32) by a pre-pass and copied with the tiles
    bool lo_mem = false;
    size_t lo_offset = 0;
};

// Ring depth of the single-CTA kernel (mirrors Cfg::kStages).
int stages_for(int bn, int prec, int kps) {
    const int stage = kps * (fle::kBM + bn) * fle::kBK * 4 * (prec == fle::kPrec3xTF32 ? 2 : 1);
    const int s = (fle::kSmemStageBudget - fle::kEpiWarps * fle::kEpiTileBytes) / stage;
    return s > 8 ? 8 : s;
}

// Ring depth of the pair kernel (mirrors PairCfg::kStages).
int pair_stages_for(int bn, int prec, int kps) {
    const int stage = kps * (fle::kBM + bn / 2) * fle::kBK * 4 * (prec == fle::kPrec3xTF32 ? 2 : 1);
    const int s = (fle::kSmemStageBudget - fle::kEpiWarps * fle::kEpiTileBytes) / stage;
    return s > 12 ? 12 : s;
}

// Fewest k-blocks (of 32) a CTA takes in the stream-K part of a schedule.
constexpr int64_t kMinSkIters = 16;

const char* sched_override() {
    static const char* v = [] {
        const char* e = std::getenv("FLE_SCHED");
        return e ? e : "";
    }();
    return v;
}

// k-blocks per ring stage: FLE_KPS=1 or 2 overrides the planner's choice
// (single-pass TF32 only; 3xTF32 stages hold one k-block).
int kps_override() {
    static int v = [] {
        const char* e = std::getenv("FLE_KPS");
        return (e && (e[0] == '1' || e[0] == '2')) ? e[0] - '0' : 0;
    }();
    return v;
}

// FLE_GELU_POLY=0 keeps the rational erf for epilogue (a) (comparisons).
bool poly_disabled() {
    static bool off = [] {
        const char* e = std::getenv("FLE_GELU_POLY");
        return e && e[0] == '0';
    }();
    return off;
}

// FLE_PAIR_BN=224, 256 or 512 fixes the direct pair tile's width (comparisons).
int pair_bn_override() {
    static int v = [] {
        const char* e = std::getenv("FLE_PAIR_BN");
        const int n = e ? std::atoi(e) : 0;
        return (n == fle::kPairBN || n == fle::kPairBNNarrow || n == fle::kPairBNWide) ? n : 0;
    }();
    return v;
}

// FLE_LO_MEM=0 keeps 3xTF32's low parts of x inside the GEMM (comparisons).
bool lo_mem_disabled() {
    static bool off = [] {
        const char* e = std::getenv("FLE_LO_MEM");
        return e && e[0] == '0';
    }();
    return off;
}

// FLE_MIX=0 keeps the 512-wide plans on a uniform grid (comparisons).
bool mix_disabled() {
    static bool off = [] {
        const char* e = std::getenv("FLE_MIX");
        return e && e[0] == '0';
    }();
    return off;
}

// Mixed widths for a 512-wide plan of more than one wave on G pairs: each
// 256-row panel r is cut into a[r] tiles 512 wide, then b[r] = ceil((N -
// 512 a[r]) / 384) tiles 384 wide, with at most G tiles of each width, so
// that every pair runs at most one of each.  The cut takes one or two values
// of a[r] (n1 panels at a1, the rest at a2): the most 512-wide tiles, then
// the most even split, so that the tiles of each wave share operand rows
// across panels.  Returns false when there is no such cut.
bool mixed_cut(int64_t panels, int64_t N, int64_t G, unsigned char* a_out, unsigned char* b_out, int* n_wide,
               int* n_narrow) {
    if (panels < 1 || panels > fle::kMaxMixPanels || G < 1) return false;
    const int64_t A = (N + fle::kMixWide - 1) / fle::kMixWide;
    // at most one tile of each width per pair: no cut exists beyond 2G tiles
    // of 512 (this also bounds the search below: A <= 2G / panels)
    if (A > 255 || panels * A > 2 * G) return false;
    auto b_of = [&](int64_t a) {
        const int64_t rest = N - fle::kMixWide * a;
        return rest > 0 ? (rest + fle::kMixNarrow - 1) / fle::kMixNarrow : int64_t(0);
    };
    int64_t best_wide = -1, best_spread = 0, best_a1 = 0, best_a2 = 0, best_n1 = 0;
    for (int64_t a1 = 0; a1 <= A; ++a1)
        for (int64_t a2 = a1; a2 <= A; ++a2)
            for (int64_t n1 = (a1 == a2 ? panels : 1); n1 <= (a1 == a2 ? panels : panels - 1); ++n1) {
                const int64_t wide = n1 * a1 + (panels - n1) * a2;
                const int64_t narrow = n1 * b_of(a1) + (panels - n1) * b_of(a2);
                if (wide > G || narrow > G || b_of(a1) > 255) continue;
                const int64_t spread = a2 - a1;
                if (wide > best_wide || (wide == best_wide && spread < best_spread)) {
                    best_wide = wide;
                    best_spread = spread;
                    best_a1 = a1;
                    best_a2 = a2;
                    best_n1 = n1;
                }
            }
    if (best_wide < 0) return false;
    int narrow = 0;
    for (int64_t r = 0; r < panels; ++r) {
        const int64_t a = r < best_n1 ? best_a1 : best_a2;
        a_out[r] = static_cast<unsigned char>(a);
        b_out[r] = static_cast<unsigned char>(b_of(a));
        narrow += b_out[r];
    }
    *n_wide = static_cast<int>(best_wide);
    *n_narrow = narrow;
    return true;
}

// FLE_PAIR=0 keeps every plan on one-CTA tiles; FLE_PAIR=1 puts every
// swapped plan on CTA pairs (comparisons).
int pair_override() {
    static int v = [] {
        const char* e = std::getenv("FLE_PAIR");
        return (e && (e[0] == '0' || e[0] == '1')) ? e[0] - '0' : -1;
    }();
    return v;
}
bool pair_disabled() { return pair_override() == 0; }

// Waves of a plan of T tiles on G (pairs of) CTAs in units of one tile's
// time, counting the last partial wave of R tiles as 1/S when make_plan
// splits it S ways (S >= 2, k-aligned parts), as R/G when it spreads that
// wave's k-blocks over all G (spread: the 3xTF32 rule of make_plan), else as
// a whole wave.
double plan_waves(int64_t T, int64_t G, int num_kb, int64_t min_iters, bool spread) {
    const int64_t R = T % G;
    double w = static_cast<double>(T / G);
    if (R == 0) return w;
    if (num_kb < 4 * min_iters) return w + 1.0;
    const int64_t S = std::min<int64_t>(G / R, num_kb / min_iters);
    if (S >= 2) return w + 1.0 / static_cast<double>(S);
    if (spread && T > G && T < 2 * G) return w + static_cast<double>(R) / static_cast<double>(G);
    return w + 1.0;
}

// sms: SMs of the device; pairs: co-resident CTA pairs of the pair kernel.
// lo_mem: 3xTF32 plans may keep x's low parts in the workspace (the fastest
// plan); without it their split warps compute them for every tile.
Plan make_plan(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d, int sms, int pairs,
               bool lo_mem = true);
Plan make_plan_core(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d, int sms, int pairs) {
    Plan pl;
    pl.prec = (d->precision == FLE_PREC_3XTF32) ? fle::kPrec3xTF32 : fle::kPrecTF32;
    pl.swap = (M <= 128) && d->kind != FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX;
    // CTA pairs: 256 A rows per tile, each CTA loading half of the B rows.
    // Swapped (skinny) shapes use them in TF32 when the weight has at least
    // a full wave of 256-row tiles (measured: the pair kernel then streams
    // the weight faster; with fewer tiles, or in 3xTF32, the one-CTA kernel
    // is faster).
    const bool pairs_ok = pairs > 0 && !pair_disabled();
    if (pl.swap)
        pl.pair = pairs_ok && ((pl.prec == fle::kPrecTF32 && (N + fle::kPairBM - 1) / fle::kPairBM >= pairs) ||
                               pair_override() == 1);
    else
        pl.pair = pairs_ok && M > 128;
    int tile_m = pl.pair ? fle::kPairBM : fle::kBM;
    // the stream-K minimum is 16 k-blocks of 32 (512 of K) per CTA
    // (FLE_MIN_KB overrides it for comparisons)
    static const int64_t min_kb_env = [] {
        const char* e = std::getenv("FLE_MIN_KB");
        const long v = e ? std::atol(e) : 0;
        return static_cast<int64_t>(v > 0 ? v : 0);
    }();
    const int64_t min_iters = min_kb_env > 0 ? min_kb_env : kMinSkIters;
    const int num_kb = static_cast<int>((K + fle::kBK - 1) / fle::kBK);
    if (pl.swap) {
        pl.bn = M <= 32 ? 32 : (M <= 64 ? 64 : 128);
    } else if (pl.pair) {
        // 256, 224 or 512 B rows per pair tile.  A plan's time is estimated
        // as columns per tile x waves on the pairs (plan_waves).
        // - 224 when it fills the waves enough better: 1024 x 8192 x 8192
        //   is 128 tiles of 256 = 2 waves on 74 pairs, or 148 tiles of 224
        //   = 2 full waves, 12.5% fewer columns per pair.  (In 3xTF32 a
        //   256-wide plan that spreads its uneven last wave over all pairs
        //   measured faster than the two whole waves of 224: 805 against
        //   850 us on 1024 x 8192 x 8192.)
        // - 512 (TF32): two 256-wide MMAs share each A tile, so a column
        //   costs 0.86 of a 256-wide one (measured per wave: 184 against
        //   2 x 107 us on 2048 x 8192 x 8192), with one TMEM accumulator and
        //   512-column partials, whose split last wave costs a quarter wave
        //   more.  Taken when at least 1.5% faster by this estimate:
        //   2048, 4096 and 1024 x 8192 x 8192 (measured -1.1%, -2.2%, -3.5%);
        //   not 256 x 8192 x 8192 (16 tiles split four ways: slower).
        const int64_t ta = (M + fle::kPairBM - 1) / fle::kPairBM;
        const int64_t G = pairs;
        const bool spread = pl.prec == fle::kPrec3xTF32;
        auto tiles_of = [&](int bn) { return ta * ((N + bn - 1) / bn); };
        const double c256 = fle::kPairBN * plan_waves(tiles_of(fle::kPairBN), G, num_kb, min_iters, spread);
        const double c224 =
            fle::kPairBNNarrow * plan_waves(tiles_of(fle::kPairBNNarrow), G, num_kb, min_iters, spread);
        pl.bn = (c224 < 0.97 * c256) ? fle::kPairBNNarrow : fle::kPairBN;
        if (pl.prec == fle::kPrecTF32) {
            const int64_t Tw = tiles_of(fle::kPairBNWide);
            double ww = plan_waves(Tw, G, num_kb, min_iters, false);
            if (Tw % G != 0 && ww != std::floor(ww)) ww += 0.25;  // split last wave of wide partials
            const double c512 = 0.86 * fle::kPairBNWide * ww;
            if (c512 < 0.985 * std::min(c256, c224)) pl.bn = fle::kPairBNWide;
            // Mixed widths: a plan of more than one wave of 512-wide tiles
            // whose last wave is short (2048 x 8192 x 8192: 128 tiles on 74
            // pairs, the second wave 54) can run one wave of 512-wide tiles
            // and one of 384-wide ones (74 + 73 tiles): each pair then does
            // 896 columns instead of 1024.  A 384-wide tile is a 256-wide and
            // a 128-wide MMA sharing the A tile; the narrow MMA reads the
            // whole A tile for half the columns, so a column costs 1.25x a
            // 512-wide one (measured on 2048 x 8192 x 8192: 178 against
            // 190 us per wave, and 368 against 380 us for the whole plan).
            if (Tw > G && pair_bn_override() == 0 && !mix_disabled()) {
                const double cmix = 0.86 * (fle::kMixWide + 1.25 * fle::kMixNarrow);
                if (cmix < 0.985 * std::min(std::min(c256, c224), c512) &&
                    mixed_cut(ta, N, G, pl.mix_a, pl.mix_b, &pl.mix_wide, &pl.mix_narrow))
                    pl.bn = fle::kPairBNWide;
            }
        }
        if (pair_bn_override() != 0) pl.bn = pair_bn_override();
        if (pl.bn > 256 && pl.prec != fle::kPrecTF32) pl.bn = fle::kPairBN;  // wide tiles: TF32 only
    } else {
        pl.bn = (pl.prec == fle::kPrec3xTF32) ? 128 : 256;
    }
    const int64_t Ma = pl.swap ? N : M;
    const int64_t Nb = pl.swap ? M : N;
    pl.tiles_a = static_cast<int>((Ma + tile_m - 1) / tile_m);
    pl.tiles_b = static_cast<int>((Nb + pl.bn - 1) / pl.bn);
    pl.tiles = pl.mix_wide > 0 ? pl.mix_wide + pl.mix_narrow : pl.tiles_a * pl.tiles_b;
    pl.bk = fle::kBK;
    pl.num_kb = static_cast<int>((K + pl.bk - 1) / pl.bk);
    // Two k-blocks per ring stage (TF32): measured faster on the swapped
    // skinny kernel and on pair plans of two or more full waves; plans with
    // fewer tiles keep the deeper one-k-block ring.
    pl.kps = 1;
    if (pl.prec == fle::kPrecTF32) {
        const int64_t tiles = static_cast<int64_t>(pl.tiles_a) * pl.tiles_b;
        if (pl.swap || (pl.pair && tiles >= 2 * static_cast<int64_t>(pairs))) pl.kps = 2;
        if (kps_override() != 0) pl.kps = kps_override();
        if (pl.bn > 256) pl.kps = 1;  // a 512-wide stage of one k-block is already 48 KB
    }
    pl.stages = pl.pair ? pair_stages_for(pl.bn, pl.prec, pl.kps) : stages_for(pl.bn, pl.prec, pl.kps);

    // The schedule runs over CTAs, or over CTA pairs in pair mode.
    const int64_t T = pl.tiles;
    const int64_t G = pl.pair ? pairs : sms;
    const int64_t iters = T * pl.num_kb;
    const char* ov = sched_override();
    const bool force_dp = std::strcmp(ov, "dp") == 0;
    const bool force_sk = std::strcmp(ov, "sk") == 0;
    const bool hybrid = std::strcmp(ov, "hybrid") == 0;
    pl.dp_tiles = static_cast<int>(T);
    pl.grid = static_cast<int>(T < G ? T : G);
    pl.sk_grid = 0;
    if (pl.mix_wide > 0) return pl;  // at most two tiles per pair, all whole
    // Splitting K costs a partial-tile round trip and a wait at the end of the
    // tile (a few microseconds); it is taken only for tiles of at least four
    // minimum-size parts (measured: at K = 1024 the whole tiles are faster).
    if (!force_dp && T % G != 0 && pl.num_kb >= 4 * min_iters) {
        if (force_sk) {
            // spread all k-blocks evenly over all SMs (measured no faster
            // than the k-aligned split below on any of the benchmark shapes,
            // and slower on some)
            const int64_t g_sk = std::min<int64_t>(G, iters / min_iters);
            if (g_sk > T || (T > G && g_sk >= 2)) {
                pl.dp_tiles = 0;
                pl.grid = static_cast<int>(g_sk);
                pl.sk_grid = pl.grid;
            }
        } else {
            // full waves data-parallel; the R tiles of the last partial wave
            // split into S k-aligned parts on R*S CTAs
            const int64_t R = T % G;
            const int64_t S = std::min<int64_t>(G / R, pl.num_kb / min_iters);
            // When the last wave cannot be split evenly (S < 2), 3xTF32 spreads
            // its k-blocks over all CTAs instead: three tensor passes per byte
            // make the lost L2 reuse cheap there (measured faster: 10% on the
            // pair plan of 1024x8192x8192, 14% on the swapped one-CTA plan of
            // 128x32768x32768), while in TF32 it costs more than the idle CTAs.
            // (Only for fewer than two waves, where the idle share is large.)
            const bool spread = hybrid || (pl.prec == fle::kPrec3xTF32 && S < 2 && T < 2 * G);
            if (spread && T > G) {
                pl.dp_tiles = static_cast<int>(T - R);
                pl.grid = static_cast<int>(G);
                pl.sk_grid = static_cast<int>(G);
            } else if (S >= 2) {
                pl.dp_tiles = static_cast<int>(T - R);
                pl.grid = static_cast<int>(T > G ? G : R * S);
                pl.sk_grid = static_cast<int>(R * S);
            }
        }
    }
    pl.sk_tiles = static_cast<int>(T - pl.dp_tiles);
    pl.sk_iters = static_cast<int64_t>(pl.sk_tiles) * pl.num_kb;
    if (pl.sk_tiles > 0) {
        // one partial slot per CTA unless some CTA's stream-K range reaches
        // into a second tile (the k-aligned split of a last wave never does)
        pl.sk_slots = 1;
        for (int64_t c = 0; c < pl.sk_grid; ++c) {
            const int64_t gb = c * pl.sk_iters / pl.sk_grid;
            const int64_t ge = (c + 1) * pl.sk_iters / pl.sk_grid;
            if (ge > gb && gb / pl.num_kb != (ge - 1) / pl.num_kb) {
                pl.sk_slots = 2;
                break;
            }
        }
        // sk_slots fp32 partial tiles of 128 x bn per stream-K CTA, then one
        // arrival counter per stream-K tile (per CTA of the pair)
        const int sk_ctas = pl.pair ? 2 * pl.sk_grid : pl.sk_grid;
        const int counters = pl.pair ? 2 * pl.sk_tiles : pl.sk_tiles;
        pl.partial_bytes = static_cast<size_t>(pl.sk_slots) * sk_ctas * fle::kBM * pl.bn * sizeof(float);
        pl.ws_bytes = pl.partial_bytes + ((static_cast<size_t>(counters) * 4 + 255) & ~size_t(255));
    }
    return pl;
}

// 3xTF32: x's low parts are split once per call into the workspace, except
// for skinny swapped shapes (M <= 64), where x is a small part of each stage
// and the pre-pass does not pay (measured no faster at M = 16), and for x
// above 1 GiB, whose low parts would make the workspace as large.  Measured
// with the low parts in memory: 2048 x 8192 x 8192 1358 -> ~1066 us of GEMM,
// 128 x 32768 x 32768 1766 -> ~1565 us, M = 256 239 -> ~198 us.
Plan make_plan(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d, int sms, int pairs, bool lo_mem) {
    Plan pl = make_plan_core(M, K, N, d, sms, pairs);
    const size_t x_bytes = static_cast<size_t>(M) * static_cast<size_t>(K) * sizeof(float);
    if (lo_mem && pl.prec == fle::kPrec3xTF32 && K > 0 && !(pl.swap && M <= 64) && x_bytes <= (size_t(1) << 30) &&
        !lo_mem_disabled()) {
        pl.lo_mem = true;
        pl.lo_offset = (pl.ws_bytes + 255) & ~size_t(255);
        pl.ws_bytes = pl.lo_offset + x_bytes;
    }
    return pl;
}

// after_prep: the previous kernel in the stream is this call's prep kernel,
// which writes nothing the GEMM reads before griddep_wait(); the GEMM is then
// launched with programmatic stream serialization and starts during it.
template <int BN, int PREC, bool SWAP, int KPS>
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& txlo, const CUtensorMap& to,
                        const KParams& p, int grid, bool after_prep, cudaStream_t st) {
    using C = fle::Cfg<BN, PREC, SWAP, KPS>;
    auto kern = fle::fle_gemm_kernel<BN, PREC, SWAP, KPS>;
    static std::atomic<bool> attr_set[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(fle::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_prep ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, txlo, to, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int PREC, int KPS, int BN = fle::kPairBN, bool SWAP = false>
cudaError_t launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb2,
                             const CUtensorMap& txlo, const CUtensorMap& to, const KParams& p, int pairs,
                             bool after_prep, cudaStream_t st) {
    using C = fle::PairCfg<PREC, KPS, BN, SWAP>;
    auto kern = fle::fle_gemm_pair_kernel<PREC, KPS, BN, SWAP>;
    static std::atomic<bool> attr_set[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cfg.blockDim = dim3(fle::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_prep ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tb2, txlo, to, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// tb2: the 64-row boxes of B for the 384-wide tiles of a mixed plan (else tb).
// txlo: 3xTF32 with x's low parts in memory, their tensor map (else ta).
cudaError_t dispatch(const Plan& pl, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb2,
                     const CUtensorMap& txlo, const CUtensorMap& to, const KParams& p, bool after_prep,
                     cudaStream_t st) {
    using namespace fle;
    const bool tf32 = pl.prec == kPrecTF32;
    const bool two = pl.kps == 2;  // TF32 only
    if (pl.pair && !pl.swap && pl.bn == kPairBNWide)
        return launch_gemm_pair<kPrecTF32, 1, kPairBNWide>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st);
    if (pl.pair && !pl.swap && pl.bn == kPairBNNarrow) {
        if (!tf32) return launch_gemm_pair<kPrec3xTF32, 1, kPairBNNarrow>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st);
        return two ? launch_gemm_pair<kPrecTF32, 2, kPairBNNarrow>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st)
                   : launch_gemm_pair<kPrecTF32, 1, kPairBNNarrow>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st);
    }
    if (pl.pair && !pl.swap) {
        if (!tf32) return launch_gemm_pair<kPrec3xTF32, 1>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st);
        return two ? launch_gemm_pair<kPrecTF32, 2>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st)
                   : launch_gemm_pair<kPrecTF32, 1>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st);
    }
    if (pl.pair) {
        switch (pl.bn) {
#define FLE_PAIR_SWAP_CASE(bn)                                                                             \
    case bn:                                                                                               \
        if (!tf32) return launch_gemm_pair<kPrec3xTF32, 1, bn, true>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st); \
        return two ? launch_gemm_pair<kPrecTF32, 2, bn, true>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st)      \
                   : launch_gemm_pair<kPrecTF32, 1, bn, true>(ta, tb, tb2, txlo, to, p, pl.grid, after_prep, st);
            FLE_PAIR_SWAP_CASE(32)
            FLE_PAIR_SWAP_CASE(64)
            FLE_PAIR_SWAP_CASE(128)
#undef FLE_PAIR_SWAP_CASE
            default: return cudaErrorInvalidConfiguration;
        }
    }
    if (!pl.swap) {
        if (tf32 && pl.bn == 256)
            return two ? launch_gemm<256, kPrecTF32, false, 2>(ta, tb, txlo, to, p, pl.grid, after_prep, st)
                       : launch_gemm<256, kPrecTF32, false, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
        if (!tf32 && pl.bn == 128) return launch_gemm<128, kPrec3xTF32, false, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
    } else {
        switch (pl.bn) {
            case 32:
                if (!tf32) return launch_gemm<32, kPrec3xTF32, true, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
                return two ? launch_gemm<32, kPrecTF32, true, 2>(ta, tb, txlo, to, p, pl.grid, after_prep, st)
                           : launch_gemm<32, kPrecTF32, true, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
            case 64:
                if (!tf32) return launch_gemm<64, kPrec3xTF32, true, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
                return two ? launch_gemm<64, kPrecTF32, true, 2>(ta, tb, txlo, to, p, pl.grid, after_prep, st)
                           : launch_gemm<64, kPrecTF32, true, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
            case 128:
                if (!tf32) return launch_gemm<128, kPrec3xTF32, true, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
                return two ? launch_gemm<128, kPrecTF32, true, 2>(ta, tb, txlo, to, p, pl.grid, after_prep, st)
                           : launch_gemm<128, kPrecTF32, true, 1>(ta, tb, txlo, to, p, pl.grid, after_prep, st);
            default: break;
        }
    }
    return cudaErrorInvalidConfiguration;
}

uint64_t timeout_ns() {
    static uint64_t t = [] {
        const char* e = std::getenv("FLE_TIMEOUT_MS");
        long ms = e ? std::atol(e) : 0;
        return static_cast<uint64_t>(ms > 0 ? ms : 1000) * 1000000ull;
    }();
    return t;
}

// Finisher mode of split tiles (fle_test_set_finisher); FLE_FINISH_AUTO in use.
std::atomic<int> g_finish_mode{FLE_FINISH_AUTO};

bool log_enabled() {
    static bool on = [] {
        const char* e = std::getenv("FLE_LOG");
        return e && e[0] == '1';
    }();
    return on;
}

bool sync_check_enabled() {
    static bool on = [] {
        const char* e = std::getenv("FLE_SYNC_CHECK");
        return e && e[0] == '1';
    }();
    return on;
}

int plan_to_string(const Plan& pl, char* buf, size_t n) {
    if (!buf || n == 0) return FLE_ERR_NULL;
    std::snprintf(buf, n,
                  "tile=%dx%d pair=%d swap=%d prec=%s stages=%d kps=%d tiles=%dx%d kblocks=%d dp_tiles=%d sk_tiles=%d "
                  "sk_kblocks=%lld sk_grid=%d slots=%d grid=%d workspace=%zu",
                  pl.pair ? fle::kPairBM : fle::kBM, pl.bn, pl.pair ? 1 : 0, pl.swap ? 1 : 0,
                  pl.prec == fle::kPrecTF32 ? "tf32" : "3xtf32", pl.stages, pl.kps,
                  pl.tiles_a, pl.tiles_b, pl.num_kb, pl.dp_tiles, pl.sk_tiles, (long long)pl.sk_iters, pl.sk_grid,
                  pl.sk_slots, pl.grid, pl.ws_bytes);
    if (pl.lo_mem) {
        const size_t used = std::strlen(buf);
        if (used + 1 < n) std::snprintf(buf + used, n - used, " xlo=mem");
    }
    if (pl.mix_wide > 0) {
        const size_t used = std::strlen(buf);
        if (used + 1 < n)
            std::snprintf(buf + used, n - used, " mix=%dx%d+%dx%d", pl.mix_wide, fle::kMixWide, pl.mix_narrow,
                          fle::kMixNarrow);
    }
    return FLE_OK;
}

}  // namespace

extern "C" {

int fle_version(void) { return 200; }

#ifndef FLE_SOURCE_HASH
#define FLE_SOURCE_HASH "unknown"
#endif
// The marker prefix lets the build script find the hash in the built file.
static const char kSourceHashTag[] = "fle-source-sha256:" FLE_SOURCE_HASH;
const char* fle_source_hash(void) { return kSourceHashTag + 18; }

const char* fle_status_string(int s) {
    switch (s) {
        case FLE_OK: return "ok";
        case FLE_ERR_NULL: return "a required pointer is NULL";
        case FLE_ERR_SHAPE: return "invalid shape (negative, >= 2^31, or N < pool_k for the pool epilogue)";
        case FLE_ERR_ALIGN: return "misaligned argument (x/W need 16-byte alignment and K % 4 == 0; out/b 4-byte)";
        case FLE_ERR_DESC: return "invalid epilogue descriptor";
        case FLE_ERR_WORKSPACE: return "workspace smaller than fle_workspace_size()";
        case FLE_ERR_ARCH: return "device is not sm_100 (B200)";
        case FLE_ERR_CUDA: return "a CUDA call failed";
        case FLE_ERR_TIMEOUT: return "a device-side bounded wait expired";
        case FLE_ERR_UNSUPPORTED: return "arguments valid but not supported by the library";
        case FLE_ERR_PROTOCOL: return "a barrier-protocol check failed (checking build)";
        default: return "unknown status";
    }
}

size_t fle_workspace_size(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d) {
    if (check_desc(d) != FLE_OK || check_shape(M, K, N, d) != FLE_OK) return 0;
    if (M == 0 || N == 0 || K == 0) return 0;
    DeviceInfo di;
    if (device_info(&di) != FLE_OK) return 0;
    return make_plan(M, K, N, d, di.sms, d->precision == FLE_PREC_3XTF32 ? di.pairs3x : di.pairs).ws_bytes;
}

size_t fle_workspace_size_min(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d) {
    if (check_desc(d) != FLE_OK || check_shape(M, K, N, d) != FLE_OK) return 0;
    if (M == 0 || N == 0 || K == 0) return 0;
    DeviceInfo di;
    if (device_info(&di) != FLE_OK) return 0;
    return make_plan(M, K, N, d, di.sms, d->precision == FLE_PREC_3XTF32 ? di.pairs3x : di.pairs, false).ws_bytes;
}

int fle_plan_string(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d, char* buf, size_t n) {
    int st = check_desc(d);
    if (st != FLE_OK) return st;
    st = check_shape(M, K, N, d);
    if (st != FLE_OK) return st;
    DeviceInfo di;
    st = device_info(&di);
    if (st != FLE_OK) return st;
    return plan_to_string(make_plan(M, K, N, d, di.sms, d->precision == FLE_PREC_3XTF32 ? di.pairs3x : di.pairs), buf, n);
}

int fle_forward(const float* x, const float* W, const float* b, int64_t M, int64_t K, int64_t N,
                const fle_epilogue_desc* d, float* out, void* workspace, size_t workspace_bytes,
                void* stream) {
    // ---- host-side argument checks: nothing is enqueued on failure
    int st = check_desc(d);
    if (st != FLE_OK) return st;
    st = check_shape(M, K, N, d);
    if (st != FLE_OK) return st;
    const bool pool = d->kind == FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX;
    if (M == 0 || (N == 0 && !pool)) return FLE_OK;
    if (!out) return FLE_ERR_NULL;
    if (K > 0 && (!x || !W)) return FLE_ERR_NULL;
    if (K > 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(W)) & 15u)) return FLE_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(out) & 3u) return FLE_ERR_ALIGN;
    if (b && (reinterpret_cast<uintptr_t>(b) & 3u)) return FLE_ERR_ALIGN;

    DeviceInfo di;
    st = device_info(&di);
    if (st != FLE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    KParams p{};
    p.bias = b;
    p.out = out;
    p.M = M;
    p.N = N;
    p.kind = d->kind;
    p.scale = d->scale;
    p.clamp_lo = d->clamp_lo;
    p.clamp_hi = d->clamp_hi;
    p.gelu_tanh = (d->flags & FLE_FLAG_GELU_TANH) ? 1 : 0;
    p.fold_scale = (d->flags & FLE_FLAG_FOLD_SCALE) ? 1 : 0;
    // (a) with its GELU input clamped into [-2, 2]: the polynomial GELU
    p.gelu_poly = (d->kind == FLE_EPI_SCALE_HARDTANH_GELU && !p.gelu_tanh && d->clamp_lo >= -2.0f &&
                   d->clamp_hi <= 2.0f && !poly_disabled())
                      ? 1 : 0;
    p.pool_k = pool ? d->pool_k : 1;
    p.pool_limit = pool ? (N / d->pool_k) * d->pool_k : N;
    p.vec_out = ((reinterpret_cast<uintptr_t>(out) & 15u) == 0 && N % 4 == 0) ? 1 : 0;
    p.vec_bias = (b && (reinterpret_cast<uintptr_t>(b) & 15u) == 0) ? 1 : 0;
    p.timeout_ns = timeout_ns();
    switch (g_finish_mode.load(std::memory_order_relaxed)) {
        case FLE_FINISH_OWN: p.sk_finish = fle::kFinishOwn; break;
        case FLE_FINISH_LAST: p.sk_finish = fle::kFinishPark; break;
        default: p.sk_finish = fle::kFinishAuto; break;
    }

    if (K == 0) {
        const int64_t n = pool ? M : M * N;
        const int threads = 256;
        const int64_t blocks = (n + threads - 1) / threads;
        fle::fle_bias_only_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
        return cudaGetLastError() == cudaSuccess ? FLE_OK : FLE_ERR_CUDA;
    }

    const int pairs = d->precision == FLE_PREC_3XTF32 ? di.pairs3x : di.pairs;
    Plan pl = make_plan(M, K, N, d, di.sms, pairs);
    // a workspace too small for x's low parts (3xTF32) runs the plan that
    // computes them inside the GEMM
    if (pl.lo_mem && (!workspace || workspace_bytes < pl.ws_bytes)) pl = make_plan(M, K, N, d, di.sms, pairs, false);
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return FLE_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FLE_ERR_ALIGN;
    }
    p.Ma = static_cast<int>(pl.swap ? N : M);
    p.Nb = static_cast<int>(pl.swap ? M : N);
    p.tiles_a = pl.tiles_a;
    p.tiles_b = pl.tiles_b;
    p.num_kb = pl.num_kb;
    p.num_tiles = pl.tiles;
    p.dp_tiles = pl.dp_tiles;
    p.sk_iters = pl.sk_iters;
    p.sk_grid = pl.sk_grid;
    p.sk_slots = pl.sk_slots;
    p.tile_n = pl.bn;
    p.lo_mem = pl.lo_mem ? 1 : 0;
    p.mix_wide = pl.mix_wide;
    std::memcpy(p.mix_a, pl.mix_a, sizeof p.mix_a);
    std::memcpy(p.mix_b, pl.mix_b, sizeof p.mix_b);
    if (pl.sk_tiles > 0) {
        p.ws = static_cast<float*>(workspace);
        p.counters = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + pl.partial_bytes);
    }

    CUtensorMap ta, tb, tb2, txlo, to;
    std::memset(&to, 0, sizeof to);
    // Elementwise kinds (direct or swapped layout) store through TMA when the
    // output rows are 16-byte multiples and the base is 16-byte aligned.
    p.tma_out = (!pool && N % 4 == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) ? 1 : 0;
    if (p.tma_out) {
        st = encode_output(&to, out, M, N);
        if (st != FLE_OK) return st;
    }
    const float* A = pl.swap ? W : x;
    const float* B = pl.swap ? x : W;
    st = encode_operand(&ta, A, p.Ma, K, fle::kBM);
    if (st != FLE_OK) return st;
    // B boxes: half of the pair tile's rows per CTA, 128 for the 512-wide
    // tile (each CTA loads its 128 rows of both 256-wide sub-tiles)
    st = encode_operand(&tb, B, p.Nb, K, pl.pair ? (pl.bn > 256 ? 128 : pl.bn / 2) : pl.bn);
    if (st != FLE_OK) return st;
    // x's low parts (3xTF32), in the workspace: the same boxes as x's own tiles
    float* x_lo = pl.lo_mem ? reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.lo_offset) : nullptr;
    txlo = ta;
    if (pl.lo_mem) {
        const int box = pl.swap ? (pl.pair ? (pl.bn > 256 ? 128 : pl.bn / 2) : pl.bn) : fle::kBM;
        st = encode_operand(&txlo, x_lo, M, K, box);
        if (st != FLE_OK) return st;
    }
    // a mixed plan's 384-wide tiles: 64 rows per CTA of their 128-wide sub-tile
    tb2 = tb;
    if (pl.mix_wide > 0) {
        st = encode_operand(&tb2, B, p.Nb, K, (fle::kMixNarrow - 256) / 2);
        if (st != FLE_OK) return st;
    }

    if (log_enabled()) {
        char line[256];
        plan_to_string(pl, line, sizeof line);
        std::fprintf(stderr, "[fle] M=%lld K=%lld N=%lld kind=%d %s\n", (long long)M, (long long)K,
                     (long long)N, d->kind, line);
    }

    if (pl.lo_mem) {
        const int64_t n4 = M * K / 4;
        const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, 16 * static_cast<int64_t>(di.sms));
        fle::fle_split_lo_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            reinterpret_cast<const float4*>(x), reinterpret_cast<float4*>(x_lo), n4);
        if (cudaGetLastError() != cudaSuccess) return FLE_ERR_CUDA;
    }
    const bool prep = pool || pl.sk_tiles > 0;
    if (prep) {
        const int threads = 256;
        const int n_counters = pl.pair ? 2 * pl.sk_tiles : pl.sk_tiles;
        const int64_t n = std::max<int64_t>(pool ? M : 0, n_counters);
        fle::fle_prep_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, s>>>(
            pool ? out : nullptr, pool ? M : 0, p.counters, n_counters);
        if (cudaGetLastError() != cudaSuccess) return FLE_ERR_CUDA;
    }
    if (dispatch(pl, ta, tb, tb2, txlo, to, p, prep, s) != cudaSuccess) return FLE_ERR_CUDA;
    if (sync_check_enabled()) return fle_device_status(stream);
    return FLE_OK;
}

int fle_plan_units(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d, int num_sms, int cta,
                   int32_t* units, int max_units, int* n_units, int* grid) {
    int st = check_desc(d);
    if (st != FLE_OK) return st;
    st = check_shape(M, K, N, d);
    if (st != FLE_OK) return st;
    if (num_sms <= 0 || cta < 0 || !n_units || (max_units > 0 && !units)) return FLE_ERR_NULL;
    *n_units = 0;
    if (grid) *grid = 0;
    if (M == 0 || N == 0 || K == 0) return FLE_OK;
    const Plan pl = make_plan(M, K, N, d, num_sms, num_sms / 2);
    if (grid) *grid = pl.grid;
    if (cta >= pl.grid) return FLE_OK;
    KParams p{};
    p.tiles_a = pl.tiles_a;
    p.tiles_b = pl.tiles_b;
    p.num_kb = pl.num_kb;
    p.num_tiles = pl.tiles;
    p.dp_tiles = pl.dp_tiles;
    p.sk_iters = pl.sk_iters;
    p.sk_grid = pl.sk_grid;
    p.sk_slots = pl.sk_slots;
    p.tile_n = pl.bn;
    p.mix_wide = pl.mix_wide;
    std::memcpy(p.mix_a, pl.mix_a, sizeof p.mix_a);
    std::memcpy(p.mix_b, pl.mix_b, sizeof p.mix_b);
    fle::Sched sc;
    sc.init(p, cta, pl.grid);
    fle::Unit u;
    int n = 0;
    while (sc.next(p, u)) {
        if (n < max_units) {
            int32_t* row = units + static_cast<size_t>(n) * 12;
            row[0] = u.t; row[1] = u.ta; row[2] = u.tb; row[3] = u.kb0; row[4] = u.kb1;
            row[10] = static_cast<int32_t>(u.col0);
            row[11] = u.w;
            row[5] = u.partial; row[6] = u.partial ? u.slot : -1;
            if (u.partial) {
                row[7] = fle::sk_cta_of(static_cast<int64_t>(u.sk_tile) * p.num_kb, p.sk_iters, pl.sk_grid);
                row[8] = fle::sk_cta_of((static_cast<int64_t>(u.sk_tile) + 1) * p.num_kb - 1, p.sk_iters, pl.sk_grid);
                row[9] = fle::sk_slot_of(cta, u.sk_tile, p.sk_iters, pl.sk_grid, p.num_kb);
            } else {
                row[7] = row[8] = row[9] = -1;
            }
        }
        ++n;
    }
    *n_units = n;
    return FLE_OK;
}

int fle_pool_weights(const float* W, const float* b, int64_t N, int64_t K, int32_t pool_k, float* W_pooled,
                     float* b_pooled, void* stream) {
    if (!is_pow2_upto32(pool_k)) return FLE_ERR_DESC;
    const int64_t lim = (int64_t(1) << 31);
    if (N < pool_k || K < 0 || N >= lim || K >= lim) return FLE_ERR_SHAPE;
    if (K % 4 != 0) return FLE_ERR_ALIGN;
    const int64_t P = N / pool_k;
    if (K > 0 && (!W || !W_pooled)) return FLE_ERR_NULL;
    if (b && !b_pooled) return FLE_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(W_pooled)) & 15u) return FLE_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(b_pooled)) & 3u) return FLE_ERR_ALIGN;
    DeviceInfo di;
    int st = device_info(&di);
    if (st != FLE_OK) return st;
    const int64_t n = std::max<int64_t>(P * (K / 4), P);
    const int threads = 256;
    fle::fle_pool_weights_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0,
                                   static_cast<cudaStream_t>(stream)>>>(W, b, P, K, pool_k, W_pooled, b_pooled);
    return cudaGetLastError() == cudaSuccess ? FLE_OK : FLE_ERR_CUDA;
}

namespace {
// The pool-folded call: desc with the pool replaced by pool_k = 1 on the
// pooled weights.
fle_epilogue_desc folded_desc(const fle_epilogue_desc* d) {
    fle_epilogue_desc f = *d;
    f.pool_k = 1;
    f.pool_stride = 1;
    return f;
}
size_t pooled_weight_bytes(int64_t P, int64_t K) {
    return ((static_cast<size_t>(P) * K * sizeof(float) + 255) & ~size_t(255)) +
           ((static_cast<size_t>(P) * sizeof(float) + 255) & ~size_t(255));
}
}  // namespace

size_t fle_workspace_size_pooled(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* d) {
    if (check_desc(d) != FLE_OK || check_shape(M, K, N, d) != FLE_OK) return 0;
    if (d->kind != FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX || M == 0) return 0;
    const int64_t P = N / d->pool_k;
    const fle_epilogue_desc f = folded_desc(d);
    return pooled_weight_bytes(P, K) + fle_workspace_size(M, K, P, &f);
}

int fle_forward_pooled(const float* x, const float* W, const float* b, int64_t M, int64_t K, int64_t N,
                       const fle_epilogue_desc* d, float* out, void* workspace, size_t workspace_bytes,
                       void* stream) {
    int st = check_desc(d);
    if (st != FLE_OK) return st;
    if (d->kind != FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX) return FLE_ERR_DESC;
    st = check_shape(M, K, N, d);
    if (st != FLE_OK) return st;
    if (M == 0) return FLE_OK;
    const int64_t P = N / d->pool_k;
    const size_t need = fle_workspace_size_pooled(M, K, N, d);
    if (!workspace || workspace_bytes < need) return FLE_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FLE_ERR_ALIGN;
    char* ws = static_cast<char*>(workspace);
    float* Wp = reinterpret_cast<float*>(ws);
    float* bp = reinterpret_cast<float*>(ws + ((static_cast<size_t>(P) * K * sizeof(float) + 255) & ~size_t(255)));
    const size_t pw = pooled_weight_bytes(P, K);
    if (K == 0) return fle_forward(x, W, b, M, K, N, d, out, nullptr, 0, stream);  // out = epilogue(b)
    st = fle_pool_weights(W, b, N, K, d->pool_k, Wp, b ? bp : nullptr, stream);
    if (st != FLE_OK) return st;
    const fle_epilogue_desc f = folded_desc(d);
    return fle_forward(x, Wp, b ? bp : nullptr, M, K, P, &f, out, ws + pw, workspace_bytes - pw, stream);
}

int fle_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FLE_ERR_CUDA;
    unsigned h[4] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(h, fle::g_status, sizeof h) != cudaSuccess) return FLE_ERR_CUDA;
    if (h[0] != 0) {
        const unsigned z[4] = {0, 0, 0, 0};
        if (cudaMemcpyToSymbol(fle::g_status, z, sizeof z) != cudaSuccess) return FLE_ERR_CUDA;
        if (log_enabled())
            std::fprintf(stderr, "[fle] device status %u at site %u block %u (count %u)\n", h[0], h[1], h[2], h[3]);
        return static_cast<int>(h[0]);
    }
    return FLE_OK;
}

int fle_test_epilogue_math(const float* in, float* out, int64_t n, int32_t which, int32_t reference,
                           void* stream) {
    if (!in || !out) return FLE_ERR_NULL;
    if (n < 0 || which < 0 || which > 4) return FLE_ERR_SHAPE;
    DeviceInfo di;
    int st = device_info(&di);
    if (st != FLE_OK) return st;
    if (n == 0) return FLE_OK;
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((n + threads - 1) / threads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (reference)
        fle::fle_math_reference_kernel<<<blocks, threads, 0, s>>>(in, out, n, which);
    else
        fle::fle_math_probe_kernel<<<blocks, threads, 0, s>>>(in, out, n, which);
    return cudaGetLastError() == cudaSuccess ? FLE_OK : FLE_ERR_CUDA;
}

int fle_test_set_finisher(int32_t mode) {
    if (mode != FLE_FINISH_AUTO && mode != FLE_FINISH_OWN && mode != FLE_FINISH_LAST) return -1;
    return g_finish_mode.exchange(mode);
}

int fle_test_finisher_counts(uint32_t* counts, int32_t reset, void* stream) {
    if (!counts) return FLE_ERR_NULL;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FLE_ERR_CUDA;
    unsigned h[2] = {0, 0};
    if (cudaMemcpyFromSymbol(h, fle::g_finish_count, sizeof h) != cudaSuccess) return FLE_ERR_CUDA;
    counts[0] = h[0];
    counts[1] = h[1];
    if (reset) {
        const unsigned z[2] = {0, 0};
        if (cudaMemcpyToSymbol(fle::g_finish_count, z, sizeof z) != cudaSuccess) return FLE_ERR_CUDA;
    }
    return FLE_OK;
}

int fle_test_bounded_wait(uint32_t timeout_us, void* stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != FLE_OK) return st;
    fle::fle_bounded_wait_test_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(timeout_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? FLE_OK : FLE_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free entry point.  Its scratch (the stream-K partial tiles and
// arrival counters that fle_forward takes from the caller's workspace) lives
// in this file-scope device array instead, so the call needs no allocation
// by anyone.  The array is part of the library's device image: every GPU
// that loads the library holds these bytes until the process exits.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FLE_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device.  In host code the array's
// name only stands in for the symbol; the address a kernel can use comes
// from cudaGetSymbolAddress, taken with that device current.
void* g_noalloc_ptr[kMaxDevices] = {};

}  // namespace

extern "C" int fle_forward_noalloc(const float* x, const float* W, const float* b, int64_t M, int64_t K,
                                   int64_t N, const fle_epilogue_desc* d, float* out, void* stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FLE_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_noalloc_ptr[dev] == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FLE_ERR_CUDA;
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // The scratch need of the plan that fits the least workspace (3xTF32:
    // x's low parts computed inside the GEMM); 0 also for invalid
    // arguments, which fle_forward then reports.
    const size_t need = fle_workspace_size_min(M, K, N, d);
    if (need > FLE_NOALLOC_SCRATCH_BYTES) return FLE_ERR_WORKSPACE;
    return fle_forward(x, W, b, M, K, N, d, out, scratch, FLE_NOALLOC_SCRATCH_BYTES, stream);
}
