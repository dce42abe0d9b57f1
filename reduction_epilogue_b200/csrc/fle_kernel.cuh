// fle_kernel.cuh -- the fused Linear + epilogue kernel for sm_100a.
//
// One persistent CTA per SM walks a list of work units.  A unit is one output
// tile (128 rows of operand A x BN rows of operand B) over a range of
// k-blocks.  The schedule is hybrid: the first tiles are data-parallel (one
// CTA per tile, the whole K), and the remaining tiles' k-blocks are divided
// evenly over the first sk_grid CTAs (stream-K).  The host (make_plan) splits
// only the last partial wave, into k-aligned parts, so CTAs that share a
// weight slab still walk K together and hit it in L2.  A tile whose k-range
// is split is finished without waits: the CTA holding its k-block 0 (which
// normally ends last) adds the parked fp32 partials of the others to its own
// accumulator; if it is not last, it parks its partial too and the last
// arrival sums them all.  Partials are summed in a fixed order, so results
// are bitwise reproducible.  Operand A is x and B is W
// ("direct"), or, for small M, A is W and B is x ("swapped"), so the large
// dimension sits on the 128-row side of the MMA; either way both operands are
// K-major, as nn.Linear stores them.
//
// Warp roles (384 threads):
//   warp 0, lane 0   TMA producer: fills a ring of shared-memory stages.
//   warp 1           allocates TMEM; lane 0 issues the tcgen05.mma chain.
//   warps 2-3        3xTF32 only: split each landed stage into TF32 hi/lo parts.
//   warps 4-11       epilogue: TMEM -> registers -> bias + epilogue -> global;
//                    two warps per TMEM lane quadrant, each with half the columns.
// The accumulator is double-buffered in TMEM, so the epilogue of one tile
// overlaps the main loop of the next.
#pragma once

#include <cuda.h>
#include <math.h>
#include <stdint.h>

#include "fle_ptx.cuh"

namespace fle {

constexpr int kBM = 128;           // MMA M: rows of operand A per tile
constexpr int kBK = 32;            // fp32 per k-block = one 128-byte swizzled row
// Mixed-width plans (see KParams): tile widths and the most 256-row panels
constexpr int kMixWide = 512;
constexpr int kMixNarrow = 384;
constexpr int kMaxMixPanels = 16;
constexpr int kUmmaK = 8;          // K of one tcgen05.mma kind::tf32
constexpr int kThreads = 384;
constexpr int kEpiWarps = 8;                 // warps 4..11
constexpr int kEpiTileBytes = 32 * 32 * 4;   // one warp's 32 x 32 fp32 block
constexpr int kSmemStageBudget = 229376;  // bytes of shared memory for stages (224 KB)

enum : int { kEpiHardtanhGelu = 0, kEpiSwish = 1, kEpiPoolMax = 2, kEpiNone = 3 };
enum : int { kPrec3xTF32 = 0, kPrecTF32 = 1 };
// Who finishes a tile whose k-range is split over CTAs (KParams::sk_finish).
// kFinishAuto is the product behaviour; the other two pin one branch for tests.
enum : int { kFinishAuto = 0, kFinishOwn = 1, kFinishPark = 2 };

// Wait-site identifiers recorded with a timeout.
enum : unsigned {
    kWhereProdEmpty = 1, kWhereMmaFull = 2, kWhereMmaAccEmpty = 3, kWhereEpiAccFull = 4,
    kWhereConvFull = 5, kWhereDrain = 6, kWhereProdDrain = 7, kWhereTest = 9
};

struct KParams {
    const float* bias;      // [N] or nullptr
    float* out;             // [M,N] or [M]
    float* ws;              // stream-K partial tiles: [sk_slots * CTAs][kBM * BN]
    unsigned* counters;     // stream-K arrival counters, one per stream-K tile
    int64_t M, N;           // output sizes
    int Ma, Nb;             // rows of operand A and operand B
    int tiles_a, tiles_b;   // tiles along A rows and along B rows
    int num_kb;             // k-blocks along K
    int num_tiles;          // tiles_a * tiles_b
    int dp_tiles;           // tiles [0, dp_tiles) are data-parallel
    int64_t sk_iters;       // (num_tiles - dp_tiles) * num_kb
    int sk_grid;            // CTAs [0, sk_grid) share the stream-K k-blocks
    int sk_slots;           // partial-tile slots per stream-K CTA (1 or 2)
    int kind;
    float scale, clamp_lo, clamp_hi;
    int gelu_tanh;          // GELU in its tanh form, (a) and (c)
    int gelu_poly;          // (a), erf form, clamp within [-2, 2]: polynomial GELU
    int fold_scale;         // (a): scale * acc + scale * b in one FMA
    int pool_k;
    int64_t pool_limit;     // columns covered by complete pool windows
    int sk_finish;          // kFinishAuto / kFinishOwn / kFinishPark
    int vec_out;            // out 16-byte aligned and N % 4 == 0
    int vec_bias;           // bias 16-byte aligned
    int tma_out;            // direct layout: write out through TMA tile stores
    uint64_t timeout_ns;
    int tile_n;             // B rows per tile (the kernel's tile width)
    int lo_mem;             // 3xTF32: the low parts of x are in memory (tensor map
                            // tmXlo), copied with the tiles; the split warps split W only
    // Mixed-width plans of the 512-wide pair kernel (data-parallel only):
    // each 256-row panel r holds mix_a[r] tiles 512 wide from column 0, then
    // mix_b[r] tiles 384 wide.  Units [0, mix_wide) are the 512-wide tiles,
    // panel by panel, the rest the 384-wide ones.  0: a uniform grid of tiles.
    int mix_wide;
    unsigned char mix_a[kMaxMixPanels];
    unsigned char mix_b[kMaxMixPanels];
};

// One unit of work: tile t over k-blocks [kb0, kb1).
struct Unit {
    int t, ta, tb;          // tile; its index along A rows and along B rows (-1: mixed plan)
    int64_t col0;           // first B row of the tile
    int w;                  // B rows of the tile
    int kb0, kb1;
    int partial;            // the tile's k-range is shared with other CTAs
    int sk_tile;            // index among the stream-K tiles
    int slot;               // 0: first tile of this CTA's stream-K range, 1: last
};

// The unit sequence of one CTA.  Every role of the CTA walks it in lockstep.
struct Sched {
    int c, G;
    int dp_next;
    int64_t g, g_begin, g_end;

    __host__ __device__ __forceinline__ void init(const KParams& p, int cta, int grid) {
        c = cta;
        G = grid;
        dp_next = c;
        if (c < p.sk_grid) {
            g_begin = (static_cast<int64_t>(c) * p.sk_iters) / p.sk_grid;
            g_end = (static_cast<int64_t>(c + 1) * p.sk_iters) / p.sk_grid;
        } else {
            g_begin = g_end = 0;
        }
        g = g_begin;
    }
    __host__ __device__ __forceinline__ bool next(const KParams& p, Unit& u) {
        if (dp_next < p.dp_tiles) {
            u.t = dp_next;
            u.kb0 = 0;
            u.kb1 = p.num_kb;
            u.partial = 0;
            u.sk_tile = -1;
            u.slot = 0;
            dp_next += G;
        } else if (g < g_end) {
            const int64_t tsk = g / p.num_kb;
            const int kb0 = static_cast<int>(g - tsk * p.num_kb);
            const int64_t left = g_end - g;
            const int kb1 = static_cast<int>(left < p.num_kb - kb0 ? kb0 + left : p.num_kb);
            u.t = p.dp_tiles + static_cast<int>(tsk);
            u.kb0 = kb0;
            u.kb1 = kb1;
            u.partial = (kb0 != 0 || kb1 != p.num_kb) ? 1 : 0;
            u.sk_tile = static_cast<int>(tsk);
            u.slot = (tsk == g_begin / p.num_kb) ? 0 : 1;
            g += kb1 - kb0;
        } else {
            return false;
        }
        if (p.mix_wide > 0) {
            // mixed widths: walk the panels to the unit's tile
            const bool wide = u.t < p.mix_wide;
            int i = wide ? u.t : u.t - p.mix_wide;
            int r = 0;
            for (; r + 1 < p.tiles_a; ++r) {
                const int n = wide ? p.mix_a[r] : p.mix_b[r];
                if (i < n) break;
                i -= n;
            }
            u.ta = r;
            u.tb = -1;
            u.w = wide ? kMixWide : kMixNarrow;
            u.col0 = wide ? static_cast<int64_t>(kMixWide) * i
                          : static_cast<int64_t>(kMixWide) * p.mix_a[r] + static_cast<int64_t>(kMixNarrow) * i;
        } else {
            u.ta = u.t % p.tiles_a;
            u.tb = u.t / p.tiles_a;
            u.w = p.tile_n;
            u.col0 = static_cast<int64_t>(u.tb) * p.tile_n;
        }
        return true;
    }
};

// The CTA whose stream-K range holds global stream-K k-block g (G = sk_grid).
__host__ __device__ __forceinline__ int sk_cta_of(int64_t g, int64_t sk_iters, int G) {
    return static_cast<int>(((g + 1) * G - 1) / sk_iters);
}

// Which of CTA c's two partial slots holds stream-K tile tsk.
__host__ __device__ __forceinline__ int sk_slot_of(int c, int64_t tsk, int64_t sk_iters, int G, int num_kb) {
    const int64_t gb = (static_cast<int64_t>(c) * sk_iters) / G;
    return (tsk == gb / num_kb) ? 0 : 1;
}

// KPS: k-blocks per ring stage.  A stage is [A of k-block 0..KPS-1 | B of
// k-block 0..KPS-1] (then the same again for the 3xTF32 low parts).  Two
// k-blocks per stage halve the producer/MMA handoffs per byte: each stage
// costs a fixed barrier round trip, which otherwise caps the bytes a CTA
// moves per microsecond.
template <int BN, int PREC, bool SWAP, int KPS = 1>
struct Cfg {
    static constexpr int kABytes = kBM * kBK * 4;                    // A rows of one k-block
    static constexpr int kBBytes = BN * kBK * 4;                     // B rows of one k-block
    static constexpr int kKbBytes = kABytes + kBBytes;
    static constexpr int kLoadBytes = KPS * kKbBytes;                // TMA bytes per full stage
    static constexpr int kStageBytes = kLoadBytes * (PREC == kPrec3xTF32 ? 2 : 1);
    // direct layout: one 32 x 32 fp32 staging tile per epilogue warp for TMA stores
    static constexpr int kEpiStageBytes = kEpiWarps * kEpiTileBytes;
    static constexpr int kStagesRaw = (kSmemStageBudget - kEpiStageBytes) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                    : (2 * BN <= 256) ? 256 : 512;
    // barriers: full, conv, empty per stage; accf, acce per buffer; drain
    static constexpr int kNumBars = 3 * kStages + 4 + 1;
    static constexpr int kSmemBytes =
        1024 /*align slack*/ + kStages * kStageBytes + kEpiStageBytes + kNumBars * 8 + 32 + (kCheckBarriers ? 64 : 0);
    static_assert(kStages >= 2, "need at least two stages");
    static_assert(KPS == 1 || KPS == 2, "one or two k-blocks per stage");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128 is a multiple of 16 in [16,256]");
    static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kSmemBytes <= 232448, "exceeds 227 KB of shared memory per block");
    static_assert(PREC != kPrec3xTF32 || KPS == 1, "3xTF32 stages hold one k-block");
};

// ----------------------------------------------------------------------------
// Epilogue math
// ----------------------------------------------------------------------------
// erf(x) by Abramowitz & Stegun, Handbook of Mathematical Functions, formula
// 7.1.26 (Hastings' rational approximation): for x >= 0,
//   erf(x) = 1 - (a1 s + a2 s^2 + a3 s^3 + a4 s^4 + a5 s^5) exp(-x^2),
//   s = 1 / (1 + p x),  |error| <= 1.5e-7,
// extended to x < 0 by oddness.  One reciprocal and one exponential instead
// of a long polynomial chain: the epilogue runs it once per output element.
__device__ __forceinline__ float erf_as7126(float x) {
    const float ax = fabsf(x);
    const float s = __fdividef(1.0f, fmaf(0.3275911f, ax, 1.0f));
    float poly = fmaf(s, 1.061405429f, -1.453152027f);
    poly = fmaf(s, poly, 1.421413741f);
    poly = fmaf(s, poly, -0.284496736f);
    poly = fmaf(s, poly, 0.254829592f);
    poly *= s;
    const float r = fmaf(-poly, __expf(-ax * ax), 1.0f);
    return copysignf(r, x);
}

// Exact-form GELU: t * Phi(t) = t * (1 + erf(t / sqrt 2)) / 2.
__device__ __forceinline__ float gelu_erf(float t) {
    return t * 0.5f * (1.0f + erf_as7126(t * 0.70710678118654752440f));
}

// GELU in its tanh form, t/2 * (1 + tanh(u)), u = sqrt(2/pi) (t + 0.044715 t^3),
// with tanh(u) = 1 - 2 / (1 + e^(2u)): one exponential and one division; it
// saturates to +-1 where e^(2u) over- or underflows.
__device__ __forceinline__ float gelu_tanh_form(float t) {
    const float u = 0.79788456080286535588f * fmaf(0.044715f * t, t * t, t);
    const float th = 1.0f - __fdividef(2.0f, 1.0f + __expf(2.0f * u));
    return 0.5f * t * (1.0f + th);
}

// Exact-form GELU on |t| <= 2 (epilogue (a) with the pages' Hardtanh bounds):
// t/2 + t^2 Q(t^2), Q a degree-7 least-squares fit of (t/2) erf(t/sqrt 2) / t^2
// (gen_gelu_poly.py beside this file writes the table); eight FMAs and no
// exponential or division.  |error| <= 1e-8 before fp32 rounding.
__device__ __forceinline__ float gelu_poly2(float t) {
    // Q(z), z = t^2, lowest degree first (gen_gelu_poly.py: T = 2, D = 7; fp64 max |error| 2.0e-09)
    constexpr float kGeluPolyQ[8] = {3.989422365e-01f, -6.649000114e-02f, 9.972453726e-03f, -1.185778469e-03f,
                                     1.142239958e-04f, -8.885020448e-06f, 5.106075654e-07f, -1.594644622e-08f};
    const float z = t * t;
    float q = kGeluPolyQ[7];
#pragma unroll
    for (int k = 6; k >= 0; --k) q = fmaf(q, z, kGeluPolyQ[k]);
    return fmaf(z, q, 0.5f * t);
}

__device__ __forceinline__ float gelu_sel(float t, const KParams& p) {
    return p.gelu_tanh ? gelu_tanh_form(t) : gelu_erf(t);
}

// GELU forms of epilogue (a), chosen once per 32-value chunk so that each
// chunk runs as straight-line code the scheduler can interleave.
enum : int { kGeluErf = 0, kGeluTanh = 1, kGeluPoly = 2 };

__device__ __forceinline__ int gelu_mode(const KParams& p) {
    return p.gelu_tanh ? kGeluTanh : (p.gelu_poly ? kGeluPoly : kGeluErf);
}

template <int KIND, int GM = kGeluErf>
__device__ __forceinline__ float epi_apply(float y, const KParams& p) {
    if constexpr (KIND == kEpiHardtanhGelu) {
        float t = p.fold_scale ? y : y * p.scale;  // folded: y already holds s*acc + s*b
        t = fminf(fmaxf(t, p.clamp_lo), p.clamp_hi);
        if constexpr (GM == kGeluPoly) return gelu_poly2(t);
        else if constexpr (GM == kGeluTanh) return gelu_tanh_form(t);
        else return gelu_erf(t);
    } else if constexpr (KIND == kEpiSwish) {
        // y * sigmoid(y); for y -> -inf, exp(-y) overflows to inf and the
        // quotient goes to 0 (the limit), never NaN.
        return __fdividef(y, 1.0f + __expf(-y)) * p.scale;
    } else {
        return y;
    }
}

// Order-preserving fp32 max through integer atomics (finite values; the
// target starts at -inf).  Non-negative floats order like signed ints,
// negative floats order inversely as unsigned ints.
__device__ __forceinline__ void atomic_max_f32(float* addr, float v) {
    v = v + 0.0f;  // -0.0 -> +0.0
    if (v >= 0.0f)
        atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
    else
        atomicMin(reinterpret_cast<unsigned*>(addr), __float_as_uint(v));
}

// v[j] = s * v[j] + s * b[n0 + j] in one FMA: (a) with the scale folded in.
__device__ __forceinline__ void fold_bias32(const KParams& p, int64_t n0, float (&v)[32]) {
    const float s = p.scale;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float bj = (p.bias != nullptr && n0 + j < p.N) ? __ldg(p.bias + n0 + j) : 0.0f;
        v[j] = fmaf(s, v[j], s * bj);
    }
}

// v[j] += b[n0 + j] for the columns that exist, four at a time (no extra
// 32-register copy of the bias).
__device__ __forceinline__ void add_bias32(const KParams& p, int64_t n0, float (&v)[32]) {
    if (p.bias == nullptr) return;
    if (p.vec_bias && n0 + 32 <= p.N) {
        const float4* b4 = reinterpret_cast<const float4*>(p.bias + n0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 t = __ldg(b4 + i);
            v[4 * i] += t.x; v[4 * i + 1] += t.y; v[4 * i + 2] += t.z; v[4 * i + 3] += t.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n0 + j < p.N) v[j] += __ldg(p.bias + n0 + j);
    }
}

// Where a direct-layout epilogue warp sends its finished 32 x 32 block: through
// its swizzled shared-memory staging tile and one TMA tile store (tmap set),
// or with plain per-thread stores.
struct EpiOut {
    const CUtensorMap* tmap;  // nullptr: plain stores
    float* stage;             // this warp's staging tile, 1024-byte aligned
    uint32_t stage_u32;
    int64_t row0;             // first output row of this warp's 32 rows
};

// Direct layout, elementwise kinds: this thread holds row m, columns n0..n0+31.
template <int KIND>
__device__ __forceinline__ void epi_store_direct(const KParams& p, const EpiOut& eo, int64_t m, int64_t n0,
                                                 float (&v)[32]) {
    if (KIND == kEpiHardtanhGelu && p.fold_scale)
        fold_bias32(p, n0, v);
    else
        add_bias32(p, n0, v);
    if constexpr (KIND == kEpiHardtanhGelu) {
        switch (gelu_mode(p)) {
            case kGeluPoly:
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND, kGeluPoly>(v[j], p);
                break;
            case kGeluTanh:
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND, kGeluTanh>(v[j], p);
                break;
            default:
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND, kGeluErf>(v[j], p);
                break;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND>(v[j], p);
    }
    if (eo.tmap != nullptr) {
        // Row r of the block goes to staging row r; its eight 16-byte pieces
        // are placed at piece index (i ^ (r % 8)), the 128-byte swizzle the
        // tensor map was encoded with, so the writes hit distinct banks.
        const int lane = threadIdx.x & 31;
        if (lane == 0) bulk_wait_read_all();  // the previous block has left this tile
        __syncwarp();
        float4* row = reinterpret_cast<float4*>(eo.stage + lane * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            row[i ^ (lane & 7)] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(eo.tmap, eo.stage_u32, static_cast<int32_t>(n0), static_cast<int32_t>(eo.row0));
            bulk_commit_group();
        }
        return;
    }
    if (m >= p.M) return;
    float* dst = p.out + m * p.N + n0;
    if (p.vec_out && n0 + 32 <= p.N) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int j = 0; j < 8; ++j) d4[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n0 + j < p.N) dst[j] = v[j];
    }
}

// Direct layout, pool kind: folds complete windows of this 32-column chunk
// into the running row maximum.
__device__ __forceinline__ void epi_pool_direct(const KParams& p, int64_t n0, float (&v)[32], float& best) {
    add_bias32(p, n0, v);
    const int k = p.pool_k;
    const float inv_k = 1.0f / static_cast<float>(k);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        acc += v[j];
        if (((j + 1) & (k - 1)) == 0) {
            if (n0 + j + 1 <= p.pool_limit) {
                float g = p.scale * gelu_sel(acc * inv_k, p);
                best = fmaxf(best, g);
            }
            acc = 0.0f;
        }
    }
}

// Swapped layout: this thread holds output column n, rows m0..m0+31.
template <int KIND>
__device__ __forceinline__ void epi_store_swapped(const KParams& p, const EpiOut& eo, int64_t n, int64_t m0,
                                                  float (&v)[32]) {
    const float bn = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + n) : 0.0f;
    const bool n_ok = n < p.N;
    const bool fold = KIND == kEpiHardtanhGelu && p.fold_scale;
    const float sbn = p.scale * bn;
    // all 32 results first (independent chains the scheduler can interleave),
    // then the stores: for each j the warp's lanes write one 128-byte line
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fold ? fmaf(p.scale, v[j], sbn) : v[j] + bn;
    if constexpr (KIND == kEpiHardtanhGelu) {
        switch (gelu_mode(p)) {
            case kGeluPoly:
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND, kGeluPoly>(v[j], p);
                break;
            case kGeluTanh:
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND, kGeluTanh>(v[j], p);
                break;
            default:
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND, kGeluErf>(v[j], p);
                break;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = epi_apply<KIND>(v[j], p);
    }
    if (eo.tmap != nullptr) {
        // The warp's 32 x 32 block of out (rows m0 + j, columns n - lane +
        // 0..31) through its staging tile and one TMA tile store: value j of
        // this lane goes to staging row j, column lane, in the 128-byte
        // swizzle of the tensor map (16-byte piece (lane / 4) ^ (j % 8)), so
        // each row's 32 writes hit 32 distinct banks.  The store clips rows
        // past M and columns past N.
        const int lane = threadIdx.x & 31;
        if (lane == 0) bulk_wait_read_all();  // the previous block has left this tile
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 32; ++j) eo.stage[j * 32 + (((lane >> 2) ^ (j & 7)) << 2) + (lane & 3)] = v[j];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(eo.tmap, eo.stage_u32, static_cast<int32_t>(n - lane), static_cast<int32_t>(m0));
            bulk_commit_group();
        }
        return;
    }
    if (n_ok) {
        const int64_t ld = p.N;
        float* o = p.out + m0 * ld + n;
        const int64_t rows = p.M - m0;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < rows) o[j * ld] = v[j];
    }
}

// Epilogue for one 32-column chunk c of a unit's tile, whose accumulator
// values (row r of the tile) are in v.  For the pool kind the chunk's complete
// windows are folded into `best`; epi_finish then combines it across CTAs.
template <bool SWAP, int BN>
__device__ __forceinline__ void epi_chunk(const KParams& p, const Unit& u, int r, int c, float (&v)[32],
                                          float& best, const EpiOut& eo) {
    if constexpr (!SWAP) {
        const int64_t m = static_cast<int64_t>(u.ta) * kBM + r;
        const int64_t n0 = u.col0 + c * 32;
        switch (p.kind) {
            case kEpiHardtanhGelu: epi_store_direct<kEpiHardtanhGelu>(p, eo, m, n0, v); break;
            case kEpiSwish: epi_store_direct<kEpiSwish>(p, eo, m, n0, v); break;
            case kEpiPoolMax: epi_pool_direct(p, n0, v, best); break;
            default: epi_store_direct<kEpiNone>(p, eo, m, n0, v); break;
        }
    } else {
        const int64_t n = static_cast<int64_t>(u.ta) * kBM + r;
        const int64_t m0 = u.col0 + c * 32;
        switch (p.kind) {
            case kEpiHardtanhGelu: epi_store_swapped<kEpiHardtanhGelu>(p, eo, n, m0, v); break;
            case kEpiSwish: epi_store_swapped<kEpiSwish>(p, eo, n, m0, v); break;
            default: epi_store_swapped<kEpiNone>(p, eo, n, m0, v); break;
        }
    }
    // Stores above may branch per lane (TMA issue, bounds); the warp must be
    // converged again for the next tcgen05.ld (.sync.aligned).
    __syncwarp();
}

template <bool SWAP>
__device__ __forceinline__ void epi_finish(const KParams& p, const Unit& u, int r, float best) {
    if constexpr (!SWAP) {
        const int64_t m = static_cast<int64_t>(u.ta) * kBM + r;
        if (p.kind == kEpiPoolMax && m < p.M && best > -INFINITY) atomic_max_f32(p.out + m, best);
    }
    __syncwarp();
}

// A global word read with acquire semantics (stream-K arrival counters,
// raised by other CTAs with atomicAdd after a __threadfence).
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// 3xTF32 low parts of one ring stage, by the 64 threads of the two split
// warps (ct = 0..63): for each of the stage's kVec float4, lo = x - hi with hi
// = x with the low 13 mantissa bits cleared (a TF32 value; x - hi is exact in
// fp32).  A batch of loads is issued before its stores: the raw and low
// halves of a stage do not overlap, and without that (or the restrict
// qualifiers) each store would have to complete before the next load issues,
// serialising the stage on the shared-memory latency.
constexpr int kSplitBatch = 8;  // float4 per thread in flight (measured: 8 = 16 > 32)

template <int kVec>
__device__ __forceinline__ void split_lo_parts(const float4* __restrict__ x4, float4* __restrict__ lo4, int ct) {
    static_assert(kVec % 64 == 0, "whole float4 rows for the 64 split threads");
    constexpr int kPer = kVec / 64;
#pragma unroll
    for (int b0 = 0; b0 < kPer; b0 += kSplitBatch) {
        float4 v[kSplitBatch];
#pragma unroll
        for (int u = 0; u < kSplitBatch; ++u)
            if (b0 + u < kPer) v[u] = x4[ct + 64 * (b0 + u)];
#pragma unroll
        for (int u = 0; u < kSplitBatch; ++u)
            if (b0 + u < kPer) {
                const float4 x = v[u];
                lo4[ct + 64 * (b0 + u)] = make_float4(x.x - __uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u),
                                                      x.y - __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u),
                                                      x.z - __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u),
                                                      x.w - __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u));
            }
    }
}

// The low parts of x for 3xTF32, written once per call into the workspace
// and copied with the tiles (each x tile is otherwise split again by every
// CTA that multiplies it): lo = x - (x with the low 13 mantissa bits
// cleared), the same value split_lo_parts computes.  n4: float4 of x.
__global__ void __launch_bounds__(256) fle_split_lo_kernel(const float4* __restrict__ x, float4* __restrict__ lo,
                                                           int64_t n4) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 v = x[i];
        lo[i] = make_float4(v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u),
                            v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u),
                            v.z - __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u),
                            v.w - __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u));
    }
}

// Barrier among the eight epilogue warps only (named barrier 1, 256 threads).
__device__ __forceinline__ void epilogue_bar_sync() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

// Limit of the wait in the kFinishOwn test mode (after it the CTA parks as usual).
constexpr uint64_t kFinishOwnWaitNs = 50000000ull;
// Limit of the default wait: the contributors of a shared tile run at the same
// time and, in the k-aligned splits, end within a few microseconds of each
// other (measured: M = 256 x 8192 x 8192 78.3 -> 74.5 us against parking at
// once, M = 16 2.5% faster).
constexpr uint64_t kFinishAutoWaitNs = 20000ull;

// Whether the CTA holding k-block 0 of a shared tile finishes it from its own
// accumulator: only when all `others` contributors have parked their partials
// (arrival counter == others).  It waits for them up to a limit: 20 us by
// default, 50 ms in the kFinishOwn test mode; kFinishPark never waits and
// never finishes.  No contributor waits for the k-block-0 CTA, so the others
// arrive whenever they run; if the limit passes first (a contributor not yet
// resident, say), the CTA parks its partial too and the last arrival
// finishes the tile, which is correct in every case.
__device__ __forceinline__ bool sk_take_own(const KParams& p, const unsigned* counter, unsigned others) {
    if (p.sk_finish == kFinishPark) return false;
    unsigned c = ld_acquire_u32(counter);
    if (c != others) {
        const uint64_t limit = (p.sk_finish == kFinishOwn) ? kFinishOwnWaitNs : kFinishAutoWaitNs;
        const uint64_t t0 = global_timer_ns();
        while (c != others && global_timer_ns() - t0 < limit) {
            __nanosleep(64);
            c = ld_acquire_u32(counter);
        }
    }
    return c == others;
}

// ----------------------------------------------------------------------------
// The kernel
// ----------------------------------------------------------------------------
template <int BN, int PREC, bool SWAP, int KPS>
__global__ void __launch_bounds__(kThreads, 1)
fle_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmXlo, const __grid_constant__ CUtensorMap tmOut,
                const KParams p) {
    using C = Cfg<BN, PREC, SWAP, KPS>;
    constexpr int S = C::kStages;
    constexpr uint32_t kIdesc = idesc_tf32(kBM, BN);
    // k-blocks per TMEM accumulation chain (see the epilogue role); a
    // multiple of KPS, so that chains and stages start on the same k-block
    constexpr int kChunkKb = (PREC == kPrec3xTF32) ? 4 : (1 << 30);
    static_assert(kChunkKb % KPS == 0, "accumulation chains hold whole stages");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t* epi_stage = smem + S * C::kStageBytes;  // C::kEpiStageBytes
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi_stage + C::kEpiStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // two slots used in turn: a slot is written again only after every
    // epilogue thread has passed a later barrier, so after its read
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
    // checking build: the work tag of each stage and accumulator buffer
    volatile uint32_t* stage_tag = reinterpret_cast<volatile uint32_t*>(tmem_slot + 8);
    volatile uint32_t* acc_tag = stage_tag + 12;
    (void)stage_tag;
    (void)acc_tag;

    auto bar_full = [&](int s) { return smem_u32(bars + s); };
    auto bar_conv = [&](int s) { return smem_u32(bars + S + s); };
    auto bar_empty = [&](int s) { return smem_u32(bars + 2 * S + s); };
    auto bar_accf = [&](int b) { return smem_u32(bars + 3 * S + b); };
    auto bar_acce = [&](int b) { return smem_u32(bars + 3 * S + 2 + b); };
    const uint32_t bar_drain = smem_u32(bars + 3 * S + 4);
    // stage s: [A hi | B hi | A lo | B lo], each part KPS k-blocks
    auto sA = [&](int s) { return sbase + s * C::kStageBytes; };
    auto sB = [&](int s) { return sbase + s * C::kStageBytes + KPS * C::kABytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_conv(s), 2);
            mbar_init(bar_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf(b), 1);
            mbar_init(bar_acce(b), 8);  // one arrival per epilogue warp
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (PREC == kPrec3xTF32 && p.lo_mem) tma_prefetch_desc(&tmXlo);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    __syncwarp();  // warp 0 branched on thread 0 above
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            Sched sc;
            sc.init(p, blockIdx.x, gridDim.x);
            Unit u;
            while (ok && sc.next(p, u)) {
                for (int kb = u.kb0; kb < u.kb1; kb += KPS) {
                    const int n = (u.kb1 - kb < KPS) ? u.kb1 - kb : KPS;  // k-blocks in this stage
                    if (!mbar_wait_bounded(bar_empty(stage), phase ^ 1u, abort_flag, p.timeout_ns,
                                           kWhereProdEmpty)) {
                        ok = false;
                        break;
                    }
                    if constexpr (kCheckBarriers) {
                        if (mbar_test_wait(bar_full(stage), phase)) record_error(kErrProtocol, kWhereProdEmpty);
                        stage_tag[stage] = work_tag(u.t, kb);
                    }
                    // 3xTF32 with x's low parts in memory: they are copied into
                    // the low half beside the tiles (x is B in the swapped
                    // order, A in the direct one)
                    const uint32_t xlo_bytes =
                        (PREC == kPrec3xTF32 && p.lo_mem) ? static_cast<uint32_t>(SWAP ? C::kBBytes : C::kABytes) : 0u;
                    mbar_arrive_expect_tx(bar_full(stage), n * (C::kKbBytes + xlo_bytes));
                    for (int j = 0; j < n; ++j) {
                        tma_load_2d(sA(stage) + j * C::kABytes, &tmA, bar_full(stage), (kb + j) * kBK, u.ta * kBM);
                        tma_load_2d(sB(stage) + j * C::kBBytes, &tmB, bar_full(stage), (kb + j) * kBK, u.tb * BN);
                        if (xlo_bytes) {
                            if constexpr (SWAP)
                                tma_load_2d(sB(stage) + C::kLoadBytes + j * C::kBBytes, &tmXlo, bar_full(stage),
                                            (kb + j) * kBK, u.tb * BN);
                            else
                                tma_load_2d(sA(stage) + C::kLoadBytes + j * C::kABytes, &tmXlo, bar_full(stage),
                                            (kb + j) * kBK, u.ta * kBM);
                        }
                    }
                    ++fills;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
            // Every issued copy must have landed before the CTA may exit.
            for (long long f = (fills > S ? fills - S : 0); f < fills; ++f) {
                const int s = static_cast<int>(f % S);
                const uint32_t ph = static_cast<uint32_t>((f / S) & 1);
                volatile int never = 0;
                mbar_wait_bounded(bar_full(s), ph, &never, kDrainTimeoutNs, kWhereProdDrain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            Sched sc;
            sc.init(p, blockIdx.x, gridDim.x);
            Unit u;
            while (ok && sc.next(p, u)) {
              // one accumulation chain per chunk of k-blocks (3xTF32) or per unit (TF32)
              for (int kc = u.kb0; ok && kc < u.kb1; kc += kChunkKb) {
                const int kce = (u.kb1 - kc > kChunkKb) ? kc + kChunkKb : u.kb1;
                if (!mbar_wait_bounded(bar_acce(buf), acc_phase ^ 1u, abort_flag, p.timeout_ns,
                                       kWhereMmaAccEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                if constexpr (kCheckBarriers) {
                    acc_tag[buf] = work_tag(u.t, kc);
                    __threadfence_block();
                }
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = kc; kb < kce; kb += KPS) {
                    const int n = (kce - kb < KPS) ? kce - kb : KPS;  // k-blocks in this stage
                    // hi x hi reads only the copied tiles: it runs as soon as
                    // they land (3xTF32: while the split warps write the low
                    // parts), the products with a low part after the split
                    if (!mbar_wait_bounded(bar_full(stage), phase, abort_flag, p.timeout_ns, kWhereMmaFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    if constexpr (kCheckBarriers) check_tag(stage_tag[stage], work_tag(u.t, kb), kWhereMmaFull);
                    for (int j = 0; j < n; ++j) {
                        const uint64_t a_hi = smem_desc_sw128(sA(stage) + j * C::kABytes);
                        const uint64_t b_hi = smem_desc_sw128(sB(stage) + j * C::kBBytes);
#pragma unroll
                        for (int k = 0; k < kBK / kUmmaK; ++k) {
                            // advance 8 fp32 = 32 bytes along K inside the swizzle atom
                            const uint64_t koff = static_cast<uint64_t>(k * 2);
                            const uint32_t acc = (kb > kc || j > 0 || k > 0) ? 1u : 0u;
                            mma_tf32(d_tmem, a_hi + koff, b_hi + koff, kIdesc, acc);
                        }
                    }
                    if constexpr (PREC == kPrec3xTF32) {
                        if (!mbar_wait_bounded(bar_conv(stage), phase, abort_flag, p.timeout_ns, kWhereMmaFull)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        for (int j = 0; j < n; ++j) {
                            const uint64_t a_hi = smem_desc_sw128(sA(stage) + j * C::kABytes);
                            const uint64_t b_hi = smem_desc_sw128(sB(stage) + j * C::kBBytes);
                            const uint64_t a_lo = smem_desc_sw128(sA(stage) + C::kLoadBytes + j * C::kABytes);
                            const uint64_t b_lo = smem_desc_sw128(sB(stage) + C::kLoadBytes + j * C::kBBytes);
#pragma unroll
                            for (int k = 0; k < kBK / kUmmaK; ++k) {
                                const uint64_t koff = static_cast<uint64_t>(k * 2);
                                mma_tf32(d_tmem, a_lo + koff, b_hi + koff, kIdesc, 1u);
                                mma_tf32(d_tmem, a_hi + koff, b_lo + koff, kIdesc, 1u);
                            }
                        }
                    }
                    mma_commit(bar_empty(stage));
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(bar_accf(buf));
                buf ^= 1;
                if (buf == 0) acc_phase ^= 1u;
              }
            }
            // All issued MMAs must be complete before TMEM is released.
            mma_commit(bar_drain);
            volatile int never = 0;
            mbar_wait_bounded(bar_drain, 0, &never, kDrainTimeoutNs, kWhereDrain);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------ 3xTF32 split
        if constexpr (PREC == kPrec3xTF32) {
            const int ct = threadIdx.x - 64;  // 0..63
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            Sched sc;
            sc.init(p, blockIdx.x, gridDim.x);
            Unit u;
            while (ok && sc.next(p, u)) {
                for (int kb = u.kb0; kb < u.kb1; kb += KPS) {
                    int got = 0;
                    if (lane == 0)
                        got = mbar_wait_bounded(bar_full(stage), phase, abort_flag, p.timeout_ns, kWhereConvFull);
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) { ok = false; break; }
                    if constexpr (kCheckBarriers) {
                        if (lane == 0) check_tag(stage_tag[stage], work_tag(u.t, kb), kWhereConvFull);
                    }
                    // hi = x with the low 13 mantissa bits cleared (a TF32
                    // value); lo = x - hi (exact in fp32) goes to the same
                    // offset in the lo half.  The tensor core reads the raw x
                    // of the hi half as exactly that hi: kind::tf32 truncates
                    // an fp32 operand to TF32 (checked on the device by the
                    // operand-conversion test).
                    const float4* x4 = reinterpret_cast<const float4*>(smem + stage * C::kStageBytes);
                    float4* lo4 = reinterpret_cast<float4*>(smem + stage * C::kStageBytes + C::kLoadBytes);
                    if (p.lo_mem) {
                        // only W's tile: A in the swapped order, B in the direct one
                        constexpr int kWOff = SWAP ? 0 : C::kABytes / 16;
                        split_lo_parts<(SWAP ? C::kABytes : C::kBBytes) / 16>(x4 + kWOff, lo4 + kWOff, ct);
                    } else {
                        split_lo_parts<C::kLoadBytes / 16>(x4, lo4, ct);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_conv(stage));
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // The stream-K counters and (kind (c)) out are set by the prep
        // kernel just before this one, which may still be running.
        griddep_wait();
        // Eight warps.  Warp w reads TMEM lane quadrant w % 4 (tile rows
        // 32*(w%4) .. +31; a warp may only touch its own quadrant) and one
        // half of the tile's 32-column chunks, so each SM sub-partition runs
        // two independent epilogue warps.
        const int q = warp & 3;
        const int half = (warp - 4) >> 2;
        const int r = q * 32 + lane;  // tile row = TMEM lane of this thread
        EpiOut eo;
        eo.tmap = p.tma_out ? &tmOut : nullptr;
        eo.stage = reinterpret_cast<float*>(epi_stage + (warp - 4) * kEpiTileBytes);
        eo.stage_u32 = smem_u32(eo.stage);
        eo.row0 = 0;
        constexpr int kChunks = BN / 32;
        constexpr int kHalf = (kChunks + 1) / 2;  // chunks per half
        const int c_lo = half * kHalf;
        int buf = 0;
        uint32_t acc_phase = 0;
        // 3xTF32 accumulates each kChunkKb-deep slice of K in a fresh TMEM
        // buffer and sums the slices here, in fp32 registers with
        // round-to-nearest: the tensor core's own accumulation rounds toward
        // zero, whose bias would otherwise grow with the length of K.
        constexpr bool kRegAcc = (PREC == kPrec3xTF32);
        float accr[kRegAcc ? kHalf * 32 : 1];
        int fsel = 0;  // next last_flag slot (the same in every epilogue thread)
        Sched sc;
        sc.init(p, blockIdx.x, gridDim.x);
        Unit u;
        bool ok = true;
        while (ok && sc.next(p, u)) {
            // 32-column chunks of this tile that hold any output, and this
            // warp's share [c_lo, c_lo + mine) of them (warp-uniform)
            const int64_t cols_left = (SWAP ? p.M : p.N) - static_cast<int64_t>(u.tb) * BN;
            const int nchunks = static_cast<int>(cols_left >= BN ? kChunks : (cols_left + 31) / 32);
            const int mine = nchunks - c_lo < 0 ? 0 : (nchunks - c_lo > kHalf ? kHalf : nchunks - c_lo);
            eo.row0 = static_cast<int64_t>(u.ta) * kBM + q * 32;

            auto wait_acc = [&](int kc) -> bool {
                int got = 0;
                if (lane == 0) {
                    got = mbar_wait_bounded(bar_accf(buf), acc_phase, abort_flag, p.timeout_ns, kWhereEpiAccFull);
                    if constexpr (kCheckBarriers) {
                        if (got) check_tag(acc_tag[buf], work_tag(u.t, kc), kWhereEpiAccFull);
                    }
                }
                got = __shfl_sync(0xffffffffu, got, 0);
                if (got) tc_fence_after_sync();
                return got != 0;
            };
            auto release_acc = [&]() {
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acce(buf));
                __syncwarp();
                buf ^= 1;
                if (buf == 0) acc_phase ^= 1u;
            };
            auto t_row = [&]() {
                return tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * BN);
            };

            uint32_t t_acc = 0;
            if constexpr (kRegAcc) {
#pragma unroll
                for (int j = 0; j < (kRegAcc ? kHalf * 32 : 1); ++j) accr[j] = 0.0f;
                for (int kc = u.kb0; kc < u.kb1; kc += kChunkKb) {
                    if (!wait_acc(kc)) { ok = false; break; }
                    const uint32_t tr = t_row();
#pragma unroll
                    for (int lc = 0; lc < kHalf; ++lc) {
                        if (lc >= mine) break;
                        float v[32];
                        tmem_ld32_wait(tr + (c_lo + lc) * 32, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) accr[lc * 32 + j] += v[j];
                    }
                    release_acc();
                }
                if (!ok) break;
            } else {
                if (!wait_acc(u.kb0)) break;
                t_acc = t_row();
            }
            // The 32 accumulator values of this warp's local chunk lc, in
            // registers (3xTF32, with compile-time lc) or in TMEM (TF32).
#define FLE_LOAD_ACC(lc, v)                                                                    \
    do {                                                                                       \
        if constexpr (kRegAcc) {                                                               \
            _Pragma("unroll") for (int j_ = 0; j_ < 32; ++j_) v[j_] = accr[(lc) * 32 + j_];    \
        } else {                                                                               \
            tmem_ld32_wait(t_acc + (c_lo + (lc)) * 32, v);                                     \
        }                                                                                      \
    } while (0)

            if (!u.partial) {
                float best = -INFINITY;
#define FLE_EPI_BODY(lc)                                     \
    {                                                        \
        float v[32];                                         \
        FLE_LOAD_ACC(lc, v);                                 \
        epi_chunk<SWAP, BN>(p, u, r, c_lo + (lc), v, best, eo);  \
    }
                if constexpr (kRegAcc) {
#pragma unroll
                    for (int lc = 0; lc < kHalf; ++lc)
                        if (lc < mine) FLE_EPI_BODY(lc)
                } else {
#pragma unroll 1
                    for (int lc = 0; lc < mine; ++lc) FLE_EPI_BODY(lc)
                }
#undef FLE_EPI_BODY
                epi_finish<SWAP>(p, u, r, best);
                if constexpr (!kRegAcc) release_acc();
            } else {
                // A unit of a tile whose k-blocks are split over CTAs first ..
                // last.  The CTA holding k-block 0 (the last unit of its range,
                // while the others ran the tile's later k-blocks as their first
                // units) normally ends last: if every other contributor has
                // already parked its partial, it adds them to its own
                // accumulator and runs the epilogue.  Otherwise it parks its
                // partial too, and whichever contributor arrives last sums all
                // partials.  No CTA ever waits for another.  Partials are summed
                // in CTA order (= k order), so the result does not depend on
                // who does it.
                const int64_t tsk = u.sk_tile;
                const int first = sk_cta_of(tsk * p.num_kb, p.sk_iters, p.sk_grid);
                const int last = sk_cta_of((tsk + 1) * p.num_kb - 1, p.sk_iters, p.sk_grid);
                const unsigned others = static_cast<unsigned>(last - first);
                unsigned* counter = p.counters + tsk;
                bool own = false;
                if (u.kb0 == 0) {
                    volatile int* lf = last_flag + fsel;
                    fsel ^= 1;
                    if (threadIdx.x == 128) *lf = sk_take_own(p, counter, others) ? 1 : 0;
                    __syncwarp();  // named barriers are .aligned: whole warps arrive
                    epilogue_bar_sync();
                    own = *lf != 0;
                }
                bool fix = own;
                if (!own) {
                    // park the partial, column-major inside the tile (element
                    // (row, col) at col * 128 + row: a warp's lanes write 32
                    // consecutive floats), then count it
                    float* slot = p.ws + static_cast<size_t>(p.sk_slots * blockIdx.x + u.slot) * kBM * BN;
#define FLE_PARK_BODY(lc)                                                                 \
    {                                                                                     \
        float v[32];                                                                      \
        FLE_LOAD_ACC(lc, v);                                                              \
        float* d = slot + static_cast<size_t>((c_lo + (lc)) * 32) * kBM + r;              \
        _Pragma("unroll") for (int j = 0; j < 32; ++j) __stcg(d + j * kBM, v[j]);         \
    }
                    if constexpr (kRegAcc) {
#pragma unroll
                        for (int lc = 0; lc < kHalf; ++lc)
                            if (lc < mine) FLE_PARK_BODY(lc)
                    } else {
#pragma unroll 1
                        for (int lc = 0; lc < mine; ++lc) FLE_PARK_BODY(lc)
                    }
#undef FLE_PARK_BODY
                    if constexpr (!kRegAcc) release_acc();
                    __threadfence();
                    epilogue_bar_sync();
                    volatile int* lf = last_flag + fsel;
                    fsel ^= 1;
                    if (threadIdx.x == 128) *lf = (atomicAdd(counter, 1u) == others) ? 1 : 0;
                    __syncwarp();
                    epilogue_bar_sync();
                    fix = *lf != 0;
                }
                if (fix) {
                    __threadfence();
                    float best = -INFINITY;
                    auto src_of = [&](int cc, int c) {
                        const int sl = sk_slot_of(cc, tsk, p.sk_iters, p.sk_grid, p.num_kb);
                        return p.ws + static_cast<size_t>(p.sk_slots * cc + sl) * kBM * BN +
                               static_cast<size_t>(c * 32) * kBM + r;
                    };
                    // start from the own accumulator (contributors first+1 ..
                    // last to add) or from zero (first .. last); loads of up to
                    // three contributors are in flight together
#define FLE_FIX_BODY(lc)                                                                      \
    {                                                                                         \
        const int c = c_lo + (lc);                                                            \
        float v[32];                                                                          \
        if (own) {                                                                            \
            FLE_LOAD_ACC(lc, v);                                                              \
        } else {                                                                              \
            _Pragma("unroll") for (int j = 0; j < 32; ++j) v[j] = 0.0f;                       \
        }                                                                                     \
        int cc = own ? first + 1 : first;                                                     \
        for (; cc + 2 <= last; cc += 3) {                                                     \
            const float* s0 = src_of(cc, c);                                                  \
            const float* s1 = src_of(cc + 1, c);                                              \
            const float* s2 = src_of(cc + 2, c);                                              \
            float t0[32], t1[32], t2[32];                                                     \
            _Pragma("unroll") for (int j = 0; j < 32; ++j) {                                  \
                t0[j] = __ldcg(s0 + j * kBM);                                                 \
                t1[j] = __ldcg(s1 + j * kBM);                                                 \
                t2[j] = __ldcg(s2 + j * kBM);                                                 \
            }                                                                                 \
            _Pragma("unroll") for (int j = 0; j < 32; ++j) v[j] = ((v[j] + t0[j]) + t1[j]) + t2[j]; \
        }                                                                                     \
        for (; cc <= last; ++cc) {                                                            \
            const float* s0 = src_of(cc, c);                                                  \
            float t0[32];                                                                     \
            _Pragma("unroll") for (int j = 0; j < 32; ++j) t0[j] = __ldcg(s0 + j * kBM);      \
            _Pragma("unroll") for (int j = 0; j < 32; ++j) v[j] += t0[j];                     \
        }                                                                                     \
        epi_chunk<SWAP, BN>(p, u, r, c, v, best, eo);                                         \
    }
                    if constexpr (kRegAcc) {
#pragma unroll
                        for (int lc = 0; lc < kHalf; ++lc)
                            if (lc < mine) FLE_FIX_BODY(lc)
                    } else {
#pragma unroll 1
                        for (int lc = 0; lc < mine; ++lc) FLE_FIX_BODY(lc)
                    }
#undef FLE_FIX_BODY
                    epi_finish<SWAP>(p, u, r, best);
                    if (threadIdx.x == 128) {
                        *counter = 0u;
                        atomicAdd(&g_finish_count[own ? 0 : 1], 1u);
                    }
                    __syncwarp();
                }
                if constexpr (!kRegAcc) {
                    if (own) release_acc();
                }
            }
#undef FLE_LOAD_ACC
        }
    }

    // Roles branch on the lane (one issuing thread per warp); reconverge every
    // warp before the CTA barrier, which whole warps must reach together.
    __syncwarp();
    // Epilogue TMA stores read the staging tiles until they complete.
    if (warp >= 4 && lane == 0) bulk_wait_all();
    __syncwarp();
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// K == 0: out = epilogue(b).  One thread per output element (elementwise
// kinds) or per row (pool kind).
__global__ void fle_bias_only_kernel(const KParams p) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (p.kind == kEpiPoolMax) {
        if (i >= p.M) return;
        float best = -INFINITY;
        for (int64_t w0 = 0; w0 + p.pool_k <= p.pool_limit; w0 += p.pool_k) {
            float acc = 0.0f;
            for (int t = 0; t < p.pool_k; ++t) acc += p.bias ? p.bias[w0 + t] : 0.0f;
            best = fmaxf(best, p.scale * gelu_sel(acc / static_cast<float>(p.pool_k), p));
        }
        p.out[i] = best;
        return;
    }
    if (i >= p.M * p.N) return;
    const float y = p.bias ? p.bias[i % p.N] : 0.0f;
    float o;
    switch (p.kind) {
        case kEpiHardtanhGelu: {
            const float yy = p.fold_scale ? p.scale * y : y;
            o = p.gelu_tanh ? epi_apply<kEpiHardtanhGelu, kGeluTanh>(yy, p) : epi_apply<kEpiHardtanhGelu>(yy, p);
            break;
        }
        case kEpiSwish: o = epi_apply<kEpiSwish>(y, p); break;
        default: o = y; break;
    }
    p.out[i] = o;
}

// Per-call preparation on the caller's stream: out[M] = -inf for the pool
// kind (the row maximum is combined with atomics) and zeroed stream-K
// arrival counters.
__global__ void fle_prep_kernel(float* fill, int64_t n_fill, unsigned* counters, int n_counters) {
    // The GEMM that follows touches these words only after griddep_wait(),
    // so it may be launched (and load its first tiles) right away.
    griddep_launch_dependents();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (fill != nullptr && i < n_fill) fill[i] = -INFINITY;
    if (counters != nullptr && i < n_counters) counters[i] = 0u;
}

// Pooled weights for epilogue (c): AvgPool1d(k, stride k) over the output
// features commutes with the Linear map, so the mean of k consecutive outputs
// equals one output of the Linear whose weight row is the mean of the k
// weight rows (and likewise for the bias).  Wp[j][:] = mean_t W[j*k + t][:],
// bp[j] = mean_t b[j*k + t], for j < P.  Each thread sums k float4 rows in
// order t = 0..k-1 and scales by 1/k (exact: k is a power of two).  K % 4 == 0.
__global__ void fle_pool_weights_kernel(const float* __restrict__ W, const float* __restrict__ b,
                                        int64_t P, int64_t K, int k, float* __restrict__ Wp,
                                        float* __restrict__ bp) {
    const int64_t kv = K / 4;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const float inv_k = 1.0f / static_cast<float>(k);
    if (i < P * kv) {
        const int64_t j = i / kv;
        const int64_t c = i - j * kv;
        const float4* src = reinterpret_cast<const float4*>(W) + (j * k) * kv + c;
        float4 acc = __ldcs(src);
        for (int t = 1; t < k; ++t) {
            const float4 w = __ldcs(src + t * kv);
            acc.x += w.x; acc.y += w.y; acc.z += w.z; acc.w += w.w;
        }
        reinterpret_cast<float4*>(Wp)[i] = make_float4(acc.x * inv_k, acc.y * inv_k, acc.z * inv_k, acc.w * inv_k);
    }
    if (b != nullptr && bp != nullptr && i < P) {
        float acc = b[i * k];
        for (int t = 1; t < k; ++t) acc += b[i * k + t];
        bp[i] = acc * inv_k;
    }
}

// Test hook: the epilogue's scalar functions on n inputs (kind 0: erf,
// 1: GELU, 2: swish with scale 1, 3: GELU in its tanh form, 4: the
// polynomial GELU of |t| <= 2), for checks against CUDA's erff / expf / tanhf.
__global__ void fle_math_probe_kernel(const float* in, float* out, int64_t n, int which) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = in[i];
    if (which == 0) out[i] = erf_as7126(v);
    else if (which == 1) out[i] = gelu_erf(v);
    else if (which == 2) out[i] = __fdividef(v, 1.0f + __expf(-v));
    else if (which == 3) out[i] = gelu_tanh_form(v);
    else out[i] = gelu_poly2(v);
}
__global__ void fle_math_reference_kernel(const float* in, float* out, int64_t n, int which) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = in[i];
    if (which == 0) out[i] = erff(v);
    else if (which == 1) out[i] = v * 0.5f * (1.0f + erff(v * 0.70710678118654752440f));
    else if (which == 2) out[i] = v / (1.0f + expf(-v));
    else if (which == 3) out[i] = 0.5f * v * (1.0f + tanhf(0.79788456080286535588f * (v + 0.044715f * v * v * v)));
    else out[i] = v * 0.5f * (1.0f + erff(v * 0.70710678118654752440f));
}

// Test hook: one thread waits on a barrier nothing arrives on.
__global__ void fle_bounded_wait_test_kernel(uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
        mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, timeout_ns, kWhereTest);
    }
}

}  // namespace fle
