// fle_kernel_pair.cuh -- the fused Linear + epilogue kernel on CTA pairs.
//
// Two CTAs of a cluster, on two SMs, compute one output tile of 256 A rows
// with tcgen05.mma.cta_group::2: each CTA loads its own 128 rows of A and its
// half of the B rows into its shared memory, and the pair's MMA reads A and
// B from both.  Per SM this halves the B operand traffic through shared memory
// compared with a single-CTA tile, at the same MMA work per SM.  The
// accumulator rows are split across the two SMs' TMEM (rows 0-127 in the even
// CTA, 128-255 in the odd one), so each CTA runs the epilogue of its own 128
// rows.  Tile widths (B rows): 256 or 224 (direct order), 512 (two 256-wide
// MMAs per k-step sharing the A tile, single-pass TF32), and 32, 64 or 128
// in the swapped order (A = W, B = x) of the skinny shapes.  The 512-wide
// kernel also runs mixed-width plans (KParams::mix_wide): 384-wide tiles are
// a 256-wide and a 128-wide MMA sharing the A tile, whose 64 B rows per CTA
// come through a second tensor map (tmB2, 64-row boxes).
//
// Roles are those of fle_gemm_kernel.  Only the even ("leader") CTA's MMA
// thread issues MMAs; the leader's commits are multicast to both CTAs' empty
// and accumulator-full barriers; both CTAs' epilogues release the leader's
// accumulator-empty barrier.  No load uses cluster multicast.
//   TF32:   both CTAs' tile copies are counted on the leader's full barrier.
//   3xTF32: each CTA's copies complete on its own full barrier; its split
//           warps then write the TF32 low parts (x minus x with the low 13
//           mantissa bits cleared; the tensor core reads the raw fp32 value
//           as that truncated high part) and arrive on the leader's split
//           barrier, which the MMA waits on.  The three products of each
//           k-step accumulate in 128-deep slices of K, summed in registers
//           (the tensor core's own accumulation rounds toward zero).
// Every signal one CTA sends the other is waited for before the receiver
// exits (the last accumulator releases by the leader's MMA thread, the rest
// by the roles that consume them, then a bounded two-way handshake), so no
// arrival can reach the shared memory of the next CTA on that SM.
#pragma once

#include "fle_kernel.cuh"

namespace fle {

constexpr int kPairBN = 256;  // pair tile N (B rows), direct operand order
constexpr int kPairBNNarrow = 224;  // the narrower direct tile (fills uneven waves better)
constexpr int kPairBNWide = 512;    // two 256-wide MMAs sharing the A tile (TF32)
constexpr int kPairBM = 256;  // pair tile M (A rows)

// KPS: k-blocks per ring stage, as in Cfg: [A k-blocks | B k-blocks].
// BN: B rows of the pair tile (each CTA loads BN / 2 of them).  SWAP: A = W
// and B = x, for the skinny shapes (BN = 32, 64, 128 covers M).
template <int PREC, int KPS = 1, int BN = kPairBN, bool SWAP = false>
struct PairCfg {
    static constexpr int kBKW = kBK;  // k-block width: 32 fp32, one 128-byte swizzle row
    static constexpr int kABytes = kBM * kBKW * 4;            // this CTA's 128 A rows, one k-block
    static constexpr int kBBytes = (BN / 2) * kBKW * 4;       // this CTA's BN / 2 B rows, one k-block
    // Tiles wider than 256 are kNSub MMAs of N = kSubN sharing the A tile;
    // each CTA holds its kSubN / 2 rows of every sub-tile, one after another.
    static constexpr int kNSub = BN > 256 ? BN / 256 : 1;
    static constexpr int kSubN = BN / kNSub;
    static constexpr int kSubBBytes = kBBytes / kNSub;
    static constexpr int kKbBytes = kABytes + kBBytes;
    static constexpr int kLoadBytes = KPS * kKbBytes;         // TMA bytes per full stage and CTA
    static constexpr int kStageBytes = kLoadBytes * (PREC == kPrec3xTF32 ? 2 : 1);
    // TMA-store staging, one 32 x 32 tile per epilogue warp
    static constexpr int kEpiStageBytes = kEpiWarps * kEpiTileBytes;
    static constexpr int kStagesRaw = (kSmemStageBudget - kEpiStageBytes) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    // TMEM accumulator buffers and columns per buffer: two of BN, or of 256
    // for BN = 224 (its second buffer starts at column 256); one of 512 for
    // the 512-wide tile, which fills the whole TMEM
    static constexpr int kNumAcc = BN > 256 ? 1 : 2;
    static constexpr int kAccCols = BN > 256 ? BN : (BN > 128 ? 256 : BN);
    static constexpr int kTmemAll = kNumAcc * kAccCols;
    static constexpr int kTmemCols = (kTmemAll <= 32) ? 32 : (kTmemAll <= 64) ? 64
                                    : (kTmemAll <= 128) ? 128 : (kTmemAll <= 256) ? 256 : 512;
    // full, split, empty per stage; accf, acce per buffer; drain; exit
    static constexpr int kNumBars = 3 * kStages + 4 + 2;
    // (the checking build keeps its stage and accumulator tags after the 32
    // bytes of TMEM address and flags)
    static constexpr int kSmemBytes =
        1024 + kStages * kStageBytes + kEpiStageBytes + kNumBars * 8 + 32 + (kCheckBarriers ? 64 : 0);
    static_assert(kStages >= 2, "need at least two stages");
    static_assert(KPS == 1 || KPS == 2, "one or two k-blocks per stage");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 512, "pair tile N: 32..512, whole 32-column chunks");
    static_assert(kSubN % 16 == 0 && kSubN <= 256, "MMA N for M = 256 is a multiple of 16, at most 256");
    static_assert(BN <= 256 || (BN % 256 == 0 && PREC == kPrecTF32 && !SWAP),
                  "wide tiles: whole 256-column sub-tiles, single-pass TF32, direct operand order");
    static_assert(kSubBBytes % 1024 == 0, "B sub-tiles keep 1024-byte alignment");
    static_assert(kTmemAll <= 512, "TMEM has 512 columns");
    static_assert(kBBytes % 1024 == 0, "B halves keep 1024-byte alignment");
    static_assert(kSmemBytes <= 232448, "exceeds 227 KB of shared memory per block");
};

template <int PREC, int KPS, int BN, bool SWAP>
__global__ void __launch_bounds__(kThreads, 1)
fle_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmXlo,
                     const __grid_constant__ CUtensorMap tmOut, const KParams p) {
    using C = PairCfg<PREC, KPS, BN, SWAP>;
    constexpr bool k3x = (PREC == kPrec3xTF32);
    constexpr int S = C::kStages;
    constexpr uint32_t kIdesc = idesc_tf32(kPairBM, C::kSubN);
    // 512-wide kernel: a 384-wide unit's second MMA is 128 wide (64 B rows
    // per CTA, the first half of the sub-tile's slot)
    constexpr bool kWide = BN > 256;
    constexpr int kNarrowSubN = kMixNarrow - 256;
    constexpr uint32_t kIdescNarrow = idesc_tf32(kPairBM, kNarrowSubN);
    static_assert(!kWide || (BN == kMixWide && C::kNSub == 2 && C::kSubN == 256),
                  "mixed plans: 512-wide tiles of two 256-wide sub-tiles");
    constexpr int kBKW = C::kBKW;
    constexpr int kChunkKb = k3x ? 128 / kBKW : (1 << 30);  // k-blocks per TMEM accumulation chain
    static_assert(kChunkKb % KPS == 0, "accumulation chains hold whole stages");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t* epi_stage = smem + S * C::kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi_stage + C::kEpiStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // two slots used in turn (see fle_gemm_kernel)
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
    // checking build: the work tag of each stage (per CTA) and of each
    // accumulator buffer (in the leader)
    volatile uint32_t* stage_tag = reinterpret_cast<volatile uint32_t*>(tmem_slot + 8);
    volatile uint32_t* acc_tag = stage_tag + 12;
    (void)stage_tag;
    (void)acc_tag;

    auto bar_full = [&](int s) { return smem_u32(bars + s); };
    auto bar_split = [&](int s) { return smem_u32(bars + S + s); };
    auto bar_empty = [&](int s) { return smem_u32(bars + 2 * S + s); };
    auto bar_accf = [&](int b) { return smem_u32(bars + 3 * S + b); };
    auto bar_acce = [&](int b) { return smem_u32(bars + 3 * S + 2 + b); };
    const uint32_t bar_drain = smem_u32(bars + 3 * S + 4);
    const uint32_t bar_exit = smem_u32(bars + 3 * S + 5);
    // stage s: [A | B | A lo | B lo]; the lo half exists for 3xTF32 only
    auto sA = [&](int s) { return sbase + s * C::kStageBytes; };
    auto sB = [&](int s) { return sbase + s * C::kStageBytes + KPS * C::kABytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader, 1: peer
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    // The peer's abort flag: a wait that times out raises it too, so that the
    // other CTA's roles stop waiting for barriers this CTA no longer signals.
    const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_split(s), 4);  // 2 split warps in each CTA of the pair
            mbar_init(bar_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf(b), 1);
            mbar_init(bar_acce(b), 16);  // 8 epilogue warps in each CTA of the pair
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_exit, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (kWide && p.mix_wide > 0) tma_prefetch_desc(&tmB2);
        if (k3x && p.lo_mem) tma_prefetch_desc(&tmXlo);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish_pair();
    }
    __syncwarp();  // warp 0 branched on thread 0 above
    tc_fence_before_sync();
    cluster_sync_all();  // both CTAs' barriers exist before either signals the other
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            Sched sc;
            sc.init(p, pair, num_pairs);
            Unit u;
            while (ok && sc.next(p, u)) {
                const int32_t ra = u.ta * kPairBM + static_cast<int32_t>(rank) * kBM;
                // B rows of sub-tile s: u.col0 + s * kSubN + rank * kSubN / 2, kSubN / 2 of them
                const int32_t rb = static_cast<int32_t>(u.col0) + static_cast<int32_t>(rank) * (C::kSubN / 2);
                // a 384-wide unit: its second sub-tile is 128 wide, 64 rows per CTA
                const bool narrow = kWide && u.w < BN;
                const int32_t rb2 = static_cast<int32_t>(u.col0) + C::kSubN + static_cast<int32_t>(rank) * (kNarrowSubN / 2);
                const uint32_t kb_bytes = narrow ? static_cast<uint32_t>(C::kABytes + C::kSubBBytes + C::kSubBBytes / 2)
                                                 : static_cast<uint32_t>(C::kKbBytes);
                for (int kb = u.kb0; kb < u.kb1; kb += KPS) {
                    const int n = (u.kb1 - kb < KPS) ? u.kb1 - kb : KPS;  // k-blocks in this stage
                    if (!mbar_wait_bounded(bar_empty(stage), phase ^ 1u, abort_flag, p.timeout_ns,
                                           kWhereProdEmpty, peer_abort)) {
                        ok = false;
                        break;
                    }
                    if constexpr (kCheckBarriers) {
                        // the full barrier in use: each CTA's own (3xTF32), the leader's (TF32)
                        if ((k3x || rank == 0) && mbar_test_wait(bar_full(stage), phase))
                            record_error(kErrProtocol, kWhereProdEmpty);
                        stage_tag[stage] = work_tag(u.t, kb);
                        fence_acq_rel_cluster();
                    }
                    if constexpr (k3x) {
                        // own barrier: this CTA's split warps wait for these bytes;
                        // x's low parts, when in memory, come with them into the
                        // low half (x is B in the swapped order, A in the direct one)
                        const uint32_t xlo_bytes = p.lo_mem ? static_cast<uint32_t>(SWAP ? C::kBBytes : C::kABytes) : 0u;
                        mbar_arrive_expect_tx(bar_full(stage), n * (C::kKbBytes + xlo_bytes));
                        for (int j = 0; j < n; ++j) {
                            tma_load_2d(sA(stage) + j * C::kABytes, &tmA, bar_full(stage), (kb + j) * kBKW, ra);
#pragma unroll
                            for (int sb = 0; sb < C::kNSub; ++sb)
                                tma_load_2d(sB(stage) + j * C::kBBytes + sb * C::kSubBBytes, &tmB, bar_full(stage),
                                            (kb + j) * kBKW, rb + sb * C::kSubN);
                            if (xlo_bytes) {
                                if constexpr (SWAP)
                                    tma_load_2d(sB(stage) + C::kLoadBytes + j * C::kBBytes, &tmXlo, bar_full(stage),
                                                (kb + j) * kBKW, rb);
                                else
                                    tma_load_2d(sA(stage) + C::kLoadBytes + j * C::kABytes, &tmXlo, bar_full(stage),
                                                (kb + j) * kBKW, ra);
                            }
                        }
                    } else {
                        // the leader expects both CTAs' bytes on its own full barrier
                        if (rank == 0) mbar_arrive_expect_tx(bar_full(stage), 2 * n * kb_bytes);
                        const uint32_t leader_full = mapa_shared(bar_full(stage), 0);
                        for (int j = 0; j < n; ++j) {
                            tma_load_2d_pair(sA(stage) + j * C::kABytes, &tmA, leader_full, (kb + j) * kBKW, ra);
#pragma unroll
                            for (int sb = 0; sb < C::kNSub; ++sb) {
                                if (kWide && sb == 1 && narrow)
                                    tma_load_2d_pair(sB(stage) + j * C::kBBytes + sb * C::kSubBBytes, &tmB2, leader_full,
                                                     (kb + j) * kBKW, rb2);
                                else
                                    tma_load_2d_pair(sB(stage) + j * C::kBBytes + sb * C::kSubBBytes, &tmB, leader_full,
                                                     (kb + j) * kBKW, rb + sb * C::kSubN);
                            }
                        }
                    }
                    ++fills;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
            // This CTA's copies land before its stages are released by the
            // leader's MMA commit; wait for that on the last stages filled.
            for (long long f = (fills > S ? fills - S : 0); f < fills; ++f) {
                const int s = static_cast<int>(f % S);
                const uint32_t ph = static_cast<uint32_t>((f / S) & 1);
                volatile int never = 0;
                mbar_wait_bounded(bar_empty(s), ph, &never, kDrainTimeoutNs, kWhereProdDrain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            Sched sc;
            sc.init(p, pair, num_pairs);
            Unit u;
            while (ok && sc.next(p, u)) {
                const bool narrow = kWide && u.w < BN;
                for (int kc = u.kb0; ok && kc < u.kb1; kc += kChunkKb) {
                    const int kce = (u.kb1 - kc > kChunkKb) ? kc + kChunkKb : u.kb1;
                    if (!mbar_wait_bounded(bar_acce(buf), acc_phase ^ 1u, abort_flag, p.timeout_ns,
                                           kWhereMmaAccEmpty, peer_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    if constexpr (kCheckBarriers) {
                        acc_tag[buf] = work_tag(u.t, kc);
                        fence_acq_rel_cluster();
                    }
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::kAccCols);
                    for (int kb = kc; kb < kce; kb += KPS) {
                        const int n = (kce - kb < KPS) ? kce - kb : KPS;  // k-blocks in this stage
                        const uint32_t wbar = k3x ? bar_split(stage) : bar_full(stage);
                        if (!mbar_wait_bounded(wbar, phase, abort_flag, p.timeout_ns, kWhereMmaFull, peer_abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        if constexpr (kCheckBarriers) {
                            // this CTA's stage and the peer's hold the same work
                            const uint32_t want = work_tag(u.t, kb);
                            check_tag(stage_tag[stage], want, kWhereMmaFull);
                            check_tag(ld_cluster_u32(mapa_shared(smem_u32(const_cast<uint32_t*>(stage_tag + stage)), 1)),
                                      want, kWhereMmaFull);
                        }
                        auto desc = [](uint32_t a) { return smem_desc_sw128(a); };
                        for (int j = 0; j < n; ++j) {
                            const uint64_t a_hi = desc(sA(stage) + j * C::kABytes);
                            const uint64_t b_hi = desc(sB(stage) + j * C::kBBytes);
#pragma unroll
                            for (int k = 0; k < kBKW / kUmmaK; ++k) {
                                // advance 8 fp32 = 32 bytes along K inside the swizzle atom
                                const uint64_t koff = static_cast<uint64_t>(k * 2);
                                const uint32_t acc = (kb > kc || j > 0 || k > 0) ? 1u : 0u;
                                if constexpr (k3x) {
                                    const uint64_t a_lo = desc(sA(stage) + C::kLoadBytes + j * C::kABytes);
                                    const uint64_t b_lo = desc(sB(stage) + C::kLoadBytes + j * C::kBBytes);
                                    mma_tf32_pair(d_tmem, a_lo + koff, b_hi + koff, kIdesc, acc);
                                    mma_tf32_pair(d_tmem, a_hi + koff, b_lo + koff, kIdesc, 1u);
                                    mma_tf32_pair(d_tmem, a_hi + koff, b_hi + koff, kIdesc, 1u);
                                } else {
#pragma unroll
                                    for (int sb = 0; sb < C::kNSub; ++sb)
                                        mma_tf32_pair(d_tmem + static_cast<uint32_t>(sb * C::kSubN), a_hi + koff,
                                                      desc(sB(stage) + j * C::kBBytes + sb * C::kSubBBytes) + koff,
                                                      (kWide && sb == 1 && narrow) ? kIdescNarrow : kIdesc, acc);
                                }
                            }
                        }
                        mma_commit_pair_multicast(bar_empty(stage), 0x3);
                        if (++stage == S) { stage = 0; phase ^= 1u; }
                    }
                    if (!ok) break;
                    mma_commit_pair_multicast(bar_accf(buf), 0x3);
                    if (++buf == C::kNumAcc) {
                        buf = 0;
                        acc_phase ^= 1u;
                    }
                }
            }
            mma_commit_pair(bar_drain);
            volatile int never = 0;
            mbar_wait_bounded(bar_drain, 0, &never, kDrainTimeoutNs, kWhereDrain);
            // Both CTAs' epilogues release each accumulator buffer with an
            // arrival on this CTA's barrier, the peer's from the other SM.
            // The last release of each buffer is never waited for by the loop
            // above; wait for it here, so that no arrival from the peer is
            // still on its way to this CTA's shared memory when it exits (it
            // would land in whichever CTA runs on this SM next).
            for (int i = 0; ok && i < C::kNumAcc; ++i) {
                if (!mbar_wait_bounded(bar_acce(buf), acc_phase ^ 1u, abort_flag, p.timeout_ns, kWhereDrain,
                                       peer_abort))
                    break;
                if (++buf == C::kNumAcc) {
                    buf = 0;
                    acc_phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------ 3xTF32 split (both CTAs)
        if constexpr (k3x) {
            const int ct = threadIdx.x - 64;  // 0..63
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            Sched sc;
            sc.init(p, pair, num_pairs);
            Unit u;
            while (ok && sc.next(p, u)) {
                for (int kb = u.kb0; kb < u.kb1; kb += KPS) {
                    int got = 0;
                    if (lane == 0)
                        got = mbar_wait_bounded(bar_full(stage), phase, abort_flag, p.timeout_ns, kWhereConvFull, peer_abort);
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) { ok = false; break; }
                    if constexpr (kCheckBarriers) {
                        if (lane == 0) check_tag(stage_tag[stage], work_tag(u.t, kb), kWhereConvFull);
                        __syncwarp();
                    }
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
                    // the leader's split warps arrive on their own CTA's barrier
                    // at CTA scope; only the peer's need a cluster-scope release
                    if (lane == 0) {
                        if (rank == 0)
                            mbar_arrive(bar_split(stage));
                        else
                            mbar_arrive_cluster(mapa_shared(bar_split(stage), 0));
                    }
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        // The stream-K counters and (kind (c)) out are set by the prep
        // kernel just before this one, which may still be running.
        griddep_wait();
        // Eight warps: lane quadrant warp % 4, half of the columns each.
        const int q = warp & 3;
        const int half = (warp - 4) >> 2;
        const int r = q * 32 + lane;
        constexpr int kChunks = BN / 32;
        constexpr int kHalf = (kChunks + 1) / 2;  // chunks per half (the most)
        EpiOut eo;
        eo.tmap = p.tma_out ? &tmOut : nullptr;
        eo.stage = reinterpret_cast<float*>(epi_stage + (warp - 4) * kEpiTileBytes);
        eo.stage_u32 = smem_u32(eo.stage);
        int buf = 0;
        uint32_t acc_phase = 0;
        float accr[k3x ? kHalf * 32 : 1];  // 3xTF32: this thread's sums of the K slices
        int fsel = 0;  // next last_flag slot (the same in every epilogue thread)
        Sched sc;
        sc.init(p, pair, num_pairs);
        Unit u;
        bool ok = true;
        while (ok && sc.next(p, u)) {
            // this unit's chunks (a 384-wide unit of a mixed plan has 12),
            // split between the two halves of the epilogue warps
            const int u_chunks = kWide ? u.w / 32 : kChunks;
            const int u_half = kWide ? u_chunks / 2 : kHalf;
            const int c_lo = half * u_half;
            const int64_t cols_left = (SWAP ? p.M : p.N) - u.col0;
            const int nchunks = static_cast<int>(cols_left >= u_chunks * 32 ? u_chunks : (cols_left + 31) / 32);
            const int mine = nchunks - c_lo < 0 ? 0 : (nchunks - c_lo > u_half ? u_half : nchunks - c_lo);
            // This CTA's 128 rows of the pair tile, as a 128-row tile index.
            Unit uh = u;
            uh.ta = 2 * u.ta + static_cast<int>(rank);
            eo.row0 = static_cast<int64_t>(uh.ta) * kBM + q * 32;
            auto wait_acc = [&](int kc) -> bool {
                int got = 0;
                if (lane == 0) {
                    got = mbar_wait_bounded(bar_accf(buf), acc_phase, abort_flag, p.timeout_ns, kWhereEpiAccFull, peer_abort);
                    if constexpr (kCheckBarriers) {
                        // the leader's MMA tagged the buffer it filled
                        if (got)
                            check_tag(ld_cluster_u32(mapa_shared(smem_u32(const_cast<uint32_t*>(acc_tag + buf)), 0)),
                                      work_tag(u.t, kc), kWhereEpiAccFull);
                    }
                }
                (void)kc;
                got = __shfl_sync(0xffffffffu, got, 0);
                if (got) tc_fence_after_sync();
                return got != 0;
            };
            auto release_acc = [&]() {
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(bar_acce(buf), 0));
                __syncwarp();
                if (++buf == C::kNumAcc) {
                    buf = 0;
                    acc_phase ^= 1u;
                }
            };
            auto t_row = [&]() {
                return tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * C::kAccCols);
            };

            uint32_t t_acc = 0;
            if constexpr (k3x) {
#pragma unroll
                for (int j = 0; j < kHalf * 32; ++j) accr[j] = 0.0f;
                for (int kc = u.kb0; kc < u.kb1; kc += kChunkKb) {
                    if (!wait_acc(kc)) { ok = false; break; }
                    const uint32_t tr = t_row();
#pragma unroll
                    for (int lc = 0; lc < kHalf; ++lc) {
                        if (lc >= mine) break;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            float v[16];
                            tmem_ld16_wait(tr + (c_lo + lc) * 32 + h * 16, v);
#pragma unroll
                            for (int j = 0; j < 16; ++j) accr[lc * 32 + h * 16 + j] += v[j];
                        }
                    }
                    release_acc();
                }
                if (!ok) break;
            } else {
                if (!wait_acc(u.kb0)) break;
                t_acc = t_row();
            }

            if (!u.partial) {
                float best = -INFINITY;
                if constexpr (k3x) {
#pragma unroll
                    for (int lc = 0; lc < kHalf; ++lc) {
                        if (lc < mine) {
                            float v[32];
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = accr[lc * 32 + j];
                            epi_chunk<SWAP, BN>(p, uh, r, c_lo + lc, v, best, eo);
                        }
                    }
                } else {
#pragma unroll 1
                    for (int lc = 0; lc < mine; ++lc) {
                        float v[32];
                        tmem_ld32_wait(t_acc + (c_lo + lc) * 32, v);
                        epi_chunk<SWAP, BN>(p, uh, r, c_lo + lc, v, best, eo);
                    }
                }
                epi_finish<SWAP>(p, uh, r, best);
                if constexpr (!k3x) release_acc();
            } else {
                // A unit of a tile split over pairs first .. last: the same
                // wait-free protocol as fle_gemm_kernel, per CTA of the pair
                // (each CTA owns 128 rows of the tile and its own counter).
                const int64_t tsk = u.sk_tile;
                const int first = sk_cta_of(tsk * p.num_kb, p.sk_iters, p.sk_grid);
                const int last = sk_cta_of((tsk + 1) * p.num_kb - 1, p.sk_iters, p.sk_grid);
                const unsigned others = static_cast<unsigned>(last - first);
                unsigned* counter = p.counters + 2 * tsk + rank;
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
                    // park this CTA's partial (column-major: element (row, col)
                    // at col * 128 + row) and count it
                    float* slot = p.ws + static_cast<size_t>(p.sk_slots * blockIdx.x + u.slot) * kBM * BN;
                    if constexpr (k3x) {
#pragma unroll
                        for (int lc = 0; lc < kHalf; ++lc) {
                            if (lc < mine) {
                                float* d = slot + static_cast<size_t>((c_lo + lc) * 32) * kBM + r;
#pragma unroll
                                for (int j = 0; j < 32; ++j) __stcg(d + j * kBM, accr[lc * 32 + j]);
                            }
                        }
                    } else {
#pragma unroll 1
                        for (int lc = 0; lc < mine; ++lc) {
                            float v[32];
                            tmem_ld32_wait(t_acc + (c_lo + lc) * 32, v);
                            float* d = slot + static_cast<size_t>((c_lo + lc) * 32) * kBM + r;
#pragma unroll
                            for (int j = 0; j < 32; ++j) __stcg(d + j * kBM, v[j]);
                        }
                        release_acc();
                    }
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
                        return p.ws + static_cast<size_t>(p.sk_slots * (2 * cc + rank) + sl) * kBM * BN +
                               static_cast<size_t>(c * 32) * kBM + r;
                    };
                    // contributors from..last added in order; loads of up to
                    // three contributors are in flight together
                    auto add_partials = [&](int c, int from, float (&v)[32]) {
                        int cc = from;
                        for (; cc + 2 <= last; cc += 3) {
                            const float* s0 = src_of(cc, c);
                            const float* s1 = src_of(cc + 1, c);
                            const float* s2 = src_of(cc + 2, c);
                            float t0[32], t1[32], t2[32];
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                t0[j] = __ldcg(s0 + j * kBM);
                                t1[j] = __ldcg(s1 + j * kBM);
                                t2[j] = __ldcg(s2 + j * kBM);
                            }
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = ((v[j] + t0[j]) + t1[j]) + t2[j];
                        }
                        for (; cc <= last; ++cc) {
                            const float* s0 = src_of(cc, c);
                            float t0[32];
#pragma unroll
                            for (int j = 0; j < 32; ++j) t0[j] = __ldcg(s0 + j * kBM);
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] += t0[j];
                        }
                    };
                    const int from = own ? first + 1 : first;
                    if constexpr (k3x) {
#pragma unroll
                        for (int lc = 0; lc < kHalf; ++lc) {
                            if (lc < mine) {
                                float v[32];
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = own ? accr[lc * 32 + j] : 0.0f;
                                add_partials(c_lo + lc, from, v);
                                epi_chunk<SWAP, BN>(p, uh, r, c_lo + lc, v, best, eo);
                            }
                        }
                    } else {
#pragma unroll 1
                        for (int lc = 0; lc < mine; ++lc) {
                            float v[32];
                            if (own) {
                                tmem_ld32_wait(t_acc + (c_lo + lc) * 32, v);
                            } else {
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = 0.0f;
                            }
                            add_partials(c_lo + lc, from, v);
                            epi_chunk<SWAP, BN>(p, uh, r, c_lo + lc, v, best, eo);
                        }
                    }
                    epi_finish<SWAP>(p, uh, r, best);
                    if (threadIdx.x == 128) {
                        *counter = 0u;
                        atomicAdd(&g_finish_count[own ? 0 : 1], 1u);
                    }
                    __syncwarp();
                }
                if constexpr (!k3x) {
                    if (own) release_acc();
                }
            }
        }
    }

    // Roles branch on the lane (one issuing thread per warp); reconverge every
    // warp before the CTA barriers, which whole warps must reach together.
    __syncwarp();
    // Epilogue TMA stores read the staging tiles until they complete.
    if (warp >= 4 && lane == 0) bulk_wait_all();
    __syncwarp();
    // Neither CTA may release TMEM or exit while the other can still signal
    // its barriers or (leader) write its TMEM: a bounded two-way handshake.
    // The other CTA arrives within one progress limit (a stalled role gives
    // up, or sees the abort this CTA raised) plus its drains.
    tc_fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_cluster(mapa_shared(bar_exit, rank ^ 1u));
        volatile int never = 0;
        mbar_wait_bounded(bar_exit, 0, &never, p.timeout_ns + 2 * kDrainTimeoutNs, kWhereDrain);
        // the wait acquires at CTA scope; the other CTA released at cluster
        // scope: order this CTA's teardown after everything it did before
        fence_acq_rel_cluster();
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

}  // namespace fle
