// gemm_pair_tc.cuh -- fused NF4-dequantise + GEMM on CTA pairs
// (tcgen05.mma.cta_group::2: one 256 x BN MMA spans the two CTAs of a cluster).
//
// It computes, in two directions of the QLoRA layer,
//   forward: D = x W~^T + bf16((alpha/r) x A^T) B^T
//   dgrad:   D = dY W~  + bf16((alpha/r) dY B) A
// ("QLoRA explained", section "The LoRA adapter path", and the chain rule
// through the frozen dequantised weight). The 4-bit codes stream into shared
// memory through TMA and are dequantised in registers (a per-block lookup of
// the 16 scaled levels) straight into the tensor core's 128-byte-swizzled
// operand layout: K-major for the forward, MN-major for dgrad. The LoRA term
// is ceil(r/64) extra reduction stages of the same accumulator (r
// zero-padded to 64). Each output tile is 256 tokens x BN columns computed by
// a pair of CTAs on two SMs:
//   CTA v of the pair loads tokens [128v, 128v+128) of the tile (A operand),
//   dequantises only half of the weight tile -- columns [v BN/2, v BN/2 + BN/2)
//   of the MMA's B operand -- into its own shared memory, and keeps rows
//   [128v, 128v+128) of the fp32 accumulator in its own tensor memory.
// The tensor core of the even CTA reads both halves of A and B directly, so
// every dequantised element is produced once per 256 tokens instead of once
// per 128, and each SM writes and the tensor core reads only half of the
// weight tile: the dequantisation ALU work and the shared-memory traffic per
// SM are both halved relative to a one-CTA tile of the same width.
//
// Synchronisation across the pair:
//   a_full  (even CTA)   both CTAs' activation loads credit their bytes here
//   b_full  (even CTA)   the dequant warps of both CTAs arrive here; the even
//                        CTA's warps arrive only once the stage's a_full phase
//                        has completed, so the MMA issuer waits on b_full alone
//                        (one barrier probe per stage on its critical path)
//   acc_empty (even CTA) the epilogue warps of both CTAs arrive here
//   consumed, acc_full (both CTAs)  one multicast tcgen05.commit; consumed[u mod
//                        kConsumedBars] completes when the MMAs of stage u have, and
//                        frees that stage's activation slot and weight slot alike:
//                        one commit per stage on the MMA issuer's critical path
// The code-tile ring is private to each CTA.
//
// Warp roles per CTA: 0..3 epilogue, 4 TMA activations, 5 TMEM owner and (even
// CTA) MMA issuer, 6 TMA codes, 7.. dequantisation (G groups of BN/2 threads
// taking every G-th stage).
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kBM = 128;            // tokens per CTA of a pair tile (MMA M = 2 kBM)
constexpr int kBK = 64;             // reduction per stage = one 64-element NF4 step
constexpr int kConsumedBars = 16;   // ring of stage-consumed barriers (a power of two)
constexpr int kEpiWarp0 = 0;
constexpr int kTmaAWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kTmaCWarp = 6;
constexpr int kDequantWarp0 = 7;

struct GemmArgs {
    int M;              // tokens
    int red;            // reduction length (forward: K, dgrad: N)
    int out;            // output columns   (forward: N, dgrad: K)
    int main_steps;     // ceil(red / 64)
    int lora_steps;     // ceil(r / 64)
    int m_tiles, n_tiles;
    int r;
    // quantised weight (always the [N, K] weight)
    int64_t Nw;         // rows of W
    int64_t Kw;         // columns of W
    int64_t kblocks;    // K / 64 (64-element steps per W row)
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    const uint16_t *lora_b;   // forward: B [N, r]; dgrad: A [r, K]
    uint16_t *D;        // [M, out] bf16
    // stream-K schedule: 0 = whole tiles round-robin
    int sk;
    float *partial;     // [pairs][2][BN/32][128][32] fp32 partial tiles
    int *flags;         // [pairs][2][4 epilogue warps], zero at launch; 1 = rows written
    float *D32;         // when non-null: the fp32 result goes here instead of D
    int bshift;         // log2(block size / 64): block of step j is j >> bshift
};


template <int BN, bool DGRAD, int G>
struct PairCfg {
    static constexpr int kBH = BN / 2;                    // B columns held by one CTA
    static constexpr int kABytes = kBM * kBK * 2;         // 16 KB
    static constexpr int kBBytes = kBH * kBK * 2;         // this CTA's half of the B tile
    static constexpr int kCBytes = kBH * kBK / 2;         // its 4-bit codes
    static constexpr int kSB = G >= 4 ? G : 2 * G;       // weight-tile stages
    static constexpr int kSC = G >= 4 ? G : 2 * G;       // code-tile stages
    static constexpr int kSAFit = (220 * 1024 - kSB * kBBytes - kSC * kCBytes) / kABytes;
    static constexpr int kSA = kSAFit > 8 ? 8 : kSAFit;
    static constexpr int kGroupWarps = kBH / 32;
    static constexpr int kThreads = 32 * (kDequantWarp0 + G * kGroupWarps);
    static constexpr int kTmemCols = (2 * BN <= 256) ? 256 : 512;
    static constexpr int kSmemBytes =
        kSA * kABytes + kSB * kBBytes + kSC * kCBytes + 1024 /*align*/ + 512 /*barriers*/;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(2 * kBM, BN, 0, DGRAD ? 1 : 0);
    static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "pair MMA N");
    static_assert(kBH % 32 == 0, "whole dequant warps");
    static_assert(!DGRAD || kBH % 64 == 0, "MN-major halves are whole 64-column swizzle atoms");
    static_assert(kBBytes % 1024 == 0 && kCBytes % 1024 == 0, "stage alignment");
    static_assert(kSC % G == 0 && kSB % G == 0, "each dequant group owns every G-th slot");
    static_assert(kSA >= 3, "pipeline depth");
    // The even CTA's dequant warps wait on a_full of stage u while the MMA may
    // still hold stage u - kSB; with kSA >= kSB the phase of stage u - kSA has
    // completed by then, so the parity they wait on names stage u alone.
    static_assert(kSA >= kSB, "activation ring at least as deep as the weight ring");
    // A producer of stage u waits on consumed[(u - S) mod R] (S = kSA or kSB):
    // that barrier's next phase needs stage u - S + R consumed, which needs
    // stage u itself when R > S, and its previous phase (stage u - S - R) was
    // waited for already when R >= G (the dequant group's previous stage).
    static_assert(kConsumedBars > kSA && kConsumedBars > kSB && kConsumedBars >= G,
                  "stage-consumed ring deeper than either operand ring");
    // barriers, then the TMEM address, the abort flag and three progress counters
    static_assert((kSA + kConsumedBars + 2 * kSC + kSB + 2 + 2 + 1) * 8 + 4 + 4 + 12 <= 512,
                  "barrier area");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// The work of one pair: segments of stages [k0, k1) of a tile.
//   Whole-tile schedule (sk = 0): tiles p, p + P, p + 2P, ... with every stage.
//   Data-parallel waves + stream-K (sk = 1): the first (floor(T / P) - 1) P
//   tiles go round-robin (pair p takes tiles p, p + P, ...) with every stage;
//   the units (tile, stage) of the remaining P + (T mod P) tiles, numbered
//   tile-major, are cut into P contiguous runs [W p / P, W (p + 1) / P) with
//   W = (P + T mod P) S. Every run spans at least one tile, so a tile there is
//   split between at most two consecutive pairs: its head (stages [0, k)) is
//   the last segment of pair p and its tail (stages [k, S)) the first segment
//   of pair p + 1. The round-robin waves keep the tiles in flight at one time
//   consecutive in the raster order below (operands shared in L2), and the
//   stream-K tail keeps the last wave from leaving pairs idle.
struct PairSeg {
    int tile, k0, k1;
};

struct PairSched {
    int S, T, P, p, sk;
    int n_dp;          // tiles of the round-robin waves
    int dp_count;      // this pair's round-robin tiles
    int64_t u0, u1;    // this pair's stream-K units, as tile * S + stage

    __device__ __forceinline__ void init(int S_, int T_, int P_, int p_, int sk_) {
        S = S_; T = T_; P = P_; p = p_; sk = sk_;
        if (!sk) {
            n_dp = T;
            u0 = u1 = 0;
        } else {
            n_dp = (T / P - 1) * P;
            const int64_t W = static_cast<int64_t>(T - n_dp) * S;
            const int64_t base = static_cast<int64_t>(n_dp) * S;
            u0 = base + (W * p) / P;
            u1 = base + (W * (p + 1)) / P;
        }
        dp_count = p < n_dp ? (n_dp - p + P - 1) / P : 0;
    }
    // units of this pair, in schedule order
    __device__ __forceinline__ int units() const {
        return dp_count * S + static_cast<int>(u1 - u0);
    }
    // the i-th unit of this pair (0 <= i < units())
    __device__ __forceinline__ void unit(int i, int &tile, int &it) const {
        if (i < dp_count * S) {
            const int j = i / S;
            tile = p + j * P;
            it = i - j * S;
        } else {
            const int64_t u = u0 + (i - dp_count * S);
            tile = static_cast<int>(u / S);
            it = static_cast<int>(u - static_cast<int64_t>(tile) * S);
        }
    }
    __device__ __forceinline__ bool sk_first(PairSeg &g) const {
        if (u0 >= u1) return false;
        const int t = static_cast<int>(u0 / S);
        const int k0 = static_cast<int>(u0 - static_cast<int64_t>(t) * S);
        const int64_t rest = u1 - static_cast<int64_t>(t) * S;
        g = {t, k0, rest < S ? static_cast<int>(rest) : S};
        return true;
    }
    __device__ __forceinline__ bool first(PairSeg &g) const {
        if (dp_count > 0) {
            g = {p, 0, S};
            return true;
        }
        return sk_first(g);
    }
    __device__ __forceinline__ bool next(PairSeg &g) const {
        if (g.tile < n_dp) {
            if (g.tile + P < n_dp) {
                g = {g.tile + P, 0, S};
                return true;
            }
            return sk_first(g);
        }
        const int t = g.tile + 1;
        const int64_t rest = u1 - static_cast<int64_t>(t) * S;
        if (g.k1 < S || rest <= 0) return false;
        g = {t, 0, rest < S ? static_cast<int>(rest) : S};
        return true;
    }
};

// Raster order of the output tiles (256 tokens x BN columns): groups of
// kRasterGroup token tiles, within a group column tile by column tile with
// the token tiles fastest. The tiles of one wave (the pairs' current tiles,
// consecutive in this order) then read about kRasterGroup activation slices
// and P / kRasterGroup weight column tiles, a working set that stays in L2.
constexpr int kRasterGroup = 4;

__device__ __forceinline__ void tile_coords(int tile, int m_pairs, int n_tiles, int &mi, int &ni) {
    const int per_group = kRasterGroup * n_tiles;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int gm = min(kRasterGroup, m_pairs - g * kRasterGroup);   // token tiles in this group
    ni = r / gm;
    mi = g * kRasterGroup + (r - ni * gm);
}

// Bounded wait until a flag in global memory becomes non-zero (acquire, GPU
// scope). It returns false if the CTA is giving up, or when the wait runs out
// of time: then NF4_ERR_TIMEOUT is recorded in the device status and the
// caller finishes its tile without what the flag guards (a wait on global
// memory has no copy in flight, so nothing needs to unwind). The cycle limit
// is the pipeline's unless a test has set g_dbg_flag_wait_limit.
__device__ __forceinline__ bool wait_flag_gpu(const int *flag, volatile int *abort_flag) {
    const long long t0 = clock64();
    const long long lim = g_dbg_flag_wait_limit > 0 ? g_dbg_flag_wait_limit : kWaitLimitCycles;
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v != 0) return true;
        if (abort_raised(abort_flag)) return false;
        if (clock64() - t0 > lim) {
            record_status(NF4_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void set_flag_gpu(int *flag) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}

// OUT32: the result is written in fp32 to args.D32 (for a later kernel that
// adds to it and rounds once) instead of bf16 to args.D.
template <int BN, bool DGRAD, int G, bool OUT32>
__global__ void __launch_bounds__(PairCfg<BN, DGRAD, G>::kThreads, 1)
qlora_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_act,    // [M, red] bf16, box {64,128}
                       const __grid_constant__ CUtensorMap tm_codes,  // [Nw, K/2] u8, box {32, rows}
                       const __grid_constant__ CUtensorMap tm_la,     // [M, r] bf16, box {64,128}
                       const GemmArgs args) {
    using Cfg = PairCfg<BN, DGRAD, G>;
    constexpr int SA = Cfg::kSA, SB = Cfg::kSB, SC = Cfg::kSC, BH = Cfg::kBH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *slot_a = smem;                              // [SA][kABytes]
    uint8_t *slot_b = slot_a + SA * Cfg::kABytes;        // [SB][kBBytes]
    uint8_t *slot_c = slot_b + SB * Cfg::kBBytes;        // [SC][kCBytes]
    uint64_t *bars = reinterpret_cast<uint64_t *>(slot_c + SC * Cfg::kCBytes);
    uint64_t *a_full = bars;                 // even CTA: both loads landed (1 + tx)
    uint64_t *consumed = a_full + SA;        // [kConsumedBars] MMAs of a stage done (pair commit)
    uint64_t *c_full = consumed + kConsumedBars;   // code TMA landed (1 + tx) or LoRA stage (1)
    uint64_t *c_empty = c_full + SC;         // codes read (one dequant group of this CTA)
    uint64_t *b_full = c_empty + SC;         // even CTA: halves written (groups of both CTAs)
    uint64_t *acc_full = b_full + SB;        // [2] accumulator complete (pair commit)
    uint64_t *acc_empty = acc_full + 2;      // [2] even CTA: drained (epilogue warps of both)
    uint64_t *mma_drain = acc_empty + 2;     // even CTA: the MMAs issued before giving up completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // even CTA, read only after giving up: activation stages issued by each
    // CTA's producer, and stages the MMA issuer consumed
    volatile int *progress = reinterpret_cast<volatile int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();             // 0 or 1 within the pair
    const int pair = static_cast<int>(cluster_id_x());
    const int npairs = static_cast<int>(cluster_count_x());

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) mbar_init(&a_full[s], 1);
        for (int s = 0; s < kConsumedBars; ++s) mbar_init(&consumed[s], 1);
        for (int s = 0; s < SC; ++s) {
            mbar_init(&c_full[s], 1);
            mbar_init(&c_empty[s], Cfg::kGroupWarps);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(&b_full[s], 2 * Cfg::kGroupWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_la);
    }
    if (warp == kMmaWarp) {
        tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();            // barriers of both CTAs initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // This grid is launched only after the kernel before it (the rank-r
    // product of the same call) has passed its own wait on everything earlier
    // in the stream, so the activations, codes, scales and adapters are final
    // now. Only what that kernel writes -- the bf16 rank-r activations read by
    // the last (LoRA) stage and the zeroed stream-K flags -- is waited for,
    // by the roles that read it, so the main loop starts while it finishes.
    griddep_launch_dependents();

    const int m_pairs = (args.M + 2 * kBM - 1) / (2 * kBM);
    const int total_tiles = m_pairs * args.n_tiles;
    const int nsteps = args.main_steps + args.lora_steps;
    PairSched sched;
    sched.init(nsteps, total_tiles, npairs, pair, args.sk);
    PairSeg sg;
    // progress of the producers and of the MMA issuer (read after giving up)
    int na = 0, nc = 0, cm = 0;

    if (warp == kTmaAWarp) {
        // ------------------------------------------------ TMA: activations
        if (lane == 0) {
            const uint32_t full0 = mapa_shared(smem_u32(a_full), 0);
            int sa = 0;
            bool la_ready = false;     // the rank-r activations are written by the kernel before
            for (bool more = sched.first(sg); more; more = sched.next(sg)) {
                int mi, ni;
                tile_coords(sg.tile, m_pairs, args.n_tiles, mi, ni);
                const int m0 = mi * (2 * kBM) + static_cast<int>(rank) * kBM;
                for (int it = sg.k0; it < sg.k1; ++it) {
                    if (na >= SA) {               // the slot's previous stage, na - SA, consumed
                        const int v = na - SA;
                        if (!mbar_wait(&consumed[v & (kConsumedBars - 1)],
                                       static_cast<uint32_t>(v / kConsumedBars) & 1u, abort_flag))
                            goto done;
                    }
                    if (it >= args.main_steps && !la_ready) {
                        griddep_wait();
                        la_ready = true;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&a_full[sa], 2 * Cfg::kABytes);
                    if (it < args.main_steps)
                        tma_load_2d_pair(slot_a + sa * Cfg::kABytes, &tm_act, full0 + 8u * sa,
                                         it * kBK, m0);
                    else
                        tma_load_2d_pair(slot_a + sa * Cfg::kABytes, &tm_la, full0 + 8u * sa,
                                         (it - args.main_steps) * kBK, m0);
                    ++na;
                    if (++sa == SA) sa = 0;
                }
            }
        }
    } else if (warp == kTmaCWarp) {
        // ------------------------------------------------ TMA: 4-bit codes
        if (lane == 0) {
            int sc = 0;
            uint32_t pc = 0;
            for (bool more = sched.first(sg); more; more = sched.next(sg)) {
                int mi, ni;
                tile_coords(sg.tile, m_pairs, args.n_tiles, mi, ni);
                const int nh = ni * BN + static_cast<int>(rank) * BH;
                for (int it = sg.k0; it < sg.k1; ++it) {
                    if (!mbar_wait(&c_empty[sc], pc ^ 1, abort_flag)) goto done;
                    uint8_t *c = slot_c + sc * Cfg::kCBytes;
                    if (it < args.main_steps) {
                        mbar_arrive_expect_tx(&c_full[sc], Cfg::kCBytes);
                        if (!DGRAD) {
                            tma_load_2d(c, &tm_codes, &c_full[sc], it * (kBK / 2), nh);
                        } else {
#pragma unroll
                            for (int kb = 0; kb < BH / 64; ++kb)
                                tma_load_2d(c + kb * 2048, &tm_codes, &c_full[sc], nh / 2 + kb * 32,
                                            it * kBK);
                        }
                    } else {
                        mbar_arrive(&c_full[sc]);      // LoRA stage: no codes
                    }
                    ++nc;
                    if (++sc == SC) { sc = 0; pc ^= 1; }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        // The whole warp walks the schedule and waits; the elected lane
        // issues every MMA and commit (so its commits track all of them).
        if (rank == 0) {
            int sa = 0, sb = 0, ab = 0;
            uint32_t pb = 0, aph = 0;
            const uint32_t a_base = smem_u32(slot_a), b_base = smem_u32(slot_b);
            for (bool more = sched.first(sg); more; more = sched.next(sg)) {
                if (!mbar_wait_warp(&acc_empty[ab], aph ^ 1, abort_flag)) goto done;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + ab * BN;
                for (int it = sg.k0; it < sg.k1; ++it) {
                    // b_full implies a_full (see the dequant role)
                    if (!mbar_wait_warp(&b_full[sb], pb, abort_flag)) goto done;
                    tc_fence_after();
                    const uint32_t a_addr = a_base + sa * Cfg::kABytes;
                    const uint32_t b_addr = b_base + sb * Cfg::kBBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bd = DGRAD ? smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                                  : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
                        umma_bf16_ss_pair_warp(d_tmem, ad, bd, Cfg::kIdesc,
                                               (it > sg.k0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit_pair_warp(&consumed[cm & (kConsumedBars - 1)], 0x3);
                    ++cm;
                    if (++sa == SA) sa = 0;
                    if (++sb == SB) { sb = 0; pb ^= 1; }
                }
                umma_commit_pair_warp(&acc_full[ab], 0x3);
                if (++ab == 2) { ab = 0; aph ^= 1; }
            }
        }
    } else if (warp < kEpiWarp0 + 4) {
        // ------------------------------------------------------- epilogue
        // Per segment: a whole tile is rounded to bf16 and stored; the tail
        // of a split tile is stored as an fp32 partial (layout [BN/32][128
        // rows][32], 128-byte rows per thread) and its flag set; the head of
        // a split tile waits for the flag of the next pair's partial, adds it
        // and stores the sum. Flags are per epilogue warp: warp q of the head
        // reads exactly the rows warp q of the tail wrote.
        const int q = warp - kEpiWarp0;                   // TMEM lane quadrant (== warp % 4)
        const uint32_t empty0 = mapa_shared(smem_u32(acc_empty), 0);
        griddep_wait();            // the stream-K flags are zeroed by the kernel before
        constexpr int kChunks = BN / 32;
        int ab = 0;
        uint32_t aph = 0;
        for (bool more = sched.first(sg); more; more = sched.next(sg)) {
            int mi, ni;
            tile_coords(sg.tile, m_pairs, args.n_tiles, mi, ni);
            const int m0 = mi * (2 * kBM) + static_cast<int>(rank) * kBM;
            const int n0 = ni * BN;
            const bool tail = sg.k0 > 0;
            const bool head = !tail && sg.k1 < nsteps;
            const int rloc = q * 32 + lane;               // row within this CTA's 128
            if (!mbar_wait(&acc_full[ab], aph, abort_flag)) goto done;
            tc_fence_after();
            if (tail) {
                float *pp = args.partial +
                            (static_cast<int64_t>(pair) * 2 + rank) * kChunks * (128 * 32) + rloc * 32;
#pragma unroll 1
                for (int c2 = 0; c2 < 2 * kChunks; ++c2) {      // 16 columns at a time
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(tmem_base + ((q * 32) << 16) + ab * BN + c2 * 16, v);
                    tmem_ld_wait();
                    float *dst = pp + (c2 >> 1) * (128 * 32) + (c2 & 1) * 16;
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(dst + e) =
                            make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                        __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                }
                tc_fence_before();
                __syncwarp();                 // this warp's 32 rows of the partial are written
                if (lane == 0) {
                    mbar_arrive_remote(empty0 + 8u * ab);
                    __threadfence();
                    if (!g_dbg_skip_flag_set) set_flag_gpu(args.flags + (pair * 2 + rank) * 4 + q);
                }
            } else {
                const float *pp = nullptr;
                bool add_partial = false;
                if (head) {
                    // rows rloc of the partial were written by warp q of the
                    // same-rank CTA of the next pair
                    const int src = (pair + 1) * 2 + static_cast<int>(rank);
                    add_partial = wait_flag_gpu(args.flags + src * 4 + q, abort_flag);
                    if (*abort_flag) goto done;
                    pp = args.partial + static_cast<int64_t>(src) * kChunks * (128 * 32) + rloc * 32;
                }
                const int row = m0 + rloc;
                uint16_t *drow = args.D + static_cast<int64_t>(row) * args.out;
#pragma unroll 1
                for (int c2 = 0; c2 < 2 * kChunks; ++c2) {      // 16 columns at a time
                    const int c = c2 >> 1;
                    // the partial's 16 values are requested before the tensor-memory
                    // load and its wait, so that the two latencies overlap
                    float4 pv4[4] = {};
                    if (add_partial) {
                        const float4 *pv = reinterpret_cast<const float4 *>(pp + c * (128 * 32) + (c2 & 1) * 16);
#pragma unroll
                        for (int i = 0; i < 4; ++i) pv4[i] = pv[i];
                    }
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(tmem_base + ((q * 32) << 16) + ab * BN + c2 * 16, v);
                    tmem_ld_wait();
                    if (row < args.M) {
#pragma unroll
                        for (int gg = 0; gg < 2; ++gg) {
                            const int g = 2 * (c2 & 1) + gg;       // 8-column group of the 32-column chunk
                            const int col = n0 + c * 32 + g * 8;
                            if (col < args.out) {
                                float f[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[gg * 8 + e]);
                                if (add_partial) {
                                    const float4 p0 = pv4[2 * gg], p1 = pv4[2 * gg + 1];
                                    f[0] += p0.x; f[1] += p0.y; f[2] += p0.z; f[3] += p0.w;
                                    f[4] += p1.x; f[5] += p1.y; f[6] += p1.z; f[7] += p1.w;
                                }
                                if constexpr (OUT32) {
                                    // fp32 result (a later kernel adds to it and rounds once)
                                    float4 *f4 = reinterpret_cast<float4 *>(args.D32 + static_cast<int64_t>(row) * args.out + col);
                                    f4[0] = make_float4(f[0], f[1], f[2], f[3]);
                                    f4[1] = make_float4(f[4], f[5], f[6], f[7]);
                                    continue;
                                }
                                uint32_t p[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
                                    p[e] = *reinterpret_cast<uint32_t *>(&h2);
                                }
                                *reinterpret_cast<uint4 *>(drow + col) =
                                    make_uint4(p[0], p[1], p[2], p[3]);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(empty0 + 8u * ab);
            }
            if (++ab == 2) { ab = 0; aph ^= 1; }
        }
    } else {
        // -------------------------------------------------- dequantisation
        // G groups of BH threads; group g takes the stages whose global index
        // is g mod G. Thread i of a group owns one work item per stage:
        //   forward: W row nh + i, block `it`
        //   dgrad:   W row 64 it + r_loc, block nh/64 + kb
        // where nh is the first B column this CTA holds. Eight consecutive
        // lanes take eight consecutive rows of one 8-row swizzle atom, so each
        // 8-lane phase of a 16-byte shared access hits distinct banks.
        const int t = threadIdx.x - kDequantWarp0 * 32;
        const int grp = t / BH;
        const int i = t % BH;
        constexpr int kBPR = BH / 64;
        const int kb = DGRAD ? (i / 8) % kBPR : 0;
        const int r_loc = DGRAD ? (i / (8 * kBPR)) * 8 + (i & 7) : i;
        const uint32_t row_off = DGRAD ? static_cast<uint32_t>(kb * 8192 + r_loc * 128)
                                       : static_cast<uint32_t>(i * 128);
        // code tiles carry the 32-byte TMA swizzle: 16-byte chunk hh of row j
        // sits at chunk hh ^ ((j >> 2) & 1)
        const uint32_t code_off = DGRAD ? static_cast<uint32_t>(kb * 2048 + r_loc * 32)
                                        : static_cast<uint32_t>(i * 32);
        const uint32_t cswz = static_cast<uint32_t>((r_loc >> 2) & 1);
        const uint32_t swz = static_cast<uint32_t>(r_loc & 7);
        const uint32_t full0 = mapa_shared(smem_u32(b_full), 0);

        // a position in this group's walk over the pair's (tile, stage) units,
        // in the order of the schedule's segments
        struct Pos {
            int tile, it;
            int64_t item;      // W row (forward) or W block column (dgrad); -1 outside W
        };
        auto item_of = [&](int tile) -> int64_t {
            int mi, ni;
            tile_coords(tile, m_pairs, args.n_tiles, mi, ni);
            const int64_t nh = static_cast<int64_t>(ni) * BN + rank * BH;
            if (!DGRAD) return nh + i < args.Nw ? nh + i : -1;
            return nh / 64 + kb < args.kblocks ? nh / 64 + kb : -1;
        };
        const int nunits = sched.units();
        const int dp_units = sched.dp_count * nsteps;
        // move from unit u to unit u + G (u + G < nunits): within the round-robin
        // tiles or within the stream-K run by stepping, across the boundary
        // between them by the schedule's unit()
        auto advance = [&](Pos &p, int u) {
            const int un = u + G;
            if (u < dp_units && un >= dp_units) {
                sched.unit(un, p.tile, p.it);
                p.item = item_of(p.tile);
                return;
            }
            const int tstep = un < dp_units ? npairs : 1;
            p.it += G;
            bool moved = false;
            while (p.it >= nsteps) {
                p.it -= nsteps;
                p.tile += tstep;
                moved = true;
            }
            if (moved) p.item = item_of(p.tile);
        };
        auto block_of = [&](const Pos &p) -> int64_t {
            if (p.tile >= total_tiles || p.it >= args.main_steps || p.item < 0) return -1;
            const int64_t bpr = args.kblocks >> args.bshift;      // blocks per W row
            if (!DGRAD) return p.item * bpr + (p.it >> args.bshift);
            const int64_t wrow = static_cast<int64_t>(p.it) * kBK + r_loc;
            return wrow < args.Nw ? wrow * bpr + (p.item >> args.bshift) : -1;
        };
        // raw scale of a block: q8 and c_g under double quantisation, else absmax
        struct RawScale { int64_t b; uint32_t q8; float v; };
        auto load_scale = [&](int64_t b) -> RawScale {
            RawScale rs{b, 0u, 0.0f};
            if (b < 0) return rs;
            if (args.dq) {
                rs.q8 = __ldg(args.q8 + b);
                rs.v = __ldg(args.cg + (b >> 8));
            } else {
                rs.v = __ldg(args.absmax + b);
            }
            return rs;
        };

        int u = grp;
        Pos cur{0, 0, -1};
        if (u < nunits) {
            sched.unit(u, cur.tile, cur.it);
            cur.item = item_of(cur.tile);
        }
        // The scale of the next item is loaded after this item's last fence,
        // so that no load is outstanding across a proxy fence.
        RawScale cs = load_scale(u < nunits ? block_of(cur) : -1);
        int sb = grp, sc = grp;
        uint32_t pc = 0;
        while (u < nunits) {
            const bool main = cur.it < args.main_steps;

            if (!mbar_wait(&c_full[sc], pc, abort_flag)) goto done;
            // this item's 64 codes go to registers, which frees the code slot
            uint4 h0 = make_uint4(0, 0, 0, 0), h1 = h0;
            float s = 0.0f;          // blocks outside W get scale 0: every level maps to +-0
            if (main) {
                const uint8_t *cp = slot_c + sc * Cfg::kCBytes + code_off;
                h0 = *reinterpret_cast<const uint4 *>(cp + 16 * cswz);
                h1 = *reinterpret_cast<const uint4 *>(cp + 16 * (cswz ^ 1));
                if (cs.b >= 0)
                    s = args.dq ? __fmul_rn(static_cast<float>(cs.q8), __fdiv_rn(cs.v, 127.0f))
                                : cs.v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&c_empty[sc]);

            // Each 8-code word becomes one 16-byte piece of the row and is stored
            // at once, so at most one piece is live in registers (no spills at
            // the 72 registers a thread has).
            if (u >= SB) {                    // the slot's previous stage, u - SB, consumed
                const int v = u - SB;
                if (!mbar_wait(&consumed[v & (kConsumedBars - 1)],
                               static_cast<uint32_t>(v / kConsumedBars) & 1u, abort_flag))
                    goto done;
            }
            uint8_t *brow = slot_b + sb * Cfg::kBBytes + row_off;
            auto put = [&](int c, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
                *reinterpret_cast<uint4 *>(brow + ((c ^ swz) << 4)) = make_uint4(w0, w1, w2, w3);
            };
            if (main) {
                const BlockLut L = make_block_lut(s);
                const uint32_t words[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                for (int wd = 0; wd < 8; ++wd) {
                    uint32_t o[4];
                    dequant8(L, words[wd], o);
                    put(wd, o[0], o[1], o[2], o[3]);
                }
            } else {
                // LoRA stage: the adapter tile comes straight from global memory
                //   forward: B[nh + i][64 ls .. +64)           (zero beyond r, N)
                //   dgrad:   A[64 ls + r_loc][64 item .. +64)  (zero beyond r, K)
                const int ls = cur.it - args.main_steps;
                const uint16_t *src = nullptr;
                int nvalid = 0;   // valid 8-element chunks
                if (cur.item >= 0) {
                    if (!DGRAD) {
                        const int j0 = 64 * ls;
                        if (j0 < args.r) {
                            src = args.lora_b + cur.item * args.r + j0;
                            nvalid = (args.r - j0) / 8 >= 8 ? 8 : (args.r - j0) / 8;
                        }
                    } else {
                        const int j = 64 * ls + r_loc;
                        const int64_t k0 = cur.item * 64;
                        if (j < args.r) {
                            src = args.lora_b + static_cast<int64_t>(j) * args.Kw + k0;
                            nvalid = (args.Kw - k0) / 8 >= 8 ? 8 : static_cast<int>((args.Kw - k0) / 8);
                        }
                    }
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (c < nvalid) v = __ldg(reinterpret_cast<const uint4 *>(src) + c);
                    put(c, v.x, v.y, v.z, v.w);
                }
            }
            // the even CTA vouches for the activation tile of this stage too
            if (rank == 0 &&
                !mbar_wait(&a_full[u % SA], static_cast<uint32_t>(u / SA) & 1u, abort_flag))
                goto done;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(full0 + 8u * sb);

            sb += G;
            if (sb >= SB) sb -= SB;
            sc += G;
            if (sc >= SC) { sc -= SC; pc ^= 1; }
            if (u + G < nunits) {
                advance(cur, u);
                cs = load_scale(block_of(cur));
            }
            u += G;
        }
    }
done:
    // ---- giving up: leave no copy or MMA in flight. A role that gave up has
    // raised this CTA's abort flag; pass it to the other CTA of the pair, whose
    // roles then leave their waits too.
    if (*abort_flag && lane == 0) {
        const uint32_t peer = mapa_shared(smem_u32(const_cast<int *>(abort_flag)), rank ^ 1u);
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
    }
    if (warp == kMmaWarp && rank == 0) {
        // the warp left its loop together (its waits vote), so it is converged
        // and elect.sync picks the lane that issued the MMAs
        __syncwarp();
        if (__any_sync(0xffffffffu, *abort_flag != 0)) {
            // the MMAs already issued complete before the operands are released
            umma_commit_pair_warp(mma_drain, 0x1);
            if (lane == 0) mbar_drain(mma_drain, 0);
        }
        if (lane == 0) progress[2] = cm;
    }
    if (lane == 0 && warp == kTmaAWarp) {
        // activation stages issued by this CTA, kept in the even CTA
        if (rank == 0) {
            progress[0] = na;
        } else {
            const uint32_t dst = mapa_shared(smem_u32(const_cast<int *>(progress)) + 4u, 0u);
            asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(dst), "r"(na) : "memory");
        }
    }
    if (lane == 0 && warp == kTmaCWarp) {
        // code tiles land in this CTA only: wait for the ones still in flight
        for (int it = nc > SC ? nc - SC : 0; it < nc; ++it)
            mbar_drain(&c_full[it % SC], static_cast<uint32_t>(it / SC) & 1u);
    }
    __syncthreads();
    cluster_sync();            // neither CTA leaves while the other may still use its memory
    if (*abort_flag) {
        // Both CTAs' activation copies complete on the even CTA's barriers,
        // which expect the two halves of a stage once the even producer has
        // issued its own. Stages the MMA issuer did not consume may still be in
        // flight; where only one producer issued a stage, the even CTA supplies
        // the other half's arrival or bytes so that the phase can complete,
        // then waits for it. (At most SA stages are outstanding, one per slot.)
        if (rank == 0 && warp == kTmaAWarp && lane == 0) {
            const int n0 = progress[0], n1 = progress[1];
            const int hi = n0 > n1 ? n0 : n1;
            for (int st = progress[2]; st < hi; ++st) {
                uint64_t *bar = &a_full[st % SA];
                if (st < n0 && st >= n1) mbar_complete_tx(bar, Cfg::kABytes);
                if (st >= n0 && st < n1) mbar_arrive_expect_tx(bar, Cfg::kABytes);
                mbar_drain(bar, static_cast<uint32_t>(st / SA) & 1u);
            }
        }
        __syncthreads();
        cluster_sync();        // the odd CTA's activation copies have landed too
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace nf4
