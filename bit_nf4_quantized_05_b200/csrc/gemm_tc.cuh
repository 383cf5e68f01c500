// gemm_tc.cuh -- fused NF4-dequantise + GEMM on sm_100a tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
// One kernel computes, for a 128-token x BN-column output tile,
//     D = act * W~op  +  lora_a * lora_b
// in two directions of the QLoRA layer:
//   forward: act = x [M, K],  W~op = W~^T      (reduce over k; W~ rows = output)
//            lora_a = bf16((alpha/r) x A^T) [M, r], lora_b = B^T
//            ("QLoRA explained", section "The LoRA adapter path":
//             x W^T + (x A^T) B^T * scale)
//   dgrad:   act = dY [M, N], W~op = W~        (reduce over n; W~ cols = output)
//            lora_a = bf16((alpha/r) dY B) [M, r], lora_b = A
//            (chain rule through the frozen dequantised weight)
// The 4-bit codes stream into shared memory through TMA; dequantisation
// warps turn each 64-code block into bf16 (two threads per block, sharing a
// per-block register lookup table) and write it directly in the tensor
// core's 128-byte-swizzled operand layout: K-major for the forward, MN-major
// for dgrad. The LoRA term is ceil(r/64) extra reduction stages (r zero-padded
// to 64).
//
// Warp roles (one CTA per SM, persistent over output tiles):
//   warps 0..3    epilogue: TMEM -> registers -> bf16 -> global (warp w reads
//                 TMEM lanes 32(w%4)..)
//   warp 4        TMA producer of activation tiles
//   warp 5        TMEM owner + MMA issuer (one thread)
//   warp 6        TMA producer of code tiles
//   warps 7..     dequantisation (2*BN threads)
// Three shared-memory rings decouple the producers: activation tiles (freed
// by the MMA), code tiles (freed as soon as the dequant warps have read them,
// so they can be fetched far ahead), and dequantised weight tiles (freed by
// the MMA). Two TMEM accumulator buffers let the epilogue of one tile overlap
// the main loop of the next.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kBM = 128;            // tokens per tile = MMA M
constexpr int kBK = 64;             // reduction per stage = one NF4 block
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
    // stream-K schedule (CTA-pair kernel only): 0 = whole tiles round-robin
    int sk;
    float *partial;     // [pairs][2][BN/32][128][32] fp32 partial tiles
    int *flags;         // [pairs][2][4 epilogue warps], zero at launch; 1 = rows written
    float *D32;         // when non-null: the fp32 result goes here instead of D
    int bshift;         // log2(block size / 64): block of step j is j >> bshift
};

template <int BN, bool DGRAD>
struct GemmCfg {
    static constexpr int kABytes = kBM * kBK * 2;        // 16 KB
    static constexpr int kBBytes = BN * kBK * 2;         // BN rows of 128 B
    static constexpr int kCBytes = BN * kBK / 2;         // 4-bit codes of the B tile
    static constexpr int kSB = BN <= 192 ? 4 : 2;        // dequantised-tile stages (even)
    static constexpr int kSC = 6;                        // code-tile stages
    static constexpr int kSA = (220 * 1024 - kSB * kBBytes - kSC * kCBytes) / kABytes > 8
                                   ? 8
                                   : (220 * 1024 - kSB * kBBytes - kSC * kCBytes) / kABytes;
    static constexpr int kGroupWarps = BN / 32;           // warps of one dequant group
    static constexpr int kDeqWarps = 2 * kGroupWarps;     // two groups take alternate stages
    static constexpr int kThreads = 32 * (kDequantWarp0 + kDeqWarps);
    static constexpr int kTmemCols = (2 * BN <= 256) ? 256 : 512;
    static constexpr int kSmemBytes =
        kSA * kABytes + kSB * kBBytes + kSC * kCBytes + 1024 /*align*/ + 512 /*barriers*/;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, BN, 0, DGRAD ? 1 : 0);
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert(kBBytes % 1024 == 0 && kCBytes % 1024 == 0, "stage alignment");
    static_assert(kSA >= 3, "pipeline depth");
    static_assert(kSB % 2 == 0, "the two dequant groups alternate over the weight-tile ring");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

template <int BN, bool DGRAD>
__global__ void __launch_bounds__(GemmCfg<BN, DGRAD>::kThreads, 1)
qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,    // [M, red] bf16, box {64,128}
                  const __grid_constant__ CUtensorMap tm_codes,  // [Nw, K/2] u8, box {32, rows}
                  const __grid_constant__ CUtensorMap tm_la,     // [M, r] bf16, box {64,128}
                  const GemmArgs args) {
    using Cfg = GemmCfg<BN, DGRAD>;
    constexpr int SA = Cfg::kSA, SB = Cfg::kSB, SC = Cfg::kSC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *slot_a = smem;                              // [SA][kABytes]
    uint8_t *slot_b = slot_a + SA * Cfg::kABytes;        // [SB][kBBytes]
    uint8_t *slot_c = slot_b + SB * Cfg::kBBytes;        // [SC][kCBytes]
    uint64_t *bars = reinterpret_cast<uint64_t *>(slot_c + SC * Cfg::kCBytes);
    uint64_t *a_full = bars;                 // TMA landed            (1 + tx)
    uint64_t *a_empty = a_full + SA;         // MMA done              (commit)
    uint64_t *c_full = a_empty + SA;         // TMA landed            (1 + tx)
    uint64_t *c_empty = c_full + SC;         // codes read            (one dequant group)
    uint64_t *b_full = c_empty + SC;         // weight tile written   (one dequant group)
    uint64_t *b_empty = b_full + SB;         // MMA done              (commit)
    uint64_t *acc_full = b_empty + SB;       // [2] accumulator complete (commit)
    uint64_t *acc_empty = acc_full + 2;      // [2] accumulator drained  (4 epilogue warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < SC; ++s) {
            mbar_init(&c_full[s], 1);
            mbar_init(&c_empty[s], Cfg::kGroupWarps);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(&b_full[s], Cfg::kGroupWarps);
            mbar_init(&b_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_la);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();
    griddep_launch_dependents();

    const int total_tiles = args.m_tiles * args.n_tiles;
    const int nsteps = args.main_steps + args.lora_steps;

    if (warp == kTmaAWarp) {
        // ------------------------------------------------ TMA: activations
        if (lane == 0) {
            int sa = 0;
            uint32_t pa = 0;
            for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
                const int m0 = (tile % args.m_tiles) * kBM;
                for (int it = 0; it < nsteps; ++it) {
                    if (!mbar_wait(&a_empty[sa], pa ^ 1, abort_flag)) goto done;
                    mbar_arrive_expect_tx(&a_full[sa], Cfg::kABytes);
                    if (it < args.main_steps)
                        tma_load_2d(slot_a + sa * Cfg::kABytes, &tm_act, &a_full[sa], it * kBK, m0);
                    else
                        tma_load_2d(slot_a + sa * Cfg::kABytes, &tm_la, &a_full[sa],
                                    (it - args.main_steps) * kBK, m0);
                    if (++sa == SA) { sa = 0; pa ^= 1; }
                }
            }
        }
    } else if (warp == kTmaCWarp) {
        // ------------------------------------------------ TMA: 4-bit codes
        if (lane == 0) {
            int sc = 0;
            uint32_t pc = 0;
            for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
                const int n0 = (tile / args.m_tiles) * BN;
                for (int it = 0; it < args.main_steps; ++it) {
                    if (!mbar_wait(&c_empty[sc], pc ^ 1, abort_flag)) goto done;
                    uint8_t *c = slot_c + sc * Cfg::kCBytes;
                    mbar_arrive_expect_tx(&c_full[sc], Cfg::kCBytes);
                    if (!DGRAD) {
                        tma_load_2d(c, &tm_codes, &c_full[sc], it * (kBK / 2), n0);
                    } else {
#pragma unroll
                        for (int kb = 0; kb < BN / 64; ++kb)
                            tma_load_2d(c + kb * 2048, &tm_codes, &c_full[sc], n0 / 2 + kb * 32,
                                        it * kBK);
                    }
                    if (++sc == SC) { sc = 0; pc ^= 1; }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            int sa = 0, sb = 0, ab = 0;
            uint32_t pa = 0, pb = 0, aph = 0;
            const uint32_t a_base = smem_u32(slot_a), b_base = smem_u32(slot_b);
            for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
                if (!mbar_wait(&acc_empty[ab], aph ^ 1, abort_flag)) goto done;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + ab * BN;
                for (int it = 0; it < nsteps; ++it) {
                    if (!mbar_wait(&a_full[sa], pa, abort_flag)) goto done;
                    if (!mbar_wait(&b_full[sb], pb, abort_flag)) goto done;
                    tc_fence_after();
                    const uint32_t a_addr = a_base + sa * Cfg::kABytes;
                    const uint32_t b_addr = b_base + sb * Cfg::kBBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bd = DGRAD ? smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                                  : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
                        umma_bf16_ss(d_tmem, ad, bd, Cfg::kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&a_empty[sa]);
                    umma_commit(&b_empty[sb]);
                    if (++sa == SA) { sa = 0; pa ^= 1; }
                    if (++sb == SB) { sb = 0; pb ^= 1; }
                }
                umma_commit(&acc_full[ab]);
                if (++ab == 2) { ab = 0; aph ^= 1; }
            }
        }
    } else if (warp < kEpiWarp0 + 4) {
        // ------------------------------------------------------- epilogue
        const int q = warp - kEpiWarp0;                   // TMEM lane quadrant (== warp % 4)
        int ab = 0;
        uint32_t aph = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const int m0 = (tile % args.m_tiles) * kBM;
            const int n0 = (tile / args.m_tiles) * BN;
            if (!mbar_wait(&acc_full[ab], aph, abort_flag)) goto done;
            tc_fence_after();
            const int row = m0 + q * 32 + lane;
            uint16_t *drow = args.D + static_cast<int64_t>(row) * args.out;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + ((q * 32) << 16) + ab * BN + c * 32, v);
                tmem_ld_wait();
                if (row < args.M) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int col = n0 + c * 32 + g * 8;
                        if (col < args.out) {
                            if (args.D32) {
                                float4 *f4 = reinterpret_cast<float4 *>(args.D32 + static_cast<int64_t>(row) * args.out + col);
                                f4[0] = make_float4(__uint_as_float(v[g * 8]), __uint_as_float(v[g * 8 + 1]),
                                                    __uint_as_float(v[g * 8 + 2]), __uint_as_float(v[g * 8 + 3]));
                                f4[1] = make_float4(__uint_as_float(v[g * 8 + 4]), __uint_as_float(v[g * 8 + 5]),
                                                    __uint_as_float(v[g * 8 + 6]), __uint_as_float(v[g * 8 + 7]));
                                continue;
                            }
                            uint32_t p[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(
                                    __uint_as_float(v[g * 8 + 2 * e]),
                                    __uint_as_float(v[g * 8 + 2 * e + 1]));
                                p[e] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            *reinterpret_cast<uint4 *>(drow + col) = make_uint4(p[0], p[1], p[2], p[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            if (++ab == 2) { ab = 0; aph ^= 1; }
        }
    } else {
        // -------------------------------------------------- dequantisation
        // Two groups of BN threads take alternate stages (group g handles the
        // stages whose global index is g mod 2), so each thread has two stage
        // times for one 64-element block. Thread i of a group owns work item i:
        //   forward: W row n0 + i, block `it` of the stage
        //   dgrad:   reduction row r_loc of the stage, output block kb
        // Eight consecutive lanes take eight consecutive rows of one 8-row
        // swizzle atom, so each 8-lane phase of a 16-byte shared access hits
        // distinct banks.
        const int t = threadIdx.x - kDequantWarp0 * 32;
        const int grp = t / BN;
        const int i = t % BN;
        constexpr int kBPR = BN / 64;
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

        // block index of (tile, stage) for this item, or -1 outside the weight
        auto block_of = [&](int tile, int it) -> int64_t {
            if (tile >= total_tiles || it >= args.main_steps) return -1;
            const int n0 = (tile / args.m_tiles) * BN;
            int64_t wrow, wblk;
            if (!DGRAD) {
                wrow = n0 + i;
                wblk = it;
            } else {
                wrow = static_cast<int64_t>(it) * kBK + r_loc;
                wblk = n0 / 64 + kb;
            }
            if (wrow >= args.Nw || wblk >= args.kblocks) return -1;
            return wrow * (args.kblocks >> args.bshift) + (wblk >> args.bshift);
        };
        struct RawScale { int64_t b; uint32_t q8; float v; };
        auto load_scale = [&](int64_t b) -> RawScale {
            RawScale rs{b, 0u, 0.0f};
            if (b < 0) return rs;
            if (args.dq) rs.q8 = __ldg(args.q8 + b);
            else rs.v = __ldg(args.absmax + b);
            return rs;
        };
        int64_t kg_group = -1;      // cached fl32(c_g / 127) of the last group seen
        float kg = 0.0f;

        // walk every (tile, stage) in order; this group acts on every other one
        int tile = blockIdx.x, it = 0;
        int64_t gstep = 0;          // global stage counter (weight-tile ring)
        int64_t mstep = 0;          // global main-stage counter (code ring)
        // the next stage of this group, and its prefetched scale
        auto advance = [&](int &tl, int &st_, int64_t &g, int64_t &m) {
            if (st_ < args.main_steps) ++m;
            ++g;
            if (++st_ == nsteps) { st_ = 0; tl += gridDim.x; }
        };
        if (grp == 1 && tile < total_tiles) advance(tile, it, gstep, mstep);
        RawScale nxt = load_scale(block_of(tile, it));
        while (tile < total_tiles) {
            const RawScale cur = nxt;
            const bool main = it < args.main_steps;
            const int n0 = (tile / args.m_tiles) * BN;
            const int sb = static_cast<int>(gstep % SB);
            const uint32_t pb = static_cast<uint32_t>((gstep / SB) & 1);
            const int sc = static_cast<int>(mstep % SC);
            const uint32_t pc = static_cast<uint32_t>((mstep / SC) & 1);
            // this group's following stage: skip the other group's one
            int ntile = tile, nit = it;
            int64_t ng = gstep, nm = mstep;
            advance(ntile, nit, ng, nm);
            if (ntile < total_tiles) advance(ntile, nit, ng, nm);
            nxt = load_scale(block_of(ntile, nit));

            uint32_t out[32];
            if (main) {
                if (!mbar_wait(&c_full[sc], pc, abort_flag)) goto done;
                const uint8_t *cp = slot_c + sc * Cfg::kCBytes + code_off;
                const uint4 h0 = *reinterpret_cast<const uint4 *>(cp + 16 * cswz);
                const uint4 h1 = *reinterpret_cast<const uint4 *>(cp + 16 * (cswz ^ 1));
                float s = 0.0f;
                if (cur.b >= 0) {
                    if (args.dq) {
                        const int64_t g = cur.b >> 8;
                        if (g != kg_group) {
                            kg_group = g;
                            kg = __fdiv_rn(__ldg(args.cg + g), 127.0f);
                        }
                        s = __fmul_rn(static_cast<float>(cur.q8), kg);
                    } else {
                        s = cur.v;
                    }
                }
                const BlockLut L = make_block_lut(s);
                const uint32_t words[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                for (int wd = 0; wd < 8; ++wd) {
                    uint32_t o[4];
                    dequant8(L, words[wd], o);
#pragma unroll
                    for (int e = 0; e < 4; ++e) out[4 * wd + e] = cur.b >= 0 ? o[e] : 0u;
                }
                // the codes are consumed (out depends on them): release the slot
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
            } else {
                // LoRA stage: the adapter tile comes straight from global memory
                //   forward: B[n0 + i][64 ls .. +64)        (zero beyond r, N)
                //   dgrad:   A[64 ls + r_loc][n0 + 64 kb .. +64)  (zero beyond r, K)
                const int ls = it - args.main_steps;
                const uint16_t *src = nullptr;
                int nvalid = 0;   // valid 8-element chunks
                if (!DGRAD) {
                    const int64_t n = n0 + i;
                    const int j0 = 64 * ls;
                    if (n < args.Nw && j0 < args.r) {
                        src = args.lora_b + n * args.r + j0;
                        nvalid = (args.r - j0) / 8 >= 8 ? 8 : (args.r - j0) / 8;
                    }
                } else {
                    const int j = 64 * ls + r_loc;
                    const int64_t k0 = static_cast<int64_t>(n0) + 64 * kb;
                    if (j < args.r && k0 < args.Kw) {
                        src = args.lora_b + static_cast<int64_t>(j) * args.Kw + k0;
                        nvalid = (args.Kw - k0) / 8 >= 8 ? 8 : static_cast<int>((args.Kw - k0) / 8);
                    }
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (c < nvalid) v = __ldg(reinterpret_cast<const uint4 *>(src) + c);
                    out[4 * c] = v.x;
                    out[4 * c + 1] = v.y;
                    out[4 * c + 2] = v.z;
                    out[4 * c + 3] = v.w;
                }
            }
            if (!mbar_wait(&b_empty[sb], pb ^ 1, abort_flag)) goto done;
            uint8_t *brow = slot_b + sb * Cfg::kBBytes + row_off;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(brow + ((c ^ swz) << 4)) =
                    make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_full[sb]);
            tile = ntile;
            it = nit;
            gstep = ng;
            mstep = nm;
        }
    }
done:
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace nf4
