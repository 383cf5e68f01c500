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
// warps turn each 64-code block into bf16 with a per-block register lookup
// table and write it directly in the tensor core's 128-byte-swizzled operand
// layout (K-major for the forward, MN-major for dgrad). The LoRA term is
// ceil(r/64) extra reduction stages whose operands TMA loads directly (r is
// zero-padded to 64 by the TMA out-of-bounds fill).
//
// Warp roles (16 warps, one CTA per SM, persistent over output tiles):
//   warp 0        TMA producer (one thread)
//   warp 1        TMEM owner + MMA issuer (one thread)
//   warps 4..7    epilogue: TMEM -> registers -> bf16 -> global
//   warps 8..15   dequantisation
// Pipelines: a ring of shared-memory stages (full / dequantised / empty
// mbarriers) and two TMEM accumulator buffers (full / empty), so the
// epilogue of one tile overlaps the main loop of the next.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kBM = 128;            // tokens per tile = MMA M
constexpr int kBK = 64;             // reduction per stage = one NF4 block
constexpr int kGemmThreads = 512;
constexpr int kDequantWarp0 = 8;
constexpr int kDequantWarps = 8;
constexpr int kEpiWarp0 = 4;

struct GemmArgs {
    int M;              // tokens
    int red;            // reduction length (forward: K, dgrad: N)
    int out;            // output columns   (forward: N, dgrad: K)
    int main_steps;     // ceil(red / 64)
    int lora_steps;     // ceil(r / 64)
    int m_tiles, n_tiles;
    // quantised weight (always the [N, K] weight)
    int64_t Nw;         // rows of W
    int64_t kblocks;    // K / 64 (blocks per W row)
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    uint16_t *D;        // [M, out] bf16
};

template <int BN, bool DGRAD>
struct GemmCfg {
    static constexpr int kABytes = kBM * kBK * 2;        // 16 KB
    static constexpr int kBBytes = BN * kBK * 2;         // BN rows of 128 B
    static constexpr int kCBytes = BN * kBK / 2;         // 4-bit codes of the B tile
    static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;
    static constexpr int kStages = (220 * 1024) / kStageBytes > 6 ? 6 : (220 * 1024) / kStageBytes;
    static constexpr int kTmemCols = (2 * BN <= 256) ? 256 : 512;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, BN, 0, DGRAD ? 1 : 0);
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kStages >= 3, "pipeline depth");
};

template <int BN, bool DGRAD>
__global__ void __launch_bounds__(kGemmThreads, 1)
qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,    // [M, red] bf16, box {64,128}
                  const __grid_constant__ CUtensorMap tm_codes,  // [Nw, K/2] u8
                  const __grid_constant__ CUtensorMap tm_la,     // [M, r] bf16, box {64,128}
                  const __grid_constant__ CUtensorMap tm_lb,     // fwd: B [N, r]; dgrad: A [r, K]
                  const GemmArgs args) {
    using Cfg = GemmCfg<BN, DGRAD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *slot_a = smem;                                        // [Cfg::kStages][kABytes]
    uint8_t *slot_b = smem + Cfg::kStages * Cfg::kABytes;               // [Cfg::kStages][kBBytes]
    uint8_t *slot_c = slot_b + Cfg::kStages * Cfg::kBBytes;             // [Cfg::kStages][kCBytes]
    uint64_t *bars = reinterpret_cast<uint64_t *>(slot_c + Cfg::kStages * Cfg::kCBytes);
    uint64_t *full = bars;                   // TMA landed         (count 1 + tx)
    uint64_t *bfull = bars + Cfg::kStages;        // B tile ready       (count kDequantWarps)
    uint64_t *empty = bars + 2 * Cfg::kStages;    // MMA done with slot (count 1, tcgen05.commit)
    uint64_t *acc_full = bars + 3 * Cfg::kStages; // [2] accumulator complete
    uint64_t *acc_empty = acc_full + 2;      // [2] accumulator drained (count 4)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bfull[s], kDequantWarps);
            mbar_init(&empty[s], 1);
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
        tma_prefetch_desc(&tm_lb);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total_tiles = args.m_tiles * args.n_tiles;
    const int nsteps = args.main_steps + args.lora_steps;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA
        int st = 0;
        uint32_t ph = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const int m0 = (tile % args.m_tiles) * kBM;
            const int n0 = (tile / args.m_tiles) * BN;
            for (int it = 0; it < nsteps; ++it) {
                if (!mbar_wait(&empty[st], ph ^ 1, abort_flag)) goto done;
                uint8_t *a = slot_a + st * Cfg::kABytes;
                uint8_t *b = slot_b + st * Cfg::kBBytes;
                uint8_t *c = slot_c + st * Cfg::kCBytes;
                if (it < args.main_steps) {
                    mbar_arrive_expect_tx(&full[st], Cfg::kABytes + Cfg::kCBytes);
                    tma_load_2d(a, &tm_act, &full[st], it * kBK, m0);
                    if (!DGRAD) {
                        tma_load_2d(c, &tm_codes, &full[st], it * (kBK / 2), n0);
                    } else {
#pragma unroll
                        for (int kb = 0; kb < BN / 64; ++kb)
                            tma_load_2d(c + kb * 2048, &tm_codes, &full[st], n0 / 2 + kb * 32,
                                        it * kBK);
                    }
                } else {
                    const int ls = it - args.main_steps;
                    mbar_arrive_expect_tx(&full[st], Cfg::kABytes + Cfg::kBBytes);
                    tma_load_2d(a, &tm_la, &full[st], ls * kBK, m0);
                    if (!DGRAD) {
                        tma_load_2d(b, &tm_lb, &full[st], ls * kBK, n0);
                    } else {
#pragma unroll
                        for (int ma = 0; ma < BN / 64; ++ma)
                            tma_load_2d(b + ma * 8192, &tm_lb, &full[st], n0 + ma * 64, ls * kBK);
                    }
                }
                if (++st == Cfg::kStages) { st = 0; ph ^= 1; }
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA
        int st = 0;
        uint32_t ph = 0;
        int ab = 0;
        uint32_t aph = 0;
        const uint32_t a_base = smem_u32(slot_a), b_base = smem_u32(slot_b);
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            if (!mbar_wait(&acc_empty[ab], aph ^ 1, abort_flag)) goto done;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + ab * BN;
            for (int it = 0; it < nsteps; ++it) {
                if (!mbar_wait(&full[st], ph, abort_flag)) goto done;
                if (!mbar_wait(&bfull[st], ph, abort_flag)) goto done;
                tc_fence_after();
                const uint32_t a_addr = a_base + st * Cfg::kABytes;
                const uint32_t b_addr = b_base + st * Cfg::kBBytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                    const uint64_t bd = DGRAD ? smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                              : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
                    umma_bf16_ss(d_tmem, ad, bd, Cfg::kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty[st]);
                if (++st == Cfg::kStages) { st = 0; ph ^= 1; }
            }
            umma_commit(&acc_full[ab]);
            if (++ab == 2) { ab = 0; aph ^= 1; }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
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
    } else if (warp >= kDequantWarp0) {
        // -------------------------------------------------- dequantisation
        // Work item of this thread: forward: W row n0 + i (one block per
        // stage); dgrad: reduction row r_loc of the stage and output block kb.
        // Eight consecutive lanes always take eight consecutive rows of one
        // 8-row swizzle atom, so their 16-byte stores hit distinct banks.
        const int i = threadIdx.x - kDequantWarp0 * 32;
        const bool active = i < BN;
        constexpr int kBPR = BN / 64;
        const int kb = DGRAD ? (i / 8) % kBPR : 0;
        const int r_loc = DGRAD ? (i / (8 * kBPR)) * 8 + (i & 7) : i;
        const uint32_t row_off = DGRAD ? static_cast<uint32_t>(kb * 8192 + r_loc * 128)
                                       : static_cast<uint32_t>(i * 128);
        // codes tiles carry the 32-byte TMA swizzle: 16-byte chunk h of row j
        // sits at chunk h ^ ((j >> 2) & 1)
        const uint32_t code_off = DGRAD ? static_cast<uint32_t>(kb * 2048 + r_loc * 32)
                                        : static_cast<uint32_t>(i * 32);
        const uint32_t cswz = static_cast<uint32_t>((r_loc >> 2) & 1);
        const uint32_t swz = static_cast<uint32_t>(r_loc & 7);

        // raw scale inputs of one (tile, step), loaded one step ahead
        struct RawScale { uint32_t q8; float v; bool valid; };
        auto load_scale = [&](int tile, int it) -> RawScale {
            RawScale rs{0u, 0.0f, false};
            if (tile >= total_tiles || it >= args.main_steps || !active) return rs;
            const int n0 = (tile / args.m_tiles) * BN;
            int64_t wrow, wblk;
            if (!DGRAD) {
                wrow = n0 + i;
                wblk = it;
            } else {
                wrow = static_cast<int64_t>(it) * kBK + r_loc;
                wblk = n0 / 64 + kb;
            }
            if (wrow >= args.Nw || wblk >= args.kblocks) return rs;
            const int64_t b = wrow * args.kblocks + wblk;
            rs.valid = true;
            if (args.dq) {
                rs.q8 = __ldg(args.q8 + b);
                rs.v = __ldg(args.cg + (b >> 8));
            } else {
                rs.v = __ldg(args.absmax + b);
            }
            return rs;
        };

        int st = 0;
        uint32_t ph = 0;
        int tile = blockIdx.x, it = 0;
        RawScale nxt = load_scale(tile, it);
        while (tile < total_tiles) {
            const RawScale cur = nxt;
            const bool main = it < args.main_steps;
            // advance to the next (tile, step) and start its scale load now
            int ntile = tile, nit = it + 1;
            if (nit == nsteps) { nit = 0; ntile += gridDim.x; }
            nxt = load_scale(ntile, nit);
            if (!mbar_wait(&full[st], ph, abort_flag)) goto done;
            if (main && active) {
                const uint8_t *cp = slot_c + st * Cfg::kCBytes + code_off;
                const uint4 c0 = *reinterpret_cast<const uint4 *>(cp + 16 * cswz);
                const uint4 c1 = *reinterpret_cast<const uint4 *>(cp + 16 * (cswz ^ 1));
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint8_t *brow = slot_b + st * Cfg::kBBytes + row_off;
                if (cur.valid) {
                    float s = cur.v;
                    if (args.dq) s = __fmul_rn(static_cast<float>(cur.q8), __fdiv_rn(cur.v, 127.0f));
                    const BlockLut L = make_block_lut(s);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t o[4];
                        dequant8(L, words[ch], o);
                        *reinterpret_cast<uint4 *>(brow + ((ch ^ swz) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                } else {
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4 *>(brow + (ch << 4)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bfull[st]);
            if (++st == Cfg::kStages) { st = 0; ph ^= 1; }
            tile = ntile;
            it = nit;
        }
    }
done:
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace nf4
