// skinny_tc.cuh -- the rank-r products of the QLoRA layer on tcgen05 tensor
// cores. Each is out[p][j] = sum_q P(p, q) Q(q, j) with j < r <= 128:
//   u  = x A^T          P = x   [M, K] (K-major),  Q = A  [r, K] (K-major)
//   v  = dY B           P = dY  [M, N] (K-major),  Q = B  [N, r] (MN-major)
//   dB = dY^T (s u)     P = dY^T: dY [M, N] read MN-major, Q = bf16(s u) [M, r] (MN-major)
//   dA^T = x^T (s v)    P = x^T:  x  [M, K] read MN-major, Q = bf16(s v) [M, r] (MN-major)
// (forward down-projection, "QLoRA explained", section "The LoRA adapter
// path"; the adapter gradients follow by the chain rule with W0 frozen).
// They stream one large operand once, so they are HBM-bound. The reduction
// is split across the CTAs of one thread-block cluster per 128-row output
// tile (at most 8 splits, sized so that the whole grid is one wave): each CTA
// streams its share into a tensor-memory accumulator, parks its fp32 partial
// in its own shared memory, and after a cluster barrier the CTAs add the
// partials of all splits in split order through distributed shared memory
// (deterministic) and write the destination with its scale, rounding and
// layout. No partial sums go to global memory. One launch may carry two
// products of the same operand layouts (the backward's dB and dA, which are
// independent) and an element-wise side task (bf16(s u) from the saved u),
// so that each launch's ramp and drain are paid once.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kSkStages = 4;     // two CTAs fit on one SM
constexpr int kSkThreads = 256;   // warp 0 TMA, warp 1 MMA, warps 4..7 dropout mask and epilogue
constexpr int kSkMaxSplits = 8;   // portable cluster size

// One product of a launch. A launch carries one or two products of the same
// operand layouts; grid rows [0, p_tiles of job 0) take job 0, the rest job 1.
struct SkinnyJob {
    int P;               // output rows (MMA M, tiles of 128)
    int p_tiles;
    int steps;           // reduction steps of 64
    int steps_per_split;
    int r;               // output columns actually written (<= RN)
    float *out_f32;      // the sum in fp32 (unscaled): [P][r], or [r][P] when transposed; or null
    uint16_t *out_bf16;  // bf16(scale * sum): [P][r], or [r][P] when transposed; or null
    float scale;
    int transposed;
    // dropout on x as the A operand (LoRA dropout: the keep mask is an input,
    // bit (e & 7) of byte e >> 3 for element e = m * kx + k of x [mx, kx], or,
    // when rng.on, drawn here from the counter-based generator):
    // 0 = none, 1 = A is x K-major (tile rows are tokens), 2 = A is x
    // MN-major (tile rows are tokens of two 64-column halves)
    int mask_mode;
    const uint8_t *keep;
    int64_t mx, kx;
    DropRng rng;
};

struct SkinnyArgs {
    SkinnyJob job[2];
    int njobs;
    int *zero_ints;      // optional: zeroed by the first CTA (flags for a later kernel)
    int zero_count;
    // optional element-wise side task over all CTAs: conv_dst[i] = bf16(conv_scale * conv_src[i])
    const float *conv_src;
    uint16_t *conv_dst;
    int64_t conv_n;
    float conv_scale;
    // optional per-row adapter selection (several stacked adapters, one per
    // output row): row p keeps only the group_width columns of adapter
    // row_group[p], scaled by gscale of that adapter; other columns, and rows
    // whose adapter is outside [0, ngroups), get zero in out_bf16
    const int32_t *row_group;
    int group_width;
    int ngroups;
    float gscale[16];
};

template <int RN, bool A_MN, bool B_MN>
struct SkCfg {
    static constexpr int kABytes = 128 * 64 * 2;                 // 16 KB
    static constexpr int kBBytes = RN * 64 * 2;                  // RN x 64 bf16
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kPartStride = RN + 4;                   // floats per partial row
    static constexpr int kSmemBytes = kSkStages * kStageBytes + 1024 + 256;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(128, RN, A_MN ? 1 : 0, B_MN ? 1 : 0);
    static_assert(RN == 64 || RN == 128, "RN");
    static_assert(128 * kPartStride * 4 <= kSkStages * kStageBytes, "partial fits the stages");
};

__device__ __forceinline__ float ld_cluster_f32(uint32_t caddr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(caddr) : "memory");
    return v;
}

// Grid (splits, p_tiles), cluster (splits, 1, 1): blockIdx.x is the split.
template <int RN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kSkThreads, 2)
skinny_cluster_kernel(const __grid_constant__ CUtensorMap tm_a0,
                      const __grid_constant__ CUtensorMap tm_b0,
                      const __grid_constant__ CUtensorMap tm_a1,
                      const __grid_constant__ CUtensorMap tm_b1, const SkinnyArgs args) {
    using Cfg = SkCfg<RN, A_MN, B_MN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *slot_a = smem;
    uint8_t *slot_b = smem + kSkStages * Cfg::kABytes;
    float *part = reinterpret_cast<float *>(smem);   // [128][kPartStride], after the main loop
    uint64_t *bars = reinterpret_cast<uint64_t *>(slot_b + kSkStages * Cfg::kBBytes);
    uint64_t *full = bars, *empty = bars + kSkStages, *done_bar = bars + 2 * kSkStages;
    uint64_t *masked = done_bar + 1;            // [stages] dropout applied to the A tile
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(masked + kSkStages);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, splits = gridDim.x;
    const int jb = (args.njobs > 1 && static_cast<int>(blockIdx.y) >= args.job[0].p_tiles) ? 1 : 0;
    const SkinnyJob &J = args.job[jb];
    const CUtensorMap *tm_a = jb ? &tm_a1 : &tm_a0;
    const CUtensorMap *tm_b = jb ? &tm_b1 : &tm_b0;
    const int p0 = (static_cast<int>(blockIdx.y) - (jb ? args.job[0].p_tiles : 0)) * 128;
    const int s0 = split * J.steps_per_split;
    const int s1 = min(J.steps, s0 + J.steps_per_split);
    const int nsteps = s1 - s0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSkStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&masked[s], 4);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(tm_a);
        tma_prefetch_desc(tm_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, RN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();
    griddep_launch_dependents();
    if (args.zero_ints && blockIdx.x == 0 && blockIdx.y == 0)
        for (int z = threadIdx.x; z < args.zero_count; z += kSkThreads) args.zero_ints[z] = 0;
    if (args.conv_n > 0) {
        const int64_t ctas = static_cast<int64_t>(gridDim.x) * gridDim.y;
        const int64_t cta = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
        for (int64_t e = cta * kSkThreads + threadIdx.x; e < args.conv_n; e += ctas * kSkThreads) {
            __nv_bfloat16 b = __float2bfloat16_rn(args.conv_scale * args.conv_src[e]);
            args.conv_dst[e] = *reinterpret_cast<uint16_t *>(&b);
        }
    }

    if (warp == 0 && lane == 0) {
        int issued = 0;
        for (int it = 0; it < nsteps; ++it) {
            const int st = it % kSkStages;
            const uint32_t ph = (it / kSkStages) & 1;
            if (!mbar_wait(&empty[st], ph ^ 1, abort_flag)) break;
            ++issued;
            uint8_t *a = slot_a + st * Cfg::kABytes;
            uint8_t *b = slot_b + st * Cfg::kBBytes;
            const int q0 = (s0 + it) * 64;
            mbar_arrive_expect_tx(&full[st], Cfg::kStageBytes);
            if (!A_MN) {
                tma_load_2d(a, tm_a, &full[st], q0, p0);
            } else {
                tma_load_2d(a, tm_a, &full[st], p0, q0);
                tma_load_2d(a + 8192, tm_a, &full[st], p0 + 64, q0);
            }
            if (!B_MN) {
                tma_load_2d(b, tm_b, &full[st], q0, 0);
            } else {
#pragma unroll
                for (int ja = 0; ja < RN / 64; ++ja)
                    tma_load_2d(b + ja * 8192, tm_b, &full[st], ja * 64, q0);
            }
        }
        // every copy issued has landed before the stage buffers are reused or
        // released (at most one stage per slot can still be in flight; after
        // a normal run all of them were consumed, so these return at once)
        for (int it = issued > kSkStages ? issued - kSkStages : 0; it < issued; ++it)
            mbar_drain(&full[it % kSkStages], static_cast<uint32_t>(it / kSkStages) & 1u);
    } else if (warp == 1 && lane == 0) {
        const uint32_t a_base = smem_u32(slot_a), b_base = smem_u32(slot_b);
        bool ok = true;
        for (int it = 0; it < nsteps; ++it) {
            const int st = it % kSkStages;
            const uint32_t ph = (it / kSkStages) & 1;
            if (!mbar_wait(J.mask_mode ? &masked[st] : &full[st], ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t aa = a_base + st * Cfg::kABytes, bb = b_base + st * Cfg::kBBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = A_MN ? smem_desc_sw128(aa + kk * 2048, 8192, 1024)
                                         : smem_desc_sw128(aa + kk * 32, 16, 1024);
                const uint64_t bd = B_MN ? smem_desc_sw128(bb + kk * 2048, 8192, 1024)
                                         : smem_desc_sw128(bb + kk * 32, 16, 1024);
                umma_bf16_ss(tmem_base, ad, bd, Cfg::kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&empty[st]);
        }
        // after giving up, the MMAs already issued must complete before the
        // stage buffers and tensor memory are released
        umma_commit(done_bar);
        if (!ok) mbar_drain(done_bar, 0);
    } else if (warp >= 4 && warp < 8) {
        if (J.mask_mode) {
            // dropout: zero the dropped elements of each landed A tile in place
            // before the MMA reads it (these warps are idle until the last MMA).
            // The tile is 128 rows of 128 bytes (64 consecutive k of one token,
            // 128-byte swizzle); a 16-byte piece holds 8 k, i.e. one keep byte,
            // so a row's keep bits are one aligned 8-byte word (kx and the tile
            // origins are multiples of 64). Thread t takes row t and fetches its
            // word before the tile lands.
            const int row = threadIdx.x - 128;
            for (int it = 0; it < nsteps; ++it) {
                const int st = it % kSkStages;
                const uint32_t ph = (it / kSkStages) & 1;
                const int q0 = (s0 + it) * 64;
                const int64_t m = J.mask_mode == 1 ? p0 + row : q0 + (row & 63);
                const int64_t k0 = J.mask_mode == 1 ? q0 : p0 + 64 * (row >> 6);
                const bool rok = m < J.mx && k0 < J.kx;
                uint64_t kw = ~0ull;
                if (rok) {
                    if (J.rng.on) {
                        // the row's 64 keep bits from the generator
                        kw = drop_keep_bits<16>(J.rng, static_cast<uint64_t>(m * J.kx + k0));
                    } else {
                        kw = __ldg(reinterpret_cast<const unsigned long long *>(J.keep + ((m * J.kx + k0) >> 3)));
                    }
                }
                if (!mbar_wait(&full[st], ph, abort_flag)) break;
                uint8_t *a = slot_a + st * Cfg::kABytes;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t kb = static_cast<uint32_t>(kw >> (8 * c)) & 0xFFu;
                    if (kb == 0xFFu) continue;                      // all eight kept
                    uint4 *piece = reinterpret_cast<uint4 *>(a + row * 128 + ((c ^ (row & 7)) << 4));
                    uint4 v = *piece;
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o[e] = w[e] & (((kb >> (2 * e)) & 1u ? 0x0000ffffu : 0u) |
                                       ((kb >> (2 * e + 1)) & 1u ? 0xffff0000u : 0u));
                    *piece = make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_proxy_async_smem();     // generic writes before the tensor core reads the tile
                __syncwarp();
                if (lane == 0) mbar_arrive(&masked[st]);
            }
        }
        // accumulator -> this CTA's partial (the stage buffers are free once
        // the last MMA has completed: every load it waited for has landed)
        const int q = warp - 4;
        float *prow = part + (q * 32 + lane) * Cfg::kPartStride;
        if (nsteps <= 0) {
            for (int j = 0; j < RN; j += 4)
                *reinterpret_cast<float4 *>(prow + j) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else if (mbar_wait(done_bar, 0, abort_flag)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < RN / 32; ++c) {
                if (c * 32 >= J.r) break;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + ((q * 32) << 16) + c * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(prow + c * 32 + e) =
                        make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                    __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();            // every split's partial is written and visible

    // Ordered sum over the splits: CTA `split` takes its share of the tile's
    // (row, column) elements, numbered column-major when the destination is
    // transposed so that consecutive threads write consecutive addresses.
    {
        const int r = J.r;
        const int E = 128 * r;
        const int e0 = static_cast<int>((static_cast<int64_t>(E) * split) / splits);
        const int e1 = static_cast<int>((static_cast<int64_t>(E) * (split + 1)) / splits);
        const uint32_t part_addr = smem_u32(part);
        for (int e = e0 + threadIdx.x; e < e1; e += kSkThreads) {
            const int row = J.transposed ? e % 128 : e / r;
            const int j = J.transposed ? e / 128 : e % r;
            const int p = p0 + row;
            if (p >= J.P) continue;
            const uint32_t off = static_cast<uint32_t>((row * Cfg::kPartStride + j) * 4);
            float acc = 0.0f;
            for (int s = 0; s < splits; ++s)
                acc += ld_cluster_f32(mapa_shared(part_addr + off, static_cast<uint32_t>(s)));
            const int64_t o = J.transposed ? static_cast<int64_t>(j) * J.P + p
                                           : static_cast<int64_t>(p) * r + j;
            if (J.out_f32) J.out_f32[o] = acc;
            if (J.out_bf16) {
                float sc = J.scale;
                if (args.row_group) {
                    const int gp = args.row_group[p];
                    const bool keep = gp >= 0 && gp < args.ngroups && j / args.group_width == gp;
                    sc = keep ? args.gscale[gp] : 0.0f;
                }
                __nv_bfloat16 b = __float2bfloat16_rn(sc * acc);
                J.out_bf16[o] = *reinterpret_cast<uint16_t *>(&b);
            }
        }
    }
    cluster_sync();            // no CTA leaves while another still reads its partial
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, RN);
    }
}

__global__ void zero_u16_kernel(uint16_t *__restrict__ p, int64_t n) {
    griddep_wait();
    griddep_launch_dependents();
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[e] = 0;
}

}  // namespace nf4
