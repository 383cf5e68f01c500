// skinny_tc.cuh -- the rank-r products of the QLoRA layer on tcgen05 tensor
// cores. Each is out[p][j] = sum_q P(p, q) Q(q, j) with j < r <= 128:
//   u  = x A^T          P = x   [M, K] (K-major),  Q = A  [r, K] (K-major)
//   v  = dY B           P = dY  [M, N] (K-major),  Q = B  [N, r] (MN-major)
//   dB = dY^T (s u)     P = dY^T: dY [M, N] read MN-major, Q = bf16(s u) [M, r] (MN-major)
//   dA^T = x^T (s v)    P = x^T:  x  [M, K] read MN-major, Q = bf16(s v) [M, r] (MN-major)
// (forward down-projection, "QLoRA explained", section "The LoRA adapter
// path"; the adapter gradients follow by the chain rule with W0 frozen).
// They stream one large operand once, so they are HBM-bound: the reduction is
// split across CTAs so that every SM streams, each CTA writes fp32 partial
// sums, and a second kernel adds the splits in a fixed order (deterministic)
// and applies the scale, rounding and layout of the destination.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kSkStages = 6;
constexpr int kSkThreads = 256;   // warp 0 TMA, warp 1 MMA, warps 4..7 epilogue

struct SkinnyArgs {
    int P;               // output rows (MMA M, tiles of 128)
    int steps;           // reduction steps of 64
    int steps_per_split;
    float *part;         // [splits][P][RN] fp32
};

template <int RN, bool A_MN, bool B_MN>
struct SkCfg {
    static constexpr int kABytes = 128 * 64 * 2;                 // 16 KB
    static constexpr int kBBytes = RN * 64 * 2;                  // RN x 64 bf16
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kSmemBytes = kSkStages * kStageBytes + 1024 + 256;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(128, RN, A_MN ? 1 : 0, B_MN ? 1 : 0);
    static_assert(RN == 64 || RN == 128, "RN");
};

template <int RN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kSkThreads, 1)
skinny_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const SkinnyArgs args) {
    using Cfg = SkCfg<RN, A_MN, B_MN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *slot_a = smem;
    uint8_t *slot_b = smem + kSkStages * Cfg::kABytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(slot_b + kSkStages * Cfg::kBBytes);
    uint64_t *full = bars, *empty = bars + kSkStages, *done_bar = bars + 2 * kSkStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p0 = blockIdx.x * 128;
    const int s0 = blockIdx.y * args.steps_per_split;
    const int s1 = min(args.steps, s0 + args.steps_per_split);
    const int nsteps = s1 - s0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSkStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, RN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        for (int it = 0; it < nsteps; ++it) {
            const int st = it % kSkStages;
            const uint32_t ph = (it / kSkStages) & 1;
            if (!mbar_wait(&empty[st], ph ^ 1, abort_flag)) break;
            uint8_t *a = slot_a + st * Cfg::kABytes;
            uint8_t *b = slot_b + st * Cfg::kBBytes;
            const int q0 = (s0 + it) * 64;
            mbar_arrive_expect_tx(&full[st], Cfg::kStageBytes);
            if (!A_MN) {
                tma_load_2d(a, &tm_a, &full[st], q0, p0);
            } else {
                tma_load_2d(a, &tm_a, &full[st], p0, q0);
                tma_load_2d(a + 8192, &tm_a, &full[st], p0 + 64, q0);
            }
            if (!B_MN) {
                tma_load_2d(b, &tm_b, &full[st], q0, 0);
            } else {
#pragma unroll
                for (int ja = 0; ja < RN / 64; ++ja)
                    tma_load_2d(b + ja * 8192, &tm_b, &full[st], ja * 64, q0);
            }
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t a_base = smem_u32(slot_a), b_base = smem_u32(slot_b);
        bool ok = true;
        for (int it = 0; it < nsteps; ++it) {
            const int st = it % kSkStages;
            const uint32_t ph = (it / kSkStages) & 1;
            if (!mbar_wait(&full[st], ph, abort_flag)) { ok = false; break; }
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
        if (ok) umma_commit(done_bar);
    } else if (warp >= 4 && warp < 8) {
        const int q = warp - 4;
        const int p = p0 + q * 32 + lane;
        float *dst = args.part + (static_cast<int64_t>(blockIdx.y) * args.P + p) * RN;
        if (nsteps <= 0) {
            if (p < args.P)
                for (int j = 0; j < RN; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else if (mbar_wait(done_bar, 0, abort_flag)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < RN / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + ((q * 32) << 16) + c * 32, v);
                tmem_ld_wait();
                if (p < args.P) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(dst + c * 32 + e) =
                            make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                        __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, RN);
    }
}

// out = sum over splits of part[s][p][j] (j < r), in split order; then
//   out_f32[p][j]  = sum                       (if out_f32)
//   out_bf16[..]   = bf16(scale * sum)         (if out_bf16; [p][j], or [j][p] when transposed)
__global__ void skinny_reduce_kernel(const float *__restrict__ part, int splits, int P, int RN, int r,
                                     float *__restrict__ out_f32, uint16_t *__restrict__ out_bf16,
                                     float scale, int transposed) {
    const int64_t total = static_cast<int64_t>(P) * r;
    const int64_t stride = static_cast<int64_t>(P) * RN;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t p = e / r, j = e % r;
        const float *src = part + p * RN + j;
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s) acc += src[s * stride];
        if (out_f32) out_f32[p * r + j] = acc;
        if (out_bf16) {
            __nv_bfloat16 b = __float2bfloat16_rn(scale * acc);
            const int64_t o = transposed ? j * P + p : p * r + j;
            out_bf16[o] = *reinterpret_cast<uint16_t *>(&b);
        }
    }
}

// dst[i] = bf16(scale * src[i])
__global__ void scale_to_bf16_kernel(const float *__restrict__ src, int64_t n, float scale,
                                     uint16_t *__restrict__ dst) {
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        __nv_bfloat16 b = __float2bfloat16_rn(scale * src[e]);
        dst[e] = *reinterpret_cast<uint16_t *>(&b);
    }
}

__global__ void zero_u16_kernel(uint16_t *__restrict__ p, int64_t n) {
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[e] = 0;
}

}  // namespace nf4
