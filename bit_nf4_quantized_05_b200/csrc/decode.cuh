// decode.cuh -- the forward of the QLoRA layer for a handful of tokens
// (M <= 16): h = x W~^T + bf16((alpha/r) x A^T) B^T, streaming the 4-bit
// weight once from HBM ("QLoRA Finetuner", flowchart "Quantized Base
// Inference": load 4-bit indices and 32-bit block scales, dequantise,
// multiply).
//
// The weight dominates the bytes (n*k/2 code bytes against a few KB of
// tokens), so the kernel is HBM-bound and built to keep HBM busy:
//   * every warp owns 16 weight rows x a quarter of k and streams their codes
//     with 8-byte loads; one CTA per 32 rows, three CTAs per SM, so the whole
//     weight is covered by one wave of CTAs;
//   * a byte of codes becomes a pair of bf16 levels through a 256-entry table
//     replicated 32 times in shared memory (lane l reads copy l: no bank
//     conflicts);
//   * the 16 x 8 x 16 products run on the tensor cores (mma.sync: the
//     dequantised fragment goes straight from registers to the MMA), because
//     at 4-16 tokens the CUDA-core FMA rate would fall below the HBM rate;
//   * each 64-element block's partial product is scaled by its block scale
//     in fp32 and accumulated, so no per-element multiply by the scale.
// Numerically this forms sum_b s_b * sum_k bf16(level) * x, which differs
// from bf16(s_b * level) * x by at most one bf16 rounding of each term.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kDecRowsPerWarp = 16;
constexpr int kDecKSplit = 4;                 // warps sharing one 16-row group
constexpr int kDecRowGroups = 2;              // 16-row groups per CTA
constexpr int kDecThreads = 32 * kDecKSplit * kDecRowGroups;
constexpr int kDecRows = kDecRowsPerWarp * kDecRowGroups;
constexpr int kDecMaxRank = 64;               // LoRA rank handled by the decode kernel

struct DecodeArgs {
    int M;                 // tokens (1..16)
    int64_t N, K;          // weight rows / columns
    int r;
    const uint8_t *codes;
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    const uint16_t *x;     // [M, K]
    const uint16_t *B;     // [N, r]
    const uint16_t *u_s;   // [M, r] bf16((alpha/r) x A^T), written by the preceding kernel
    uint16_t *h;           // [M, N]
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Scale of block b, with the group constant fl32(c_g / 127) cached by the caller.
__device__ __forceinline__ float decode_scale(const DecodeArgs &a, int64_t b, int64_t &kg_group,
                                              float &kg) {
    if (!a.dq) return __ldg(a.absmax + b);
    const int64_t g = b >> 8;
    if (g != kg_group) {
        kg_group = g;
        kg = __fdiv_rn(__ldg(a.cg + g), 127.0f);
    }
    return __fmul_rn(static_cast<float>(__ldg(a.q8 + b)), kg);
}

// TG = number of 8-token groups (1 for M <= 8, 2 for M <= 16). One CTA per
// 32 weight rows: warp (rg, ks) takes 16 rows and the ks-th quarter of k.
//
// Fragment bookkeeping (m16n8k16, thread (g, t) = (lane / 4, lane % 4)):
// the A fragment holds rows g and g+8 and four k slots per row; the
// reduction order inside one MMA is free, so k slot assignments are chosen
// such that thread t's slots over the block's four MMAs are the 16
// consecutive elements [16t, 16t+16) of the block: the 8 code bytes at
// [8t, 8t+8) of each of its rows, and 16 consecutive x values per token.
template <int TG>
__global__ void __launch_bounds__(kDecThreads, 3)
qlora_decode_kernel(const DecodeArgs a) {
    __shared__ uint32_t lut[256 * 32];                              // 32 KB
    __shared__ float red[kDecRowGroups][kDecKSplit - 1][32][4 * TG];
    __shared__ __align__(16) uint16_t b_tile[kDecRows * kDecMaxRank];
    __shared__ __align__(16) uint16_t u_tile[16 * kDecMaxRank];

    // level pairs: byte b -> (bf16(level[b >> 4]) low half, bf16(level[b & 15]) high half);
    // thread b writes the 32 copies of entry b, chunk order rotated by lane so
    // that a warp's 16-byte stores spread over the banks
    {
        const int b = threadIdx.x;   // kDecThreads == 256: one entry per thread
        __nv_bfloat162 p = __floats2bfloat162_rn(c_levels[b >> 4], c_levels[b & 15]);
        const uint32_t v = *reinterpret_cast<uint32_t *>(&p);
        uint4 *dst = reinterpret_cast<uint4 *>(&lut[b * 32]);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[(c + b) & 7] = make_uint4(v, v, v, v);
    }
    // the CTA's rows of B [n, r] for the LoRA epilogue (coalesced 16-byte loads)
    {
        const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kDecRows;
        const int chunks = kDecRows * a.r / 8;
        for (int c = threadIdx.x; c < chunks; c += kDecThreads) {
            const int rr = (c * 8) / a.r, j = (c * 8) % a.r;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row0 + rr < a.N) v = __ldg(reinterpret_cast<const uint4 *>(a.B + (row0 + rr) * a.r + j));
            *reinterpret_cast<uint4 *>(b_tile + rr * a.r + j) = v;
        }
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rg = warp / kDecKSplit, ks = warp % kDecKSplit;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n_lo = static_cast<int64_t>(blockIdx.x) * kDecRows + rg * kDecRowsPerWarp + g;
    const int64_t n_hi = n_lo + 8;
    const bool v_lo = n_lo < a.N, v_hi = n_hi < a.N;
    const int64_t kblocks = a.K / kBlock;
    const int64_t kb0 = kblocks * ks / kDecKSplit, kb1 = kblocks * (ks + 1) / kDecKSplit;
    const uint8_t *c_lo = a.codes + n_lo * (a.K / 2) + 8 * t;
    const uint8_t *c_hi = a.codes + n_hi * (a.K / 2) + 8 * t;
    const uint32_t *lutl = lut + lane;

    // token rows of this thread's B fragments: g (group 0) and g + 8 (group 1)
    const uint16_t *xr[TG];
    bool xv[TG];
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
        const int m = tg * 8 + g;
        xv[tg] = m < a.M;
        xr[tg] = a.x + static_cast<int64_t>(xv[tg] ? m : 0) * a.K + 16 * t;
    }

    float acc[TG][4];
#pragma unroll
    for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[tg][e] = 0.0f;

    int64_t kgg_lo = -1, kgg_hi = -1;
    float kg_lo = 0.f, kg_hi = 0.f;

#pragma unroll 2
    for (int64_t kb = kb0; kb < kb1; ++kb) {
        // 8 code bytes per row: elements [16t, 16t+16) of the block
        uint2 wl = make_uint2(0x77777777u, 0x77777777u), wh = wl;
        if (v_lo) wl = __ldg(reinterpret_cast<const uint2 *>(c_lo + kb * 32));
        if (v_hi) wh = __ldg(reinterpret_cast<const uint2 *>(c_hi + kb * 32));
        const float s_lo = v_lo ? decode_scale(a, n_lo * kblocks + kb, kgg_lo, kg_lo) : 0.f;
        const float s_hi = v_hi ? decode_scale(a, n_hi * kblocks + kb, kgg_hi, kg_hi) : 0.f;
        // x values [16t, 16t+16) of the block for each token row
        uint4 xa[TG], xb[TG];
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) {
            if (xv[tg]) {
                xa[tg] = __ldg(reinterpret_cast<const uint4 *>(xr[tg] + kb * 64));
                xb[tg] = __ldg(reinterpret_cast<const uint4 *>(xr[tg] + kb * 64) + 1);
            } else {
                xa[tg] = make_uint4(0, 0, 0, 0);
                xb[tg] = xa[tg];
            }
        }
        const uint32_t cl[2] = {wl.x, wl.y}, chh[2] = {wh.x, wh.y};
        float part[TG][4];
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
            for (int e = 0; e < 4; ++e) part[tg][e] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // MMA i covers elements 16t + 4i + {0,1} (slots 2t, 2t+1) and
            // 16t + 4i + {2,3} (slots 2t+8, 2t+9): code bytes 2i and 2i+1
            const uint32_t bl0 = (cl[i >> 1] >> (16 * (i & 1))) & 0xFFu;
            const uint32_t bl1 = (cl[i >> 1] >> (16 * (i & 1) + 8)) & 0xFFu;
            const uint32_t bh0 = (chh[i >> 1] >> (16 * (i & 1))) & 0xFFu;
            const uint32_t bh1 = (chh[i >> 1] >> (16 * (i & 1) + 8)) & 0xFFu;
            uint32_t af[4];
            af[0] = lutl[bl0 * 32];
            af[1] = lutl[bh0 * 32];
            af[2] = lutl[bl1 * 32];
            af[3] = lutl[bh1 * 32];
#pragma unroll
            for (int tg = 0; tg < TG; ++tg) {
                const uint4 &q = (i < 2) ? xa[tg] : xb[tg];
                const uint32_t b0 = (i & 1) ? q.z : q.x;
                const uint32_t b1 = (i & 1) ? q.w : q.y;
                mma_bf16_16816(part[tg], af, b0, b1);
            }
        }
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) {
            acc[tg][0] = fmaf(s_lo, part[tg][0], acc[tg][0]);
            acc[tg][1] = fmaf(s_lo, part[tg][1], acc[tg][1]);
            acc[tg][2] = fmaf(s_hi, part[tg][2], acc[tg][2]);
            acc[tg][3] = fmaf(s_hi, part[tg][3], acc[tg][3]);
        }
    }

    // reduce the k quarters of each row group in a fixed order (0 + 1 + 2 + 3)
    if (ks > 0) {
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
            for (int e = 0; e < 4; ++e) red[rg][ks - 1][lane][4 * tg + e] = acc[tg][e];
    }
    __syncthreads();
    if (ks != 0) return;
#pragma unroll
    for (int s = 0; s < kDecKSplit - 1; ++s)
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[tg][e] += red[rg][s][lane][4 * tg + e];

    // LoRA up-projection: needs bf16((alpha/r) x A^T) from the preceding kernel
    griddep_wait();
    griddep_launch_dependents();
    {
        const int chunks = a.M * a.r / 8;
        for (int c = lane; c < chunks; c += 32)
            *reinterpret_cast<uint4 *>(u_tile + c * 8) =
                *reinterpret_cast<const uint4 *>(a.u_s + c * 8);
    }
    __syncwarp();
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = tg * 8 + 2 * t + (e & 1);
            const int rloc = rg * kDecRowsPerWarp + g + (e < 2 ? 0 : 8);
            const int64_t n = (e < 2) ? n_lo : n_hi;
            if (m >= a.M || n >= a.N) continue;
            float l = 0.0f;
            const uint16_t *br = b_tile + rloc * a.r;
            const uint16_t *ur = u_tile + m * a.r;
            for (int j = 0; j < a.r; j += 8) {
                const uint4 bv = *reinterpret_cast<const uint4 *>(br + j);
                const uint4 uv = *reinterpret_cast<const uint4 *>(ur + j);
                const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    l = fmaf(__uint_as_float(bw[q] << 16), __uint_as_float(uw[q] << 16), l);
                    l = fmaf(__uint_as_float(bw[q] & 0xFFFF0000u), __uint_as_float(uw[q] & 0xFFFF0000u), l);
                }
            }
            __nv_bfloat16 hv = __float2bfloat16_rn(acc[tg][e] + l);
            a.h[static_cast<int64_t>(m) * a.N + n] = *reinterpret_cast<uint16_t *>(&hv);
        }
    }
}

// u = x A^T for a few tokens (M <= 16): one CTA per rank column j, threads
// split k, fixed-order reduction; writes u (fp32, optional) and
// bf16(scale * u). Lets the decode kernel that follows start right away.
constexpr int kDecUThreads = 256;

__global__ void __launch_bounds__(kDecUThreads)
decode_lora_u_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ A, int M,
                     int64_t K, int r, float scale, float *__restrict__ u_out,
                     uint16_t *__restrict__ u_s) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float red[kDecUThreads / 32][16];
    const int j = blockIdx.x;
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = 0.0f;
    const uint16_t *ar = A + static_cast<int64_t>(j) * K;
    for (int64_t k = 8 * threadIdx.x; k < K; k += 8 * kDecUThreads) {
        const uint4 av = __ldg(reinterpret_cast<const uint4 *>(ar + k));
        const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            if (m >= M) break;
            const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + m * K + k));
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[m] = fmaf(__uint_as_float(aw[q] << 16), __uint_as_float(xw[q] << 16), acc[m]);
                acc[m] = fmaf(__uint_as_float(aw[q] & 0xFFFF0000u), __uint_as_float(xw[q] & 0xFFFF0000u), acc[m]);
            }
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        float v = acc[m];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][m] = v;
    }
    __syncthreads();
    if (threadIdx.x < M) {
        const int m = threadIdx.x;
        float v = 0.0f;
        for (int w = 0; w < kDecUThreads / 32; ++w) v += red[w][m];
        if (u_out) u_out[static_cast<int64_t>(m) * r + j] = v;
        __nv_bfloat16 b = __float2bfloat16_rn(scale * v);
        u_s[static_cast<int64_t>(m) * r + j] = *reinterpret_cast<uint16_t *>(&b);
    }
}

}  // namespace nf4
