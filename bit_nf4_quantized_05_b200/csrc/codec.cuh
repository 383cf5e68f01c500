// codec.cuh -- NF4 quantisation (with optional double quantisation) and
// dequantisation kernels.
//
// Quantisation follows "QLoRA Finetuner -- Juan Martos", section 2 (absmax per
// 64-element block, normalise to [-1, 1], nearest of the 16 NF4 quantiles)
// and "Parameter-Efficient Fine-Tuning: From LoRA to QLoRA", Pillar 1 (byte
// packing, first element in the high nibble) and Pillar 2 (8-bit codes for
// the scales in groups of 256 blocks, one fp32 constant per group).
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

// Scale used by dequantisation of block b (fp32 s_b, or q8_b * (c_g / 127)).
__device__ __forceinline__ float dq_block_scale(const float *absmax, const uint8_t *q8,
                                                const float *cg, int dq, int64_t b) {
    if (!dq) return __ldg(absmax + b);
    const float kg = __fdiv_rn(__ldg(cg + (b >> 8)), 127.0f);
    return __fmul_rn(static_cast<float>(__ldg(q8 + b)), kg);
}

// Quantisation. Persistent CTAs walk the groups of 256 blocks (16384
// weights); each half-warp owns one block at a time: 16 lanes x 4 consecutive
// fp32 = 64 elements, loaded as float4. Blocks are taken four at a time, and
// the next four are loaded (across group boundaries) while the current four
// are coded.
//
// The code of w is #{i : fl32(w / s) > t_i}, where the 15 decision thresholds
// t_i are the level midpoints rounded toward -inf in fp32, so that a value on
// a midpoint falls to the lower level. Instead of dividing and comparing with
// every threshold, each element forms p = fl32(w * fl32(1/s)), which differs
// from fl32(w / s) by at most 2.5 units in the last place (two roundings of
// relative size 2^-24 each, plus the half unit of the exact quotient), and
// looks up p's bucket in a table of 32 equal buckets over [-1, 1]: the table
// gives the number of thresholds below the bucket and the one threshold
// inside it (no bucket holds two, and no threshold lies within 1/1024 of a
// bucket boundary, so a bucket misplaced by rounding gives the same count).
// The table is held in 32 copies, one per lane, so the data-dependent lookups
// of a warp never collide on a shared-memory bank.
// When p is within kQuantGuard of that threshold the element falls back to
// the exact quotient and the full comparison.
constexpr int kQuantThreads = 256;
constexpr int kQuantBuckets = 32;
constexpr float kQuantGuard = 4.76837158203125e-07f;   // 2^-21 > 2.5 ulp of any |p| <= 1

constexpr int kQuantCtasPerSm = 3;

__global__ void __launch_bounds__(kQuantThreads, kQuantCtasPerSm)
nf4_quantize_kernel(const float *__restrict__ W, int64_t nb, int dq, uint8_t *__restrict__ codes,
                    float *__restrict__ absmax, uint8_t *__restrict__ q8, float *__restrict__ cg) {
    __shared__ float s_abs[kGroup];
    __shared__ float s_red[kQuantThreads / 32];
    __shared__ float s_t[16];
    __shared__ float2 s_tab[kQuantBuckets * 32];   // [bucket][lane copy]: {threshold inside or +inf, count below}

    if (threadIdx.x < 15)
        s_t[threadIdx.x] = __double2float_rd((static_cast<double>(c_levels[threadIdx.x]) +
                                              static_cast<double>(c_levels[threadIdx.x + 1])) * 0.5);
    __syncthreads();
    for (int idx = threadIdx.x; idx < kQuantBuckets * 32; idx += kQuantThreads) {
        const int bkt = idx >> 5;
        const float lo = -1.0f + static_cast<float>(bkt) * (2.0f / kQuantBuckets);   // exact
        const float hi = -1.0f + static_cast<float>(bkt + 1) * (2.0f / kQuantBuckets);
        int below = 0;
        float inside = __int_as_float(0x7f800000);   // +inf: no threshold in this bucket
#pragma unroll
        for (int i = 0; i < 15; ++i) {
            if (s_t[i] < lo) ++below;
            else if (s_t[i] < hi) inside = s_t[i];
        }
        s_tab[idx] = make_float2(inside, __int_as_float(below));
    }
    float t[15];
#pragma unroll
    for (int i = 0; i < 15; ++i) t[i] = s_t[i];
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    const int hw = warp * 2 + half;                 // half-warp 0..15
    // the two half-warps may take different branches below (ragged last group)
    const unsigned hmask = half ? 0xffff0000u : 0x0000ffffu;
    const int64_t ngroups = (nb + kGroup - 1) / kGroup;
    bool bad = false;

    static_assert(kQuantBuckets == 32, "bucket = top 5 mantissa bits of p + 3");
    auto code_of = [&](float e, float s, float inv) -> uint32_t {
        const float p = __fmul_rn(e, inv);
        // p + 3 lies in [2, 4) (clamped), where the exponent is fixed and the
        // top five mantissa bits are floor(16 (p + 1)); its rounding (2^-22)
        // is far below the distance of any threshold from a bucket boundary
        const float p3 = fminf(fmaxf(p + 3.0f, 2.0f), 3.99999976f);
        const uint32_t bkt = (__float_as_uint(p3) >> 18) & 31u;
        const float2 tb = s_tab[bkt * 32 + lane];
        if (fabsf(p - tb.x) > kQuantGuard)
            return static_cast<uint32_t>(__float_as_int(tb.y)) + (p > tb.x ? 1u : 0u);
        // within the guard of a threshold: the exact quotient decides
        const float wn = __fdiv_rn(e, s);
        uint32_t c = 0;
#pragma unroll
        for (int l = 0; l < 15; ++l) c += (wn > t[l]) ? 1u : 0u;
        return c;
    };

    // the half-warp's quads of blocks in order: (group g, first block j0 = hw + 64 k), k = 0..3
    auto load_quad = [&](int64_t g, int j0, float4 (&v)[4]) {
        const int64_t b0 = g * kGroup;
        const int nblk = g < ngroups ? ((nb - b0 < kGroup) ? static_cast<int>(nb - b0) : kGroup) : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 16 * u;
            v[u] = j < nblk ? __ldg(reinterpret_cast<const float4 *>(W + (b0 + j) * kBlock) + hl)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    float4 nxt[4];
    load_quad(blockIdx.x, hw, nxt);
    for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
        const int64_t b0 = g * kGroup;
        const int nblk = (nb - b0 < kGroup) ? static_cast<int>(nb - b0) : kGroup;
#pragma unroll 1
        for (int j0 = hw; j0 < kGroup; j0 += 4 * 16) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = nxt[u];
            if (j0 + 64 < kGroup) load_quad(g, j0 + 64, nxt);
            else load_quad(g + gridDim.x, hw, nxt);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + 16 * u;
                if (j >= nblk) {
                    if (hl == 0) s_abs[j] = 0.0f;
                    continue;
                }
                const int64_t b = b0 + j;
                // absmax as the integer max of |w|'s bit patterns: the order of
                // non-negative floats, with NaN above +inf, so one compare per
                // block flags any non-finite element
                uint32_t sb = max(max(__float_as_uint(v[u].x) & 0x7fffffffu, __float_as_uint(v[u].y) & 0x7fffffffu),
                                  max(__float_as_uint(v[u].z) & 0x7fffffffu, __float_as_uint(v[u].w) & 0x7fffffffu));
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) sb = max(sb, __shfl_xor_sync(hmask, sb, o));
                bad |= sb >= 0x7f800000u;
                const float s = __uint_as_float(sb);
                uint32_t q[4] = {7u, 7u, 7u, 7u};
                if (s != 0.0f) {
                    const float inv = __frcp_rn(s);
                    q[0] = code_of(v[u].x, s, inv);
                    q[1] = code_of(v[u].y, s, inv);
                    q[2] = code_of(v[u].z, s, inv);
                    q[3] = code_of(v[u].w, s, inv);
                }
                const uint16_t packed = static_cast<uint16_t>(((q[0] << 4) | q[1]) |
                                                              (((q[2] << 4) | q[3]) << 8));
                reinterpret_cast<uint16_t *>(codes + b * (kBlock / 2))[hl] = packed;
                if (hl == 0) {
                    absmax[b] = s;
                    s_abs[j] = s;
                }
            }
        }
        if (dq) {
            __syncthreads();
            // group constant c_g = max of the block scales of this group
            float m = s_abs[threadIdx.x];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) s_red[warp] = m;
            __syncthreads();
            float c = s_red[0];
#pragma unroll
            for (int i = 1; i < kQuantThreads / 32; ++i) c = fmaxf(c, s_red[i]);
            const int j = threadIdx.x;
            if (j < nblk) {
                uint8_t code = 0;
                if (c > 0.0f) {
                    // fl32(fl32(s / c) * 127), rounded half to even
                    const float ratio = __fdiv_rn(s_abs[j], c);
                    code = static_cast<uint8_t>(__float2int_rn(__fmul_rn(ratio, 127.0f)));
                }
                q8[b0 + j] = code;
            }
            if (threadIdx.x == 0) cg[g] = c;
        }
        __syncthreads();      // s_abs is reused by the next group
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(NF4_ERR_NONFINITE);
}

// Dequantisation, one thread per 64-element block.
//   bf16 output: per-block register lookup table (the same routine that
//   produces the tensor-core operand in the fused matmuls).
//   fp32 output: fl32(scale * level) per element.
__global__ void __launch_bounds__(256)
nf4_dequantize_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ absmax,
                      const uint8_t *__restrict__ q8, const float *__restrict__ cg, int dq,
                      int64_t nb, int out_bf16, void *__restrict__ out) {
    for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < nb;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float s = dq_block_scale(absmax, q8, cg, dq, b);
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + b * (kBlock / 2));
        const uint4 c0 = __ldg(src), c1 = __ldg(src + 1);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        if (out_bf16) {
            const BlockLut L = make_block_lut(s);
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + b * kBlock);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t o[4];
                dequant8(L, words[i], o);
                dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        } else {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + b * kBlock);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t w = words[i];
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t byte = (w >> (8 * e)) & 0xFFu;
                    f[2 * e] = __fmul_rn(s, c_levels[byte >> 4]);
                    f[2 * e + 1] = __fmul_rn(s, c_levels[byte & 15u]);
                }
                dst[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
                dst[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
    }
}

}  // namespace nf4
