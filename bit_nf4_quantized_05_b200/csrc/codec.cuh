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

// One CTA per group of 256 blocks (16384 weights). Each half-warp owns one
// block per step: 16 lanes x 4 consecutive fp32 = 64 elements, loaded as
// float4 so that a warp reads 512 contiguous bytes. The 15 decision
// thresholds are the level midpoints rounded toward -inf in fp32, so that
// `w' > t_i` holds exactly when w' is above the exact midpoint: a value on a
// midpoint falls to the lower level.
constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
nf4_quantize_kernel(const float *__restrict__ W, int64_t nb, int dq, uint8_t *__restrict__ codes,
                    float *__restrict__ absmax, uint8_t *__restrict__ q8, float *__restrict__ cg) {
    __shared__ float s_abs[kGroup];
    __shared__ float s_red[kQuantThreads / 32];

    float t[15];
#pragma unroll
    for (int i = 0; i < 15; ++i)
        t[i] = __double2float_rd((static_cast<double>(c_levels[i]) +
                                  static_cast<double>(c_levels[i + 1])) * 0.5);

    const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kGroup;
    const int nblk = (nb - b0 < kGroup) ? static_cast<int>(nb - b0) : kGroup;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    // the two half-warps may take different branches below (odd block counts)
    const unsigned hmask = half ? 0xffff0000u : 0x0000ffffu;
    bool bad = false;

    for (int j = warp * 2 + half; j < kGroup; j += (kQuantThreads / 32) * 2) {
        if (j >= nblk) {
            if (hl == 0) s_abs[j] = 0.0f;
            continue;
        }
        const int64_t b = b0 + j;
        const float4 v = __ldg(reinterpret_cast<const float4 *>(W + b * kBlock) + hl);
        bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
        float s = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) s = fmaxf(s, __shfl_xor_sync(hmask, s, o));
        const float e[4] = {v.x, v.y, v.z, v.w};
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (s == 0.0f) {
                q[i] = 7;
            } else {
                const float wn = __fdiv_rn(e[i], s);
                uint32_t c = 0;
#pragma unroll
                for (int l = 0; l < 15; ++l) c += (wn > t[l]) ? 1u : 0u;
                q[i] = c;
            }
        }
        const uint16_t packed = static_cast<uint16_t>(((q[0] << 4) | q[1]) |
                                                      (((q[2] << 4) | q[3]) << 8));
        reinterpret_cast<uint16_t *>(codes + b * (kBlock / 2))[hl] = packed;
        if (hl == 0) {
            absmax[b] = s;
            s_abs[j] = s;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(NF4_ERR_NONFINITE);
    if (!dq) return;

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
    if (threadIdx.x == 0) cg[blockIdx.x] = c;
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
