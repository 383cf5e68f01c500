// codec.cuh -- NF4 quantisation (with optional double quantisation) and
// dequantisation kernels.
//
// Quantisation follows "QLoRA Finetuner -- Juan Martos", section 2 (absmax per
// 64-element block, normalise to [-1, 1], nearest of the 16 NF4 quantiles)
// and "Parameter-Efficient Fine-Tuning: From LoRA to QLoRA", Pillar 1 (byte
// packing, first element in the high nibble) and Pillar 2 (8-bit codes for
// the scales in groups of 256 blocks, one fp32 constant per group).
#pragma once

#include <cuda_fp16.h>

#include "nf4_common.cuh"

namespace nf4 {

// Scale used by dequantisation of block b (fp32 s_b, or q8_b * (c_g / 127)).
__device__ __forceinline__ float dq_block_scale(const float *absmax, const uint8_t *q8,
                                                const float *cg, int dq, int64_t b) {
    if (!dq) return __ldg(absmax + b);
    const float kg = __fdiv_rn(__ldg(cg + (b >> 8)), 127.0f);
    return __fmul_rn(static_cast<float>(__ldg(q8 + b)), kg);
}

// Quantisation. Persistent CTAs (two per SM) walk the groups of 256 blocks
// (16384 weights, 64 KB of fp32). A producer lane streams each group into
// shared memory by TMA, a quarter group (64 blocks, 16 KB) per stage through
// a ring of kQzStages stages, with the 128-byte swizzle. Eight consumer warps
// code a stage: four lanes per 64-element block (eight per 128-element
// block), each lane 16 consecutive elements (elements [16q, 16q + 16) of its
// block), read as 16-byte pieces whose swizzled addresses fall on eight
// distinct bank groups in every quarter warp. The absmax is an integer max
// over |w|'s bit patterns (NaN above +inf, so one compare flags any
// non-finite block), then shuffles across the block's lanes.
//
// The code of w is #{i : fl32(w / s) > t_i}, where the 15 decision thresholds
// t_i are the level midpoints rounded toward -inf in fp32, so that a value on
// a midpoint falls to the lower level. Instead of dividing and comparing with
// every threshold, each element forms p = fl32(w * rcp(s)) with the hardware
// reciprocal (at most 1 ulp from 1/s), so that |p - fl32(w / s)| <= 2.4e-7 for
// |w| <= s, and looks up p's bucket in a table of 32 equal buckets over
// [-1, 1] plus one on either side: the table gives the number of thresholds
// below the bucket and the one threshold inside it (no bucket holds two, and
// no threshold lies within 1/1024 of a bucket boundary, so a bucket misplaced
// by the rounding of p + 3 gives the same count). The bucket is read from bits
// 18..23 of fl32(p + 3) (masked, so every bit pattern addresses the table);
// the table is held in 32 copies, one per lane, so data-dependent lookups
// never collide on a bank.
// When p is within kQuantGuard (2^-21) of that threshold, or s is so small or
// large that its reciprocal loses precision, the lane recomputes its 16 codes
// from the exact quotient and the full comparison.
constexpr int kQzConsumerWarps = 8;
constexpr int kQzThreads = 32 * (kQzConsumerWarps + 1);   // the last warp issues the TMA copies
constexpr int kQzStages = 5;
constexpr int kQzStageElems = 4096;                        // a stage: 64 blocks of 64 or 32 of 128
constexpr int kQzStageBytes = kQzStageElems * 4;            // 16 KB: one stage slot (fp32 fills it)

// Element type of W0: fp32, or a 16-bit type converted exactly to fp32 on
// load ("QLoRA explained", section "The quantization backbone": weights are
// quantised from 16-bit FP16/BF16). A 16-bit block is one 128-byte row.
enum QzKind { kQzF32 = 0, kQzBF16 = 1, kQzF16 = 2 };
constexpr int kQzTabRows = 64;                              // bits 18..23 of fl32(p + 3)
constexpr int kQzCtasPerSm = 2;
constexpr int kQzTabOff = kQzStages * kQzStageBytes;                // float2 [34][32]
constexpr int kQzAbsOff = kQzTabOff + kQzTabRows * 32 * 8;          // float [2][256]
constexpr int kQzBarOff = kQzAbsOff + 2 * kGroup * 4;               // full, empty, group
constexpr int kQzSmemBytes = kQzBarOff + (2 * kQzStages + 2) * 8 + 16 + 1024;
constexpr float kQuantGuard = 4.76837158203125e-07f;   // 2^-21 > 2.4e-7 bound on |p - fl32(w/s)|
static_assert(kQzConsumerWarps * 32 == kGroup, "one consumer thread per block of a group");
static_assert(kQzStageElems == kQzConsumerWarps * 32 * 16, "16 elements per consumer lane and stage");

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
    float2 v;
    asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Exact code of one element: the quotient rounded once, compared with every
// threshold.
__device__ __forceinline__ uint32_t nf4_code_exact(float w, float s, const float (&t)[15]) {
    const float wn = __fdiv_rn(w, s);
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < 15; ++i) c += (wn > t[i]) ? 1u : 0u;
    return c;
}

// tm_w views W0 as 128-byte rows: fp32 [numel / 32, 32] with box {32, 128},
// or 16-bit [numel / 64, 64] with box {64, 64}; either way a stage is 4096
// elements. BS (64 or 128) elements per block: BS / 16 lanes code a block.
template <int KIND, int BS>
__global__ void __launch_bounds__(kQzThreads, kQzCtasPerSm)
nf4_quantize_kernel(const __grid_constant__ CUtensorMap tm_w,
                    int64_t nb, int dq, uint8_t *__restrict__ codes, float *__restrict__ absmax,
                    uint8_t *__restrict__ q8, float *__restrict__ cg) {
    extern __shared__ uint8_t qsm_raw[];
    uint8_t *qsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(qsm_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    float2 *tab = reinterpret_cast<float2 *>(qsm + kQzTabOff);
    float *s_abs = reinterpret_cast<float *>(qsm + kQzAbsOff);
    uint64_t *full = reinterpret_cast<uint64_t *>(qsm + kQzBarOff);
    uint64_t *empty = full + kQzStages;
    uint64_t *grp = empty + kQzStages;                 // [2] all consumer warps done with a group
    volatile int *abort_flag = reinterpret_cast<volatile int *>(grp + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // thresholds: the exact (fp64) midpoints of adjacent levels, rounded toward -inf
    float t[15];
#pragma unroll
    for (int i = 0; i < 15; ++i)
        t[i] = __double2float_rd((static_cast<double>(c_levels[i]) + static_cast<double>(c_levels[i + 1])) * 0.5);
    for (int idx = threadIdx.x; idx < kQzTabRows * 32; idx += kQzThreads) {
        // Row i holds bucket k = min((i + 1) mod 64, 33) of p. For |p| <= 1 + 2^-22,
        // fl32(p + 3) lies in [2 - 2^-22, 4]; its bits 18..23 are 63 below 2
        // (bucket 0: everything below -1), 0..31 on [2, 4) (bucket k = 1..32:
        // p in [-1 + (k - 1) / 16, -1 + k / 16)) and 32 at 4 (bucket 33:
        // everything from 1 up). Rows 33..62 are never addressed.
        const int k = min(((idx >> 5) + 1) & 63, 33);
        const float inf = __int_as_float(0x7f800000);
        const float lo = k == 0 ? -inf : -1.0f + static_cast<float>(k - 1) * 0.0625f;
        const float hi = k == 33 ? inf : -1.0f + static_cast<float>(k) * 0.0625f;
        int below = 0;
        float inside = inf;
#pragma unroll
        for (int i = 0; i < 15; ++i) {
            if (t[i] < lo) ++below;
            else if (t[i] < hi) inside = t[i];
        }
        tab[idx] = make_float2(inside, __int_as_float(below));
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kQzStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kQzConsumerWarps);
        }
        mbar_init(&grp[0], kQzConsumerWarps);
        mbar_init(&grp[1], kQzConsumerWarps);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_w);
    }
    __syncthreads();

    constexpr int kLanes = BS / 16;                  // lanes per block
    constexpr int kStageBlocks = kQzStageElems / BS;
    constexpr int kRowsPerBlock = KIND == kQzF32 ? BS / 32 : BS / 64;   // 128-byte rows
    const int64_t ngroups = (nb + kGroup - 1) / kGroup;
    if (warp == kQzConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int n = 0;
            for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
                for (int qq = 0; qq < kGroup / kStageBlocks; ++qq) {
                    const int64_t b0 = g * kGroup + qq * kStageBlocks;
                    if (b0 >= nb) break;
                    const int s = n % kQzStages;
                    const uint32_t ph = static_cast<uint32_t>(n / kQzStages) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) goto drain;
                    mbar_arrive_expect_tx(&full[s], KIND == kQzF32 ? kQzStageBytes : kQzStageBytes / 2);
                    tma_load_2d(qsm + s * kQzStageBytes, &tm_w, &full[s], 0,
                                static_cast<int32_t>(kRowsPerBlock * b0));
                    ++n;
                }
            }
        drain:
            // every copy issued has landed before the CTA's memory is released
            for (int m = n - kQzStages > 0 ? n - kQzStages : 0; m < n; ++m)
                mbar_drain(&full[m % kQzStages], static_cast<uint32_t>(m / kQzStages) & 1u);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int bq = lane / kLanes;                // block of this lane among the warp's 32 / kLanes
    const int q = lane % kLanes;                 // elements [16q, 16q + 16) of that block
    const int lb = warp * (32 / kLanes) + bq;    // block within a stage
    // 128-byte row within the stage, and the 16-byte pieces of the lane's
    // elements: an fp32 row holds 32 elements (two lanes), a 16-bit row 64
    // (four lanes). In every quarter warp the eight lanes' pieces fall on
    // eight distinct 16-byte bank groups after the swizzle.
    const int row = KIND == kQzF32 ? kRowsPerBlock * lb + (q >> 1) : kRowsPerBlock * lb + (q >> 2);
    constexpr int kPieces = KIND == kQzF32 ? 4 : 2;
    uint32_t off[kPieces];
#pragma unroll
    for (int j = 0; j < kPieces; ++j) {
        const int piece = KIND == kQzF32 ? 4 * (q & 1) + j : 2 * (q & 3) + j;
        off[j] = static_cast<uint32_t>(row * 128 + ((piece ^ (row & 7)) << 4));
    }
    const uint32_t mytab = smem_u32(tab) + 8u * lane;
    bool bad = false;
    int n = 0, gi = 0;
    for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x, ++gi) {
        float *sa = s_abs + (gi & 1) * kGroup;
        for (int qq = 0; qq < kGroup / kStageBlocks; ++qq) {
            const int64_t b0 = g * kGroup + qq * kStageBlocks;
            if (b0 >= nb) break;
            const int s = n % kQzStages;
            const uint32_t ph = static_cast<uint32_t>(n / kQzStages) & 1u;
            ++n;
            if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
            const uint8_t *st = qsm + s * kQzStageBytes;
            float x[16];
            if constexpr (KIND == kQzF32) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 v = *reinterpret_cast<const float4 *>(st + off[j]);
                    x[4 * j] = v.x;
                    x[4 * j + 1] = v.y;
                    x[4 * j + 2] = v.z;
                    x[4 * j + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(st + off[j]);
                    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if constexpr (KIND == kQzBF16) {
                            // a bf16 value is the upper half of its fp32 value
                            x[8 * j + 2 * e] = __uint_as_float(wd[e] << 16);
                            x[8 * j + 2 * e + 1] = __uint_as_float(wd[e] & 0xffff0000u);
                        } else {
                            x[8 * j + 2 * e] = __half2float(__ushort_as_half(static_cast<unsigned short>(wd[e] & 0xffffu)));
                            x[8 * j + 2 * e + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(wd[e] >> 16)));
                        }
                    }
                }
            }
            // |w| bit patterns, reduced as a tree
            uint32_t mm[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                mm[e] = max(__float_as_uint(x[e]) & 0x7fffffffu, __float_as_uint(x[e + 8]) & 0x7fffffffu);
#pragma unroll
            for (int e = 0; e < 4; ++e) mm[e] = max(mm[e], mm[e + 4]);
            uint32_t m = max(max(mm[0], mm[1]), max(mm[2], mm[3]));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if constexpr (kLanes == 8) m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
            const float sc = __uint_as_float(m);
            uint32_t c[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) c[e] = 7u;          // all-zero block: the exact zero level
            if (m >= 0x7f800000u) {
                bad = true;                                  // non-finite input: codes unspecified
            } else if (m != 0u) {
                // a reciprocal of s this small or large loses precision: exact path
                bool near = !(sc >= 0x1p-125f && sc <= 0x1p125f);
                if (!near) {
                    const float inv = rcp_approx(sc);
                    float dmin = 1.0f;           // smallest distance of p to its bucket's threshold
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p = x[e] * inv;
                        const uint32_t row = (__float_as_uint(p + 3.0f) >> 10) & 0x3F00u;   // 256 bytes per row
                        const float2 te = lds_f2(mytab + row);
                        const float d = p - te.x;
                        c[e] = static_cast<uint32_t>(__float_as_int(te.y)) + (d > 0.0f ? 1u : 0u);
                        dmin = fminf(dmin, fabsf(d));
                    }
                    near = dmin <= kQuantGuard;
                }
                if (near) {
                    // some element lies within the guard of its threshold: the
                    // exact quotient decides all sixteen (rare)
#pragma unroll
                    for (int e = 0; e < 16; ++e) c[e] = nf4_code_exact(x[e], sc, t);
                }
            }
            // byte j of the lane's 8: element 2j in the high nibble, 2j + 1 in the low
            uint32_t w0 = 0, w1 = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w0 |= ((c[2 * j] << 4) | c[2 * j + 1]) << (8 * j);
                w1 |= ((c[8 + 2 * j] << 4) | c[8 + 2 * j + 1]) << (8 * j);
            }
            const int64_t b = b0 + lb;
            if (b < nb) {
                *reinterpret_cast<uint2 *>(codes + b * (BS / 2) + 8 * q) = make_uint2(w0, w1);
                if (q == 0) absmax[b] = sc;
            }
            if (q == 0) sa[qq * kStageBlocks + lb] = sc;
            // the stage's values are consumed (the stores above depend on all of them)
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (dq) {
            // double quantisation of this group's 256 scales: every consumer
            // warp has written its scales before the group barrier completes
            __syncwarp();
            if (lane == 0) mbar_arrive(&grp[gi & 1]);
            if (!mbar_wait(&grp[gi & 1], static_cast<uint32_t>(gi >> 1) & 1u, abort_flag)) goto done;
            const int64_t gb = g * kGroup;
            float cmax = 0.0f;
#pragma unroll
            for (int k = 0; k < kGroup / 32; ++k)
                if (gb + lane + 32 * k < nb) cmax = fmaxf(cmax, sa[lane + 32 * k]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
            const int j = warp * 32 + lane;
            if (gb + j < nb) {
                uint8_t code = 0;
                if (cmax > 0.0f) {
                    // fl32(fl32(s / c) * 127), rounded half to even
                    const float ratio = __fdiv_rn(sa[j], cmax);
                    code = static_cast<uint8_t>(__float2int_rn(__fmul_rn(ratio, 127.0f)));
                }
                q8[gb + j] = code;
            }
            if (warp == 0 && lane == 0) cg[g] = cmax;
        }
    }
done:
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(NF4_ERR_NONFINITE);
}

// Dequantisation, one thread per 64 elements (a block, or half of a
// 128-element block: scale index b >> bshift).
//   bf16 output: per-block register lookup table (the same routine that
//   produces the tensor-core operand in the fused matmuls).
//   fp32 output: fl32(scale * level) per element.
__global__ void __launch_bounds__(256)
nf4_dequantize_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ absmax,
                      const uint8_t *__restrict__ q8, const float *__restrict__ cg, int dq,
                      int64_t nb, int bshift, int out_bf16, void *__restrict__ out) {
    for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < nb;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float s = dq_block_scale(absmax, q8, cg, dq, b >> bshift);
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
