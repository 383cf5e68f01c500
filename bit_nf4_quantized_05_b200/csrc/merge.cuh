// merge.cuh -- the adapters folded into the frozen weight for inference
// without adapters ("QLoRA explained: fine-tuning in 4-bit precision",
// section "Merging and deploying"; "How Fine-Tuning LLMs with LoRA and QLoRA
// Works", FAQ on merging: W_new = W + (alpha/r) B A):
//
//     out[n][k] = w~[n][k] + s * sum_j B[n][j] A[j][k],   s = fl32(alpha / r)
//
// with w~ = fl32(scale * NF4[q]) the dequantised base weight in fp32. The
// rank-r product is accumulated in fp32 on the tensor cores (mma.sync
// fragments; r <= 128, zero-padded to a multiple of 16), then one fused
// multiply-add with w~ and one rounding to the output type (bf16 for the
// 16-bit merged model, fp32 for re-quantisation with nf4_quantize).
//
// A CTA owns one 128-column stripe of out and walks its 64-row tiles (every
// gridDim.y-th): the stripe's columns of A (stored transposed, so that each
// MMA's B fragment is one 32-bit word) are staged once, and the next tile's
// rows of B and 4-bit codes arrive by cp.async while the current tile is
// computed (two buffers). Warp w takes rows [16 (w % 4), +16) and the 64
// columns (one NF4 block per row) [64 (w / 4), +64) of a tile; each warp's
// results go through a padded shared buffer so that every row leaves as
// 16-byte stores.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kMgRows = 64;
constexpr int kMgCols = 128;
constexpr int kMgThreads = 256;
constexpr int kMgMaxRank = 128;
constexpr int kMgCodeStride = 80;    // bytes per staged code row (64 used; padded against bank conflicts)

struct MergeArgs {
    int64_t N, K;
    int r, rp;                 // rank and rank padded to a multiple of 16
    const uint8_t *codes;
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    const uint16_t *A;         // [r, K]
    const uint16_t *B;         // [N, r]
    float scale;               // fl32(alpha / r)
    void *out;                 // [N, K] bf16 or fp32
    int block;                 // elements per NF4 block (64 or 128)
};

// Shared-memory layout of one CTA (bytes), for padded rank rp.
__host__ __device__ constexpr int merge_bs_stride(int rp) { return rp + 8; }    // bf16 per B row
__host__ __device__ inline int merge_smem_bytes(int rp, bool out_bf16) {
    return kMgCols * merge_bs_stride(rp) * 2          // A columns (transposed)
           + 2 * kMgRows * merge_bs_stride(rp) * 2    // B rows, two buffers
           + 2 * kMgRows * kMgCodeStride              // codes, two buffers
           + 16 * 4                                   // levels
           + 8 * 16 * (out_bf16 ? (64 + 8) * 2 : (64 + 4) * 4);   // per-warp output staging
}
// RQ = padded rank / 16 (1..8), a compile-time constant so that the rank
// loops unroll without guards.
template <bool OUT_BF16, int RQ>
__global__ void __launch_bounds__(kMgThreads, 4) qlora_merge_kernel(const MergeArgs a) {
    extern __shared__ __align__(16) uint8_t msm[];
    constexpr int rs = merge_bs_stride(16 * RQ);
    uint16_t *Ats = reinterpret_cast<uint16_t *>(msm);                      // [128][rs]
    uint16_t *Bs2 = Ats + kMgCols * rs;                                     // [2][64][rs]
    uint8_t *cs2 = reinterpret_cast<uint8_t *>(Bs2 + 2 * kMgRows * rs);     // [2][64][kMgCodeStride]
    float *lv = reinterpret_cast<float *>(cs2 + 2 * kMgRows * kMgCodeStride);    // [16]
    uint8_t *stage = reinterpret_cast<uint8_t *>(lv + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kMgCols;
    const int row_tiles = static_cast<int>((a.N + kMgRows - 1) / kMgRows);

    griddep_wait();
    griddep_launch_dependents();

    // tile rt's rows of B (zero beyond N and r) and codes into buffer buf
    auto prefetch = [&](int rt, int buf) {
        const int64_t n0 = static_cast<int64_t>(rt) * kMgRows;
        uint16_t *Bs = Bs2 + buf * kMgRows * rs;
        for (int idx = tid; idx < kMgRows * (a.rp / 8); idx += kMgThreads) {
            const int row = idx / (a.rp / 8), ch = idx % (a.rp / 8);
            const bool ok = n0 + row < a.N && ch * 8 < a.r;
            cp_async16(Bs + row * rs + ch * 8, ok ? a.B + (n0 + row) * a.r + ch * 8 : a.B, ok);
        }
        {
            const int row = tid >> 2, ch = tid & 3;
            const bool ok = n0 + row < a.N && k0 + ch * 32 < a.K;
            cp_async16(cs2 + buf * kMgRows * kMgCodeStride + row * kMgCodeStride + ch * 16,
                       ok ? a.codes + (n0 + row) * (a.K / 2) + k0 / 2 + ch * 16 : a.codes, ok);
        }
        cp_async_commit();
    };
    int rt = static_cast<int>(blockIdx.y);
    if (rt < row_tiles) prefetch(rt, 0);

    if (tid < 16) lv[tid] = c_levels[tid];
    // A columns k0..k0+127 as rows of Ats (Ats[c][j] = A[j][k0 + c]), zero beyond K and r;
    // consecutive threads take consecutive j, so each 16-bit store of a warp
    // lands on consecutive addresses
    for (int idx = tid; idx < a.rp * (kMgCols / 8); idx += kMgThreads) {
        const int j = idx % a.rp, ch = idx / a.rp;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (j < a.r && k0 + ch * 8 < a.K)
            v = __ldg(reinterpret_cast<const uint4 *>(a.A + static_cast<int64_t>(j) * a.K + k0) + ch);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            Ats[(ch * 8 + e) * rs + j] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
    }

    const int rw = 16 * (warp & 3);          // first tile row of this warp
    const int cw = 64 * (warp >> 2);         // first tile column of this warp
    const bool cols_ok = k0 + cw < a.K;      // K is a multiple of 64: a warp's block is all in or all out
    uint8_t *st = stage + warp * 16 * (OUT_BF16 ? (64 + 8) * 2 : (64 + 4) * 4);

    for (int buf = 0; rt < row_tiles; rt += static_cast<int>(gridDim.y), buf ^= 1) {
        // this tile's rows of B and codes have landed (the only copies in
        // flight), and every warp is done with the previous tile and its
        // buffer, which takes the next tile now
        cp_async_wait_all();
        __syncthreads();
        if (rt + static_cast<int>(gridDim.y) < row_tiles) prefetch(rt + static_cast<int>(gridDim.y), buf ^ 1);
        const int64_t n0 = static_cast<int64_t>(rt) * kMgRows;
        const uint16_t *Bs = Bs2 + buf * kMgRows * rs;
        const uint8_t *cs = cs2 + buf * kMgRows * kMgCodeStride;

        // block scales of rows rw + g and rw + g + 8 (a warp's 64 columns lie in one block)
        float sc[2] = {0.0f, 0.0f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t n = n0 + rw + g + 8 * h;
            if (n < a.N && cols_ok) {
                const int64_t b = n * (a.K / a.block) + (k0 + cw) / a.block;
                sc[h] = a.dq ? __fmul_rn(static_cast<float>(__ldg(a.q8 + b)), __fdiv_rn(__ldg(a.cg + (b >> 8)), 127.0f))
                             : __ldg(a.absmax + b);
            }
        }

        // rows rw + g, rw + g + 8 of B as MMA A fragments, one set per 16 ranks
        uint32_t af[RQ][4];
#pragma unroll
        for (int q = 0; q < RQ; ++q) {
            const int ks = 16 * q;
            af[q][0] = *reinterpret_cast<const uint32_t *>(Bs + (rw + g) * rs + ks + 2 * t);
            af[q][1] = *reinterpret_cast<const uint32_t *>(Bs + (rw + g + 8) * rs + ks + 2 * t);
            af[q][2] = *reinterpret_cast<const uint32_t *>(Bs + (rw + g) * rs + ks + 2 * t + 8);
            af[q][3] = *reinterpret_cast<const uint32_t *>(Bs + (rw + g + 8) * rs + ks + 2 * t + 8);
        }

        // per 8-column tile i: the rank-r product, then out = fma(s, BA, w~) for
        // elements (row, 8 i + 2 t) and (row, 8 i + 2 t + 1), rows g and g + 8
        const uint8_t *crow0 = cs + (rw + g) * kMgCodeStride + cw / 2;
        const uint8_t *crow1 = crow0 + 8 * kMgCodeStride;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const uint16_t *bc = Ats + (cw + 8 * i + g) * rs + 2 * t;
#pragma unroll
            for (int q = 0; q < RQ; ++q)
                mma_bf16_16816(acc, af[q], *reinterpret_cast<const uint32_t *>(bc + 16 * q),
                               *reinterpret_cast<const uint32_t *>(bc + 16 * q + 8));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t byte = (h ? crow1 : crow0)[4 * i + t];
                const float w0 = __fmul_rn(sc[h], lv[byte >> 4]);
                const float w1 = __fmul_rn(sc[h], lv[byte & 15u]);
                const float o0 = fmaf(a.scale, acc[2 * h], w0);
                const float o1 = fmaf(a.scale, acc[2 * h + 1], w1);
                const int rl = g + 8 * h, cl = 8 * i + 2 * t;
                if (OUT_BF16) {
                    __nv_bfloat162 p = __floats2bfloat162_rn(o0, o1);
                    *reinterpret_cast<__nv_bfloat162 *>(st + (rl * (64 + 8) + cl) * 2) = p;
                } else {
                    *reinterpret_cast<float2 *>(st + (rl * (64 + 4) + cl) * 4) = make_float2(o0, o1);
                }
            }
        }
        __syncwarp();
        if (cols_ok) {
            // 16 rows of 64 outputs leave as 16-byte stores, consecutive lanes along a row
            constexpr int kChunksPerRow = OUT_BF16 ? 8 : 16;
#pragma unroll
            for (int c = lane; c < 16 * kChunksPerRow; c += 32) {
                const int rl = c / kChunksPerRow, ch = c % kChunksPerRow;
                const int64_t n = n0 + rw + rl;
                if (n >= a.N) continue;
                const int64_t col = k0 + cw + ch * (OUT_BF16 ? 8 : 4);
                if (OUT_BF16) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(st + (rl * (64 + 8) + ch * 8) * 2);
                    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + n * a.K + col) = v;
                } else {
                    const uint4 v = *reinterpret_cast<const uint4 *>(st + (rl * (64 + 4) + ch * 4) * 4);
                    *reinterpret_cast<uint4 *>(static_cast<float *>(a.out) + n * a.K + col) = v;
                }
            }
        }
        __syncwarp();            // the staging buffer is read before the next tile writes it
    }
}

}  // namespace nf4

namespace nf4 {

// ---------------------------------------------------------------------------
// The adapter part of dX under LoRA dropout: with dropout on the adapter input,
// the gradient that reaches x through the adapters is masked element-wise,
//     dX[m][k] += keep[m][k] * sum_j Vs[m][j] A[j][k],   Vs = bf16((alpha/r)/(1-p) v)
// (the chain rule through inverted dropout; "QLoRA Finetuner", section 1,
// h = W0 x + (alpha/r) B(A(dropout x))). base holds dY W~ in fp32 (written by
// the dgrad GEMM); the sum is accumulated in fp32 on mma.sync fragments and
// one rounding of base + kept sum gives dX in bf16. Same tiling as the merge kernel: 64 rows (tokens) x 128 columns
// per CTA, warp w on rows [16 (w % 4), +16) and columns [64 (w / 4), +64).
// ---------------------------------------------------------------------------
struct LoraAddArgs {
    int64_t M, K;
    int r, rp;
    const uint16_t *Vs;        // [M, r]
    const uint16_t *A;         // [r, K]
    const uint8_t *keep;       // bit mask over [M, K] (when rng.on is 0)
    DropRng rng;               // the mask drawn from the generator (rng.on)
    const float *base;         // [M, K] fp32: dY W~
    uint16_t *dX;              // [M, K] bf16 result
};

__host__ __device__ inline int lora_add_smem_bytes(int rp) {
    return kMgRows * merge_bs_stride(rp) * 2 + kMgCols * merge_bs_stride(rp) * 2 + 8 * 16 * (64 + 4) * 4;
}

template <int RQ>
__global__ void __launch_bounds__(kMgThreads, 4) qlora_lora_add_kernel(const LoraAddArgs a) {
    extern __shared__ __align__(16) uint8_t msm[];
    constexpr int rs = merge_bs_stride(16 * RQ);
    uint16_t *Vsm = reinterpret_cast<uint16_t *>(msm);                      // [64][rs]
    uint16_t *Ats = Vsm + kMgRows * rs;                                     // [128][rs]
    uint8_t *stage = reinterpret_cast<uint8_t *>(Ats + kMgCols * rs);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kMgRows;
    const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kMgCols;

    griddep_wait();
    griddep_launch_dependents();

    for (int idx = tid; idx < kMgRows * (a.rp / 8); idx += kMgThreads) {
        const int row = idx / (a.rp / 8), ch = idx % (a.rp / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m0 + row < a.M && ch * 8 < a.r)
            v = __ldg(reinterpret_cast<const uint4 *>(a.Vs + (m0 + row) * a.r) + ch);
        *reinterpret_cast<uint4 *>(Vsm + row * rs + ch * 8) = v;
    }
    for (int idx = tid; idx < a.rp * (kMgCols / 8); idx += kMgThreads) {
        const int j = idx % a.rp, ch = idx / a.rp;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (j < a.r && k0 + ch * 8 < a.K)
            v = __ldg(reinterpret_cast<const uint4 *>(a.A + static_cast<int64_t>(j) * a.K + k0) + ch);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            Ats[(ch * 8 + e) * rs + j] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
    }
    __syncthreads();

    const int rw = 16 * (warp & 3), cw = 64 * (warp >> 2);
    if (k0 + cw >= a.K) return;            // K is a multiple of 64: a warp's columns are all in or out
    uint32_t af[RQ][4];
#pragma unroll
    for (int q = 0; q < RQ; ++q) {
        const int ks = 16 * q;
        af[q][0] = *reinterpret_cast<const uint32_t *>(Vsm + (rw + g) * rs + ks + 2 * t);
        af[q][1] = *reinterpret_cast<const uint32_t *>(Vsm + (rw + g + 8) * rs + ks + 2 * t);
        af[q][2] = *reinterpret_cast<const uint32_t *>(Vsm + (rw + g) * rs + ks + 2 * t + 8);
        af[q][3] = *reinterpret_cast<const uint32_t *>(Vsm + (rw + g + 8) * rs + ks + 2 * t + 8);
    }
    float *st = reinterpret_cast<float *>(stage + warp * 16 * (64 + 4) * 4);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint16_t *bc = Ats + (cw + 8 * i + g) * rs + 2 * t;
#pragma unroll
        for (int q = 0; q < RQ; ++q)
            mma_bf16_16816(acc, af[q], *reinterpret_cast<const uint32_t *>(bc + 16 * q),
                           *reinterpret_cast<const uint32_t *>(bc + 16 * q + 8));
        *reinterpret_cast<float2 *>(st + g * (64 + 4) + 8 * i + 2 * t) = make_float2(acc[0], acc[1]);
        *reinterpret_cast<float2 *>(st + (g + 8) * (64 + 4) + 8 * i + 2 * t) = make_float2(acc[2], acc[3]);
    }
    __syncwarp();
    // 16 rows x 8 pieces of 8 columns: fp32 base plus the kept adapter terms, one rounding
#pragma unroll
    for (int c = lane; c < 16 * 8; c += 32) {
        const int rl = c >> 3, ch = c & 7;
        const int64_t m = m0 + rw + rl;
        if (m >= a.M) continue;
        const int64_t k = k0 + cw + 8 * ch;
        const uint32_t kb = a.rng.on ? drop_keep8(a.rng, static_cast<uint64_t>(m * a.K + k))
                                     : a.keep[(m * a.K + k) >> 3];
        uint4 *px = reinterpret_cast<uint4 *>(a.dX + m * a.K + k);
        const float4 b0 = *reinterpret_cast<const float4 *>(a.base + m * a.K + k);
        const float4 b1 = *reinterpret_cast<const float4 *>(a.base + m * a.K + k + 4);
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        const float4 l0 = *reinterpret_cast<const float4 *>(st + rl * (64 + 4) + 8 * ch);
        const float4 l1 = *reinterpret_cast<const float4 *>(st + rl * (64 + 4) + 8 * ch + 4);
        const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = bv[2 * e] + ((kb >> (2 * e)) & 1u ? lv[2 * e] : 0.0f);
            const float x1 = bv[2 * e + 1] + ((kb >> (2 * e + 1)) & 1u ? lv[2 * e + 1] : 0.0f);
            __nv_bfloat162 p = __floats2bfloat162_rn(x0, x1);
            o[e] = *reinterpret_cast<uint32_t *>(&p);
        }
        *px = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace nf4
