// lora_small.cuh -- the rank-r side products of the QLoRA layer:
//   u  = x A^T            (forward down-projection, "QLoRA explained",
//                          section "The LoRA adapter path": x @ lora_A.t())
//   v  = dY B             (backward through the up-projection)
//   dB = s dY^T u,  dA = s v^T x   (adapter gradients; s = alpha / r)
// These are skinny products (r <= 128 columns) that read one large operand
// once; they run on the CUDA cores with shared-memory tiles.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// out[m][j] = sum_k P[m][k] * Q[j][k]      P: [M, Kd] bf16, Q: [r, Kd] bf16
// out_f32 (nullable) gets the fp32 sums; out_bf16 (nullable) gets
// bf16(scale * sum).  One CTA per 32 rows; 256 threads; thread t owns row
// t % 32 and columns j = t / 32 + 8 * jj.
constexpr int kRowdotRows = 32;
constexpr int kRowdotKC = 64;

__global__ void __launch_bounds__(256)
rowdot_kernel(const uint16_t *__restrict__ P, const uint16_t *__restrict__ Q, int M, int Kd, int r,
              float *__restrict__ out_f32, uint16_t *__restrict__ out_bf16, float scale) {
    __shared__ float Ps[kRowdotKC][kRowdotRows + 1];
    __shared__ float Qs[128][kRowdotKC + 1];
    const int m0 = blockIdx.x * kRowdotRows;
    const int t = threadIdx.x;
    const int row = t % kRowdotRows, jg = t / kRowdotRows;
    float acc[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.0f;

    for (int k0 = 0; k0 < Kd; k0 += kRowdotKC) {
        for (int e = t; e < kRowdotRows * kRowdotKC; e += 256) {
            const int rr = e / kRowdotKC, kc = e % kRowdotKC;
            const int m = m0 + rr, k = k0 + kc;
            Ps[kc][rr] = (m < M && k < Kd) ? bf16_bits_to_f32(P[static_cast<int64_t>(m) * Kd + k]) : 0.0f;
        }
        for (int e = t; e < r * kRowdotKC; e += 256) {
            const int j = e / kRowdotKC, kc = e % kRowdotKC;
            const int k = k0 + kc;
            Qs[j][kc] = (k < Kd) ? bf16_bits_to_f32(Q[static_cast<int64_t>(j) * Kd + k]) : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int kc = 0; kc < kRowdotKC; ++kc) {
            const float p = Ps[kc][row];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = jg + 8 * jj;
                if (j < r) acc[jj] = fmaf(p, Qs[j][kc], acc[jj]);
            }
        }
        __syncthreads();
    }
    const int m = m0 + row;
    if (m < M) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            const int j = jg + 8 * jj;
            if (j < r) {
                if (out_f32) out_f32[static_cast<int64_t>(m) * r + j] = acc[jj];
                if (out_bf16) {
                    __nv_bfloat16 b = __float2bfloat16_rn(scale * acc[jj]);
                    out_bf16[static_cast<int64_t>(m) * r + j] = *reinterpret_cast<uint16_t *>(&b);
                }
            }
        }
    }
}

// Partial column products over a chunk of rows:
//   part[s][c][j] = sum_{m in chunk s} P[m][c] * U[m][j]
// P: [M, C] bf16, U: [M, r] fp32. Grid (ceil(C/64), S); thread t owns column
// c0 + t % 64 and columns j = t / 64 + 4 * jj of the rank dimension.
constexpr int kColTile = 64;
constexpr int kColRows = 32;

__global__ void __launch_bounds__(256)
colprod_partial_kernel(const uint16_t *__restrict__ P, const float *__restrict__ U, int M, int C,
                       int r, int rows_per_split, float *__restrict__ part) {
    __shared__ float Ps[kColRows][kColTile + 1];
    __shared__ float Us[kColRows][128 + 1];
    const int c0 = blockIdx.x * kColTile;
    const int s = blockIdx.y;
    const int mb = s * rows_per_split;
    const int me = min(M, mb + rows_per_split);
    const int t = threadIdx.x;
    const int cl = t % kColTile, jg = t / kColTile;
    float acc[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) acc[jj] = 0.0f;

    for (int m0 = mb; m0 < me; m0 += kColRows) {
        for (int e = t; e < kColRows * kColTile; e += 256) {
            const int rr = e / kColTile, cc = e % kColTile;
            const int m = m0 + rr, c = c0 + cc;
            Ps[rr][cc] = (m < me && c < C) ? bf16_bits_to_f32(P[static_cast<int64_t>(m) * C + c]) : 0.0f;
        }
        for (int e = t; e < kColRows * r; e += 256) {
            const int rr = e / r, j = e % r;
            const int m = m0 + rr;
            Us[rr][j] = (m < me) ? U[static_cast<int64_t>(m) * r + j] : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int rr = 0; rr < kColRows; ++rr) {
            const float p = Ps[rr][cl];
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const int j = jg + 4 * jj;
                if (j < r) acc[jj] = fmaf(p, Us[rr][j], acc[jj]);
            }
        }
        __syncthreads();
    }
    const int c = c0 + cl;
    if (c < C) {
        float *dst = part + (static_cast<int64_t>(s) * C + c) * r;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
            const int j = jg + 4 * jj;
            if (j < r) dst[j] = acc[jj];
        }
    }
}

// out = bf16(scale * sum_s part[s][c][j]); transposed == 0 writes out[c][j]
// ([C, r]), transposed == 1 writes out[j][c] ([r, C]). Sums in split order.
__global__ void colprod_reduce_kernel(const float *__restrict__ part, int S, int C, int r,
                                      float scale, int transposed, uint16_t *__restrict__ out) {
    const int64_t total = static_cast<int64_t>(C) * r;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = 0.0f;
        for (int s = 0; s < S; ++s) acc += part[static_cast<int64_t>(s) * total + e];
        const int c = static_cast<int>(e / r), j = static_cast<int>(e % r);
        __nv_bfloat16 b = __float2bfloat16_rn(scale * acc);
        const int64_t o = transposed ? static_cast<int64_t>(j) * C + c : e;
        out[o] = *reinterpret_cast<uint16_t *>(&b);
    }
}

// Bt[j][n] = B[n][j]
__global__ void transpose_nr_kernel(const uint16_t *__restrict__ B, int N, int r,
                                    uint16_t *__restrict__ Bt) {
    const int64_t total = static_cast<int64_t>(N) * r;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t n = e / r, j = e % r;
        Bt[j * N + n] = B[e];
    }
}

__global__ void zero_u16_kernel(uint16_t *__restrict__ p, int64_t n) {
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[e] = 0;
}

}  // namespace nf4
