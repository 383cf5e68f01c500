// decode.cuh -- pieces shared by the decode-shaped forward (M <= 16 tokens):
// the m16n8k16 bf16 tensor-core product used on register fragments, and the
// small kernel that forms partial sums of u = x A^T ("QLoRA explained",
// section "The LoRA adapter path") ahead of the weight-streaming kernel in
// decode3.cuh.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Partial sums of u = x A^T for a few tokens (M <= 16): CTA (j, s) reduces
// the s-th of kDecUSplits k-slices for rank column j and all tokens, in a
// fixed order, and writes upart[s][m][j]. The decode kernel that follows adds
// the kDecUSplits partials of each u[m][j] in order of s. Splitting k spreads
// the reads of x over r * kDecUSplits CTAs.
constexpr int kDecUThreads = 128;
constexpr int kDecUSplits = 8;

__global__ void __launch_bounds__(kDecUThreads)
decode_lora_u_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ A, int M,
                     int64_t K, int r, float *__restrict__ upart) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float red[kDecUThreads / 32][16];
    const int j = blockIdx.x, sl = blockIdx.y;
    const int64_t k0 = K * sl / kDecUSplits / 8 * 8, k1 = K * (sl + 1) / kDecUSplits / 8 * 8;
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = 0.0f;
    const uint16_t *ar = A + static_cast<int64_t>(j) * K;
    for (int64_t k = k0 + 8 * threadIdx.x; k < k1; k += 8 * kDecUThreads) {
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
        upart[(static_cast<int64_t>(sl) * M + m) * r + j] = v;
    }
}

}  // namespace nf4
