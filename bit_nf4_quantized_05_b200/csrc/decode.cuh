// decode.cuh -- pieces shared by the decode-shaped forward (M <= 16 tokens):
// the m16n8k16 bf16 tensor-core product used on register fragments, and the
// small kernel that forms u = x A^T and bf16((alpha/r) u) ("QLoRA explained",
// section "The LoRA adapter path") ahead of the weight-streaming kernel in
// decode2.cuh.
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
