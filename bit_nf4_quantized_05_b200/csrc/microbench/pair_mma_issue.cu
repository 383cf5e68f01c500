// pair_mma_issue.cu -- issue-rate microbenchmark of the fused GEMM's CTA-pair
// MMA sequence (a standalone program; not part of the library).
//
// On every SM pair of the GPU (74 clusters of 2 CTAs), warp 0 of the even CTA
// issues, per stage, the fused GEMM's four 256 x 256 x 16 bf16 pair MMAs
// (tcgen05.mma.cta_group::2, K-major 128-byte-swizzled operands, rotating over
// four 16 KB operand slots of static shared memory) and one multicast commit,
// for 4000 stages; it reports the SM cycles per stage (512 is the tensor
// core's rate for four such MMAs). The other warps of both CTAs (`noise
// warps`, 0, 12 or 20 of them) run byte permutes and logic ops without pause
// until the issuer is done, standing in for the dequantisation warps that
// share the issuer's schedulers. Issue forms (template `mode`):
//   2   one lane in divergent code: probe of a complete barrier, fence, MMAs,
//       commit (the form the fused GEMM used before)
//   6   whole warp: every lane probes, elect.sync issues
//   7   whole warp: lane 0 probes and broadcasts, elect.sync issues
//   8   whole warp: every lane probes, warp vote, lane 0 issues by predicate
//   9   whole warp: every lane probes, warp vote, elect.sync issues (the form
//       the fused GEMM uses now)
// Other modes in the kernel (0, 1, 3, 4, 5, 10) are variants not launched by
// main(). Every wait is bounded; operands are zero-filled.
//
// Build and run on a B200 from the repository root:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -lineinfo \
//        -o pair_mma_issue bit_nf4_quantized_05_b200/csrc/microbench/pair_mma_issue.cu -lcuda
//   ./pair_mma_issue
#include "../nf4_common.cuh"
#include <cstdio>
#include <vector>
#include <algorithm>
using namespace nf4;

constexpr int kSlots = 4;
constexpr int kSlotBytes = 16384;
constexpr int kSmem = 2 * kSlots * kSlotBytes + 1024 + 512;

__device__ __forceinline__ void umma_pair_elect(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(acc)
                 : "memory");
}
__device__ __forceinline__ void commit_pair_elect(uint64_t *bar, uint16_t mask) {
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
                 " [%0], %1;\n\t}" ::"r"(smem_u32(bar)), "h"(mask)
                 : "memory");
}
__device__ __forceinline__ void umma_pair_pred(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc, uint32_t issue) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "setp.ne.b32 e, %5, 0;\n\t"
                 "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(issue)
                 : "memory");
}
__device__ __forceinline__ void commit_pair_pred(uint64_t *bar, uint16_t mask, uint32_t issue) {
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "setp.ne.b32 e, %2, 0;\n\t"
                 "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
                 " [%0], %1;\n\t}" ::"r"(smem_u32(bar)), "h"(mask), "r"(issue)
                 : "memory");
}
__device__ __forceinline__ bool drain_ok(uint64_t *bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > 2000000000LL) return false;
    return true;
}

// mode 0: lane 0, 4 MMAs + commit per stage
// mode 1: lane 0, 4 MMAs per stage, no per-stage commit
// mode 2: lane 0, probe of a complete barrier + fence + 4 MMAs + commit per stage
// mode 3: whole warp, elect-one issue, 4 MMAs + commit per stage
// mode 4: lane 0, 8 MMAs + commit per stage (half the stages)
// mode 5: lane 0, 4 MMAs per stage, each MMA on the same (slot 0) operands, commit per stage
// modes 6-10: whole warp, as listed at the top of the file (10: every lane
// probes, no vote, lane 0 issues by predicate)
template <int mode>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(1024, 1)
pair_mma_bench(int stages, long long *out, uint32_t *sink) {
    extern __shared__ uint8_t raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sa = sm, *sb = sm + kSlots * kSlotBytes;
    uint64_t *consumed = reinterpret_cast<uint64_t *>(sm + 2 * kSlots * kSlotBytes);
    uint64_t *done_bar = consumed + 16;
    uint64_t *ready = done_bar + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(ready + 1);
    volatile int *stop = reinterpret_cast<volatile int *>(tslot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    for (int i = threadIdx.x; i < 2 * kSlots * kSlotBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(sm)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 16; ++i) mbar_init(&consumed[i], 1);
        mbar_init(done_bar, 1);
        mbar_init(ready, 1);
        *stop = 0;
        fence_mbar_init();
        mbar_arrive(ready);    // phase 0 complete: a probe of parity 0 succeeds
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc_pair(tslot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t idesc = idesc_bf16_f32(256, 256, 0, 0);
    const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
    bool ok = true;
    if (warp > 0) {
        // ALU pressure: byte permutes and logic ops until the issuer is done
        uint32_t x = threadIdx.x * 0x9E3779B9u, y = x ^ 0x85EBCA6Bu, z = x + 0xC2B2AE35u;
        const long long t0 = clock64();
        while (true) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                x = prmt(x, y, z & 0x7777u);
                y = (x & ~z) | (y & z);
                z += x ^ (y << 4);
            }
            if (*stop || clock64() - t0 > 200000000LL) break;
        }
        sink[blockIdx.x * blockDim.x + threadIdx.x] = x ^ y ^ z;
    }
    if (rank == 0 && warp == 0) {
        const long long c0 = clock64();
        if constexpr (mode == 3 || mode >= 6) {
            for (int i = 0; i < stages; ++i) {
                if constexpr (mode == 6) {
                    if (!mbar_try_wait(ready, 0)) { ok = false; break; }
                    tc_fence_after();
                } else if constexpr (mode == 8 || mode == 9) {
                    const int r = __all_sync(0xffffffffu, mbar_try_wait(ready, 0) ? 1 : 0);
                    if (!r) { ok = false; break; }
                    tc_fence_after();
                } else if constexpr (mode == 10) {
                    if (!mbar_try_wait(ready, 0)) { ok = false; break; }
                    tc_fence_after();
                } else if constexpr (mode == 7) {
                    int r = 0;
                    if (lane == 0) r = mbar_try_wait(ready, 0) ? 1 : 0;
                    r = __shfl_sync(0xffffffffu, r, 0);
                    if (!r) { ok = false; break; }
                    tc_fence_after();
                }
                const uint32_t aa = a0 + (i % kSlots) * kSlotBytes, bb = b0 + (i % kSlots) * kSlotBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if constexpr (mode == 8 || mode == 10)
                        umma_pair_pred(tmem, smem_desc_sw128(aa + kk * 32, 16, 1024), smem_desc_sw128(bb + kk * 32, 16, 1024),
                                       idesc, (i | kk) ? 1u : 0u, lane == 0 ? 1u : 0u);
                    else
                        umma_pair_elect(tmem, smem_desc_sw128(aa + kk * 32, 16, 1024), smem_desc_sw128(bb + kk * 32, 16, 1024),
                                        idesc, (i | kk) ? 1u : 0u);
                }
                if constexpr (mode == 8 || mode == 10) commit_pair_pred(&consumed[i & 15], 0x3, lane == 0 ? 1u : 0u);
                else commit_pair_elect(&consumed[i & 15], 0x3);
            }
            __syncwarp();
            if (lane == 0) {
                umma_commit_pair(done_bar, 0x1);
                ok = drain_ok(done_bar, 0);
            }
        } else {
          if (lane == 0) {
            const int n = mode == 4 ? stages / 2 : stages;
            for (int i = 0; i < n; ++i) {
                if constexpr (mode == 2) {
                    if (!mbar_try_wait(ready, 0)) { ok = false; break; }
                    tc_fence_after();
                }
                const int s = mode == 5 ? 0 : i % kSlots;
                const uint32_t aa = a0 + s * kSlotBytes, bb = b0 + s * kSlotBytes;
                const int nk = mode == 4 ? 8 : 4;
                for (int kk = 0; kk < nk; ++kk) {
                    const int k4 = kk & 3;
                    const uint32_t ax = (mode == 4 && kk >= 4) ? a0 + ((i + 1) % kSlots) * kSlotBytes : aa;
                    const uint32_t bx = (mode == 4 && kk >= 4) ? b0 + ((i + 1) % kSlots) * kSlotBytes : bb;
                    umma_bf16_ss_pair(tmem, smem_desc_sw128(ax + k4 * 32, 16, 1024), smem_desc_sw128(bx + k4 * 32, 16, 1024),
                                      idesc, (i | kk) ? 1u : 0u);
                }
                if (mode != 1) umma_commit_pair(&consumed[i & 15], 0x3);
            }
            umma_commit_pair(done_bar, 0x1);
            ok = ok && drain_ok(done_bar, 0);
          }
        }
        const long long c1 = clock64();
        if (lane == 0) {
            *stop = 1;
            const uint32_t peer = mapa_shared(smem_u32(const_cast<int *>(stop)), 1u);
            asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
            out[blockIdx.x / 2 * 2 + 0] = ok ? (c1 - c0) : -1;
            out[blockIdx.x / 2 * 2 + 1] = stages;
        }
    }
    __syncthreads();
    tc_fence_before();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

int main() {
    cudaFuncSetAttribute(pair_mma_bench<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    cudaFuncSetAttribute(pair_mma_bench<6>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    cudaFuncSetAttribute(pair_mma_bench<7>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    cudaFuncSetAttribute(pair_mma_bench<9>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    cudaFuncSetAttribute(pair_mma_bench<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    long long *d_out;
    cudaMalloc(&d_out, 148 * 2 * sizeof(long long));
    uint32_t *d_sink;
    cudaMalloc(&d_sink, 148 * 1024 * sizeof(uint32_t));
    const int stages = 4000;
    const int pairs = 74;
    for (int nw : {0, 12, 20}) {
        for (int mode : {2, 6, 7, 8, 9}) {
            for (int rep = 0; rep < 2; ++rep) {
                cudaMemset(d_out, 0, 148 * 2 * sizeof(long long));
                cudaEvent_t e0, e1;
                cudaEventCreate(&e0); cudaEventCreate(&e1);
                cudaEventRecord(e0);
                {
                    dim3 g(2 * pairs), b(32 * (1 + nw));
                    if (mode == 2) pair_mma_bench<2><<<g, b, kSmem>>>(stages, d_out, d_sink);
                    if (mode == 6) pair_mma_bench<6><<<g, b, kSmem>>>(stages, d_out, d_sink);
                    if (mode == 7) pair_mma_bench<7><<<g, b, kSmem>>>(stages, d_out, d_sink);
                    if (mode == 8) pair_mma_bench<8><<<g, b, kSmem>>>(stages, d_out, d_sink);
                    if (mode == 9) pair_mma_bench<9><<<g, b, kSmem>>>(stages, d_out, d_sink);
                }
                cudaEventRecord(e1);
                cudaError_t err = cudaDeviceSynchronize();
                if (err != cudaSuccess) { printf("mode %d: %s\n", mode, cudaGetErrorString(err)); return 1; }
                float ms; cudaEventElapsedTime(&ms, e0, e1);
                std::vector<long long> h(148 * 2);
                cudaMemcpy(h.data(), d_out, h.size() * sizeof(long long), cudaMemcpyDeviceToHost);
                std::vector<double> cyc;
                bool bad = false;
                for (int p = 0; p < pairs; ++p) {
                    if (h[2 * p] < 0) bad = true;
                    cyc.push_back(double(h[2 * p]) / stages);
                }
                std::sort(cyc.begin(), cyc.end());
                printf("noise warps %2d mode %d rep %d: cycles/stage med %.1f min %.1f max %.1f  kernel %.3f ms  %s\n", nw,
                       mode, rep, cyc[cyc.size() / 2], cyc.front(), cyc.back(), ms, bad ? "TIMEOUT" : "");
            }
        }
    }
    return 0;
}
