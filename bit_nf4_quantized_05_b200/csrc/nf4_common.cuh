// nf4_common.cuh -- shared device helpers of the sm_100a QLoRA library:
// the NF4 level table, the device status word, and thin wrappers over the
// PTX of mbarriers, TMA and tcgen05 (tensor memory + 5th-gen tensor cores).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora_nf4.h"

namespace nf4 {

// ---------------------------------------------------------------------------
// NF4 levels: the 16-value lookup table printed in "QLoRA explained:
// fine-tuning in 4-bit precision" (section "Common misconceptions"), index
// order as in the level table of "Parameter-Efficient Fine-Tuning: From LoRA
// to QLoRA" (Pillar 1). Written as hex floats; every value is an exact fp32.
// ---------------------------------------------------------------------------
#define NF4_LEVEL_LIST                                                          \
    -0x1.000000p+0f, -0x1.647362p-1f, -0x1.0cd660p-1f, -0x1.946540p-2f,         \
    -0x1.23449ap-2f, -0x1.7a6a7ep-3f, -0x1.74f0e2p-4f, 0x0.0p+0f,               \
    0x1.45f5fep-4f, 0x1.4995c6p-3f, 0x1.f809bap-3f, 0x1.5a0674p-2f,            \
    0x1.c34970p-2f, 0x1.200f56p-1f, 0x1.722766p-1f, 0x1.000000p+0f

__constant__ float c_levels[16] = {NF4_LEVEL_LIST};

// Elements per NF4 block: 64 or 128. The kernels walk K in 64-element steps
// (kBlock); a 128-element block is two consecutive steps that share one
// scale, block index = step >> block_shift.
constexpr int kBlock = 64;
__host__ __device__ constexpr int block_shift_of(int block_size) { return block_size == 128 ? 1 : 0; }
constexpr int kGroup = 256;      // blocks per double-quant group

// ---------------------------------------------------------------------------
// Device status word (first error wins). Read and cleared by the host.
// ---------------------------------------------------------------------------
__device__ unsigned int g_status;

__device__ __forceinline__ void record_status(unsigned int code) {
    atomicCAS(&g_status, 0u, code);
}

// Pipeline waits give up after this many SM cycles (about 2 s at the
// B200's clocks), record NF4_ERR_TIMEOUT and unwind.
constexpr long long kWaitLimitCycles = 4000000000LL;

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// A waiting thread is suspended in try_wait until the phase completes or this
// many nanoseconds pass, so a warp that waits (for a whole tile, say) costs
// a few issue slots rather than a spin loop's worth; the bounded waits below
// still look at their clock and at the abort flag after every return.
constexpr uint32_t kSuspendHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// The CTA's abort flag, read from shared memory.
__device__ __forceinline__ int abort_raised(volatile int *abort_flag) {
    int v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];"
                 : "=r"(v)
                 : "r"(smem_u32(const_cast<int *>(abort_flag)))
                 : "memory");
    return v;
}

// Bounded wait for the phase with the given parity. Returns false (and
// raises the CTA's abort flag) when the wait runs out of time or another
// role of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (abort_raised(abort_flag)) return false;
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitLimitCycles) {
            record_status(NF4_ERR_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// mbar_wait by every lane of a converged warp; the lanes agree on the outcome
// (any lane that gave up makes the whole warp give up), so the warp stays
// converged on both paths.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag)) != 0;
}

// Bounded wait that ignores the abort flag: used on the way out of a kernel
// that gave up, so that the copies (or tensor-core operations) it has already
// issued land before its shared memory and tensor memory are released.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitLimitCycles) return;
}

// complete_tx of `bytes` on an mbarrier of this CTA (bytes that will never be
// copied: lets a phase whose copy was never issued complete).
__device__ __forceinline__ void mbar_complete_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Test hooks of the stream-K flag wait (set through nf4_debug_flag_wait):
// when g_dbg_skip_flag_set is nonzero the tails of split tiles do not raise
// their flags, and a nonzero g_dbg_flag_wait_limit replaces the flag wait's
// cycle limit, so a test can make that one wait run out.
__device__ int g_dbg_skip_flag_set;
__device__ long long g_dbg_flag_wait_limit;

// ---------------------------------------------------------------------------
// Programmatic dependent launch. Every kernel of this library that is launched
// as a programmatic dependent first waits for the grid before it in the stream
// (complete, memory visible), then lets the next grid launch; so a kernel may
// run its set-up while its predecessor finishes, and any grid that starts early
// finds every grid two places before it complete.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters: ranks, cluster addresses, remote arrivals
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// Arrive on an mbarrier given by its cluster address (possibly the other CTA
// of a pair), with the default release semantics at CTA scope. What the
// arrival publishes is read by tensor-core operations (the async proxy) that
// are issued after the phase completes: the arriving threads make their
// shared-memory writes visible to that proxy with fence.proxy.async first,
// and tensor-memory reads are ordered by tcgen05.fence::before_thread_sync.
// A cluster-scope release here would add a fence per arrival that the pair
// pipeline does not need; it cost about 4% of the fused GEMM's time.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// Generic-proxy writes to shared memory become visible to the async proxy
// (tensor core operand reads, TMA) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), 2-D tiles into shared memory
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only); with valid false
// nothing is read and the 16 bytes are zero-filled (src must still be a
// valid address).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier when every tcgen05 op issued so far by this
// thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// ---- CTA-pair forms (cta_group::2): one MMA spans the two CTAs of a cluster
// pair; CTA v of the pair holds rows [128v, 128v+128) of A and of the
// accumulator, and columns [vN/2, vN/2 + N/2) of B. Allocation, relinquish
// and deallocation are issued by the same warp in both CTAs.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void umma_bf16_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// The same MMA executed by a whole converged warp with warp-uniform operands
// and issued by the lane that elect.sync picks (the same lane every time the
// full warp executes it). A lone thread issuing from divergent code is slowed
// by the other warps sharing its scheduler; the converged, elected form keeps
// the tensor pipe fed under that load.
__device__ __forceinline__ void umma_bf16_ss_pair_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at this offset in each CTA of `mask` when the
// pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(mask)
        : "memory");
}
// umma_commit_pair executed by a converged warp: the elected lane (the one
// that issued the warp's MMAs) commits.
__device__ __forceinline__ void umma_commit_pair_warp(uint64_t *bar, uint16_t mask) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "h"(mask)
        : "memory");
}
// Tiled 2-D load into this CTA's shared memory whose completion is counted on
// an mbarrier that may live in the other CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map,
                                                 uint32_t bar_cluster, int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

// 32 TMEM lanes x 32 consecutive 32-bit columns; thread i of the warp gets
// lane (quadrant*32 + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
// The same for 16 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 form): start address, leading and
// stride byte offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;   // version
    d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, M x N, A/B major-ness
// (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4)                                  // D format fp32
           | (1u << 7)                                // A bf16
           | (1u << 10)                               // B bf16
           | (static_cast<uint32_t>(a_mn_major) << 15)
           | (static_cast<uint32_t>(b_mn_major) << 16)
           | (static_cast<uint32_t>(N >> 3) << 17)
           | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// NF4 block dequantisation into packed bf16 pairs (register-resident lookup)
//
// A block of 64 codes shares one scale s. The 16 possible outputs
// bf16(fl32(s * level_j)) are computed once per block and kept as byte planes
// in 8 registers; each code then selects its output with byte permutes, so
// no shared-memory lookup (and no bank conflict) is needed per element.
// ---------------------------------------------------------------------------
struct BlockLut {
    uint32_t lo[4];   // lo[q] bytes: low bytes of entries 4q..4q+3
    uint32_t hi[4];   // hi[q] bytes: high bytes of entries 4q..4q+3
};

__device__ __forceinline__ BlockLut make_block_lut(float s) {
    uint32_t pair[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        // fp32 product, then one rounding to bf16 (nearest even); entry 2i in
        // the low half, 2i+1 in the high half
        __nv_bfloat162 p = __floats2bfloat162_rn(s * c_levels[2 * i], s * c_levels[2 * i + 1]);
        pair[i] = *reinterpret_cast<uint32_t *>(&p);
    }
    BlockLut L;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        L.lo[q] = __byte_perm(pair[2 * q], pair[2 * q + 1], 0x6420);
        L.hi[q] = __byte_perm(pair[2 * q], pair[2 * q + 1], 0x7531);
    }
    return L;
}

// PRMT with the selector used as given (a selector nibble with bit 3 set
// replicates the sign bit of the selected byte across the output byte).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Dequantise the 8 codes of one 32-bit word (bytes in memory order; byte b
// holds element 2b in its high nibble and 2b+1 in its low nibble) into 4
// packed bf16x2 words, element order preserved (lower element in the low
// half).
__device__ __forceinline__ void dequant8(const BlockLut &L, uint32_t w, uint32_t (&out)[4]) {
    const uint32_t w4 = w << 4;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const uint32_t sel = (half ? (w >> 16) : w) & 0x7777u;
        // byte mask of codes >= 8, output byte order = nibble order of `sel`
        const uint32_t m = prmt(w, w4, half ? 0xBFAEu : 0x9D8Cu);
        const uint32_t la = __byte_perm(L.lo[0], L.lo[1], sel);
        const uint32_t lb = __byte_perm(L.lo[2], L.lo[3], sel);
        const uint32_t ha = __byte_perm(L.hi[0], L.hi[1], sel);
        const uint32_t hb = __byte_perm(L.hi[2], L.hi[3], sel);
        const uint32_t lo = (la & ~m) | (lb & m);
        const uint32_t hi = (ha & ~m) | (hb & m);
        // nibble order in `sel` is (odd, even, odd, even) elements; rebuild
        // bf16 pairs (even element low)
        out[2 * half + 0] = __byte_perm(lo, hi, 0x4051);
        out[2 * half + 1] = __byte_perm(lo, hi, 0x6273);
    }
}

// ---------------------------------------------------------------------------
// LoRA dropout drawn in the kernels ("QLoRA Finetuner -- Juan Martos",
// section 1: dropout on the adapter input). The draw is Philox4x32-10, the
// counter-based generator of Salmon et al. ("Parallel random numbers: as easy
// as 1, 2, 3", SC'11): element e of x [M, k] takes word e % 4 of the
// generator at counter (e / 4 as two 32-bit words, offset as two words) with
// key (seed as two words), and is dropped when that word is below
// floor(p * 2^32). Any kernel that needs the mask of some elements computes
// exactly those words, so the backward regenerates the forward's mask and no
// mask is stored.
// ---------------------------------------------------------------------------
struct DropRng {
    uint32_t k0, k1;       // key: the seed's low and high words
    uint32_t o0, o1;       // counter words 2 and 3: the offset's low and high words
    uint32_t thresh;       // an element is dropped when its word is below this
    int on;                // 0: no generated mask
};

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;     // Weyl sequence of the round keys
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
        const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ k1;
        c1 = static_cast<uint32_t>(p1);
        c3 = static_cast<uint32_t>(p0);
        c0 = n0;
        c2 = n2;
    }
    return make_uint4(c0, c1, c2, c3);
}

// Keep bits of the 4 * CALLS elements [e0, e0 + 4 CALLS) of x (e0 % 4 == 0):
// bit i is 1 when element e0 + i is kept. The generator calls are independent
// and computed four at a time, so that their multiply chains overlap.
template <int CALLS>
__device__ __forceinline__ uint64_t drop_keep_bits(const DropRng &d, uint64_t e0) {
    static_assert(CALLS >= 1 && CALLS <= 16, "at most 64 bits");
    constexpr int kBatch = CALLS < 4 ? CALLS : 4;
    uint64_t bits = 0;
    const uint64_t g0 = e0 >> 2;
#pragma unroll
    for (int q = 0; q < CALLS; q += kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const uint64_t g = g0 + q + j;
            v[j] = philox4x32_10(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), d.o0, d.o1, d.k0,
                                 d.k1);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const uint64_t nib = (v[j].x >= d.thresh ? 1u : 0u) | (v[j].y >= d.thresh ? 2u : 0u) |
                                 (v[j].z >= d.thresh ? 4u : 0u) | (v[j].w >= d.thresh ? 8u : 0u);
            bits |= nib << (4 * (q + j));
        }
    }
    return bits;
}

// Keep bits of the eight elements [e0, e0 + 8) of x (e0 % 8 == 0).
__device__ __forceinline__ uint32_t drop_keep8(const DropRng &d, uint64_t e0) {
    return static_cast<uint32_t>(drop_keep_bits<2>(d, e0));
}

}  // namespace nf4
