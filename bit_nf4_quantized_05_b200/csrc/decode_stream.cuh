// decode_stream.cuh -- the forward of the QLoRA layer for a handful of tokens
// (M <= 16): h = x W~^T + bf16((alpha/r) x A^T) B^T, streaming the 4-bit
// weight once from HBM ("QLoRA Finetuner", flowchart "Quantized Base
// Inference": load 4-bit indices and 32-bit block scales, dequantise,
// multiply).
//
// The weight dominates the bytes (n*k/2 code bytes against a few KB of
// tokens) and the dequantisation dominates the instructions, so the kernel is
// built to issue as few instructions per code byte as it can:
//   * persistent CTAs of 16 warps, one per SM, walk tiles of 32 weight rows;
//     the 16 warps split k sixteen ways, and each warp covers both 16-row
//     groups of the tile, so one token-fragment load serves 32 weight rows;
//   * each warp fetches its k range of a tile in chunks of CB blocks -- 32
//     rows x CB * 32 contiguous bytes -- with one 2-D TMA copy into a
//     two-slot ring; chunk c + 1 is requested as soon as chunk c has landed
//     (its slot held chunk c - 1, already consumed);
//   * a byte of codes becomes a pair of bf16 levels through a 256-entry table
//     in shared memory whose entry b, copy l sits at address
//     65536 + 256 b + 4 l: a single byte permute turns (code byte, lane) into
//     the lookup address, and lane l always reads copy l (no bank conflicts).
//     The other half of each 256-byte table row holds the k-split partials
//     of the tile being finished;
//   * the 16 x 8 x 16 products run on the tensor cores (mma.sync, the
//     dequantised fragment goes straight from registers to the MMA);
//   * u = x A^T ("QLoRA explained", section "The LoRA adapter path") is formed
//     by a small kernel on a few SMs that this grid leaves free, so it runs
//     beside the weight stream instead of in front of it;
//   * each 64-element block's partial product is scaled by its block scale
//     in fp32 and accumulated, so no per-element multiply by the scale; one
//     of the four lanes that share a row forms each (row, block) scale, from
//     values fetched a whole chunk ahead, and shuffles it to the others.
// Numerically this forms sum_b s_b * sum_k bf16(level) * x, which differs
// from bf16(s_b * level) * x by at most one bf16 rounding of each term.
#pragma once

#include "nf4_common.cuh"

namespace nf4 {

constexpr int kDsWarps = 16;                  // k split across the warps of a CTA
constexpr int kDsThreads = 32 * kDsWarps;
constexpr int kDsRows = 32;                   // weight rows per tile (two 16-row MMA groups)
constexpr int kDsMaxRank = 64;
constexpr int kDsMaxChunk = 5;                // blocks per TMA chunk (160 bytes per row)
constexpr int kDsDynBytes = 227 * 1024;       // the largest dynamic allocation of a CTA on B200
constexpr int kDsUCtas = 4;                   // SMs left to the u kernel
// Fixed shared addresses. The table takes [65536, 131072): row b is 256
// bytes, the first 128 the 32 lane copies of entry b, the last 128 one row
// of partials. Ring slots fill the rest of the window below and above it.
constexpr uint32_t kDsLutAddr = 65536;
constexpr uint32_t kDsHighAddr = 131072;
// the start of the dynamic window: chunk barriers and the abort flag, then u
constexpr int kDsUOff = 512;
constexpr int kDsLowBytes = kDsUOff + 16 * kDsMaxRank * 2;
static_assert(kDsWarps * 2 * 8 + 16 <= kDsUOff, "barrier area");

struct DecodeArgs {
    int M;                 // tokens (1..16)
    int64_t N, K;          // weight rows / columns
    int r;
    int rb;                // blocks per warp: ceil(K / 64 / 16)
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    const uint16_t *x;     // [M, K]
    const uint16_t *B;     // [N, r]
    const uint16_t *A;     // [r, K]
    float *upart;          // [kDsUCtas][M][r] partial sums of x A^T from the u kernel
    float scale;           // fl32(alpha / r)
    float *u_out;          // [M, r] fp32 x A^T (optional; written by CTA 0)
    uint16_t *h;           // [M, N]
    int bshift;            // log2(block size / 64): block of 64-element step j is j >> bshift
};

// Per-token adapter selection over stacked adapters (multi-adapter forward):
// token m keeps the group_width rank columns of adapter row_group[m], scaled
// by gscale of that adapter (no adapter term when row_group[m] is outside
// [0, ngroups)). The single-adapter instantiations take the empty type.
struct DsNoGroups {};
struct DsGroups {
    const int32_t *row_group;
    int group_width;
    int ngroups;
    float gscale[16];
};

// Table lookup by shared address. The table is written once before a
// barrier and never again, and every lookup address is derived from code
// words read after that barrier, so the load needs no ordering of its own.
__device__ __forceinline__ uint32_t ds_lut(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
// Ring loads. They are free to be scheduled among the table lookups and
// products; what keeps them after the chunk's barrier wait is that their
// addresses take a zero produced by an ordered instruction after the wait.
__device__ __forceinline__ uint2 ds_lds64(uint32_t addr) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t after_wait_zero() {
    uint32_t z;
    asm volatile("mov.u32 %0, 0;" : "=r"(z)::"memory");
    return z;
}

// Lookup address of code byte I of word w for this lane: the byte permute
// builds 65536 + 256 b + 4 lane from byte 0 = 4 lane, byte 1 = the code
// byte, byte 2 = 1, byte 3 = 0. Selector nibble k picks output byte k from
// {lanew (bytes 4..7), w (bytes 0..3)}: nibbles (from byte 3 down) 7, 6, I, 4.
template <int I>
__device__ __forceinline__ uint32_t ds_addr(uint32_t w, uint32_t lanew) {
    static_assert(I >= 0 && I < 4, "code byte");
    return prmt(w, lanew, 0x7604u | (static_cast<uint32_t>(I) << 4));
}

// d += a b (m16n8k16, bf16 inputs, fp32 accumulator)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d = a b (m16n8k16, bf16 inputs, fp32 result, zero accumulator in)
__device__ __forceinline__ void ds_mma_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// The raw block scales of one lane's row over one chunk: the 8-bit codes and
// the (at most two) group constants they refer to, or the fp32 absmax.
template <int CB>
struct DsScales {
    uint32_t raw[CB];      // q8 code, or the absmax bits
    float c0, c1;          // c_g of the chunk's first and last block
    int split;             // first block (chunk-relative) that uses c1
};

// TG = number of 8-token groups (1 for M <= 8, 2 for M <= 16); CB = blocks
// per chunk (it divides rb, the blocks of a warp in every tile).
//
// Fragment bookkeeping (m16n8k16, thread (g, t) = (lane / 4, lane % 4)): the
// A fragment holds rows g and g+8 of a 16-row group and four k slots per
// row; the reduction order inside one MMA is free, so the slots are chosen
// such that thread t's slots over a block's four MMAs are the 16 consecutive
// elements [16t, 16t+16) of the block: code bytes [8t, 8t+8) of each of its
// rows, and 16 consecutive x values per token.
//
// Warp w takes blocks [w rb, w rb + rb) of every tile, in chunks of CB
// blocks. Its chunks are numbered c = 0, 1, ... over all of the CTA's tiles;
// chunk c goes to ring slot c % 2, and the other slot takes chunk c + 1 as soon as
// every lane has read chunk c.
// GT: DsNoGroups, or DsGroups for per-token adapter selection.
template <int TG, int CB, class GT>
__global__ void __launch_bounds__(kDsThreads, 1)
qlora_decode_stream_kernel(const __grid_constant__ CUtensorMap tm_codes,   // [N, K/2] u8, box {32 CB, 32}
                           const DecodeArgs a, const GT grp) {
    constexpr bool GROUPS = sizeof(GT) > 1;
    extern __shared__ __align__(1024) uint8_t dsm[];
    constexpr uint32_t kSlot = 1024u * CB;           // bytes of one chunk (32 rows x 32 CB)
    constexpr uint32_t kRowStride = 32u * CB;        // bytes per row in a slot
    const uint32_t sbase = smem_u32(dsm);
    const uint32_t low0 = (sbase + kDsLowBytes + 127u) & ~127u;
    const uint32_t win_end = sbase + kDsDynBytes;
    const uint32_t nlow = low0 <= kDsLutAddr ? (kDsLutAddr - low0) / kSlot : 0u;
    const uint32_t nhigh = win_end >= kDsHighAddr ? (win_end - kDsHighAddr) / kSlot : 0u;
    if (sbase + kDsLowBytes > kDsLutAddr || win_end < kDsHighAddr || nlow + nhigh < 2u * kDsWarps) {
        if (threadIdx.x == 0) record_status(NF4_ERR_CUDA);   // the fixed addresses are not ours
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsm);                          // [warp][slot]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsm + kDsWarps * 2 * 8);
    uint16_t *u_tile = reinterpret_cast<uint16_t *>(dsm + kDsUOff);               // [M][r]
    uint8_t *lut_g = dsm + (kDsLutAddr - sbase);                                  // table rows

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDsWarps * 2; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_codes);
    }
    __syncthreads();

    const int kblocks = static_cast<int>(a.K / kBlock);
    const int Nrows = static_cast<int>(a.N);
    const int kb0 = warp * a.rb;
    const int nkb = max(0, min(a.rb, kblocks - kb0));
    const int nch = (nkb + CB - 1) / CB;
    const int ntiles = (Nrows + kDsRows - 1) / kDsRows;
    const int nt = static_cast<int>(blockIdx.x) < ntiles
                       ? (ntiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                             static_cast<int>(gridDim.x)
                       : 0;
    const int nchunks = nt * nch;
    // this warp's ring slots: numbered 2 warp, 2 warp + 1 over the window,
    // below the table first
    uint32_t slot0, slot1;
    {
        const uint32_t i0 = 2u * warp, i1 = i0 + 1u;
        slot0 = i0 < nlow ? low0 + i0 * kSlot : kDsHighAddr + (i0 - nlow) * kSlot;
        slot1 = i1 < nlow ? low0 + i1 * kSlot : kDsHighAddr + (i1 - nlow) * kSlot;
    }

    // chunk cc of this warp: tile cc / nch, blocks kb0 + (cc % nch) CB .. +CB
    auto issue = [&](int cc) {
        if (cc >= nchunks || lane != 0) return;
        const int ti = cc / nch, ch = cc - ti * nch;
        const int tile = static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x);
        uint64_t *bar = &bars[warp * 2 + (cc & 1)];
        // the slot's previous contents were read through the generic proxy
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, kSlot);
        tma_load_2d(dsm + (((cc & 1) ? slot1 : slot0) - sbase), &tm_codes, bar, (kb0 + ch * CB) * 32,
                    tile * kDsRows);
    };

    // the raw scales of chunk cc for this lane's row
    const int srow = (t >> 1) * 16 + g + 8 * (t & 1);
    auto load_scales = [&](int cc) -> DsScales<CB> {
        DsScales<CB> s;
#pragma unroll
        for (int i = 0; i < CB; ++i) s.raw[i] = 0u;
        s.c0 = s.c1 = 0.0f;
        s.split = CB;
        if (cc >= nchunks) return s;
        const int ti = cc / nch, ch = cc - ti * nch;
        const int n = (static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x)) * kDsRows + srow;
        if (n >= Nrows) return s;
        const int nb = min(CB, nkb - ch * CB);
        const int kbase = kb0 + ch * CB;                 // the chunk's first 64-element step
        const int rowb = n * (kblocks >> a.bshift);      // first block of row n
        const int b = rowb + (kbase >> a.bshift);
        if (a.dq) {
#pragma unroll
            for (int i = 0; i < CB; ++i)
                if (i < nb) s.raw[i] = __ldg(a.q8 + rowb + ((kbase + i) >> a.bshift));
            s.c0 = __ldg(a.cg + (b >> 8));
            s.c1 = __ldg(a.cg + ((rowb + ((kbase + nb - 1) >> a.bshift)) >> 8));
            // the first step of the chunk whose block is in the next group
            s.split = (((kbase >> a.bshift) + 256 - (b & 255)) << a.bshift) - kbase;
        } else {
#pragma unroll
            for (int i = 0; i < CB; ++i)
                if (i < nb) s.raw[i] = __float_as_uint(__ldg(a.absmax + rowb + ((kbase + i) >> a.bshift)));
        }
        return s;
    };

    // token fragments: block kbx, rolling over this warp's blocks (the same
    // blocks in every tile)
    const uint16_t *xrow[TG];
    bool xok[TG];
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
        const int m = tg * 8 + g;
        xok[tg] = m < a.M;
        xrow[tg] = a.x + static_cast<int64_t>(xok[tg] ? m : 0) * a.K + 16 * t;
    }
    int kbx = kb0;
    auto load_x = [&](uint4 (&xa)[TG], uint4 (&xb)[TG]) {
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) {
            if (nkb > 0 && xok[tg]) {
                const uint4 *p = reinterpret_cast<const uint4 *>(xrow[tg] + kbx * 64);
                xa[tg] = __ldg(p);
                xb[tg] = __ldg(p + 1);
            } else {
                xa[tg] = make_uint4(0, 0, 0, 0);
                xb[tg] = xa[tg];
            }
        }
        kbx = (kbx + 1 == kb0 + nkb) ? kb0 : kbx + 1;
    };

    // The next kernel may start now (it waits for this one to finish before
    // it reads anything). The codes, scales and tokens read below were
    // complete before this grid was launched: the u kernel in front of it
    // triggers this launch only after its own wait on the kernel before.
    griddep_launch_dependents();

    // the first chunk and its scales
    issue(0);
    DsScales<CB> sc = load_scales(0);

    // the first two blocks' tokens
    // The lookup table is filled while the first chunks are in flight.
    // level pairs: byte b -> (bf16(level[b >> 4]) low half, bf16(level[b & 15]) high half)
    for (int idx = threadIdx.x; idx < 256 * 32; idx += kDsThreads) {
        const int b = idx >> 5, l = idx & 31;
        __nv_bfloat162 p = __floats2bfloat162_rn(c_levels[b >> 4], c_levels[b & 15]);
        *reinterpret_cast<uint32_t *>(lut_g + b * 256 + 4 * l) = *reinterpret_cast<uint32_t *>(&p);
    }
    __syncthreads();

    uint4 xa0[TG], xb0[TG], xa1[TG], xb1[TG];
    load_x(xa0, xb0);
    load_x(xa1, xb1);

    const uint32_t lanew = (static_cast<uint32_t>(lane) << 2) | (1u << 16);
    float acc[2][TG][4];
    int c = 0;                // this warp's next chunk
    // partial buffers: two (one barrier per tile) when a tile's partials
    // take half of the spare half-rows (M <= 8), else one
    constexpr int kParkBufs = TG == 1 ? 2 : 1;

    for (int ti = 0; ti < nt; ++ti) {
        const int tile = static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x);
        // this lane's share of the LoRA rank columns for the tile's output
        // step, fetched now so the loads are long done by then:
        // B[n][j + 16 i] for row n of half-warp (row, j)
        const int fj = lane & 15;
        const int frow = (warp & 3) + 8 * (warp >> 2) + 4 * ((lane >> 4) & 1);
        const int fn = tile * kDsRows + frow;
        float bq[kDsMaxRank / 16];
#pragma unroll
        for (int i = 0; i < kDsMaxRank / 16; ++i) {
            const int q = fj + 16 * i;
            bq[i] = (fn < Nrows && q < a.r)
                        ? __uint_as_float(static_cast<uint32_t>(__ldg(a.B + static_cast<int64_t>(fn) * a.r + q)) << 16)
                        : 0.0f;
        }
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[rg][tg][e] = 0.0f;

        for (int ch = 0; ch < nch; ++ch, ++c) {
            // this chunk's block scales for this lane's row, then the next
            // chunk's raw values
            float s_blk[CB];
            {
                float kg0 = 0.0f, kg1 = 0.0f;
                if (a.dq) {
                    kg0 = __fdiv_rn(sc.c0, 127.0f);
                    kg1 = sc.split < CB ? __fdiv_rn(sc.c1, 127.0f) : kg0;
                }
#pragma unroll
                for (int i = 0; i < CB; ++i)
                    s_blk[i] = a.dq ? __fmul_rn(static_cast<float>(sc.raw[i]), i < sc.split ? kg0 : kg1)
                                    : __uint_as_float(sc.raw[i]);
            }
            sc = load_scales(c + 1);
            if (!mbar_wait(&bars[warp * 2 + (c & 1)], static_cast<uint32_t>(c >> 1) & 1u, abort_flag))
                goto done;
            // the next chunk goes out as soon as this one has landed, into the
            // slot of the chunk before, which every lane has finished reading:
            // at start-up each SM first fetches one chunk per warp, so the
            // first tile's data arrives before the rest of the burst
            issue(c + 1);
            const uint32_t cbase = ((c & 1) ? slot1 : slot0) + static_cast<uint32_t>(g) * kRowStride + 8u * t +
                                   after_wait_zero();
            const int nbc = min(CB, nkb - ch * CB);
            // one block of the chunk: i is a constant after inlining
            auto block = [&](const int i) {
                // s[rg][hi] (rows rg*16 + g + 8 hi) comes from lane (g, 2 rg + hi)
                float s[2][2];
#pragma unroll
                for (int rg = 0; rg < 2; ++rg)
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi)
                        s[rg][hi] = __shfl_sync(0xffffffffu, s_blk[i], (lane & ~3) | (2 * rg + hi));

                uint2 cw[2][2];    // [rg][hi]: code bytes [8t, 8t+8) of row rg*16 + g + 8 hi
#pragma unroll
                for (int rg = 0; rg < 2; ++rg)
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi)
                        cw[rg][hi] = ds_lds64(cbase + (rg * 16 + 8 * hi) * kRowStride + i * 32);

                float pp[2][TG][4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // MMA q covers elements 16t + 4q + {0,1} (slots 2t, 2t+1) and
                    // 16t + 4q + {2,3} (slots 2t+8, 2t+9): code bytes 2q and 2q+1
                    uint32_t b0[TG], b1[TG];
#pragma unroll
                    for (int tg = 0; tg < TG; ++tg) {
                        const uint4 &xv = (q < 2) ? xa0[tg] : xb0[tg];
                        b0[tg] = (q & 1) ? xv.z : xv.x;
                        b1[tg] = (q & 1) ? xv.w : xv.y;
                    }
#pragma unroll
                    for (int rg = 0; rg < 2; ++rg) {
                        const uint32_t wl = (q < 2) ? cw[rg][0].x : cw[rg][0].y;
                        const uint32_t wh = (q < 2) ? cw[rg][1].x : cw[rg][1].y;
                        uint32_t af[4];
                        if (q & 1) {
                            af[0] = ds_lut(ds_addr<2>(wl, lanew));
                            af[1] = ds_lut(ds_addr<2>(wh, lanew));
                            af[2] = ds_lut(ds_addr<3>(wl, lanew));
                            af[3] = ds_lut(ds_addr<3>(wh, lanew));
                        } else {
                            af[0] = ds_lut(ds_addr<0>(wl, lanew));
                            af[1] = ds_lut(ds_addr<0>(wh, lanew));
                            af[2] = ds_lut(ds_addr<1>(wl, lanew));
                            af[3] = ds_lut(ds_addr<1>(wh, lanew));
                        }
#pragma unroll
                        for (int tg = 0; tg < TG; ++tg) {
                            if (q == 0) ds_mma_zero(pp[rg][tg], af, b0[tg], b1[tg]);
                            else mma_bf16_16816(pp[rg][tg], af, b0[tg], b1[tg]);
                        }
                    }
                }
#pragma unroll
                for (int rg = 0; rg < 2; ++rg)
#pragma unroll
                    for (int tg = 0; tg < TG; ++tg) {
                        acc[rg][tg][0] = fmaf(s[rg][0], pp[rg][tg][0], acc[rg][tg][0]);
                        acc[rg][tg][1] = fmaf(s[rg][0], pp[rg][tg][1], acc[rg][tg][1]);
                        acc[rg][tg][2] = fmaf(s[rg][1], pp[rg][tg][2], acc[rg][tg][2]);
                        acc[rg][tg][3] = fmaf(s[rg][1], pp[rg][tg][3], acc[rg][tg][3]);
                    }
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    xa0[tg] = xa1[tg];
                    xb0[tg] = xb1[tg];
                }
                load_x(xa1, xb1);
            };
            if (nbc == CB) {
#pragma unroll
                for (int i = 0; i < CB; ++i) block(i);
            } else {
                for (int i = 0; i < nbc; ++i) block(i);
            }
            __syncwarp();        // every lane has read the chunk
        }

        // ---- the tile's k-split partials -> one ordered sum with the LoRA
        // term, then the output. Each warp parks its partial in the free
        // halves of the table rows, [warp][rg][tg][e] x 32 lanes, the lane
        // index rotated by the warp index; half-warp (row, j) then holds warp
        // j's partial in lane j, and a four-step butterfly adds the sixteen
        // in a fixed order.
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int pr = (ti % kParkBufs) * 128 + warp * (8 * TG) + (rg * TG + tg) * 4 + e;
                    *reinterpret_cast<float *>(lut_g + pr * 256 + 128 + 4 * ((lane + warp) & 31)) =
                        acc[rg][tg][e];
                }
        if (ti == 0) {
            // u = x A^T from the u kernel's partials, summed in order; the
            // up-projection uses bf16((alpha/r) u)
            griddep_wait();
            for (int cc = threadIdx.x; cc < a.M * a.r; cc += kDsThreads) {
                float u = 0.0f;
#pragma unroll
                for (int j = 0; j < kDsUCtas; ++j) u += a.upart[j * a.M * a.r + cc];
                if (a.u_out && blockIdx.x == 0) a.u_out[cc] = u;
                float sc = a.scale;
                if constexpr (GROUPS) {
                    const int gp = grp.row_group[cc / a.r];
                    const bool keep = gp >= 0 && gp < grp.ngroups && (cc % a.r) / grp.group_width == gp;
                    sc = keep ? grp.gscale[gp] : 0.0f;
                }
                __nv_bfloat16 ub = __float2bfloat16_rn(__fmul_rn(sc, u));
                u_tile[cc] = *reinterpret_cast<uint16_t *>(&ub);
            }
        }
        __syncthreads();
        {
            // rows (frow, frow + 4) share a warp, so the two halves read
            // disjoint banks of the rotated partials
            const int rg = frow >> 4, rr = frow & 15;
#pragma unroll
            for (int m = 0; m < 8 * TG; ++m) {
                if (m >= a.M) break;
                const int tg = m >> 3, tt = m & 7;
                const int e = (rr >> 3) * 2 + (tt & 1);
                const int ln = (rr & 7) * 4 + (tt >> 1);
                const int pr = (ti % kParkBufs) * 128 + fj * (8 * TG) + (rg * TG + tg) * 4 + e;
                float v = *reinterpret_cast<const float *>(lut_g + pr * 256 + 128 + 4 * ((ln + fj) & 31));
#pragma unroll
                for (int i = 0; i < kDsMaxRank / 16; ++i) {
                    const int q = fj + 16 * i;
                    if (q < a.r) v = fmaf(__uint_as_float(static_cast<uint32_t>(u_tile[m * a.r + q]) << 16), bq[i], v);
                }
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                if (fj == 0 && fn < Nrows) {
                    __nv_bfloat16 hb = __float2bfloat16_rn(v);
                    a.h[static_cast<int64_t>(m) * a.N + fn] = *reinterpret_cast<uint16_t *>(&hb);
                }
            }
        }
        // with one buffer, the partials are consumed before they are rewritten;
        // with two, the next tile's barrier orders this tile's reads before
        // the tile after it parks here again
        if (kParkBufs == 1) __syncthreads();
    }
done:
    // Leave no copy in flight into shared memory this CTA is about to release.
    // The only wait of the loop is on chunk c, and chunk c + 1 is issued only
    // after it succeeds, so after giving up there, chunk c is the one copy
    // that may still be landing (after a normal end, c == nchunks).
    if (lane == 0 && c < nchunks)
        mbar_drain(&bars[warp * 2 + (c & 1)], static_cast<uint32_t>(c >> 1) & 1u);
    __syncwarp();
}

// ---------------------------------------------------------------------------
// u = x A^T for the decode path, as kDsUCtas partial sums over contiguous k
// ranges (CTA j writes upart[j][m][rank]). The decode grid leaves kDsUCtas
// SMs free for these CTAs, so they run beside the weight stream; the decode
// kernel adds the partials in order of j when it first needs u.
//
// Within a CTA the 16 warps split the CTA's k blocks into contiguous
// shares. A warp multiplies with the ranks as the MMA rows and the tokens as
// its columns (m16n8k16; per block thread t covers elements [16t, 16t + 16),
// four MMAs); the sixteen warp partials go to shared memory, the lane index
// rotated by the warp index, and half-warp (output, j) adds them in warp
// order with a butterfly. Rank groups of 16 are done kPerRound at a time so
// that the partials fit 256 rows of 32 floats.
// ---------------------------------------------------------------------------
constexpr int kDsUParkBytes = 256 * 32 * 4;

template <int TG>
__global__ void __launch_bounds__(kDsThreads, 1)
qlora_decode_u_kernel(const DecodeArgs a, const uint8_t *__restrict__ keep, const DropRng rng) {
    extern __shared__ __align__(16) float upark[];     // [256][32]
    // x may come from the kernel before this one
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int kblocks = static_cast<int>(a.K / kBlock);
    const int lo = static_cast<int>(static_cast<int64_t>(kblocks) * blockIdx.x / gridDim.x);
    const int hi = static_cast<int>(static_cast<int64_t>(kblocks) * (blockIdx.x + 1) / gridDim.x);
    const int kb_lo = lo + (hi - lo) * warp / kDsWarps, kb_hi = lo + (hi - lo) * (warp + 1) / kDsWarps;
    float *out = a.upart + static_cast<int64_t>(blockIdx.x) * a.M * a.r;

    const uint16_t *xrow[TG];
    bool xok[TG];
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
        const int m = tg * 8 + g;
        xok[tg] = m < a.M;
        xrow[tg] = a.x + static_cast<int64_t>(xok[tg] ? m : 0) * a.K + 16 * t;
    }
    constexpr int kPerRound = 4 / TG;    // 16 warps x kPerRound x TG x 4 rows = 256
    const int nrg = (a.r + 15) / 16;
    for (int rg0 = 0; rg0 < nrg; rg0 += kPerRound) {
        float ua[kPerRound][TG][4];
#pragma unroll
        for (int p = 0; p < kPerRound; ++p)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) ua[p][tg][e] = 0.0f;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
            uint4 xa[TG], xb[TG];
#pragma unroll
            for (int tg = 0; tg < TG; ++tg) {
                if (xok[tg]) {
                    const uint4 *px = reinterpret_cast<const uint4 *>(xrow[tg] + kb * 64);
                    xa[tg] = __ldg(px);
                    xb[tg] = __ldg(px + 1);
                    if (keep || rng.on) {
                        // LoRA dropout: zero the dropped tokens' elements (16 k: two keep
                        // bytes of the mask, or drawn from the generator)
                        const int m = tg * 8 + g;
                        const int64_t e = static_cast<int64_t>(m) * a.K + kb * 64 + 16 * t;
                        const uint32_t kbits =
                            rng.on ? static_cast<uint32_t>(drop_keep_bits<4>(rng, static_cast<uint64_t>(e)))
                                   : (keep[e >> 3] | (static_cast<uint32_t>(keep[(e >> 3) + 1]) << 8));
                        uint32_t w[8] = {xa[tg].x, xa[tg].y, xa[tg].z, xa[tg].w,
                                         xb[tg].x, xb[tg].y, xb[tg].z, xb[tg].w};
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            w[i] &= ((kbits >> (2 * i)) & 1u ? 0x0000ffffu : 0u) |
                                    ((kbits >> (2 * i + 1)) & 1u ? 0xffff0000u : 0u);
                        xa[tg] = make_uint4(w[0], w[1], w[2], w[3]);
                        xb[tg] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                } else {
                    xa[tg] = make_uint4(0, 0, 0, 0);
                    xb[tg] = xa[tg];
                }
            }
#pragma unroll
            for (int p = 0; p < kPerRound; ++p) {
                if (rg0 + p >= nrg) break;
                // rank rows j0 = 16 (rg0 + p) + g and j0 + 8, elements [16t, 16t + 16) of the block
                const int j0 = (rg0 + p) * 16 + g;
                uint4 ag[2], ah[2];
                if (j0 < a.r) {
                    const uint4 *pa = reinterpret_cast<const uint4 *>(a.A + static_cast<int64_t>(j0) * a.K + kb * 64 + 16 * t);
                    ag[0] = __ldg(pa);
                    ag[1] = __ldg(pa + 1);
                } else {
                    ag[0] = ag[1] = make_uint4(0, 0, 0, 0);
                }
                if (j0 + 8 < a.r) {
                    const uint4 *pa = reinterpret_cast<const uint4 *>(a.A + static_cast<int64_t>(j0 + 8) * a.K + kb * 64 + 16 * t);
                    ah[0] = __ldg(pa);
                    ah[1] = __ldg(pa + 1);
                } else {
                    ah[0] = ah[1] = make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // MMA q: element pairs 2q (slots 2t, 2t+1) and 2q + 1 (slots 2t+8, 2t+9)
                    const uint4 &gq = ag[q >> 1], &hq = ah[q >> 1];
                    uint32_t af[4];
                    af[0] = (q & 1) ? gq.z : gq.x;
                    af[1] = (q & 1) ? hq.z : hq.x;
                    af[2] = (q & 1) ? gq.w : gq.y;
                    af[3] = (q & 1) ? hq.w : hq.y;
#pragma unroll
                    for (int tg = 0; tg < TG; ++tg) {
                        const uint4 &xv = (q < 2) ? xa[tg] : xb[tg];
                        mma_bf16_16816(ua[p][tg], af, (q & 1) ? xv.z : xv.x, (q & 1) ? xv.w : xv.y);
                    }
                }
            }
        }
        // park [warp][p][tg][e] x 32 lanes, the lane rotated by the warp index
#pragma unroll
        for (int p = 0; p < kPerRound; ++p)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int hr = ((warp * kPerRound + p) * TG + tg) * 4 + e;
                    upark[hr * 32 + ((lane + warp) & 31)] = ua[p][tg][e];
                }
        __syncthreads();
        // half-warp (output o, lane j) holds warp j's partial of output o:
        // o = m * 16 kPerRound + (rank - 16 rg0)
        const int j = lane & 15;
        for (int o0 = 0; o0 < a.M * 16 * kPerRound; o0 += 2 * kDsWarps) {
            const int o = o0 + (threadIdx.x >> 4);
            const int m = o / (16 * kPerRound), jj = o - m * (16 * kPerRound);
            const int p = jj >> 4, jr = jj & 15, rank = (rg0 + p) * 16 + jr;
            const bool ok = m < a.M && rg0 + p < nrg && rank < a.r;
            float v = 0.0f;
            if (ok) {
                const int tg = m >> 3, tt = m & 7;
                const int ln = (jr & 7) * 4 + (tt >> 1), e = (jr >> 3) * 2 + (tt & 1);
                const int hr = ((j * kPerRound + p) * TG + tg) * 4 + e;
                v = upark[hr * 32 + ((ln + j) & 31)];
            }
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            if (ok && j == 0) out[m * a.r + rank] = v;
        }
        __syncthreads();      // the rows are free again
    }
}

}  // namespace nf4
