// decode2.cuh -- the forward of the QLoRA layer for a handful of tokens
// (M <= 16): h = x W~^T + bf16((alpha/r) x A^T) B^T, streaming the 4-bit
// weight once from HBM ("QLoRA Finetuner", flowchart "Quantized Base
// Inference": load 4-bit indices and 32-bit block scales, dequantise,
// multiply).
//
// The weight dominates the bytes (n*k/2 code bytes against a few KB of
// tokens), so the kernel is HBM-bound when each code byte costs only a few
// instructions. The design keeps that count low:
//   * persistent CTAs of 16 warps, one per SM, walk tiles of 32 weight rows;
//     the 16 warps of a CTA split k sixteen ways, and each warp covers both
//     16-row groups of the tile, so one load of a token fragment serves 32
//     weight rows;
//   * a byte of codes becomes a pair of bf16 levels through a 256-entry table
//     in shared memory whose entry b, copy l sits at address
//     65536 + 256 b + 4 l: one byte permute turns (code byte, lane) into the
//     lookup address, and lane l always reads copy l (no bank conflicts);
//   * the 16 x 8 x 16 products run on the tensor cores (mma.sync, the
//     dequantised fragment goes straight from registers to the MMA);
//   * each 64-element block's partial product is scaled by its block scale
//     in fp32 and accumulated, so no per-element multiply by the scale;
//   * the codes, scales and token fragments of the next block are loaded
//     while the current one is multiplied.
// Numerically this forms sum_b s_b * sum_k bf16(level) * x, which differs
// from bf16(s_b * level) * x by at most one bf16 rounding of each term.
#pragma once

#include "decode.cuh"

namespace nf4 {

constexpr int kDc2Warps = 16;                  // k split across the warps of a CTA
constexpr int kDc2Threads = 32 * kDc2Warps;
constexpr int kDc2Rows = 32;                   // weight rows per tile (two 16-row MMA groups)
constexpr int kDc2MaxRank = 64;
constexpr uint32_t kDc2LutAddr = 65536;        // shared address of the level-pair table
constexpr int kDc2SmemBytes = 2 * 65536;       // covers [start, start + 128 KB) for start <= 64 KB
// low region (below the table): k-split partials, the tile's rows of B, u
constexpr int kDc2PartFloats = kDc2Warps * 2 * 2 * 4 * 32;   // [ks][rg][tg][e][lane]
constexpr int kDc2BtileOff = kDc2PartFloats * 4;             // bytes
constexpr int kDc2UtileOff = kDc2BtileOff + kDc2Rows * kDc2MaxRank * 2;
constexpr int kDc2LowBytes = kDc2UtileOff + 16 * kDc2MaxRank * 2;

struct Decode2Args {
    int M;                 // tokens (1..16)
    int64_t N, K;          // weight rows / columns
    int r;
    const uint8_t *codes;
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    const uint16_t *x;     // [M, K]
    const uint16_t *B;     // [N, r]
    const uint16_t *u_s;   // [M, r] bf16((alpha/r) x A^T), written by the preceding kernel
    uint16_t *h;           // [M, N]
};

constexpr uint32_t kDc2RingAddr = 2 * 65536;   // shared address of the per-warp code rings
constexpr int kDc2Slots = 4;                   // blocks in flight per warp
constexpr int kDc2SlotBytes = kDc2Rows * 32;   // one block of codes of the tile's 32 rows
constexpr int kDc2DynBytes = 3 * 65536;        // table at 64 KB, rings at 128 KB
static_assert(kDc2RingAddr + kDc2Warps * kDc2Slots * kDc2SlotBytes <= 3 * 65536, "ring fits");
static_assert(kDc2LowBytes <= 60 * 1024, "low region stays below the table (checked against the start at run time)");

// Table lookup by address. The table is written once before a barrier and
// never again, and every lookup address is derived from code words read
// after that barrier, so the load needs no ordering constraint of its own.
__device__ __forceinline__ uint32_t dc2_lut(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
// Ring loads: the "memory" clobber keeps them after the copy wait.
__device__ __forceinline__ uint2 dc2_lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}
// 16-byte asynchronous copy global -> shared; src_bytes == 0 writes zeros
__device__ __forceinline__ void dc2_cp16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void dc2_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void dc2_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Lookup address of code byte I of word w for this lane: byte 0 = 4 lane,
// byte 1 = the code byte, byte 2 = 1 (the table's 64 KB base). Selector
// nibble k picks output byte k from {lanew (bytes 4..7), w (bytes 0..3)}:
// nibbles (from byte 3 down) 7, 6, I, 4.
template <int I>
__device__ __forceinline__ uint32_t dc2_addr(uint32_t w, uint32_t lanew) {
    static_assert(I >= 0 && I < 4, "code byte");
    return prmt(w, lanew, 0x7604u | (static_cast<uint32_t>(I) << 4));
}

// d = a b (m16n8k16, bf16 inputs, fp32 result, zero accumulator in)
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                 uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// Raw scale of one (row, block): q8 and c_g (double quantisation) or absmax.
struct Dc2Raw {
    uint32_t q8;
    float v;
};

__device__ __forceinline__ Dc2Raw dc2_load_scale(const Decode2Args &a, bool valid, int b) {
    Dc2Raw r{0u, 0.0f};
    if (!valid) return r;
    if (a.dq) {
        r.q8 = __ldg(a.q8 + b);
        r.v = __ldg(a.cg + (b >> 8));
    } else {
        r.v = __ldg(a.absmax + b);
    }
    return r;
}

// TG = number of 8-token groups (1 for M <= 8, 2 for M <= 16).
//
// Fragment bookkeeping (m16n8k16, thread (g, t) = (lane / 4, lane % 4)): the
// A fragment holds rows g and g+8 of a 16-row group and four k slots per
// row; the reduction order inside one MMA is free, so the slots are chosen
// such that thread t's slots over a block's four MMAs are the 16 consecutive
// elements [16t, 16t+16) of the block: code bytes [8t, 8t+8) of each of its
// rows, and 16 consecutive x values per token.
template <int TG>
__global__ void __launch_bounds__(kDc2Threads, 1) qlora_decode2_kernel(const Decode2Args a) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    const uint32_t sbase = smem_u32(dsm);
    if (sbase + kDc2LowBytes > kDc2LutAddr) {      // the fixed table address is not ours
        if (threadIdx.x == 0) record_status(NF4_ERR_CUDA);
        return;
    }
    float *part = reinterpret_cast<float *>(dsm);                        // [ks][rg][tg][e][lane]
    uint16_t *u_tile = reinterpret_cast<uint16_t *>(dsm + kDc2UtileOff); // [M][r]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    // level pairs: byte b -> (bf16(level[b >> 4]) low half, bf16(level[b & 15]) high half),
    // 32 copies at 256-byte stride
    {
        uint32_t *lut = reinterpret_cast<uint32_t *>(dsm + (kDc2LutAddr - sbase));
        for (int idx = threadIdx.x; idx < 256 * 32; idx += kDc2Threads) {
            const int b = idx >> 5, l = idx & 31;
            __nv_bfloat162 p = __floats2bfloat162_rn(c_levels[b >> 4], c_levels[b & 15]);
            lut[b * 64 + l] = *reinterpret_cast<uint32_t *>(&p);
        }
    }
    __syncthreads();

    const int64_t kblocks = a.K / kBlock;
    const int ks = warp;
    const int kb0 = static_cast<int>(kblocks * ks / kDc2Warps);
    const int kb1 = static_cast<int>(kblocks * (ks + 1) / kDc2Warps);
    const int nkb = kb1 - kb0;
    const int ntiles = static_cast<int>((a.N + kDc2Rows - 1) / kDc2Rows);
    const int Nrows = static_cast<int>(a.N);
    const int kbl = static_cast<int>(kblocks);   // n * kbl + kb < 2^31 (checked by the host)
    const int nt = blockIdx.x < ntiles
                       ? static_cast<int>((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x)
                       : 0;
    const int njobs = nt * nkb;                    // (tile, block) pairs of this warp
    const uint32_t lanew = (static_cast<uint32_t>(lane) << 2) | (1u << 16);
    const uint32_t ring = kDc2RingAddr + static_cast<uint32_t>(warp) * (kDc2Slots * kDc2SlotBytes);
    const int64_t krow = a.K / 2;                  // code bytes per weight row

    // Jobs are the (tile, block) pairs of this warp in order: block kb0..kb1-1
    // of tile blockIdx.x, then of tile blockIdx.x + gridDim.x, ... Three
    // cursors walk them incrementally: the job whose codes are being issued
    // (3 ahead), the job whose scales and tokens are being loaded (2 ahead)
    // and the current job.
    struct Cursor {
        int tile;
        int kb;
    };
    auto advance = [&](Cursor &c) {
        if (++c.kb == kb1) {
            c.kb = kb0;
            c.tile += gridDim.x;
        }
    };
    auto at_job = [&](int jj) -> Cursor {   // start-up only
        Cursor c{blockIdx.x, kb0};
        for (int q = 0; q < jj; ++q) advance(c);
        return c;
    };

    // codes: 64 copies of 16 bytes per job (two per lane: rows lane/2 and 16 + lane/2)
    const int crow = lane >> 1, chalf = lane & 1;
    Cursor ci = at_job(0);
    const uint8_t *csrc[2] = {nullptr, nullptr};
    bool cok[2] = {false, false};
    int ctile = -1;
    uint32_t ji = 0;          // jobs issued so far; job ji goes to slot ji % kDc2Slots
    auto issue = [&]() {
        if (nkb > 0 && ci.tile < ntiles) {
            if (ci.tile != ctile) {
                ctile = ci.tile;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int n = ctile * kDc2Rows + crow + 16 * c2;
                    cok[c2] = n < Nrows;
                    csrc[c2] = a.codes + (cok[c2] ? static_cast<int64_t>(n) * krow : 0) + chalf * 16;
                }
            }
            const uint32_t slot = ring + (ji % kDc2Slots) * kDc2SlotBytes;
            ++ji;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2)
                dc2_cp16(slot + (crow + 16 * c2) * 32 + chalf * 16, csrc[c2] + ci.kb * 32, cok[c2] ? 16u : 0u);
            advance(ci);
        }
        dc2_commit();
    };
    // scales and tokens: cursor two jobs ahead
    const int srow = (t >> 1) * 16 + g + 8 * (t & 1);   // this lane's scale row in the tile
    Cursor cs = at_job(0);
    int stile = -1, sbrow = 0;
    bool sok = false;
    auto scale_raw = [&]() -> Dc2Raw {
        if (nkb == 0 || cs.tile >= ntiles) return Dc2Raw{0u, 0.0f};
        if (cs.tile != stile) {
            stile = cs.tile;
            const int n = stile * kDc2Rows + srow;
            sok = n < Nrows;
            sbrow = n * kbl;
        }
        return dc2_load_scale(a, sok, sbrow + cs.kb);
    };
    const uint16_t *xrow[TG];
    bool xok[TG];
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
        const int m = tg * 8 + g;
        xok[tg] = m < a.M;
        xrow[tg] = a.x + static_cast<int64_t>(xok[tg] ? m : 0) * a.K + 16 * t;
    }
    auto load_x = [&](uint4 (&xa)[TG], uint4 (&xb)[TG]) {
        const bool live = nkb > 0 && cs.tile < ntiles;
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) {
            if (live && xok[tg]) {
                const uint4 *p = reinterpret_cast<const uint4 *>(xrow[tg] + cs.kb * 64);
                xa[tg] = __ldg(p);
                xb[tg] = __ldg(p + 1);
            } else {
                xa[tg] = make_uint4(0, 0, 0, 0);
                xb[tg] = xa[tg];
            }
        }
    };

    // prologue: codes of the first kDc2Slots - 1 jobs, scales and tokens of the first two
#pragma unroll
    for (int p = 0; p < kDc2Slots - 1; ++p) issue();
    uint4 xa0[TG], xb0[TG], xa1[TG], xb1[TG];
    Dc2Raw rs0 = scale_raw();
    load_x(xa0, xb0);
    if (nkb > 0) advance(cs);
    Dc2Raw rs1 = scale_raw();
    load_x(xa1, xb1);
    if (nkb > 0) advance(cs);
    int cur_brow = 0;         // (row of this lane's scale) * blocks per row, current tile
    int kg_group = -1;        // cached fl32(c_g / 127) of this lane's scale row
    float kg = 0.0f;
    bool lora_ready = false;

    float acc[2][TG][4];
#pragma unroll
    for (int rg = 0; rg < 2; ++rg)
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[rg][tg][e] = 0.0f;

    // one job: the current block of the current tile; its scales and token
    // fragments arrive in (rs, xa, xb), which are then refilled for the job
    // two places later
    int ti = 0, kbi = 0;      // position of the current job
    auto job = [&](int j, Dc2Raw &rs, uint4 (&xa)[TG], uint4 (&xb)[TG]) {
        issue();
        float s_mine = 0.0f;
        if (a.dq) {
            const int grp = (cur_brow + kb0 + kbi) >> 8;
            if (grp != kg_group) {
                kg_group = grp;
                kg = __fdiv_rn(rs.v, 127.0f);
            }
            s_mine = __fmul_rn(static_cast<float>(rs.q8), kg);
        } else {
            s_mine = rs.v;
        }
        // s[rg][hi] comes from lane (g, 2 rg + hi)
        float s[2][2];
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                s[rg][hi] = __shfl_sync(0xffffffffu, s_mine, (lane & ~3) | (2 * rg + hi));

        dc2_wait<kDc2Slots - 1>();
        __syncwarp();
        const uint32_t slot = ring + (static_cast<uint32_t>(j) % kDc2Slots) * kDc2SlotBytes;
        uint2 cw[2][2];    // [rg][hi]: code bytes [8t, 8t+8) of row rg*16 + g + 8 hi
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                cw[rg][hi] = dc2_lds64(slot + (rg * 16 + g + 8 * hi) * 32 + 8 * t);

        float pp[2][TG][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // MMA i covers elements 16t + 4i + {0,1} (slots 2t, 2t+1) and
            // 16t + 4i + {2,3} (slots 2t+8, 2t+9): code bytes 2i and 2i+1
            uint32_t b0[TG], b1[TG];
#pragma unroll
            for (int tg = 0; tg < TG; ++tg) {
                const uint4 &q = (i < 2) ? xa[tg] : xb[tg];
                b0[tg] = (i & 1) ? q.z : q.x;
                b1[tg] = (i & 1) ? q.w : q.y;
            }
#pragma unroll
            for (int rg = 0; rg < 2; ++rg) {
                const uint32_t wl = (i < 2) ? cw[rg][0].x : cw[rg][0].y;
                const uint32_t wh = (i < 2) ? cw[rg][1].x : cw[rg][1].y;
                uint32_t af[4];
                if (i & 1) {
                    af[0] = dc2_lut(dc2_addr<2>(wl, lanew));
                    af[1] = dc2_lut(dc2_addr<2>(wh, lanew));
                    af[2] = dc2_lut(dc2_addr<3>(wl, lanew));
                    af[3] = dc2_lut(dc2_addr<3>(wh, lanew));
                } else {
                    af[0] = dc2_lut(dc2_addr<0>(wl, lanew));
                    af[1] = dc2_lut(dc2_addr<0>(wh, lanew));
                    af[2] = dc2_lut(dc2_addr<1>(wl, lanew));
                    af[3] = dc2_lut(dc2_addr<1>(wh, lanew));
                }
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    if (i == 0) mma_bf16_16816_z(pp[rg][tg], af, b0[tg], b1[tg]);
                    else mma_bf16_16816(pp[rg][tg], af, b0[tg], b1[tg]);
                }
            }
        }
        __syncwarp();      // every lane has read the slot before it is refilled
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg) {
                acc[rg][tg][0] = fmaf(s[rg][0], pp[rg][tg][0], acc[rg][tg][0]);
                acc[rg][tg][1] = fmaf(s[rg][0], pp[rg][tg][1], acc[rg][tg][1]);
                acc[rg][tg][2] = fmaf(s[rg][1], pp[rg][tg][2], acc[rg][tg][2]);
                acc[rg][tg][3] = fmaf(s[rg][1], pp[rg][tg][3], acc[rg][tg][3]);
            }
        rs = scale_raw();
        load_x(xa, xb);
        advance(cs);
    };

    // the tile's k-split partials -> ordered sum, LoRA term, output
    auto finish_tile = [&]() {
        const int tile = blockIdx.x + ti * gridDim.x;
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    part[(((ks * 2 + rg) * 2 + tg) * 4 + e) * 32 + lane] = acc[rg][tg][e];
                    acc[rg][tg][e] = 0.0f;
                }
        if (!lora_ready) {
            // bf16((alpha/r) x A^T) comes from the preceding kernel
            griddep_wait();
            griddep_launch_dependents();
            for (int c = threadIdx.x; c < a.M * a.r; c += kDc2Threads) u_tile[c] = a.u_s[c];
            lora_ready = true;
        }
        __syncthreads();
        {
            const int row = threadIdx.x >> 4, token = threadIdx.x & 15;
            const int n = tile * kDc2Rows + row;
            if (token < a.M && n < Nrows) {
                const int rg = row >> 4, rr = row & 15, tg = token >> 3, tt = token & 7;
                const int e = (rr >> 3) * 2 + (tt & 1);
                const int ln = (rr & 7) * 4 + (tt >> 1);
                float sum = 0.0f;
#pragma unroll 4
                for (int w = 0; w < kDc2Warps; ++w)
                    sum += part[(((w * 2 + rg) * 2 + tg) * 4 + e) * 32 + ln];
                // LoRA term sum_j u[token][j] B[n][j], eight bf16 at a time (r % 8 == 0)
                float lora = 0.0f;
                const uint4 *br = reinterpret_cast<const uint4 *>(a.B + static_cast<int64_t>(n) * a.r);
                const uint4 *ur = reinterpret_cast<const uint4 *>(u_tile + token * a.r);
                for (int c8 = 0; c8 < a.r / 8; ++c8) {
                    const uint4 bv = __ldg(br + c8), uv = ur[c8];
                    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        lora = fmaf(__uint_as_float(uw[q] << 16), __uint_as_float(bw[q] << 16), lora);
                        lora = fmaf(__uint_as_float(uw[q] & 0xFFFF0000u), __uint_as_float(bw[q] & 0xFFFF0000u), lora);
                    }
                }
                __nv_bfloat16 hb = __float2bfloat16_rn(sum + lora);
                a.h[static_cast<int64_t>(token) * a.N + n] = *reinterpret_cast<uint16_t *>(&hb);
            }
        }
        __syncthreads();      // partials consumed before the next tile writes them
        ++ti;
        kbi = 0;
        cur_brow = ((blockIdx.x + ti * gridDim.x) * kDc2Rows + srow) * kbl;
    };

    cur_brow = (blockIdx.x * kDc2Rows + srow) * kbl;
    if (nkb == 0) {
        while (ti < nt) finish_tile();
    } else {
        // jobs in pairs so that the two buffers alternate without copies
        for (int j = 0; j < njobs; j += 2) {
            job(j, rs0, xa0, xb0);
            if (++kbi == nkb) finish_tile();
            if (j + 1 < njobs) {
                job(j + 1, rs1, xa1, xb1);
                if (++kbi == nkb) finish_tile();
            }
        }
    }
    dc2_wait<0>();
}

}  // namespace nf4
