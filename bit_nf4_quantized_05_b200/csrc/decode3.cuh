// decode3.cuh -- the forward of the QLoRA layer for a handful of tokens
// (M <= 16): h = x W~^T + bf16((alpha/r) x A^T) B^T, streaming the 4-bit
// weight once from HBM ("QLoRA Finetuner", flowchart "Quantized Base
// Inference": load 4-bit indices and 32-bit block scales, dequantise,
// multiply).
//
// The weight dominates the bytes (n*k/2 code bytes against a few KB of
// tokens), so the kernel is built around streaming the codes:
//   * persistent CTAs of 16 warps, one per SM, walk tiles of 32 weight rows;
//     the 16 warps split k sixteen ways, and each warp covers both 16-row
//     groups of the tile, so one token-fragment load serves 32 weight rows;
//   * each warp fetches its k range of a tile -- 32 rows x up to five blocks,
//     a run of up to 160 contiguous bytes per row -- with one 2-D TMA copy
//     into a two-slot ring, so the next chunk streams in while the current
//     one is multiplied;
//   * a byte of codes becomes a pair of bf16 levels through a 256-entry table
//     in shared memory whose entry b, copy l sits at address
//     32768 + 128 b + 4 l: one byte permute and one shift turn (code byte,
//     lane) into the lookup address, and lane l always reads copy l (no bank
//     conflicts);
//   * the 16 x 8 x 16 products run on the tensor cores (mma.sync, the
//     dequantised fragment goes straight from registers to the MMA);
//   * each 64-element block's partial product is scaled by its block scale
//     in fp32 and accumulated, so no per-element multiply by the scale; one
//     of the four lanes that share a row forms each (row, block) scale and
//     shuffles it to the others.
// Numerically this forms sum_b s_b * sum_k bf16(level) * x, which differs
// from bf16(s_b * level) * x by at most one bf16 rounding of each term.
#pragma once

#include "decode.cuh"

namespace nf4 {

constexpr int kDc3Warps = 16;                  // k split across the warps of a CTA
constexpr int kDc3Threads = 32 * kDc3Warps;
constexpr int kDc3Rows = 32;                   // weight rows per tile (two 16-row MMA groups)
constexpr int kDc3MaxRank = 64;
constexpr int kDc3MaxChunk = 5;                // blocks per TMA chunk (160 bytes per row)
constexpr uint32_t kDc3LutAddr = 32768;        // shared address of the level-pair table (32 KB)
constexpr uint32_t kDc3RingAddr = 65536;       // shared address of the per-warp chunk rings
// below the table: u (M x r bf16), then the chunk barriers and the abort flag
constexpr int kDc3UBytes = 16 * kDc3MaxRank * 2;
constexpr int kDc3LowBytes = kDc3UBytes + kDc3Warps * 2 * 8 + 16;
// the largest dynamic allocation a CTA may have on B200
constexpr int kDc3DynBytes = 227 * 1024;

struct Decode3Args {
    int M;                 // tokens (1..16)
    int64_t N, K;          // weight rows / columns
    int r;
    int rb;                // blocks per warp: ceil(K / 64 / 16)
    int cb;                // blocks per chunk (divides rb, <= kDc3MaxChunk)
    int slot_bytes;        // bytes of one ring slot: max(32 * 32 * cb, 2048)
    const float *absmax;
    const uint8_t *q8;
    const float *cg;
    int dq;
    const uint16_t *x;     // [M, K]
    const uint16_t *B;     // [N, r]
    const float *upart;    // [kDecUSplits][M][r] partial sums of x A^T, from the preceding kernel
    float scale;           // fl32(alpha / r)
    float *u_out;          // [M, r] fp32 x A^T (optional; written by CTA 0)
    uint16_t *h;           // [M, N]
};

// Table lookup by address. The table is written once before a barrier and
// never again, and every lookup address is derived from code words read
// after that barrier, so the load needs no ordering constraint of its own.
__device__ __forceinline__ uint32_t dc3_lut(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
// Ring loads: the "memory" clobber keeps them after the chunk barrier wait.
__device__ __forceinline__ uint2 dc3_lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

// Lookup address of code byte I of word w for this lane: the byte permute
// builds 65536 + 256 b + 8 lane (byte 0 = 8 lane, byte 1 = the code byte,
// byte 2 = 1), and the shift halves it to 32768 + 128 b + 4 lane. Selector
// nibble k picks output byte k from {lanew (bytes 4..7), w (bytes 0..3)}:
// nibbles (from byte 3 down) 7, 6, I, 4.
template <int I>
__device__ __forceinline__ uint32_t dc3_addr(uint32_t w, uint32_t lanew) {
    static_assert(I >= 0 && I < 4, "code byte");
    return prmt(w, lanew, 0x7604u | (static_cast<uint32_t>(I) << 4)) >> 1;
}

// d = a b (m16n8k16, bf16 inputs, fp32 result, zero accumulator in)
__device__ __forceinline__ void mma_bf16_16816_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                    uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// Raw scale of one (row, block): q8 and c_g (double quantisation) or absmax.
struct Dc3Raw {
    uint32_t q8;
    float v;
};

__device__ __forceinline__ Dc3Raw dc3_load_scale(const Decode3Args &a, bool valid, int b) {
    Dc3Raw r{0u, 0.0f};
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
//
// Warp w takes blocks [w rb, w rb + rb) of every tile, in chunks of cb blocks
// (cb divides rb). Its chunks are numbered c = 0, 1, ... over all of the
// CTA's tiles; chunk c goes to ring slot c % 2. A slot is refilled with chunk
// c + 2 right after chunk c is consumed, except after a tile's last chunk,
// whose slot then holds the warp's k-split partial until the tile's output
// is written.
template <int TG>
__global__ void __launch_bounds__(kDc3Threads, 1)
qlora_decode3_kernel(const __grid_constant__ CUtensorMap tm_codes,   // [N, K/2] u8, box {32 cb, 32}
                     const Decode3Args a) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    const uint32_t sbase = smem_u32(dsm);
    const uint32_t ring_end = kDc3RingAddr + kDc3Warps * 2 * static_cast<uint32_t>(a.slot_bytes);
    if (sbase + kDc3LowBytes > kDc3LutAddr || ring_end > sbase + kDc3DynBytes) {
        if (threadIdx.x == 0) record_status(NF4_ERR_CUDA);   // the fixed addresses are not ours
        return;
    }
    uint16_t *u_tile = reinterpret_cast<uint16_t *>(dsm);                       // [M][r]
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsm + kDc3UBytes);           // [warp][slot]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + kDc3Warps * 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    // level pairs: byte b -> (bf16(level[b >> 4]) low half, bf16(level[b & 15]) high half),
    // 32 copies at 128-byte stride
    {
        uint32_t *lut = reinterpret_cast<uint32_t *>(dsm + (kDc3LutAddr - sbase));
        for (int idx = threadIdx.x; idx < 256 * 32; idx += kDc3Threads) {
            const int b = idx >> 5, l = idx & 31;
            __nv_bfloat162 p = __floats2bfloat162_rn(c_levels[b >> 4], c_levels[b & 15]);
            lut[b * 32 + l] = *reinterpret_cast<uint32_t *>(&p);
        }
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDc3Warps * 2; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_codes);
    }
    __syncthreads();

    const int kblocks = static_cast<int>(a.K / kBlock);
    const int Nrows = static_cast<int>(a.N);
    auto blocks_of = [&](int w) -> int {        // blocks of warp w in every tile
        const int n = kblocks - w * a.rb;
        return n < 0 ? 0 : (n > a.rb ? a.rb : n);
    };
    const int ks = warp;
    const int kb0 = ks * a.rb;
    const int nkb = blocks_of(ks);
    const int nch = (nkb + a.cb - 1) / a.cb;
    const int ntiles = (Nrows + kDc3Rows - 1) / kDc3Rows;
    const int nt = static_cast<int>(blockIdx.x) < ntiles
                       ? (ntiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                             static_cast<int>(gridDim.x)
                       : 0;
    const int nchunks = nt * nch;
    const uint32_t ring = kDc3RingAddr + static_cast<uint32_t>(warp) * 2 * a.slot_bytes;
    const uint32_t rowstride = 32u * a.cb;      // bytes per row in a slot
    uint8_t *ring_g = dsm + (ring - sbase);     // generic view of this warp's ring

    // chunk c of this warp: tile c / nch, blocks kb0 + (c % nch) cb .. +cb
    auto issue = [&](int c) {
        if (c >= nchunks) return;
        if (lane == 0) {
            const int ti = c / nch, ch = c - (c / nch) * nch;
            const int tile = static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x);
            // the slot's previous contents were read through the generic proxy
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bars[warp * 2 + (c & 1)], 32u * rowstride);
            tma_load_2d(ring_g + (c & 1) * a.slot_bytes, &tm_codes, &bars[warp * 2 + (c & 1)],
                        (kb0 + ch * a.cb) * 32, tile * kDc3Rows);
        }
    };

    // cursor over this warp's (tile, block) jobs, for the scale and token prefetch
    struct Cursor {
        int tile, kb;
    };
    auto advance = [&](Cursor &c) {
        if (++c.kb == kb0 + nkb) {
            c.kb = kb0;
            c.tile += gridDim.x;
        }
    };
    const int srow = (t >> 1) * 16 + g + 8 * (t & 1);   // this lane's scale row in the tile
    Cursor cs{static_cast<int>(blockIdx.x), kb0};
    auto scale_raw = [&]() -> Dc3Raw {
        if (nkb == 0 || cs.tile >= ntiles) return Dc3Raw{0u, 0.0f};
        const int n = cs.tile * kDc3Rows + srow;
        return dc3_load_scale(a, n < Nrows, n * kblocks + cs.kb);
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

    // prologue: the first two chunks, the scales and tokens of the first two jobs
    issue(0);
    issue(1);
    uint4 xa0[TG], xb0[TG], xa1[TG], xb1[TG];
    Dc3Raw rs0 = scale_raw();
    load_x(xa0, xb0);
    if (nkb > 0) advance(cs);
    Dc3Raw rs1 = scale_raw();
    load_x(xa1, xb1);
    if (nkb > 0) advance(cs);

    const uint32_t lanew = (static_cast<uint32_t>(lane) << 3) | (1u << 16);
    int kg_group = -1;        // cached fl32(c_g / 127) of this lane's scale row
    float kg = 0.0f;
    bool lora_ready = false;
    float acc[2][TG][4];
    int c = 0;                // this warp's next chunk

    for (int ti = 0; ti < nt; ++ti) {
        const int tile = static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x);
        const int cur_brow = (tile * kDc3Rows + srow) * kblocks;
#pragma unroll
        for (int rg = 0; rg < 2; ++rg)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[rg][tg][e] = 0.0f;

        for (int ch = 0; ch < nch; ++ch, ++c) {
            if (!mbar_wait(&bars[warp * 2 + (c & 1)], static_cast<uint32_t>(c >> 1) & 1u, abort_flag))
                goto done;
            const uint32_t slot = ring + static_cast<uint32_t>(c & 1) * a.slot_bytes;
            const int nbc = (nkb - ch * a.cb) < a.cb ? (nkb - ch * a.cb) : a.cb;
            for (int cbi = 0; cbi < nbc; ++cbi) {
                // this job's scales, then the next-but-one job's raw values
                float s_mine = 0.0f;
                if (a.dq) {
                    const int grp = (cur_brow + kb0 + ch * a.cb + cbi) >> 8;
                    if (grp != kg_group) {
                        kg_group = grp;
                        kg = __fdiv_rn(rs0.v, 127.0f);
                    }
                    s_mine = __fmul_rn(static_cast<float>(rs0.q8), kg);
                } else {
                    s_mine = rs0.v;
                }
                // s[rg][hi] comes from lane (g, 2 rg + hi)
                float s[2][2];
#pragma unroll
                for (int rg = 0; rg < 2; ++rg)
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi)
                        s[rg][hi] = __shfl_sync(0xffffffffu, s_mine, (lane & ~3) | (2 * rg + hi));

                uint2 cw[2][2];    // [rg][hi]: code bytes [8t, 8t+8) of row rg*16 + g + 8 hi
#pragma unroll
                for (int rg = 0; rg < 2; ++rg)
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi)
                        cw[rg][hi] = dc3_lds64(slot + (rg * 16 + g + 8 * hi) * rowstride + cbi * 32 + 8 * t);

                float pp[2][TG][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // MMA i covers elements 16t + 4i + {0,1} (slots 2t, 2t+1) and
                    // 16t + 4i + {2,3} (slots 2t+8, 2t+9): code bytes 2i and 2i+1
                    uint32_t b0[TG], b1[TG];
#pragma unroll
                    for (int tg = 0; tg < TG; ++tg) {
                        const uint4 &q = (i < 2) ? xa0[tg] : xb0[tg];
                        b0[tg] = (i & 1) ? q.z : q.x;
                        b1[tg] = (i & 1) ? q.w : q.y;
                    }
#pragma unroll
                    for (int rg = 0; rg < 2; ++rg) {
                        const uint32_t wl = (i < 2) ? cw[rg][0].x : cw[rg][0].y;
                        const uint32_t wh = (i < 2) ? cw[rg][1].x : cw[rg][1].y;
                        uint32_t af[4];
                        if (i & 1) {
                            af[0] = dc3_lut(dc3_addr<2>(wl, lanew));
                            af[1] = dc3_lut(dc3_addr<2>(wh, lanew));
                            af[2] = dc3_lut(dc3_addr<3>(wl, lanew));
                            af[3] = dc3_lut(dc3_addr<3>(wh, lanew));
                        } else {
                            af[0] = dc3_lut(dc3_addr<0>(wl, lanew));
                            af[1] = dc3_lut(dc3_addr<0>(wh, lanew));
                            af[2] = dc3_lut(dc3_addr<1>(wl, lanew));
                            af[3] = dc3_lut(dc3_addr<1>(wh, lanew));
                        }
#pragma unroll
                        for (int tg = 0; tg < TG; ++tg) {
                            if (i == 0) mma_bf16_16816_zero(pp[rg][tg], af, b0[tg], b1[tg]);
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
                rs0 = rs1;
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    xa0[tg] = xa1[tg];
                    xb0[tg] = xb1[tg];
                }
                rs1 = scale_raw();
                load_x(xa1, xb1);
                advance(cs);
            }
            __syncwarp();        // every lane has read the chunk
            if (ch + 1 < nch) issue(c + 2);
        }

        // ---- the tile's k-split partials -> ordered sum, LoRA term, output.
        // Each warp parks its partial [rg][tg][e][lane] in the slot of its
        // last chunk of this tile (slot 0 if it has no blocks).
        {
            float *mine = reinterpret_cast<float *>(ring_g + (nch > 0 ? ((c - 1) & 1) : 0) * a.slot_bytes);
#pragma unroll
            for (int rg = 0; rg < 2; ++rg)
#pragma unroll
                for (int tg = 0; tg < 2; ++tg)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        mine[((rg * 2 + tg) * 4 + e) * 32 + lane] = tg < TG ? acc[rg][tg][e] : 0.0f;
        }
        if (!lora_ready) {
            // u = x A^T from the preceding kernel's partials, summed in order;
            // the up-projection uses bf16((alpha/r) u)
            griddep_wait();
            griddep_launch_dependents();
            for (int cc = threadIdx.x; cc < a.M * a.r; cc += kDc3Threads) {
                float u = 0.0f;
#pragma unroll
                for (int sl = 0; sl < kDecUSplits; ++sl) u += a.upart[sl * a.M * a.r + cc];
                if (a.u_out && blockIdx.x == 0) a.u_out[cc] = u;
                __nv_bfloat16 ub = __float2bfloat16_rn(__fmul_rn(a.scale, u));
                u_tile[cc] = *reinterpret_cast<uint16_t *>(&ub);
            }
            lora_ready = true;
        }
        __syncthreads();
        {
            const int row = threadIdx.x >> 4, token = threadIdx.x & 15;
            const int n = tile * kDc3Rows + row;
            if (token < a.M && n < Nrows) {
                const int rg = row >> 4, rr = row & 15, tg = token >> 3, tt = token & 7;
                const int e = (rr >> 3) * 2 + (tt & 1);
                const int ln = (rr & 7) * 4 + (tt >> 1);
                float sum = 0.0f;
                for (int w = 0; w < kDc3Warps; ++w) {
                    const int nch_w = (blocks_of(w) + a.cb - 1) / a.cb;
                    const int slot_w = nch_w > 0 ? (((ti + 1) * nch_w - 1) & 1) : 0;
                    const float *pw = reinterpret_cast<const float *>(
                        dsm + (kDc3RingAddr - sbase) + (w * 2 + slot_w) * a.slot_bytes);
                    sum += pw[((rg * 2 + tg) * 4 + e) * 32 + ln];
                }
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
        __syncthreads();      // every partial is consumed before its slot is refilled
        if (nch > 0) issue(c + 1);   // the slot of this tile's last chunk (c - 1) takes chunk c + 1
    }
done:
    // leave no copy in flight into shared memory this CTA is about to release
    if (lane == 0) {
        for (int q = 0; q < 2; ++q) {
            const int cq = c + q;           // chunks issued but not consumed: c and c + 1
            if (cq < nchunks && cq >= 0) mbar_wait(&bars[warp * 2 + (cq & 1)], static_cast<uint32_t>(cq >> 1) & 1u, abort_flag);
        }
    }
    __syncwarp();
}

}  // namespace nf4
