/*
 * nf4_oracle.c -- plain, slow CPU oracle for the QLoRA linear layer
 * (NF4-quantized frozen weight plus a LoRA branch).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or
 * call this file: only the test suite, the package entry point's smoke check
 * and the benchmark's CPU-baseline leg use it. It shares no code, header,
 * table or constant with the CUDA library; the two are compared against each
 * other on identical seeded inputs.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC
 * (no contraction, no fast math: every float operation below is one IEEE-754
 * operation in the precision written).
 *
 * Sources (web pages; cited by title and section):
 *   [P1] "QLoRA Finetuner -- Juan Martos", sections "1. Low-Rank Adaptation
 *        (LoRA)" and "2. Block-by-Block NormalFloat4 (NF4) Quantization".
 *   [P2] "QLoRA Specification for EMEP Fine-Tuning", "NF4 Quantization" and
 *        "Hyperparameters" table.
 *   [P3] "QLoRA explained: fine-tuning in 4-bit precision", sections
 *        "Double quantization", "The LoRA adapter path" and "Common
 *        misconceptions" (the NF4 lookup table).
 *   [P4] "How Fine-Tuning LLMs with LoRA and QLoRA Works", "Merging and
 *        Deployment Strategies".
 *   [P5] "Parameter-Efficient Fine-Tuning: From LoRA to QLoRA", sections
 *        "Vanilla Uniform Quantization", "Block-Wise (Chunking) Quantization",
 *        "Pillar 1: 4-bit NormalFloat (NF4) Quantization" (level table and the
 *        numerical step-by-step example) and "Pillar 2: Double Quantization".
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   R1  normalisation w' = fl32(w / s), one IEEE fp32 division.
 *   R2  nearest level by |w' - c_j| over the 16 levels; an exact tie goes to
 *       the lower index (the more negative level).
 *   R3  an all-zero block stores s = 0 and every code is 7 (the exact zero).
 *   R4  double quantisation: groups of 256 consecutive blocks; c_g = max s_i
 *       over the group; q8_i = RNE(fl32(fl32(s_i / c_g) * 127)); dequantised
 *       scale fl32(q8_i * fl32(c_g / 127)); c_g = 0 gives q8 = 0.
 *   R5  NF4 codes are always computed against the unquantised fp32 s_i.
 *   R6  the matmul operand is RNE_bf16(fl32(scale * c[q])).
 *   R7  W0 is stored [n_out, k_in] row-major; x is [M, k_in]; A is [r, k_in];
 *       B is [n_out, r]; h = x W~^T + (alpha/r) (x A^T) B^T.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* NF4 levels as printed, to 16 digits, in [P3] "Common misconceptions"     */
/* (the NF4 lookup table). Every printed value is an exact fp32 number.     */
/* Index 0 = -1, index 7 = 0, index 15 = +1 (order as in [P5] level table). */
/* ------------------------------------------------------------------------ */
static const float NF4_LEVELS[16] = {
    -1.0f,
    -0.6961928009986877f,
    -0.5250730514526367f,
    -0.39491748809814453f,
    -0.28444138169288635f,
    -0.18477343022823334f,
    -0.09105003625154495f,
    0.0f,
    0.07958029955625534f,
    0.16093020141124725f,
    0.24611230194568634f,
    0.33791524171829224f,
    0.44070982933044434f,
    0.5626170039176941f,
    0.7229568362236023f,
    1.0f,
};

enum {
    ORACLE_OK = 0,
    ORACLE_ERR_ARG = 1,
    ORACLE_ERR_NONFINITE = 4,
};

void oracle_nf4_levels(float out[16]) { memcpy(out, NF4_LEVELS, sizeof NF4_LEVELS); }

/* Nearest of the 16 levels to a normalised value ([P1] section 2,
 * "Normalization"; [P5] Pillar 1 "Map to Closest NF4 Bin").
 * Distances are taken in fp64. For fp32 w' and fp32 levels the difference is
 * exact whenever two candidate distances are close enough for rounding to
 * matter (near a midpoint both operands have comparable exponents), so the
 * argmin is the exact one. Strict '<' keeps the lower index on a tie (R2). */
int oracle_nearest_level(float wn)
{
    int best = 0;
    double best_d = fabs((double)wn - (double)NF4_LEVELS[0]);
    for (int j = 1; j < 16; ++j) {
        double d = fabs((double)wn - (double)NF4_LEVELS[j]);
        if (d < best_d) {
            best_d = d;
            best = j;
        }
    }
    return best;
}

/* Blockwise NF4 quantisation with optional double quantisation.
 *   W       numel fp32 values, flattened row-major ([P5] "Block-Wise
 *           (Chunking) Quantization": slice the flattened tensor into
 *           contiguous chunks).
 *   block   block size (64 in the layer; any even size here, e.g. 6 for the
 *           [P5] numerical example).
 *   codes   numel/2 bytes; element 2j in the HIGH nibble of byte j
 *           ([P5] Pillar 1 "Byte Packing": [1,8] -> 24).
 *   absmax  numel/block fp32 scales s_i = max_j |w_ij| ([P1] section 2,
 *           "Absmax Scale").
 *   dq      when nonzero, also writes q8 (one byte per block) and cg (one fp32
 *           per group of dq_group blocks) per reading R4 ([P5] Pillar 2;
 *           [P3] "Double quantization"; the int8 absmax formula of [P5]
 *           "Vanilla Uniform Quantization").
 * Returns ORACLE_ERR_NONFINITE if any input is NaN or infinite. */
int oracle_nf4_quantize(const float *W, int64_t numel, int32_t block, int32_t dq,
                        int32_t dq_group, uint8_t *codes, float *absmax,
                        uint8_t *q8, float *cg)
{
    if (block <= 0 || (block % 2) != 0 || numel < 0 || (numel % block) != 0)
        return ORACLE_ERR_ARG;
    if (dq && dq_group <= 0)
        return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < numel; ++i)
        if (!isfinite(W[i]))
            return ORACLE_ERR_NONFINITE;

    const int64_t nb = numel / block;
    memset(codes, 0, (size_t)(numel / 2));

    /* First pass: absmax, normalise, nearest level, pack. Blocks are
     * independent (an even block size never splits a byte), so they are
     * spread over threads. */
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        const float *w = W + b * block;
        float s = 0.0f;
        for (int32_t j = 0; j < block; ++j) {
            float a = fabsf(w[j]);
            if (a > s)
                s = a;
        }
        absmax[b] = s;
        for (int32_t j = 0; j < block; ++j) {
            int q;
            if (s == 0.0f) {
                q = 7; /* R3 */
            } else {
                float wn = w[j] / s; /* R1: one fp32 division */
                q = oracle_nearest_level(wn);
            }
            int64_t e = b * block + j;
            if ((e & 1) == 0)
                codes[e / 2] |= (uint8_t)(q << 4);
            else
                codes[e / 2] |= (uint8_t)q;
        }
    }

    /* Second pass: 8-bit quantisation of the scales in groups (R4, R5). */
    if (dq) {
        const int64_t ng = (nb + dq_group - 1) / dq_group;
        for (int64_t g = 0; g < ng; ++g) {
            int64_t b0 = g * dq_group;
            int64_t b1 = b0 + dq_group < nb ? b0 + dq_group : nb;
            float c = 0.0f;
            for (int64_t b = b0; b < b1; ++b)
                if (absmax[b] > c)
                    c = absmax[b];
            cg[g] = c;
            for (int64_t b = b0; b < b1; ++b) {
                if (c == 0.0f) {
                    q8[b] = 0;
                } else {
                    float t = absmax[b] / c;   /* fl32(s / c) */
                    float u = t * 127.0f;      /* fl32(. * 127) */
                    q8[b] = (uint8_t)nearbyintf(u); /* round half to even */
                }
            }
        }
    }
    return ORACLE_OK;
}

/* Dequantised scale of block b: s_b itself, or fl32(q8_b * fl32(c_g / 127))
 * with double quantisation (R4). */
static float oracle_block_scale(int64_t b, const float *absmax, const uint8_t *q8,
                                const float *cg, int32_t dq, int32_t dq_group)
{
    if (!dq)
        return absmax[b];
    float kg = cg[b / dq_group] / 127.0f;
    return (float)q8[b] * kg;
}

void oracle_block_scales(int64_t nb, const float *absmax, const uint8_t *q8,
                         const float *cg, int32_t dq, int32_t dq_group, float *out)
{
    for (int64_t b = 0; b < nb; ++b)
        out[b] = oracle_block_scale(b, absmax, q8, cg, dq, dq_group);
}

/* w~ = fl32(scale * NF4[q]) ([P1] section 2, "On-the-Fly Dequantization";
 * [P1] flowchart "Dynamic Dequantization"). */
void oracle_nf4_dequantize(const uint8_t *codes, const float *absmax,
                           const uint8_t *q8, const float *cg, int64_t numel,
                           int32_t block, int32_t dq, int32_t dq_group, float *out)
{
    for (int64_t e = 0; e < numel; ++e) {
        uint8_t byte = codes[e / 2];
        int q = (e & 1) == 0 ? (byte >> 4) : (byte & 15);
        float s = oracle_block_scale(e / block, absmax, q8, cg, dq, dq_group);
        out[e] = s * NF4_LEVELS[q];
    }
}

/* Round an fp32 value to bf16 (round to nearest, ties to even), returned as
 * the 16 stored bits. Written from the definition: keep the top 16 bits of
 * the fp32 encoding after adding half an ulp of bf16 plus the tie bias. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

double oracle_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

void oracle_f32_to_bf16_array(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_bf16(in[i]);
}

/* Widen a bf16 array to fp64. */
static double *widen_bf16(const uint16_t *p, int64_t n)
{
    double *d = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!d)
        return NULL;
    for (int64_t i = 0; i < n; ++i)
        d[i] = oracle_bf16_to_f64(p[i]);
    return d;
}

/* Dequantised weight as the bf16 matmul operand (R6), held as fp32 (every
 * bf16 value is exact in fp32) and widened to fp64 where it is used:
 * Wt[n][k] = RNE_bf16(fl32(scale * NF4[q])). */
void oracle_dequant_operand(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                            const float *cg, int64_t N, int64_t K, int32_t dq, float *w)
{
    int64_t numel = N * K;
    oracle_nf4_dequantize(codes, absmax, q8, cg, numel, 64, dq, 256, w);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < numel; ++i)
        w[i] = (float)oracle_bf16_to_f64(oracle_f32_to_bf16(w[i]));
}

static float *dequant_operand(const uint8_t *codes, const float *absmax,
                               const uint8_t *q8, const float *cg, int64_t N,
                               int64_t K, int32_t dq)
{
    float *w = (float *)malloc(sizeof(float) * (size_t)(N * K));
    if (!w)
        return NULL;
    oracle_dequant_operand(codes, absmax, q8, cg, N, K, dq, w);
    return w;
}

/* Forward of the layer for a subset of token rows ([P1] section 1, forward
 * step h = W0 x + (alpha/r) B(A(dropout x)) with dropout p = 0; [P3] "The
 * LoRA adapter path": base = x W^T, lora = (x A^T) B^T * scale). Everything in
 * fp64 from the bf16 inputs and the bf16 dequantised operand.
 *   rows[i]     token index of output row i (0 <= rows[i] < M)
 *   h_out       nrows x N fp64
 *   u_out       nrows x r fp64 (u = x A^T), may be NULL
 * Returns 0, or ORACLE_ERR_ARG on allocation failure / bad shapes. */
int oracle_qlora_fwd_rows_op(const float *Wt, int64_t N, int64_t K,
                             const uint16_t *x, int64_t M, const uint16_t *A,
                             const uint16_t *B, int32_t r, double alpha,
                             const int64_t *rows, int64_t nrows, double *h_out, double *u_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || M < 0 || !Wt)
        return ORACLE_ERR_ARG;
    double *Ad = widen_bf16(A, (int64_t)r * K);
    double *Bd = widen_bf16(B, N * r);
    if (!Ad || !Bd) {
        free(Ad); free(Bd);
        return ORACLE_ERR_ARG;
    }
    const double s = alpha / (double)r;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows[i];
        if (m < 0 || m >= M) {
            err = 1;
            continue;
        }
        double *xr = widen_bf16(x + m * K, K);
        double *u = (double *)malloc(sizeof(double) * (size_t)r);
        if (!xr || !u) {
            free(xr); free(u);
            err = 1;
            continue;
        }
        for (int32_t j = 0; j < r; ++j) {           /* u = x A^T */
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += xr[k] * Ad[(int64_t)j * K + k];
            u[j] = acc;
            if (u_out)
                u_out[i * r + j] = acc;
        }
        for (int64_t n = 0; n < N; ++n) {
            double base = 0.0;                       /* x W~^T */
            for (int64_t k = 0; k < K; ++k)
                base += xr[k] * (double)Wt[n * K + k];
            double lora = 0.0;                       /* (x A^T) B^T */
            for (int32_t j = 0; j < r; ++j)
                lora += u[j] * Bd[n * r + j];
            h_out[i * N + n] = base + s * lora;
        }
        free(xr);
        free(u);
    }
    free(Ad); free(Bd);
    return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* The forward from the quantised weight: its dequantised operand is formed
 * (oracle_dequant_operand) and the forward above runs on it. */
int oracle_qlora_fwd_rows(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                          const float *cg, int32_t dq, int64_t N, int64_t K,
                          const uint16_t *x, int64_t M, const uint16_t *A,
                          const uint16_t *B, int32_t r, double alpha,
                          const int64_t *rows, int64_t nrows, double *h_out, double *u_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || M < 0)
        return ORACLE_ERR_ARG;
    float *Wt = dequant_operand(codes, absmax, q8, cg, N, K, dq);
    if (!Wt)
        return ORACLE_ERR_ARG;
    int rc = oracle_qlora_fwd_rows_op(Wt, N, K, x, M, A, B, r, alpha, rows, nrows, h_out, u_out);
    free(Wt);
    return rc;
}

/* Backward of the layer (chain rule; the frozen weight gets no gradient:
 * [P3] "The LoRA adapter path", the dequantised base weight is a constant in
 * backprop; [P4] "Mathematical Foundation", W frozen, only A and B trained):
 *   v  = dY B                      (M x r)
 *   u  = x A^T                     (M x r)
 *   dX = dY W~ + s v A             (rows listed in dx_rows only)
 *   dA = s v^T x                   (r x K, full)
 *   dB = s dY^T u                  (N x r, full)
 * All in fp64 from bf16 inputs. dx_out is ndx x K; dA_out r x K; dB_out N x r.
 * Any output pointer may be NULL to skip it. */
int oracle_qlora_bwd_op(const float *Wt, int64_t N, int64_t K,
                        const uint16_t *x, int64_t M, const uint16_t *A,
                        const uint16_t *B, int32_t r, double alpha, const uint16_t *dY,
                        const int64_t *dx_rows, int64_t ndx, double *dx_out,
                        double *dA_out, double *dB_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || M < 0)
        return ORACLE_ERR_ARG;
    const double s = alpha / (double)r;
    double *Ad = widen_bf16(A, (int64_t)r * K);
    double *Bd = widen_bf16(B, N * r);
    double *v = (double *)calloc((size_t)(M * r + 1), sizeof(double));
    double *u = (double *)calloc((size_t)(M * r + 1), sizeof(double));
    if (!Ad || !Bd || !v || !u) {
        free(Ad); free(Bd); free(v); free(u);
        return ORACLE_ERR_ARG;
    }

    /* v[m][j] = sum_n dY[m][n] B[n][j];  u[m][j] = sum_k x[m][k] A[j][k] */
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double g = oracle_bf16_to_f64(dY[m * N + n]);
            for (int32_t j = 0; j < r; ++j)
                v[m * r + j] += g * Bd[n * r + j];
        }
        for (int32_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += oracle_bf16_to_f64(x[m * K + k]) * Ad[(int64_t)j * K + k];
            u[m * r + j] = acc;
        }
    }

    int err = 0;
    if (dx_out && ndx > 0) {
        if (!Wt) {
            err = 1;
        } else {
#pragma omp parallel for schedule(dynamic, 1)
            for (int64_t i = 0; i < ndx; ++i) {
                int64_t m = dx_rows[i];
                if (m < 0 || m >= M) {
                    err = 1;
                    continue;
                }
                double *row = dx_out + i * K;
                for (int64_t k = 0; k < K; ++k)
                    row[k] = 0.0;
                for (int64_t n = 0; n < N; ++n) {    /* dY W~ */
                    double g = oracle_bf16_to_f64(dY[m * N + n]);
                    for (int64_t k = 0; k < K; ++k)
                        row[k] += g * (double)Wt[n * K + k];
                }
                for (int64_t k = 0; k < K; ++k) {    /* + s v A */
                    double acc = 0.0;
                    for (int32_t j = 0; j < r; ++j)
                        acc += v[m * r + j] * Ad[(int64_t)j * K + k];
                    row[k] += s * acc;
                }
            }
        }
    }

    if (dA_out) {
        /* dA[j][k] = s sum_m v[m][j] x[m][k] */
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < K; ++k) {
            for (int32_t j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t m = 0; m < M; ++m)
                    acc += v[m * r + j] * oracle_bf16_to_f64(x[m * K + k]);
                dA_out[(int64_t)j * K + k] = s * acc;
            }
        }
    }

    if (dB_out) {
        /* dB[n][j] = s sum_m dY[m][n] u[m][j]; each thread owns a range of n
         * and walks m in order, so every sum runs over m = 0..M-1. */
        for (int64_t i = 0; i < N * r; ++i)
            dB_out[i] = 0.0;
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            double *acc = dB_out + n * r;
            for (int64_t m = 0; m < M; ++m) {
                double g = oracle_bf16_to_f64(dY[m * N + n]);
                for (int32_t j = 0; j < r; ++j)
                    acc[j] += g * u[m * r + j];
            }
            for (int32_t j = 0; j < r; ++j)
                acc[j] *= s;
        }
    }

    free(Ad); free(Bd); free(v); free(u);
    return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* The backward from the quantised weight: the dequantised operand is formed
 * only when dX rows are asked for. */
int oracle_qlora_bwd(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                     const float *cg, int32_t dq, int64_t N, int64_t K,
                     const uint16_t *x, int64_t M, const uint16_t *A,
                     const uint16_t *B, int32_t r, double alpha, const uint16_t *dY,
                     const int64_t *dx_rows, int64_t ndx, double *dx_out,
                     double *dA_out, double *dB_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || M < 0)
        return ORACLE_ERR_ARG;
    float *Wt = NULL;
    if (dx_out && ndx > 0)
        Wt = dequant_operand(codes, absmax, q8, cg, N, K, dq);
    int rc = oracle_qlora_bwd_op(Wt, N, K, x, M, A, B, r, alpha, dY, dx_rows, ndx, dx_out,
                                 dA_out, dB_out);
    free(Wt);
    return rc;
}

/* Adapter merge ([P3] "Merging and deploying": the adapters are folded into
 * the base weight for inference; [P4] FAQ on merging: W_new = W + (alpha/r) B A):
 *   out[n][k] = W~[n][k] + (alpha/r) sum_j B[n][j] A[j][k]
 * where W~ is the dequantised base weight in fp32 (fl32(scale * NF4[q]), the
 * value before any rounding to a 16-bit compute type), and B, A are the bf16
 * adapters. Computed in fp64; out is N x K. Returns 0 or ORACLE_ERR_ARG. */
int oracle_qlora_merge(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                       const float *cg, int32_t dq, int64_t N, int64_t K,
                       const uint16_t *A, const uint16_t *B, int32_t r, double alpha,
                       double *out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0)
        return ORACLE_ERR_ARG;
    float *W = (float *)malloc(sizeof(float) * (size_t)(N * K));
    double *Ad = widen_bf16(A, (int64_t)r * K);
    double *Bd = widen_bf16(B, N * r);
    if (!W || !Ad || !Bd) {
        free(W); free(Ad); free(Bd);
        return ORACLE_ERR_ARG;
    }
    oracle_nf4_dequantize(codes, absmax, q8, cg, N * K, 64, dq, 256, W);
    const double s = alpha / (double)r;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double ba = 0.0;
            for (int32_t j = 0; j < r; ++j)
                ba += Bd[n * r + j] * Ad[(int64_t)j * K + k];
            out[n * K + k] = (double)W[n * K + k] + s * ba;
        }
    }
    free(W); free(Ad); free(Bd);
    return ORACLE_OK;
}

/* Forward of one NF4 base with several adapters, one per token ([P5] "The
 * PEFT Strategy (LoRA + QLoRA + Multi-Adapter Serving)": one quantised base
 * resident, the adapter chosen per request; [P4] "Merging and Deployment
 * Strategies": adapters swapped over one quantised base):
 *   h[m] = x[m] W~^T + (alpha_a / r) (x[m] A_a^T) B_a^T,   a = adapter[m]
 * and no adapter term when adapter[m] < 0. The n_ad adapters are stacked:
 * A_all is [n_ad * r, K] (rows a*r .. a*r + r - 1 are A_a), B_all is
 * [N, n_ad * r] (columns a*r .. a*r + r - 1 are B_a). fp64 from the bf16
 * inputs and the bf16 dequantised operand, as the single-adapter forward.
 *   rows[i]   token index of output row i;  h_out nrows x N. */
int oracle_qlora_multi_fwd_rows(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                                const float *cg, int32_t dq, int64_t N, int64_t K,
                                const uint16_t *x, int64_t M, const uint16_t *A_all,
                                const uint16_t *B_all, int32_t r, int32_t n_ad,
                                const double *alphas, const int32_t *adapter,
                                const int64_t *rows, int64_t nrows, double *h_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || n_ad <= 0 || M < 0)
        return ORACLE_ERR_ARG;
    const int64_t R = (int64_t)n_ad * r;
    float *Wt = dequant_operand(codes, absmax, q8, cg, N, K, dq);
    double *Ad = widen_bf16(A_all, R * K);
    double *Bd = widen_bf16(B_all, N * R);
    if (!Wt || !Ad || !Bd) {
        free(Wt); free(Ad); free(Bd);
        return ORACLE_ERR_ARG;
    }
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows[i];
        if (m < 0 || m >= M || adapter[m] >= n_ad) {
            err = 1;
            continue;
        }
        const int32_t a = adapter[m];
        double *xr = widen_bf16(x + m * K, K);
        double *u = (double *)malloc(sizeof(double) * (size_t)r);
        if (!xr || !u) {
            free(xr); free(u);
            err = 1;
            continue;
        }
        if (a >= 0)
            for (int32_t j = 0; j < r; ++j) {        /* u = x A_a^T */
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += xr[k] * Ad[((int64_t)a * r + j) * K + k];
                u[j] = acc;
            }
        const double s = a >= 0 ? alphas[a] / (double)r : 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double base = 0.0;                       /* x W~^T */
            for (int64_t k = 0; k < K; ++k)
                base += xr[k] * (double)Wt[n * K + k];
            double lora = 0.0;                       /* (x A_a^T) B_a^T */
            if (a >= 0)
                for (int32_t j = 0; j < r; ++j)
                    lora += u[j] * Bd[n * R + (int64_t)a * r + j];
            h_out[i * N + n] = base + s * lora;
        }
        free(xr);
        free(u);
    }
    free(Wt); free(Ad); free(Bd);
    return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* LoRA dropout ([P1] section 1: h = W0 x + (alpha/r) B(A(dropout x)); the    */
/* recipe in [P3] uses lora_dropout = 0.05). The random draw is an input:     */
/* keep is a bit mask over x, bit (e & 7) of byte e >> 3 for element          */
/* e = m K + k, 1 = kept. Inverted dropout: a kept element is scaled by       */
/* 1 / (1 - p), a dropped one is zero; the scale is applied to the LoRA       */
/* branch as a whole, (alpha/r)/(1-p), so the masked x is exact.              */
/* ------------------------------------------------------------------------ */
static int keep_bit(const uint8_t *keep, int64_t e) { return (keep[e >> 3] >> (e & 7)) & 1; }

/* Forward rows with dropout on the LoRA input:
 *   u[m] = (keep . x[m]) A^T,   h[m] = x[m] W~^T + (alpha / r) / (1 - p) u[m] B^T
 * u_out (may be NULL) receives u without the 1/(1-p) factor. */
int oracle_qlora_fwd_rows_dropout(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                                  const float *cg, int32_t dq, int64_t N, int64_t K,
                                  const uint16_t *x, int64_t M, const uint16_t *A,
                                  const uint16_t *B, int32_t r, double alpha, double p,
                                  const uint8_t *keep, const int64_t *rows, int64_t nrows,
                                  double *h_out, double *u_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || M < 0 || !(p >= 0.0 && p < 1.0) || !keep)
        return ORACLE_ERR_ARG;
    float *Wt = dequant_operand(codes, absmax, q8, cg, N, K, dq);
    double *Ad = widen_bf16(A, (int64_t)r * K);
    double *Bd = widen_bf16(B, N * r);
    if (!Wt || !Ad || !Bd) {
        free(Wt); free(Ad); free(Bd);
        return ORACLE_ERR_ARG;
    }
    const double s = alpha / (double)r / (1.0 - p);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows[i];
        if (m < 0 || m >= M) {
            err = 1;
            continue;
        }
        double *xr = widen_bf16(x + m * K, K);
        double *u = (double *)malloc(sizeof(double) * (size_t)r);
        if (!xr || !u) {
            free(xr); free(u);
            err = 1;
            continue;
        }
        for (int32_t j = 0; j < r; ++j) {           /* u = (keep . x) A^T */
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                if (keep_bit(keep, m * K + k))
                    acc += xr[k] * Ad[(int64_t)j * K + k];
            u[j] = acc;
            if (u_out)
                u_out[i * r + j] = acc;
        }
        for (int64_t n = 0; n < N; ++n) {
            double base = 0.0;                       /* x W~^T, without dropout */
            for (int64_t k = 0; k < K; ++k)
                base += xr[k] * (double)Wt[n * K + k];
            double lora = 0.0;
            for (int32_t j = 0; j < r; ++j)
                lora += u[j] * Bd[n * r + j];
            h_out[i * N + n] = base + s * lora;
        }
        free(xr);
        free(u);
    }
    free(Wt); free(Ad); free(Bd);
    return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* Backward with dropout on the LoRA input (chain rule through the mask):
 *   v  = dY B,  u = (keep . x) A^T,  s' = (alpha / r) / (1 - p)
 *   dX = dY W~ + s' keep . (v A)       (rows in dx_rows)
 *   dA = s' v^T (keep . x)
 *   dB = s' dY^T u */
int oracle_qlora_bwd_dropout(const uint8_t *codes, const float *absmax, const uint8_t *q8,
                             const float *cg, int32_t dq, int64_t N, int64_t K,
                             const uint16_t *x, int64_t M, const uint16_t *A,
                             const uint16_t *B, int32_t r, double alpha, double p,
                             const uint8_t *keep, const uint16_t *dY,
                             const int64_t *dx_rows, int64_t ndx, double *dx_out,
                             double *dA_out, double *dB_out)
{
    if (N <= 0 || K <= 0 || K % 64 != 0 || r <= 0 || M < 0 || !(p >= 0.0 && p < 1.0) || !keep)
        return ORACLE_ERR_ARG;
    const double s = alpha / (double)r / (1.0 - p);
    double *Ad = widen_bf16(A, (int64_t)r * K);
    double *Bd = widen_bf16(B, N * r);
    double *v = (double *)calloc((size_t)(M * r + 1), sizeof(double));
    double *u = (double *)calloc((size_t)(M * r + 1), sizeof(double));
    if (!Ad || !Bd || !v || !u) {
        free(Ad); free(Bd); free(v); free(u);
        return ORACLE_ERR_ARG;
    }
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double g = oracle_bf16_to_f64(dY[m * N + n]);
            for (int32_t j = 0; j < r; ++j)
                v[m * r + j] += g * Bd[n * r + j];
        }
        for (int32_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                if (keep_bit(keep, m * K + k))
                    acc += oracle_bf16_to_f64(x[m * K + k]) * Ad[(int64_t)j * K + k];
            u[m * r + j] = acc;
        }
    }
    int err = 0;
    if (dx_out && ndx > 0) {
        float *Wt = dequant_operand(codes, absmax, q8, cg, N, K, dq);
        if (!Wt) {
            err = 1;
        } else {
#pragma omp parallel for schedule(dynamic, 1)
            for (int64_t i = 0; i < ndx; ++i) {
                int64_t m = dx_rows[i];
                if (m < 0 || m >= M) {
                    err = 1;
                    continue;
                }
                double *row = dx_out + i * K;
                for (int64_t k = 0; k < K; ++k)
                    row[k] = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double g = oracle_bf16_to_f64(dY[m * N + n]);
                    for (int64_t k = 0; k < K; ++k)
                        row[k] += g * (double)Wt[n * K + k];
                }
                for (int64_t k = 0; k < K; ++k) {
                    if (!keep_bit(keep, m * K + k))
                        continue;
                    double acc = 0.0;
                    for (int32_t j = 0; j < r; ++j)
                        acc += v[m * r + j] * Ad[(int64_t)j * K + k];
                    row[k] += s * acc;
                }
            }
            free(Wt);
        }
    }
    if (dA_out) {
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < K; ++k) {
            for (int32_t j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t m = 0; m < M; ++m)
                    if (keep_bit(keep, m * K + k))
                        acc += v[m * r + j] * oracle_bf16_to_f64(x[m * K + k]);
                dA_out[(int64_t)j * K + k] = s * acc;
            }
        }
    }
    if (dB_out) {
        for (int64_t i = 0; i < N * r; ++i)
            dB_out[i] = 0.0;
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            double *acc = dB_out + n * r;
            for (int64_t m = 0; m < M; ++m) {
                double g = oracle_bf16_to_f64(dY[m * N + n]);
                for (int32_t j = 0; j < r; ++j)
                    acc[j] += g * u[m * r + j];
            }
            for (int32_t j = 0; j < r; ++j)
                acc[j] *= s;
        }
    }
    free(Ad); free(Bd); free(v); free(u);
    return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* LoRA dropout with the mask drawn from a counter-based generator.          */
/* ------------------------------------------------------------------------ */
/* [P1] section 1 puts dropout on the LoRA input and [P3]'s recipe uses
 * lora_dropout = 0.05; the pages name no random generator. Reading: the
 * draw comes from Philox4x32-10, the counter-based generator of Salmon,
 * Moraes, Dror and Shaw ("Parallel random numbers: as easy as 1, 2, 3",
 * SC'11), so that the backward can regenerate the forward's mask from
 * (seed, offset) instead of storing it.
 *
 * One Philox round on the counter (c0, c1, c2, c3) with round key (k0, k1):
 * the two 32x32 -> 64-bit products hi0:lo0 = 0xD2511F53 * c0 and
 * hi1:lo1 = 0xCD9E8D57 * c2 give the new counter
 * (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0). Ten rounds; the key is bumped by
 * the Weyl constants (0x9E3779B9, 0xBB67AE85) between rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Drop threshold of probability p: the element is dropped when its 32-bit
 * draw is below t = floor(p * 2^32), so P(drop) = t / 2^32 (within 2^-32 of
 * p). p * 2^32 is exact in fp64 for an fp32 p. */
uint32_t oracle_dropout_threshold(float p)
{
    double t = floor((double)p * 4294967296.0);
    if (!(t > 0.0))
        return 0u;
    if (t > 4294967295.0)
        return 4294967295u;
    return (uint32_t)t;
}

/* Keep mask of x [M, K] for one (seed, offset): element e = m*K + k takes
 * word (e mod 4) of Philox4x32-10 at counter (g_lo, g_hi, offset_lo,
 * offset_hi), g = e div 4, key (seed_lo, seed_hi); it is kept when that word
 * is >= oracle_dropout_threshold(p). Written as the bit mask the keep-mask
 * functions above read: bit (e & 7) of byte e >> 3, 1 = kept; keep holds
 * ceil(M*K/8) bytes. */
void oracle_dropout_keep_mask(int64_t M, int64_t K, float p, uint64_t seed, uint64_t offset,
                              uint8_t *keep)
{
    const int64_t n = M * K;
    const uint32_t t = oracle_dropout_threshold(p);
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    memset(keep, 0, (size_t)((n + 7) / 8));
#pragma omp parallel for schedule(static)
    for (int64_t byte = 0; byte < (n + 7) / 8; ++byte) {
        uint8_t bits = 0;
        for (int b = 0; b < 8; ++b) {
            const int64_t e = byte * 8 + b;
            if (e >= n)
                break;
            const uint64_t g = (uint64_t)e >> 2;
            const uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), (uint32_t)offset,
                                     (uint32_t)(offset >> 32)};
            uint32_t w[4];
            oracle_philox4x32_10(ctr, key, w);
            if (w[e & 3] >= t)
                bits |= (uint8_t)(1u << b);
        }
        keep[byte] = bits;
    }
}
