/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA linear-layer library.
 *
 * The layer computes, for a frozen weight W0 stored as 4-bit NormalFloat
 * (NF4) codes with blockwise scales, and trainable low-rank adapters A, B:
 *
 *     h = x W~^T + (alpha / r) (x A^T) B^T
 *
 * ("QLoRA Finetuner -- Juan Martos", section 1, forward step of the LoRA
 * layer, and its flowchart "Quantized Base Inference"; "QLoRA explained:
 * fine-tuning in 4-bit precision", section "The LoRA adapter path").
 *
 * Shapes and layouts (all row-major, all device memory owned by the caller):
 *   W0  [n, k] fp32      n = output features, k = input features. The pages
 *                        write W0 as d x k with A r x d and B k x r; here
 *                        d == k (input) and the pages' k == n (output), stored
 *                        out-by-in like a torch Linear weight.
 *   x   [M, k] bf16      tokens
 *   A   [r, k] bf16      down-projection
 *   B   [n, r] bf16      up-projection
 *   h   [M, n] bf16
 *   dY  [M, n] bf16      gradient of the loss w.r.t. h
 *   dX  [M, k] bf16, dA [r, k] bf16, dB [n, r] bf16
 * bf16 values travel as uint16_t bit patterns.
 *
 * Conventions:
 *   - The library never allocates device memory. Scratch space is passed in
 *     (`workspace`, sized by the *_workspace_bytes queries).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every
 *     entry point is asynchronous: NF4_OK means the arguments were valid and
 *     the kernels were launched. Conditions detected on the device
 *     (non-finite weight values, a pipeline wait that ran out of time) are
 *     recorded in a per-device status word read by nf4_device_status().
 *   - Requirements (violations return an error and launch nothing):
 *       block_size 64 or 128, k % block_size == 0, k >= block_size,
 *       n % 8 == 0, n >= 8, M >= 0, 1 <= r <= 128 and r % 8 == 0,
 *       alpha finite, every pointer 16-byte aligned.
 *   - No C++ exception crosses this boundary. Entry points are reentrant;
 *     calls on one stream are ordered, calls on different streams that share
 *     output or workspace buffers race.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NF4_OK = 0,
    NF4_ERR_INVALID_ARG = 1,       /* null pointer where one is required, bad flag */
    NF4_ERR_UNSUPPORTED_SHAPE = 2, /* a shape requirement above is violated */
    NF4_ERR_ALIGNMENT = 3,         /* a pointer is not 16-byte aligned */
    NF4_ERR_NONFINITE = 4,         /* (device) NaN or Inf in the weight to quantise */
    NF4_ERR_TIMEOUT = 5,           /* (device) a pipeline wait ran out of time */
    NF4_ERR_CUDA = 6,              /* a CUDA runtime/driver call failed */
    NF4_ERR_WORKSPACE = 7,         /* workspace missing or smaller than required */
} nf4_status;

/* A quantised frozen weight. The struct lives in host memory; the arrays it
 * points to are device memory owned by the caller.
 *   codes      n*k/2 bytes. Element e of the flattened weight is a 4-bit
 *              index into the 16 NF4 levels; element 2j is the HIGH nibble of
 *              byte j ("Parameter-Efficient Fine-Tuning: From LoRA to QLoRA",
 *              Pillar 1, byte packing step of the numerical example).
 *   absmax     nb = n*k/block_size fp32 block scales s_i = max |w| over each
 *              run of block_size consecutive elements ("QLoRA Finetuner",
 *              section 2: one absmax per block of 64 or 128 weights). Always
 *              written by nf4_quantize; read by the other entry points only
 *              when double_quant == 0.
 *   absmax_q8  nb bytes in [0, 127]: 8-bit codes of the block scales
 *              (double_quant == 1 only).
 *   absmax_c   ceil(nb/256) fp32 group constants: the largest s_i in each run
 *              of 256 consecutive blocks (double_quant == 1 only). The scale
 *              used by dequantisation is then q8_i * (c_g / 127) in fp32
 *              ("Parameter-Efficient Fine-Tuning", Pillar 2: 8-bit
 *              quantisation of the scales in blocks of 256). */
typedef struct {
    int64_t n;
    int64_t k;
    int32_t block_size;   /* 64 or 128 elements per block; k % block_size == 0 */
    int32_t double_quant; /* 0 or 1 */
    uint8_t *codes;
    float *absmax;
    uint8_t *absmax_q8;
    float *absmax_c;
} nf4_weight;

/* Blockwise NF4 quantisation of W0 [n, k] fp32 into w ("QLoRA Finetuner",
 * section 2: absmax per block of w->block_size (64 or 128) consecutive
 * elements, normalise to [-1, 1], nearest of the 16 NF4 quantiles; "Parameter-Efficient Fine-Tuning", Pillar 1 and the
 * numerical step-by-step example; Pillar 2 for double quantisation).
 * Normalisation is one IEEE fp32 division w / s. A value exactly halfway
 * between two levels takes the lower level. An all-zero block stores s = 0
 * and code 7 (the exact zero level). With double_quant, each group of 256
 * blocks stores c_g = max s_i and q8_i = round_half_even((s_i / c_g) * 127)
 * in fp32; the NF4 codes are always taken against the unquantised s_i.
 * A NaN/Inf in W0 sets NF4_ERR_NONFINITE in the device status (the outputs
 * are then unspecified). Writes codes, absmax, and (if double_quant)
 * absmax_q8 and absmax_c. */
QLORA_API nf4_status nf4_quantize(const float *W0, const nf4_weight *w, void *stream);

/* Element types of W0 accepted by nf4_quantize_typed. */
typedef enum { NF4_DTYPE_F32 = 0, NF4_DTYPE_BF16 = 1, NF4_DTYPE_F16 = 2 } nf4_dtype;

/* nf4_quantize for a W0 stored as fp32, bf16 or fp16 ([n, k] row-major, device
 * memory): pretrained weights usually come as 16-bit floats ("QLoRA
 * explained", section "The quantization backbone"). A 16-bit value converts
 * to fp32 exactly, so the result equals nf4_quantize of the fp32 image of W0,
 * bit for bit. Same outputs, requirements and device status as nf4_quantize;
 * an unknown dtype returns NF4_ERR_INVALID_ARG. */
QLORA_API nf4_status nf4_quantize_typed(const void *W0, int32_t dtype, const nf4_weight *w, void *stream);

/* Dequantisation w~ = fl32(scale_i * NF4[q]) for every element ("QLoRA
 * Finetuner", section 2, on-the-fly dequantization). out is n*k elements:
 * fp32 when out_bf16 == 0, else bf16 (round to nearest even of the fp32
 * value). The bf16 result is exactly the operand the layer's matmuls use. */
QLORA_API nf4_status nf4_dequantize(const nf4_weight *w, void *out, int32_t out_bf16, void *stream);

/* Workspace needed by qlora_linear_fwd for M tokens at rank r. */
QLORA_API size_t qlora_fwd_workspace_bytes(int64_t M, int64_t n, int64_t k, int32_t r);

/* Forward of the layer: h = x W~^T + (alpha/r) (x A^T) B^T, with W~ the bf16
 * dequantised weight and fp32 accumulation ("QLoRA explained", section "The
 * LoRA adapter path"; "QLoRA Finetuner", section 1 with dropout p = 0).
 * The scaled down-projection (alpha/r)(x A^T) is rounded to bf16 before the
 * up-projection. u_out (nullable, [M, r] fp32) receives u = x A^T for the
 * backward. workspace: at least qlora_fwd_workspace_bytes(M, n, k, r) bytes
 * of device memory, 256-byte aligned. M == 0 is a no-op. */
QLORA_API nf4_status qlora_linear_fwd(const nf4_weight *w, const uint16_t *x, int64_t M,
                            const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                            uint16_t *h, float *u_out, void *workspace, size_t ws_bytes,
                            void *stream);

/* The forward of qlora_linear_fwd for callers that cannot allocate device
 * memory at call time: processes that reserve their whole memory budget at
 * start-up and forbid later allocations (for example a serving process that
 * has handed every free byte to its own pool), or code that runs inside a
 * memory allocator's own callback, where calling cudaMalloc would re-enter
 * it. Instead of a caller-provided workspace it uses a fixed 4 MiB scratch
 * array that is part of this library's device image: every GPU that loads
 * the library holds those 4 MiB until the process exits. No pages give this
 * entry point: it is an interface variant of this library, not part of the
 * method.
 *   - Same arguments and results as qlora_linear_fwd, minus the workspace.
 *   - Limit: the scaled rank-r activations, M * 2 r bytes, must fit in
 *     4 MiB (128 K tokens at r = 16, 32 K at r = 64, 16 K at r = 128);
 *     larger M returns NF4_ERR_UNSUPPORTED_SHAPE and launches nothing.
 *   - The first call on a device looks up the scratch array's device address
 *     (once per device); make that first call before any stream capture.
 *   - Every call on a device shares the one scratch array, and a call only
 *     reads scratch it has written itself, so nothing needs clearing between
 *     calls; calls whose kernels overlap on the GPU (different streams, or
 *     different host threads) race on it and must be serialised by the
 *     caller. */
QLORA_API nf4_status qlora_linear_fwd_noalloc(const nf4_weight *w, const uint16_t *x, int64_t M,
                                              const uint16_t *A, const uint16_t *B, int32_t r,
                                              float alpha, uint16_t *h, float *u_out,
                                              void *stream);

/* Forward and backward with LoRA dropout on the adapter input ("QLoRA
 * Finetuner", section 1: h = W0 x + (alpha/r) B(A(dropout x)); the recipe in
 * "QLoRA explained" uses lora_dropout = 0.05). The random draw is an input:
 * keep is a DEVICE bit mask over x, (M * k) / 8 bytes, where bit (e & 7) of
 * byte e >> 3 keeps element e = m * k + kk of x (1 = kept, 0 = dropped).
 * Inverted dropout with 0 <= p < 1: the kept elements are scaled by 1/(1-p),
 * applied to the adapter branch as a whole, so
 *     u  = (keep . x) A^T            (u_out receives this, without 1/(1-p))
 *     h  = x W~^T + s' u B^T,        s' = (alpha/r)/(1-p), s' u rounded to bf16
 *     dX = dY W~ + keep . (bf16(s' v) A),   v = dY B
 *     dA = bf16(s' v)^T (keep . x),  dB = dY^T bf16(s' u)
 * The base product uses x unmasked. In the backward, u (if given) must be the
 * forward's u_out for the same mask; dY W~ is kept in fp32 in the workspace and
 * the masked adapter part added to it before the one rounding to bf16, so the
 * backward's workspace is qlora_bwd_dropout_workspace_bytes (M * k * 4 bytes
 * more than qlora_bwd_workspace_bytes). Otherwise as qlora_linear_fwd /
 * qlora_linear_bwd; a null keep (allowed only when M == 0) or p outside
 * [0, 1) returns NF4_ERR_INVALID_ARG. */
QLORA_API nf4_status qlora_linear_fwd_dropout(const nf4_weight *w, const uint16_t *x, int64_t M,
                                              const uint16_t *A, const uint16_t *B, int32_t r,
                                              float alpha, float p, const uint8_t *keep,
                                              uint16_t *h, float *u_out, void *workspace,
                                              size_t ws_bytes, void *stream);
QLORA_API size_t qlora_bwd_dropout_workspace_bytes(int64_t M, int64_t n, int64_t k, int32_t r);
QLORA_API nf4_status qlora_linear_bwd_dropout(const nf4_weight *w, const uint16_t *x, int64_t M,
                                              const uint16_t *A, const uint16_t *B, int32_t r,
                                              float alpha, float p, const uint8_t *keep,
                                              const uint16_t *dY, const float *u, uint16_t *dX,
                                              uint16_t *dA, uint16_t *dB, void *workspace,
                                              size_t ws_bytes, void *stream);

/* The same forward and backward with the dropout mask drawn inside the
 * kernels instead of passed in. The pages fix no random generator; the draw is
 * the counter-based Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 * random numbers: as easy as 1, 2, 3", SC'11): element e = m * k + kk of x
 * takes word (e mod 4) of Philox4x32-10 at counter (e div 4 as two 32-bit
 * words, low first; offset as two words) with key (seed as two words) and is
 * dropped when that word is below floor(p * 2^32). Each kernel that needs the
 * mask computes the words of the elements it touches, so no mask is stored:
 * the backward, given the forward's (p, seed, offset), regenerates exactly the
 * forward's mask. Use a new offset (or seed) for every training step. All else
 * (scaling, rounding, u, workspace sizes, requirements) is as in
 * qlora_linear_fwd_dropout / qlora_linear_bwd_dropout; p outside [0, 1)
 * returns NF4_ERR_INVALID_ARG. */
QLORA_API nf4_status qlora_linear_fwd_dropout_philox(const nf4_weight *w, const uint16_t *x,
                                                     int64_t M, const uint16_t *A,
                                                     const uint16_t *B, int32_t r, float alpha,
                                                     float p, uint64_t seed, uint64_t offset,
                                                     uint16_t *h, float *u_out, void *workspace,
                                                     size_t ws_bytes, void *stream);
QLORA_API nf4_status qlora_linear_bwd_dropout_philox(const nf4_weight *w, const uint16_t *x,
                                                     int64_t M, const uint16_t *A,
                                                     const uint16_t *B, int32_t r, float alpha,
                                                     float p, uint64_t seed, uint64_t offset,
                                                     const uint16_t *dY, const float *u,
                                                     uint16_t *dX, uint16_t *dA, uint16_t *dB,
                                                     void *workspace, size_t ws_bytes,
                                                     void *stream);

/* Forward of one NF4 base with several adapters, one chosen per token, as a
 * server keeps one quantised base resident and applies each request's own
 * adapter ("Parameter-Efficient Fine-Tuning: From LoRA to QLoRA", "The PEFT
 * Strategy (LoRA + QLoRA + Multi-Adapter Serving)"):
 *     h[m] = x[m] W~^T + (alphas[a] / r) (x[m] A_a^T) B_a^T,   a = adapter_of_token[m]
 * The n_adapters adapters of rank r are stacked: A_all is [n_adapters * r, k]
 * (rows a*r .. a*r + r - 1 are A_a), B_all is [n, n_adapters * r] (columns
 * a*r .. a*r + r - 1 are B_a), bf16. alphas is a HOST array of n_adapters
 * floats; adapter_of_token is a DEVICE array of M int32 values, and a value
 * outside [0, n_adapters) means no adapter term for that token.
 * Requirements: 1 <= n_adapters <= 16, r % 8 == 0, n_adapters * r <= 128;
 * the other requirements of qlora_linear_fwd. workspace: at least
 * qlora_fwd_workspace_bytes(M, n, k, n_adapters * r) bytes, 256-byte aligned.
 * Rounding as qlora_linear_fwd: each token's (alphas[a] / r)(x A_a^T) is
 * rounded to bf16 before the up-projection. */
QLORA_API nf4_status qlora_multi_lora_fwd(const nf4_weight *w, const uint16_t *x, int64_t M,
                                          const uint16_t *A_all, const uint16_t *B_all, int32_t r,
                                          int32_t n_adapters, const float *alphas,
                                          const int32_t *adapter_of_token, uint16_t *h,
                                          void *workspace, size_t ws_bytes, void *stream);

/* Workspace needed by qlora_linear_bwd for M tokens at rank r. */
QLORA_API size_t qlora_bwd_workspace_bytes(int64_t M, int64_t n, int64_t k, int32_t r);

/* Backward of the layer; the frozen weight gets no gradient ("QLoRA
 * explained", section "The LoRA adapter path": the dequantised base weight is
 * a constant in backprop and only the adapters are trained):
 *     v  = dY B                  (fp32, [M, r])
 *     dX = dY W~ + s v A         (s = alpha / r; v rounded to bf16 as s*v)
 *     dA = s v^T x
 *     dB = s dY^T u,   u = x A^T (taken from `u` when non-null, else recomputed)
 * dX may be NULL (first layer: no input gradient). dA and dB are required.
 * M == 0 writes zeros to dA and dB. */
QLORA_API nf4_status qlora_linear_bwd(const nf4_weight *w, const uint16_t *x, int64_t M,
                            const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                            const uint16_t *dY, const float *u, uint16_t *dX, uint16_t *dA,
                            uint16_t *dB, void *workspace, size_t ws_bytes, void *stream);

/* qlora_linear_bwd with the adapter gradients written in fp32: dA [r, k] and
 * dB [n, r] receive the fp32 sums of their products (the same sums that
 * qlora_linear_bwd rounds to bf16), so that data-parallel ranks add their
 * gradients in fp32 before the optimiser step (the adapters are the only
 * trained parameters, "QLoRA explained", section "The LoRA adapter path").
 * dX stays bf16. Same arguments, requirements and workspace as
 * qlora_linear_bwd; M == 0 writes zeros. */
QLORA_API nf4_status qlora_linear_bwd_f32grad(const nf4_weight *w, const uint16_t *x, int64_t M,
                                              const uint16_t *A, const uint16_t *B, int32_t r,
                                              float alpha, const uint16_t *dY, const float *u,
                                              uint16_t *dX, float *dA, float *dB, void *workspace,
                                              size_t ws_bytes, void *stream);

/* Adapter merge for inference without adapters ("QLoRA explained", section
 * "Merging and deploying"; "How Fine-Tuning LLMs with LoRA and QLoRA Works",
 * FAQ on merging: W_new = W + (alpha/r) B A):
 *     out[n][k] = w~[n][k] + s * sum_j B[n][j] A[j][k],   s = fl32(alpha / r)
 * with w~ = fl32(scale * NF4[q]) the dequantised weight in fp32. The rank-r
 * sum is accumulated in fp32, added to w~ with one fused multiply-add and
 * rounded once to the output type: out is [n, k] row-major, bf16 when
 * out_is_bf16 == 1 (the 16-bit merged weight), fp32 when 0 (for example to
 * re-quantise it with nf4_quantize). A is [r, k], B is [n, r] (bf16), with
 * the same requirements on r and alpha as the layer. */
QLORA_API nf4_status qlora_merge(const nf4_weight *w, const uint16_t *A, const uint16_t *B,
                                 int32_t r, float alpha, void *out, int32_t out_is_bf16,
                                 void *stream);

/* Synchronises `stream`, then returns and clears the status word that the
 * kernels of the current device set (NF4_OK if nothing was recorded). */
QLORA_API nf4_status nf4_device_status(void *stream);

/* Test hook of the failure-detection path (no counterpart on the pages).
 * Every wait inside the kernels is bounded: a pipeline wait that runs out
 * records NF4_ERR_TIMEOUT, lets the copies and tensor-core operations already
 * issued complete, and returns; the wait of a split tile's first half for the
 * partial sum of its second half (computed by the next CTA pair) records
 * NF4_ERR_TIMEOUT and finishes the tile without it. With skip_flag_set = 1 the
 * second halves do not signal their partial sums, and limit_cycles > 0
 * replaces that one wait's limit (SM clock cycles), so a test can make it run
 * out in microseconds and check the status and a following clean call.
 * (0, 0) restores normal operation. Applies to the current device, between
 * calls (it is not ordered with kernels in flight: synchronise first). */
QLORA_API nf4_status nf4_debug_flag_wait(int32_t skip_flag_set, int64_t limit_cycles);

/* Per-kernel timing, for benchmarks. While enabled, every kernel the library
 * launches is bracketed by two CUDA events recorded on the stream it is
 * launched on; nf4_profile_read() synchronises those events and reports, per
 * kernel kind, the number of launches and their summed duration.
 * nf4_profiling(1) enables and clears the records, nf4_profiling(0) disables
 * recording (records are kept until the next enable). Not thread-safe with
 * respect to concurrent enable/read; launches from several threads are
 * recorded under a lock. */
typedef struct {
    const char *name;   /* static string: kernel kind */
    int64_t launches;
    double total_ms;
} nf4_kernel_time;

QLORA_API nf4_status nf4_profiling(int32_t enable);

/* Fills up to `max` entries and returns how many kernel kinds were recorded
 * (or -1 if reading an event failed). */
QLORA_API int32_t nf4_profile_read(nf4_kernel_time *out, int32_t max);

/* When an entry point returned NF4_ERR_CUDA: the failing CUDA call's error
 * string and where in the library it came from (the last such failure on the
 * calling thread; empty if none). Never NULL; valid until the thread's next
 * failing call. */
QLORA_API const char *nf4_last_cuda_error(void);

/* Static description of a status code. Never NULL. */
QLORA_API const char *nf4_status_string(nf4_status s);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
