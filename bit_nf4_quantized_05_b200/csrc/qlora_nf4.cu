// qlora_nf4.cu -- C ABI of the sm_100a QLoRA linear-layer library: argument
// validation, workspace layout, TMA descriptor set-up and kernel dispatch.
// The whole library is this one translation unit (the kernels live in the
// included headers), so the device status word has a single definition.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "codec.cuh"
#include "gemm_pair_tc.cuh"
#include "skinny_tc.cuh"
#include "decode_stream.cuh"
#include "merge.cuh"

using namespace nf4;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxAdapters = 16;   // stacked adapters of one multi-adapter forward

// The description of the last NF4_ERR_CUDA returned on this thread: the
// failing CUDA call's error string and where it came from.
thread_local char t_last_error[256] = "";

nf4_status cuda_fail(cudaError_t e, int line) {
    std::snprintf(t_last_error, sizeof t_last_error, "%s (qlora_nf4.cu line %d)", cudaGetErrorString(e), line);
    return NF4_ERR_CUDA;
}

nf4_status map_fail(int line) {
    std::snprintf(t_last_error, sizeof t_last_error, "tensor map encoding failed (qlora_nf4.cu line %d)", line);
    return NF4_ERR_CUDA;
}

#define NF4_TRY_CUDA(expr)                                  \
    do {                                                    \
        const cudaError_t nf4_e_ = (expr);                  \
        if (nf4_e_ != cudaSuccess) return cuda_fail(nf4_e_, __LINE__); \
    } while (0)

// ---------------------------------------------------------------------------
// Optional per-kernel event timing (nf4_profiling / nf4_profile_read)
// ---------------------------------------------------------------------------
enum KernelKind {
    KK_QUANTIZE, KK_DEQUANTIZE, KK_LORA_U, KK_LORA_V, KK_LORA_DBDA, KK_ZERO, KK_GEMM_FWD, KK_GEMM_DGRAD, KK_DECODE, KK_DECODE_U, KK_MERGE, KK_LORA_ADD, KK_COUNT
};
const char *const kKindNames[KK_COUNT] = {
    "nf4_quantize", "nf4_dequantize", "lora_u", "lora_v", "lora_dB_dA", "zero_fill", "qlora_gemm_fwd", "qlora_gemm_dgrad", "qlora_decode",
    "decode_lora_u", "qlora_merge", "lora_dX_add"};

struct ProfRecord {
    int kind;
    int device;
    cudaEvent_t start, stop;
};

struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<ProfRecord> recs;
    std::vector<ProfRecord> pool;   // spare event pairs (kind unused)

    bool take(int device, cudaEvent_t *a, cudaEvent_t *b) {
        for (size_t i = 0; i < pool.size(); ++i) {
            if (pool[i].device == device) {
                *a = pool[i].start;
                *b = pool[i].stop;
                pool.erase(pool.begin() + static_cast<long>(i));
                return true;
            }
        }
        return cudaEventCreate(a) == cudaSuccess && cudaEventCreate(b) == cudaSuccess;
    }
};

Profiler &profiler() {
    static Profiler p;
    return p;
}

// Brackets one launch with events on its stream when profiling is enabled.
class LaunchTimer {
  public:
    LaunchTimer(int kind, cudaStream_t s) : kind_(kind), s_(s) {
        Profiler &p = profiler();
        std::lock_guard<std::mutex> g(p.mu);
        if (!p.on) return;
        if (cudaGetDevice(&dev_) != cudaSuccess) return;
        if (!p.take(dev_, &a_, &b_)) return;
        active_ = cudaEventRecord(a_, s_) == cudaSuccess;
    }
    void stop() {
        if (!active_) return;
        active_ = false;
        Profiler &p = profiler();
        std::lock_guard<std::mutex> g(p.mu);
        if (cudaEventRecord(b_, s_) == cudaSuccess) p.recs.push_back({kind_, dev_, a_, b_});
        else p.pool.push_back({kind_, dev_, a_, b_});
    }
    ~LaunchTimer() { stop(); }

  private:
    int kind_;
    cudaStream_t s_;
    int dev_ = 0;
    cudaEvent_t a_{}, b_{};
    bool active_ = false;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch as a programmatic dependent of the previous grid in the stream (the
// kernel waits for it before touching memory), optionally as clusters of
// cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t stream, unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int num_sms(int dev) {
    static int cache[kMaxDevices] = {0};
    if (dev < 0 || dev >= kMaxDevices) return 148;
    if (cache[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [outer, inner] of `elem` bytes per element.
bool make_map(CUtensorMap *map, CUtensorMapDataType dt, size_t elem, const void *base,
              uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * elem};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

nf4_status check_weight(const nf4_weight *w, bool need_scales) {
    if (!w) return NF4_ERR_INVALID_ARG;
    if ((w->block_size != 64 && w->block_size != 128) || (w->double_quant != 0 && w->double_quant != 1))
        return NF4_ERR_INVALID_ARG;
    if (w->n < 8 || w->k < w->block_size || (w->n % 8) != 0 || (w->k % w->block_size) != 0)
        return NF4_ERR_UNSUPPORTED_SHAPE;
    if (w->n > (int64_t(1) << 31) - 1 || w->k > (int64_t(1) << 31) - 1) return NF4_ERR_UNSUPPORTED_SHAPE;
    if (!w->codes || !w->absmax) {
        if (!w->codes || !(w->double_quant || !need_scales)) return NF4_ERR_INVALID_ARG;
    }
    if (w->double_quant && (!w->absmax_q8 || !w->absmax_c)) return NF4_ERR_INVALID_ARG;
    if (!aligned16(w->codes) || (w->absmax && !aligned16(w->absmax)) ||
        (w->absmax_q8 && !aligned16(w->absmax_q8)) || (w->absmax_c && !aligned16(w->absmax_c)))
        return NF4_ERR_ALIGNMENT;
    return NF4_OK;
}

nf4_status check_layer(const nf4_weight *w, const void *x, int64_t M, const void *A, const void *B,
                       int32_t r, float alpha) {
    nf4_status st = check_weight(w, true);
    if (st != NF4_OK) return st;
    if (M < 0 || M > (int64_t(1) << 30)) return NF4_ERR_UNSUPPORTED_SHAPE;
    if (r < 1 || r > 128 || (r % 8) != 0) return NF4_ERR_UNSUPPORTED_SHAPE;
    if (!std::isfinite(alpha)) return NF4_ERR_INVALID_ARG;
    if (!A || !B || (M > 0 && !x)) return NF4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(A) || !aligned16(B)) return NF4_ERR_ALIGNMENT;
    return NF4_OK;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Split plan of one rank-r product: P output rows (tiles of 128), Q reduction
// elements (steps of 64). The splits of one tile form a cluster of at most
// kSkMaxSplits CTAs, and the grid is sized to about one CTA per SM. (At r <= 64
// two CTAs fit on an SM, which lets the clusters pack into one wave; more
// splits than one per SM measured slower on B200.)
// Stream-K scratch of one fused GEMM launch: per CTA pair one fp32 partial
// tile (2 CTAs x 128 rows x 256 columns) and 8 flags (2 CTAs x 4 epilogue
// warps). Sized for sms / 2 pairs, the most that can be resident.
constexpr int kSkFlagsPerPair = 8;
int sk_pairs_max(int sms) { return std::max(1, sms / 2); }
size_t sk_flag_bytes(int sms) { return size_t(sk_pairs_max(sms)) * kSkFlagsPerPair * 4; }
size_t sk_partial_bytes(int sms) { return size_t(sk_pairs_max(sms)) * 2 * 128 * 256 * 4; }

struct SkBuf {
    float *partial;
    int *flags;
    int pairs_max;
};

struct FwdLayout {
    size_t us, upart, flags, partial, total;
};

// us: bf16 rank-r activations; upart: the decode path's partial sums of
// x A^T (M <= 16 tokens only); flags/partial: stream-K scratch (with_sk =
// false: the whole-tile schedule, none)
FwdLayout fwd_layout(int64_t M, int32_t r, int sms, bool with_sk = true) {
    FwdLayout L{};
    size_t off = 0;
    L.us = off;   off = align256(off + size_t(M) * r * 2);
    L.upart = off;
    if (M <= 16) off = align256(off + size_t(kDsUCtas) * size_t(M) * r * 4);
    if (with_sk) {
        L.flags = off;   off = align256(off + sk_flag_bytes(sms));
        L.partial = off; off = align256(off + sk_partial_bytes(sms));
    }
    L.total = off;
    return L;
}

struct BwdLayout {
    size_t us, vs, flags, partial, total;
};

BwdLayout bwd_layout(int64_t M, int32_t r, int sms) {
    BwdLayout L{};
    size_t off = 0;
    L.us = off;      off = align256(off + size_t(M) * r * 2);
    L.vs = off;      off = align256(off + size_t(M) * r * 2);
    L.flags = off;   off = align256(off + sk_flag_bytes(sms));
    L.partial = off; off = align256(off + sk_partial_bytes(sms));
    L.total = off;
    return L;
}

enum class Major { K, MN };

// Rank-r product out[p][j] = sum_q P(p,q) Q(q,j) through the clustered
// skinny tcgen05 kernel (split reduction included).
//   a: row-major bf16 [a_rows, a_cols]; K-major: p = row, q = col; MN-major: q = row, p = col
//   b: row-major bf16 [b_rows, b_cols]; K-major: j = row, q = col; MN-major: q = row, j = col
struct SkinnySpec {
    const void *a;
    int64_t a_rows, a_cols;
    Major am;
    const void *b;
    int64_t b_rows, b_cols;
    Major bm;
    int32_t r;
    float *out_f32;
    uint16_t *out_bf16;
    float scale;
    int transposed;
    int mask_mode = 0;                 // dropout on x as the A operand (see SkinnyJob)
    const uint8_t *keep = nullptr;
    int64_t mx = 0, kx = 0;
    DropRng rng{};                     // the mask drawn from the generator instead of keep
};

// Tensor maps and job fields of one product; splits is the launch's split count.
bool skinny_job(const SkinnySpec &sp, int RN, int splits, CUtensorMap *ta, CUtensorMap *tb,
                SkinnyJob *job) {
    const int64_t P = sp.am == Major::K ? sp.a_rows : sp.a_cols;
    const int64_t Q = sp.am == Major::K ? sp.a_cols : sp.a_rows;
    bool ok = sp.am == Major::K
                  ? make_map(ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.a, sp.a_cols, sp.a_rows, 64, 128,
                             CU_TENSOR_MAP_SWIZZLE_128B)
                  : make_map(ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.a, sp.a_cols, sp.a_rows, 64, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && (sp.bm == Major::K
                    ? make_map(tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.b, sp.b_cols, sp.b_rows, 64,
                               static_cast<uint32_t>(RN), CU_TENSOR_MAP_SWIZZLE_128B)
                    : make_map(tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.b, sp.b_cols, sp.b_rows, 64, 64,
                               CU_TENSOR_MAP_SWIZZLE_128B));
    job->P = static_cast<int>(P);
    job->p_tiles = static_cast<int>((P + 127) / 128);
    job->steps = static_cast<int>((Q + 63) / 64);
    job->steps_per_split = (job->steps + splits - 1) / splits;
    job->r = sp.r;
    job->out_f32 = sp.out_f32;
    job->out_bf16 = sp.out_bf16;
    job->scale = sp.scale;
    job->transposed = sp.transposed;
    job->mask_mode = sp.mask_mode;
    job->keep = sp.keep;
    job->rng = sp.rng;
    job->mx = sp.mx;
    job->kx = sp.kx;
    return ok;
}

// One launch of one or two products (n = 1, 2) with the same operand layouts
// and rank, plus optional flag zeroing and an element-wise side task.
// Per-row adapter selection for the bf16 output of a one-product launch.
struct RowGroups {
    const int32_t *row_group = nullptr;
    int group_width = 0;
    int ngroups = 0;
    const float *gscale = nullptr;   // host array [ngroups]
};

nf4_status skinny_launch(int kind, const SkinnySpec *sp, int n, cudaStream_t stream,
                         int *zero_ints = nullptr, int zero_count = 0, const float *conv_src = nullptr,
                         uint16_t *conv_dst = nullptr, int64_t conv_n = 0, float conv_scale = 0.f,
                         const RowGroups *groups = nullptr) {
    const int sms = num_sms(current_device());
    const int RN = sp[0].r <= 64 ? 64 : 128;
    int p_tiles = 0, steps = 1;
    for (int i = 0; i < n; ++i) {
        if (sp[i].am != sp[0].am || sp[i].bm != sp[0].bm || sp[i].r != sp[0].r) return NF4_ERR_INVALID_ARG;
        const int64_t P = sp[i].am == Major::K ? sp[i].a_rows : sp[i].a_cols;
        const int64_t Q = sp[i].am == Major::K ? sp[i].a_cols : sp[i].a_rows;
        p_tiles += static_cast<int>((P + 127) / 128);
        steps = std::max(steps, static_cast<int>((Q + 63) / 64));
    }
    // one wave: the splits of all tiles fill the CTA slots once (two CTAs fit
    // on an SM; clusters of at most 8)
    int splits = std::max(1, 2 * sms / std::max(1, p_tiles));
    splits = std::min({splits, kSkMaxSplits, steps});
    const int sps = (steps + splits - 1) / splits;
    splits = (steps + sps - 1) / sps;            // every split has at least one step
    SkinnyArgs args{};
    CUtensorMap ta[2], tb[2];
    for (int i = 0; i < n; ++i)
        if (!skinny_job(sp[i], RN, splits, &ta[i], &tb[i], &args.job[i])) return map_fail(__LINE__);
    if (n == 1) {
        ta[1] = ta[0];
        tb[1] = tb[0];
        args.job[1] = args.job[0];
    }
    args.njobs = n;
    args.zero_ints = zero_ints;
    args.zero_count = zero_count;
    args.conv_src = conv_src;
    args.conv_dst = conv_dst;
    args.conv_n = conv_n;
    args.conv_scale = conv_scale;
    if (groups && groups->row_group) {
        args.row_group = groups->row_group;
        args.group_width = groups->group_width;
        args.ngroups = groups->ngroups;
        for (int i = 0; i < groups->ngroups && i < 16; ++i) args.gscale[i] = groups->gscale[i];
    }
    const dim3 grid(static_cast<unsigned>(splits), static_cast<unsigned>(p_tiles));
    const Major am = sp[0].am, bm = sp[0].bm;
    cudaError_t e = cudaErrorInvalidValue;
    {
        LaunchTimer t(kind, stream);
#define NF4_SKINNY_CASE(RN_, AMN, BMN)                                                      \
    if (RN == RN_ && (am == Major::MN) == AMN && (bm == Major::MN) == BMN) {                \
        auto kern = skinny_cluster_kernel<RN_, AMN, BMN>;                                   \
        NF4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                          SkCfg<RN_, AMN, BMN>::kSmemBytes));               \
        e = launch_ex(kern, grid, dim3(kSkThreads), SkCfg<RN_, AMN, BMN>::kSmemBytes, stream, \
                      static_cast<unsigned>(splits), ta[0], tb[0], ta[1], tb[1], args);     \
    }
        NF4_SKINNY_CASE(64, false, false)
        NF4_SKINNY_CASE(128, false, false)
        NF4_SKINNY_CASE(64, false, true)
        NF4_SKINNY_CASE(128, false, true)
        NF4_SKINNY_CASE(64, true, true)
        NF4_SKINNY_CASE(128, true, true)
#undef NF4_SKINNY_CASE
        t.stop();
    }
    if (e != cudaSuccess) return cuda_fail(e, __LINE__);
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

nf4_status skinny_product(int kind, const void *a, int64_t a_rows, int64_t a_cols, Major am,
                          const void *b, int64_t b_rows, int64_t b_cols, Major bm, int32_t r,
                          float *out_f32, uint16_t *out_bf16, float scale, int transposed,
                          cudaStream_t stream, int *zero_ints = nullptr, int zero_count = 0) {
    const SkinnySpec sp{a, a_rows, a_cols, am, b, b_rows, b_cols, bm, r, out_f32, out_bf16, scale, transposed};
    return skinny_launch(kind, &sp, 1, stream, zero_ints, zero_count);
}

// Clusters of two CTAs of one pair-kernel configuration that can be resident
// at once on the device (0 if the query fails).
template <int BN, bool DGRAD, int G>
int pair_capacity(int dev) {
    using Cfg = PairCfg<BN, DGRAD, G>;
    static int cache[kMaxDevices] = {0};
    if (dev < 0 || dev >= kMaxDevices) return 0;
    if (cache[dev] == 0) {
        auto kern = qlora_gemm_pair_kernel<BN, DGRAD, G, false>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::kSmemBytes) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 74);
        cfg.blockDim = dim3(Cfg::kThreads);
        cfg.dynamicSmemBytes = Cfg::kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            return 0;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

// sk: stream-K scratch, or null for the whole-tile schedule. Stream-K runs
// when there are more tiles than resident pairs and they do not divide evenly.
template <int BN, bool DGRAD, int G>
nf4_status launch_gemm_pair(const nf4_weight *w, const uint16_t *act, int64_t M, int64_t red,
                            int64_t out, const uint16_t *la, int32_t r, const uint16_t *lb,
                            uint16_t *D, cudaStream_t stream, const SkBuf *sk = nullptr,
                            float *D32 = nullptr) {
    using Cfg = PairCfg<BN, DGRAD, G>;
    CUtensorMap tm_act, tm_codes, tm_la;
    const int64_t N = w->n, K = w->k;
    bool ok = make_map(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, act, red, M, kBK, kBM,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    // 4-bit codes of this CTA's half tile: one 32-byte block column per box
    // (BN/2 rows forward, 64 rows dgrad), 32-byte swizzle
    ok = ok && make_map(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, K / 2, N, kBK / 2,
                        DGRAD ? kBK : Cfg::kBH, CU_TENSOR_MAP_SWIZZLE_32B);
    // no LoRA stage when la is null (the adapter term is added by another kernel)
    if (la)
        ok = ok && make_map(&tm_la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, la, r, M, kBK, kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    else
        tm_la = tm_act;
    if (!ok) return map_fail(__LINE__);

    GemmArgs a{};
    a.M = static_cast<int>(M);
    a.red = static_cast<int>(red);
    a.out = static_cast<int>(out);
    a.main_steps = static_cast<int>((red + kBK - 1) / kBK);
    a.lora_steps = la ? (r + kBK - 1) / kBK : 0;
    a.m_tiles = static_cast<int>((M + kBM - 1) / kBM);
    a.n_tiles = static_cast<int>((out + BN - 1) / BN);
    a.r = r;
    a.Nw = N;
    a.Kw = K;
    a.kblocks = K / kBlock;
    a.bshift = block_shift_of(w->block_size);
    a.absmax = w->absmax;
    a.q8 = w->absmax_q8;
    a.cg = w->absmax_c;
    a.dq = w->double_quant;
    a.lora_b = lb;
    a.D = D;
    a.D32 = D32;

    const int dev = current_device();
    const int cap = pair_capacity<BN, DGRAD, G>(dev);
    if (cap <= 0) {
        std::snprintf(t_last_error, sizeof t_last_error, "no CTA pair of the fused GEMM can be resident");
        return NF4_ERR_CUDA;
    }
    const int64_t m_pairs = (M + 2 * kBM - 1) / (2 * kBM);
    const int64_t tiles = m_pairs * a.n_tiles;
    const bool use_sk = BN == 256 && sk && sk->partial && sk->flags && cap <= sk->pairs_max &&
                        tiles > cap && tiles % cap != 0;
    const int pairs = use_sk ? cap : static_cast<int>(std::min<int64_t>(tiles, cap));
    if (use_sk) {
        a.sk = 1;
        a.partial = sk->partial;
        a.flags = sk->flags;
    }
    LaunchTimer t(DGRAD ? KK_GEMM_DGRAD : KK_GEMM_FWD, stream);
    const cudaError_t e =
        D32 ? (cudaFuncSetAttribute(qlora_gemm_pair_kernel<BN, DGRAD, G, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) != cudaSuccess
                   ? cudaErrorInvalidValue
                   : launch_ex(qlora_gemm_pair_kernel<BN, DGRAD, G, true>, dim3(static_cast<unsigned>(2 * pairs)),
                        dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, 2u, tm_act, tm_codes, tm_la, a))
            : launch_ex(qlora_gemm_pair_kernel<BN, DGRAD, G, false>, dim3(static_cast<unsigned>(2 * pairs)),
                        dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, 2u, tm_act, tm_codes, tm_la, a);
    t.stop();
    if (e != cudaSuccess) return cuda_fail(e, __LINE__);
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

// One instantiation of the decode kernel per (token groups, chunk blocks,
// per-token adapter selection).
template <int TG, int CB, class GT>
cudaError_t launch_decode_stream_t(unsigned grid, cudaStream_t stream, const CUtensorMap &tm,
                                   const DecodeArgs &a, const GT &grp) {
    auto k = qlora_decode_stream_kernel<TG, CB, GT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kDsDynBytes);
    if (e != cudaSuccess) return e;
    return launch_ex(k, dim3(grid), dim3(kDsThreads), kDsDynBytes, stream, 0u, tm, a, grp);
}

template <int TG, class GT>
cudaError_t launch_decode_stream_cb(int cb, unsigned grid, cudaStream_t stream, const CUtensorMap &tm,
                                    const DecodeArgs &a, const GT &grp) {
    switch (cb) {
        case 1: return launch_decode_stream_t<TG, 1>(grid, stream, tm, a, grp);
        case 2: return launch_decode_stream_t<TG, 2>(grid, stream, tm, a, grp);
        case 3: return launch_decode_stream_t<TG, 3>(grid, stream, tm, a, grp);
        case 4: return launch_decode_stream_t<TG, 4>(grid, stream, tm, a, grp);
        case 5: return launch_decode_stream_t<TG, 5>(grid, stream, tm, a, grp);
        default: return cudaErrorInvalidValue;
    }
}

template <class GT>
cudaError_t launch_decode_stream(int tg, int cb, unsigned grid, cudaStream_t stream, const CUtensorMap &tm,
                                 const DecodeArgs &a, const GT &grp) {
    return tg == 1 ? launch_decode_stream_cb<1>(cb, grid, stream, tm, a, grp)
                   : launch_decode_stream_cb<2>(cb, grid, stream, tm, a, grp);
}

// Forward for M <= 16 tokens: partial sums of u = x A^T on a few SMs, then
// the decode kernel on the rest, launched as a programmatic dependent of the
// first so that it streams the weight while u is being formed (it adds the
// partials once it needs u).
constexpr int64_t kDecodeMaxTokens = 16;

// The decode kernel keeps u tiles of rank <= kDsMaxRank in shared memory.
bool decode_shape(const nf4_weight *w, int64_t M, int32_t r) {
    return M <= kDecodeMaxTokens && r <= kDsMaxRank &&
           w->n * (w->k / kBlock) < (int64_t(1) << 31);   // 32-bit block indices
}

nf4_status launch_decode(const nf4_weight *w, const uint16_t *x, int64_t M, const uint16_t *A,
                         const uint16_t *B, int32_t r, float scale, uint16_t *h, float *u_out,
                         float *upart, cudaStream_t stream, const RowGroups *groups = nullptr,
                         const uint8_t *keep = nullptr, const DropRng &rng = DropRng{}) {
    // each of the 16 warps takes rb blocks of every 32-row tile, fetched in
    // chunks of cb blocks (the largest divisor of rb that is at most 5)
    const int64_t kblocks = w->k / kBlock;
    const int rb = static_cast<int>((kblocks + kDsWarps - 1) / kDsWarps);
    int cb = 1;
    for (int d = kDsMaxChunk; d >= 1; --d)
        if (rb % d == 0) {
            cb = d;
            break;
        }
    DecodeArgs a;
    a.M = static_cast<int>(M);
    a.N = w->n;
    a.K = w->k;
    a.r = r;
    a.rb = rb;
    a.absmax = w->absmax;
    a.q8 = w->absmax_q8;
    a.cg = w->absmax_c;
    a.dq = w->double_quant;
    a.x = x;
    a.B = B;
    a.A = A;
    a.upart = upart;
    a.scale = scale;
    a.u_out = u_out;
    a.h = h;
    a.bshift = block_shift_of(w->block_size);
    CUtensorMap tm_codes;
    if (!make_map(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, w->k / 2, w->n,
                  static_cast<uint32_t>(32 * cb), kDsRows, CU_TENSOR_MAP_SWIZZLE_NONE))
        return map_fail(__LINE__);
    const int64_t tiles = (w->n + kDsRows - 1) / kDsRows;
    // the decode grid leaves kDsUCtas SMs to the u kernel
    const int sms = num_sms(current_device());
    const unsigned grid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(tiles, sms - kDsUCtas)));
    const int tg = M <= 8 ? 1 : 2;
    {
        // u = x A^T on kDsUCtas CTAs, beside the decode grid
        LaunchTimer t(KK_DECODE_U, stream);
        auto ku = tg == 1 ? qlora_decode_u_kernel<1> : qlora_decode_u_kernel<2>;
        NF4_TRY_CUDA(cudaFuncSetAttribute(ku, cudaFuncAttributeMaxDynamicSharedMemorySize, kDsUParkBytes));
        const cudaError_t e = launch_ex(ku, dim3(kDsUCtas), dim3(kDsThreads), kDsUParkBytes, stream, 0u, a, keep, rng);
        t.stop();
        if (e != cudaSuccess) return cuda_fail(e, __LINE__);
    }
    LaunchTimer t(KK_DECODE, stream);
    cudaError_t e;
    if (groups && groups->row_group) {
        DsGroups gr{};
        gr.row_group = groups->row_group;
        gr.group_width = groups->group_width;
        gr.ngroups = groups->ngroups;
        for (int i = 0; i < groups->ngroups && i < 16; ++i) gr.gscale[i] = groups->gscale[i];
        e = launch_decode_stream(tg, cb, grid, stream, tm_codes, a, gr);
    } else {
        e = launch_decode_stream(tg, cb, grid, stream, tm_codes, a, DsNoGroups{});
    }
    t.stop();
    if (e != cudaSuccess) return cuda_fail(e, __LINE__);
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

// Pair-tile width: the candidate with the smallest (rounds of 256-token
// tiles over the resident pairs) x (time of one tile). A tile's time is
// modelled as proportional to (width + 320): measured on B200, a stage costs
// nearly as much at width 128 as at 256 (activation loads and pipeline
// latency do not shrink with the width). Dgrad halves must be whole 64-column
// swizzle atoms, so dgrad chooses between 256 and 128.
int pick_pair_bn(int64_t M, int64_t out, int pairs, bool dgrad) {
    const int64_t m_pairs = (M + 2 * kBM - 1) / (2 * kBM);
    int best = 256;
    int64_t best_cost = -1;
    for (int bn : {256, 192, 128}) {
        if (dgrad && bn == 192) continue;
        const int64_t tiles = m_pairs * ((out + bn - 1) / bn);
        const int64_t cost = ((tiles + pairs - 1) / pairs) * (bn + 320);
        if (best_cost < 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

// Dequantisation groups per CTA of the pair kernel (each takes every
// kPairGroups-th stage). Measured on B200 at 5120x5120, 2048 tokens (forward
// us): 2 groups 187, 3 163, 4 146, 5 134, 6 135 (6 groups leave 64 registers
// per thread).
constexpr int kPairGroups = 5;

// sk: stream-K scratch (null: whole tiles only). With it, problems with more
// 256-column tiles than resident pairs run 256-wide tiles under stream-K
// (the tensor core takes as long for a 192-wide tile as for a 256-wide one).
template <bool DGRAD>
nf4_status launch_gemm_auto(const nf4_weight *w, const uint16_t *act, int64_t M, int64_t red,
                            int64_t out, const uint16_t *la, int32_t r, const uint16_t *lb,
                            uint16_t *D, cudaStream_t stream, const SkBuf *sk = nullptr,
                            float *D32 = nullptr) {
    const int dev = current_device();
    const int pairs = pair_capacity<256, DGRAD, kPairGroups>(dev);
    if (pairs > 0) {
        const int64_t tiles256 = ((M + 2 * kBM - 1) / (2 * kBM)) * ((out + 255) / 256);
        if (sk && tiles256 > pairs)
            return launch_gemm_pair<256, DGRAD, kPairGroups>(w, act, M, red, out, la, r, lb, D,
                                                             stream, sk, D32);
        switch (pick_pair_bn(M, out, pairs, DGRAD)) {
        case 128:
            return launch_gemm_pair<128, DGRAD, kPairGroups>(w, act, M, red, out, la, r, lb, D, stream, nullptr, D32);
        case 192:
            if constexpr (!DGRAD)
                return launch_gemm_pair<192, DGRAD, kPairGroups>(w, act, M, red, out, la, r, lb, D,
                                                                 stream, nullptr, D32);
            break;
        default:
            return launch_gemm_pair<256, DGRAD, kPairGroups>(w, act, M, red, out, la, r, lb, D, stream, nullptr, D32);
        }
    }
    // no CTA pair of this kernel can be resident (not the case on a B200)
    std::snprintf(t_last_error, sizeof t_last_error, "no CTA pair of the fused GEMM can be resident");
    return NF4_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Fixed device scratch for qlora_linear_fwd_noalloc. It is part of the
// library's image: every device that loads the library holds these bytes
// until the process exits, and every call of that entry point on a device
// shares them.
// ---------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB
__device__ __align__(256) uint8_t g_fwd_static_scratch[kStaticScratchBytes];

// Device address of the static scratch on the current device. Host code may
// not use the array's name as a pointer (it names a host-side stand-in), so
// the address is looked up once per device with that device current.
void *static_scratch_on_current_device() {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {nullptr};
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fwd_static_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

const char *nf4_last_cuda_error(void) { return t_last_error; }

const char *nf4_status_string(nf4_status s) {
    switch (s) {
        case NF4_OK: return "ok";
        case NF4_ERR_INVALID_ARG: return "invalid argument";
        case NF4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case NF4_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case NF4_ERR_NONFINITE: return "non-finite value in the weight";
        case NF4_ERR_TIMEOUT: return "device pipeline wait timed out";
        case NF4_ERR_CUDA: return "CUDA call failed";
        case NF4_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

nf4_status nf4_profiling(int32_t enable) {
    Profiler &p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    if (enable) {
        for (auto &r : p.recs) p.pool.push_back(r);
        p.recs.clear();
    }
    p.on = enable != 0;
    return NF4_OK;
}

int32_t nf4_profile_read(nf4_kernel_time *out, int32_t max) {
    Profiler &p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    int64_t n[KK_COUNT] = {0};
    double ms[KK_COUNT] = {0};
    for (auto &r : p.recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess ||
            cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            return -1;
        n[r.kind] += 1;
        ms[r.kind] += t;
    }
    int32_t cnt = 0;
    for (int k = 0; k < KK_COUNT; ++k) {
        if (n[k] == 0) continue;
        if (out && cnt < max) out[cnt] = {kKindNames[k], n[k], ms[k]};
        ++cnt;
    }
    return cnt;
}

nf4_status nf4_debug_flag_wait(int32_t skip_flag_set, int64_t limit_cycles) {
    if (limit_cycles < 0 || (skip_flag_set != 0 && skip_flag_set != 1)) return NF4_ERR_INVALID_ARG;
    const int skip = skip_flag_set;
    const long long lim = limit_cycles;
    NF4_TRY_CUDA(cudaMemcpyToSymbol(g_dbg_skip_flag_set, &skip, sizeof skip));
    NF4_TRY_CUDA(cudaMemcpyToSymbol(g_dbg_flag_wait_limit, &lim, sizeof lim));
    return NF4_OK;
}

nf4_status nf4_device_status(void *stream) {
    NF4_TRY_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    unsigned int v = 0, zero = 0;
    NF4_TRY_CUDA(cudaMemcpyFromSymbol(&v, g_status, sizeof v));
    if (v != 0) NF4_TRY_CUDA(cudaMemcpyToSymbol(g_status, &zero, sizeof zero));
    return static_cast<nf4_status>(v);
}

nf4_status nf4_quantize_typed(const void *W0, int32_t dtype, const nf4_weight *w, void *stream) {
    nf4_status st = check_weight(w, false);
    if (st != NF4_OK) return st;
    if (!W0 || !w->absmax) return NF4_ERR_INVALID_ARG;
    if (dtype != NF4_DTYPE_F32 && dtype != NF4_DTYPE_BF16 && dtype != NF4_DTYPE_F16) return NF4_ERR_INVALID_ARG;
    if (!aligned16(W0)) return NF4_ERR_ALIGNMENT;
    const int64_t numel = w->n * w->k;
    const int64_t nb = numel / w->block_size;
    const int64_t groups = (nb + kGroup - 1) / kGroup;
    // TMA row coordinates (128-byte rows: 32 fp32 or 64 16-bit elements) are 32-bit
    if (numel / 32 > 0x7fffffffLL) return NF4_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap tm_w;
    bool ok;
    if (dtype == NF4_DTYPE_F32)
        ok = make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, W0, 32, static_cast<uint64_t>(numel / 32), 32,
                      kQzStageElems / 32, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ok = make_map(&tm_w,
                      dtype == NF4_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                      2, W0, 64, static_cast<uint64_t>(numel / 64), 64, kQzStageElems / 64,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return map_fail(__LINE__);
    // persistent: kQzCtasPerSm CTAs per SM walk the groups
    const int64_t grid = std::min<int64_t>(groups, int64_t(kQzCtasPerSm) * num_sms(current_device()));
    void (*kern)(const CUtensorMap, int64_t, int, uint8_t *, float *, uint8_t *, float *);
    if (w->block_size == 64)
        kern = dtype == NF4_DTYPE_F32 ? nf4_quantize_kernel<kQzF32, 64>
               : dtype == NF4_DTYPE_BF16 ? nf4_quantize_kernel<kQzBF16, 64> : nf4_quantize_kernel<kQzF16, 64>;
    else
        kern = dtype == NF4_DTYPE_F32 ? nf4_quantize_kernel<kQzF32, 128>
               : dtype == NF4_DTYPE_BF16 ? nf4_quantize_kernel<kQzBF16, 128> : nf4_quantize_kernel<kQzF16, 128>;
    NF4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQzSmemBytes));
    LaunchTimer t(KK_QUANTIZE, static_cast<cudaStream_t>(stream));
    kern<<<static_cast<unsigned>(grid), kQzThreads, kQzSmemBytes, static_cast<cudaStream_t>(stream)>>>(
        tm_w, nb, w->double_quant, w->codes, w->absmax, w->absmax_q8, w->absmax_c);
    t.stop();
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

nf4_status nf4_quantize(const float *W0, const nf4_weight *w, void *stream) {
    return nf4_quantize_typed(W0, NF4_DTYPE_F32, w, stream);
}

nf4_status nf4_dequantize(const nf4_weight *w, void *out, int32_t out_bf16, void *stream) {
    nf4_status st = check_weight(w, true);
    if (st != NF4_OK) return st;
    if (!out || (out_bf16 != 0 && out_bf16 != 1)) return NF4_ERR_INVALID_ARG;
    if (!aligned16(out)) return NF4_ERR_ALIGNMENT;
    const int64_t nb = w->n * w->k / kBlock;       // 64-element steps
    const int dev = current_device();
    const int grid = static_cast<int>(std::min<int64_t>((nb + 255) / 256, int64_t(num_sms(dev)) * 16));
    LaunchTimer t(KK_DEQUANTIZE, static_cast<cudaStream_t>(stream));
    nf4_dequantize_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        w->codes, w->absmax, w->absmax_q8, w->absmax_c, w->double_quant, nb, block_shift_of(w->block_size),
        out_bf16, out);
    t.stop();
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

nf4_status qlora_merge(const nf4_weight *w, const uint16_t *A, const uint16_t *B, int32_t r,
                       float alpha, void *out, int32_t out_is_bf16, void *stream) {
    nf4_status st = check_weight(w, true);
    if (st != NF4_OK) return st;
    if (r < 1 || r > kMgMaxRank || (r % 8) != 0) return NF4_ERR_UNSUPPORTED_SHAPE;
    if (!std::isfinite(alpha)) return NF4_ERR_INVALID_ARG;
    if (!A || !B || !out || (out_is_bf16 != 0 && out_is_bf16 != 1)) return NF4_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(out)) return NF4_ERR_ALIGNMENT;
    if ((w->n + kMgRows - 1) / kMgRows > 65535) return NF4_ERR_UNSUPPORTED_SHAPE;
    MergeArgs a{};
    a.N = w->n;
    a.K = w->k;
    a.r = r;
    a.rp = (r + 15) / 16 * 16;
    a.codes = w->codes;
    a.absmax = w->absmax;
    a.q8 = w->absmax_q8;
    a.cg = w->absmax_c;
    a.dq = w->double_quant;
    a.A = A;
    a.B = B;
    a.scale = alpha / static_cast<float>(r);
    a.out = out;
    a.block = w->block_size;
    const int smem = merge_smem_bytes(a.rp, out_is_bf16 != 0);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void (*kern)(const MergeArgs) = nullptr;
#define NF4_MERGE_CASE(RQ_)                                                                    \
    case RQ_:                                                                                  \
        kern = out_is_bf16 ? qlora_merge_kernel<true, RQ_> : qlora_merge_kernel<false, RQ_>; \
        break;
    switch (a.rp / 16) {
        NF4_MERGE_CASE(1) NF4_MERGE_CASE(2) NF4_MERGE_CASE(3) NF4_MERGE_CASE(4)
        NF4_MERGE_CASE(5) NF4_MERGE_CASE(6) NF4_MERGE_CASE(7) NF4_MERGE_CASE(8)
        default: return NF4_ERR_UNSUPPORTED_SHAPE;
    }
#undef NF4_MERGE_CASE
    NF4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    // one wave: the column stripes times enough CTAs per stripe to fill the
    // resident CTA slots, each walking every gy-th row tile of its stripe
    int per_sm = 0;
    NF4_TRY_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kMgThreads, static_cast<size_t>(smem)));
    const int64_t gx = (w->k + kMgCols - 1) / kMgCols, row_tiles = (w->n + kMgRows - 1) / kMgRows;
    const int64_t slots = static_cast<int64_t>(std::max(1, per_sm)) * num_sms(current_device());
    const int64_t gy = std::max<int64_t>(1, std::min<int64_t>(row_tiles, slots / gx));
    const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    LaunchTimer t(KK_MERGE, s);
    const cudaError_t e = launch_ex(kern, grid, dim3(kMgThreads), static_cast<size_t>(smem), s, 0u, a);
    t.stop();
    if (e != cudaSuccess) return cuda_fail(e, __LINE__);
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

size_t qlora_fwd_workspace_bytes(int64_t M, int64_t n, int64_t k, int32_t r) {
    if (M <= 0 || n <= 0 || k <= 0 || r <= 0) return 256;
    return fwd_layout(M, r, num_sms(current_device())).total;
}

// Forward, with LoRA dropout when keep is non-null or rng.on (inverted dropout
// on the adapter input with the keep mask given, or drawn in the kernels; the
// branch is scaled by (alpha/r)/(1-p)).
nf4_status fwd_impl(const nf4_weight *w, const uint16_t *x, int64_t M, const uint16_t *A,
                    const uint16_t *B, int32_t r, float alpha, float p, const uint8_t *keep,
                    uint16_t *h, float *u_out, void *workspace, size_t ws_bytes, void *stream,
                    const DropRng &rng = DropRng{}) {
    nf4_status st = check_layer(w, x, M, A, B, r, alpha);
    if (st != NF4_OK) return st;
    const bool masked = keep != nullptr || rng.on;
    if (masked && !(p >= 0.0f && p < 1.0f)) return NF4_ERR_INVALID_ARG;
    if (M == 0) return NF4_OK;
    if (!h) return NF4_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(u_out) || !aligned16(keep)) return NF4_ERR_ALIGNMENT;
    const int sms = num_sms(current_device());
    const FwdLayout L = fwd_layout(M, r, sms);
    if (!workspace || ws_bytes < L.total) return NF4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NF4_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *u_s = reinterpret_cast<uint16_t *>(ws + L.us);
    const SkBuf sk{reinterpret_cast<float *>(ws + L.partial), reinterpret_cast<int *>(ws + L.flags),
                   sk_pairs_max(sms)};
    float scale = alpha / static_cast<float>(r);
    if (masked) scale = scale / (1.0f - p);
    if (decode_shape(w, M, r))
        return launch_decode(w, x, M, A, B, r, scale, h, u_out, reinterpret_cast<float *>(ws + L.upart), s,
                             nullptr, keep, rng);
    // u = x A^T (fp32, optional; under dropout the dropped elements of x are
    // zero) and bf16(scale u) for the up-projection stage; this kernel also
    // clears the GEMM's stream-K flags
    SkinnySpec su{x, M, w->k, Major::K, A, r, w->k, Major::K, r, u_out, u_s, scale, 0};
    if (masked) {
        su.mask_mode = 1;
        su.keep = keep;
        su.rng = rng;
        su.mx = M;
        su.kx = w->k;
    }
    st = skinny_launch(KK_LORA_U, &su, 1, s, sk.flags, sk.pairs_max * kSkFlagsPerPair);
    if (st != NF4_OK) return st;
    return launch_gemm_auto<false>(w, x, M, w->k, w->n, u_s, r, B, h, s, &sk);
}

nf4_status qlora_linear_fwd(const nf4_weight *w, const uint16_t *x, int64_t M, const uint16_t *A,
                            const uint16_t *B, int32_t r, float alpha, uint16_t *h, float *u_out,
                            void *workspace, size_t ws_bytes, void *stream) {
    return fwd_impl(w, x, M, A, B, r, alpha, 0.0f, nullptr, h, u_out, workspace, ws_bytes, stream);
}

nf4_status qlora_linear_fwd_dropout(const nf4_weight *w, const uint16_t *x, int64_t M,
                                    const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                                    float p, const uint8_t *keep, uint16_t *h, float *u_out,
                                    void *workspace, size_t ws_bytes, void *stream) {
    // an empty batch has an empty mask: keep may be null only then
    if ((M > 0 && !keep) || !(p >= 0.0f && p < 1.0f)) return NF4_ERR_INVALID_ARG;
    return fwd_impl(w, x, M, A, B, r, alpha, p, keep, h, u_out, workspace, ws_bytes, stream);
}

nf4_status qlora_multi_lora_fwd(const nf4_weight *w, const uint16_t *x, int64_t M,
                                const uint16_t *A_all, const uint16_t *B_all, int32_t r,
                                int32_t n_adapters, const float *alphas,
                                const int32_t *adapter_of_token, uint16_t *h, void *workspace,
                                size_t ws_bytes, void *stream) {
    if (n_adapters < 1 || n_adapters > kMaxAdapters || !alphas) return NF4_ERR_INVALID_ARG;
    const int32_t R = r * n_adapters;
    if (r < 8 || (r % 8) != 0 || R > 128) return NF4_ERR_UNSUPPORTED_SHAPE;
    float gscale[kMaxAdapters];
    for (int i = 0; i < n_adapters; ++i) {
        if (!std::isfinite(alphas[i])) return NF4_ERR_INVALID_ARG;
        gscale[i] = alphas[i] / static_cast<float>(r);
    }
    nf4_status st = check_layer(w, x, M, A_all, B_all, R, 1.0f);
    if (st != NF4_OK) return st;
    if (M == 0) return NF4_OK;
    if (!h || !adapter_of_token) return NF4_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(adapter_of_token)) return NF4_ERR_ALIGNMENT;
    const int sms = num_sms(current_device());
    const FwdLayout L = fwd_layout(M, R, sms);
    if (!workspace || ws_bytes < L.total) return NF4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NF4_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *u_s = reinterpret_cast<uint16_t *>(ws + L.us);
    const SkBuf sk{reinterpret_cast<float *>(ws + L.partial), reinterpret_cast<int *>(ws + L.flags),
                   sk_pairs_max(sms)};
    RowGroups groups;
    groups.row_group = adapter_of_token;
    groups.group_width = r;
    groups.ngroups = n_adapters;
    groups.gscale = gscale;
    if (decode_shape(w, M, R))
        return launch_decode(w, x, M, A_all, B_all, R, 1.0f, h, nullptr,
                             reinterpret_cast<float *>(ws + L.upart), s, &groups);
    // u = x A_all^T for every stacked adapter; each token keeps its own adapter's
    // columns, scaled by that adapter's alpha / r; the launch also clears the GEMM's flags
    const SkinnySpec su{x, M, w->k, Major::K, A_all, R, w->k, Major::K, R, nullptr, u_s, 1.0f, 0};
    st = skinny_launch(KK_LORA_U, &su, 1, s, sk.flags, sk.pairs_max * kSkFlagsPerPair, nullptr, nullptr,
                       0, 0.f, &groups);
    if (st != NF4_OK) return st;
    return launch_gemm_auto<false>(w, x, M, w->k, w->n, u_s, R, B_all, h, s, &sk);
}

nf4_status qlora_linear_fwd_noalloc(const nf4_weight *w, const uint16_t *x, int64_t M,
                                    const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                                    uint16_t *h, float *u_out, void *stream) {
    nf4_status st = check_layer(w, x, M, A, B, r, alpha);
    if (st != NF4_OK) return st;
    if (M == 0) return NF4_OK;
    if (!h) return NF4_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(u_out)) return NF4_ERR_ALIGNMENT;
    // scratch: bf16 (alpha/r) x A^T [M, r], the workspace of qlora_linear_fwd
    const FwdLayout L = fwd_layout(M, r, 0, false);   // whole-tile schedule: no stream-K scratch
    if (L.total > kStaticScratchBytes) return NF4_ERR_UNSUPPORTED_SHAPE;
    uint8_t *ws = static_cast<uint8_t *>(static_scratch_on_current_device());
    if (!ws) {
        std::snprintf(t_last_error, sizeof t_last_error, "the scratch array's device address was not found");
        return NF4_ERR_CUDA;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint16_t *u_s = reinterpret_cast<uint16_t *>(ws + L.us);
    const float scale = alpha / static_cast<float>(r);
    // same dispatch as qlora_linear_fwd: a few tokens take the decode kernel
    if (decode_shape(w, M, r))
        return launch_decode(w, x, M, A, B, r, scale, h, u_out, reinterpret_cast<float *>(ws + L.upart), s);
    st = skinny_product(KK_LORA_U, x, M, w->k, Major::K, A, r, w->k, Major::K, r, u_out, u_s,
                        scale, 0, s);
    if (st != NF4_OK) return st;
    return launch_gemm_auto<false>(w, x, M, w->k, w->n, u_s, r, B, h, s);
}

size_t qlora_bwd_workspace_bytes(int64_t M, int64_t n, int64_t k, int32_t r) {
    if (M < 0 || n <= 0 || k <= 0 || r <= 0) return 256;
    return bwd_layout(std::max<int64_t>(M, 1), r, num_sms(current_device())).total;
}

// dX += keep . (Vs A) on the tensor cores (the adapter part of dX under dropout).
nf4_status lora_add(const float *base, const uint16_t *Vs, const uint16_t *A, const uint8_t *keep,
                    const DropRng &rng, int64_t M, int64_t K, int32_t r, uint16_t *dX, cudaStream_t s) {
    LoraAddArgs a{};
    a.base = base;
    a.M = M;
    a.K = K;
    a.r = r;
    a.rp = (r + 15) / 16 * 16;
    a.Vs = Vs;
    a.A = A;
    a.keep = keep;
    a.rng = rng;
    a.dX = dX;
    if ((M + kMgRows - 1) / kMgRows > 65535) return NF4_ERR_UNSUPPORTED_SHAPE;
    const dim3 grid(static_cast<unsigned>((K + kMgCols - 1) / kMgCols), static_cast<unsigned>((M + kMgRows - 1) / kMgRows));
    const int smem = lora_add_smem_bytes(a.rp);
    void (*kern)(const LoraAddArgs) = nullptr;
    switch (a.rp / 16) {
        case 1: kern = qlora_lora_add_kernel<1>; break;
        case 2: kern = qlora_lora_add_kernel<2>; break;
        case 3: kern = qlora_lora_add_kernel<3>; break;
        case 4: kern = qlora_lora_add_kernel<4>; break;
        case 5: kern = qlora_lora_add_kernel<5>; break;
        case 6: kern = qlora_lora_add_kernel<6>; break;
        case 7: kern = qlora_lora_add_kernel<7>; break;
        case 8: kern = qlora_lora_add_kernel<8>; break;
        default: return NF4_ERR_UNSUPPORTED_SHAPE;
    }
    NF4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    LaunchTimer t(KK_LORA_ADD, s);
    const cudaError_t e = launch_ex(kern, grid, dim3(kMgThreads), static_cast<size_t>(smem), s, 0u, a);
    t.stop();
    if (e != cudaSuccess) return cuda_fail(e, __LINE__);
    NF4_TRY_CUDA(cudaGetLastError());
    return NF4_OK;
}

// Backward, with LoRA dropout when keep is non-null or rng.on (u, when given,
// is the forward's masked u = (keep . x) A^T).
// Adapter gradients in bf16 (dA, dB) or, when grads32 is set, in fp32 (the
// same pointers, as float).
nf4_status bwd_impl(const nf4_weight *w, const uint16_t *x, int64_t M, const uint16_t *A,
                    const uint16_t *B, int32_t r, float alpha, float p, const uint8_t *keep,
                    const uint16_t *dY, const float *u, uint16_t *dX, void *dA, void *dB,
                    void *workspace, size_t ws_bytes, void *stream, bool grads32 = false,
                    const DropRng &rng = DropRng{}) {
    nf4_status st = check_layer(w, x, M, A, B, r, alpha);
    if (st != NF4_OK) return st;
    const bool masked = keep != nullptr || rng.on;
    if (masked && !(p >= 0.0f && p < 1.0f)) return NF4_ERR_INVALID_ARG;
    if (!dA || !dB || (M > 0 && !dY)) return NF4_ERR_INVALID_ARG;
    if (!aligned16(dY) || !aligned16(u) || !aligned16(dX) || !aligned16(dA) || !aligned16(dB) ||
        !aligned16(keep))
        return NF4_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t N = w->n, K = w->k;
    if (M == 0) {
        LaunchTimer t(KK_ZERO, s);
        // zero gradients: 2-byte words, twice as many for fp32
        const int64_t per = grads32 ? 2 : 1;
        const cudaError_t e1 = launch_ex(zero_u16_kernel, dim3(64), dim3(256), 0, s, 0u,
                                         static_cast<uint16_t *>(dA), per * int64_t(r) * K);
        const cudaError_t e2 = launch_ex(zero_u16_kernel, dim3(64), dim3(256), 0, s, 0u,
                                         static_cast<uint16_t *>(dB), per * N * r);
        t.stop();
        if (e1 != cudaSuccess || e2 != cudaSuccess) return cuda_fail(e1 != cudaSuccess ? e1 : e2, __LINE__);
        NF4_TRY_CUDA(cudaGetLastError());
        return NF4_OK;
    }
    const int sms = num_sms(current_device());
    const BwdLayout L = bwd_layout(M, r, sms);
    // under dropout the workspace also holds dY W~ in fp32 ([M, k]) for the masked add
    const size_t need = masked ? L.total + align256(size_t(M) * size_t(K) * 4) : L.total;
    if (!workspace || ws_bytes < need) return NF4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NF4_ERR_ALIGNMENT;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *u_s = reinterpret_cast<uint16_t *>(ws + L.us);
    uint16_t *v_s = reinterpret_cast<uint16_t *>(ws + L.vs);
    float *base32 = reinterpret_cast<float *>(ws + L.total);
    const SkBuf sk{reinterpret_cast<float *>(ws + L.partial), reinterpret_cast<int *>(ws + L.flags),
                   sk_pairs_max(sms)};
    float scale = alpha / static_cast<float>(r);
    if (masked) scale = scale / (1.0f - p);

    // bf16(s u): recomputed from x here (masked under dropout), or converted from
    // the saved u by the v launch
    if (!u) {
        SkinnySpec su{x, M, K, Major::K, A, r, K, Major::K, r, nullptr, u_s, scale, 0};
        if (masked) {
            su.mask_mode = 1;
            su.keep = keep;
            su.rng = rng;
            su.mx = M;
            su.kx = K;
        }
        st = skinny_launch(KK_LORA_U, &su, 1, s);
        if (st != NF4_OK) return st;
    }
    // v = dY B  ->  bf16(s v)
    {
        const SkinnySpec sv{dY, M, N, Major::K, B, N, r, Major::MN, r, nullptr, v_s, scale, 0};
        st = skinny_launch(KK_LORA_V, &sv, 1, s, nullptr, 0, u, u ? u_s : nullptr, u ? M * r : 0, scale);
        if (st != NF4_OK) return st;
    }
    // dB = dY^T bf16(s u) ([N, r]) and dA = (x^T bf16(s v))^T ([r, K]) in one launch (under
    // dropout dA takes the masked x), which also clears the dgrad GEMM's stream-K flags
    {
        SkinnySpec j[2] = {{dY, M, N, Major::MN, u_s, M, r, Major::MN, r, nullptr, nullptr, 1.0f, 0},
                           {x, M, K, Major::MN, v_s, M, r, Major::MN, r, nullptr, nullptr, 1.0f, 1}};
        if (grads32) {
            j[0].out_f32 = static_cast<float *>(dB);
            j[1].out_f32 = static_cast<float *>(dA);
        } else {
            j[0].out_bf16 = static_cast<uint16_t *>(dB);
            j[1].out_bf16 = static_cast<uint16_t *>(dA);
        }
        if (masked) {
            j[1].mask_mode = 2;
            j[1].keep = keep;
            j[1].rng = rng;
            j[1].mx = M;
            j[1].kx = K;
        }
        st = skinny_launch(KK_LORA_DBDA, j, 2, s, sk.flags, sk.pairs_max * kSkFlagsPerPair);
        if (st != NF4_OK) return st;
    }
    if (!dX) return NF4_OK;
    // dX = dY W~ + bf16(s v) A; under dropout the adapter part is masked
    // element-wise, so it is added by its own kernel after the GEMM
    if (!masked) return launch_gemm_auto<true>(w, dY, M, N, K, v_s, r, A, dX, s, &sk);
    st = launch_gemm_auto<true>(w, dY, M, N, K, nullptr, r, A, dX, s, &sk, base32);
    if (st != NF4_OK) return st;
    return lora_add(base32, v_s, A, keep, rng, M, K, r, dX, s);
}

nf4_status qlora_linear_bwd(const nf4_weight *w, const uint16_t *x, int64_t M, const uint16_t *A,
                            const uint16_t *B, int32_t r, float alpha, const uint16_t *dY,
                            const float *u, uint16_t *dX, uint16_t *dA, uint16_t *dB,
                            void *workspace, size_t ws_bytes, void *stream) {
    return bwd_impl(w, x, M, A, B, r, alpha, 0.0f, nullptr, dY, u, dX, dA, dB, workspace, ws_bytes,
                    stream);
}

nf4_status qlora_linear_bwd_f32grad(const nf4_weight *w, const uint16_t *x, int64_t M,
                                    const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                                    const uint16_t *dY, const float *u, uint16_t *dX, float *dA,
                                    float *dB, void *workspace, size_t ws_bytes, void *stream) {
    return bwd_impl(w, x, M, A, B, r, alpha, 0.0f, nullptr, dY, u, dX, dA, dB, workspace, ws_bytes,
                    stream, true);
}

size_t qlora_bwd_dropout_workspace_bytes(int64_t M, int64_t n, int64_t k, int32_t r) {
    if (M < 0 || n <= 0 || k <= 0 || r <= 0) return 256;
    return bwd_layout(std::max<int64_t>(M, 1), r, num_sms(current_device())).total +
           align256(size_t(std::max<int64_t>(M, 1)) * size_t(k) * 4);
}

nf4_status qlora_linear_bwd_dropout(const nf4_weight *w, const uint16_t *x, int64_t M,
                                    const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                                    float p, const uint8_t *keep, const uint16_t *dY, const float *u,
                                    uint16_t *dX, uint16_t *dA, uint16_t *dB, void *workspace,
                                    size_t ws_bytes, void *stream) {
    // an empty batch has an empty mask: keep may be null only then
    if ((M > 0 && !keep) || !(p >= 0.0f && p < 1.0f)) return NF4_ERR_INVALID_ARG;
    return bwd_impl(w, x, M, A, B, r, alpha, p, keep, dY, u, dX, dA, dB, workspace, ws_bytes, stream);
}

// The generator's parameters of one (p, seed, offset): the drop threshold is
// floor(p * 2^32), exact in fp64 for an fp32 p.
DropRng make_drop_rng(float p, uint64_t seed, uint64_t offset) {
    DropRng d{};
    d.k0 = static_cast<uint32_t>(seed);
    d.k1 = static_cast<uint32_t>(seed >> 32);
    d.o0 = static_cast<uint32_t>(offset);
    d.o1 = static_cast<uint32_t>(offset >> 32);
    const double t = std::floor(static_cast<double>(p) * 4294967296.0);
    d.thresh = t > 0.0 ? (t < 4294967295.0 ? static_cast<uint32_t>(t) : 0xFFFFFFFFu) : 0u;
    d.on = 1;
    return d;
}

nf4_status qlora_linear_fwd_dropout_philox(const nf4_weight *w, const uint16_t *x, int64_t M,
                                           const uint16_t *A, const uint16_t *B, int32_t r,
                                           float alpha, float p, uint64_t seed, uint64_t offset,
                                           uint16_t *h, float *u_out, void *workspace,
                                           size_t ws_bytes, void *stream) {
    if (!(p >= 0.0f && p < 1.0f)) return NF4_ERR_INVALID_ARG;
    return fwd_impl(w, x, M, A, B, r, alpha, p, nullptr, h, u_out, workspace, ws_bytes, stream,
                    make_drop_rng(p, seed, offset));
}

nf4_status qlora_linear_bwd_dropout_philox(const nf4_weight *w, const uint16_t *x, int64_t M,
                                           const uint16_t *A, const uint16_t *B, int32_t r,
                                           float alpha, float p, uint64_t seed, uint64_t offset,
                                           const uint16_t *dY, const float *u, uint16_t *dX,
                                           uint16_t *dA, uint16_t *dB, void *workspace,
                                           size_t ws_bytes, void *stream) {
    if (!(p >= 0.0f && p < 1.0f)) return NF4_ERR_INVALID_ARG;
    return bwd_impl(w, x, M, A, B, r, alpha, p, nullptr, dY, u, dX, dA, dB, workspace, ws_bytes,
                    stream, false, make_drop_rng(p, seed, offset));
}

}  // extern "C"
