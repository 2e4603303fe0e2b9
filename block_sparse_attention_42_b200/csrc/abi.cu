// abi.cu -- the extern "C" entry points of libbsa.so declared in include/bsa.h: argument
// validation (synchronous, nothing launched on error), workspace carving, TMA descriptor
// encoding and kernel launches.  No device memory is allocated here.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "../../include/bsa.h"
#include "internal.h"

namespace bsa {

__device__ unsigned g_device_error;  // per-device error word (kDevErr* bits)
constexpr int kTileCounters = 64;
__device__ int g_tile_counter[kTileCounters];  // per-launch counters of the dynamic tile schedule

namespace {

thread_local std::string g_last_error;

bsa_status_t fail(bsa_status_t st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

bsa_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(BSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int elt_bytes(int32_t dtype) { return dtype == BSA_BF16 ? 2 : (dtype == BSA_FP8_E4M3 ? 1 : (dtype == BSA_FP32 ? 4 : 0)); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bsa_status_t check_tensor(const bsa_tensor_t& t, const char* name, bool need_b) {
    if (t.ptr == nullptr) return fail(BSA_ERR_INVALID_ARG, "%s: null pointer", name);
    const int eb = elt_bytes(t.dtype);
    if (eb == 0) return fail(BSA_ERR_INVALID_ARG, "%s: unknown dtype %d", name, t.dtype);
    if (!aligned16(t.ptr)) return fail(BSA_ERR_INVALID_ARG, "%s: base pointer not 16-byte aligned", name);
    if (t.stride_t <= 0 || t.stride_h <= 0 || (need_b && t.stride_b <= 0))
        return fail(BSA_ERR_INVALID_ARG, "%s: strides must be positive", name);
    if ((t.stride_t * eb) % 16 || (t.stride_h * eb) % 16 || (need_b && (t.stride_b * eb) % 16))
        return fail(BSA_ERR_INVALID_ARG, "%s: strides must be multiples of 16 bytes", name);
    if (t.dtype == BSA_FP8_E4M3 && !(t.scale > 0.f && std::isfinite(t.scale)))
        return fail(BSA_ERR_INVALID_ARG, "%s: FP8 scale must be positive and finite", name);
    return BSA_OK;
}

TensorArg targ(const bsa_tensor_t& t) {
    TensorArg a;
    a.ptr = t.ptr;
    a.sb = t.stride_b;
    a.st = t.stride_t;
    a.sh = t.stride_h;
    a.scale = t.dtype == BSA_FP8_E4M3 ? t.scale : 1.f;
    return a;
}

unsigned* device_error_word(bsa_status_t* st) {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *st = cuda_fail(e, "cudaGetDevice");
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (addr[dev] == nullptr) {
        e = cudaGetSymbolAddress(&addr[dev], g_device_error);
        if (e != cudaSuccess) {
            addr[dev] = nullptr;
            *st = cuda_fail(e, "cudaGetSymbolAddress(device error word)");
            return nullptr;
        }
    }
    *st = BSA_OK;
    return static_cast<unsigned*>(addr[dev]);
}

// A tile counter for one attention launch, zeroed on `stream` ahead of it.  Launches take the
// per-device slots in turn, so two launches in flight share one only when 64 others were
// issued between them.
int* tile_counter(cudaStream_t stream, bsa_status_t* st) {
    static std::mutex mu;
    static void* base[64] = {};
    static unsigned turn[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *st = cuda_fail(e, "cudaGetDevice");
        return nullptr;
    }
    int* p = nullptr;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (base[dev] == nullptr) {
            e = cudaGetSymbolAddress(&base[dev], g_tile_counter);
            if (e != cudaSuccess) {
                base[dev] = nullptr;
                *st = cuda_fail(e, "cudaGetSymbolAddress(tile counters)");
                return nullptr;
            }
        }
        p = static_cast<int*>(base[dev]) + (turn[dev]++ % kTileCounters);
    }
    e = cudaMemsetAsync(p, 0, sizeof(int), stream);
    if (e != cudaSuccess) {
        *st = cuda_fail(e, "cudaMemsetAsync(tile counter)");
        return nullptr;
    }
    *st = BSA_OK;
    return p;
}

// ---------------------------------------------------------------- TPD budget (host copy)

int64_t tpd_kstar(int32_t nb, double density) {
    const int64_t T = static_cast<int64_t>(nb) * (nb + 1) / 2;
    const int64_t sum_m = 2 * static_cast<int64_t>(nb) - 1;
    int64_t k = static_cast<int64_t>(std::floor(density * static_cast<double>(T) + 0.5));
    if (k < sum_m) k = sum_m;
    if (k > T) k = T;
    return k;
}

bool tpd_args_ok(int32_t nb, double density, double decay) {
    return nb >= 1 && nb <= kMaxBlocks * 16 && density > 0.0 && density <= 1.0 && (decay == 0.0 || decay == 0.5);
}

// ---------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(bsa_status_t* st) {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    *st = fn ? BSA_OK : cuda_fail(err == cudaSuccess ? cudaErrorNotSupported : err, "cuTensorMapEncodeTiled lookup");
    return fn;
}

// 4-D tiled map over [d, rows, heads, outer] with 128-byte swizzle; box = 128 bytes of d x
// box_rows x 1 x 1.  Out-of-range boxes read zeros.
bsa_status_t make_map(CUtensorMap* m, const void* base, int eb, uint64_t d, uint64_t rows, uint64_t heads,
                      uint64_t outer, int64_t s_rows, int64_t s_heads, int64_t s_outer, uint32_t box_rows,
                      const char* name) {
    bsa_status_t st;
    EncodeTiledFn fn = encode_fn(&st);
    if (!fn) return st;
    const cuuint64_t dims[4] = {d, rows, heads, outer};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(s_rows) * eb, static_cast<cuuint64_t>(s_heads) * eb,
                                   static_cast<cuuint64_t>(s_outer) * eb};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / eb), box_rows, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = eb == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = fn(m, dt, 4,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(BSA_ERR_INVALID_ARG, "%s: cuTensorMapEncodeTiled failed (%d)", name, (int)r);
    return BSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// An NVTX range around one entry point, so a profiler's timeline shows each call of the C ABI
// with the kernels it launched (header-only NVTX; a no-op unless a tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Attention kernel.  Default: ws3 (attn_ws3.cu: persistent, two pipelined CTAs per SM with a
// TMA producer warp, an MMA warp and a softmax warpgroup; BF16 at d = 128 / block 128, whose
// stages do not fit two CTAs per SM that way, runs ws2 with P in TMEM).  BSA_ATTN_VARIANT picks
// another kernel for cross-checks: "serial" (attn.cu, one tile per CTA, no overlap inside a
// CTA) or "ws2".  All compute the same result and the tests cross-check every one.
cudaError_t launch_attn(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnArgs& a, cudaStream_t s) {
    const char* v = std::getenv("BSA_ATTN_VARIANT");
    if (v && std::strcmp(v, "serial") == 0) return launch_attention(fp8, paged, tq, tk, tv, a, s);
    if (v && std::strcmp(v, "ws2") == 0) return launch_attention_ws2(fp8, paged, tq, tk, tv, a, s);
    return launch_attention_ws3(fp8, paged, tq, tk, tv, a, s);
}

bsa_status_t attn_common_checks(const bsa_tensor_t& q, const bsa_tensor_t& k, const bsa_tensor_t& v,
                                const bsa_tensor_t& out, int32_t Hq, int32_t Hkv, int32_t d, int32_t block,
                                const int32_t* row_ptr, const int32_t* col_idx, int64_t max_k) {
    if (q.dtype != k.dtype || q.dtype != v.dtype)
        return fail(BSA_ERR_INVALID_ARG, "q, k and v must share a dtype");
    if (q.dtype != BSA_BF16 && q.dtype != BSA_FP8_E4M3)
        return fail(BSA_ERR_UNSUPPORTED, "attention supports BF16 or FP8_E4M3 inputs");
    if (out.dtype != BSA_BF16) return fail(BSA_ERR_UNSUPPORTED, "out must be BF16");
    if (Hq < 1 || Hkv < 1 || Hq % Hkv) return fail(BSA_ERR_INVALID_ARG, "Hq must be a positive multiple of Hkv");
    if (d != 64 && d != 128) return fail(BSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (block != 64 && block != 128) return fail(BSA_ERR_UNSUPPORTED, "block must be 64 or 128");
    if (q.dtype == BSA_FP8_E4M3 && (d != 128 || block != 128))
        return fail(BSA_ERR_UNSUPPORTED, "FP8 attention needs head_dim 128 and block 128");
    if (!row_ptr || !col_idx) return fail(BSA_ERR_INVALID_ARG, "row_ptr/col_idx are null");
    if (max_k < 1) return fail(BSA_ERR_INVALID_ARG, "max_k must be positive");
    return BSA_OK;
}


bsa_status_t prefill_checks(const bsa_tensor_t& q, const bsa_tensor_t& k, const bsa_tensor_t& v,
                            const bsa_tensor_t& out, int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                            int32_t block, const int32_t* row_ptr, const int32_t* col_idx, int64_t max_k) {
    bsa_status_t st;
    if ((st = check_tensor(q, "q", B > 1)) || (st = check_tensor(k, "k", B > 1)) || (st = check_tensor(v, "v", B > 1)) ||
        (st = check_tensor(out, "out", B > 1)))
        return st;
    if ((st = attn_common_checks(q, k, v, out, Hq, Hkv, d, block, row_ptr, col_idx, max_k))) return st;
    if (B < 1 || B > kMaxBatch || N < 1) return fail(BSA_ERR_INVALID_ARG, "bad B=%d / N=%d", B, N);
    const int nb = (N + block - 1) / block;
    if (nb > kMaxBlocks) return fail(BSA_ERR_UNSUPPORTED, "at most %d blocks per sequence", kMaxBlocks);
    if (static_cast<int64_t>(Hkv) * nb * (Hq / Hkv) > 0x7FFFFFFFll) return fail(BSA_ERR_UNSUPPORTED, "grid too large");
    return BSA_OK;
}

bsa_status_t prefill_launch(const bsa_tensor_t& q, const bsa_tensor_t& k, const bsa_tensor_t& v,
                            const bsa_tensor_t& out, int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                            int32_t block, const int32_t* row_ptr, int32_t row_ptr_stride, int32_t row_ptr_hstride,
                            int32_t allow_empty, const int32_t* col_idx, int64_t max_k, float softmax_scale,
                            float* lse, cudaStream_t stream, bool group = false, double skip_lambda = 0.0,
                            unsigned long long* skip_stats = nullptr) {
    bsa_status_t st;
    const int nb = (N + block - 1) / block;
    bsa_status_t est;
    unsigned* err = device_error_word(&est);
    if (!err) return est;
    const int eb = elt_bytes(q.dtype);
    CUtensorMap tq, tk, tv;
    if ((st = make_map(&tq, q.ptr, eb, d, N, Hq, B, q.stride_t, q.stride_h, B > 1 ? q.stride_b : q.stride_t * N, 128, "q")) ||
        (st = make_map(&tk, k.ptr, eb, d, N, Hkv, B, k.stride_t, k.stride_h, B > 1 ? k.stride_b : k.stride_t * N, block, "k")) ||
        (st = make_map(&tv, v.ptr, eb, d, N, Hkv, B, v.stride_t, v.stride_h, B > 1 ? v.stride_b : v.stride_t * N, block, "v")))
        return st;
    AttnArgs a;
    std::memset(&a, 0, sizeof a);
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.d = d;
    a.block = block;
    a.nb_max = nb;
    a.N = N;
    a.cu_seqlens = nullptr;
    for (int b = 0; b < B; ++b) a.seqlen[b] = N;
    a.row_ptr = row_ptr;
    a.row_ptr_stride = row_ptr_stride;
    a.row_ptr_hstride = row_ptr_hstride;
    a.allow_empty = allow_empty;
    a.col_idx = col_idx;
    a.max_k = max_k;
    const float tau = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
    const bool fp8 = q.dtype == BSA_FP8_E4M3;
    a.scale_log2 = tau * 1.4426950408889634f * (fp8 ? q.scale * k.scale : 1.f);
    a.out_scale = fp8 ? v.scale : 1.f;
    a.out = out.ptr;
    a.osb = out.stride_b;
    a.ost = out.stride_t;
    a.osh = out.stride_h;
    a.lse = lse;
    a.lse_stride = N;
    a.err = err;
    a.list_per_group = group ? 1 : 0;
    a.skip_on = skip_lambda > 0.0 ? 1 : 0;
    a.skip_log2 = skip_lambda > 0.0 ? static_cast<float>(std::log2(skip_lambda)) : 0.f;
    a.skip_stats = skip_stats;
    if (!(a.tile_counter = tile_counter(stream, &est))) return est;
    // Group-shared lists: the GQA-packed kernel where it applies (BSA_ATTN_VARIANT still picks a
    // per-head kernel for cross-checks), else the per-head kernels on the shared lists.
    const char* var = std::getenv("BSA_ATTN_VARIANT");
    const bool packed = group && attention_group_packed(fp8, a) && (!var || std::strcmp(var, "group") == 0);
    cudaError_t e = packed
                        ? launch_attention_group(fp8, false, tq, tk, tv, a, stream)
                        : launch_attn(fp8, false, tq, tk, tv, a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "bsa_prefill launch");
    return BSA_OK;
}


// bsa_prefill_mask workspace: row_ptr [B*Hq][nb+1] | col_idx [B*Hq][nb(nb+1)/2].
size_t mask_ws_bytes(int32_t B, int32_t Hq, int32_t nb) {
    return align256(sizeof(int32_t) * size_t(B) * Hq * (nb + 1)) +
           sizeof(int32_t) * size_t(B) * Hq * (size_t(nb) * (nb + 1) / 2);
}

bsa_status_t mask_checks(const uint8_t* mask, int64_t mask_stride, int32_t B, int32_t Hq, int32_t nb) {
    if (!mask) return fail(BSA_ERR_INVALID_ARG, "block_mask is null");
    if (B < 1 || B > kMaxBatch || Hq < 1) return fail(BSA_ERR_INVALID_ARG, "bad B=%d / Hq=%d", B, Hq);
    if (nb < 1 || nb > kMaxBlocks) return fail(BSA_ERR_UNSUPPORTED, "nb must be in [1, %d]", kMaxBlocks);
    if (mask_stride < nb || mask_stride % 16 != 0)
        return fail(BSA_ERR_INVALID_ARG, "mask_stride (%lld) must be >= nb (%d) and a multiple of 16",
                    static_cast<long long>(mask_stride), nb);
    if (reinterpret_cast<uintptr_t>(mask) & 15u) return fail(BSA_ERR_INVALID_ARG, "block_mask must be 16-byte aligned");
    // one warp per mask row, eight rows per CTA, grid.x < 2^31
    if (static_cast<int64_t>(B) * Hq * nb > 8ll * 0x7FFFFFFFll) return fail(BSA_ERR_UNSUPPORTED, "grid too large");
    return BSA_OK;
}

}  // namespace

void set_last_error(const char* msg) { g_last_error = msg; }

}  // namespace bsa

using namespace bsa;

extern "C" {

int64_t bsa_tpd_budget(int32_t nb, double density, double tpd_decay, int32_t* k_out) {
    if (!tpd_args_ok(nb, density, tpd_decay)) return -1;
    const int64_t kstar = tpd_kstar(nb, density);
    if (!k_out) return kstar;
    const bool half = tpd_decay == 0.5;
    auto share = [&](double c, int i) -> int64_t {
        const double n = static_cast<double>(i + 1), m = i == 0 ? 1.0 : 2.0;
        const double w = half ? std::sqrt(n) : n;
        volatile double t = c * w;  // one rounding, no contraction
        double tt = t;
        if (tt < m) tt = m;
        if (tt > n) tt = n;
        volatile double sc = tt * 4294967296.0;
        return static_cast<int64_t>(std::floor(static_cast<double>(sc)));
    };
    const int64_t target = kstar * (int64_t(1) << 32);
    double lo = 0.0, hi = static_cast<double>(nb);
    for (int it = 0; it < 64; ++it) {
        volatile double sum = lo + hi;
        const double mid = sum * 0.5;
        int64_t tot = 0;
        for (int i = 0; i < nb; ++i) tot += share(mid, i);
        if (tot >= target)
            hi = mid;
        else
            lo = mid;
    }
    int64_t whole = 0;
    struct Rem {
        uint32_t f;
        int32_t i;
    };
    Rem* rem = new Rem[nb];
    int nrem = 0;
    for (int i = 0; i < nb; ++i) {
        const int64_t F = share(hi, i);
        k_out[i] = static_cast<int32_t>(F >> 32);
        whole += k_out[i];
        if (k_out[i] < i + 1) rem[nrem++] = Rem{static_cast<uint32_t>(F & 0xFFFFFFFFll), i};
    }
    int64_t R = kstar - whole;
    // Partial selection of the R largest fractions (earlier row first on ties).
    for (int64_t r = 0; r < R && r < nrem; ++r) {
        int best = static_cast<int>(r);
        for (int q = static_cast<int>(r) + 1; q < nrem; ++q)
            if (rem[q].f > rem[best].f || (rem[q].f == rem[best].f && rem[q].i < rem[best].i)) best = q;
        Rem t = rem[r];
        rem[r] = rem[best];
        rem[best] = t;
        k_out[rem[r].i] += 1;
    }
    delete[] rem;
    return kstar;
}

size_t bsa_score_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t nb, int32_t d) {
    if (B < 1 || Hq < 1 || Hkv < 1 || nb < 1 || d < 1) return 0;
    return 2 * align256(sizeof(float) * size_t(B) * Hq * nb * d) +
           2 * align256(sizeof(float) * size_t(B) * Hkv * nb * d) + align256(sizeof(float) * size_t(B) * Hkv * nb);
}

size_t bsa_score_group_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t nb, int32_t d) {
    const size_t base = bsa_score_workspace_bytes(B, Hq, Hkv, nb, d);
    if (base == 0) return 0;
    return base + 2 * align256(sizeof(float) * size_t(B) * Hkv * nb * d);
}

}  // extern "C"

namespace bsa {
namespace {

// stem_score and stem_score_group: pool (a1), then the score GEMM (a2) with one query row per
// query head, or (group) one per KV-head group from the group mean of the heads' pooled Q.
bsa_status_t score_common(bool group, const bsa_tensor_t& q, const bsa_tensor_t& k, const bsa_tensor_t& v, int32_t B,
                          int32_t N, int32_t Hq, int32_t Hkv, int32_t d, int32_t block, int32_t metric,
                          float softmax_scale, float* scores, int32_t nb_stride, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
    bsa_status_t st;
    if ((st = check_tensor(q, "q", B > 1)) || (st = check_tensor(k, "k", B > 1)) || (st = check_tensor(v, "v", B > 1)))
        return st;
    if (q.dtype != k.dtype || q.dtype != v.dtype) return fail(BSA_ERR_INVALID_ARG, "q, k and v must share a dtype");
    if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv)
        return fail(BSA_ERR_INVALID_ARG, "bad sizes (B=%d N=%d Hq=%d Hkv=%d)", B, N, Hq, Hkv);
    if (d != 64 && d != 128) return fail(BSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (block != 64 && block != 128) return fail(BSA_ERR_UNSUPPORTED, "block must be 64 or 128");
    if (metric < BSA_METRIC_OAM || metric > BSA_METRIC_OAM_MUL) return fail(BSA_ERR_INVALID_ARG, "unknown metric");
    const int nb = (N + block - 1) / block;
    if (B > 65535 || Hq > 65535) return fail(BSA_ERR_UNSUPPORTED, "B and Hq must be <= 65535");
    if (!scores) return fail(BSA_ERR_INVALID_ARG, "scores is null");
    if (nb_stride < nb) return fail(BSA_ERR_INVALID_ARG, "nb_stride (%d) < number of blocks (%d)", nb_stride, nb);
    const size_t need = group ? bsa_score_group_workspace_bytes(B, Hq, Hkv, nb, d)
                              : bsa_score_workspace_bytes(B, Hq, Hkv, nb, d);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(BSA_ERR_WORKSPACE, "workspace must be >= %zu bytes and 256-byte aligned", need);
    // Workspace: [qhi | qlo | khi | klo | vbar (| ghi | glo)], each part 256-byte aligned.
    const size_t qbytes = align256(sizeof(float) * size_t(B) * Hq * nb * d);
    const size_t kbytes = align256(sizeof(float) * size_t(B) * Hkv * nb * d);
    const size_t vbytes = align256(sizeof(float) * size_t(B) * Hkv * nb);
    char* w = static_cast<char*>(ws);
    float* qhi = reinterpret_cast<float*>(w);
    float* qlo = reinterpret_cast<float*>(w + qbytes);
    float* khi = reinterpret_cast<float*>(w + 2 * qbytes);
    float* klo = reinterpret_cast<float*>(w + 2 * qbytes + kbytes);
    float* vbar = reinterpret_cast<float*>(w + 2 * qbytes + 2 * kbytes);
    const float tau = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
    const int dt = q.dtype == BSA_BF16 ? 0 : (q.dtype == BSA_FP8_E4M3 ? 1 : 2);
    cudaError_t e =
        launch_pool(dt, targ(q), targ(k), targ(v), B, N, Hq, Hkv, d, block, qhi, qlo, khi, klo, vbar, stream);
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    int Hrows = Hq;  // query-side heads of the score GEMM
    if (group) {
        float* ghi = reinterpret_cast<float*>(w + 2 * qbytes + 2 * kbytes + vbytes);
        float* glo = reinterpret_cast<float*>(w + 2 * qbytes + 3 * kbytes + vbytes);
        e = launch_group_mean(qhi, qlo, B, Hq, Hkv, nb, d, ghi, glo, stream);
        if (e != cudaSuccess) return cuda_fail(e, "group mean launch");
        qhi = ghi;
        qlo = glo;
        Hrows = Hkv;
    }
    // Score GEMM on the tensor cores (3xTF32, score_tc.cu); BSA_SCORE_VARIANT=simt selects the
    // fp32 FMA kernel (score.cu), which computes the same scores to fp32 rounding.
    const char* sv = std::getenv("BSA_SCORE_VARIANT");
    if (sv && std::strcmp(sv, "simt") == 0) {
        e = launch_score(qhi, qlo, khi, klo, vbar, B, Hrows, Hkv, nb, d, tau, metric, scores, nb_stride, stream);
    } else {
        bsa_status_t est;
        unsigned* err = device_error_word(&est);
        if (err == nullptr) return est;
        CUtensorMap mqh, mql, mkh, mkl;
        const int64_t ro = d, qh = int64_t(nb) * d, kh = int64_t(nb) * d;
        if ((st = make_map(&mqh, qhi, 4, d, nb, Hrows, B, ro, qh, qh * Hrows, 128, "qhi")) ||
            (st = make_map(&mql, qlo, 4, d, nb, Hrows, B, ro, qh, qh * Hrows, 128, "qlo")) ||
            (st = make_map(&mkh, khi, 4, d, nb, Hkv, B, ro, kh, kh * Hkv, 128, "khi")) ||
            (st = make_map(&mkl, klo, 4, d, nb, Hkv, B, ro, kh, kh * Hkv, 128, "klo")))
            return st;
        e = launch_score_tc(mqh, mql, mkh, mkl, vbar, B, Hrows, Hkv, nb, d, tau, metric, scores, nb_stride, err,
                            stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, "score launch");
    return BSA_OK;
}

// stem_score_select: the score matrix of one chunk of KV-head groups of one sequence at a time,
// so that at most kScoreChunkBytes of it exist at once (about the size of the L2), consumed by
// the top-k.  (Each chunk costs a score and three select launches; at 128K tokens 64 MiB chunks
// took 0.69 ms against 0.66 ms for 128 MiB.)
constexpr size_t kScoreChunkBytes = size_t(128) << 20;

int score_select_groups(int32_t Hq, int32_t Hkv, int nb) {
    const size_t per_group = sizeof(float) * size_t(Hq / Hkv) * nb * nb;
    int cg = static_cast<int>(kScoreChunkBytes / per_group);
    if (cg < 1) cg = 1;
    if (cg > Hkv) cg = Hkv;
    while (Hkv % cg) --cg;
    return cg;
}

}  // namespace
}  // namespace bsa

extern "C" {

bsa_status_t stem_score(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N, int32_t Hq,
                        int32_t Hkv, int32_t d, int32_t block, int32_t metric, float softmax_scale, float* scores,
                        int32_t nb_stride, void* ws, size_t ws_bytes, cudaStream_t stream) {
    NvtxRange nvtx_range("stem_score");
    return score_common(false, q, k, v, B, N, Hq, Hkv, d, block, metric, softmax_scale, scores, nb_stride, ws,
                        ws_bytes, stream);
}

bsa_status_t stem_score_group(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N, int32_t Hq,
                              int32_t Hkv, int32_t d, int32_t block, int32_t metric, float softmax_scale,
                              float* scores, int32_t nb_stride, void* ws, size_t ws_bytes, cudaStream_t stream) {
    NvtxRange nvtx_range("stem_score_group");
    return score_common(true, q, k, v, B, N, Hq, Hkv, d, block, metric, softmax_scale, scores, nb_stride, ws,
                        ws_bytes, stream);
}

size_t bsa_score_select_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t N, int32_t block,
                                        int32_t d) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || N < 1 || block < 1 || d < 1) return 0;
    const int nb = (N + block - 1) / block;
    const int cg = score_select_groups(Hq, Hkv, nb);
    return bsa_score_workspace_bytes(B, Hq, Hkv, nb, d) +
           align256(sizeof(float) * size_t(cg) * (Hq / Hkv) * nb * nb);
}

bsa_status_t stem_score_select(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N, int32_t Hq,
                               int32_t Hkv, int32_t d, int32_t block, int32_t metric, float softmax_scale,
                               double density, double tpd_decay, int32_t* row_ptr, int32_t* col_idx, int64_t max_k,
                               void* ws, size_t ws_bytes, cudaStream_t stream) {
    NvtxRange nvtx_range("stem_score_select");
    bsa_status_t st;
    if ((st = check_tensor(q, "q", B > 1)) || (st = check_tensor(k, "k", B > 1)) || (st = check_tensor(v, "v", B > 1)))
        return st;
    if (q.dtype != k.dtype || q.dtype != v.dtype) return fail(BSA_ERR_INVALID_ARG, "q, k and v must share a dtype");
    if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv)
        return fail(BSA_ERR_INVALID_ARG, "bad sizes (B=%d N=%d Hq=%d Hkv=%d)", B, N, Hq, Hkv);
    if (B > kMaxBatch) return fail(BSA_ERR_UNSUPPORTED, "B must be in [1, %d]", kMaxBatch);
    if (d != 64 && d != 128) return fail(BSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (block != 64 && block != 128) return fail(BSA_ERR_UNSUPPORTED, "block must be 64 or 128");
    if (metric < BSA_METRIC_OAM || metric > BSA_METRIC_OAM_MUL) return fail(BSA_ERR_INVALID_ARG, "unknown metric");
    const int nb = (N + block - 1) / block;
    if (nb > kMaxBlocks) return fail(BSA_ERR_UNSUPPORTED, "at most %d blocks per sequence", kMaxBlocks);
    if (!row_ptr || !col_idx) return fail(BSA_ERR_INVALID_ARG, "row_ptr/col_idx are null");
    if (!(density > 0.0 && density <= 1.0)) return fail(BSA_ERR_INVALID_ARG, "density must be in (0, 1]");
    if (!(tpd_decay == 0.0 || tpd_decay == 0.5)) return fail(BSA_ERR_UNSUPPORTED, "tpd_decay must be 0 or 0.5");
    const int64_t kstar = tpd_kstar(nb, density);
    if (kstar > max_k)
        return fail(BSA_ERR_INVALID_ARG, "max_k=%lld is below the budget %lld", (long long)max_k, (long long)kstar);
    const size_t need = bsa_score_select_workspace_bytes(B, Hq, Hkv, N, block, d);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(BSA_ERR_WORKSPACE, "workspace must be >= %zu bytes and 256-byte aligned", need);
    bsa_status_t est;
    unsigned* err = device_error_word(&est);
    if (err == nullptr) return est;
    // Workspace: the pooled means as in stem_score, then the score chunk.
    const size_t qbytes = align256(sizeof(float) * size_t(B) * Hq * nb * d);
    const size_t kbytes = align256(sizeof(float) * size_t(B) * Hkv * nb * d);
    const size_t vbytes = align256(sizeof(float) * size_t(B) * Hkv * nb);
    char* w = static_cast<char*>(ws);
    float* qhi = reinterpret_cast<float*>(w);
    float* qlo = reinterpret_cast<float*>(w + qbytes);
    float* khi = reinterpret_cast<float*>(w + 2 * qbytes);
    float* klo = reinterpret_cast<float*>(w + 2 * qbytes + kbytes);
    float* vbar = reinterpret_cast<float*>(w + 2 * qbytes + 2 * kbytes);
    float* chunk = reinterpret_cast<float*>(w + 2 * qbytes + 2 * kbytes + vbytes);
    const float tau = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
    const int dt = q.dtype == BSA_BF16 ? 0 : (q.dtype == BSA_FP8_E4M3 ? 1 : 2);
    cudaError_t e =
        launch_pool(dt, targ(q), targ(k), targ(v), B, N, Hq, Hkv, d, block, qhi, qlo, khi, klo, vbar, stream);
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    SelectSeqs all;
    all.B = B;
    for (int b = 0; b < B; ++b) {
        all.nb[b] = nb;
        all.kstar[b] = kstar;
    }
    e = launch_tpd_budget(all, nb, tpd_decay == 0.5, row_ptr, stream);
    if (e != cudaSuccess) return cuda_fail(e, "budget launch");
    SelectSeqs one;
    one.B = 1;
    one.nb[0] = nb;
    one.kstar[0] = kstar;
    const int G = Hq / Hkv, cg = score_select_groups(Hq, Hkv, nb);
    const int64_t hs = int64_t(nb) * d;  // floats per head of a pooled tensor
    for (int b = 0; b < B; ++b) {
        for (int hk0 = 0; hk0 < Hkv; hk0 += cg) {
            const int h0 = hk0 * G;
            CUtensorMap mqh, mql, mkh, mkl;
            const int64_t qo = (int64_t(b) * Hq + h0) * hs, ko = (int64_t(b) * Hkv + hk0) * hs;
            if ((st = make_map(&mqh, qhi + qo, 4, d, nb, cg * G, 1, d, hs, hs * Hq, 128, "qhi")) ||
                (st = make_map(&mql, qlo + qo, 4, d, nb, cg * G, 1, d, hs, hs * Hq, 128, "qlo")) ||
                (st = make_map(&mkh, khi + ko, 4, d, nb, cg, 1, d, hs, hs * Hkv, 128, "khi")) ||
                (st = make_map(&mkl, klo + ko, 4, d, nb, cg, 1, d, hs, hs * Hkv, 128, "klo")))
                return st;
            e = launch_score_tc(mqh, mql, mkh, mkl, vbar + (int64_t(b) * Hkv + hk0) * nb, 1, cg * G, cg, nb, d, tau,
                                metric, chunk, nb, err, stream);
            if (e != cudaSuccess) return cuda_fail(e, "score launch");
            e = launch_select_rows(chunk, one, cg * G, nb, row_ptr + int64_t(b) * (nb + 1),
                                   col_idx + (int64_t(b) * Hq + h0) * max_k, max_k, stream);
            if (e != cudaSuccess) return cuda_fail(e, "select launch");
        }
    }
    return BSA_OK;
}

bsa_status_t stem_select(const float* scores, int32_t B, int32_t Hq, const int32_t* nb_per_seq, int32_t nb_stride,
                         double density, double tpd_decay, int32_t* row_ptr, int32_t* col_idx, int64_t max_k,
                         cudaStream_t stream) {
    NvtxRange nvtx_range("stem_select");
    if (!scores || !nb_per_seq || !row_ptr || !col_idx) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
    if (B < 1 || B > kMaxBatch) return fail(BSA_ERR_UNSUPPORTED, "B must be in [1, %d]", kMaxBatch);
    if (Hq < 1) return fail(BSA_ERR_INVALID_ARG, "Hq must be positive");
    if (nb_stride < 1 || nb_stride > kMaxBlocks)
        return fail(BSA_ERR_UNSUPPORTED, "nb_stride must be in [1, %d]", kMaxBlocks);
    if (!(density > 0.0 && density <= 1.0)) return fail(BSA_ERR_INVALID_ARG, "density must be in (0, 1]");
    if (!(tpd_decay == 0.0 || tpd_decay == 0.5)) return fail(BSA_ERR_UNSUPPORTED, "tpd_decay must be 0 or 0.5");
    SelectSeqs seqs;
    seqs.B = B;
    for (int b = 0; b < B; ++b) {
        const int nb = nb_per_seq[b];
        if (nb < 1 || nb > nb_stride) return fail(BSA_ERR_INVALID_ARG, "nb_per_seq[%d]=%d out of [1, nb_stride]", b, nb);
        seqs.nb[b] = nb;
        seqs.kstar[b] = tpd_kstar(nb, density);
        if (seqs.kstar[b] > max_k)
            return fail(BSA_ERR_INVALID_ARG, "max_k=%lld is below the budget %lld of sequence %d", (long long)max_k,
                        (long long)seqs.kstar[b], b);
    }
    cudaError_t e = launch_select(scores, seqs, Hq, nb_stride, tpd_decay == 0.5, row_ptr, col_idx, max_k, stream);
    if (e != cudaSuccess) return cuda_fail(e, "select launch");
    return BSA_OK;
}

bsa_status_t bsa_prefill(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out, int32_t B, int32_t N,
                         int32_t Hq, int32_t Hkv, int32_t d, int32_t block, const int32_t* row_ptr,
                         int32_t row_ptr_stride, const int32_t* col_idx, int64_t max_k, float softmax_scale,
                         float* lse, cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_prefill");
    bsa_status_t st;
    if ((st = prefill_checks(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, col_idx, max_k))) return st;
    const int nb = (N + block - 1) / block;
    if (row_ptr_stride < nb + 1) return fail(BSA_ERR_INVALID_ARG, "row_ptr_stride must be >= nb + 1");
    return prefill_launch(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, row_ptr_stride, 0, 0, col_idx, max_k,
                          softmax_scale, lse, stream);
}

bsa_status_t bsa_prefill_skip(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out, int32_t B,
                              int32_t N, int32_t Hq, int32_t Hkv, int32_t d, int32_t block, const int32_t* row_ptr,
                              int32_t row_ptr_stride, const int32_t* col_idx, int64_t max_k, float softmax_scale,
                              double skip_lambda, float* lse, unsigned long long* skip_stats,
                              cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_prefill_skip");
    bsa_status_t st;
    if ((st = prefill_checks(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, col_idx, max_k))) return st;
    const int nb = (N + block - 1) / block;
    if (row_ptr_stride < nb + 1) return fail(BSA_ERR_INVALID_ARG, "row_ptr_stride must be >= nb + 1");
    if (!(skip_lambda >= 0.0 && skip_lambda < 1.0))
        return fail(BSA_ERR_INVALID_ARG, "skip_lambda must be in [0, 1)");
    if (skip_lambda > 0.0 && q.dtype == BSA_BF16 && d == 128 && block == 128)
        return fail(BSA_ERR_UNSUPPORTED, "the threshold skip runs FP8, or BF16 with head_dim 64 or block 64");
    const char* var = std::getenv("BSA_ATTN_VARIANT");
    if (skip_lambda > 0.0 && var && std::strcmp(var, "ws3") != 0)
        return fail(BSA_ERR_UNSUPPORTED, "the threshold skip runs in the default attention kernel only");
    if (skip_stats && (reinterpret_cast<uintptr_t>(skip_stats) & 7u))
        return fail(BSA_ERR_INVALID_ARG, "skip_stats must be 8-byte aligned");
    // lambda = 0 runs the plain kernel; its statistics are then all zero and left untouched
    return prefill_launch(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, row_ptr_stride, 0, 0, col_idx, max_k,
                          softmax_scale, lse, stream, false, skip_lambda, skip_stats);
}

bsa_status_t bsa_prefill_group(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out, int32_t B,
                               int32_t N, int32_t Hq, int32_t Hkv, int32_t d, int32_t block, const int32_t* row_ptr,
                               int32_t row_ptr_stride, const int32_t* col_idx, int64_t max_k, float softmax_scale,
                               float* lse, cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_prefill_group");
    bsa_status_t st;
    if ((st = prefill_checks(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, col_idx, max_k))) return st;
    const int nb = (N + block - 1) / block;
    if (row_ptr_stride < nb + 1) return fail(BSA_ERR_INVALID_ARG, "row_ptr_stride must be >= nb + 1");
    return prefill_launch(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, row_ptr_stride, 0, 0, col_idx, max_k,
                          softmax_scale, lse, stream, true);
}

size_t bsa_mask_workspace_bytes(int32_t B, int32_t Hq, int32_t nb) {
    if (B < 1 || Hq < 1 || nb < 1 || nb > kMaxBlocks) return 0;
    return mask_ws_bytes(B, Hq, nb);
}

bsa_status_t bsa_mask_to_lists(const uint8_t* block_mask, int64_t mask_stride, int32_t B, int32_t Hq, int32_t nb,
                               int32_t* row_ptr, int32_t* col_idx, int64_t max_k, cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_mask_to_lists");
    bsa_status_t st;
    if ((st = mask_checks(block_mask, mask_stride, B, Hq, nb))) return st;
    if (!row_ptr || !col_idx) return fail(BSA_ERR_INVALID_ARG, "row_ptr/col_idx are null");
    if (max_k < static_cast<int64_t>(nb) * (nb + 1) / 2)
        return fail(BSA_ERR_INVALID_ARG, "max_k (%lld) < nb(nb+1)/2 = %lld", static_cast<long long>(max_k),
                    static_cast<long long>(nb) * (nb + 1) / 2);
    MaskListArgs m;
    std::memset(&m, 0, sizeof m);
    m.mask = block_mask;
    m.mask_stride = mask_stride;
    m.Hq = Hq;
    m.nb = nb;
    m.N = 0;  // no outputs: an empty row is just an empty list
    m.block = 1;
    m.d = 0;
    m.row_ptr = row_ptr;
    m.col_idx = col_idx;
    m.cap = max_k;
    cudaError_t e = launch_mask_lists(m, B, stream);
    if (e != cudaSuccess) return cuda_fail(e, "mask list launch");
    return BSA_OK;
}

bsa_status_t bsa_validate_lists(const int32_t* row_ptr, int64_t row_ptr_stride, int64_t row_ptr_head_stride,
                                const int32_t* col_idx, int64_t max_k, int32_t B, int32_t Hq,
                                const int32_t* nb_per_seq, int32_t allow_empty, cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_validate_lists");
    if (!row_ptr || !col_idx || !nb_per_seq) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
    if (B < 1 || B > kMaxBatch) return fail(BSA_ERR_UNSUPPORTED, "B must be in [1, %d]", kMaxBatch);
    if (Hq < 1) return fail(BSA_ERR_INVALID_ARG, "Hq must be positive");
    if (max_k < 1) return fail(BSA_ERR_INVALID_ARG, "max_k must be positive");
    ListCheckArgs c;
    std::memset(&c, 0, sizeof c);
    int nbmax = 0;
    for (int b = 0; b < B; ++b) {
        if (nb_per_seq[b] < 1 || nb_per_seq[b] > kMaxBlocks)
            return fail(BSA_ERR_UNSUPPORTED, "nb_per_seq[%d] = %d outside [1, %d]", b, nb_per_seq[b], kMaxBlocks);
        c.nb[b] = nb_per_seq[b];
        nbmax = nb_per_seq[b] > nbmax ? nb_per_seq[b] : nbmax;
    }
    if (row_ptr_head_stride < 0 || (row_ptr_head_stride > 0 && row_ptr_head_stride < nbmax + 1) ||
        row_ptr_stride < (row_ptr_head_stride > 0 ? row_ptr_head_stride * Hq : nbmax + 1))
        return fail(BSA_ERR_INVALID_ARG, "row_ptr strides too small for %d blocks x %d heads", nbmax, Hq);
    bsa_status_t est;
    unsigned* err = device_error_word(&est);
    if (!err) return est;
    c.B = B;
    c.Hq = Hq;
    c.row_ptr = row_ptr;
    c.rp_stride = row_ptr_stride;
    c.rp_hstride = row_ptr_head_stride;
    c.col_idx = col_idx;
    c.max_k = max_k;
    c.allow_empty = allow_empty ? 1 : 0;
    c.err = err;
    cudaError_t e = launch_validate_lists(c, stream);
    if (e != cudaSuccess) return cuda_fail(e, "list validation launch");
    return BSA_OK;
}

bsa_status_t bsa_prefill_mask(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out, int32_t B, int32_t N,
                              int32_t Hq, int32_t Hkv, int32_t d, int32_t block, const uint8_t* block_mask,
                              int64_t mask_stride, float softmax_scale, float* lse, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_prefill_mask");
    bsa_status_t st;
    if (!ws) return fail(BSA_ERR_WORKSPACE, "workspace is null");
    // (the list pointers are checked once they are carved out of the workspace)
    const int nb = N > 0 && block > 0 ? (N + block - 1) / block : 0;
    if ((st = prefill_checks(q, k, v, out, B, N, Hq, Hkv, d, block, static_cast<const int32_t*>(ws),
                             static_cast<const int32_t*>(ws), 1)))
        return st;
    if ((st = mask_checks(block_mask, mask_stride, B, Hq, nb))) return st;
    const size_t need = mask_ws_bytes(B, Hq, nb);
    if (ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return fail(BSA_ERR_WORKSPACE, "workspace must be >= %zu bytes and 256-byte aligned", need);
    int32_t* row_ptr = static_cast<int32_t*>(ws);
    int32_t* col_idx = reinterpret_cast<int32_t*>(static_cast<char*>(ws) +
                                                  align256(sizeof(int32_t) * size_t(B) * Hq * (nb + 1)));
    const int64_t cap = static_cast<int64_t>(nb) * (nb + 1) / 2;
    MaskListArgs m;
    std::memset(&m, 0, sizeof m);
    m.mask = block_mask;
    m.mask_stride = mask_stride;
    m.Hq = Hq;
    m.nb = nb;
    m.N = N;
    m.block = block;
    m.d = d;
    m.row_ptr = row_ptr;
    m.col_idx = col_idx;
    m.cap = cap;
    m.out = out.ptr;
    m.osb = out.stride_b;
    m.ost = out.stride_t;
    m.osh = out.stride_h;
    m.lse = lse;
    m.lse_stride = N;
    cudaError_t e = launch_mask_lists(m, B, stream);
    if (e != cudaSuccess) return cuda_fail(e, "mask list launch");
    return prefill_launch(q, k, v, out, B, N, Hq, Hkv, d, block, row_ptr, Hq * (nb + 1), nb + 1, 1, col_idx, cap,
                          softmax_scale, lse, stream);
}

namespace {

// bsa_prefill_paged and bsa_prefill_paged_group: checks, tensor maps and the launch; `group`
// selects one list per KV-head group (col_idx [B, Hkv, max_k]).
bsa_status_t paged_launch(bsa_tensor_t q, bsa_tensor_t out, const int32_t* cu_seqlens, const int32_t* seqlens_host,
                          int32_t B, bsa_tensor_t k_cache, bsa_tensor_t v_cache, int32_t num_pages,
                          int32_t page_size, const int32_t* page_table, int32_t max_pages, int32_t Hq, int32_t Hkv,
                          int32_t d, int32_t block, const int32_t* row_ptr, int32_t row_ptr_stride,
                          const int32_t* col_idx, int64_t max_k, float softmax_scale, float* lse,
                          cudaStream_t stream, bool group) {
    bsa_status_t st;
    if ((st = check_tensor(q, "q", false)) || (st = check_tensor(out, "out", false)) ||
        (st = check_tensor(k_cache, "k_cache", true)) || (st = check_tensor(v_cache, "v_cache", true)))
        return st;
    if ((st = attn_common_checks(q, k_cache, v_cache, out, Hq, Hkv, d, block, row_ptr, col_idx, max_k))) return st;
    if (!cu_seqlens || !seqlens_host || !page_table) return fail(BSA_ERR_INVALID_ARG, "null pointer argument");
    if (B < 1 || B > kMaxBatch) return fail(BSA_ERR_UNSUPPORTED, "B must be in [1, %d]", kMaxBatch);
    if (page_size != 64 || block % page_size) return fail(BSA_ERR_UNSUPPORTED, "page_size must be 64 and divide block");
    if (num_pages < 1 || max_pages < 1) return fail(BSA_ERR_INVALID_ARG, "num_pages/max_pages must be positive");
    AttnArgs a;
    std::memset(&a, 0, sizeof a);
    int64_t total = 0;
    int nb_max = 0, n_max = 0;
    for (int b = 0; b < B; ++b) {
        const int n = seqlens_host[b];
        if (n < 1) return fail(BSA_ERR_INVALID_ARG, "seqlens_host[%d]=%d must be positive", b, n);
        const int nb = (n + block - 1) / block;
        if (nb > kMaxBlocks) return fail(BSA_ERR_UNSUPPORTED, "at most %d blocks per sequence", kMaxBlocks);
        if ((n + page_size - 1) / page_size > max_pages)
            return fail(BSA_ERR_INVALID_ARG, "sequence %d needs more than max_pages pages", b);
        a.seqlen[b] = n;
        total += n;
        nb_max = nb > nb_max ? nb : nb_max;
        n_max = n > n_max ? n : n_max;
    }
    if (row_ptr_stride < nb_max + 1) return fail(BSA_ERR_INVALID_ARG, "row_ptr_stride must be >= max nb + 1");
    bsa_status_t est;
    unsigned* err = device_error_word(&est);
    if (!err) return est;
    const int eb = elt_bytes(q.dtype);
    CUtensorMap tq, tk, tv;
    if ((st = make_map(&tq, q.ptr, eb, d, total, Hq, 1, q.stride_t, q.stride_h, q.stride_t * total, 128, "q")) ||
        (st = make_map(&tk, k_cache.ptr, eb, d, page_size, Hkv, num_pages, k_cache.stride_t, k_cache.stride_h,
                       k_cache.stride_b, 64, "k_cache")) ||
        (st = make_map(&tv, v_cache.ptr, eb, d, page_size, Hkv, num_pages, v_cache.stride_t, v_cache.stride_h,
                       v_cache.stride_b, 64, "v_cache")))
        return st;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.d = d;
    a.block = block;
    a.nb_max = nb_max;
    a.N = n_max;
    a.cu_seqlens = cu_seqlens;
    a.row_ptr = row_ptr;
    a.row_ptr_stride = row_ptr_stride;
    a.col_idx = col_idx;
    a.max_k = max_k;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.page_size = page_size;
    a.num_pages = num_pages;
    const float tau = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
    const bool fp8 = q.dtype == BSA_FP8_E4M3;
    a.scale_log2 = tau * 1.4426950408889634f * (fp8 ? q.scale * k_cache.scale : 1.f);
    a.out_scale = fp8 ? v_cache.scale : 1.f;
    a.out = out.ptr;
    a.osb = 0;
    a.ost = out.stride_t;
    a.osh = out.stride_h;
    a.lse = lse;
    a.lse_stride = n_max;
    a.err = err;
    a.list_per_group = group ? 1 : 0;
    if (!(a.tile_counter = tile_counter(stream, &est))) return est;
    // Group-shared lists: the GQA-packed kernel where it applies (BSA_ATTN_VARIANT still picks a
    // per-head kernel for cross-checks), else the per-head kernels on the shared lists.
    const char* var = std::getenv("BSA_ATTN_VARIANT");
    const bool packed = group && attention_group_packed(fp8, a) && (!var || std::strcmp(var, "group") == 0);
    cudaError_t e = packed ? launch_attention_group(fp8, true, tq, tk, tv, a, stream)
                           : launch_attn(fp8, true, tq, tk, tv, a, stream);
    if (e != cudaSuccess) return cuda_fail(e, group ? "bsa_prefill_paged_group launch" : "bsa_prefill_paged launch");
    return BSA_OK;
}

}  // namespace

bsa_status_t bsa_prefill_paged(bsa_tensor_t q, bsa_tensor_t out, const int32_t* cu_seqlens, const int32_t* seqlens_host,
                               int32_t B, bsa_tensor_t k_cache, bsa_tensor_t v_cache, int32_t num_pages,
                               int32_t page_size, const int32_t* page_table, int32_t max_pages, int32_t Hq,
                               int32_t Hkv, int32_t d, int32_t block, const int32_t* row_ptr,
                               int32_t row_ptr_stride, const int32_t* col_idx, int64_t max_k, float softmax_scale,
                               float* lse, cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_prefill_paged");
    return paged_launch(q, out, cu_seqlens, seqlens_host, B, k_cache, v_cache, num_pages, page_size, page_table,
                        max_pages, Hq, Hkv, d, block, row_ptr, row_ptr_stride, col_idx, max_k, softmax_scale, lse,
                        stream, false);
}

bsa_status_t bsa_prefill_paged_group(bsa_tensor_t q, bsa_tensor_t out, const int32_t* cu_seqlens,
                                     const int32_t* seqlens_host, int32_t B, bsa_tensor_t k_cache,
                                     bsa_tensor_t v_cache, int32_t num_pages, int32_t page_size,
                                     const int32_t* page_table, int32_t max_pages, int32_t Hq, int32_t Hkv,
                                     int32_t d, int32_t block, const int32_t* row_ptr, int32_t row_ptr_stride,
                                     const int32_t* col_idx, int64_t max_k, float softmax_scale, float* lse,
                                     cudaStream_t stream) {
    NvtxRange nvtx_range("bsa_prefill_paged_group");
    return paged_launch(q, out, cu_seqlens, seqlens_host, B, k_cache, v_cache, num_pages, page_size, page_table,
                        max_pages, Hq, Hkv, d, block, row_ptr, row_ptr_stride, col_idx, max_k, softmax_scale, lse,
                        stream, true);
}

const char* bsa_last_error(void) { return g_last_error.c_str(); }

bsa_status_t bsa_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
    if (limit_ns < 1000ull || limit_ns > 1000000000ull) return fail(BSA_ERR_INVALID_ARG, "limit_ns must be in [1e3, 1e9]");
    bsa_status_t est;
    unsigned* err = device_error_word(&est);
    if (err == nullptr) return est;
    const cudaError_t e = launch_wait_timeout_selftest(err, limit_ns, stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait-timeout self-test launch");
    return BSA_OK;
}

bsa_status_t bsa_check_device_error(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned v = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    if (v & kDevErrTimeout) return fail(BSA_ERR_TIMEOUT, "a kernel wait ran out of time");
    if (v & kDevErrInvalidList) return fail(BSA_ERR_INVALID_LIST, "a list entry was outside [0, query block]");
    if (v & kDevErrSmemAlign)
        return fail(BSA_ERR_CUDA, "an attention kernel found its dynamic shared memory not 1024-byte aligned");
    if (v & kDevErrInvalidPage)
        return fail(BSA_ERR_INVALID_PAGE, "a page-table entry of a token inside its sequence was outside [0, num_pages)");
    return BSA_OK;
}

}  // extern "C"
