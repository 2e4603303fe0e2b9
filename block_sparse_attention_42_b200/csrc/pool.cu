// pool.cu -- a1: per-block mean of Q and K token vectors and mean L2 norm of V token vectors.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.1 Stem算子优化: compact block-level
//  representations of Q and K are precomputed so that one GEMM gives every block score;
//  §3.2 OAM: the value amplitude enters the metric.]
//
// HBM-bound streaming reduction.  One CTA reduces one block of tokens of one tensor
// (blockIdx.z: 0 Q, 1 K, 2 V) over all heads: every thread owns a 16-byte column vector of
// the [token, head*d] rows and walks a strided subset of the block's tokens, so each token
// row is read once with fully coalesced 16-byte loads.  Sums are kept in fp64 (cheap here:
// the kernel waits on HBM) so the pooled means carry only the final fp32 rounding.  What
// bounds it is the number of 16-byte loads in flight per SM, so the E4M3 instantiation keeps
// its fp64 sums in shared memory and its registers at 64 per thread, for four CTAs per SM.
// Each Q/K mean is written as two fp32 arrays, a TF32-exact high part and the remainder,
// which the tensor-core score GEMM consumes directly (score_tc.cu).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"

namespace bsa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kBatch = 8;  // tokens whose loads each thread issues together

template <int DT>
struct Elem;
template <>
struct Elem<0> {  // bf16
    static constexpr int kVec = 8;
    __device__ static void decode(const uint4& raw, float (&f)[8]) {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct Elem<1> {  // e4m3: summed through the f16x2 path in pool_kernel, no float decode
    static constexpr int kVec = 16;
};
// Two E4M3 codes (low 16 bits of w >> 16*half) -> f16x2, exact; NaN codes give NaN.
__device__ __forceinline__ uint32_t cvt_e4m3x2(uint32_t w, int half) {
    uint32_t d;
    if (half == 0)
        asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}" : "=r"(d) : "r"(w));
    else
        asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}" : "=r"(d) : "r"(w));
    return d;
}

// c + the low / high f16 half of h2, rounded once to fp32 (sm_100 mixed-precision add).
__device__ __forceinline__ float add_f16lo(uint32_t h2, float c) {
    float d;
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.f16 %0, l, %2;\n\t}" : "=f"(d) : "r"(h2), "f"(c));
    return d;
}
__device__ __forceinline__ float add_f16hi(uint32_t h2, float c) {
    float d;
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.f16 %0, h, %2;\n\t}" : "=f"(d) : "r"(h2), "f"(c));
    return d;
}
// c + half * half (low / high half of h2), one fp32 rounding.
__device__ __forceinline__ float sq_f16lo(uint32_t h2, float c) {
    float d;
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.f16 %0, l, l, %2;\n\t}" : "=f"(d) : "r"(h2), "f"(c));
    return d;
}
__device__ __forceinline__ float sq_f16hi(uint32_t h2, float c) {
    float d;
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.f16 %0, h, h, %2;\n\t}" : "=f"(d) : "r"(h2), "f"(c));
    return d;
}

template <>
struct Elem<2> {  // fp32
    static constexpr int kVec = 4;
    __device__ static void decode(const uint4& raw, float (&f)[4]) {
        f[0] = __uint_as_float(raw.x);
        f[1] = __uint_as_float(raw.y);
        f[2] = __uint_as_float(raw.z);
        f[3] = __uint_as_float(raw.w);
    }
};

struct PoolArgs {
    TensorArg t[3];
    int H[3];
    float* mean_out[3];  // TF32 high part of each mean; nullptr for V
    float* lo_out[3];    // fp32 remainder: mean = mean_out + lo_out exactly
    float* vnorm_out;
    int N, d, block, nb;
};

// Stores a pooled mean as hi + lo: hi keeps the sign, exponent and top 10 mantissa bits (exact
// in TF32, so the tensor cores read it unchanged) and lo = m - hi is exact in fp32.  A
// non-finite mean keeps lo = 0 so that hi + lo still gives it back.
__device__ __forceinline__ void store_split(const PoolArgs& a, int which, int64_t o, float m) {
    const float hi = __uint_as_float(__float_as_uint(m) & 0xFFFFE000u);
    a.mean_out[which][o] = hi;
    a.lo_out[which][o] = isfinite(m) ? m - hi : 0.f;
}

template <int DT>
__global__ void __launch_bounds__(kPoolThreads, DT == 1 ? 4 : 2) pool_kernel(const PoolArgs a) {
    constexpr int V = Elem<DT>::kVec;
    const int which = blockIdx.z;
    const TensorArg x = a.t[which];
    const int H = a.H[which];
    const int i = blockIdx.x, b = blockIdx.y;
    const int d = a.d;
    const int vec_per_head = d / V;
    const int vpt = H * vec_per_head;                   // 16-byte vectors per token row
    const int tg_count = vpt >= kPoolThreads ? 1 : kPoolThreads / vpt;
    const int t_lo = i * a.block;
    const int t_hi = min(a.N, t_lo + a.block);
    const double inv_cnt = 1.0 / static_cast<double>(t_hi - t_lo);
    const double scale = static_cast<double>(x.scale);
    const bool is_v = (which == 2);

    __shared__ double red[kPoolThreads][V + 1];

    const int tg = threadIdx.x / (vpt >= kPoolThreads ? kPoolThreads : vpt);
    // Threads past tg_count * vpt only take part in the warp shuffles.
    const bool active_tg = tg < tg_count;
    for (int v0 = 0; v0 < (vpt >= kPoolThreads ? vpt : 1); v0 += kPoolThreads) {
        const int v = (vpt >= kPoolThreads ? v0 + threadIdx.x : threadIdx.x % vpt);
        const bool live = active_tg && v < vpt;
        const int h = live ? v / vec_per_head : 0;
        const int c0 = live ? (v % vec_per_head) * V : 0;
        // fp64 sums: in registers for BF16 / fp32; for E4M3, in this thread's row of `red`
        // (read and written only by this thread until the reduction below), which leaves the
        // registers to keep more loads in flight.
        double acc[DT == 1 ? 1 : V];
#pragma unroll
        for (int e = 0; e < V; ++e) {
            if constexpr (DT == 1)
                red[threadIdx.x][e] = 0.0;
            else
                acc[e] = 0.0;
        }
        double nacc = 0.0;
        // E4M3: values are multiples of 2^-9 below 2^9, so any sum of up to 64 of them is exact
        // in fp32; such partial sums are flushed into the fp64 sums every kFlush batches.  Each
        // pair of codes becomes an f16x2 word (a hardware conversion, exact, NaN codes to NaN)
        // whose halves are added into the fp32 sums directly (sm_100 mixed-precision add).
        float facc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) facc[e] = 0.f;
        constexpr int kFlush = 64 / kBatch;
        int nbatch = 0;
        const char* base = static_cast<const char*>(x.ptr);
        const int esz = DT == 0 ? 2 : (DT == 1 ? 1 : 4);
        // Tokens in batches of kBatch per thread: all of a batch's 16-byte loads are issued
        // before any is consumed, so each thread keeps several HBM requests in flight.  The trip
        // count is uniform across the CTA so the warp shuffles below never diverge.
        for (int tb = t_lo; tb < t_hi; tb += tg_count * kBatch) {
            uint4 raw[kBatch];
            bool okb[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int t = tb + u * tg_count + tg;
                okb[u] = live && t < t_hi;
                raw[u] = make_uint4(0u, 0u, 0u, 0u);
                if (okb[u]) {
                    const int64_t off = static_cast<int64_t>(b) * x.sb + static_cast<int64_t>(t) * x.st +
                                        static_cast<int64_t>(h) * x.sh + c0;
                    raw[u] = __ldg(reinterpret_cast<const uint4*>(base + off * esz));
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                if constexpr (DT == 1) {
                    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
                    float ss = 0.f;  // V: fp32 sum of squares (relative error ~1e-7 in the norm)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t h01 = cvt_e4m3x2(w[q], 0), h23 = cvt_e4m3x2(w[q], 1);
                        facc[4 * q + 0] = add_f16lo(h01, facc[4 * q + 0]);
                        facc[4 * q + 1] = add_f16hi(h01, facc[4 * q + 1]);
                        facc[4 * q + 2] = add_f16lo(h23, facc[4 * q + 2]);
                        facc[4 * q + 3] = add_f16hi(h23, facc[4 * q + 3]);
                        if (is_v) ss = sq_f16hi(h23, sq_f16lo(h23, sq_f16hi(h01, sq_f16lo(h01, ss))));
                    }
                    if (is_v) {
                        for (int o = 1; o < vec_per_head; o <<= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
                        if (okb[u]) nacc += static_cast<double>(sqrtf(ss));
                    }
                } else {
                    float f[V];
                    Elem<DT>::decode(raw[u], f);  // zero bits decode to +0 in every format
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] += static_cast<double>(f[e]);
                    if (is_v) {
                        double ss = 0.0;
#pragma unroll
                        for (int e = 0; e < V; ++e) ss += static_cast<double>(f[e]) * static_cast<double>(f[e]);
                        // Sum of squares over the head's d/V lanes (aligned power-of-two lane groups).
                        for (int o = 1; o < vec_per_head; o <<= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
                        if (okb[u]) nacc += sqrt(ss);
                    }
                }
            }
            if constexpr (DT == 1) {
                if (++nbatch == kFlush) {
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        red[threadIdx.x][e] += static_cast<double>(facc[e]);
                        facc[e] = 0.f;
                    }
                    nbatch = 0;
                }
            }
        }
        if constexpr (DT == 1) {
#pragma unroll
            for (int e = 0; e < V; ++e) red[threadIdx.x][e] += static_cast<double>(facc[e]);
        }
        auto sum_at = [&](int e) -> double {
            if constexpr (DT == 1)
                return red[threadIdx.x][e];
            else
                return acc[e];
        };
        if (vpt >= kPoolThreads) {
            if (live) {
                const int64_t o = ((static_cast<int64_t>(b) * H + h) * a.nb + i) * d + c0;
                if (!is_v) {
#pragma unroll
                    for (int e = 0; e < V; ++e) store_split(a, which, o + e, static_cast<float>(sum_at(e) * inv_cnt * scale));
                } else if (c0 == 0) {
                    a.vnorm_out[(static_cast<int64_t>(b) * H + h) * a.nb + i] =
                        static_cast<float>(nacc * inv_cnt * scale);
                }
            }
        } else {
            if constexpr (DT != 1) {
#pragma unroll
                for (int e = 0; e < V; ++e) red[threadIdx.x][e] = acc[e];
            }
            red[threadIdx.x][V] = nacc;
            __syncthreads();
            if (live && tg == 0) {
                for (int g = 1; g < tg_count; ++g) {
#pragma unroll
                    for (int e = 0; e <= V; ++e) red[threadIdx.x][e] += red[g * vpt + threadIdx.x][e];
                }
                const int64_t o = ((static_cast<int64_t>(b) * H + h) * a.nb + i) * d + c0;
                if (!is_v) {
#pragma unroll
                    for (int e = 0; e < V; ++e)
                        store_split(a, which, o + e, static_cast<float>(red[threadIdx.x][e] * inv_cnt * scale));
                } else if (c0 == 0) {
                    a.vnorm_out[(static_cast<int64_t>(b) * H + h) * a.nb + i] =
                        static_cast<float>(red[threadIdx.x][V] * inv_cnt * scale);
                }
            }
        }
    }
}

// Group-shared selection: the mean over the G query heads of a KV-head group of their pooled
// Q means, as hi + lo like the per-head means.  One thread per output element; each head's mean
// is read as hi + lo (exactly the fp32 mean) and the G of them are summed in fp64, so the group
// mean carries one final fp32 rounding.
__global__ void __launch_bounds__(256) group_mean_kernel(const float* __restrict__ qhi, const float* __restrict__ qlo,
                                                         int B, int Hq, int Hkv, int nb, int d,
                                                         float* __restrict__ ghi, float* __restrict__ glo) {
    const int64_t n_out = static_cast<int64_t>(B) * Hkv * nb * d;
    const int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (o >= n_out) return;
    const int G = Hq / Hkv;
    const int64_t per_head = static_cast<int64_t>(nb) * d;
    const int64_t bk = o / per_head, rest = o % per_head;  // bk = b * Hkv + hk
    const int64_t b = bk / Hkv, hk = bk % Hkv;
    double acc = 0.0;
    for (int g = 0; g < G; ++g) {
        const int64_t src = (b * Hq + hk * G + g) * per_head + rest;
        acc += static_cast<double>(qhi[src]) + static_cast<double>(qlo[src]);
    }
    const float m = static_cast<float>(acc / G);
    const float hi = __uint_as_float(__float_as_uint(m) & 0xFFFFE000u);
    ghi[o] = hi;
    glo[o] = isfinite(m) ? m - hi : 0.f;
}

}  // namespace

cudaError_t launch_group_mean(const float* qhi, const float* qlo, int B, int Hq, int Hkv, int nb, int d, float* ghi,
                              float* glo, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(B) * Hkv * nb * d;
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
    group_mean_kernel<<<blocks, 256, 0, s>>>(qhi, qlo, B, Hq, Hkv, nb, d, ghi, glo);
    return cudaGetLastError();
}

cudaError_t launch_pool(int dtype, TensorArg q, TensorArg k, TensorArg v, int B, int N, int Hq, int Hkv, int d,
                        int block, float* qbar, float* qlo, float* kbar, float* klo, float* vbar, cudaStream_t s) {
    PoolArgs a;
    a.t[0] = q;
    a.t[1] = k;
    a.t[2] = v;
    a.H[0] = Hq;
    a.H[1] = Hkv;
    a.H[2] = Hkv;
    a.mean_out[0] = qbar;
    a.mean_out[1] = kbar;
    a.mean_out[2] = nullptr;
    a.lo_out[0] = qlo;
    a.lo_out[1] = klo;
    a.lo_out[2] = nullptr;
    a.vnorm_out = vbar;
    a.N = N;
    a.d = d;
    a.block = block;
    a.nb = (N + block - 1) / block;
    dim3 grid(a.nb, B, 3);
    if (dtype == 0)
        pool_kernel<0><<<grid, kPoolThreads, 0, s>>>(a);
    else if (dtype == 1)
        pool_kernel<1><<<grid, kPoolThreads, 0, s>>>(a);
    else
        pool_kernel<2><<<grid, kPoolThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace bsa
