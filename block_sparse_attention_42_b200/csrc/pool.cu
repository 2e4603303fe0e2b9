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
// the kernel waits on HBM) so the pooled means carry only the final fp32 rounding.
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
struct Elem<1> {  // e4m3
    static constexpr int kVec = 16;
    __device__ static void decode(const uint4& raw, float (&f)[16]) {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFFu), __NV_E4M3);
            __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
            float2 a = __half22float2(*reinterpret_cast<__half2*>(&lo));
            float2 b = __half22float2(*reinterpret_cast<__half2*>(&hi));
            f[4 * i] = a.x;
            f[4 * i + 1] = a.y;
            f[4 * i + 2] = b.x;
            f[4 * i + 3] = b.y;
        }
    }
};
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
    float* mean_out[3];  // nullptr for V
    float* vnorm_out;
    int N, d, block, nb;
};

template <int DT>
__global__ void __launch_bounds__(kPoolThreads, 2) pool_kernel(const PoolArgs a) {
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
        double acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.0;
        double nacc = 0.0;
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
        if (vpt >= kPoolThreads) {
            if (live) {
                const int64_t o = ((static_cast<int64_t>(b) * H + h) * a.nb + i) * d + c0;
                if (!is_v) {
#pragma unroll
                    for (int e = 0; e < V; ++e)
                        a.mean_out[which][o + e] = static_cast<float>(acc[e] * inv_cnt * x.scale);
                } else if (c0 == 0) {
                    a.vnorm_out[(static_cast<int64_t>(b) * H + h) * a.nb + i] =
                        static_cast<float>(nacc * inv_cnt * x.scale);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < V; ++e) red[threadIdx.x][e] = acc[e];
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
                        a.mean_out[which][o + e] = static_cast<float>(red[threadIdx.x][e] * inv_cnt * x.scale);
                } else if (c0 == 0) {
                    a.vnorm_out[(static_cast<int64_t>(b) * H + h) * a.nb + i] =
                        static_cast<float>(red[threadIdx.x][V] * inv_cnt * x.scale);
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_pool(int dtype, TensorArg q, TensorArg k, TensorArg v, int B, int N, int Hq, int Hkv, int d,
                        int block, float* qbar, float* kbar, float* vbar, cudaStream_t s) {
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
