// score.cu -- a2: OAM block scores from the pooled representations.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.1 Stem算子优化: because the metric
//  is purely additive (no softmax, no gather), one standard GEMM of the block-level Q and K
//  representations gives every block score; §3.2 OAM: the score is weighted by the value
//  amplitude.]
//
//   S[b,h,i,j] = tau * Qbar[b,h,i] . Kbar[b,h/G,j]  (+ ln vbar[b,h/G,j] for OAM,
//                                                   * vbar for OAM_MUL), j <= i; -inf above.
//
// Per query head this is a [nb x d] x [d x nb] product restricted to the causal lower
// triangle.  64x64 output tiles, tiles wholly above the diagonal are skipped, fp32 FMA
// accumulation (the scores must be fp32-accurate: they decide the top-k lists).
#include <cmath>

#include "internal.h"

namespace bsa {
namespace {

constexpr int kTile = 64;
constexpr int kKc = 32;

__device__ __forceinline__ float4 load_mean(const float* hi, const float* lo, int64_t o) {
    const float4 h = *reinterpret_cast<const float4*>(hi + o);
    const float4 l = *reinterpret_cast<const float4*>(lo + o);
    return make_float4(h.x + l.x, h.y + l.y, h.z + l.z, h.w + l.w);
}

__global__ void __launch_bounds__(256)
    score_kernel(const float* __restrict__ qhi, const float* __restrict__ qlo, const float* __restrict__ khi,
                 const float* __restrict__ klo, const float* __restrict__ vbar, int Hq, int Hkv, int nb, int d,
                 float tau, int metric, float* __restrict__ S, int nbs) {
    __shared__ __align__(16) float As[kKc][kTile + 4];
    __shared__ __align__(16) float Bs[kKc][kTile + 4];
    __shared__ float lv[kTile];

    // Lower-triangular tile pair (ti, tj), tj <= ti.
    const int x = blockIdx.x;
    int ti = static_cast<int>((sqrtf(8.f * x + 1.f) - 1.f) * 0.5f);
    while ((ti + 1) * (ti + 2) / 2 <= x) ++ti;
    while (ti * (ti + 1) / 2 > x) --ti;
    const int tj = x - ti * (ti + 1) / 2;
    const int h = blockIdx.y, b = blockIdx.z;
    const int hk = h / (Hq / Hkv);
    const int i0 = ti * kTile, j0 = tj * kTile;

    const int64_t qo = (static_cast<int64_t>(b) * Hq + h) * nb * d;
    const int64_t ko = (static_cast<int64_t>(b) * Hkv + hk) * nb * d;
    const float* vb = vbar + (static_cast<int64_t>(b) * Hkv + hk) * nb;

    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    if (tid < kTile) {
        const int j = j0 + tid;
        const float a = j < nb ? vb[j] : 1.f;
        lv[tid] = metric == 0 ? logf(a) : a;
    }

    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kKc) {
        // 64 rows x 32 columns per operand: two float4 per thread each.
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int idx = tid + rep * 256;     // 0..511
            const int row = idx / 8, q4 = (idx % 8) * 4;
            float4 av = make_float4(0.f, 0.f, 0.f, 0.f), bv = av;
            // The pooled means are stored as hi + lo; the fp32 sum is exact.
            if (i0 + row < nb) av = load_mean(qhi, qlo, qo + static_cast<int64_t>(i0 + row) * d + k0 + q4);
            if (j0 + row < nb) bv = load_mean(khi, klo, ko + static_cast<int64_t>(j0 + row) * d + k0 + q4);
            As[q4 + 0][row] = av.x;
            As[q4 + 1][row] = av.y;
            As[q4 + 2][row] = av.z;
            As[q4 + 3][row] = av.w;
            Bs[q4 + 0][row] = bv.x;
            Bs[q4 + 1][row] = bv.y;
            Bs[q4 + 2][row] = bv.z;
            Bs[q4 + 3][row] = bv.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kKc; ++kk) {
            const float4 a4 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
            const float4 b4 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
            const float ar[4] = {a4.x, a4.y, a4.z, a4.w};
            const float br[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(ar[r], br[c], acc[r][c]);
        }
        __syncthreads();
    }

    float* out = S + (static_cast<int64_t>(b) * Hq + h) * nbs * nbs;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = i0 + ty * 4 + r;
        if (i >= nb) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = j0 + tx * 4 + c;
            if (j >= nb) continue;
            float s;
            if (j > i) {
                s = -INFINITY;
            } else {
                s = tau * acc[r][c];
                const float a = lv[tx * 4 + c];
                if (metric == 0)
                    s = s + a;
                else if (metric == 2)
                    s = s * a;
            }
            out[static_cast<int64_t>(i) * nbs + j] = s;
        }
    }
}

}  // namespace

cudaError_t launch_score(const float* qhi, const float* qlo, const float* khi, const float* klo, const float* vbar,
                         int B, int Hq, int Hkv, int nb, int d, float tau, int metric, float* scores, int nb_stride,
                         cudaStream_t s) {
    const int nt = (nb + kTile - 1) / kTile;
    dim3 grid(nt * (nt + 1) / 2, Hq, B);
    score_kernel<<<grid, 256, 0, s>>>(qhi, qlo, khi, klo, vbar, Hq, Hkv, nb, d, tau, metric, scores, nb_stride);
    return cudaGetLastError();
}

}  // namespace bsa
