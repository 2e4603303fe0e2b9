// score_tc.cu -- a2: OAM block scores on the tcgen05 tensor cores, fp32-accurate.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.1 Stem算子优化: because the metric
//  is purely additive (no softmax, no gather), one standard GEMM of the block-level Q and K
//  representations gives every block score; §3.2 OAM: the score is weighted by the value
//  amplitude.]
//
//   S[b,h,i,j] = tau * Qbar[b,h,i] . Kbar[b,h/G,j]  (+ ln vbar[b,h/G,j] for OAM,
//                                                   * vbar for OAM_MUL), j <= i; -inf above.
//
// The scores decide integer top-k lists, so the product must be fp32-accurate; TF32 or BF16
// alone would move scores by ~1e-3 and reorder near-equal candidates.  Each fp32 operand is
// split into hi = x with its 13 low mantissa bits cleared (exactly representable in TF32) and
// lo = x - hi (exact in fp32), and the tensor cores accumulate hi*hi + hi*lo + lo*hi in fp32
// (kind::tf32).  The dropped lo*lo term and the TF32 truncation of lo are ~2^-20 of the
// product.
//
// One CTA (128 threads) computes one 128 x 128 tile (query blocks x key blocks) of one query
// head; tiles wholly above the diagonal are not launched.  The contraction runs over head_dim
// in chunks of 32 values (one 128-byte swizzled row): all threads load the fp32 chunk of Qbar
// and Kbar, split it and store hi / lo into shared memory in the 128-byte-swizzled K-major
// layout; thread 0 issues the 3 x 4 MMAs of the chunk into TMEM and commits them to an
// mbarrier that gates the next chunk.  The epilogue reads the accumulator row of each thread
// from TMEM and writes the scores.  Every wait is bounded.
#include <cmath>

#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kTileS = 128;       // query blocks x key blocks per CTA
constexpr int kChunk = 32;        // fp32 values of head_dim per chunk (one 128-byte row)
constexpr int kOpBytes = kTileS * 128;  // one operand chunk in shared memory (16 KB)

struct ScoreSmem {
    uint8_t a_hi[kOpBytes], a_lo[kOpBytes], b_hi[kOpBytes], b_lo[kOpBytes];
    float lv[kTileS];
    uint64_t mma_done;
    uint32_t tmem_slot;
    int abort_flag;
};

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// 128 rows x 32 fp32 of `src` (row stride d floats, rows >= n_valid read as zero) -> hi / lo
// operands in the 128-byte-swizzled K-major layout.
__device__ __forceinline__ void stage_chunk(const float* __restrict__ src, int row0, int n_valid, int d, int k0,
                                            uint8_t* hi, uint8_t* lo) {
#pragma unroll
    for (int rep = 0; rep < kTileS * 8 / 128; ++rep) {
        const int idx = threadIdx.x + rep * 128;  // 0 .. 1023
        const int r = idx / 8, c = idx % 8;        // row, 16-byte chunk within the 128-byte row
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row0 + r < n_valid) v = __ldg(reinterpret_cast<const float4*>(src + static_cast<int64_t>(row0 + r) * d + k0) + c);
        const float4 vh = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
        const float4 vl = make_float4(v.x - vh.x, v.y - vh.y, v.z - vh.z, v.w - vh.w);
        const int off = r * 128 + ((c ^ (r & 7)) * 16);
        *reinterpret_cast<float4*>(hi + off) = vh;
        *reinterpret_cast<float4*>(lo + off) = vl;
    }
}

template <int D>
__global__ void __launch_bounds__(128) score_tf32x3_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                           const float* __restrict__ vbar, int Hq, int Hkv, int nb,
                                                           float tau, int metric, float* __restrict__ S, int nbs,
                                                           unsigned* err) {
    extern __shared__ uint8_t smem_raw[];
    ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid / 32;

    // Lower-triangular tile pair (ti, tj), tj <= ti.
    const int x = blockIdx.x;
    int ti = static_cast<int>((sqrtf(8.f * x + 1.f) - 1.f) * 0.5f);
    while ((ti + 1) * (ti + 2) / 2 <= x) ++ti;
    while (ti * (ti + 1) / 2 > x) --ti;
    const int tj = x - ti * (ti + 1) / 2;
    const int h = blockIdx.y, b = blockIdx.z;
    const int hk = h / (Hq / Hkv);
    const int i0 = ti * kTileS, j0 = tj * kTileS;
    const float* A = qbar + (static_cast<int64_t>(b) * Hq + h) * nb * D;
    const float* Bm = kbar + (static_cast<int64_t>(b) * Hkv + hk) * nb * D;
    const float* vb = vbar + (static_cast<int64_t>(b) * Hkv + hk) * nb;

    if (tid == 0) {
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
    }
    {
        const int j = j0 + tid;
        const float a = j < nb ? vb[j] : 1.f;
        sm.lv[tid] = metric == 0 ? logf(a) : a;
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_slot, kTileS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_slot;
    const uint32_t idesc = make_idesc(kTileS, kTileS, 2u /* TF32 */, false, false);

    bool ok = true;
    constexpr int NCH = D / kChunk;
#pragma unroll 1
    for (int ch = 0; ch < NCH; ++ch) {
        if (ch > 0) {
            // The previous chunk's MMAs have read the shared-memory operands.
            ok = mbar_wait(&sm.mma_done, (ch - 1) & 1, &sm.abort_flag, err);
            if (__syncthreads_or(!ok)) break;
            tc_fence_after();
        }
        stage_chunk(A, i0, nb, D, ch * kChunk, sm.a_hi, sm.a_lo);
        stage_chunk(Bm, j0, nb, D, ch * kChunk, sm.b_hi, sm.b_lo);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ah = smem_u32(sm.a_hi), al = smem_u32(sm.a_lo);
            const uint32_t bh = smem_u32(sm.b_hi), bl = smem_u32(sm.b_lo);
#pragma unroll
            for (int kk = 0; kk < kChunk / 8; ++kk) {  // 8 tf32 = 32 bytes of K per MMA
                const uint32_t o = kk * 32;
                const uint32_t first = (ch == 0 && kk == 0) ? 0u : 1u;
                mma_tf32_ss(tmem, smem_desc_sw128(ah + o, 16, 1024), smem_desc_sw128(bh + o, 16, 1024), idesc, first);
                mma_tf32_ss(tmem, smem_desc_sw128(ah + o, 16, 1024), smem_desc_sw128(bl + o, 16, 1024), idesc, 1u);
                mma_tf32_ss(tmem, smem_desc_sw128(al + o, 16, 1024), smem_desc_sw128(bh + o, 16, 1024), idesc, 1u);
            }
            tc_commit(&sm.mma_done);
        }
        __syncwarp();
    }
    if (ok) {
        ok = mbar_wait(&sm.mma_done, (NCH - 1) & 1, &sm.abort_flag, err);
        ok = !__syncthreads_or(!ok);
    }
    if (ok) {
        tc_fence_after();
        // Epilogue: thread t owns accumulator row t (TMEM lane t).
        const int i = i0 + tid;
        const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        float* out = S + (static_cast<int64_t>(b) * Hq + h) * nbs * nbs + static_cast<int64_t>(i) * nbs;
#pragma unroll
        for (int c0 = 0; c0 < kTileS; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(trow + c0, r);
            if (i < nb) {
#pragma unroll
                for (int q = 0; q < 32; q += 4) {
                    float v4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int jj = c0 + q + e, j = j0 + jj;
                        float sc = tau * __uint_as_float(r[q + e]);
                        if (metric == 0)
                            sc += sm.lv[jj];
                        else if (metric == 2)
                            sc *= sm.lv[jj];
                        v4[e] = j > i ? -INFINITY : sc;
                    }
                    const int j = j0 + c0 + q;
                    // A 16-byte store only where the row stride leaves out + j 16-byte aligned.
                    if (j + 3 < nb && (reinterpret_cast<uintptr_t>(out + j) & 15u) == 0) {
                        *reinterpret_cast<float4*>(out + j) = make_float4(v4[0], v4[1], v4[2], v4[3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (j + e < nb) out[j + e] = v4[e];
                    }
                }
            }
        }
    } else if (tid == 0) {
        // Drain the MMAs in flight before the shared memory and TMEM go away.
        volatile int no_abort = 0;
        tc_commit(&sm.mma_done);
        mbar_wait(&sm.mma_done, NCH & 1, &no_abort, err);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTileS);
}

}  // namespace

cudaError_t launch_score_tc(const float* qbar, const float* kbar, const float* vbar, int B, int Hq, int Hkv, int nb,
                            int d, float tau, int metric, float* scores, int nb_stride, unsigned* err,
                            cudaStream_t s) {
    const int nt = (nb + kTileS - 1) / kTileS;
    dim3 grid(nt * (nt + 1) / 2, Hq, B);
    const int smem = static_cast<int>(sizeof(ScoreSmem)) + 1024;
    if (d == 128) {
        cudaError_t e = cudaFuncSetAttribute(score_tf32x3_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        score_tf32x3_kernel<128><<<grid, 128, smem, s>>>(qbar, kbar, vbar, Hq, Hkv, nb, tau, metric, scores, nb_stride, err);
    } else if (d == 64) {
        cudaError_t e = cudaFuncSetAttribute(score_tf32x3_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        score_tf32x3_kernel<64><<<grid, 128, smem, s>>>(qbar, kbar, vbar, Hq, Hkv, nb, tau, metric, scores, nb_stride, err);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace bsa
