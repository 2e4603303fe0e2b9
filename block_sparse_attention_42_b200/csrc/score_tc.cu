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
// alone would move scores by ~1e-3 and reorder near-equal candidates.  The pooling kernel
// stores each pooled fp32 value x split as hi = x with its 13 low mantissa bits cleared (exact
// in TF32) and lo = x - hi (exact in fp32), and the tensor cores accumulate hi*hi + hi*lo +
// lo*hi in fp32 (kind::tf32).  The dropped lo*lo term and the TF32 truncation of lo are ~2^-20
// of the product.
//
// A persistent GEMM over the causal 128 x 128 tiles (query blocks x key blocks) of every
// query head, one CTA per SM (6 warps):
//   warp 0      TMA producer: per 32-value chunk of head_dim, the hi / lo rows of the tile's
//               Qbar and Kbar (4 x 16 KB, 128-byte swizzle, rows past nb read as zeros) into a
//               ring of 3 stages
//   warp 1      MMA issuer (TMEM owner): 3 x 4 MMAs per chunk into one of two TMEM
//               accumulators (128 columns each), so the next tile runs while the last drains
//   warps 2-9   epilogue, two warps per TMEM lane quarter, each with half of the columns:
//               ln vbar of the tile's 128 key blocks once into shared memory (one per thread
//               of the first half), then per 32 columns tcgen05.ld of the thread's row,
//               tau * acc (+ ln vbar), -inf above the diagonal, and a transpose through a
//               per-warp shared buffer so that each store instruction writes whole 128-byte
//               score-row segments
// Every wait is bounded (sm100.cuh).
#include <cmath>

#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kTileS = 128;
constexpr int kChunk = 32;              // fp32 values of head_dim per chunk (one 128-byte row)
constexpr int kOpBytes = kTileS * 128;  // one operand chunk (16 KB)
constexpr int kStageBytes = 4 * kOpBytes;
constexpr int kStagesS = 3;
constexpr int kThreadsS = 320;

struct ScoreBars {
    uint64_t full[kStagesS], empty[kStagesS];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain, tmem_free;
    uint32_t tmem_slot;
    int abort_flag;
};
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
static_assert(kThreadsS == 64 + kEpiThreads, "producer + MMA warps + epilogue");
constexpr int kTrBytes = kEpiWarps * 32 * 32 * 4;  // epilogue transpose buffers, 32 x 32 fp32 per warp
constexpr int kLvBytes = 2 * kTileS * 4;    // per-column terms of the last two tiles
constexpr int kScoreSmem = kStagesS * kStageBytes + kTrBytes + kLvBytes + 256 + 1024;  // + barriers, slack
static_assert(kScoreSmem <= 227 * 1024, "shared memory per CTA");

// Barrier 1 over the epilogue warps, returning whether `p` held in every thread.
__device__ __forceinline__ bool epilogue_all(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, 256, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(p))
        : "memory");
    return r != 0;
}

struct TileRC {
    int b, h, hk, i0, j0;
};

// Tile t -> (sequence, head, first query block, first key block); per head the causal tile
// pairs (ti, tj), tj <= ti, in row-major order.
__device__ __forceinline__ TileRC decode_score_tile(int t, int nt, int Hq, int G) {
    const int per = nt * (nt + 1) / 2;
    const int bh = t / per;
    const int x = t % per;
    int ti = static_cast<int>((sqrtf(8.f * x + 1.f) - 1.f) * 0.5f);
    while ((ti + 1) * (ti + 2) / 2 <= x) ++ti;
    while (ti * (ti + 1) / 2 > x) --ti;
    const int tj = x - ti * (ti + 1) / 2;
    TileRC r;
    r.h = bh % Hq;
    r.b = bh / Hq;
    r.hk = r.h / G;
    r.i0 = ti * kTileS;
    r.j0 = tj * kTileS;
    return r;
}

template <int D>
__global__ void __launch_bounds__(kThreadsS, 1)
    score_tf32x3_kernel(const __grid_constant__ CUtensorMap mqh, const __grid_constant__ CUtensorMap mql,
                        const __grid_constant__ CUtensorMap mkh, const __grid_constant__ CUtensorMap mkl,
                        const float* __restrict__ vbar, int Hq, int Hkv, int nb, float tau, int metric,
                        float* __restrict__ S, int nbs, int total_tiles, unsigned* err) {
    constexpr int NCH = D / kChunk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* tr_all = reinterpret_cast<float*>(smem + kStagesS * kStageBytes);
    float* lv_all = reinterpret_cast<float*>(smem + kStagesS * kStageBytes + kTrBytes);
    ScoreBars* bars = reinterpret_cast<ScoreBars*>(smem + kStagesS * kStageBytes + kTrBytes + kLvBytes);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nt = (nb + kTileS - 1) / kTileS;
    const int G = Hq / Hkv;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesS; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->acc_full[a], 1);
            mbar_init(&bars->acc_empty[a], kEpiThreads);
        }
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->tmem_free, kEpiThreads);
        bars->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&mqh);
        tma_prefetch_desc(&mql);
        tma_prefetch_desc(&mkh);
        tma_prefetch_desc(&mkl);
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc(&bars->tmem_slot, 2 * kTileS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t ring = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
                const TileRC r = decode_score_tile(t, nt, Hq, G);
                for (int c = 0; ok && c < NCH; ++c) {
                    const int st = ring % kStagesS;
                    ok = mbar_wait(&bars->empty[st], ((ring / kStagesS) & 1) ^ 1, abort_flag, err);
                    if (!ok) break;
                    uint8_t* dst = smem + st * kStageBytes;
                    uint64_t* fb = &bars->full[st];
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    tma_load_4d(dst, &mqh, fb, c * kChunk, r.i0, r.h, r.b);
                    tma_load_4d(dst + kOpBytes, &mql, fb, c * kChunk, r.i0, r.h, r.b);
                    tma_load_4d(dst + 2 * kOpBytes, &mkh, fb, c * kChunk, r.j0, r.hk, r.b);
                    tma_load_4d(dst + 3 * kOpBytes, &mkl, fb, c * kChunk, r.j0, r.hk, r.b);
                    ++ring;
                }
            }
            // Every issued copy must land before the shared memory goes away.
            volatile int no_abort = 0;
            for (uint32_t q = ring > kStagesS ? ring - kStagesS : 0; q < ring; ++q)
                mbar_wait(&bars->full[q % kStagesS], (q / kStagesS) & 1, &no_abort, err);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc(kTileS, kTileS, 2u /* TF32 */, false, false);
            uint32_t ring = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x, ++tc) {
                const uint32_t ab = tc & 1;
                if (tc >= 2) {
                    // The epilogue has drained this accumulator's previous tile.
                    ok = mbar_wait(&bars->acc_empty[ab], ((tc / 2) - 1) & 1, abort_flag, err);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t acc = tmem + ab * kTileS;
                for (int c = 0; ok && c < NCH; ++c) {
                    const int st = ring % kStagesS;
                    ok = mbar_wait(&bars->full[st], (ring / kStagesS) & 1, abort_flag, err);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t ah = smem_u32(smem + st * kStageBytes);
                    const uint32_t al = ah + kOpBytes, bh = ah + 2 * kOpBytes, bl = ah + 3 * kOpBytes;
#pragma unroll
                    for (int kk = 0; kk < kChunk / 8; ++kk) {  // 8 tf32 = 32 bytes of K per MMA
                        const uint32_t o = kk * 32;
                        const uint32_t first = (c == 0 && kk == 0) ? 0u : 1u;
                        mma_tf32_ss(acc, smem_desc_sw128(ah + o, 16, 1024), smem_desc_sw128(bh + o, 16, 1024), idesc,
                                    first);
                        mma_tf32_ss(acc, smem_desc_sw128(ah + o, 16, 1024), smem_desc_sw128(bl + o, 16, 1024), idesc, 1u);
                        mma_tf32_ss(acc, smem_desc_sw128(al + o, 16, 1024), smem_desc_sw128(bh + o, 16, 1024), idesc, 1u);
                    }
                    tc_commit(&bars->empty[st]);
                    ++ring;
                }
                if (ok) tc_commit(&bars->acc_full[ab]);
            }
            tc_commit(&bars->drain);
            volatile int no_abort = 0;
            mbar_wait(&bars->drain, 0, &no_abort, err);
            mbar_wait(&bars->tmem_free, 0, &no_abort, err);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kTileS);
        return;
    } else {
        // ------------------------------------------------------------ epilogue (warps 2-9)
        const int ew = warp - 2;
        const int quad = warp % 4;          // TMEM lanes 32 * quad .. 32 * quad + 31
        const int half = ew / 4;            // columns 64 * half .. 64 * half + 63
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        float* tr = tr_all + ew * 32 * 32;
        // 16-byte stores need every score row segment 16-byte aligned.
        const bool vec_ok = (nbs % 4) == 0 && (reinterpret_cast<uintptr_t>(S) & 15u) == 0;
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tc) {
            const uint32_t ab = tc & 1;
            const TileRC r = decode_score_tile(t, nt, Hq, G);
            // This tile's per-column term: ln vbar (OAM), vbar (OAM_MUL); one column per thread
            // of the first half.  lv_all holds two tiles' terms, so the write below cannot race
            // the reads of the previous tile: every epilogue thread has passed that tile's
            // barrier, which comes after its reads of the tile before.
            float* lv = lv_all + ab * kTileS;
            if (half == 0) {
                const int j = r.j0 + row;
                float a = 0.f;
                if (metric != 1 && j < nb) {
                    a = __ldg(vbar + (static_cast<int64_t>(r.b) * Hkv + r.hk) * nb + j);
                    if (metric == 0) a = logf(a);
                }
                lv[row] = a;
            }
            // One barrier per tile for all epilogue threads, also on the way out: a thread whose
            // wait gave up makes every epilogue thread leave at the same tile.
            const bool ok = mbar_wait(&bars->acc_full[ab], (tc / 2) & 1, abort_flag, err);
            if (!epilogue_all(ok)) break;
            tc_fence_after();
            const bool diag = r.i0 == r.j0;  // the only tiles with entries above the diagonal
            float* out_head = S + (static_cast<int64_t>(r.b) * Hq + r.h) * nbs * nbs;
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                const int c0 = half * 64 + g * 32;
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + ab * kTileS + c0, v);
                if (g == 1) {
                    // The accumulator is in registers: the MMA warp may reuse it.
                    tc_fence_before();
                    mbar_arrive(&bars->acc_empty[ab]);
                }
                // Row `lane` of this warp's 32 x 32 buffer, 16-byte chunks rotated by the row
                // (chunk q at q ^ (row & 7)) so that both the row writes here and the column
                // reads below are free of bank conflicts.
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 l4 = *reinterpret_cast<const float4*>(lv + c0 + q * 4);
                    const float la[4] = {l4.x, l4.y, l4.z, l4.w};
                    float o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float acc = __uint_as_float(v[q * 4 + e]);
                        float sc;
                        if (metric == 0)
                            sc = fmaf(tau, acc, la[e]);
                        else if (metric == 2)
                            sc = tau * acc * la[e];
                        else
                            sc = tau * acc;
                        if (diag && c0 + q * 4 + e > row) sc = -INFINITY;
                        o[e] = sc;
                    }
                    *reinterpret_cast<float4*>(tr + lane * 32 + ((q ^ (lane & 7)) * 4)) =
                        make_float4(o[0], o[1], o[2], o[3]);
                }
                __syncwarp();
                // 8 lanes per score row, 4 rows per instruction.
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int rr = p * 4 + lane / 8, cq = lane % 8;
                    const float4 o = *reinterpret_cast<const float4*>(tr + rr * 32 + ((cq ^ (rr & 7)) * 4));
                    const int gi = r.i0 + quad * 32 + rr, gj = r.j0 + c0 + cq * 4;
                    if (gi < nb) {
                        float* dst = out_head + static_cast<int64_t>(gi) * nbs + gj;
                        if (vec_ok && gj + 3 < nb) {
                            *reinterpret_cast<float4*>(dst) = o;
                        } else {
                            const float oe[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (gj + e < nb) dst[e] = oe[e];
                        }
                    }
                }
                __syncwarp();
            }
        }
        tc_fence_before();
        mbar_arrive(&bars->tmem_free);
        return;
    }
}

}  // namespace

cudaError_t launch_score_tc(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                            const CUtensorMap& mkl, const float* vbar, int B, int Hq, int Hkv, int nb, int d,
                            float tau, int metric, float* scores, int nb_stride, unsigned* err, cudaStream_t s) {
    const int nt = (nb + kTileS - 1) / kTileS;
    const long long total = static_cast<long long>(nt) * (nt + 1) / 2 * Hq * B;
    if (total > 0x7FFFFFFFll) return cudaErrorInvalidValue;  // tile indices are int
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
    if (d == 128) {
        cudaError_t e = cudaFuncSetAttribute(score_tf32x3_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kScoreSmem);
        if (e != cudaSuccess) return e;
        score_tf32x3_kernel<128><<<grid, kThreadsS, kScoreSmem, s>>>(mqh, mql, mkh, mkl, vbar, Hq, Hkv, nb, tau, metric,
                                                                      scores, nb_stride, static_cast<int>(total), err);
    } else if (d == 64) {
        cudaError_t e = cudaFuncSetAttribute(score_tf32x3_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kScoreSmem);
        if (e != cudaSuccess) return e;
        score_tf32x3_kernel<64><<<grid, kThreadsS, kScoreSmem, s>>>(mqh, mql, mkh, mkl, vbar, Hq, Hkv, nb, tau, metric,
                                                                     scores, nb_stride, static_cast<int>(total), err);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace bsa
