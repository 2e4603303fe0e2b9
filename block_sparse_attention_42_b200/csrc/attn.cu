// attn.cu -- a5: block-sparse causal prefill attention on tcgen05 tensor cores.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: the list of KV blocks
//  to visit is built before the inner loop, the loop visits only those blocks and its body is
//  the dense attention body; a skipped block is mathematically a block of -inf scores, so the
//  softmax needs no change.  Paged KV is loaded page by page; FP8 doubles MMA throughput.]
//
// One CTA computes one 128-row query tile (query block i of head h; for 64-token blocks the
// upper 64 rows are padding).  Per kept KV block j, in list order:
//   TMA    K_j, V_j -> shared memory (128-byte swizzle; paged: one box per 64-token page)
//   MMA    S = Q K_j^T          (tcgen05, A and B from shared memory, FP32 in TMEM cols 0..)
//   all    128 threads, one query row each: tcgen05.ld S, scale, causal mask on the diagonal
//          block only, online max / sum, P = exp2(S - m) -> BF16 (or E4M3 x 256) in shared
//          memory; O in TMEM is rescaled when the row max moved
//   MMA    O += P V_j           (V as an MN-major B operand, FP32 in TMEM cols 128..)
// then O / l -> BF16 global, and the natural-log LSE.
//
// Every mbarrier wait is bounded (sm100.cuh); on a timeout the CTA stops issuing work,
// drains its in-flight copies and MMAs with a bounded wait, frees its TMEM and exits.
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBM = 128;
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 128;

template <bool FP8, int D, int BN>
struct Cfg {
    static constexpr int EB = FP8 ? 1 : 2;          // bytes per element
    static constexpr int PW = 128 / EB;             // elements per 128-byte panel row
    static constexpr int QP = D * EB / 128;         // panels across head_dim
    static constexpr int Q_BYTES = kBM * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int P_BYTES = kBM * BN * EB;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KV_BYTES;
    static constexpr int OFF_P = OFF_V + KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;  // 4 mbarriers + tmem slot + abort flag
    static constexpr int OFF_LIST = OFF_BAR + 64;
    // + alignment slack; at least 78 KB so no more than two CTAs (2 x 256 TMEM columns) share an SM
    static constexpr int SMEM_RAW = OFF_LIST + kMaxBlocks * 4 + 1024;
    static constexpr int SMEM = SMEM_RAW > 78 * 1024 ? SMEM_RAW : 78 * 1024;
    static constexpr int KSTEPS_S = D * EB / 32;    // MMA K-steps (32 bytes of K each)
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;  // V rows consumed per PV K-step
    static_assert(QP >= 1 && BN * EB % 128 == 0, "unsupported tile");
};

template <bool FP8, int D, int BN, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
    using C = Cfg<FP8, D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;
    uint8_t* sP = smem + C::OFF_P;
    uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_kv = bar_q + 1;
    uint64_t* bar_s = bar_q + 2;
    uint64_t* bar_o = bar_q + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 32);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 40);
    int32_t* list = reinterpret_cast<int32_t*>(smem + C::OFF_LIST);

    const int tid = threadIdx.x, warp = tid / 32;
    const int G = a.Hq / a.Hkv;

    // Work tile: KV-head-major, then query blocks from the last (longest list) down, then the
    // G query heads of the group, so concurrently running CTAs share K/V in L2.
    int x = blockIdx.x;
    const int g = x % G;
    x /= G;
    const int i = a.nb_max - 1 - (x % a.nb_max);
    const int hk = x / a.nb_max;
    const int h = hk * G + g;
    const int b = blockIdx.y;
    const int n_tok = a.seqlen[b];
    const int bs = a.block;
    const int nb = (n_tok + bs - 1) / bs;
    if (i >= nb) return;
    // A row with no kept block (allowed only where its output is written elsewhere): leave
    // before any barrier or TMEM allocation.
    if (a.allow_empty) {
        const int32_t* rp0 =
            a.row_ptr + static_cast<int64_t>(b) * a.row_ptr_stride + static_cast<int64_t>(h) * a.row_ptr_hstride;
        if (rp0[i + 1] == rp0[i]) return;
    }
    const int tok0 = PAGED ? a.cu_seqlens[b] : 0;  // packed row of token 0 of this sequence

    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_kv, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // The list of this (b, h, i): validated once, before the loop.
    const int32_t* rp = a.row_ptr + static_cast<int64_t>(b) * a.row_ptr_stride + static_cast<int64_t>(h) * a.row_ptr_hstride;
    const int l_begin = rp[i];
    const int n_list = rp[i + 1] - l_begin;
    const int64_t lrow = a.list_per_group ? static_cast<int64_t>(b) * a.Hkv + h / (a.Hq / a.Hkv)
                                          : static_cast<int64_t>(b) * a.Hq + h;
    const int32_t* gl = a.col_idx + lrow * a.max_k + l_begin;
    bool bad = n_list < 1 || n_list > kMaxBlocks || l_begin < 0 || l_begin + static_cast<int64_t>(n_list) > a.max_k;
    const int n_use = bad ? 0 : n_list;
    for (int n = tid; n < n_use; n += kThreads) {
        const int j = gl[n];
        const bool ok = j >= 0 && j <= i;
        list[n] = ok ? j : -1;
        bad |= !ok;
    }
    if (bad) atomicOr(a.err, kDevErrInvalidList);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base;
    const uint32_t tO = tmem + lane_base + kTmemO;

    const uint32_t idesc_s = make_idesc(kBM, BN, FP8 ? 0u : 1u, false, false);
    const uint32_t idesc_o = make_idesc(kBM, D, FP8 ? 0u : 1u, false, true);
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);

    bool kv_inflight = false, mma_inflight = false;
    unsigned page_bad = 0;  // kDevErrInvalidPage if thread 0 met a page-table entry out of range
    uint32_t mma_parity = 0;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
        for (int p = 0; p < C::QP; ++p)
            tma_load_4d(sQ + p * kBM * 128, &tq, bar_q, p * C::PW, tok0 + i * bs, h, PAGED ? 0 : b);
    }

    const int row = tid;                          // query row within the tile
    const int t_row = i * bs + row;               // token index within the sequence
    float m_run = -INFINITY, l_run = 0.f;
    int c = 0;                                    // blocks processed
    bool q_ready = false;
    for (int n = 0; n < n_use; ++n) {
        const int j = list[n];
        if (j < 0) continue;
        // ---- issue: K/V loads, then S = Q K^T
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_kv, 2 * C::KV_BYTES);
            kv_inflight = true;
#pragma unroll
            for (int p = 0; p < C::QP; ++p) {
                if constexpr (PAGED) {
#pragma unroll
                    for (int pg = 0; pg < BN / 64; ++pg) {
                        const int lp = j * (BN / 64) + pg;
                        const int phys = physical_page(a, b, lp, n_tok, page_bad);
                        tma_load_4d(sK + p * BN * 128 + pg * 64 * 128, &tk, bar_kv, p * C::PW, 0, hk, phys);
                        tma_load_4d(sV + p * BN * 128 + pg * 64 * 128, &tv, bar_kv, p * C::PW, 0, hk, phys);
                    }
                } else {
                    tma_load_4d(sK + p * BN * 128, &tk, bar_kv, p * C::PW, j * bs, hk, b);
                    tma_load_4d(sV + p * BN * 128, &tv, bar_kv, p * C::PW, j * bs, hk, b);
                }
            }
            bool ok = true;
            if (!q_ready) ok = mbar_wait(bar_q, 0, abort_flag, a.err);
            q_ready = true;
            ok = ok && mbar_wait(bar_kv, c & 1, abort_flag, a.err);
            if (ok) {
                kv_inflight = false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS_S; ++kk) {
                    const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                    const uint64_t da = smem_desc_sw128(aQ + pan * kBM * 128 + within, 16, 1024);
                    const uint64_t db = smem_desc_sw128(aK + pan * BN * 128 + within, 16, 1024);
                    if constexpr (FP8)
                        mma_f8_ss(tmem, da, db, idesc_s, kk > 0);
                    else
                        mma_f16_ss(tmem, da, db, idesc_s, kk > 0);
                }
                tc_commit(bar_s);
                mma_inflight = true;
            }
        }
        __syncwarp();
        // ---- softmax on S (every thread owns one row)
        bool s_ok = mbar_wait(bar_s, c & 1, abort_flag, a.err);
        if (tid == 0 && s_ok) mma_inflight = false;
        s_ok = __all_sync(0xFFFFFFFFu, s_ok);  // the TMEM loads below are warp-collective
        if (s_ok) {
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) {
                uint32_t r[32];
                tmem_ld32(tS + ch * 32, r);
#pragma unroll
                for (int e = 0; e < 32; ++e) s[ch * 32 + e] = __uint_as_float(r[e]) * a.scale_log2;
            }
            if (j == i) {
#pragma unroll
                for (int e = 0; e < BN; ++e)
                    if (e > row) s[e] = -INFINITY;
            }
            float mx = m_run;
#pragma unroll
            for (int e = 0; e < BN; ++e) mx = fmaxf(mx, s[e]);
            const float alpha = fast_exp2(m_run - mx);
            float sum = 0.f;
#pragma unroll
            for (int e = 0; e < BN; ++e) {
                s[e] = fast_exp2(s[e] - mx);
                sum += s[e];
            }
            l_run = l_run * alpha + sum;
            m_run = mx;
            // Rescale the running output when any row of the warp moved its max.
            if (c > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t r[32];
                    tmem_ld32(tO + ch * 32, r);
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    tmem_st32(tO + ch * 32, r);
                }
                tmem_st_wait();
            }
            // P -> shared memory in the 128-byte-swizzled K-major layout of the A operand.
            if constexpr (FP8) {
#pragma unroll
                for (int ch = 0; ch < BN / 16; ++ch) {
                    uint32_t w[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int e = ch * 16 + q * 4;
                        const uint32_t lo = pack_e4m3x2(s[e] * 256.f, s[e + 1] * 256.f);
                        const uint32_t hi = pack_e4m3x2(s[e + 2] * 256.f, s[e + 3] * 256.f);
                        w[q] = lo | (hi << 16);
                    }
                    const int pan = ch / 8, cc = ch % 8;
                    uint8_t* dst = sP + pan * kBM * 128 + row * 128 + ((cc ^ (row & 7)) * 16);
                    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
#pragma unroll
                for (int ch = 0; ch < BN / 8; ++ch) {
                    uint32_t w[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) w[q] = pack_bf16x2(s[ch * 8 + 2 * q], s[ch * 8 + 2 * q + 1]);
                    const int pan = ch / 8, cc = ch % 8;
                    uint8_t* dst = sP + pan * kBM * 128 + row * 128 + ((cc ^ (row & 7)) * 16);
                    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
        }
        tc_fence_before();
        if (__syncthreads_or(*abort_flag != 0)) break;
        // ---- O += P V
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
                const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                const uint64_t da = smem_desc_sw128(aP + pan * kBM * 128 + within, 16, 1024);
                const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                if constexpr (FP8)
                    mma_f8_ss(tmem + kTmemO, da, db, idesc_o, (c > 0 || kk > 0) ? 1u : 0u);
                else
                    mma_f16_ss(tmem + kTmemO, da, db, idesc_o, (c > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(bar_o);
            mma_inflight = true;
        }
        __syncwarp();
        const bool o_ok = mbar_wait(bar_o, c & 1, abort_flag, a.err);
        if (tid == 0 && o_ok) mma_inflight = false;
        mma_parity = (c + 1) & 1;
        ++c;
        if (__syncthreads_or(*abort_flag != 0)) break;
        tc_fence_after();
    }

    const bool aborted = *abort_flag != 0;
    if (!aborted && c > 0) {
        tc_fence_after();
        const float inv = (l_run > 0.f ? 1.f / l_run : 0.f) * a.out_scale * (FP8 ? (1.f / 256.f) : 1.f);
        const bool store = row < bs && t_row < n_tok;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
        const int64_t orow = PAGED ? static_cast<int64_t>(tok0 + t_row) * a.ost
                                   : static_cast<int64_t>(b) * a.osb + static_cast<int64_t>(t_row) * a.ost;
        uint8_t* dst = reinterpret_cast<uint8_t*>(out + orow + static_cast<int64_t>(h) * a.osh);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t r[32];
            tmem_ld32(tO + ch * 32, r);
            if (store) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(r[q * 8 + 2 * e]) * inv,
                                           __uint_as_float(r[q * 8 + 2 * e + 1]) * inv);
                    *reinterpret_cast<uint4*>(dst + (ch * 32 + q * 8) * 2) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        if (store && a.lse != nullptr)
            a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.lse_stride + t_row] =
                (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
    if (aborted && tid == 0) {
        // Drain whatever this CTA still has in flight before its shared memory and TMEM go away.
        volatile int no_abort = 0;
        if (kv_inflight) mbar_wait(bar_kv, c & 1, &no_abort, a.err);
        if (mma_inflight) {
            tc_commit(bar_o);
            mbar_wait(bar_o, mma_parity, &no_abort, a.err);
        }
    }
    if (page_bad) atomicOr(a.err, page_bad);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

template <bool FP8, int D, int BN, bool PAGED>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                     cudaStream_t s) {
    using C = Cfg<FP8, D, BN>;
    auto kern = attn_fwd_kernel<FP8, D, BN, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hkv * a.nb_max * (a.Hq / a.Hkv), a.B);
    kern<<<grid, kThreads, C::SMEM, s>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (fp8) {
        if (a.d != 128 || a.block != 128) return cudaErrorInvalidValue;
        return paged ? launch_t<true, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_t<true, 128, 128, false>(tq, tk, tv, a, s);
    }
    if (a.d == 128 && a.block == 128)
        return paged ? launch_t<false, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_t<false, 128, 128, false>(tq, tk, tv, a, s);
    if (a.d == 128 && a.block == 64)
        return paged ? launch_t<false, 128, 64, true>(tq, tk, tv, a, s)
                     : launch_t<false, 128, 64, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 128)
        return paged ? launch_t<false, 64, 128, true>(tq, tk, tv, a, s)
                     : launch_t<false, 64, 128, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 64)
        return paged ? launch_t<false, 64, 64, true>(tq, tk, tv, a, s)
                     : launch_t<false, 64, 64, false>(tq, tk, tv, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
