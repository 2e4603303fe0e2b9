// attn_pipe.cu -- a5: block-sparse causal prefill attention, one query tile per CTA with the
// MMAs and copies pipelined under the softmax.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; a skipped block is a block of -inf
//  scores, so the softmax needs no change.]
//
// One CTA (128 threads, one query row each, up to 255 registers, two CTAs per SM) computes one
// 128-row query tile.  Thread 0 also issues the copies and MMAs, so every role shares one
// warpgroup and the whole 128-column S row fits in registers:
//   ring      K_j and V_j of the kept blocks stream through NS shared-memory stages (TMA,
//             128-byte swizzle); ring index 2n holds K of list entry n, 2n + 1 its V.  A stage
//             is refilled as soon as the MMA that read it is known to be complete.
//   S(n+1)    = Q K^T is issued as soon as every thread has copied S(n) out of TMEM, so it runs
//             under the softmax of block n.
//   softmax   tcgen05.ld of the row (one read), max over 8 chains, a running max that is only
//             refreshed when it grows by more than 2^T, P = exp2(S * scale - m) (a share of
//             them through an FMA-pipe polynomial), row sum over 4 packed chains.
//   P(n)      -> shared memory once PV(n-1) has read P(n-1); O is rescaled in TMEM when the
//             running max moved.
//   PV(n)     O += P V is issued by thread 0 once all rows wrote P, and runs under the next
//             block's softmax.
// TMEM (256 columns): S | O.  Every wait is bounded (sm100.cuh); on a timeout the CTA stops
// issuing, drains its copies and MMAs with bounded waits, frees TMEM and exits.
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBMp = 128;
constexpr int kThreadsP = 128;
constexpr int kSmemTwoPerSm = 115712;  // per-CTA limit for two CTAs per SM
constexpr int kSmemOnePerSm = 232448;  // per-CTA limit for one CTA per SM
constexpr int kMaxStagesP = 8;

template <bool FP8, int D, int BN>
struct CfgP {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;
    static constexpr int QP = D * EB / 128;
    static constexpr int Q_BYTES = kBMp * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int P_BYTES = kBMp * BN * EB;
    static constexpr int FIXED = Q_BYTES + P_BYTES + 256 + 1024;  // + barriers, alignment slack
    static constexpr int NS_TWO = (kSmemTwoPerSm - FIXED) / KV_BYTES;
    // Two CTAs per SM when four stages fit (K(n+1) must be in flight a block ahead), else one.
    static constexpr bool TWO_PER_SM = NS_TWO >= 4;
    static constexpr int NS_FIT = TWO_PER_SM ? NS_TWO : (kSmemOnePerSm - FIXED) / KV_BYTES;
    static constexpr int NS = NS_FIT > kMaxStagesP ? kMaxStagesP : NS_FIT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = Q_BYTES;
    static constexpr int OFF_RING = OFF_P + P_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    static constexpr int SMEM_RAW = OFF_BAR + 256 + 1024;
    // At least 78 KB, so that no more than two CTAs (2 x 256 TMEM columns) share an SM.
    static constexpr int SMEM = SMEM_RAW > 78 * 1024 ? SMEM_RAW : 78 * 1024;
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static constexpr int UNITS = BN * EB / 16;  // 16-byte P units per row
    static_assert(NS >= 4, "the ring needs four stages");
    static_assert(SMEM <= kSmemOnePerSm, "shared memory budget");
};

// BF16: refresh the running max only when it grows by more than 2^8 (P <= 256 unscaled);
// E4M3: beyond 2^5 with P scaled by 2^3, so P <= 2^8 fits E4M3 and values down to 2^-12 of the
// row max keep E4M3 precision.
template <bool FP8>
constexpr float kRescaleP = FP8 ? 5.f : 8.f;
template <bool FP8>
constexpr float kPScaleP = FP8 ? 3.f : 0.f;
// Exponentials through the FMA-pipe polynomial: kPolyP of every 8 pairs, degree kPolyDegP.
// Off: measured on B200 it slowed this kernel (the ALU work it adds outweighs the MUFU relief),
// and it maps a masked -inf score to 2^-126 rather than 0.
template <bool FP8>
constexpr int kPolyP = 0;
template <bool FP8>
constexpr int kPolyDegP = FP8 ? 2 : 3;

struct BarsP {
    uint64_t kv_full[kMaxStagesP];
    uint64_t q_full, s_full, s_free, p_full, o_done, drain;
    uint32_t tmem_slot;
    int abort_flag;
};
static_assert(sizeof(BarsP) <= 256, "barrier region");

template <bool FP8, int D, int BN, bool PAGED>
__global__ void __launch_bounds__(kThreadsP, 1)
    attn_pipe_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
    using C = CfgP<FP8, D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BarsP* bars = reinterpret_cast<BarsP*>(smem + C::OFF_BAR);
    volatile int* abort_flag = &bars->abort_flag;
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
    const int32_t* rp = a.row_ptr + static_cast<int64_t>(b) * a.row_ptr_stride + static_cast<int64_t>(h) * a.row_ptr_hstride;
    const int l_begin = rp[i];
    const int n_list = rp[i + 1] - l_begin;
    if (n_list == 0 && a.allow_empty) return;
    if (n_list < 1 || n_list > kMaxBlocks || l_begin < 0 || l_begin + static_cast<int64_t>(n_list) > a.max_k) {
        if (tid == 0) atomicOr(a.err, kDevErrInvalidList);
        return;
    }
    const int32_t* gl = a.col_idx + (static_cast<int64_t>(b) * a.Hq + h) * a.max_k + l_begin;
    const int tok0 = PAGED ? a.cu_seqlens[b] : 0;  // packed row of token 0 of this sequence

    if (tid == 0) {
        for (int t = 0; t < C::NS; ++t) mbar_init(&bars->kv_full[t], 1);
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, kThreadsP);
        mbar_init(&bars->p_full, kThreadsP);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&bars->tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base;
    const uint32_t tO = tmem + lane_base + 128;
    uint8_t* sP = smem + C::OFF_P;

    // ---- thread 0's issue state
    uint32_t r_issued = 0;  // ring indices issued so far (loads)
    const uint32_t r_total = 2u * n_list;
    unsigned bad = 0;  // kDevErr* bits found by thread 0's loads
    // Issues the loads of ring indices [r_issued, r_end).
    auto issue_loads = [&](uint32_t r_end) {
        if (r_end > r_total) r_end = r_total;
        for (; r_issued < r_end; ++r_issued) {
            const int n = static_cast<int>(r_issued >> 1);
            int j = __ldg(gl + n);
            if (j < 0 || j > i) {  // out of the causal range: flagged; the softmax zeroes it
                bad |= kDevErrInvalidList;
                j = 0;
            }
            const int st = r_issued % C::NS;
            uint8_t* dst = smem + C::OFF_RING + st * C::KV_BYTES;
            const CUtensorMap* map = (r_issued & 1) ? &tv : &tk;
            uint64_t* fb = &bars->kv_full[st];
            mbar_arrive_expect_tx(fb, C::KV_BYTES);
#pragma unroll
            for (int p = 0; p < C::QP; ++p) {
                if constexpr (PAGED) {
#pragma unroll
                    for (int pg = 0; pg < BN / 64; ++pg) {
                        const int lp = j * (BN / 64) + pg;
                        const int phys = physical_page(a, b, lp, n_tok, bad);
                        tma_load_4d(dst + p * BN * 128 + pg * 64 * 128, map, fb, p * C::PW, 0, hk, phys);
                    }
                } else {
                    tma_load_4d(dst + p * BN * 128, map, fb, p * C::PW, j * bs, hk, b);
                }
            }
        }
    };
    const uint32_t idesc_s = make_idesc(kBMp, BN, FP8 ? 0u : 1u, false, false);
    const uint32_t idesc_o = make_idesc(kBMp, D, FP8 ? 0u : 1u, false, true);
    const uint32_t aQ = smem_u32(smem + C::OFF_Q), aP = smem_u32(sP);
    // S = Q K^T from ring index r.
    auto mma_s = [&](uint32_t r) -> bool {
        const int st = r % C::NS;
        if (!mbar_wait(&bars->kv_full[st], (r / C::NS) & 1, abort_flag, a.err)) return false;
        tc_fence_after();
        const uint32_t aK = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS_S; ++kk) {
            const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
            const uint64_t da = smem_desc_sw128(aQ + pan * kBMp * 128 + within, 16, 1024);
            const uint64_t db = smem_desc_sw128(aK + pan * BN * 128 + within, 16, 1024);
            if constexpr (FP8)
                mma_f8_ss(tmem, da, db, idesc_s, kk > 0);
            else
                mma_f16_ss(tmem, da, db, idesc_s, kk > 0);
        }
        tc_commit(&bars->s_full);
        return true;
    };
    // O (+)= P V with V from ring index r.
    auto mma_pv = [&](uint32_t r, bool accumulate) -> bool {
        const int st = r % C::NS;
        if (!mbar_wait(&bars->kv_full[st], (r / C::NS) & 1, abort_flag, a.err)) return false;
        tc_fence_after();
        const uint32_t aV = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
            const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
            const uint64_t da = smem_desc_sw128(aP + pan * kBMp * 128 + within, 16, 1024);
            const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
            const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
            if constexpr (FP8)
                mma_f8_ss(tmem + 128, da, db, idesc_o, acc);
            else
                mma_f16_ss(tmem + 128, da, db, idesc_o, acc);
        }
        tc_commit(&bars->o_done);
        return true;
    };

    bool ok = true;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
#pragma unroll
        for (int p = 0; p < C::QP; ++p)
            tma_load_4d(smem + C::OFF_Q + p * kBMp * 128, &tq, &bars->q_full, p * C::PW, tok0 + i * bs, h,
                        PAGED ? 0 : b);
        issue_loads(C::NS);
        ok = mbar_wait(&bars->q_full, 0, abort_flag, a.err) && mma_s(0);
    }

    const int row = tid;
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY, l_run = 0.f;
    int j_next = __ldg(gl);
    for (int n = 0; n < n_list; ++n) {
        int j = j_next;
        if (n + 1 < n_list) j_next = __ldg(gl + n + 1);
        if (j > i) j = -1;  // out of range: a skipped block
        // ---- S(n) -> registers
        bool w_ok = mbar_wait(&bars->s_full, n & 1, abort_flag, a.err);
        w_ok = __all_sync(0xFFFFFFFFu, w_ok);
        if (!w_ok) {
            ok = false;
            break;
        }
        tc_fence_after();
        uint32_t rr[BN];
        if constexpr (BN == 128)
            tmem_ld128(tS, rr);
        else
            tmem_ld64(tS, rr);
        tc_fence_before();
        mbar_arrive(&bars->s_free);
        // ---- thread 0: S(n+1) as soon as every row has read S(n)
        if (tid == 0 && ok && n + 1 < n_list) {
            ok = mbar_wait(&bars->s_free, n & 1, abort_flag, a.err) && mma_s(2u * (n + 1));
        }
        __syncwarp();
        // ---- softmax of row `row` over this block.  Masked scores become -inf here, outside the
        // exponential loop: the causal part of the diagonal block, and all of a skipped block.
        if (j == i) {
#pragma unroll
            for (int e = 0; e < BN; ++e)
                if (e > row) rr[e] = __float_as_uint(-INFINITY);
        } else if (j < 0) {
#pragma unroll
            for (int e = 0; e < BN; ++e) rr[e] = __float_as_uint(-INFINITY);
        }
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
        for (int e = 0; e < BN; e += 2)
            m8[(e / 2) % 8] = max3f(m8[(e / 2) % 8], __uint_as_float(rr[e]), __uint_as_float(rr[e + 1]));
        const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        const float m_blk = mx * sl2;
        float m_new = m_used;
        if (m_blk > m_used + kRescaleP<FP8>) m_new = m_blk;
        const float alpha = (m_new == m_used) ? 1.f : fast_exp2(m_used - m_new);
        const float mref = (m_new == -INFINITY) ? 0.f : m_new - kPScaleP<FP8>;
        const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
        const uint64_t negm = pack_f32x2(-mref, -mref);
        uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
            const uint64_t xx = fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])), sl2x2, negm);
            float x0, x1, p0, p1;
            unpack_f32x2(xx, x0, x1);
            if ((e / 2) % 8 < kPolyP<FP8>) {
                exp2_poly_x2<kPolyDegP<FP8>>(x0, x1, p0, p1);
            } else {
                p0 = fast_exp2(x0);
                p1 = fast_exp2(x1);
            }
            sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(p0, p1));
            rr[e] = __float_as_uint(p0);
            rr[e + 1] = __float_as_uint(p1);
        }
        // ---- PV(n-1) must be complete: it reads P (rewritten below) and writes O (rescaled below)
        if (n > 0) {
            w_ok = mbar_wait(&bars->o_done, (n - 1) & 1, abort_flag, a.err);
            w_ok = __all_sync(0xFFFFFFFFu, w_ok);
            if (!w_ok) {
                ok = false;
                break;
            }
            tc_fence_after();
        }
        // Every MMA issued before PV(n-1) is complete, so ring indices <= 2n are free.
        if (tid == 0 && ok) issue_loads(2u * n + 1 + C::NS);
        __syncwarp();
        // ---- P -> shared memory (128-byte-swizzled K-major A operand of the PV MMA)
#pragma unroll
        for (int u = 0; u < C::UNITS; ++u) {
            uint32_t w4[4];
            if constexpr (FP8) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = u * 16 + q * 4;
                    w4[q] = pack_e4m3x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])) |
                            (static_cast<uint32_t>(pack_e4m3x2(__uint_as_float(rr[e + 2]), __uint_as_float(rr[e + 3])))
                             << 16);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    w4[q] = pack_bf16x2(__uint_as_float(rr[u * 8 + 2 * q]), __uint_as_float(rr[u * 8 + 2 * q + 1]));
            }
            const int pan = u / 8, cc = u % 8;
            *reinterpret_cast<uint4*>(sP + pan * kBMp * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        // ---- O rescale when some row of the warp moved its max
        if (n > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t ro[32];
                tmem_ld32(tO + ch * 32, ro);
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const uint64_t v = mul_f32x2(pack_f32x2(__uint_as_float(ro[e]), __uint_as_float(ro[e + 1])),
                                                 pack_f32x2(alpha, alpha));
                    float v0, v1;
                    unpack_f32x2(v, v0, v1);
                    ro[e] = __float_as_uint(v0);
                    ro[e + 1] = __float_as_uint(v1);
                }
                tmem_st32(tO + ch * 32, ro);
            }
            tmem_st_wait();
        }
        float s0, s1, s2, s3, s4, s5, s6, s7;
        unpack_f32x2(sum4[0], s0, s1);
        unpack_f32x2(sum4[1], s2, s3);
        unpack_f32x2(sum4[2], s4, s5);
        unpack_f32x2(sum4[3], s6, s7);
        l_run = l_run * alpha + (((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)));
        m_used = m_new;
        tc_fence_before();
        mbar_arrive(&bars->p_full);
        // ---- thread 0: PV(n) once every row wrote P(n)
        if (tid == 0 && ok) {
            ok = mbar_wait(&bars->p_full, n & 1, abort_flag, a.err) && mma_pv(2u * n + 1, n > 0);
        }
        __syncwarp();
    }

    bool fail = !ok;
    if (!fail) {
        bool w_ok = mbar_wait(&bars->o_done, (n_list - 1) & 1, abort_flag, a.err);
        fail = !__all_sync(0xFFFFFFFFu, w_ok);
    }
    fail = __syncthreads_or(fail || *abort_flag != 0);
    if (!fail) {
        tc_fence_after();
        const int t_row = i * bs + row;
        const bool store = row < bs && t_row < n_tok;
        const float inv = (l_run > 0.f ? 1.f / l_run : 0.f) * a.out_scale;
        const int64_t orow = PAGED ? static_cast<int64_t>(tok0 + t_row) * a.ost
                                   : static_cast<int64_t>(b) * a.osb + static_cast<int64_t>(t_row) * a.ost;
        uint8_t* dst = reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.out) + orow +
                                                  static_cast<int64_t>(h) * a.osh);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ro[32];
            tmem_ld32(tO + ch * 32, ro);
            if (store) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w4[e] = pack_bf16x2(__uint_as_float(ro[q * 8 + 2 * e]) * inv,
                                            __uint_as_float(ro[q * 8 + 2 * e + 1]) * inv);
                    *reinterpret_cast<uint4*>(dst + (ch * 32 + q * 8) * 2) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        }
        if (store && a.lse != nullptr)
            a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.lse_stride + t_row] =
                (m_used + __log2f(l_run) - kPScaleP<FP8>) * 0.69314718055994531f;
    } else if (tid == 0) {
        // Drain every copy and MMA still in flight before the shared memory and TMEM go away.
        volatile int no_abort = 0;
        for (uint32_t r = r_issued > C::NS ? r_issued - C::NS : 0; r < r_issued; ++r)
            mbar_wait(&bars->kv_full[r % C::NS], (r / C::NS) & 1, &no_abort, a.err);
        mbar_wait(&bars->q_full, 0, &no_abort, a.err);
        tc_commit(&bars->drain);
        mbar_wait(&bars->drain, 0, &no_abort, a.err);
    }
    if (tid == 0 && bad) atomicOr(a.err, bad);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

template <bool FP8, int D, int BN, bool PAGED>
cudaError_t launch_pipe_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                          cudaStream_t s) {
    using C = CfgP<FP8, D, BN>;
    auto kern = attn_pipe_kernel<FP8, D, BN, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hkv * a.nb_max * (a.Hq / a.Hkv), a.B);
    kern<<<grid, kThreadsP, C::SMEM, s>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_pipe(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (fp8) {
        if (a.d != 128 || a.block != 128) return cudaErrorInvalidValue;
        return paged ? launch_pipe_t<true, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_pipe_t<true, 128, 128, false>(tq, tk, tv, a, s);
    }
    if (a.d == 128 && a.block == 128)
        return paged ? launch_pipe_t<false, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_pipe_t<false, 128, 128, false>(tq, tk, tv, a, s);
    if (a.d == 128 && a.block == 64)
        return paged ? launch_pipe_t<false, 128, 64, true>(tq, tk, tv, a, s)
                     : launch_pipe_t<false, 128, 64, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 128)
        return paged ? launch_pipe_t<false, 64, 128, true>(tq, tk, tv, a, s)
                     : launch_pipe_t<false, 64, 128, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 64)
        return paged ? launch_pipe_t<false, 64, 64, true>(tq, tk, tv, a, s)
                     : launch_pipe_t<false, 64, 64, false>(tq, tk, tv, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
