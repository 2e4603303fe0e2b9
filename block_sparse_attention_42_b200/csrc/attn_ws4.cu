// attn_ws4.cu -- a5: block-sparse causal prefill, two pipelined CTAs per SM, with the softmax
// of every query tile split by key columns over two warpgroups.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; skipped blocks are -inf.]
//
// The softmax of a 128 x 128 score tile is bound by the exponentials (16 per clock per SM on
// the MUFU unit) and, between them, by latency: TMEM loads, barrier waits and O rescales.  Four
// softmax warps per SM sub-partition hide that latency where two cannot, so each CTA (10 warps,
// persistent, two per SM) gives a query tile two softmax warpgroups:
//   warps 0-3   softmax, key columns [0, BN/2) of S, one query row per thread (TMEM lane
//               quadrant = warp % 4)
//   warps 4-7   softmax, key columns [BN/2, BN) of the same rows
//   warp 8      TMA producer: Q, then K_j and V_j of every kept block into a ring of stages
//   warp 9      MMA issuer (TMEM owner): S(k+1) = Q K^T as soon as both halves have read S(k)
//               out of TMEM, and O += P(k) V once both halves have written P(k)
// The two threads that own a row trade their partial row maxima through shared memory (a
// bounded mbarrier wait per block) and so take the same running max, rescale decision and
// exponent reference; each keeps its own partial row sum, rescales its own half of O's columns
// and stores its half of the output.  A share of the exponentials (NPOLY of every 8 pairs) is
// evaluated by a polynomial on the FMA pipe so the MUFU and FMA pipes share the load.
// TMEM (256 columns per CTA): S | O.  P goes to shared memory (128-byte swizzled K-major A
// operand of the PV MMA); P(k) is written after PV(k-1) has read P(k-1).
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBM4 = 128;
constexpr int kThreads4 = 320;
constexpr int kSmem4Limit = 115712;  // two CTAs per SM
constexpr int kMaxStages4 = 6;
constexpr int kListChunk4 = 128;

template <bool FP8, int D, int BN>
struct Cfg4 {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;
    static constexpr int QP = D * EB / 128;
    static constexpr int Q_BYTES = kBM4 * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int P_BYTES = kBM4 * BN * EB;
    static constexpr int BAR_BYTES = 4096;
    static constexpr int NS_FIT = (kSmem4Limit - BAR_BYTES - 1024 - Q_BYTES - P_BYTES) / KV_BYTES;
    static constexpr int NS = NS_FIT > kMaxStages4 ? kMaxStages4 : NS_FIT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = Q_BYTES;
    static constexpr int OFF_RING = OFF_P + P_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static constexpr int C = BN / 2;                // key columns per softmax half
    static constexpr int DH = D / 2;                // O columns per softmax half
    static constexpr int UNITS = C * EB / 16;       // 16-byte P units per half row
    static_assert(NS >= 3, "the ring needs three stages: K(k+1) is consumed before V(k)");
    static_assert(SMEM <= kSmem4Limit, "shared memory budget");
    static_assert(C == 32 || C == 64, "half-row width");
};

// BF16: refresh the running max only when it grows by more than 2^8 (P <= 256 unscaled);
// E4M3: beyond 2^5 with P scaled by 2^3, so P <= 2^8 fits E4M3 and values down to 2^-12 of the
// row max keep E4M3 precision.
template <bool FP8>
constexpr float kRescale4 = FP8 ? 5.f : 8.f;
template <bool FP8>
constexpr float kPScale4 = FP8 ? 3.f : 0.f;
// Exponentials through the FMA-pipe polynomial: NPOLY of every 8 pairs, of degree DEG (the
// degree-2 fit, relative error 1.7e-3, is far below E4M3's 2^-4 spacing; BF16 takes degree 3).
template <bool FP8>
constexpr int kPoly4 = 0;  // off: a masked -inf score must give exactly 0
template <bool FP8>
constexpr int kPolyDeg4 = FP8 ? 2 : 3;

struct Bars4 {
    uint64_t kv_full[kMaxStages4], kv_empty[kMaxStages4];
    uint64_t q_full, q_empty, s_full, s_free, p_full, o_done, drain, tmem_free;
    uint64_t xchg[2][4];  // partial-row exchange, by exchange parity and lane quadrant
    uint32_t tmem_slot;
    int abort_flag;
    float xval[2][2][kBM4];  // [parity][half][row]
    int lst[kListChunk4];
};
static_assert(sizeof(Bars4) <= 4096, "barrier region");

// Trades one value per row with the thread of the other half that owns the same row.  Slot
// n & 1 is rewritten two exchanges later, after the partner has arrived at the exchange in
// between, i.e. after it read the slot.
__device__ __forceinline__ bool exchange_row(Bars4* bars, uint32_t& xc, int half, int quad, int row, float mine,
                                             float& theirs, volatile int* abort_flag, unsigned* err) {
    const int p = xc & 1;
    bars->xval[p][half][row] = mine;
    mbar_arrive(&bars->xchg[p][quad]);
    const bool ok = mbar_wait(&bars->xchg[p][quad], (xc >> 1) & 1, abort_flag, err);
    theirs = bars->xval[p][half ^ 1][row];
    ++xc;
    return ok;
}

template <bool FP8, int D, int BN, bool PAGED>
__global__ void __launch_bounds__(kThreads4, 2)
    attn_ws4_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const AttnArgs a, int total_tiles) {
    using C = Cfg4<FP8, D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars4* bars = reinterpret_cast<Bars4*>(smem + C::OFF_BAR);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int t = 0; t < C::NS; ++t) {
            mbar_init(&bars->kv_full[t], 1);
            mbar_init(&bars->kv_empty[t], 1);
        }
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 256);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->tmem_free, 256);
        for (int p = 0; p < 2; ++p)
            for (int q = 0; q < 4; ++q) mbar_init(&bars->xchg[p][q], 64);
        bars->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncwarp();
    if (warp == 9) {
        tmem_alloc(&bars->tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        TileIter it;
        it.init(0, blockIdx.x, gridDim.x, total_tiles);
        it.next(a);
        uint32_t ring = 0, qc = 0;
        unsigned bad = 0;
        bool ok = true;
        while (ok && it.active) {
            const Tile T = it.T;
            if (lane == 0) {
                ok = mbar_wait(&bars->q_empty, (qc & 1) ^ 1, abort_flag, a.err);
                if (ok) {
                    uint8_t* dst = smem + C::OFF_Q;
                    mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
                    const int tok0 = PAGED ? a.cu_seqlens[T.b] : 0;
#pragma unroll
                    for (int p = 0; p < C::QP; ++p)
                        tma_load_4d(dst + p * kBM4 * 128, &tq, &bars->q_full, p * C::PW, tok0 + T.i * a.block, T.h,
                                    PAGED ? 0 : T.b);
                    ++qc;
                }
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            for (int kb = 0; ok && kb < T.n_list; kb += kListChunk4) {
                __syncwarp();
                for (int e = lane; e < kListChunk4; e += 32)
                    if (kb + e < T.n_list) bars->lst[e] = list_entry(a, T, kb + e);
                __syncwarp();
                if (lane == 0) {
                    const int kend = min(T.n_list, kb + kListChunk4);
                    for (int k = kb; ok && k < kend; ++k) {
                        int j = bars->lst[k - kb];
                        if (j < 0) {
                            bad |= kDevErrInvalidList;
                            j = 0;
                        }
                        for (int v = 0; ok && v < 2; ++v) {
                            const int st = ring % C::NS;
                            ok = mbar_wait(&bars->kv_empty[st], ((ring / C::NS) & 1) ^ 1, abort_flag, a.err);
                            if (!ok) break;
                            uint8_t* dst = smem + C::OFF_RING + st * C::KV_BYTES;
                            const CUtensorMap* map = v ? &tv : &tk;
                            uint64_t* fb = &bars->kv_full[st];
                            mbar_arrive_expect_tx(fb, C::KV_BYTES);
#pragma unroll
                            for (int p = 0; p < C::QP; ++p) {
                                if constexpr (PAGED) {
#pragma unroll
                                    for (int pg = 0; pg < BN / 64; ++pg) {
                                        const int lp = j * (BN / 64) + pg;
                                        const int phys = physical_page(a, T.b, lp, T.n_tok, bad);
                                        tma_load_4d(dst + p * BN * 128 + pg * 64 * 128, map, fb, p * C::PW, 0, T.hk, phys);
                                    }
                                } else {
                                    tma_load_4d(dst + p * BN * 128, map, fb, p * C::PW, j * a.block, T.hk, T.b);
                                }
                            }
                            ++ring;
                        }
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            }
            it.next(a);
        }
        if (lane == 0) {
            if (bad) atomicOr(a.err, bad);
            // Every issued copy must land before the CTA's shared memory goes away.
            volatile int no_abort = 0;
            for (uint32_t r = ring > C::NS ? ring - C::NS : 0; r < ring; ++r)
                mbar_wait(&bars->kv_full[r % C::NS], (r / C::NS) & 1, &no_abort, a.err);
            if (qc > 0) mbar_wait(&bars->q_full, (qc - 1) & 1, &no_abort, a.err);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = make_idesc(kBM4, BN, FP8 ? 0u : 1u, false, false);
            const uint32_t idesc_o = make_idesc(kBM4, D, FP8 ? 0u : 1u, false, true);
            const uint32_t aQ = smem_u32(smem + C::OFF_Q);
            const uint32_t aP = smem_u32(smem + C::OFF_P);
            uint32_t rbase = 0, qc = 0, pc = 0, sf = 0;
            bool ok = true, first_s = true;
            TileIter it;
            it.init(0, blockIdx.x, gridDim.x, total_tiles);
            it.next(a);
            // S = Q K^T from ring index r (K of a block sits at 2k, its V at 2k + 1).
            auto mma_s = [&](uint32_t r) -> bool {
                // S is overwritten: both halves must have read the previous S.
                if (!first_s) {
                    if (!mbar_wait(&bars->s_free, sf & 1, abort_flag, a.err)) return false;
                    ++sf;
                }
                first_s = false;
                const int st = r % C::NS;
                if (!mbar_wait(&bars->kv_full[st], (r / C::NS) & 1, abort_flag, a.err)) return false;
                tc_fence_after();
                const uint32_t aK = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS_S; ++kk) {
                    const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                    const uint64_t da = smem_desc_sw128(aQ + pan * kBM4 * 128 + within, 16, 1024);
                    const uint64_t db = smem_desc_sw128(aK + pan * BN * 128 + within, 16, 1024);
                    if constexpr (FP8)
                        mma_f8_ss(tmem, da, db, idesc_s, kk > 0);
                    else
                        mma_f16_ss(tmem, da, db, idesc_s, kk > 0);
                }
                tc_commit(&bars->kv_empty[st]);
                tc_commit(&bars->s_full);
                return true;
            };
            // O (+)= P V with V from ring index r and P from shared memory.
            auto mma_pv = [&](uint32_t r, bool accumulate) -> bool {
                if (!mbar_wait(&bars->p_full, pc & 1, abort_flag, a.err)) return false;
                ++pc;
                const int st = r % C::NS;
                if (!mbar_wait(&bars->kv_full[st], (r / C::NS) & 1, abort_flag, a.err)) return false;
                tc_fence_after();
                const uint32_t aV = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
                    const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                    const uint64_t da = smem_desc_sw128(aP + pan * kBM4 * 128 + within, 16, 1024);
                    const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                    const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
                    if constexpr (FP8)
                        mma_f8_ss(tmem + 128, da, db, idesc_o, acc);
                    else
                        mma_f16_ss(tmem + 128, da, db, idesc_o, acc);
                }
                tc_commit(&bars->kv_empty[st]);
                tc_commit(&bars->o_done);
                return true;
            };
            while (ok && it.active) {
                const int n = it.T.n_list;
                ok = mbar_wait(&bars->q_full, qc & 1, abort_flag, a.err);
                ++qc;
                ok = ok && mma_s(rbase);
                if (ok && n == 1) tc_commit(&bars->q_empty);
                for (int k = 0; ok && k < n; ++k) {
                    // S(k+1) goes ahead of PV(k): it only needs both halves to have read S(k).
                    if (k + 1 < n) {
                        ok = mma_s(rbase + 2 * (k + 1));
                        if (ok && k + 2 == n) tc_commit(&bars->q_empty);  // last S of the tile
                    }
                    ok = ok && mma_pv(rbase + 2 * k + 1, k > 0);
                }
                rbase += 2 * n;
                it.next(a);
            }
            tc_commit(&bars->drain);
            volatile int no_abort = 0;
            mbar_wait(&bars->drain, 0, &no_abort, a.err);
            mbar_wait(&bars->tmem_free, 0, &no_abort, a.err);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
        return;
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int half = warp / 4;
        const int quad = warp % 4;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tmem + lane_base + half * C::C;
        const uint32_t tO = tmem + lane_base + 128 + half * C::DH;
        uint8_t* sP = smem + C::OFF_P;
        const int col0 = half * C::C;  // first key column of this half
        uint32_t scount = 0, ocount = 0, xc = 0;
        const float sl2 = a.scale_log2;
        bool ok = true;
        TileIter it;
        it.init(0, blockIdx.x, gridDim.x, total_tiles);
        it.next(a);
        while (ok && it.active) {
            const Tile T = it.T;
            float m_used = -INFINITY, l_run = 0.f;
            int j_next = list_entry(a, T, 0);
            for (int k = 0; k < T.n_list; ++k) {
                const int j = j_next;
                if (k + 1 < T.n_list) j_next = list_entry(a, T, k + 1);
                bool w_ok = mbar_wait(&bars->s_full, scount & 1, abort_flag, a.err);
                ++scount;
                w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                if (!w_ok) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const bool diag = (j == T.i);
                // This half of the S row in registers with one TMEM read; then S may be overwritten.
                uint32_t rr[C::C];
                if constexpr (C::C == 64)
                    tmem_ld64(tS, rr);
                else
                    tmem_ld32(tS, rr);
                tc_fence_before();
                mbar_arrive(&bars->s_free);
                // Masked scores become -inf here, outside the exponential loop: the causal part of
                // the diagonal block, and all of a skipped block.
                if (diag) {
#pragma unroll
                    for (int e = 0; e < C::C; ++e)
                        if (col0 + e > row) rr[e] = __float_as_uint(-INFINITY);
                } else if (j < 0) {
#pragma unroll
                    for (int e = 0; e < C::C; ++e) rr[e] = __float_as_uint(-INFINITY);
                }
                float mx;
                {
                    float m8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
                    for (int e = 0; e < C::C; e += 2)
                        m8[(e / 2) % 8] = max3f(m8[(e / 2) % 8], __uint_as_float(rr[e]), __uint_as_float(rr[e + 1]));
                    mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                }
                float mx_other;
                w_ok = exchange_row(bars, xc, half, quad, row, mx, mx_other, abort_flag, a.err);
                w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                if (!w_ok) {
                    ok = false;
                    break;
                }
                mx = fmaxf(mx, mx_other);
                const float m_blk = mx * sl2;
                float m_new = m_used;
                if (m_blk > m_used + kRescale4<FP8>) m_new = m_blk;
                const float alpha = (m_new == m_used) ? 1.f : fast_exp2(m_used - m_new);
                const float mref = (m_new == -INFINITY) ? 0.f : m_new - kPScale4<FP8>;
                // P = exp2(S * sl2 - mref) in place, four packed partial sums.
                const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
                const uint64_t negm = pack_f32x2(-mref, -mref);
                uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int e = 0; e < C::C; e += 2) {
                    const uint64_t x = fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])),
                                                 sl2x2, negm);
                    float x0, x1, p0, p1;
                    unpack_f32x2(x, x0, x1);
                    if ((e / 2) % 8 < kPoly4<FP8>) {
                        exp2_poly_x2<kPolyDeg4<FP8>>(x0, x1, p0, p1);
                    } else {
                        p0 = fast_exp2(x0);
                        p1 = fast_exp2(x1);
                    }
                    sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(p0, p1));
                    rr[e] = __float_as_uint(p0);
                    rr[e + 1] = __float_as_uint(p1);
                }
                if (k > 0) {
                    // PV(k-1) reads P (rewritten below) and writes O (maybe rescaled below).
                    w_ok = mbar_wait(&bars->o_done, ocount & 1, abort_flag, a.err);
                    ++ocount;
                    w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                    if (!w_ok) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                // This half of the P row -> shared memory (128-byte-swizzled K-major PV A operand).
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
                    const int ug = half * C::UNITS + u;  // 16-byte unit within the full P row
                    const int pan = ug / 8, cc = ug % 8;
                    *reinterpret_cast<uint4*>(sP + pan * kBM4 * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                fence_proxy_async_smem();
                if (k > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
                    for (int ch = 0; ch < C::DH / 32; ++ch) {
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
                }
                float s0, s1, s2, s3, s4, s5, s6, s7;
                unpack_f32x2(sum4[0], s0, s1);
                unpack_f32x2(sum4[1], s2, s3);
                unpack_f32x2(sum4[2], s4, s5);
                unpack_f32x2(sum4[3], s6, s7);
                const float sum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
                l_run = l_run * alpha + sum;
                m_used = m_new;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->p_full);
            }
            if (!ok) break;
            bool w_ok = mbar_wait(&bars->o_done, ocount & 1, abort_flag, a.err);
            ++ocount;
            float l_other = 0.f;
            w_ok = w_ok && exchange_row(bars, xc, half, quad, row, l_run, l_other, abort_flag, a.err);
            w_ok = __all_sync(0xFFFFFFFFu, w_ok);
            if (!w_ok) break;
            tc_fence_after();
            const float l_tot = l_run + l_other;
            const int t_row = T.i * a.block + row;
            const bool store = row < a.block && t_row < T.n_tok;
            const float inv = (l_tot > 0.f ? 1.f / l_tot : 0.f) * a.out_scale;
            const int64_t orow = PAGED ? static_cast<int64_t>(a.cu_seqlens[T.b] + t_row) * a.ost
                                       : static_cast<int64_t>(T.b) * a.osb + static_cast<int64_t>(t_row) * a.ost;
            uint8_t* dst = reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.out) + orow +
                                                      static_cast<int64_t>(T.h) * a.osh + half * C::DH);
#pragma unroll
            for (int ch = 0; ch < C::DH / 32; ++ch) {
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
            if (half == 0 && store && a.lse != nullptr)
                a.lse[(static_cast<int64_t>(T.b) * a.Hq + T.h) * a.lse_stride + t_row] =
                    (m_used + __log2f(l_tot) - kPScale4<FP8>) * 0.69314718055994531f;
            tc_fence_before();
            it.next(a);
        }
        tc_fence_before();
        mbar_arrive(&bars->tmem_free);
        return;
    }
}

template <bool FP8, int D, int BN, bool PAGED>
cudaError_t launch_ws4_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                         cudaStream_t s) {
    using C = Cfg4<FP8, D, BN>;
    auto kern = attn_ws4_kernel<FP8, D, BN, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long total = static_cast<long long>(a.B) * a.Hkv * a.nb_max * (a.Hq / a.Hkv);
    long long grid = 2LL * sms;
    if (grid > total) grid = total;
    kern<<<static_cast<unsigned>(grid), kThreads4, C::SMEM, s>>>(tq, tk, tv, a, static_cast<int>(total));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_ws4(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (fp8) {
        if (a.d != 128 || a.block != 128) return cudaErrorInvalidValue;
        return paged ? launch_ws4_t<true, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_ws4_t<true, 128, 128, false>(tq, tk, tv, a, s);
    }
    if (a.d == 128 && a.block == 128)  // the BF16 stages do not fit two CTAs per SM
        return launch_attention(fp8, paged, tq, tk, tv, a, s);
    if (a.d == 128 && a.block == 64)
        return paged ? launch_ws4_t<false, 128, 64, true>(tq, tk, tv, a, s)
                     : launch_ws4_t<false, 128, 64, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 128)
        return paged ? launch_ws4_t<false, 64, 128, true>(tq, tk, tv, a, s)
                     : launch_ws4_t<false, 64, 128, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 64)
        return paged ? launch_ws4_t<false, 64, 64, true>(tq, tk, tv, a, s)
                     : launch_ws4_t<false, 64, 64, false>(tq, tk, tv, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
