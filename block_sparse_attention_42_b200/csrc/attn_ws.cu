// attn_ws.cu -- a5: warp-specialised, persistent block-sparse causal prefill on tcgen05.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; skipped blocks are -inf.]
//
// One CTA per SM, 12 warps, two query tiles ("slots" s = 0, 1) in flight:
//   warp 0      TMA producer: per slot, its Q tile and a private ring of K/V stages
//   warp 1      MMA issuer (and TMEM owner): S_s = Q_s K^T, then O_s += P_s V with P_s read
//               from tensor memory (it overwrites S_s in place)
//   warps 4-7   softmax of slot 0, warps 8-11 softmax of slot 1: one query row per thread;
//               tcgen05.ld S, online max/sum, P -> TMEM (BF16 or E4M3), O rescale in TMEM when
//               the row max grew enough, and the tile epilogue (O / l -> BF16, LSE)
// The producer and the MMA warp poll both slots and serve whichever is ready, so the two
// slots run independently and one slot's softmax overlaps the other slot's MMAs.
// TMEM (512 columns): S_0/P_0 | S_1/P_1 | O_0 | O_1, 128 columns each.
// Each slot walks its own static sequence of work tiles (tile = query block i of head h), in
// KV-head-major order with the longest lists first.
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBM = 128;
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kSmemLimit = 232448;  // 227 KB of dynamic shared memory per CTA
constexpr int kMaxStages = 6;       // K/V stages per slot
constexpr int kListChunk = 128;     // list entries the producer stages in shared memory per slot
// Polling loops give up after this many SM cycles without progress (about 2 s).
constexpr long long kPollLimitCycles = 4000000000ll;
// Register split.  The kernel is launched with 168 registers per thread (384 x 168 = 64512; the
// build refuses an attn_ws_kernel compiled at any other count).  Warpgroup 0 (producer, MMA,
// two idle warps) then gives registers back and the two softmax warpgroups take them:
// 128 x 56 + 256 x 224 = 64512, exactly the launch pool.
constexpr int kRegsLaunch = 168;
constexpr int kRegsLow = 56;
constexpr int kRegsHigh = 224;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split exceeds the launch pool");

template <bool FP8, int D, int BN>
struct WsCfg {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;
    static constexpr int QP = D * EB / 128;
    static constexpr int Q_BYTES = kBM * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int NSS_FIT = (kSmemLimit - 5120 - 2 * Q_BYTES) / (2 * KV_BYTES);
    static constexpr int NSS = NSS_FIT > kMaxStages ? kMaxStages : NSS_FIT;  // stages per slot
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = 2 * Q_BYTES;
    static constexpr int OFF_BAR = OFF_RING + 2 * NSS * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + 2048 + 1024;  // barriers, list buffers + alignment slack
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static_assert(NSS >= 2, "each slot needs at least two K/V stages");
    static_assert(SMEM <= kSmemLimit, "shared memory budget");
};

// Online-softmax policy.  BF16: refresh the running max only when it grows by more than 2^8,
// P unscaled (P <= 256).  E4M3: refresh beyond 2^3 and scale P by 2^5, so P <= 2^8 stays
// inside E4M3's range while values down to 2^-14 of the row max keep their precision.
template <bool FP8>
constexpr float kRescaleLog2 = FP8 ? 3.f : 8.f;
template <bool FP8>
constexpr float kPScaleLog2 = FP8 ? 5.f : 0.f;

struct Bars {
    uint64_t kv_full[2][kMaxStages], kv_empty[2][kMaxStages];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t drain, tmem_free;
    uint32_t tmem_slot;
    int abort_flag;
    int lst[2][kListChunk];  // producer's staged list entries per slot
};
static_assert(sizeof(Bars) <= 2048, "barrier region");

template <bool FP8, int D, int BN, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    attn_ws_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnArgs a, int total_tiles) {
    using C = WsCfg<FP8, D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int stride = 2 * gridDim.x, base = 2 * blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            for (int t = 0; t < C::NSS; ++t) {
                mbar_init(&bars->kv_full[s][t], 1);
                mbar_init(&bars->kv_empty[s][t], 1);
            }
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], 128);
            mbar_init(&bars->o_done[s], 1);
        }
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->tmem_free, 256);
        bars->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc(&bars->tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;

    if (warp < 4) regs_dec<kRegsLow>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp walks the schedule (uniform control flow); lane 0 tests barriers and
        // issues the copies, and all lanes stage list entries into shared memory in bulk.
        TileIter rit[2], qit[2];     // K/V ring walk and Q walk of each slot
        int ld[2] = {0, 0};          // next load of the ring tile: K0 V0 K1 V1 ...
        int lbase[2] = {-1, -1};     // first list entry staged in bars->lst[s]
        uint32_t ring[2] = {0, 0}, qc[2] = {0, 0};
        unsigned bad = 0;
        bool ok = true;
        for (int s = 0; s < 2; ++s) {
            rit[s].init(s, base, stride, total_tiles);
            rit[s].next(a);
            qit[s] = rit[s];
        }
        int idle = 0;
        long long t_idle = 0;
        while (ok && (rit[0].active || rit[1].active || qit[0].active || qit[1].active)) {
            bool prog = false;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                if (qit[s].active) {
                    const bool qready = __shfl_sync(0xFFFFFFFFu, lane == 0 ? mbar_test(&bars->q_empty[s], (qc[s] & 1) ^ 1) : 0u, 0);
                    if (qready) {
                        if (lane == 0) {
                            const Tile& T = qit[s].T;
                            uint8_t* dst = smem + C::OFF_Q + s * C::Q_BYTES;
                            mbar_arrive_expect_tx(&bars->q_full[s], C::Q_BYTES);
                            const int tok0 = PAGED ? a.cu_seqlens[T.b] : 0;
#pragma unroll
                            for (int p = 0; p < C::QP; ++p)
                                tma_load_4d(dst + p * kBM * 128, &tq, &bars->q_full[s], p * C::PW, tok0 + T.i * a.block,
                                            T.h, PAGED ? 0 : T.b);
                        }
                        ++qc[s];
                        qit[s].next(a);
                        prog = true;
                    }
                }
                if (!rit[s].active) continue;
                const Tile& T = rit[s].T;
                const int kb = ld[s] >> 1;
                if (lbase[s] < 0 || kb >= lbase[s] + kListChunk) {
                    // Stage entries kb .. kb+127 of this tile's list.
                    __syncwarp();
                    for (int e = lane; e < kListChunk; e += 32)
                        if (kb + e < T.n_list) bars->lst[s][e] = list_entry(a, T, kb + e);
                    lbase[s] = kb;
                    __syncwarp();
                }
                const int st = ring[s] % C::NSS;
                const bool sready =
                    __shfl_sync(0xFFFFFFFFu, lane == 0 ? mbar_test(&bars->kv_empty[s][st], ((ring[s] / C::NSS) & 1) ^ 1) : 0u, 0);
                if (!sready) continue;
                if (lane == 0) {
                    const bool is_v = ld[s] & 1;
                    int j = bars->lst[s][kb - lbase[s]];
                    if (j < 0) {
                        bad = 1;
                        j = 0;
                    }
                    uint8_t* dst = smem + C::OFF_RING + (s * C::NSS + st) * C::KV_BYTES;
                    const CUtensorMap* map = is_v ? &tv : &tk;
                    uint64_t* fb = &bars->kv_full[s][st];
                    mbar_arrive_expect_tx(fb, C::KV_BYTES);
#pragma unroll
                    for (int p = 0; p < C::QP; ++p) {
                        if constexpr (PAGED) {
#pragma unroll
                            for (int pg = 0; pg < BN / 64; ++pg) {
                                const int lp = j * (BN / 64) + pg;
                                const int phys =
                                    lp * 64 < T.n_tok ? __ldg(a.page_table + static_cast<int64_t>(T.b) * a.max_pages + lp)
                                                      : a.num_pages;  // past the end of the sequence: zeros
                                tma_load_4d(dst + p * BN * 128 + pg * 64 * 128, map, fb, p * C::PW, 0, T.hk, phys);
                            }
                        } else {
                            tma_load_4d(dst + p * BN * 128, map, fb, p * C::PW, j * a.block, T.hk, T.b);
                        }
                    }
                }
                ++ring[s];
                if (++ld[s] == 2 * T.n_list) {
                    ld[s] = 0;
                    lbase[s] = -1;
                    rit[s].next(a);
                }
                prog = true;
            }
            if (prog) {
                idle = 0;
            } else {
                if (++idle == 1) t_idle = clock64();
                if ((idle & 255) == 0) {
                    if (*abort_flag) {
                        ok = false;
                    } else if (clock64() - t_idle > kPollLimitCycles) {
                        if (lane == 0) {
                            *abort_flag = 1;
                            atomicOr(a.err, kDevErrTimeout);
                        }
                        ok = false;
                    }
                    ok = __all_sync(0xFFFFFFFFu, ok);
                }
                __nanosleep(20);
            }
        }
        if (lane == 0) {
            if (bad) atomicOr(a.err, kDevErrInvalidList);
            // Every issued copy must land before the CTA's shared memory goes away.
            volatile int no_abort = 0;
            for (int s = 0; s < 2; ++s) {
                for (uint32_t r = ring[s] > C::NSS ? ring[s] - C::NSS : 0; r < ring[s]; ++r)
                    mbar_wait(&bars->kv_full[s][r % C::NSS], (r / C::NSS) & 1, &no_abort, a.err);
                if (qc[s] > 0) mbar_wait(&bars->q_full[s], (qc[s] - 1) & 1, &no_abort, a.err);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = make_idesc(kBM, BN, FP8 ? 0u : 1u, false, false);
            const uint32_t idesc_o = make_idesc(kBM, D, FP8 ? 0u : 1u, false, true);
            TileIter it[2];
            int kblk[2] = {0, 0};
            bool need_s[2] = {true, true}, q_seen[2] = {false, false}, p_seen[2] = {false, false};
            uint32_t rc[2] = {0, 0}, qc[2] = {0, 0}, pc[2] = {0, 0}, pv_issued[2] = {0, 0}, oc[2] = {0, 0};
            bool ok = true;
            for (int s = 0; s < 2; ++s) {
                it[s].init(s, base, stride, total_tiles);
                it[s].next(a);
            }
            int idle = 0;
            long long t_idle = 0;
            while (ok && (it[0].active || it[1].active)) {
                bool prog = false;
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    if (!it[s].active) continue;
                    const int st = rc[s] % C::NSS;
                    if (need_s[s]) {
                        // S(k) = Q K^T: its Q has landed, its K stage is full, and the previous
                        // PV (which reads P from these TMEM columns) is complete.
                        if (kblk[s] == 0 && !q_seen[s]) {
                            if (!mbar_test(&bars->q_full[s], qc[s] & 1)) continue;
                            q_seen[s] = true;
                            ++qc[s];
                        }
                        if (oc[s] < pv_issued[s]) {
                            if (!mbar_test(&bars->o_done[s], oc[s] & 1)) continue;
                            ++oc[s];
                        }
                        if (!mbar_test(&bars->kv_full[s][st], (rc[s] / C::NSS) & 1)) continue;
                        tc_fence_after();
                        const uint32_t aQ = smem_u32(smem + C::OFF_Q + s * C::Q_BYTES);
                        const uint32_t aK = smem_u32(smem + C::OFF_RING + (s * C::NSS + st) * C::KV_BYTES);
#pragma unroll
                        for (int kk = 0; kk < C::KSTEPS_S; ++kk) {
                            const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                            const uint64_t da = smem_desc_sw128(aQ + pan * kBM * 128 + within, 16, 1024);
                            const uint64_t db = smem_desc_sw128(aK + pan * BN * 128 + within, 16, 1024);
                            if constexpr (FP8)
                                mma_f8_ss(tmem + s * 128, da, db, idesc_s, kk > 0);
                            else
                                mma_f16_ss(tmem + s * 128, da, db, idesc_s, kk > 0);
                        }
                        tc_commit(&bars->kv_empty[s][st]);
                        tc_commit(&bars->s_full[s]);
                        if (kblk[s] == it[s].T.n_list - 1) {
                            tc_commit(&bars->q_empty[s]);  // last S of the tile: Q_s may be reloaded
                            q_seen[s] = false;
                        }
                        ++rc[s];
                        need_s[s] = false;
                        prog = true;
                    } else {
                        // O += P V: P written to TMEM by the softmax, V stage full.
                        if (!p_seen[s]) {
                            if (!mbar_test(&bars->p_full[s], pc[s] & 1)) continue;
                            p_seen[s] = true;
                            ++pc[s];
                        }
                        if (!mbar_test(&bars->kv_full[s][st], (rc[s] / C::NSS) & 1)) continue;
                        tc_fence_after();
                        const uint32_t aV = smem_u32(smem + C::OFF_RING + (s * C::NSS + st) * C::KV_BYTES);
#pragma unroll
                        for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
                            const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                            const uint32_t acc = (kblk[s] > 0 || kk > 0) ? 1u : 0u;
                            if constexpr (FP8)
                                mma_f8_ts(tmem + 256 + s * 128, tmem + s * 128 + kk * 8, db, idesc_o, acc);
                            else
                                mma_f16_ts(tmem + 256 + s * 128, tmem + s * 128 + kk * 8, db, idesc_o, acc);
                        }
                        tc_commit(&bars->kv_empty[s][st]);
                        tc_commit(&bars->o_done[s]);
                        ++pv_issued[s];
                        ++rc[s];
                        p_seen[s] = false;
                        need_s[s] = true;
                        if (++kblk[s] == it[s].T.n_list) {
                            kblk[s] = 0;
                            it[s].next(a);
                        }
                        prog = true;
                    }
                }
                if (prog) {
                    idle = 0;
                } else {
                    if (++idle == 1) t_idle = clock64();
                    if ((idle & 255) == 0) {
                        if (*abort_flag) {
                            ok = false;
                        } else if (clock64() - t_idle > kPollLimitCycles) {
                            *abort_flag = 1;
                            atomicOr(a.err, kDevErrTimeout);
                            ok = false;
                        }
                    }
                    __nanosleep(20);
                }
            }
            // Drain: wait until every MMA issued by this thread has completed.
            tc_commit(&bars->drain);
            volatile int no_abort = 0;
            mbar_wait(&bars->drain, 0, &no_abort, a.err);
            // Every softmax thread has finished with TMEM (bounded: the softmax warps exit
            // their loops on abort too).
            mbar_wait(&bars->tmem_free, 0, &no_abort, a.err);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
        return;
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax, slot s
        regs_inc<kRegsHigh>();
        const int s = (warp - 4) / 4;
        const int quad = warp % 4;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tmem + lane_base + s * 128;  // S, then P in place
        const uint32_t tO = tmem + lane_base + 256 + s * 128;
        uint32_t scount = 0, ocount = 0;
        const float sl2 = a.scale_log2;
        bool ok = true;
        TileIter it;
        it.init(s, base, stride, total_tiles);
        it.next(a);
        while (ok && it.active) {
            const Tile T = it.T;
            float m_used = -INFINITY, l_run = 0.f;
            int j_next = list_entry(a, T, 0);
            for (int k = 0; k < T.n_list; ++k) {
                const int j = j_next;
                if (k + 1 < T.n_list) j_next = list_entry(a, T, k + 1);  // prefetch the next entry
                bool w_ok = mbar_wait(&bars->s_full[s], scount & 1, abort_flag, a.err);
                ++scount;
                w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                if (!w_ok) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Only the diagonal block needs the causal mask (and an out-of-range entry, all -inf).
                const bool diag = (j == T.i);
                // The whole S row in registers: one TMEM round trip per block.
                uint32_t rr[BN];
                if constexpr (BN == 128)
                    tmem_ld128(tS, rr);
                else
                    tmem_ld64(tS, rr);
                // Row max with eight independent chains.
                float mx = -INFINITY;
                if (j >= 0) {
                    float m8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
                    if (!diag) {
#pragma unroll
                        for (int e = 0; e < BN; e += 2)
                            m8[(e / 2) % 8] = max3f(m8[(e / 2) % 8], __uint_as_float(rr[e]), __uint_as_float(rr[e + 1]));
                    } else {
#pragma unroll
                        for (int e = 0; e < BN; ++e)
                            if (e <= row) m8[e % 8] = fmaxf(m8[e % 8], __uint_as_float(rr[e]));
                    }
                    mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                }
                const float m_blk = mx * sl2;
                float m_new = m_used;
                if (m_blk > m_used + kRescaleLog2<FP8>) m_new = m_blk;
                const float alpha = (m_new == m_used) ? 1.f : fast_exp2(m_used - m_new);
                // exp2(s * sl2 - mref) = 2^(s - m_new) * P scale
                const float mref = (m_new == -INFINITY) ? 0.f : m_new - kPScaleLog2<FP8>;
                if (k > 0) {
                    // PV(k-1) writes O_s: it must be done before the rescale below.
                    w_ok = mbar_wait(&bars->o_done[s], ocount & 1, abort_flag, a.err);
                    ++ocount;
                    w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                    if (!w_ok) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (__any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll 1
                        for (int ch = 0; ch < D / 32; ++ch) {
                            uint32_t ro[32];
                            tmem_ld32(tO + ch * 32, ro);
#pragma unroll
                            for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
                            tmem_st32(tO + ch * 32, ro);
                        }
                    }
                }
                // P = exp2(S * sl2 - mref) on packed pairs, four packed partial sums; P is packed
                // (BF16 pairs or E4M3 quads) into the first columns of S_s as the TMEM A operand
                // of the PV MMA (S is already in registers).
                const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
                const uint64_t negm = pack_f32x2(-mref, -mref);
                // Most exponentials on the FMA pipe (polynomial), one pair in eight on MUFU; P is
                // then packed with one hardware conversion per pair (E4M3 or BF16).
                constexpr int kDeg = FP8 ? 2 : 3;
                uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int e = 0; e < BN; e += 2) {
                    const uint64_t x = fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])),
                                                 sl2x2, negm);
                    float x0, x1;
                    unpack_f32x2(x, x0, x1);
                    if (diag || j < 0) {
                        if (j < 0 || e > row) x0 = -INFINITY;
                        if (j < 0 || e + 1 > row) x1 = -INFINITY;
                    }
                    float p0, p1;
                    if ((e / 2) % 8 == 7) {
                        p0 = fast_exp2(x0);
                        p1 = fast_exp2(x1);
                    } else {
                        exp2_poly_x2<kDeg>(x0, x1, p0, p1);
                        if (diag || j < 0) {  // the polynomial maps -inf to ~2^-126, not 0
                            if (j < 0 || e > row) p0 = 0.f;
                            if (j < 0 || e + 1 > row) p1 = 0.f;
                        }
                    }
                    sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(p0, p1));
                    rr[e] = __float_as_uint(p0);
                    rr[e + 1] = __float_as_uint(p1);
                }
                if constexpr (FP8) {
                    uint32_t pk[BN / 4];
#pragma unroll
                    for (int q = 0; q < BN / 4; ++q)
                        pk[q] = pack_e4m3x2(__uint_as_float(rr[4 * q]), __uint_as_float(rr[4 * q + 1])) |
                                (static_cast<uint32_t>(pack_e4m3x2(__uint_as_float(rr[4 * q + 2]),
                                                                   __uint_as_float(rr[4 * q + 3])))
                                 << 16);
                    if constexpr (BN == 128)
                        tmem_st32(tS, pk);
                    else
                        tmem_st16(tS, pk);
                } else {
#pragma unroll
                    for (int hf = 0; hf < BN / 64; ++hf) {
                        uint32_t pk[32];
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            pk[q] = pack_bf16x2(__uint_as_float(rr[hf * 64 + 2 * q]), __uint_as_float(rr[hf * 64 + 2 * q + 1]));
                        tmem_st32(tS + hf * 32, pk);
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
                mbar_arrive(&bars->p_full[s]);
            }
            if (!ok) break;
            // Epilogue: the last PV of the tile must be done.
            bool w_ok = mbar_wait(&bars->o_done[s], ocount & 1, abort_flag, a.err);
            ++ocount;
            w_ok = __all_sync(0xFFFFFFFFu, w_ok);
            if (!w_ok) break;
            tc_fence_after();
            const int t_row = T.i * a.block + row;
            const bool store = row < a.block && t_row < T.n_tok;
            const float inv = (l_run > 0.f ? 1.f / l_run : 0.f) * a.out_scale;
            const int64_t orow = PAGED ? static_cast<int64_t>(a.cu_seqlens[T.b] + t_row) * a.ost
                                       : static_cast<int64_t>(T.b) * a.osb + static_cast<int64_t>(t_row) * a.ost;
            uint8_t* dst = reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.out) + orow +
                                                      static_cast<int64_t>(T.h) * a.osh);
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t rr[32];
                tmem_ld32(tO + ch * 32, rr);
                if (store) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w4[e] = pack_bf16x2(__uint_as_float(rr[q * 8 + 2 * e]) * inv,
                                                __uint_as_float(rr[q * 8 + 2 * e + 1]) * inv);
                        *reinterpret_cast<uint4*>(dst + (ch * 32 + q * 8) * 2) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            if (store && a.lse != nullptr)
                a.lse[(static_cast<int64_t>(T.b) * a.Hq + T.h) * a.lse_stride + t_row] =
                    (m_used + __log2f(l_run) - kPScaleLog2<FP8>) * 0.69314718055994531f;
            // The next tile's first PV overwrites O_s; the p_full arrival that lets the MMA warp
            // issue it comes after these loads.
            tc_fence_before();
            it.next(a);
        }
        tc_fence_before();
        mbar_arrive(&bars->tmem_free);
        return;
    }
}

template <bool FP8, int D, int BN, bool PAGED>
cudaError_t launch_ws_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                        cudaStream_t s) {
    using C = WsCfg<FP8, D, BN>;
    auto kern = attn_ws_kernel<FP8, D, BN, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long total = static_cast<long long>(a.B) * a.Hkv * a.nb_max * (a.Hq / a.Hkv);
    long long grid = (total + 1) / 2;
    if (grid > sms) grid = sms;
    kern<<<static_cast<unsigned>(grid), kThreads, C::SMEM, s>>>(tq, tk, tv, a, static_cast<int>(total));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_ws(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (fp8) {
        if (a.d != 128 || a.block != 128) return cudaErrorInvalidValue;
        return paged ? launch_ws_t<true, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_ws_t<true, 128, 128, false>(tq, tk, tv, a, s);
    }
    if (a.d == 128 && a.block == 128)
        return paged ? launch_ws_t<false, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_ws_t<false, 128, 128, false>(tq, tk, tv, a, s);
    if (a.d == 128 && a.block == 64)
        return paged ? launch_ws_t<false, 128, 64, true>(tq, tk, tv, a, s)
                     : launch_ws_t<false, 128, 64, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 128)
        return paged ? launch_ws_t<false, 64, 128, true>(tq, tk, tv, a, s)
                     : launch_ws_t<false, 64, 128, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 64)
        return paged ? launch_ws_t<false, 64, 64, true>(tq, tk, tv, a, s)
                     : launch_ws_t<false, 64, 64, false>(tq, tk, tv, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
