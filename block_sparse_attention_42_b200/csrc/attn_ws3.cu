// attn_ws3.cu -- a5: block-sparse causal prefill, two independent pipelined CTAs per SM, with
// the next S computed while the softmax still works on the current block.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; skipped blocks are -inf.]
//
// Each CTA (6 warps, persistent, two per SM, 168 registers per thread) owns one query tile at
// a time:
//   warp 0      TMA producer: Q, then K_j and V_j of every kept block into a ring of stages
//   warp 1      MMA issuer (TMEM owner): S(k+1) = Q K^T as soon as the softmax has read S(k)
//               out of TMEM, and O += P(k) V once P(k) is in shared memory
//   warps 2-5   softmax, one query row per thread (TMEM lane quadrant = warp % 4): tcgen05.ld S,
//               online max/sum, P -> shared memory (128-byte swizzled K-major A operand),
//               O rescale when the row max grew enough, epilogue O / l -> BF16 and LSE
// The softmax never waits for the next S to be computed after its own P; before writing P(k)
// (and rescaling O) it waits for PV(k-1), normally long finished.
// The two CTAs on an SM interleave: one's softmax runs while the other's MMAs do.
// TMEM (256 columns per CTA): S | O.
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBM3 = 128;
constexpr int kThreads3 = 192;
constexpr int kSmem3Limit = 115712;  // two CTAs per SM
constexpr int kMaxStages3 = 6;
constexpr int kListChunk3 = 128;
constexpr int kBar3Bytes = 1024;  // barriers, tile ring, list buffer

template <bool FP8, int D, int BN>
struct Cfg3 {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;
    static constexpr int QP = D * EB / 128;
    static constexpr int Q_BYTES = kBM3 * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int P_TILE = kBM3 * BN * EB;
    // Two P buffers when four K/V stages still fit beside them: P(k) then waits for PV(k-2),
    // not PV(k-1).  The tiles start at the (1024-byte aligned) base of dynamic shared memory
    // with the barrier block after them, so E4M3 at d = 128 fits Q, two P buffers and four
    // stages exactly.
    static constexpr int NP = (kSmem3Limit - kBar3Bytes - Q_BYTES - 2 * P_TILE) / KV_BYTES >= 4 ? 2 : 1;
    static constexpr int P_BYTES = NP * P_TILE;
    static constexpr int NS_FIT = (kSmem3Limit - kBar3Bytes - Q_BYTES - P_BYTES) / KV_BYTES;
    static constexpr int NS = NS_FIT > kMaxStages3 ? kMaxStages3 : NS_FIT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = Q_BYTES;
    static constexpr int OFF_RING = OFF_P + P_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + kBar3Bytes;
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static_assert(NS >= 3, "the ring needs three stages: K(k+1) is consumed before V(k)");
    static_assert(SMEM <= kSmem3Limit, "shared memory budget");
};

// BF16: refresh the running max only when it grows by more than 2^8 (P <= 256 unscaled);
// E4M3: beyond 2^5 with P scaled by 2^3, so P <= 2^8 fits E4M3 and values down to 2^-12 of the
// row max keep E4M3 precision.
template <bool FP8>
constexpr float kRescale3 = FP8 ? 5.f : 8.f;
template <bool FP8>
constexpr float kPScale3 = FP8 ? 3.f : 0.f;

struct Bars3 {
    uint64_t kv_full[kMaxStages3], kv_empty[kMaxStages3];
    uint64_t q_full, q_empty, s_full, s_free, drain, tmem_free;
    // Per P buffer: block g's P is written into buffer g % NP (p_full[g % NP]) and its PV
    // completes o_done[g % NP].  With one barrier pair per buffer the softmax cannot complete a
    // p_full phase twice before the MMA warp has consumed it: reusing the buffer first needs
    // the PV issued after that phase.
    uint64_t p_full[2], o_done[2];
    uint32_t tmem_slot;
    int abort_flag;
    // Threshold skip: need[g % NP] == g + 1 when some row of block g kept it, so its PV runs.
    int need[2];
    TileRing tiles;  // the dynamic tile schedule; a slot is freed by the MMA and the 4 softmax warps
    int lst[kListChunk3];
};
static_assert(sizeof(Bars3) <= kBar3Bytes, "barrier region");

// SKIP: the threshold-skip instantiation (bsa_prefill_skip); the default one has none of its code.
template <bool FP8, int D, int BN, bool PAGED, bool SKIP>
__global__ void __launch_bounds__(kThreads3, 2)
    attn_ws3_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const AttnArgs a, int total_tiles) {
    using C = Cfg3<FP8, D, BN>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // The 128-byte-swizzled tiles need 1024-byte alignment and there is no slack to align up:
    // a base that is not aligned is reported (no thread has touched anything yet).
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0) atomicOr(a.err, kDevErrSmemAlign);
        return;
    }
    uint8_t* smem = smem_raw;
    Bars3* bars = reinterpret_cast<Bars3*>(smem + C::OFF_BAR);
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
        mbar_init(&bars->s_free, 128);
        mbar_init(&bars->p_full[0], 128);
        mbar_init(&bars->p_full[1], 128);
        mbar_init(&bars->o_done[0], 1);
        mbar_init(&bars->o_done[1], 1);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->tmem_free, 128);
        tile_ring_init(bars->tiles, 5);
        bars->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc(&bars->tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        uint32_t ring = 0, qc = 0, tn = 0;
        unsigned bad = 0;
        bool ok = true;
        while (ok) {
            // The next tile of the launch, handed on to the MMA and softmax warps.
            int t = -1;
            if (lane == 0) ok = tile_ring_put(bars->tiles, tn++, a, total_tiles, t, abort_flag);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            t = __shfl_sync(0xFFFFFFFFu, t, 0);
            if (!ok || t < 0) break;
            const Tile T = decode_tile(a, t);
            if (lane == 0) {
                ok = mbar_wait(&bars->q_empty, (qc & 1) ^ 1, abort_flag, a.err);
                if (ok) {
                    uint8_t* dst = smem + C::OFF_Q;
                    mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
                    const int tok0 = PAGED ? a.cu_seqlens[T.b] : 0;
#pragma unroll
                    for (int p = 0; p < C::QP; ++p)
                        tma_load_4d(dst + p * kBM3 * 128, &tq, &bars->q_full, p * C::PW, tok0 + T.i * a.block, T.h,
                                    PAGED ? 0 : T.b);
                    ++qc;
                }
            }
            for (int kb = 0; ok && kb < T.n_list; kb += kListChunk3) {
                __syncwarp();
                for (int e = lane; e < kListChunk3; e += 32)
                    if (kb + e < T.n_list) bars->lst[e] = list_entry(a, T, kb + e);
                __syncwarp();
                if (lane == 0) {
                    // K of block j (v = 0) or its V (v = 1) into the next ring stage.
                    auto issue = [&](int j, int v) -> bool {
                        if (j < 0) {
                            bad |= kDevErrInvalidList;
                            j = 0;
                        }
                        const int st = ring % C::NS;
                        if (!mbar_wait(&bars->kv_empty[st], ((ring / C::NS) & 1) ^ 1, abort_flag, a.err))
                            return false;
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
                        return true;
                    };
                    // The MMA warp's order: S(0), then S(k+1) ahead of PV(k).  The loads follow it,
                    // K(0), then K(k+1) before V(k), so a K block is requested one block earlier
                    // than a V block and the ring is consumed in the order it is filled.
                    const int kend = min(T.n_list, kb + kListChunk3);
                    if (kb == 0) ok = issue(bars->lst[0], 0);
                    for (int k = kb; ok && k < kend; ++k) {
                        if (k + 1 < T.n_list)
                            ok = issue(k + 1 < kend ? bars->lst[k + 1 - kb] : list_entry(a, T, k + 1), 0);
                        if (ok) ok = issue(bars->lst[k - kb], 1);
                    }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            }
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
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = make_idesc(kBM3, BN, FP8 ? 0u : 1u, false, false);
            const uint32_t idesc_o = make_idesc(kBM3, D, FP8 ? 0u : 1u, false, true);
            const uint32_t aQ = smem_u32(smem + C::OFF_Q);
            const uint32_t aP = smem_u32(smem + C::OFF_P);
            uint32_t rbase = 0, qc = 0, pc = 0, sf = 0;
            unsigned long long n_pv_skipped = 0;  // threshold skip: products not issued
            bool ok = true, first_s = true;
            uint32_t tn = 0;
            Tile T;
            // S = Q K^T with K from ring position r.
            auto mma_s = [&](uint32_t r) -> bool {
                // S is overwritten: the softmax must have read the previous S.
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
                    const uint64_t da = smem_desc_sw128(aQ + pan * kBM3 * 128 + within, 16, 1024);
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
            // O (+)= P V with V from ring index r and P from shared-memory buffer pc % NP.
            auto mma_pv = [&](uint32_t r, bool accumulate) -> bool {
                const uint32_t pb = pc % C::NP;
                if (!mbar_wait(&bars->p_full[pb], (pc / C::NP) & 1, abort_flag, a.err)) return false;
                // With the threshold skip, a block that every row skipped has P = 0: no product.
                const bool run = !SKIP || *reinterpret_cast<volatile int*>(&bars->need[pb]) ==
                                              static_cast<int>(pc + 1);
                if (SKIP) n_pv_skipped += run ? 0 : 1;
                ++pc;
                const int st = r % C::NS;
                if (!mbar_wait(&bars->kv_full[st], (r / C::NS) & 1, abort_flag, a.err)) return false;
                tc_fence_after();
                const uint32_t aV = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < (run ? C::KSTEPS_O : 0); ++kk) {
                    const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                    const uint64_t da = smem_desc_sw128(aP + pb * C::P_TILE + pan * kBM3 * 128 + within, 16, 1024);
                    const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                    const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
                    if constexpr (FP8)
                        mma_f8_ss(tmem + 128, da, db, idesc_o, acc);
                    else
                        mma_f16_ss(tmem + 128, da, db, idesc_o, acc);
                }
                tc_commit(&bars->kv_empty[st]);
                tc_commit(&bars->o_done[pb]);
                return true;
            };
            while (ok) {
                const int nt = tile_ring_get(bars->tiles, tn++, a, T, abort_flag);
                if (nt <= 0) {
                    ok = nt == 0;
                    break;
                }
                const int n = T.n_list;
                ok = mbar_wait(&bars->q_full, qc & 1, abort_flag, a.err);
                ++qc;
                // Ring positions of the tile (the producer's order K0, K1, V0, K2, V1, ..., V(n-1)):
                // K(k) at 2k - 1 for k >= 1, V(k) at 2k + 2 for k < n - 1, V(n - 1) at 2n - 1.
                ok = ok && mma_s(rbase);
                if (ok && n == 1) tc_commit(&bars->q_empty);
                for (int k = 0; ok && k < n; ++k) {
                    // S(k+1) goes ahead of PV(k): it only needs the softmax to have read S(k).
                    if (k + 1 < n) {
                        ok = mma_s(rbase + 2 * k + 1);
                        if (ok && k + 2 == n) tc_commit(&bars->q_empty);  // last S of the tile
                    }
                    ok = ok && mma_pv(rbase + (k + 1 < n ? 2 * k + 2 : 2 * n - 1), k > 0);
                }
                rbase += 2 * n;
            }
            if (SKIP && a.skip_stats != nullptr) {
                atomicAdd(a.skip_stats + 2, static_cast<unsigned long long>(pc));
                atomicAdd(a.skip_stats + 3, n_pv_skipped);
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
        // ------------------------------------------------------------ softmax (warps 2-5)
        const int quad = warp % 4;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tmem + lane_base;
        uint8_t* sP = smem + C::OFF_P;
        const uint32_t tO = tmem + lane_base + 128;
        uint32_t scount = 0;
        uint32_t g = 0;  // blocks this CTA's softmax has finished (all tiles)
        // Waits until PV of global block gg is complete (it read P buffer gg % NP, wrote O).
        auto wait_pv = [&](uint32_t gg) -> bool {
            const bool w = mbar_wait(&bars->o_done[gg % C::NP], (gg / C::NP) & 1, abort_flag, a.err);
            return __all_sync(0xFFFFFFFFu, w);
        };
        const float sl2 = a.scale_log2;
        uint32_t n_vis = 0, n_skipped = 0;  // threshold skip: row-blocks of real rows, and skipped
        bool ok = true;
        uint32_t tn = 0;
        while (ok) {
            Tile T;
            if (tile_ring_get_warp(bars->tiles, tn++, a, T, abort_flag, lane) <= 0) break;
            float m_used = -INFINITY, l_run = 0.f;
            float m_true = -INFINITY;  // exact running max (log2 units), for the threshold skip
            // The tile's list, 32 entries per warp-wide load: lane e holds entry 32c + e of the
            // current chunk c, and the next chunk is loaded a chunk ahead, so no block waits on
            // a global load; block k's entry is a shuffle.
            int jl = list_entry_raw(a, T, lane);
            int jl_next = list_entry_raw(a, T, 32 + lane);
            for (int k = 0; k < T.n_list; ++k) {
                if ((k & 31) == 0 && k > 0) {
                    jl = jl_next;
                    jl_next = list_entry_raw(a, T, k + 32 + lane);
                }
                const int j = list_entry_check(T, __shfl_sync(0xFFFFFFFFu, jl, k & 31));
                bool w_ok = mbar_wait(&bars->s_full, scount & 1, abort_flag, a.err);
                ++scount;
                w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                if (!w_ok) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const bool diag = (j == T.i);
                // The S row in registers (E4M3: two 64-column TMEM reads, the second in flight
                // while the max of the first half is taken); after them S may be overwritten.  Masked scores
                // become -inf here, outside the exponential loop: the causal part of the diagonal
                // block, and all of a skipped block.
                uint32_t rr[BN];
                float m8[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
                auto mask_max = [&](int base) {
                    if (diag || j < 0) {
                        // keys past lim are masked: the causal part of the diagonal block, or all
                        const int lim = j < 0 ? -1 : row - base;
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (e > lim) rr[base + e] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                    for (int e = 0; e < 64; e += 2)
                        m8[(e / 2) % 8] =
                            max3f(m8[(e / 2) % 8], __uint_as_float(rr[base + e]), __uint_as_float(rr[base + e + 1]));
                };
                if constexpr (BN == 128 && FP8) {
                    tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[64]>(rr));
                    tmem_ld64_nowait(tS + 64, *reinterpret_cast<uint32_t(*)[64]>(rr + 64));
                    mask_max(0);
                    tmem_ld_wait64(*reinterpret_cast<uint32_t(*)[64]>(rr + 64));
                    tc_fence_before();
                    mbar_arrive(&bars->s_free);
                    mask_max(64);
                } else if constexpr (BN == 128) {
                    // (BF16, d = 64: the overlapped form spills at this register budget)
                    tmem_ld128(tS, rr);
                    tc_fence_before();
                    mbar_arrive(&bars->s_free);
                    mask_max(0);
                    mask_max(64);
                } else {
                    tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[64]>(rr));
                    tc_fence_before();
                    mbar_arrive(&bars->s_free);
                    mask_max(0);
                }
                const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                float m_blk = mx * sl2;
                // Threshold skip ([BLASST] §2.1): the row drops this block when its max trails the
                // running max by more than log2(lambda); the block then adds nothing (P = 0).
                bool skip = false;
                if constexpr (SKIP) {
                    skip = m_blk - m_true < a.skip_log2;
                    m_true = fmaxf(m_true, m_blk);
                    if (skip) m_blk = -INFINITY;
                    if (row < a.block && T.i * a.block + row < T.n_tok) {
                        ++n_vis;
                        n_skipped += skip ? 1 : 0;
                    }
                }
                const bool warp_skip = SKIP && __all_sync(0xFFFFFFFFu, skip);
                float m_new = m_used;
                if (m_blk > m_used + kRescale3<FP8>) m_new = m_blk;
                const bool moved = m_new != m_used;
                const float mref = skip ? INFINITY : ((m_new == -INFINITY) ? 0.f : m_new - kPScale3<FP8>);
                // P = exp2(S * sl2 - mref) in place, four packed partial sums (a skipped row: 0).
                const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
                const uint64_t negm = pack_f32x2(-mref, -mref);
                uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int e = 0; e < (warp_skip ? 0 : BN); e += 2) {
                    const uint64_t x = fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])),
                                                 sl2x2, negm);
                    float x0, x1;
                    unpack_f32x2(x, x0, x1);
                    float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(p0, p1));
                    rr[e] = __float_as_uint(p0);
                    rr[e + 1] = __float_as_uint(p1);
                }
                // The PV that last read this P buffer must be complete.
                if (g >= static_cast<uint32_t>(C::NP)) {
                    if (!wait_pv(g - C::NP)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                uint8_t* sPg = sP + (g % C::NP) * C::P_TILE;
                if (SKIP && !warp_skip && lane == 0) bars->need[g % C::NP] = static_cast<int>(g + 1);
                // P -> shared memory in the 128-byte-swizzled K-major layout of the PV A operand.
                if constexpr (FP8) {
#pragma unroll
                    for (int unit = 0; unit < BN / 16; ++unit) {  // 16 keys of e4m3 per 16 bytes
                        uint32_t w4[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int e = unit * 16 + q * 4;
                            w4[q] = warp_skip ? 0u
                                              : pack_e4m3x4(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1]),
                                                            __uint_as_float(rr[e + 2]), __uint_as_float(rr[e + 3]));
                        }
                        const int pan = unit / 8, cc = unit % 8;
                        *reinterpret_cast<uint4*>(sPg + pan * kBM3 * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                } else {
#pragma unroll
                    for (int unit = 0; unit < BN / 8; ++unit) {  // 8 keys of bf16 per 16 bytes
                        uint32_t w4[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            w4[q] = warp_skip ? 0u
                                              : pack_bf16x2(__uint_as_float(rr[unit * 8 + 2 * q]),
                                                            __uint_as_float(rr[unit * 8 + 2 * q + 1]));
                        const int pan = unit / 8, cc = unit % 8;
                        *reinterpret_cast<uint4*>(sPg + pan * kBM3 * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
                fence_proxy_async_smem();
                float s0, s1, s2, s3, s4, s5, s6, s7;
                unpack_f32x2(sum4[0], s0, s1);
                unpack_f32x2(sum4[1], s2, s3);
                unpack_f32x2(sum4[2], s4, s5);
                unpack_f32x2(sum4[3], s6, s7);
                const float sum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
                float alpha = 1.f;
                if (k > 0 && __any_sync(0xFFFFFFFFu, moved)) {
                    // O *= alpha once PV(k-1) has finished accumulating into it.  P is in shared
                    // memory, so rr is free: both 64-column halves of the O row are read at once
                    // (the partial sums were reduced above to leave the registers for them).  (At
                    // k = 0 there is no O yet and l_run is 0, so the factor is not needed.)
                    if (moved) alpha = fast_exp2(m_used - m_new);
                    if (C::NP > 1) {
                        if (!wait_pv(g - 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const uint64_t a2 = pack_f32x2(alpha, alpha);
                    auto scale64 = [&](uint32_t(&ro)[64]) {
#pragma unroll
                        for (int e = 0; e < 64; e += 2) {
                            float v0, v1;
                            unpack_f32x2(mul_f32x2(pack_f32x2(__uint_as_float(ro[e]), __uint_as_float(ro[e + 1])), a2), v0, v1);
                            ro[e] = __float_as_uint(v0);
                            ro[e + 1] = __float_as_uint(v1);
                        }
                    };
                    if constexpr (D == 128 && BN == 128) {
                        uint32_t(&ra)[64] = *reinterpret_cast<uint32_t(*)[64]>(rr);
                        uint32_t(&rb)[64] = *reinterpret_cast<uint32_t(*)[64]>(rr + 64);
                        tmem_ld64_nowait(tO, ra);
                        tmem_ld64_nowait(tO + 64, rb);
                        tmem_ld_wait64(rb);
                        tmem_ld_wait64(ra);
                        scale64(ra);
                        scale64(rb);
                        tmem_st64(tO, ra);
                        tmem_st64(tO + 64, rb);
                    } else {
#pragma unroll 1
                        for (int ch = 0; ch < D / 64; ++ch) {
                            uint32_t ro[64];
                            tmem_ld64(tO + ch * 64, ro);
                            scale64(ro);
                            tmem_st64(tO + ch * 64, ro);
                        }
                    }
                }
                l_run = l_run * alpha + sum;
                m_used = m_new;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->p_full[g % C::NP]);
                ++g;
            }
            if (!ok) break;
            if (!wait_pv(g - 1)) break;
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
                a.lse[(static_cast<int64_t>(T.b) * a.Hq + T.h) * a.lse_stride + t_row] =
                    (m_used + __log2f(l_run) - kPScale3<FP8>) * 0.69314718055994531f;
            tc_fence_before();
        }
        if (SKIP && a.skip_stats != nullptr) {
            unsigned long long v0 = n_vis, v1 = n_skipped;
            for (int o = 16; o > 0; o >>= 1) {
                v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, o);
                v1 += __shfl_xor_sync(0xFFFFFFFFu, v1, o);
            }
            if (lane == 0) {
                atomicAdd(a.skip_stats + 0, v0);
                atomicAdd(a.skip_stats + 1, v1);
            }
        }
        tc_fence_before();
        mbar_arrive(&bars->tmem_free);
        return;
    }
}

template <bool FP8, int D, int BN, bool PAGED>
cudaError_t launch_ws3_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                         cudaStream_t s) {
    using C = Cfg3<FP8, D, BN>;
    if (a.tile_counter == nullptr) return cudaErrorInvalidValue;
    auto kern = a.skip_on ? attn_ws3_kernel<FP8, D, BN, PAGED, true> : attn_ws3_kernel<FP8, D, BN, PAGED, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long total = static_cast<long long>(a.B) * a.Hkv * a.nb_max * (a.Hq / a.Hkv);
    long long grid = 2LL * sms;
    if (grid > total) grid = total;
    kern<<<static_cast<unsigned>(grid), kThreads3, C::SMEM, s>>>(tq, tk, tv, a, static_cast<int>(total));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_ws3(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (fp8) {
        if (a.d != 128 || a.block != 128) return cudaErrorInvalidValue;
        return paged ? launch_ws3_t<true, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_ws3_t<true, 128, 128, false>(tq, tk, tv, a, s);
    }
    if (a.d == 128 && a.block == 128)  // the BF16 stages do not fit two CTAs per SM
        return launch_attention_ws2(fp8, paged, tq, tk, tv, a, s);
    if (a.d == 128 && a.block == 64)
        return paged ? launch_ws3_t<false, 128, 64, true>(tq, tk, tv, a, s)
                     : launch_ws3_t<false, 128, 64, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 128)
        return paged ? launch_ws3_t<false, 64, 128, true>(tq, tk, tv, a, s)
                     : launch_ws3_t<false, 64, 128, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 64)
        return paged ? launch_ws3_t<false, 64, 64, true>(tq, tk, tv, a, s)
                     : launch_ws3_t<false, 64, 64, false>(tq, tk, tv, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
