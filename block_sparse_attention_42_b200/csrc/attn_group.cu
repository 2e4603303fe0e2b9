// attn_group.cu -- a5 with group-shared lists: GQA-packed block-sparse causal prefill.  One CTA
// per SM serves two query heads of a KV-head group for one query block at a time; the two heads
// share the group's kept-block list, so every kept K/V block is loaded once for both.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; skipped blocks are -inf.  The pages
//  say nothing about grouped-query attention: sharing one list across a group's heads, and with
//  it each K/V load, is this library's extension.]
//
// The CTA (12 warps, persistent) owns one work unit at a time: (sequence, KV head, query block,
// pair of query heads of the group).  The pair's two heads are the two slots.  Registers are
// split by warpgroup with setmaxnreg: the control warpgroup (warps 0-3) drops to 56 per thread,
// the two softmax warpgroups rise to 224.
//   warp 0      TMA producer: takes the next unit from the launch's counter (handing it to the
//               other roles through a ring in shared memory), loads both slots' Q tiles of the
//               unit (one transaction), then K_j and V_j of every kept block into one ring of
//               stages shared by the slots, in the order the MMA warps consume them
//   warps 1, 3  MMA issuers of slot 0 and slot 1 (warp 1 owns tensor memory): S(k+1) = Q K^T as
//               soon as the slot's softmax has read S(k), O += P(k) V once P(k) is in shared
//               memory.  A ring stage is free once both slots' products have read it.
//   warp 2      idle (it only completes the control warpgroup's register release)
//   warps 4-7   softmax of slot 0, warps 8-11 softmax of slot 1: one query row per thread (TMEM
//               lane quadrant = warp % 4), as in the per-head kernels.
// Per slot two P buffers: P(k) only waits for PV(k-2).
// Paged K/V (bsa_prefill_paged_group): the producer loads a kept block as its 64-token pages
// through the page table, as the per-head kernels do; Q and O are the packed varlen rows.
// The two slots read the same blocks, so their S products land together and, left alone, their
// exponential phases would run at the same time: the MUFU (16 ex2 per clock per SM) would be
// shared while both exponentiate and idle while both do the rest of a block.  A token makes the
// slots take turns at the exponentials, so one slot's exponentials overlap the other's loads,
// max, P stores and rescale (measured at fp8-128k, before later changes: 52.3 ms against 56.7 ms
// without it).
// Tensor memory (512 columns): S slot 0 | S slot 1 | O slot 0 | O slot 1.
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBMg = 128;            // query rows per tile
constexpr int kThreadsG = 384;       // 12 warps: the control warpgroup and two softmax warpgroups
constexpr int kSlotsG = 2;           // query heads per work unit
constexpr int kSmemGLimit = 232448;  // 227 KB, one CTA per SM
constexpr int kMaxStagesG = 8;
constexpr int kListChunkG = 128;
// Register split (setmaxnreg): the launch grants 168 per thread (65536 / 384, rounded down to 8);
// the control warpgroup gives back what the softmax warpgroups take.
constexpr int kRegsLaunchG = 168;
constexpr int kRegsCtrlG = 56;
constexpr int kRegsSoftG = 224;
static_assert(128 * kRegsCtrlG + 256 * kRegsSoftG <= kThreadsG * kRegsLaunchG, "register split exceeds the launch");

template <bool FP8, int D, int BN>
struct CfgG {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;      // elements per 128-byte row of a panel
    static constexpr int QP = D * EB / 128;  // 128-byte panels per Q / K / V row
    static constexpr int Q_BYTES = kBMg * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int P_TILE = kBMg * BN * EB;
    static constexpr int NP = 2;             // P buffers per slot
    static constexpr int BAR_BYTES = 2048;
    static constexpr int FIXED = kSlotsG * (Q_BYTES + NP * P_TILE) + BAR_BYTES + 1024;
    static constexpr int NS_FIT = (kSmemGLimit - FIXED) / KV_BYTES;
    static constexpr int NS = NS_FIT > kMaxStagesG ? kMaxStagesG : NS_FIT;  // shared ring stages
    static constexpr int OFF_P = kSlotsG * Q_BYTES;
    static constexpr int OFF_RING = OFF_P + kSlotsG * NP * P_TILE;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static_assert(NS >= 4, "the shared ring needs four stages");
    static_assert(SMEM <= kSmemGLimit, "shared memory budget");
};

// E4M3: the running max moves only when the row max grew by more than 2^5, with P scaled by
// 2^3, so P <= 2^8 fits E4M3 and values down to 2^-12 of the row max keep E4M3 precision.
constexpr float kRescaleG = 5.f;
// A slot waits at most this long for its turn, then goes on without it (the token only orders
// the slots' exponentials; it is never needed for correctness).
constexpr uint64_t kTurnLimitNs = 20000;
constexpr float kPScaleG = 3.f;

struct SlotBarsG {
    uint64_t s_full, s_free, drain;
    // Block g of the slot writes P buffer g % 2 (p_full[g % 2]); its PV completes o_done[g % 2].
    uint64_t p_full[2], o_done[2];
};
struct BarsG {
    uint64_t kv_full[kMaxStagesG], kv_empty[kMaxStagesG];
    uint64_t q_full, q_empty;
    SlotBarsG sl[kSlotsG];
    uint64_t tmem_free;
    // Exponential-phase token: slot s waits on turn[s] before its exponentials and hands the
    // turn to the other slot after them, so the two slots' exponentials alternate.
    uint64_t turn[kSlotsG];
    uint32_t tmem_slot;
    int abort_flag;
    TileRing units;        // the dynamic unit schedule; freed by both MMA warps and 8 softmax warps
    int lst[kListChunkG];  // list entries staged by the producer warp
};
static_assert(sizeof(BarsG) <= 2048, "barrier region");

// Work unit u -> the per-head tile of the pair's first head: units are ordered like the per-head
// tiles (sequence, KV head, query block from the last one down), then by head pair.
__device__ __forceinline__ int unit_to_tile(const AttnArgs& a, int u) {
    const int G = a.Hq / a.Hkv, P = G / 2;
    const int per_b = a.Hkv * a.nb_max * P;
    const int b = u / per_b, x = u % per_b;
    const int p = x % P, y = x / P;  // y = hk * nb_max + (query blocks counted from the last)
    return b * a.Hkv * a.nb_max * G + y * G + 2 * p;
}

// The launch's counter runs over units; the ring carries the tile of the pair's first head.
struct UnitToTile {
    const AttnArgs* a;
    __device__ __forceinline__ int operator()(int u) const { return unit_to_tile(*a, u); }
};

template <bool PAGED>
__global__ void __launch_bounds__(kThreadsG, 1)
    attn_group_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const AttnArgs a, int total_units) {
    constexpr bool FP8 = true;
    constexpr int D = 128, BN = 128;
    using C = CfgG<FP8, D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BarsG* bars = reinterpret_cast<BarsG*>(smem + C::OFF_BAR);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int t = 0; t < C::NS; ++t) {
            mbar_init(&bars->kv_full[t], 1);
            mbar_init(&bars->kv_empty[t], kSlotsG);
        }
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, kSlotsG);
        for (int s = 0; s < kSlotsG; ++s) {
            SlotBarsG& B = bars->sl[s];
            mbar_init(&B.s_full, 1);
            mbar_init(&B.s_free, 128);
            mbar_init(&B.p_full[0], 128);
            mbar_init(&B.p_full[1], 128);
            mbar_init(&B.o_done[0], 1);
            mbar_init(&B.o_done[1], 1);
            mbar_init(&B.drain, 1);
        }
        mbar_init(&bars->tmem_free, 256);
        mbar_init(&bars->turn[0], 128);
        mbar_init(&bars->turn[1], 128);
        tile_ring_init(bars->units, 2 + 8);
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

    // Each warpgroup changes its register count at the top of its own branch, and no code after
    // the change is shared between the two register regimes.
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsCtrlG));
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            uint32_t ring = 0, qc = 0, tn = 0;
            unsigned bad = 0;
            bool ok = true;
            while (ok) {
                // The next unit of the launch, handed on to the MMA and softmax warps.
                int t = -1;
                if (lane == 0) ok = tile_ring_put(bars->units, tn++, a, total_units, t, abort_flag, UnitToTile{&a});
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                t = __shfl_sync(0xFFFFFFFFu, t, 0);
                if (!ok || t < 0) break;
                const Tile T = decode_tile(a, t);  // of the pair's first head; the second is T.h + 1
                if (lane == 0) {
                    ok = mbar_wait(&bars->q_empty, (qc & 1) ^ 1, abort_flag, a.err);
                    if (ok) {
                        mbar_arrive_expect_tx(&bars->q_full, kSlotsG * C::Q_BYTES);
                        const int tok0 = PAGED ? a.cu_seqlens[T.b] : 0;
#pragma unroll
                        for (int s = 0; s < kSlotsG; ++s)
#pragma unroll
                            for (int p = 0; p < C::QP; ++p)
                                tma_load_4d(smem + s * C::Q_BYTES + p * kBMg * 128, &tq, &bars->q_full, p * C::PW,
                                            tok0 + T.i * a.block, T.h + s, PAGED ? 0 : T.b);
                        ++qc;
                    }
                }
                for (int kb = 0; ok && kb < T.n_list; kb += kListChunkG) {
                    __syncwarp();
                    for (int e = lane; e < kListChunkG; e += 32)
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
                                        tma_load_4d(dst + p * BN * 128 + pg * 64 * 128, map, fb, p * C::PW, 0, T.hk,
                                                    phys);
                                    }
                                } else {
                                    tma_load_4d(dst + p * BN * 128, map, fb, p * C::PW, j * a.block, T.hk, T.b);
                                }
                            }
                            ++ring;
                            return true;
                        };
                        // The MMA warps' order: S(0), then S(k+1) ahead of PV(k); the loads follow
                        // it (K(0), then K(k+1) before V(k)), so the ring is consumed in the order
                        // it is filled.
                        const int kend = min(T.n_list, kb + kListChunkG);
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
            return;
        } else if (warp == 1 || warp == 3) {
            // ------------------------------------------------------------ MMA issuer of one slot
            const int slot = warp / 2;
            SlotBarsG& B = bars->sl[slot];
            if (lane == 0) {
                const uint32_t idesc_s = make_idesc(kBMg, BN, 0u, false, false);
                const uint32_t idesc_o = make_idesc(kBMg, D, 0u, false, true);
                const uint32_t aQ = smem_u32(smem + slot * C::Q_BYTES);
                const uint32_t tS = tmem + slot * BN;
                const uint32_t tO = tmem + 256 + slot * D;
                uint32_t rbase = 0, qc = 0, pc = 0, sf = 0, tn = 0;
                bool ok = true, first_s = true;
                Tile T;
                // S = Q K^T with K from ring position r.
                auto mma_s = [&](uint32_t r) -> bool {
                    // S is overwritten: the softmax must have read the previous S.
                    if (!first_s) {
                        if (!mbar_wait(&B.s_free, sf & 1, abort_flag, a.err)) return false;
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
                        const uint64_t da = smem_desc_sw128(aQ + pan * kBMg * 128 + within, 16, 1024);
                        const uint64_t db = smem_desc_sw128(aK + pan * BN * 128 + within, 16, 1024);
                        mma_f8_ss(tS, da, db, idesc_s, kk > 0);
                    }
                    tc_commit(&bars->kv_empty[st]);
                    tc_commit(&B.s_full);
                    return true;
                };
                // O (+)= P V with V from ring index r and P from the slot's buffer pc % 2.
                auto mma_pv = [&](uint32_t r, bool accumulate) -> bool {
                    const uint32_t pb = pc % C::NP;
                    if (!mbar_wait(&B.p_full[pb], (pc / C::NP) & 1, abort_flag, a.err)) return false;
                    ++pc;
                    const int st = r % C::NS;
                    if (!mbar_wait(&bars->kv_full[st], (r / C::NS) & 1, abort_flag, a.err)) return false;
                    tc_fence_after();
                    const uint32_t aP = smem_u32(smem + C::OFF_P + (slot * C::NP + pb) * C::P_TILE);
                    const uint32_t aV = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                    for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
                        const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                        const uint64_t da = smem_desc_sw128(aP + pan * kBMg * 128 + within, 16, 1024);
                        const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                        mma_f8_ss(tO, da, db, idesc_o, (accumulate || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&bars->kv_empty[st]);
                    tc_commit(&B.o_done[pb]);
                    return true;
                };
                while (ok) {
                    const int nt = tile_ring_get(bars->units, tn++, a, T, abort_flag);
                    if (nt <= 0) {
                        ok = nt == 0;
                        break;
                    }
                    const int n = T.n_list;
                    ok = mbar_wait(&bars->q_full, qc & 1, abort_flag, a.err);
                    ++qc;
                    // Ring positions of the unit (the producer's order K0, K1, V0, K2, V1, ...,
                    // V(n-1)): K(k) at 2k - 1 for k >= 1, V(k) at 2k + 2 for k < n - 1, V(n - 1) at 2n - 1.
                    ok = ok && mma_s(rbase);
                    if (ok && n == 1) tc_commit(&bars->q_empty);
                    for (int k = 0; ok && k < n; ++k) {
                        // S(k+1) goes ahead of PV(k): it only needs the softmax to have read S(k).
                        if (k + 1 < n) {
                            ok = mma_s(rbase + 2 * k + 1);
                            if (ok && k + 2 == n) tc_commit(&bars->q_empty);  // last S of the unit
                        }
                        ok = ok && mma_pv(rbase + (k + 1 < n ? 2 * k + 2 : 2 * n - 1), k > 0);
                    }
                    rbase += 2 * n;
                }
                tc_commit(&B.drain);
                volatile int no_abort = 0;
                mbar_wait(&B.drain, 0, &no_abort, a.err);
                if (slot == 0) mbar_wait(&bars->tmem_free, 0, &no_abort, a.err);
            }
            __syncwarp();
            if (slot == 0) {
                // The allocating warp frees tensor memory once both slots' MMAs have drained and
                // every softmax thread is done with it.
                if (lane == 0) {
                    volatile int no_abort = 0;
                    mbar_wait(&bars->sl[1].drain, 0, &no_abort, a.err);
                }
                __syncwarp();
                tc_fence_after();
                tmem_dealloc(tmem, 512);
            }
            return;
        }
        return;
    }
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftG));
    // ------------------------------------------------------------ softmax (warps 4-11)
    const int slot = (warp - 4) / 4;
    SlotBarsG& B = bars->sl[slot];
    const int quad = warp % 4;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + slot * BN;
    const uint32_t tO = tmem + lane_base + 256 + slot * D;
    uint8_t* sP = smem + C::OFF_P + slot * C::NP * C::P_TILE;
    uint32_t scount = 0;
    uint32_t g = 0;  // blocks this slot's softmax has finished (all units)
    // Waits until PV of block gg of this slot is complete (it read P buffer gg % 2, wrote O).
    auto wait_pv = [&](uint32_t gg) -> bool {
        const bool w = mbar_wait(&B.o_done[gg % C::NP], (gg / C::NP) & 1, abort_flag, a.err);
        return __all_sync(0xFFFFFFFFu, w);
    };
    const float sl2 = a.scale_log2;
    bool ok = true;
    // Slot 0 takes the first turn: slot 1 hands it over once at the start.
    if (slot == 1) mbar_arrive(&bars->turn[0]);
    uint32_t turns = 0;
    uint32_t tn = 0;
    while (ok) {
        Tile T;
        if (tile_ring_get_warp(bars->units, tn++, a, T, abort_flag, lane) <= 0) break;
        const int h = T.h + slot;
        float m_used = -INFINITY, l_run = 0.f;
        // The unit's list, 32 entries per warp-wide load (lane e: entry 32c + e), a chunk ahead of
        // its use; block k's entry is a shuffle.
        int jl = list_entry_raw(a, T, lane);
        int jl_next = list_entry_raw(a, T, 32 + lane);
        for (int k = 0; k < T.n_list; ++k) {
            if ((k & 31) == 0 && k > 0) {
                jl = jl_next;
                jl_next = list_entry_raw(a, T, k + 32 + lane);
            }
            const int j = list_entry_check(T, __shfl_sync(0xFFFFFFFFu, jl, k & 31));
            bool w_ok = mbar_wait(&B.s_full, scount & 1, abort_flag, a.err);
            ++scount;
            w_ok = __all_sync(0xFFFFFFFFu, w_ok);
            if (!w_ok) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool diag = (j == T.i);
            // The S row in registers: two 64-column TMEM reads, the second in flight while the
            // max of the first half is taken; after them S may be overwritten.  Masked scores
            // become -inf before the max: the causal part of the diagonal block, and all of a
            // skipped (invalid) block.
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
            tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[64]>(rr));
            tmem_ld64_nowait(tS + 64, *reinterpret_cast<uint32_t(*)[64]>(rr + 64));
            mask_max(0);
            tmem_ld_wait64(*reinterpret_cast<uint32_t(*)[64]>(rr + 64));
            tc_fence_before();
            mbar_arrive(&B.s_free);
            mask_max(64);
            const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
            const float m_blk = mx * sl2;
            float m_new = m_used;
            if (m_blk > m_used + kRescaleG) m_new = m_blk;
            const bool moved = m_new != m_used;
            const float mref = (m_new == -INFINITY) ? 0.f : m_new - kPScaleG;
            // Wait for this slot's turn (bounded: past the limit it goes on without it).
            {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bars->turn[slot], turns & 1))
                    if (globaltimer_ns() - t0 > kTurnLimitNs) break;
                ++turns;
            }
            // P = exp2(S * sl2 - mref) in place, four packed partial sums.
            const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
            const uint64_t negm = pack_f32x2(-mref, -mref);
            uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int e = 0; e < BN; e += 2) {
                const uint64_t x =
                    fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])), sl2x2, negm);
                float x0, x1;
                unpack_f32x2(x, x0, x1);
                const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(p0, p1));
                rr[e] = __float_as_uint(p0);
                rr[e + 1] = __float_as_uint(p1);
            }
            mbar_arrive(&bars->turn[slot ^ 1]);
            // The PV that last read this P buffer (block g - 2) must be complete.
            if (g >= static_cast<uint32_t>(C::NP)) {
                if (!wait_pv(g - C::NP)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            uint8_t* sPg = sP + (g % C::NP) * C::P_TILE;
            // P -> shared memory in the 128-byte-swizzled K-major layout of the PV A operand.
#pragma unroll
            for (int unit = 0; unit < BN / 16; ++unit) {  // 16 keys of e4m3 per 16 bytes
                uint32_t w4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = unit * 16 + q * 4;
                    w4[q] = pack_e4m3x4(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1]),
                                        __uint_as_float(rr[e + 2]), __uint_as_float(rr[e + 3]));
                }
                const int pan = unit / 8, cc = unit % 8;
                *reinterpret_cast<uint4*>(sPg + pan * kBMg * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                    make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async_smem();
            float s0, s1, s2, s3, s4, s5, s6, s7;
            unpack_f32x2(sum4[0], s0, s1);
            unpack_f32x2(sum4[1], s2, s3);
            unpack_f32x2(sum4[2], s4, s5);
            unpack_f32x2(sum4[3], s6, s7);
            const float sum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
            bool rescaled = false;
            float alpha = 1.f;
            if (k > 0 && __any_sync(0xFFFFFFFFu, moved)) {
                // O *= alpha once PV(g - 1) has finished accumulating into it; both 64-column
                // halves of the O row at once (P is in shared memory, rr is free).  (At k = 0
                // there is no O yet and l_run is 0, so the factor is not needed.)
                if (moved) alpha = fast_exp2(m_used - m_new);
                if (!wait_pv(g - 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t a2 = pack_f32x2(alpha, alpha);
                uint32_t(&ra)[64] = *reinterpret_cast<uint32_t(*)[64]>(rr);
                uint32_t(&rb)[64] = *reinterpret_cast<uint32_t(*)[64]>(rr + 64);
                tmem_ld64_nowait(tO, ra);
                tmem_ld64_nowait(tO + 64, rb);
                tmem_ld_wait64(rb);
                tmem_ld_wait64(ra);
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    float v0, v1;
                    unpack_f32x2(mul_f32x2(pack_f32x2(__uint_as_float(ra[e]), __uint_as_float(ra[e + 1])), a2), v0, v1);
                    ra[e] = __float_as_uint(v0);
                    ra[e + 1] = __float_as_uint(v1);
                    unpack_f32x2(mul_f32x2(pack_f32x2(__uint_as_float(rb[e]), __uint_as_float(rb[e + 1])), a2), v0, v1);
                    rb[e] = __float_as_uint(v0);
                    rb[e + 1] = __float_as_uint(v1);
                }
                tmem_st64(tO, ra);
                tmem_st64(tO + 64, rb);
                rescaled = true;
            }
            if (rescaled) tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&B.p_full[g % C::NP]);
            ++g;
            l_run = l_run * alpha + sum;
            m_used = m_new;
        }
        if (!ok) break;
        if (!wait_pv(g - 1)) break;
        tc_fence_after();
        const int t_row = T.i * a.block + row;
        const bool store = row < a.block && t_row < T.n_tok;
        const float inv = (l_run > 0.f ? 1.f / l_run : 0.f) * a.out_scale;
        const int64_t orow = PAGED ? static_cast<int64_t>(a.cu_seqlens[T.b] + t_row) * a.ost
                                   : static_cast<int64_t>(T.b) * a.osb + static_cast<int64_t>(t_row) * a.ost;
        uint8_t* dst =
            reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.out) + orow + static_cast<int64_t>(h) * a.osh);
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
            a.lse[(static_cast<int64_t>(T.b) * a.Hq + h) * a.lse_stride + t_row] =
                (m_used + __log2f(l_run) - kPScaleG) * 0.69314718055994531f;
        tc_fence_before();
    }
    tc_fence_before();
    mbar_arrive(&bars->tmem_free);
}

template <bool PAGED>
cudaError_t launch_group_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                           cudaStream_t s) {
    using C = CfgG<true, 128, 128>;
    if (a.tile_counter == nullptr) return cudaErrorInvalidValue;
    auto kern = attn_group_kernel<PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = static_cast<long long>(a.B) * a.Hkv * a.nb_max * (a.Hq / a.Hkv / 2);
    long long grid = sms;
    if (grid > units) grid = units;
    kern<<<static_cast<unsigned>(grid), kThreadsG, C::SMEM, s>>>(tq, tk, tv, a, static_cast<int>(units));
    return cudaGetLastError();
}

}  // namespace

bool attention_group_packed(bool fp8, const AttnArgs& a) {
    return fp8 && a.d == 128 && a.block == 128 && a.list_per_group && (a.Hq / a.Hkv) % 2 == 0;
}

cudaError_t launch_attention_group(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                   const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (!attention_group_packed(fp8, a)) return cudaErrorInvalidValue;
    return paged ? launch_group_t<true>(tq, tk, tv, a, s) : launch_group_t<false>(tq, tk, tv, a, s);
}

}  // namespace bsa
