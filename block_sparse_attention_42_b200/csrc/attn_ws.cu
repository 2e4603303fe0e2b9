// attn_ws.cu -- a5: warp-specialised, persistent block-sparse causal prefill on tcgen05.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; skipped blocks are -inf.]
//
// One CTA per SM, 12 warps:
//   warp 0      TMA producer: Q tiles and a ring of K/V stages, in exactly the order the MMA
//               warp consumes them
//   warp 1      MMA issuer (and TMEM owner): S_s = Q_s K^T and O_s += P_s V for two query
//               tiles ("slots" s = 0, 1) in flight at once, so the tensor cores work on one
//               slot while the other slot's softmax runs
//   warps 4-7   softmax of slot 0, warps 8-11 softmax of slot 1: one query row per thread;
//               tcgen05.ld S, online max/sum, P -> shared memory, O rescale in TMEM when the
//               row max moved, and the tile epilogue (O / l -> BF16, LSE)
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1, 128 columns each.
// Each slot walks its own static sequence of work tiles (tile = query block i of head h), in
// KV-head-major order with the longest lists first.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBM = 128;
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kSmemLimit = 232448;  // 227 KB of dynamic shared memory per CTA

template <bool FP8, int D, int BN>
struct WsCfg {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;
    static constexpr int QP = D * EB / 128;
    static constexpr int Q_BYTES = kBM * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int P_BYTES = kBM * BN * EB;
    static constexpr int FIXED = 2 * Q_BYTES + 2 * P_BYTES;
    static constexpr int NS_FIT = (kSmemLimit - 2048 - FIXED) / KV_BYTES;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;  // K/V ring stages
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_RING = OFF_P + 2 * P_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + 1024 + 1024;  // barriers + alignment slack
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static_assert(NS >= 2, "K/V ring needs at least two stages");
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
    uint64_t kv_full[8], kv_empty[8];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t drain;
    uint32_t tmem_slot;
    int abort_flag;
};

// Work tile t -> (b, hk, i, g); tiles are ordered sequence-major, then KV head, then query
// block from the last one down, then the G query heads of the group.
struct Tile {
    int b, h, hk, i, n_tok, nb, n_list, l_begin;
    bool valid;
};

__device__ __forceinline__ Tile decode_tile(const AttnArgs& a, int t) {
    Tile T;
    const int G = a.Hq / a.Hkv;
    const int per_b = a.Hkv * a.nb_max * G;
    T.b = t / per_b;
    int x = t % per_b;
    const int g = x % G;
    x /= G;
    T.i = a.nb_max - 1 - (x % a.nb_max);
    T.hk = x / a.nb_max;
    T.h = T.hk * G + g;
    T.n_tok = a.seqlen[T.b];
    T.nb = (T.n_tok + a.block - 1) / a.block;
    T.valid = T.i < T.nb;
    T.n_list = 0;
    T.l_begin = 0;
    if (T.valid) {
        const int32_t* rp = a.row_ptr + static_cast<int64_t>(T.b) * a.row_ptr_stride;
        T.l_begin = rp[T.i];
        T.n_list = rp[T.i + 1] - T.l_begin;
        if (T.n_list < 1 || T.n_list > kMaxBlocks || T.l_begin < 0 ||
            T.l_begin + static_cast<int64_t>(T.n_list) > a.max_k) {
            T.n_list = 0;  // corrupt row pointer: the tile is skipped (and flagged by the producer)
        }
    }
    return T;
}

// List entry n of the tile; -1 if out of [0, i] (skipped block: scores all -inf).
__device__ __forceinline__ int list_entry(const AttnArgs& a, const Tile& T, int n) {
    const int j = __ldg(a.col_idx + (static_cast<int64_t>(T.b) * a.Hq + T.h) * a.max_k + T.l_begin + n);
    return (j >= 0 && j <= T.i) ? j : -1;
}

// Both the producer and the MMA warp run this same event sequence, so ring stages are
// filled and consumed in the same order.  Per slot: Q load, S(0), then PV(k), S(k+1) ...
struct Sched {
    int tile[2], n[2], a[2], round[2];
    bool active[2];
    int total, stride, base;
    __device__ void start(const AttnArgs& aa, int s) {
        // next non-empty tile of slot s
        while (true) {
            const int t = base + s + round[s] * stride;
            round[s]++;
            if (t >= total) {
                active[s] = false;
                return;
            }
            Tile T = decode_tile(aa, t);
            if (T.valid && T.n_list > 0) {
                tile[s] = t;
                n[s] = T.n_list;
                a[s] = 0;
                active[s] = true;
                return;
            }
        }
    }
};

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

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], 128);
            mbar_init(&bars->o_done[s], 1);
        }
        mbar_init(&bars->drain, 1);
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

    Sched sc;
    sc.total = total_tiles;
    sc.stride = 2 * gridDim.x;
    sc.base = 2 * blockIdx.x;
    sc.round[0] = sc.round[1] = 0;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t ring = 0, qcount[2] = {0, 0};
            bool ok = true;
            unsigned bad = 0;
            auto load_q = [&](int s) {
                Tile T = decode_tile(a, sc.tile[s]);
                ok = ok && mbar_wait(&bars->q_empty[s], (qcount[s] & 1) ^ 1, abort_flag, a.err);
                if (!ok) return;
                ++qcount[s];
                uint8_t* dst = smem + C::OFF_Q + s * C::Q_BYTES;
                mbar_arrive_expect_tx(&bars->q_full[s], C::Q_BYTES);
                const int tok0 = PAGED ? a.cu_seqlens[T.b] : 0;
#pragma unroll
                for (int p = 0; p < C::QP; ++p)
                    tma_load_4d(dst + p * kBM * 128, &tq, &bars->q_full[s], p * C::PW, tok0 + T.i * a.block, T.h,
                                PAGED ? 0 : T.b);
            };
            auto load_kv = [&](int s, int k, bool is_v) {
                Tile T = decode_tile(a, sc.tile[s]);
                int j = list_entry(a, T, k);
                if (j < 0) {
                    bad = 1;
                    j = 0;
                }
                const int st = ring % C::NS;
                ok = ok && mbar_wait(&bars->kv_empty[st], ((ring / C::NS) & 1) ^ 1, abort_flag, a.err);
                if (!ok) return;
                ++ring;
                uint8_t* dst = smem + C::OFF_RING + st * C::KV_BYTES;
                const CUtensorMap* map = is_v ? &tv : &tk;
                mbar_arrive_expect_tx(&bars->kv_full[st], C::KV_BYTES);
#pragma unroll
                for (int p = 0; p < C::QP; ++p) {
                    if constexpr (PAGED) {
#pragma unroll
                        for (int pg = 0; pg < BN / 64; ++pg) {
                            const int lp = j * (BN / 64) + pg;
                            const int phys = lp * 64 < T.n_tok
                                                 ? __ldg(a.page_table + static_cast<int64_t>(T.b) * a.max_pages + lp)
                                                 : a.num_pages;  // past the end of the sequence: zeros
                            tma_load_4d(dst + p * BN * 128 + pg * 64 * 128, map, &bars->kv_full[st], p * C::PW, 0,
                                        T.hk, phys);
                        }
                    } else {
                        tma_load_4d(dst + p * BN * 128, map, &bars->kv_full[st], p * C::PW, j * a.block, T.hk, T.b);
                    }
                }
            };
            for (int s = 0; s < 2; ++s) {
                sc.start(a, s);
                if (sc.active[s]) {
                    load_q(s);
                    load_kv(s, 0, false);
                    sc.a[s] = 1;
                }
            }
            while (ok && (sc.active[0] || sc.active[1])) {
                for (int s = 0; s < 2 && ok; ++s) {
                    if (!sc.active[s]) continue;
                    load_kv(s, sc.a[s] - 1, true);  // V for PV(a-1)
                    if (sc.a[s] < sc.n[s]) {
                        load_kv(s, sc.a[s], false);  // K for S(a)
                        sc.a[s]++;
                    } else {
                        sc.start(a, s);
                        if (sc.active[s]) {
                            load_q(s);
                            load_kv(s, 0, false);
                            sc.a[s] = 1;
                        }
                    }
                }
            }
            if (bad) atomicOr(a.err, kDevErrInvalidList);
            // Every issued copy must land before the CTA's shared memory goes away.
            volatile int no_abort = 0;
            const uint32_t issued = ring;
            for (uint32_t r = issued > C::NS ? issued - C::NS : 0; r < issued; ++r)
                mbar_wait(&bars->kv_full[r % C::NS], (r / C::NS) & 1, &no_abort, a.err);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = make_idesc(kBM, BN, FP8 ? 0u : 1u, false, false);
            const uint32_t idesc_o = make_idesc(kBM, D, FP8 ? 0u : 1u, false, true);
            uint32_t ring = 0, qcount[2] = {0, 0}, pcount[2] = {0, 0};
            bool ok = true;
            auto mma_s = [&](int s) {
                if (sc.a[s] == 0) {  // first block of a tile: its Q must have landed
                    ok = ok && mbar_wait(&bars->q_full[s], qcount[s] & 1, abort_flag, a.err);
                    ++qcount[s];
                }
                const int st = ring % C::NS;
                ok = ok && mbar_wait(&bars->kv_full[st], (ring / C::NS) & 1, abort_flag, a.err);
                if (!ok) return;
                ++ring;
                tc_fence_after();
                const uint32_t aQ = smem_u32(smem + C::OFF_Q + s * C::Q_BYTES);
                const uint32_t aK = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
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
                tc_commit(&bars->kv_empty[st]);
                tc_commit(&bars->s_full[s]);
                if (sc.a[s] == sc.n[s] - 1) tc_commit(&bars->q_empty[s]);  // last S of the tile
            };
            auto mma_pv = [&](int s, int k) {
                ok = ok && mbar_wait(&bars->p_full[s], pcount[s] & 1, abort_flag, a.err);
                ++pcount[s];
                const int st = ring % C::NS;
                ok = ok && mbar_wait(&bars->kv_full[st], (ring / C::NS) & 1, abort_flag, a.err);
                if (!ok) return;
                ++ring;
                tc_fence_after();
                const uint32_t aP = smem_u32(smem + C::OFF_P + s * C::P_BYTES);
                const uint32_t aV = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
                    const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                    const uint64_t da = smem_desc_sw128(aP + pan * kBM * 128 + within, 16, 1024);
                    const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                    const uint32_t acc = (k > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (FP8)
                        mma_f8_ss(tmem + 256 + s * 128, da, db, idesc_o, acc);
                    else
                        mma_f16_ss(tmem + 256 + s * 128, da, db, idesc_o, acc);
                }
                tc_commit(&bars->kv_empty[st]);
                tc_commit(&bars->o_done[s]);
            };
            for (int s = 0; s < 2; ++s) {
                sc.start(a, s);
                if (sc.active[s]) {
                    mma_s(s);
                    sc.a[s] = 1;
                }
            }
            while (ok && (sc.active[0] || sc.active[1])) {
                for (int s = 0; s < 2 && ok; ++s) {
                    if (!sc.active[s]) continue;
                    mma_pv(s, sc.a[s] - 1);
                    if (sc.a[s] < sc.n[s]) {
                        mma_s(s);
                        sc.a[s]++;
                    } else {
                        sc.start(a, s);
                        if (sc.active[s]) {
                            mma_s(s);
                            sc.a[s] = 1;
                        }
                    }
                }
            }
            // Drain: wait until every MMA issued by this thread has completed.
            tc_commit(&bars->drain);
            volatile int no_abort = 0;
            mbar_wait(&bars->drain, 0, &no_abort, a.err);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax, slot s
        const int s = (warp - 4) / 4;
        const int quad = warp % 4;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tmem + lane_base + s * 128;
        const uint32_t tO = tmem + lane_base + 256 + s * 128;
        uint8_t* sP = smem + C::OFF_P + s * C::P_BYTES;
        uint32_t scount = 0, ocount = 0;
        const float sl2 = a.scale_log2;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const int t = sc.base + s + r * sc.stride;
            if (t >= total_tiles) break;
            Tile T = decode_tile(a, t);
            if (!T.valid || T.n_list == 0) continue;
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
                // Pass 1: row max, 64 TMEM columns per load, eight independent max chains.
                float mx = -INFINITY;
                if (j >= 0) {
                    float m8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
                    for (int hf = 0; hf < BN / 64; ++hf) {
                        uint32_t rr[64];
                        tmem_ld64(tS + hf * 64, rr);
                        if (!diag) {
#pragma unroll
                            for (int e = 0; e < 64; e += 2)
                                m8[(e / 2) % 8] = max3f(m8[(e / 2) % 8], __uint_as_float(rr[e]), __uint_as_float(rr[e + 1]));
                        } else {
#pragma unroll
                            for (int e = 0; e < 64; ++e)
                                if (hf * 64 + e <= row) m8[e % 8] = fmaxf(m8[e % 8], __uint_as_float(rr[e]));
                        }
                    }
                    mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                }
                const float m_blk = mx * sl2;
                // The running max is refreshed only when a block's max exceeds it by more than
                // kRescaleLog2 (log2 units); P is formed as 2^(s - m) * kPScale, so P <= 2^(8) stays
                // inside BF16 and E4M3, and the O rescale below is rare.
                float m_new = m_used;
                if (m_blk > m_used + kRescaleLog2<FP8>) m_new = m_blk;
                const float alpha = (m_new == m_used) ? 1.f : fast_exp2(m_used - m_new);
                // exp2(s * sl2 - mref) = 2^(s - m_new) * kPScale
                const float mref = (m_new == -INFINITY) ? 0.f : m_new - kPScaleLog2<FP8>;
                if (k > 0) {
                    // PV(k-1) must be done: it reads P_s (rewritten below) and writes O_s.
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
                            uint32_t rr[32];
                            tmem_ld32(tO + ch * 32, rr);
#pragma unroll
                            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
                            tmem_st32(tO + ch * 32, rr);
                        }
                        tmem_st_wait();
                    }
                }
                // Pass 2: P = exp2(S * sl2 - mref) on packed pairs, four packed partial sums, and
                // P -> shared memory (128-byte swizzled K-major A operand of the PV MMA).
                const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
                const uint64_t negm = pack_f32x2(-mref, -mref);
                uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int hf = 0; hf < BN / 64; ++hf) {
                    uint32_t rr[64];
                    tmem_ld64(tS + hf * 64, rr);
                    float pv[64];
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const uint64_t x = fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])),
                                                     sl2x2, negm);
                        float x0, x1;
                        unpack_f32x2(x, x0, x1);
                        pv[e] = fast_exp2(x0);
                        pv[e + 1] = fast_exp2(x1);
                    }
                    if (diag || j < 0) {
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (j < 0 || hf * 64 + e > row) pv[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 64; e += 2)
                        sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(pv[e], pv[e + 1]));
                    if constexpr (FP8) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {  // four 16-key units of e4m3
                            uint32_t w4[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int e = u * 16 + q * 4;
                                w4[q] = pack_e4m3x2(pv[e], pv[e + 1]) | (static_cast<uint32_t>(pack_e4m3x2(pv[e + 2], pv[e + 3])) << 16);
                            }
                            const int unit = hf * 4 + u, pan = unit / 8, cc = unit % 8;
                            *reinterpret_cast<uint4*>(sP + pan * kBM * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                                make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {  // eight 8-key units of bf16
                            uint32_t w4[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) w4[q] = pack_bf16x2(pv[u * 8 + 2 * q], pv[u * 8 + 2 * q + 1]);
                            const int unit = hf * 8 + u, pan = unit / 8, cc = unit % 8;
                            *reinterpret_cast<uint4*>(sP + pan * kBM * 128 + row * 128 + ((cc ^ (row & 7)) * 16)) =
                                make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
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
                fence_proxy_async_smem();
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
            // The next tile's first PV overwrites O_s; its p_full arrival (after these loads)
            // is what lets the MMA warp issue it.
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
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
