// attn_ws2.cu -- a5: block-sparse causal prefill, two independent pipelined CTAs per SM.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: data movement and
//  compute run as a pipeline; the KV-block list is built before the inner loop, which then
//  visits only valid blocks with the dense-attention body; skipped blocks are -inf.]
//
// Each CTA (6 warps, persistent, two per SM, 168 registers per thread) owns one query tile at
// a time:
//   warp 0      TMA producer: Q, then K_j and V_j of every kept block into a ring of stages
//   warp 1      MMA issuer (TMEM owner): S = Q K^T; after the softmax has written P (over S in
//               tensor memory), O += P V and, right behind it in issue order, the next S
//   warps 2-5   softmax, one query row per thread (TMEM lane quadrant = warp % 4): tcgen05.ld S,
//               online max/sum, P -> TMEM,
//               O rescale when the row max grew enough, epilogue O / l -> BF16 and LSE
// The two CTAs on an SM interleave: one's softmax runs while the other's MMAs do.
// TMEM (256 columns per CTA): S/P | O.
#include <cuda_bf16.h>

#include "attn_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

constexpr int kBM2 = 128;
constexpr int kThreads2 = 192;
constexpr int kSmem2Limit = 115712;  // two CTAs per SM
constexpr int kMaxStages2 = 6;
constexpr int kListChunk2 = 128;

template <bool FP8, int D, int BN>
struct Cfg2 {
    static constexpr int EB = FP8 ? 1 : 2;
    static constexpr int PW = 128 / EB;
    static constexpr int QP = D * EB / 128;
    static constexpr int Q_BYTES = kBM2 * D * EB;
    static constexpr int KV_BYTES = BN * D * EB;
    static constexpr int NS_FIT = (kSmem2Limit - 3072 - Q_BYTES) / KV_BYTES;
    static constexpr int NS = NS_FIT > kMaxStages2 ? kMaxStages2 : NS_FIT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = Q_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + 2048 + 1024;  // barriers, list buffer + alignment slack
    static constexpr int KSTEPS_S = D * EB / 32;
    static constexpr int KSTEPS_O = BN * EB / 32;
    static constexpr int ROWS_PER_KSTEP = 32 / EB;
    static_assert(NS >= 2, "the ring needs at least two stages");
    static_assert(SMEM <= kSmem2Limit, "shared memory budget");
};

// BF16: refresh the running max only when it grows by more than 2^8 (P <= 256 unscaled);
// E4M3: beyond 2^3 with P scaled by 2^5, so P <= 2^8 fits E4M3 with room below.
template <bool FP8>
constexpr float kRescale2 = FP8 ? 3.f : 8.f;
template <bool FP8>
constexpr float kPScale2 = FP8 ? 5.f : 0.f;

struct Bars2 {
    uint64_t kv_full[kMaxStages2], kv_empty[kMaxStages2];
    uint64_t q_full, q_empty, s_full, p_full, o_done, drain, tmem_free;
    uint32_t tmem_slot;
    int abort_flag;
    TileRing tiles;  // the dynamic tile schedule; a slot is freed by the MMA and the 4 softmax warps
    int lst[kListChunk2];
};
static_assert(sizeof(Bars2) <= 2048, "barrier region");

template <bool FP8, int D, int BN, bool PAGED>
__global__ void __launch_bounds__(kThreads2, 2)
    attn_ws2_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const AttnArgs a, int total_tiles) {
    using C = Cfg2<FP8, D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars2* bars = reinterpret_cast<Bars2*>(smem + C::OFF_BAR);
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
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->o_done, 1);
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
                        tma_load_4d(dst + p * kBM2 * 128, &tq, &bars->q_full, p * C::PW, tok0 + T.i * a.block, T.h,
                                    PAGED ? 0 : T.b);
                    ++qc;
                }
            }
            for (int kb = 0; ok && kb < T.n_list; kb += kListChunk2) {
                __syncwarp();
                for (int e = lane; e < kListChunk2; e += 32)
                    if (kb + e < T.n_list) bars->lst[e] = list_entry(a, T, kb + e);
                __syncwarp();
                if (lane == 0) {
                    const int kend = min(T.n_list, kb + kListChunk2);
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
            const uint32_t idesc_s = make_idesc(kBM2, BN, FP8 ? 0u : 1u, false, false);
            const uint32_t idesc_o = make_idesc(kBM2, D, FP8 ? 0u : 1u, false, true);
            const uint32_t aQ = smem_u32(smem + C::OFF_Q);
            uint32_t ring = 0, qc = 0, pc = 0, tn = 0;
            bool ok = true;
            Tile T;
            // S = Q K^T from ring stage `ring`
            auto mma_s = [&]() -> bool {
                const int st = ring % C::NS;
                if (!mbar_wait(&bars->kv_full[st], (ring / C::NS) & 1, abort_flag, a.err)) return false;
                tc_fence_after();
                const uint32_t aK = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS_S; ++kk) {
                    const uint32_t byte = kk * 32, pan = byte / 128, within = byte % 128;
                    const uint64_t da = smem_desc_sw128(aQ + pan * kBM2 * 128 + within, 16, 1024);
                    const uint64_t db = smem_desc_sw128(aK + pan * BN * 128 + within, 16, 1024);
                    if constexpr (FP8)
                        mma_f8_ss(tmem, da, db, idesc_s, kk > 0);
                    else
                        mma_f16_ss(tmem, da, db, idesc_s, kk > 0);
                }
                tc_commit(&bars->kv_empty[st]);
                tc_commit(&bars->s_full);
                ++ring;
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
                ok = ok && mma_s();
                if (ok && n == 1) tc_commit(&bars->q_empty);
                for (int k = 0; ok && k < n; ++k) {
                    // O += P V once the softmax has written P (over S, in TMEM).
                    ok = mbar_wait(&bars->p_full, pc & 1, abort_flag, a.err);
                    ++pc;
                    const int st = ring % C::NS;
                    ok = ok && mbar_wait(&bars->kv_full[st], (ring / C::NS) & 1, abort_flag, a.err);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t aV = smem_u32(smem + C::OFF_RING + st * C::KV_BYTES);
#pragma unroll
                    for (int kk = 0; kk < C::KSTEPS_O; ++kk) {
                        const uint64_t db = smem_desc_sw128(aV + kk * C::ROWS_PER_KSTEP * 128, BN * 128, 1024);
                        const uint32_t acc = (k > 0 || kk > 0) ? 1u : 0u;
                        if constexpr (FP8)
                            mma_f8_ts(tmem + 128, tmem + kk * 8, db, idesc_o, acc);
                        else
                            mma_f16_ts(tmem + 128, tmem + kk * 8, db, idesc_o, acc);
                    }
                    tc_commit(&bars->kv_empty[st]);
                    tc_commit(&bars->o_done);
                    ++ring;
                    // The next S overwrites the P columns this PV reads; tcgen05.mma instructions
                    // from one thread execute in issue order, so it can be issued right away.
                    if (k + 1 < n) {
                        ok = mma_s();
                        if (ok && k + 2 == n) tc_commit(&bars->q_empty);  // last S of the tile
                    }
                }
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
        const uint32_t tS = tmem + lane_base;        // S, then P in place
        const uint32_t tO = tmem + lane_base + 128;
        uint32_t scount = 0, ocount = 0;
        const float sl2 = a.scale_log2;
        bool ok = true;
        uint32_t tn = 0;
        while (ok) {
            Tile T;
            if (tile_ring_get_warp(bars->tiles, tn++, a, T, abort_flag, lane) <= 0) break;
            float m_used = -INFINITY, l_run = 0.f;
            // The tile's list, 32 entries per warp-wide load, loaded a chunk ahead of its use.
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
                // The S row in registers, one TMEM read.  Masked scores become -inf before the
                // max: the causal part of the diagonal block, all of a skipped block.
                uint32_t rr[BN];
                float m8[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
                auto mask_max = [&](int base) {
                    if (diag || j < 0) {
                        const int lim = j < 0 ? -1 : row - base;  // keys past lim are masked
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (e > lim) rr[base + e] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                    for (int e = 0; e < 64; e += 2)
                        m8[(e / 2) % 8] = max3f(m8[(e / 2) % 8], __uint_as_float(rr[base + e]), __uint_as_float(rr[base + e + 1]));
                };
                if constexpr (BN == 128) {
                    // (one 128-column read: overlapping the halves spills at this register budget)
                    tmem_ld128(tS, rr);
                    mask_max(0);
                    mask_max(64);
                } else {
                    tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[64]>(rr));
                    mask_max(0);
                }
                const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                const float m_blk = mx * sl2;
                float m_new = m_used;
                if (m_blk > m_used + kRescale2<FP8>) m_new = m_blk;
                const bool moved = m_new != m_used;
                const float mref = (m_new == -INFINITY) ? 0.f : m_new - kPScale2<FP8>;
                // P = exp2(S * sl2 - mref) in place, four packed partial sums.
                const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
                const uint64_t negm = pack_f32x2(-mref, -mref);
                uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int e = 0; e < BN; e += 2) {
                    const uint64_t x = fma_f32x2(pack_f32x2(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1])), sl2x2, negm);
                    float x0, x1;
                    unpack_f32x2(x, x0, x1);
                    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    sum4[(e / 2) % 4] = add_f32x2(sum4[(e / 2) % 4], pack_f32x2(p0, p1));
                    rr[e] = __float_as_uint(p0);
                    rr[e + 1] = __float_as_uint(p1);
                }
                // P packed (BF16 pairs or E4M3 quads) over the S columns, as the TMEM A operand
                // of PV (S(k) was computed after PV(k-1) had read P(k-1) from them).
                // (8 TMEM columns per store, so few registers beyond the P row are live)
#pragma unroll
                for (int c = 0; c < BN / (FP8 ? 32 : 16); ++c) {
                    uint32_t pk[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if constexpr (FP8)
                            pk[q] = pack_e4m3x4(__uint_as_float(rr[c * 32 + 4 * q]), __uint_as_float(rr[c * 32 + 4 * q + 1]),
                                                __uint_as_float(rr[c * 32 + 4 * q + 2]), __uint_as_float(rr[c * 32 + 4 * q + 3]));
                        else
                            pk[q] = pack_bf16x2(__uint_as_float(rr[c * 16 + 2 * q]), __uint_as_float(rr[c * 16 + 2 * q + 1]));
                    }
                    tmem_st8(tS + c * 8, pk);
                }
                float s0, s1, s2, s3, s4, s5, s6, s7;
                unpack_f32x2(sum4[0], s0, s1);
                unpack_f32x2(sum4[1], s2, s3);
                unpack_f32x2(sum4[2], s4, s5);
                unpack_f32x2(sum4[3], s6, s7);
                const float sum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
                float alpha = 1.f;
                if (k > 0) {
                    // PV(k-1) has finished accumulating into O (the commit of S(k) already implies
                    // it: the two were issued in that order by one thread).
                    w_ok = mbar_wait(&bars->o_done, ocount & 1, abort_flag, a.err);
                    ++ocount;
                    if (!__all_sync(0xFFFFFFFFu, w_ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (__any_sync(0xFFFFFFFFu, moved)) {
                        // O *= alpha, the O row read 64 columns at a time, both halves at once
                        // where D = 128 and rr (128 registers, P already in TMEM) holds them.
                        if (moved) alpha = fast_exp2(m_used - m_new);
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
                }
                l_run = l_run * alpha + sum;
                m_used = m_new;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->p_full);
            }
            if (!ok) break;
            bool w_ok = mbar_wait(&bars->o_done, ocount & 1, abort_flag, a.err);
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
                    (m_used + __log2f(l_run) - kPScale2<FP8>) * 0.69314718055994531f;
            tc_fence_before();
        }
        tc_fence_before();
        mbar_arrive(&bars->tmem_free);
        return;
    }
}

template <bool FP8, int D, int BN, bool PAGED>
cudaError_t launch_ws2_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                         cudaStream_t s) {
    using C = Cfg2<FP8, D, BN>;
    if (a.tile_counter == nullptr) return cudaErrorInvalidValue;
    auto kern = attn_ws2_kernel<FP8, D, BN, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long total = static_cast<long long>(a.B) * a.Hkv * a.nb_max * (a.Hq / a.Hkv);
    long long grid = 2LL * sms;
    if (grid > total) grid = total;
    kern<<<static_cast<unsigned>(grid), kThreads2, C::SMEM, s>>>(tq, tk, tv, a, static_cast<int>(total));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_ws2(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
    if (fp8) {
        if (a.d != 128 || a.block != 128) return cudaErrorInvalidValue;
        return paged ? launch_ws2_t<true, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_ws2_t<true, 128, 128, false>(tq, tk, tv, a, s);
    }
    if (a.d == 128 && a.block == 128)
        return paged ? launch_ws2_t<false, 128, 128, true>(tq, tk, tv, a, s)
                     : launch_ws2_t<false, 128, 128, false>(tq, tk, tv, a, s);
    if (a.d == 128 && a.block == 64)
        return paged ? launch_ws2_t<false, 128, 64, true>(tq, tk, tv, a, s)
                     : launch_ws2_t<false, 128, 64, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 128)
        return paged ? launch_ws2_t<false, 64, 128, true>(tq, tk, tv, a, s)
                     : launch_ws2_t<false, 64, 128, false>(tq, tk, tv, a, s);
    if (a.d == 64 && a.block == 64)
        return paged ? launch_ws2_t<false, 64, 64, true>(tq, tk, tv, a, s)
                     : launch_ws2_t<false, 64, 64, false>(tq, tk, tv, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
