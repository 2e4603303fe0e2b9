// select.cu -- a3 + a4: TPD budget generation and per-row top-k selection.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §3.1 TPD: a position-dependent budget
//  that re-distributes a fixed total toward early positions; §二.2.1: budget generation and
//  the selection sort are fused into one operator.]
//
// Budget rule (one CTA per sequence; data-independent, bit-exact with the host rule):
//   n_i = i+1, m_i = 1 (row 0) or 2, K* = clamp(round(density * sum n), sum m, sum n),
//   t_i(c) = min(n_i, max(m_i, c * w_i)) with w_i = sqrt(n_i) (decay 1/2) or n_i (uniform),
//   64 bisection steps for the smallest c with sum floor(t_i(c) * 2^32) >= K* * 2^32,
//   k_i = floor(t_i), and the K* - sum k_i leftover blocks go to the non-full rows with the
//   largest fractional parts (earlier row first).  Every operation is a correctly rounded
//   fp64 multiply, sqrt, min/max or an exact integer step, so any IEEE machine agrees.
//
// Selection (one warp per (sequence, head, query block) row): the row's causal scores
// S[i][0..i] are turned into order-preserving 32-bit keys (NaN -> -inf, -0 -> +0; the sink,
// the diagonal and j > i get a key below every score), a 4-pass 8-bit radix select finds
// the (k_i - 2)-th largest key, and ballots emit the kept blocks in ascending order with
// equal keys taken smallest-j first.
#include <cmath>

#include "internal.h"

namespace bsa {
namespace {

constexpr int kBudgetThreads = 256;
constexpr int kRowsPerThread = kMaxBlocks / kBudgetThreads;  // 8
static_assert(kMaxBlocks <= 2048, "the leftover search takes row indices below 2^11");

// Sum of v over the CTA with one barrier, for 0 <= v < 2^46 (a thread's fixed-point shares:
// at most 8 rows of at most 2^43 each).  Each warp adds the low 22 and the high 24 bits of v
// separately with one warp reduction each (sums below 2^27 and 2^29: no overflow), lane 0
// stores the warp's sum in red[par] (the buffer alternates between calls, so a call's writes
// cannot race a slower thread's reads of the call before), and every thread adds up the warp
// sums in the same order.
__device__ __forceinline__ long long block_sum_i64(long long v, long long (*red)[32], int& par) {
    const uint32_t lo = __reduce_add_sync(0xFFFFFFFFu, static_cast<uint32_t>(v & 0x3FFFFF));
    const uint32_t hi = __reduce_add_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 22));
    const int w = threadIdx.x / 32;
    if (threadIdx.x % 32 == 0) red[par][w] = (static_cast<long long>(hi) << 22) + lo;
    __syncthreads();
    long long t = 0;
#pragma unroll
    for (int q = 0; q < kBudgetThreads / 32; ++q) t += red[par][q];
    par ^= 1;
    return t;
}

__device__ __forceinline__ long long fixed_share(double c, double w, double n, double m) {
    double t = __dmul_rn(c, w);
    t = fmax(t, m);
    t = fmin(t, n);
    return static_cast<long long>(floor(__dmul_rn(t, 4294967296.0)));
}

__global__ void __launch_bounds__(kBudgetThreads) tpd_budget_kernel(const SelectSeqs seqs, int decay_half,
                                                                    int32_t* __restrict__ row_ptr, int nbs) {
    __shared__ long long red[2][32];
    __shared__ int wsum[33];
    int par = 0;
    const int b = blockIdx.x;
    const int nb = seqs.nb[b];
    const long long kstar = seqs.kstar[b];
    const long long target = kstar * (1ll << 32);

    // Rows tid*R .. tid*R+R-1 (contiguous, so the final prefix sum is a plain block scan).
    double w[kRowsPerThread];
    bool valid[kRowsPerThread];
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int i = threadIdx.x * kRowsPerThread + r;
        valid[r] = i < nb;
        const double n = static_cast<double>(i + 1);
        w[r] = decay_half ? __dsqrt_rn(n) : n;
    }
    double lo = 0.0, hi = static_cast<double>(nb);
    for (int it = 0; it < 64; ++it) {
        const double mid = __dmul_rn(__dadd_rn(lo, hi), 0.5);
        long long part = 0;
#pragma unroll
        for (int r = 0; r < kRowsPerThread; ++r) {
            const int i = threadIdx.x * kRowsPerThread + r;
            if (valid[r]) part += fixed_share(mid, w[r], static_cast<double>(i + 1), i == 0 ? 1.0 : 2.0);
        }
        const long long tot = block_sum_i64(part, red, par);
        if (tot >= target)
            hi = mid;
        else
            lo = mid;
    }
    int k[kRowsPerThread];
    unsigned long long key[kRowsPerThread];
    long long whole = 0;
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int i = threadIdx.x * kRowsPerThread + r;
        k[r] = 0;
        key[r] = 0;
        if (!valid[r]) continue;
        const long long F = fixed_share(hi, w[r], static_cast<double>(i + 1), i == 0 ? 1.0 : 2.0);
        k[r] = static_cast<int>(F >> 32);
        whole += k[r];
        // Leftover ranking key: larger fraction first, then the earlier row; 0 = not eligible.
        if (k[r] < i + 1)
            key[r] = (static_cast<unsigned long long>(F & 0xFFFFFFFFll) << 32) |
                     (0xFFFFFFFFull - static_cast<unsigned long long>(i));
    }
    const long long R = kstar - block_sum_i64(whole, red, par);
    if (R > 0) {
        // The R-th largest key (keys are distinct) by a bitwise search on its value.  Bits
        // 31..11 are set in every eligible key (row indices are below 2048), so once the
        // fraction is found they are set without a count.
        unsigned long long thr = 0;
        for (int bit = 63; bit >= 0; --bit) {
            if (bit == 31) {
                thr |= 0xFFFFF800ull;
                bit = 11;
                continue;
            }
            const unsigned long long cand = thr | (1ull << bit);
            long long cnt = 0;
#pragma unroll
            for (int r = 0; r < kRowsPerThread; ++r) cnt += key[r] >= cand ? 1 : 0;
            if (block_sum_i64(cnt, red, par) >= R) thr = cand;
        }
#pragma unroll
        for (int r = 0; r < kRowsPerThread; ++r)
            if (key[r] != 0 && key[r] >= thr) k[r] += 1;
    }
    // Exclusive prefix sum over rows -> row_ptr[b][0..nb], then pad to nbs.
    int mine = 0;
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) mine += k[r];
    int incl = mine;
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int v = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
            if (lane >= o) v += y;
        }
        wsum[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    int base = incl - mine + (wid > 0 ? wsum[wid - 1] : 0);
    int32_t* rp = row_ptr + static_cast<int64_t>(b) * (nbs + 1);
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int i = threadIdx.x * kRowsPerThread + r;
        if (i < nb) rp[i] = base;
        base += k[r];
    }
    for (int i = nb + threadIdx.x; i <= nbs; i += kBudgetThreads) rp[i] = static_cast<int32_t>(kstar);
}

// ------------------------------------------------------------------------------ selection

constexpr int kSelWarps = 8;

// Query blocks of a sequence with nb blocks that fall in [i_lo, i_hi).
__host__ __device__ __forceinline__ int class_rows(int nb, int i_lo, int i_hi) {
    const int hi = nb < i_hi ? nb : i_hi;
    return hi > i_lo ? hi - i_lo : 0;
}

__device__ __forceinline__ uint32_t order_key(float s) {
    if (s != s) s = -INFINITY;   // NaN ranks as -inf
    if (s == 0.f) s = 0.f;       // -0 and +0 tie
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Rows whose query block i lies in [i_lo, i_hi) (i_hi <= 32 * MAXPL), so that each launch is
// compiled for the longest row it sees and short rows issue no work for positions they lack.
template <int MAXPL>
__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(const float* __restrict__ S, const SelectSeqs seqs,
                                                                int Hq, int nbs, const int32_t* __restrict__ row_ptr,
                                                                int32_t* __restrict__ col_idx, int64_t max_k,
                                                                long long total_rows, int i_lo, int i_hi) {
    __shared__ uint32_t hist_all[kSelWarps][256];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    uint32_t* hist = hist_all[wid];
    const unsigned lt_mask = (1u << lane) - 1u;

    for (long long row = static_cast<long long>(blockIdx.x) * kSelWarps + wid; row < total_rows;
         row += static_cast<long long>(gridDim.x) * kSelWarps) {
        // Row order: sequence-major, then longest rows (largest i) first.
        long long rr = row;
        int b = 0;
        while (rr >= static_cast<long long>(class_rows(seqs.nb[b], i_lo, i_hi)) * Hq) {
            rr -= static_cast<long long>(class_rows(seqs.nb[b], i_lo, i_hi)) * Hq;
            ++b;
        }
        const int nb = seqs.nb[b];
        const int i = min(nb, i_hi) - 1 - static_cast<int>(rr / Hq);
        const int h = static_cast<int>(rr % Hq);
        const int32_t* rp = row_ptr + static_cast<int64_t>(b) * (nbs + 1);
        const int start = rp[i];
        const int k_i = rp[i + 1] - start;
        int32_t* out = col_idx + (static_cast<int64_t>(b) * Hq + h) * max_k + start;
        if (i == 0) {
            if (lane == 0) out[0] = 0;
            continue;
        }
        const int want_total = k_i - 2;  // picks among 1..i-1
        const float* srow = S + ((static_cast<int64_t>(b) * Hq + h) * nbs + i) * nbs;

        uint32_t key[MAXPL];
#pragma unroll
        for (int r = 0; r < MAXPL; ++r) {
            const int j = r * 32 + lane;
            key[r] = (j >= 1 && j < i) ? order_key(__ldg(srow + j)) : 0u;
        }

        uint32_t thr = 0xFFFFFFFFu;
        int want = want_total;
        if (want_total > 0) {
            uint32_t prefix = 0, pmask = 0;
            // High bytes shared by every candidate key (typical: the scores of a row have close
            // exponents) are the same in the threshold; their passes would pick that byte with
            // nothing above it, so they are skipped.
            uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
#pragma unroll
            for (int r = 0; r < MAXPL; ++r) {
                if (r * 32 < i + 1 && key[r] != 0u) {
                    kmn = min(kmn, key[r]);
                    kmx = max(kmx, key[r]);
                }
            }
            kmn = __reduce_min_sync(0xFFFFFFFFu, kmn);
            kmx = __reduce_max_sync(0xFFFFFFFFu, kmx);
            int pass0 = 0;
            while (pass0 < 4 && ((kmn ^ kmx) >> (24 - 8 * pass0)) == 0u) {
                prefix |= kmx & (0xFFu << (24 - 8 * pass0));
                pmask |= 0xFFu << (24 - 8 * pass0);
                ++pass0;
            }
#pragma unroll 1
            for (int pass = pass0; pass < 4; ++pass) {
                const int shift = 24 - 8 * pass;
#pragma unroll
                for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0;
                __syncwarp();
#pragma unroll
                for (int r = 0; r < MAXPL; ++r)
                    if (r * 32 < i + 1 && (key[r] & pmask) == prefix && key[r] != 0u)
                        atomicAdd(&hist[(key[r] >> shift) & 255u], 1u);
                __syncwarp();
                // lane l owns digits 255-8l .. 248-8l (high to low)
                uint32_t c[8], csum = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    c[q] = hist[255 - 8 * lane - q];
                    csum += c[q];
                }
                uint32_t incl = csum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += y;
                }
                const unsigned hit = __ballot_sync(0xFFFFFFFFu, incl >= static_cast<uint32_t>(want));
                const int L = __ffs(hit) - 1;
                uint32_t digit = 0, above = 0;
                if (lane == L) {
                    uint32_t acc = incl - csum;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (acc + c[q] >= static_cast<uint32_t>(want)) {
                            digit = 255 - 8 * lane - q;
                            break;
                        }
                        acc += c[q];
                    }
                    above = acc;
                }
                digit = __shfl_sync(0xFFFFFFFFu, digit, L);
                above = __shfl_sync(0xFFFFFFFFu, above, L);
                want -= static_cast<int>(above);
                prefix |= digit << shift;
                pmask |= 0xFFu << shift;
                __syncwarp();
            }
            thr = prefix;
        }
        // Emit 0, the kept candidates in ascending j, then i.
        if (lane == 0) out[0] = 0;
        int written = 1, eq_seen = 0;
        if (want_total > 0) {
#pragma unroll
            for (int r = 0; r < MAXPL; ++r) {
                if (r * 32 >= i + 1) break;
                const bool gt = key[r] != 0u && key[r] > thr;
                const bool eq = key[r] != 0u && key[r] == thr;
                const unsigned eqm = __ballot_sync(0xFFFFFFFFu, eq);
                const bool take = gt || (eq && eq_seen + __popc(eqm & lt_mask) < want);
                eq_seen += __popc(eqm);
                const unsigned tm = __ballot_sync(0xFFFFFFFFu, take);
                if (take) out[written + __popc(tm & lt_mask)] = r * 32 + lane;
                written += __popc(tm);
            }
        }
        if (lane == 0) out[written] = i;
        __syncwarp();
    }
}

template <int MAXPL>
cudaError_t launch_sel(const float* scores, const SelectSeqs& seqs, int Hq, int nbs, const int32_t* row_ptr,
                       int32_t* col_idx, int64_t max_k, cudaStream_t s) {
    const int i_lo = MAXPL == 8 ? 0 : 16 * MAXPL, i_hi = 32 * MAXPL;
    long long total = 0;
    for (int b = 0; b < seqs.B; ++b) total += static_cast<long long>(class_rows(seqs.nb[b], i_lo, i_hi)) * Hq;
    if (total == 0) return cudaSuccess;
    long long blocks = (total + kSelWarps - 1) / kSelWarps;
    if (blocks > 148 * 16) blocks = 148 * 16;
    select_kernel<MAXPL><<<static_cast<unsigned>(blocks), kSelWarps * 32, 0, s>>>(scores, seqs, Hq, nbs, row_ptr,
                                                                                  col_idx, max_k, total, i_lo, i_hi);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tpd_budget(const SelectSeqs& seqs, int nb_stride, bool decay_half, int32_t* row_ptr,
                              cudaStream_t s) {
    tpd_budget_kernel<<<seqs.B, kBudgetThreads, 0, s>>>(seqs, decay_half ? 1 : 0, row_ptr, nb_stride);
    return cudaGetLastError();
}

cudaError_t launch_select_rows(const float* scores, const SelectSeqs& seqs, int Hq, int nb_stride,
                               const int32_t* row_ptr, int32_t* col_idx, int64_t max_k, cudaStream_t s) {
    cudaError_t e;
    // One launch per row-length class, longest rows first: i in [1024, 2048), [512, 1024),
    // [256, 512), [0, 256).
    if ((e = launch_sel<64>(scores, seqs, Hq, nb_stride, row_ptr, col_idx, max_k, s)) != cudaSuccess) return e;
    if ((e = launch_sel<32>(scores, seqs, Hq, nb_stride, row_ptr, col_idx, max_k, s)) != cudaSuccess) return e;
    if ((e = launch_sel<16>(scores, seqs, Hq, nb_stride, row_ptr, col_idx, max_k, s)) != cudaSuccess) return e;
    return launch_sel<8>(scores, seqs, Hq, nb_stride, row_ptr, col_idx, max_k, s);
}

cudaError_t launch_select(const float* scores, const SelectSeqs& seqs, int Hq, int nb_stride, bool decay_half,
                          int32_t* row_ptr, int32_t* col_idx, int64_t max_k, cudaStream_t s) {
    cudaError_t e = launch_tpd_budget(seqs, nb_stride, decay_half, row_ptr, s);
    if (e != cudaSuccess) return e;
    return launch_select_rows(scores, seqs, Hq, nb_stride, row_ptr, col_idx, max_k, s);
}

}  // namespace bsa
