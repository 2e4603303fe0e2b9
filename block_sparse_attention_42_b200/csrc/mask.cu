// mask.cu -- block mask -> per-head kept-block lists, for bsa_prefill_mask / bsa_mask_to_lists.
//
// ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §二.2.2 BSA算子优化: the selection reaches
//  the sparse kernel as a block mask, which the kernel caches on chip and turns into the list of
//  kept blocks before its inner loop; a skipped block is a block of -inf scores.]
//
// Here the list is built once per call by this kernel, as compact CSR per (sequence, query
// head): row_ptr [B*Hq][nb+1], col_idx [B*Hq][T] with T = nb(nb+1)/2 (room for every causal
// block).  Row (b, h, i) keeps, in ascending order, every j <= i with mask[b][h][i][j] != 0;
// entries above the diagonal are ignored.  A row that keeps nothing gets O = 0 and
// LSE = -inf here (the attention kernels skip it).
//
// Three launches, so that the whole GPU works on every step: (1) one warp per row counts the
// nonzero mask bytes at j <= i (16 bytes per lane per load) into row_ptr; (2) one CTA per
// (b, h) turns the counts into offsets in place (block scan); (3) one warp per row writes the
// kept j in ascending order (4 bytes per lane per step, a warp scan of the per-lane counts).
// The mask rows are read twice; the second read finds them in L2.
#include <cmath>

#include <cuda_bf16.h>

#include "internal.h"

namespace bsa {
namespace {

constexpr int kRowWarps = 8;       // rows per CTA in the count and compaction kernels
constexpr int kScanThreads = 1024; // one thread per two rows (nb <= 2048)

// Bytes of w that are nonzero, as a mask of their high bits.
__device__ __forceinline__ uint32_t nonzero_bits(uint32_t w) {
    // A byte's high bit ends up set iff the byte is nonzero: low 7 bits + 0x7F carry into bit 7.
    return (((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u;
}

// Keeps the bytes of w at positions j0 .. j0+3 that are <= i.
__device__ __forceinline__ uint32_t clip_bytes(uint32_t w, int j0, int i) {
    const int valid = i + 1 - j0;
    if (valid >= 4) return w;
    return valid <= 0 ? 0u : (w & ((1u << (8 * valid)) - 1u));
}

// (1) row_ptr[bh][i] = kept-block count of row (b, h, i).
__global__ void __launch_bounds__(kRowWarps * 32) mask_count_kernel(const MaskListArgs m, int64_t rows) {
    const int lane = threadIdx.x % 32;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + threadIdx.x / 32;
    if (row >= rows) return;
    const int64_t bh = row / m.nb;
    const int i = static_cast<int>(row % m.nb);
    const uint4* p = reinterpret_cast<const uint4*>(m.mask + (bh * m.nb + i) * m.mask_stride);
    int c = 0;
    for (int v = lane; 16 * v <= i; v += 32) {
        const uint4 x = __ldg(p + v);
        const int j0 = 16 * v;
        c += __popc(nonzero_bits(clip_bytes(x.x, j0, i))) + __popc(nonzero_bits(clip_bytes(x.y, j0 + 4, i))) +
             __popc(nonzero_bits(clip_bytes(x.z, j0 + 8, i))) + __popc(nonzero_bits(clip_bytes(x.w, j0 + 12, i)));
    }
    c = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(c)));
    if (lane == 0) m.row_ptr[bh * (m.nb + 1) + i] = c;
}

// (2) counts -> exclusive offsets in place, total at [nb]; thread t owns rows 2t, 2t+1.
__global__ void __launch_bounds__(kScanThreads) mask_scan_kernel(const MaskListArgs m) {
    __shared__ int wsum[32];
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    const int nb = m.nb;
    int32_t* rp = m.row_ptr + static_cast<int64_t>(blockIdx.x) * (nb + 1);
    const int r0 = 2 * threadIdx.x, r1 = r0 + 1;
    const int c0 = r0 < nb ? rp[r0] : 0, c1 = r1 < nb ? rp[r1] : 0;
    int incl = c0 + c1;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();  // also: every count is read before any offset is written
    if (warp == 0) {
        int v = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
            if (lane >= o) v += y;
        }
        wsum[lane] = v;
    }
    __syncthreads();
    const int excl = incl - (c0 + c1) + (warp > 0 ? wsum[warp - 1] : 0);
    if (r0 < nb) rp[r0] = excl;
    if (r1 < nb) rp[r1] = excl + c0;
    if (threadIdx.x == kScanThreads - 1) rp[nb] = wsum[31];
}

// (3) the lists, ascending; rows that keep nothing get their outputs here.
__global__ void __launch_bounds__(kRowWarps * 32) mask_compact_kernel(const MaskListArgs m, int64_t rows) {
    const int lane = threadIdx.x % 32;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + threadIdx.x / 32;
    if (row >= rows) return;
    const int64_t bh = row / m.nb;
    const int i = static_cast<int>(row % m.nb);
    const int32_t* rp = m.row_ptr + bh * (m.nb + 1);
    const int base = rp[i];
    if (rp[i + 1] == base) {
        // No kept block: O = 0 and LSE = -inf for the block's query tokens of head h.
        const int b = static_cast<int>(bh / m.Hq), h = static_cast<int>(bh % m.Hq);
        const int t_lo = i * m.block, t_hi = min(m.N, t_lo + m.block);
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(m.out);
        const __nv_bfloat16 zero = __float2bfloat16(0.f);
        for (int e = lane; e < (t_hi - t_lo) * m.d; e += 32) {
            const int t = t_lo + e / m.d, c = e % m.d;
            o[static_cast<int64_t>(b) * m.osb + static_cast<int64_t>(t) * m.ost + static_cast<int64_t>(h) * m.osh + c] =
                zero;
        }
        if (m.lse)
            for (int t = t_lo + lane; t < t_hi; t += 32) m.lse[bh * m.lse_stride + t] = -INFINITY;
        return;
    }
    const uint32_t* p = reinterpret_cast<const uint32_t*>(m.mask + (bh * m.nb + i) * m.mask_stride);
    int32_t* ci = m.col_idx + bh * m.cap + base;
    int written = 0;
    for (int w0 = 0; 4 * w0 <= i; w0 += 32) {
        const int w = w0 + lane;
        const int j0 = 4 * w;
        const uint32_t nz = j0 <= i ? nonzero_bits(clip_bytes(__ldg(p + w), j0, i)) : 0u;
        const int c = __popc(nz);
        int incl = c;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        int pos = written + incl - c;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (nz & (0x80u << (8 * q))) ci[pos++] = j0 + q;
        written += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
}

}  // namespace

cudaError_t launch_mask_lists(const MaskListArgs& m, int B, cudaStream_t s) {
    const int64_t rows = static_cast<int64_t>(B) * m.Hq * m.nb;
    const unsigned grid = static_cast<unsigned>((rows + kRowWarps - 1) / kRowWarps);
    mask_count_kernel<<<grid, kRowWarps * 32, 0, s>>>(m, rows);
    mask_scan_kernel<<<B * m.Hq, kScanThreads, 0, s>>>(m);
    mask_compact_kernel<<<grid, kRowWarps * 32, 0, s>>>(m, rows);
    return cudaGetLastError();
}

}  // namespace bsa
