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
// One CTA per (b, h), 32 warps: (1) one warp per row counts the nonzero mask bytes at
// j <= i, 4 bytes per lane per load; (2) a block-wide exclusive scan of the counts gives
// row_ptr; (3) one warp per row writes the kept j in ascending order by ballot.  The mask
// rows are read twice; the second read comes from L2.
#include <cmath>

#include <cuda_bf16.h>

#include "internal.h"

namespace bsa {
namespace {

constexpr int kMaskThreads = 1024;

// Number of nonzero bytes of w among its first `valid` bytes (0..4).
__device__ __forceinline__ int nonzero_bytes(uint32_t w, int valid) {
    if (valid < 4) w &= (1u << (8 * valid)) - 1u;
    // A byte's high bit is set iff the byte is nonzero: low 7 bits + 0x7F carry into bit 7.
    const uint32_t nz = (((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u;
    return __popc(nz);
}

__global__ void __launch_bounds__(kMaskThreads) mask_lists_kernel(const MaskListArgs m) {
    __shared__ int off[kMaxBlocks + 1];
    __shared__ int wsum[32];
    const int bh = blockIdx.x;
    const int b = bh / m.Hq, h = bh % m.Hq;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    const int nb = m.nb;
    const uint8_t* mrows = m.mask + static_cast<int64_t>(bh) * nb * m.mask_stride;

    // (1) kept-block count of every row.
    for (int i = warp; i < nb; i += kMaskThreads / 32) {
        const uint32_t* row = reinterpret_cast<const uint32_t*>(mrows + static_cast<int64_t>(i) * m.mask_stride);
        int c = 0;
        for (int w = lane; 4 * w <= i; w += 32) c += nonzero_bytes(__ldg(row + w), min(4, i + 1 - 4 * w));
        c = __reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(c));
        if (lane == 0) off[i] = c;
    }
    __syncthreads();

    // (2) exclusive scan -> row_ptr; thread t owns rows 2t, 2t+1.
    const int r0 = 2 * threadIdx.x, r1 = r0 + 1;
    const int c0 = r0 < nb ? off[r0] : 0, c1 = r1 < nb ? off[r1] : 0;
    int incl = c0 + c1;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
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
    int32_t* rp = m.row_ptr + static_cast<int64_t>(bh) * (nb + 1);
    if (r0 < nb) {
        off[r0] = excl;
        rp[r0] = excl;
    }
    if (r1 < nb) {
        off[r1] = excl + c0;
        rp[r1] = excl + c0;
    }
    if (threadIdx.x == kMaskThreads - 1) {
        off[nb] = wsum[31];
        rp[nb] = wsum[31];
    }
    __syncthreads();

    // (3) the lists, ascending; empty rows get their outputs here.
    const unsigned lt_mask = (1u << lane) - 1u;
    int32_t* ci = m.col_idx + static_cast<int64_t>(bh) * m.cap;
    for (int i = warp; i < nb; i += kMaskThreads / 32) {
        const uint8_t* row = mrows + static_cast<int64_t>(i) * m.mask_stride;
        const int base = off[i];
        if (off[i + 1] == base) {
            // No kept block: O = 0 and LSE = -inf for the block's query tokens of head h.
            const int t_lo = i * m.block, t_hi = min(m.N, t_lo + m.block);
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(m.out);
            const __nv_bfloat16 zero = __float2bfloat16(0.f);
            for (int e = lane; e < (t_hi - t_lo) * m.d; e += 32) {
                const int t = t_lo + e / m.d, c = e % m.d;
                o[static_cast<int64_t>(b) * m.osb + static_cast<int64_t>(t) * m.ost + static_cast<int64_t>(h) * m.osh + c] =
                    zero;
            }
            if (m.lse)
                for (int t = t_lo + lane; t < t_hi; t += 32)
                    m.lse[static_cast<int64_t>(bh) * m.lse_stride + t] = -INFINITY;
            continue;
        }
        int written = 0;
        for (int j0 = 0; j0 <= i; j0 += 32) {
            const int j = j0 + lane;
            const bool keep = j <= i && row[j] != 0;
            const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
            if (keep) ci[base + written + __popc(bal & lt_mask)] = j;
            written += __popc(bal);
        }
    }
}

}  // namespace

cudaError_t launch_mask_lists(const MaskListArgs& m, int B, cudaStream_t s) {
    mask_lists_kernel<<<B * m.Hq, kMaskThreads, 0, s>>>(m);
    return cudaGetLastError();
}

}  // namespace bsa
