// validate.cu -- debug check of kept-block lists (bsa_validate_lists).
//
// The attention kernels trust the lists they are given: an entry outside [0, i] is the one
// corruption they detect on the fly (the block is read as all -inf and the error word is
// set).  A repeated entry would count a block twice, and lists out of order break the
// ascending order that stem_select and bsa_mask_to_lists promise.  This kernel checks every
// row of a CSR list set once, without touching the attention path, and records
// kDevErrInvalidList in the device error word on the first violation it meets:
//   - 0 <= row_ptr[i] <= row_ptr[i + 1] and row_ptr[i + 1] <= max_k;
//   - a row holds at most i + 1 entries, and at least one unless empty rows are allowed;
//   - entries strictly ascending, each in [0, i].
// One warp per (sequence, query head, query block); entries 32 at a time.
#include "internal.h"

namespace bsa {
namespace {

constexpr int kValWarps = 8;

__global__ void __launch_bounds__(kValWarps * 32) validate_lists_kernel(const ListCheckArgs c, int64_t rows) {
    const int lane = threadIdx.x % 32;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kValWarps + threadIdx.x / 32;
    if (row >= rows) return;
    // row -> (b, h, i): sequences in order, then heads, then query blocks
    int64_t r = row;
    int b = 0;
    while (r >= static_cast<int64_t>(c.nb[b]) * c.Hq) {
        r -= static_cast<int64_t>(c.nb[b]) * c.Hq;
        ++b;
    }
    const int h = static_cast<int>(r / c.nb[b]);
    const int i = static_cast<int>(r % c.nb[b]);
    const int32_t* rp = c.row_ptr + static_cast<int64_t>(b) * c.rp_stride + static_cast<int64_t>(h) * c.rp_hstride;
    const int64_t lo = rp[i], hi = rp[i + 1];
    bool bad = lo < 0 || hi < lo || hi > c.max_k || hi - lo > i + 1 || (hi == lo && !c.allow_empty);
    if (!bad) {
        const int32_t* list = c.col_idx + (static_cast<int64_t>(b) * c.Hq + h) * c.max_k + lo;
        const int n = static_cast<int>(hi - lo);
        int carry = -1;  // last entry of the previous chunk
        for (int n0 = 0; n0 < n; n0 += 32) {
            const int e = n0 + lane;
            const int j = e < n ? list[e] : 0x7FFFFFFF;
            int prev = __shfl_up_sync(0xFFFFFFFFu, j, 1);
            if (lane == 0) prev = carry;
            const bool ok = e >= n || (j >= 0 && j <= i && j > prev);
            bad |= !__all_sync(0xFFFFFFFFu, ok);
            carry = __shfl_sync(0xFFFFFFFFu, j, 31);
        }
    }
    if (bad && lane == 0) atomicOr(c.err, kDevErrInvalidList);
}

}  // namespace

cudaError_t launch_validate_lists(const ListCheckArgs& c, cudaStream_t s) {
    int64_t rows = 0;
    for (int b = 0; b < c.B; ++b) rows += static_cast<int64_t>(c.nb[b]) * c.Hq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((rows + kValWarps - 1) / kValWarps);
    validate_lists_kernel<<<grid, kValWarps * 32, 0, s>>>(c, rows);
    return cudaGetLastError();
}

}  // namespace bsa
