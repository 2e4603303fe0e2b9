// internal.h -- launch interfaces shared between the C-ABI front end (abi.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace bsa {

// Device error word bits (read back by bsa_check_device_error).
constexpr unsigned kDevErrInvalidList = 1u;
constexpr unsigned kDevErrTimeout = 2u;
constexpr unsigned kDevErrInvalidPage = 4u;
constexpr unsigned kDevErrSmemAlign = 8u;  // dynamic shared memory not 1024-byte aligned (nothing ran)

constexpr int kMaxBatch = 256;     // sequences per call
constexpr int kMaxBlocks = 2048;   // query blocks per sequence

struct TensorArg {
    const void* ptr;
    int64_t sb, st, sh;  // element strides
    float scale;
};

// a1: pooled block representations.  Writes the Q means [B,Hq,nb,d] as qbar = qhi + qlo (qhi
// exact in TF32, qlo the fp32 remainder), the K means [B,Hkv,nb,d] as khi + klo, and the mean
// V norms vbar [B,Hkv,nb] (fp32).  dtype: 0 bf16, 1 e4m3, 2 fp32.
cudaError_t launch_pool(int dtype, TensorArg q, TensorArg k, TensorArg v, int B, int N, int Hq, int Hkv, int d,
                        int block, float* qhi, float* qlo, float* khi, float* klo, float* vbar, cudaStream_t s);

// a1, group-shared selection: ghi + glo [B, Hkv, nb, d] = mean over the G = Hq / Hkv query heads
// of each KV-head group of qhi + qlo [B, Hq, nb, d] (fp64 sum, one fp32 rounding, hi / lo split).
cudaError_t launch_group_mean(const float* qhi, const float* qlo, int B, int Hq, int Hkv, int nb, int d, float* ghi,
                              float* glo, cudaStream_t s);

// a2: block scores from pooled representations.
// tcgen05 3xTF32 GEMM (score_tc.cu) over 4-D tensor maps of qhi, qlo [d, nb, Hq, B] and khi,
// klo [d, nb, Hkv, B] (fp32, 128-byte swizzle, box 32 x 128); err = device error word.
cudaError_t launch_score_tc(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                            const CUtensorMap& mkl, const float* vbar, int B, int Hq, int Hkv, int nb, int d,
                            float tau, int metric, float* scores, int nb_stride, unsigned* err, cudaStream_t s);
// fp32 FMA version (score.cu); reads qhi + qlo and khi + klo.
cudaError_t launch_score(const float* qhi, const float* qlo, const float* khi, const float* klo, const float* vbar,
                         int B, int Hq, int Hkv, int nb, int d, float tau, int metric, float* scores, int nb_stride,
                         cudaStream_t s);

struct SelectSeqs {
    int32_t B;
    int32_t nb[kMaxBatch];
    int64_t kstar[kMaxBatch];
};

// a3 + a4: TPD budgets into row_ptr, then per-row top-k lists into col_idx.
cudaError_t launch_select(const float* scores, const SelectSeqs& seqs, int Hq, int nb_stride, bool decay_half,
                          int32_t* row_ptr, int32_t* col_idx, int64_t max_k, cudaStream_t s);
// The two halves of launch_select: the budget (row_ptr [B, nb_stride + 1]) and the per-row top-k
// of scores [B, Hq, nb_stride, nb_stride] into col_idx [B, Hq, max_k] (row_ptr already written).
cudaError_t launch_tpd_budget(const SelectSeqs& seqs, int nb_stride, bool decay_half, int32_t* row_ptr,
                              cudaStream_t s);
cudaError_t launch_select_rows(const float* scores, const SelectSeqs& seqs, int Hq, int nb_stride,
                               const int32_t* row_ptr, int32_t* col_idx, int64_t max_k, cudaStream_t s);

// a5: block-sparse prefill.
struct AttnArgs {
    int B, Hq, Hkv, d, block;
    int nb_max;                  // max blocks over sequences
    int N;                       // dense layout: sequence length
    const int32_t* cu_seqlens;   // paged layout: device prefix offsets (nullptr for dense)
    int32_t seqlen[kMaxBatch];   // per-sequence lengths (dense: all N)
    const int32_t* row_ptr;
    int row_ptr_stride;          // entries between sequences
    int row_ptr_hstride;         // entries between query heads (0: one row_ptr for all heads)
    int allow_empty;             // 1: an empty list is a row with no kept block (its output
                                 // is written elsewhere), not an error
    const int32_t* col_idx;      // [B, Hq, max_k], or [B, Hkv, max_k] with list_per_group
    int64_t max_k;
    int list_per_group;          // 1: one list per KV-head group, shared by its query heads
    const int32_t* page_table;   // paged only
    int max_pages, page_size, num_pages;
    float scale_log2;            // softmax scale * log2(e) (* q_scale * k_scale for FP8)
    int skip_on;                 // 1: skip a block for a row whose block max trails its running max
    float skip_log2;             //    by more than log2(lambda) = skip_log2 (threshold skip)
    unsigned long long* skip_stats;  // nullable [4]: row-blocks visited, row-blocks skipped,
                                     // tile-blocks, tile-blocks whose P.V product was skipped
    float out_scale;             // multiplies the normalised output (v_scale for FP8)
    void* out;
    int64_t osb, ost, osh;       // out element strides
    float* lse;
    int64_t lse_stride;          // tokens per (b, h) row of lse
    unsigned* err;
    int* tile_counter;           // zeroed before the launch: the next tile index of a dynamic
                                 // tile schedule (attn_ws3.cu)
};

// Persistent, two independent pipelined CTAs per SM, one query tile each (attn_ws2.cu).
cudaError_t launch_attention_ws2(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s);

// As ws2, but P goes through shared memory so S(k+1) is computed while the softmax still works
// on block k (attn_ws3.cu).  FP8, and BF16 shapes whose stages fit two CTAs per SM.
cudaError_t launch_attention_ws3(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s);
// Group-shared lists (a.list_per_group): one CTA per SM serves two query heads of a KV-head group
// for a query block, loading each kept K/V block once for both (attn_group.cu).  Applies to FP8
// at d = 128 / block 128 with an even group size (attention_group_packed).
bool attention_group_packed(bool fp8, const AttnArgs& a);
cudaError_t launch_attention_group(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                                   const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s);

// Block mask -> per-head CSR lists (mask.cu).  mask [B, Hq, nb, mask_stride] uint8 (16-byte
// aligned, mask_stride a multiple of 16 and >= nb); row_ptr [B*Hq][nb+1]; col_idx [B*Hq][cap]
// with cap >= nb(nb+1)/2.  Rows that keep nothing get O = 0 (BF16 out, element strides) and
// LSE = -inf (if lse is not null) for their query tokens.
struct MaskListArgs {
    const uint8_t* mask;
    int64_t mask_stride;
    int Hq, nb, N, block, d;
    int32_t* row_ptr;
    int32_t* col_idx;
    int64_t cap;
    void* out;
    int64_t osb, ost, osh;
    float* lse;
    int64_t lse_stride;
};
cudaError_t launch_mask_lists(const MaskListArgs& m, int B, cudaStream_t s);

// Debug check of a CSR list set (validate.cu): records kDevErrInvalidList in *err on a
// row_ptr out of order or past max_k, a row longer than i + 1 (or empty, unless allowed), or
// entries not strictly ascending within [0, i].
struct ListCheckArgs {
    int B, Hq;
    int32_t nb[kMaxBatch];
    const int32_t* row_ptr;
    int64_t rp_stride, rp_hstride;  // entries between sequences / query heads (0: shared)
    const int32_t* col_idx;         // [B, Hq, max_k]
    int64_t max_k;
    int allow_empty;
    unsigned* err;
};
cudaError_t launch_validate_lists(const ListCheckArgs& c, cudaStream_t s);

// Sets the message bsa_last_error() returns on this thread.
void set_last_error(const char* msg);
cudaError_t launch_wait_timeout_selftest(unsigned* err, uint64_t limit_ns, cudaStream_t s);

// One query tile per CTA, serial load -> S -> softmax -> PV per kept block (attn.cu).
cudaError_t launch_attention(bool fp8, bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s);

}  // namespace bsa
