/*
 * bsa.h -- C ABI of the B200 (sm_100a) Stem block-sparse prefill library (libbsa.so).
 *
 * The path has three steps, each a call below:
 *   stem_score   OAM block scoring: pooled per-block Q/K representations and one GEMM,
 *                weighted by the key block's mean value norm.
 *                ["腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486), §3.2 输出感知度量（OAM）
 *                 and §二.2.1 Stem算子优化: block-level Q/K representations + one standard GEMM,
 *                 no softmax, no gather.]
 *   stem_select  TPD budget generation fused with per-row top-k selection, emitting compact
 *                ascending KV-block lists per (sequence, query head, query block).
 *                [same page, §3.1 Token位置衰减策略（TPD） and §二.2.1: budget generation and
 *                 selection sort fused into one operator.]
 *   bsa_prefill / bsa_prefill_paged
 *                block-sparse causal prefill attention that loops only over the prebuilt
 *                list; a skipped block contributes exactly nothing (all of its scores are
 *                -inf).  The paged variant reads K/V from a page pool through a page table.
 *                [same page, §二.2.2 BSA算子优化.]
 *   bsa_mask_to_lists / bsa_prefill_mask
 *                the same attention with the selection given as a uint8 block mask per
 *                (sequence, query head), the form HPC-BSA takes it in [same page, §二.2.2].
 *   stem_score_select
 *                stem_score + stem_select in one call without the score matrix [same page,
 *                §二.2.1: no large intermediates].
 *   stem_score_group / bsa_prefill_group / bsa_prefill_paged_group
 *                one list per KV-head group shared by its query heads, and attention that loads
 *                each kept K/V block once for two heads (an extension; the pages say nothing
 *                about grouped-query attention).
 *   bsa_prefill_skip
 *                bsa_prefill with a threshold skip on top of the lists ["BLASST: Dynamic BLocked
 *                Attention Sparsity via Softmax Thresholding", §2.1].
 *
 * Conventions shared by every call:
 *   - All pointers except those marked "host" are device pointers on the current device.
 *     The caller owns every buffer; the library allocates no device memory in these calls.
 *   - Calls are asynchronous on `stream`.  Argument errors are returned synchronously, with
 *     nothing launched, and the message is available from bsa_last_error().  A failed launch
 *     returns BSA_ERR_CUDA.  Errors found by kernels while running (an out-of-range list
 *     entry, an out-of-range page-table entry, an internal wait that ran out of time, a
 *     dynamic shared-memory base without the 1024-byte alignment the attention tiles need) are
 *     recorded in a per-device error word that bsa_check_device_error() reads.
 *   - Tensors are described by bsa_tensor_t: element strides of batch, token and head; the
 *     feature (head_dim) dimension is contiguous; the base pointer and every stride must be
 *     16-byte aligned in bytes.  `scale` is the per-tensor dequantisation scale of FP8 data
 *     (value = code * scale) and is ignored for BF16/FP32.
 *   - Supported shapes: head_dim d in {64, 128}; block in {64, 128}; Hq % Hkv == 0;
 *     query and key lengths are equal (prefill without a prefix); at most 2048 blocks per
 *     sequence.  FP8 attention requires d = 128.  softmax_scale <= 0 means 1/sqrt(d).
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,  /* a null pointer, a bad size, stride or alignment */
    BSA_ERR_UNSUPPORTED = 2,  /* a valid request outside the supported shapes/dtypes */
    BSA_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a launch failed */
    BSA_ERR_WORKSPACE = 4,    /* the workspace is missing or too small */
    BSA_ERR_INVALID_LIST = 5, /* (device) a list entry was outside [0, query block] */
    BSA_ERR_TIMEOUT = 6,      /* (device) an internal pipeline wait ran out of time */
    BSA_ERR_INVALID_PAGE = 7  /* (device) a page-table entry was outside [0, num_pages) */
} bsa_status_t;

typedef enum { BSA_BF16 = 0, BSA_FP8_E4M3 = 1, BSA_FP32 = 2 } bsa_dtype_t;

/* Block metric.  OAM (default): S = tau * Qbar.Kbar + ln(vbar); SAM: S = tau * Qbar.Kbar
 * (attention score only, the prior-art metric); OAM_MUL: S = tau * Qbar.Kbar * vbar. */
typedef enum { BSA_METRIC_OAM = 0, BSA_METRIC_SAM = 1, BSA_METRIC_OAM_MUL = 2 } bsa_metric_t;

typedef struct {
    void* ptr;        /* element [0, 0, 0, 0] */
    int32_t dtype;    /* bsa_dtype_t */
    float scale;      /* FP8 dequantisation scale; ignored otherwise */
    int64_t stride_b; /* elements between batch entries (pages, for a paged cache) */
    int64_t stride_t; /* elements between tokens (slots, for a paged cache) */
    int64_t stride_h; /* elements between heads */
} bsa_tensor_t;

/* TPD budget of one sequence with nb query blocks, computed on the HOST (the same rule the
 * select kernel runs on the device): k_out[i] (host array of nb) receives the number of KV
 * blocks kept by query block i; returns their sum K*, or -1 for invalid arguments.
 * density in (0, 1]; tpd_decay in {0 (uniform), 0.5 (keep ratio ~ (i+1)^-1/2)}.  With
 * k_out = NULL only K* is computed (no per-row budget, O(1)).  Use it to size col_idx
 * (max_k >= K* of every sequence).  [cn486 page, §3.1 TPD.] */
int64_t bsa_tpd_budget(int32_t nb, double density, double tpd_decay, int32_t* k_out);

/* Bytes of device workspace stem_score needs for B sequences of nb blocks. */
size_t bsa_score_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t nb, int32_t d);

/* OAM block scores.  q [B, N, Hq, d], k and v [B, N, Hkv, d] (all the same dtype: BF16,
 * FP8_E4M3 or FP32).  For every (b, query head h, query block i, key block j <= i):
 *     scores[b, h, i, j] = tau * Qbar[b,h,i] . Kbar[b,h/G,j]  (+ ln vbar[b,h/G,j] for OAM)
 * with Qbar/Kbar the means of the block's token vectors (dequantised), vbar the mean L2 norm
 * of the block's value vectors, tau = softmax_scale.  scores is fp32 [B, Hq, nb_stride,
 * nb_stride] (nb_stride >= nb = ceil(N/block)); entries with j > i inside the 128x128 tiles
 * that touch the diagonal are -inf, tiles wholly above it are not written.  The product runs
 * on the tensor cores as three TF32 products (hi*hi + hi*lo + lo*hi of each operand's split),
 * fp32-accurate.  ws: device workspace of at least bsa_score_workspace_bytes() bytes, 256-byte
 * aligned; it receives the pooled means (each split into that TF32 high part and its fp32
 * remainder) and the value norms. */
bsa_status_t stem_score(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N,
                        int32_t Hq, int32_t Hkv, int32_t d, int32_t block, int32_t metric,
                        float softmax_scale, float* scores, int32_t nb_stride, void* ws,
                        size_t ws_bytes, cudaStream_t stream);

/* TPD budget + per-row top-k.  scores as written by stem_score; nb_per_seq (host, B entries)
 * gives each sequence's block count (<= nb_stride).  Outputs:
 *   row_ptr [B, nb_stride + 1] int32: row_ptr[b][i] is the offset of query block i's list
 *           inside col_idx[b][h][...] (identical for every head of a sequence); entries past
 *           nb_b repeat the total.
 *   col_idx [B, Hq, max_k] int32: the list of row (b, h, i) is the sink block 0, the diagonal
 *           block i and the k_i - 2 highest-scoring blocks among 1..i-1 (NaN counts as -inf,
 *           equal scores prefer the smaller index), in ascending order.
 * max_k must be >= the budget total of every sequence (bsa_tpd_budget). */
bsa_status_t stem_select(const float* scores, int32_t B, int32_t Hq, const int32_t* nb_per_seq,
                         int32_t nb_stride, double density, double tpd_decay, int32_t* row_ptr,
                         int32_t* col_idx, int64_t max_k, cudaStream_t stream);

/* Score and select in one call, without the score matrix [cn486 page, §二.2.1 Stem算子优化:
 * budget generation and the selection sort are fused, with no large intermediates].  Computes
 * exactly what stem_score followed by stem_select computes (the same lists, bit for bit: the
 * same per-tile score products and the same per-row selection), for B sequences of N tokens
 * (nb = ceil(N / block) blocks each), without a [B, Hq, nb, nb] score buffer.  The scores of one
 * chunk of KV-head groups of one sequence exist at a time, in `ws` (at most 128 MiB of it, or one
 * group when a group alone is larger), and are consumed by the top-k before the next chunk is
 * scored.  Outputs: row_ptr [B, nb + 1] and col_idx [B, Hq, max_k] as stem_select writes them;
 * max_k >= bsa_tpd_budget(nb, density, tpd_decay, NULL).  ws: at least
 * bsa_score_select_workspace_bytes() bytes, 256-byte aligned.  Arguments and errors otherwise as
 * in stem_score and stem_select; bsa_score_select_workspace_bytes returns 0 for invalid sizes. */
size_t bsa_score_select_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t N, int32_t block,
                                        int32_t d);
bsa_status_t stem_score_select(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N,
                               int32_t Hq, int32_t Hkv, int32_t d, int32_t block, int32_t metric,
                               float softmax_scale, double density, double tpd_decay,
                               int32_t* row_ptr, int32_t* col_idx, int64_t max_k, void* ws,
                               size_t ws_bytes, cudaStream_t stream);

/* Block-sparse causal prefill.  q [B, N, Hq, d]; k, v [B, N, Hkv, d] (BF16, or FP8_E4M3 with
 * per-tensor scales); out [B, N, Hq, d] BF16.  For token t of head h the allowed keys are the
 * tokens s <= t whose block is in the list (row_ptr/col_idx as produced by stem_select, with
 * row_ptr_stride ints per sequence); out = softmax over the allowed keys of
 * softmax_scale * q.k, times v.  lse (nullable) receives fp32 [B, Hq, N] natural-log
 * log-sum-exp of the scaled scores. */
bsa_status_t bsa_prefill(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out,
                         int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d, int32_t block,
                         const int32_t* row_ptr, int32_t row_ptr_stride, const int32_t* col_idx,
                         int64_t max_k, float softmax_scale, float* lse, cudaStream_t stream);

/* bsa_prefill with a threshold skip on top of the lists ["BLASST: Dynamic BLocked Attention
 * Sparsity via Softmax Thresholding" (gist.science), §2.1: skip a block whose local maximum
 * trails the running maximum by more than ln(lambda)].  For each query row the kept blocks are
 * visited in list order with an exact running maximum m of the scaled scores seen so far; a
 * block whose largest scaled score over the row's allowed keys is below m + ln(skip_lambda) is
 * skipped for that row (it contributes nothing; the output is the softmax over the other
 * blocks' keys).  A warp whose 32 rows all skip a block skips its exponentials, and when every
 * row of a query block skips it the P.V product is not issued.  skip_lambda in [0, 1); 0 skips
 * nothing and computes exactly what bsa_prefill computes.  Runs FP8 (d 128, block 128), or BF16
 * with head_dim 64 or block 64 (BSA_ERR_UNSUPPORTED otherwise); arguments, outputs and errors
 * otherwise as in bsa_prefill.  The decisions are taken on fp32 scores, so a block whose max
 * trails by almost exactly ln(skip_lambda) may be decided either way.
 * skip_stats (nullable, device, 8-byte aligned, four uint64 the caller zeroes) is incremented by:
 * [0] (row, kept block) pairs visited, over the rows that are tokens of the sequence; [1] how
 * many of them were skipped; [2] (query block, kept block) pairs; [3] how many of those had
 * every row skip, so that no P.V product was issued.  With skip_lambda = 0 it is not touched. */
bsa_status_t bsa_prefill_skip(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out,
                              int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                              int32_t block, const int32_t* row_ptr, int32_t row_ptr_stride,
                              const int32_t* col_idx, int64_t max_k, float softmax_scale,
                              double skip_lambda, float* lse, unsigned long long* skip_stats,
                              cudaStream_t stream);

/* Group-shared selection with GQA-packed attention.  The pages select per query head and say
 * nothing about grouped-query attention.  This extension gives the G = Hq / Hkv query heads of
 * a KV-head group one kept-block list, so that the heads sharing a list can share every K/V
 * load [a reading of cn486 page, §二.2.2 BSA算子优化: the list is built before the inner loop,
 * which then only visits valid blocks].
 *
 * stem_score_group: stem_score with one score row per KV-head group.  The query-side
 * representation is the mean over the group's G heads of their pooled Q:
 *     scores[b, hk, i, j] = tau * Gbar[b,hk,i] . Kbar[b,hk,j]  (+ ln vbar[b,hk,j] for OAM),
 *     Gbar[b,hk,i] = (1/G) * sum over the heads h of group hk of Qbar[b,h,i],
 * which is the mean of the G heads' stem_score rows (every metric is linear in Qbar).
 * scores is fp32 [B, Hkv, nb_stride, nb_stride]; ws needs bsa_score_group_workspace_bytes()
 * bytes, 256-byte aligned.  Arguments and errors otherwise as in stem_score.  stem_select then
 * runs on these scores with Hq := Hkv and writes col_idx [B, Hkv, max_k].
 *
 * bsa_prefill_group: bsa_prefill whose col_idx is [B, Hkv, max_k], one list per KV-head group,
 * shared by the group's query heads (row_ptr as stem_select writes it).  FP8 at d = 128, block
 * 128, with G even, runs the GQA-packed kernel: one CTA serves two query heads of a group for a
 * query block and loads each kept K/V block once for both.  Every other shape runs the per-head
 * kernel on the shared lists.  Arguments, outputs and errors otherwise as in bsa_prefill.
 * bsa_score_group_workspace_bytes returns 0 for invalid sizes. */
size_t bsa_score_group_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t nb, int32_t d);
bsa_status_t stem_score_group(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N,
                              int32_t Hq, int32_t Hkv, int32_t d, int32_t block, int32_t metric,
                              float softmax_scale, float* scores, int32_t nb_stride, void* ws,
                              size_t ws_bytes, cudaStream_t stream);
bsa_status_t bsa_prefill_group(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out,
                               int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                               int32_t block, const int32_t* row_ptr, int32_t row_ptr_stride,
                               const int32_t* col_idx, int64_t max_k, float softmax_scale,
                               float* lse, cudaStream_t stream);

/* Block-mask input [cn486 page, §二.2.2 BSA算子优化: the sparse kernel receives the selection
 * as a block mask and derives the kept-block list from it before its inner loop].
 * block_mask (device, uint8) is [B, Hq, nb, mask_stride] with nb = ceil(N / block): row
 * (b, h, i) keeps block j <= i iff block_mask[b][h][i][j] != 0; entries above the diagonal
 * are ignored.  mask_stride >= nb and a multiple of 16; block_mask 16-byte aligned.
 *
 * bsa_mask_to_lists writes the per-head lists: row_ptr [B*Hq][nb+1] (offsets into the
 * (b, h) row of col_idx) and col_idx [B*Hq][max_k], max_k >= nb(nb+1)/2, kept blocks in
 * ascending order.  An empty row is an empty list.  Errors: a null, misaligned or
 * badly strided mask, max_k < nb(nb+1)/2 or null lists -> BSA_ERR_INVALID_ARG; nb outside
 * [1, 2048] or a row grid past the launch limit -> BSA_ERR_UNSUPPORTED; nothing launched.
 *
 * bsa_prefill_mask runs bsa_mask_to_lists into `ws` (bsa_mask_workspace_bytes(B, Hq, nb)
 * bytes, 256-byte aligned) and then the bsa_prefill kernel on those lists; arguments and
 * outputs otherwise as in bsa_prefill.  A query block whose mask row keeps nothing has
 * out = 0 and lse = -inf for its tokens.  A missing, misaligned (256 bytes) or short
 * workspace -> BSA_ERR_WORKSPACE; the mask and tensor checks as above and in bsa_prefill.
 * bsa_mask_workspace_bytes returns 0 for invalid sizes. */
size_t bsa_mask_workspace_bytes(int32_t B, int32_t Hq, int32_t nb);
bsa_status_t bsa_mask_to_lists(const uint8_t* block_mask, int64_t mask_stride, int32_t B,
                               int32_t Hq, int32_t nb, int32_t* row_ptr, int32_t* col_idx,
                               int64_t max_k, cudaStream_t stream);
bsa_status_t bsa_prefill_mask(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, bsa_tensor_t out,
                              int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                              int32_t block, const uint8_t* block_mask, int64_t mask_stride,
                              float softmax_scale, float* lse, void* ws, size_t ws_bytes,
                              cudaStream_t stream);

/* Debug check of a kept-block list set, for lists that did not come from this library (or
 * were edited).  row_ptr entries of (b, h) start at b * row_ptr_stride + h *
 * row_ptr_head_stride (head stride 0: one row_ptr for all heads, as stem_select writes;
 * nb + 1 with row_ptr_stride Hq * (nb + 1): bsa_mask_to_lists's layout); col_idx is
 * [B, Hq, max_k]; nb_per_seq (host, B entries) gives each sequence's block count.  Checks
 * every row (b, h, i): 0 <= row_ptr[i] <= row_ptr[i + 1] <= max_k, at most i + 1 entries
 * (at least one unless allow_empty), entries strictly ascending within [0, i].  A violation
 * is recorded in the device error word: bsa_check_device_error then returns
 * BSA_ERR_INVALID_LIST.  Argument errors are returned synchronously (INVALID_ARG for null
 * pointers, max_k < 1 or strides too small; UNSUPPORTED for B or nb out of range). */
bsa_status_t bsa_validate_lists(const int32_t* row_ptr, int64_t row_ptr_stride,
                                int64_t row_ptr_head_stride, const int32_t* col_idx,
                                int64_t max_k, int32_t B, int32_t Hq, const int32_t* nb_per_seq,
                                int32_t allow_empty, cudaStream_t stream);

/* Paged-KV variant.  q and out are packed varlen [sum N_b, Hq, d] (stride_b unused);
 * cu_seqlens (device, B+1) gives each sequence's first token; seqlens_host (host, B) its
 * length.  k_cache/v_cache are page pools [num_pages, page_size, Hkv, d] described with
 * stride_b = page stride and stride_t = slot stride; page_table [B, max_pages] int32 maps a
 * sequence's logical page p (tokens p*page_size ...) to a physical page.  page_size must be
 * 64 and divide `block`.  Lists and lse ([B, Hq, max_b N_b]) as in bsa_prefill.  A page entry
 * outside [0, num_pages) for a page that holds tokens of the sequence is read as zeros and
 * recorded (bsa_check_device_error then returns BSA_ERR_INVALID_PAGE). */
bsa_status_t bsa_prefill_paged(bsa_tensor_t q, bsa_tensor_t out, const int32_t* cu_seqlens,
                               const int32_t* seqlens_host, int32_t B, bsa_tensor_t k_cache,
                               bsa_tensor_t v_cache, int32_t num_pages, int32_t page_size,
                               const int32_t* page_table, int32_t max_pages, int32_t Hq,
                               int32_t Hkv, int32_t d, int32_t block, const int32_t* row_ptr,
                               int32_t row_ptr_stride, const int32_t* col_idx, int64_t max_k,
                               float softmax_scale, float* lse, cudaStream_t stream);

/* bsa_prefill_paged with group-shared lists: col_idx is [B, Hkv, max_k], one list per KV-head
 * group shared by the group's query heads (row_ptr [B, row_ptr_stride] as stem_select writes
 * it for stem_score_group's scores).  FP8 at d = 128, block 128, with G even, runs the
 * GQA-packed kernel of bsa_prefill_group on the page pool: one CTA serves two query heads of
 * a group for a query block and loads each kept block's pages once for both.  Every other
 * shape runs the per-head paged kernel on the shared lists.  Arguments, page rules, outputs
 * and errors otherwise as in bsa_prefill_paged.  (An extension: the pages select per query
 * head and say nothing about grouped-query attention.) */
bsa_status_t bsa_prefill_paged_group(bsa_tensor_t q, bsa_tensor_t out, const int32_t* cu_seqlens,
                                     const int32_t* seqlens_host, int32_t B, bsa_tensor_t k_cache,
                                     bsa_tensor_t v_cache, int32_t num_pages, int32_t page_size,
                                     const int32_t* page_table, int32_t max_pages, int32_t Hq,
                                     int32_t Hkv, int32_t d, int32_t block, const int32_t* row_ptr,
                                     int32_t row_ptr_stride, const int32_t* col_idx, int64_t max_k,
                                     float softmax_scale, float* lse, cudaStream_t stream);

/* stem_score without a workspace argument, for callers that cannot allocate device memory:
 * for example a plain C host program that links only this library and has no device
 * allocator of its own, or a serving runtime whose memory pool owns all of HBM and does not
 * let a library call cudaMalloc (which would also synchronise the device mid-stream).  It
 * has no counterpart on the Stem pages; it is a deployment convenience.
 *
 * Arguments, layouts, results and errors are those of stem_score.  The pooled Q/K
 * representations and value norms that stem_score keeps in `ws` live instead in a fixed
 * 32 MiB array inside the library, which every GPU that loads the library holds until the
 * process exits.  Problems that need more than that (bsa_score_workspace_bytes() > 32 MiB,
 * e.g. beyond about 58K tokens at 64 query / 8 KV heads, d = 128, block 128) are rejected
 * with BSA_ERR_UNSUPPORTED and a message naming both sizes; nothing is launched.  The call
 * itself allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on each device looks up the array's device address (with that device
 *     current) and caches it; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.  Nothing in it has
 *     to start at zero: every call rewrites all of the scratch it reads.  Calls whose work
 *     overlaps on the GPU (other streams, or other host threads on the same device) race on
 *     the array and must be serialised by the caller. */
bsa_status_t stem_score_noalloc(bsa_tensor_t q, bsa_tensor_t k, bsa_tensor_t v, int32_t B, int32_t N,
                                int32_t Hq, int32_t Hkv, int32_t d, int32_t block, int32_t metric,
                                float softmax_scale, float* scores, int32_t nb_stride,
                                cudaStream_t stream);

/* Self-test of the failure path that every pipeline wait in the library shares.  It has no
 * counterpart on the Stem pages; it exists so that the timeout handling can be checked on a
 * real GPU without faulting or hanging it.  Launches one CTA on `stream` that allocates tensor
 * memory, waits on an mbarrier that nothing ever arrives at, gives up after limit_ns
 * nanoseconds (1e3 <= limit_ns <= 1e9, else BSA_ERR_INVALID_ARG and nothing is launched),
 * records BSA_ERR_TIMEOUT in the current device's error word, frees its tensor memory and
 * exits.  Returns BSA_OK once launched; a following bsa_check_device_error() returns
 * BSA_ERR_TIMEOUT (and clears the word), and the context stays usable. */
bsa_status_t bsa_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

/* Message of the last error returned on the calling thread ("" if none). */
const char* bsa_last_error(void);

/* Synchronises `stream`, then reads and clears the current device's error word: returns
 * BSA_ERR_TIMEOUT, BSA_ERR_INVALID_LIST, BSA_ERR_CUDA (an attention kernel found its dynamic
 * shared memory not 1024-byte aligned and did nothing) or BSA_ERR_INVALID_PAGE if a kernel
 * recorded one (in that order of precedence), else BSA_OK. */
bsa_status_t bsa_check_device_error(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
