/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the Stem block-sparse prefill path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this
 * file: only tests/, the smoke check in __graft_entry__.py and the CPU-baseline leg of
 * bench.py use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (page title, then section):
 *   [P1] "腾讯混元Stem稀疏注意力算法：长文推理加速新SOTA" (cn486.com):
 *        §3.1 Token位置衰减策略（TPD）, §3.2 输出感知度量（OAM）,
 *        §二.2.1 Stem算子优化 (pooled block representations + one GEMM; fused budget+sort),
 *        §二.2.2 BSA算子优化 (skipped block == all scores -inf).
 *   [P5] "BLASST: Dynamic BLocked Attention Sparsity via Softmax Thresholding" (gist.science):
 *        §2.1 (skip a block whose local max trails the running max by more than ln(lambda)).
 *   [P4] "Tencent Hunyuan introduces Stem sparse attention algorithm" (setupai.cc):
 *        "Technical Deep Dive" (TPD: position-dependent top-k, more budget to early
 *        positions; OAM: approximate output magnitude using value information).
 * The pages lost the OAM and TPD formulas in extraction; the readings used here are:
 *   - OAM score  S_ij = tau * (Qbar_i . Kbar_j) + ln(vbar_j)   (log of e^score * amplitude)
 *   - SAM score  S_ij = tau * (Qbar_i . Kbar_j)
 *   - OAM_MUL    S_ij = tau * (Qbar_i . Kbar_j) * vbar_j       (literal product, kept as option)
 *   - TPD budget k_i proportional to (i+1)^(1-beta) blocks (keep ratio ~ (i+1)^-beta),
 *     normalised so that sum k_i = round(density * causal block count); sink block 0 and
 *     the diagonal block are always kept.
 *
 * Parity status of each function (what pins it, in tests/test_oracle_pins.py):
 *   orc_decode_*        pinned: exhaustive against torch's casts (all codes).
 *   orc_pool_mean       pinned: brute-force mean of all token-pair logits == pooled score.
 *   orc_pool_vnorm      pinned: closed forms (constant rows, one-hot rows).
 *   orc_score           pinned: the pooled-GEMM equivalence above; -inf above the diagonal.
 *   orc_group_mean      pinned: the group's score rows equal the mean of its heads' score rows
 *                       (every metric is linear in the pooled query), and the brute-force mean
 *                       over the group's heads and all token pairs; G = 1 is the identity.
 *   orc_tpd_budget      invariants pinned (sum, bounds, monotone keep ratio, density 1,
 *                       beta 0 uniform, hand-worked fixture).  The decay LAW itself is a
 *                       reading of the pages: parity unpinned.
 *   orc_select          pinned: brute-force full sort; kept scores dominate dropped ones.
 *   orc_attention_rows  pinned: density 1 == library dense causal SDPA (fp64); skipped
 *                       blocks' contents are irrelevant; single-key closed form.  Its amp
 *                       output == library SDPA with |V| as the values; single key: |v|.
 *   orc_attention_rows_skip  pinned: lambda = 0 gives orc_attention_rows exactly; a block whose
 *                       max trails by more / less than ln(lambda) is skipped / kept (closed
 *                       form); with its skip decisions, == library SDPA under the per-row mask.
 *   orc_attention_rows_mask  pinned: an all-ones mask == library dense causal SDPA; a
 *                       diagonal-only mask == library SDPA over the block's own keys; an
 *                       empty row gives 0 / -inf; entries above the diagonal are ignored.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <omp.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2
#define ORC_F64 3

#define ORC_METRIC_OAM 0
#define ORC_METRIC_SAM 1
#define ORC_METRIC_OAM_MUL 2

/* A strided [B, N, H, D] view; the last (feature) dimension is contiguous.
 * Every decoded element is multiplied by `scale` (the per-tensor FP8 scale; 1 otherwise). */
typedef struct {
    const void* data;
    int32_t dtype;
    int32_t pad_;
    double scale;
    int64_t sb, st, sh; /* element strides of batch, token, head */
} orc_tensor;

/* ---------------------------------------------------------------- element decoding */

/* bf16 is the top half of an IEEE binary32 word. */
double orc_decode_bf16(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; exponent field 0 is subnormal (m/8 * 2^-6). */
double orc_decode_e4m3(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(8.0 + (double)m, e - 10);
    return sign ? -mag : mag;
}

static double load_elem(const orc_tensor* x, int64_t b, int64_t t, int64_t h, int64_t c) {
    int64_t off = b * x->sb + t * x->st + h * x->sh + c;
    double v;
    switch (x->dtype) {
        case ORC_F32: v = (double)((const float*)x->data)[off]; break;
        case ORC_BF16: v = orc_decode_bf16(((const uint16_t*)x->data)[off]); break;
        case ORC_E4M3: v = orc_decode_e4m3(((const uint8_t*)x->data)[off]); break;
        default: v = ((const double*)x->data)[off]; break;
    }
    return v * x->scale;
}

void orc_decode_tensor(const orc_tensor* x, int64_t B, int64_t N, int64_t H, int64_t D,
                       double* out /* [B][N][H][D] */) {
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < N; ++t)
            for (int64_t h = 0; h < H; ++h)
                for (int64_t c = 0; c < D; ++c)
                    out[((b * N + t) * H + h) * D + c] = load_elem(x, b, t, h, c);
}

/* ---------------------------------------------------------------- a1: pooling */

/* Qbar / Kbar: per (batch, head, block) mean of the block's token vectors.  A partial last
 * block averages its valid tokens only.  [P1 §二.2.1: compact block-level Q and K
 * representations computed before the score GEMM.] */
void orc_pool_mean(const orc_tensor* x, int B, int N, int H, int D, int bs,
                   double* out /* [B][H][nb][D] */) {
    int nb = (N + bs - 1) / bs;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < nb; ++i) {
                int lo = i * bs, hi = (i + 1) * bs < N ? (i + 1) * bs : N;
                for (int c = 0; c < D; ++c) {
                    double acc = 0.0;
                    for (int t = lo; t < hi; ++t) acc += load_elem(x, b, t, h, c);
                    out[(((int64_t)b * H + h) * nb + i) * D + c] = acc / (double)(hi - lo);
                }
            }
}

/* vbar: per (batch, kv head, block) mean over the block's tokens of the L2 norm of the
 * value vector -- the "value amplitude" that OAM weights by.  [P1 §3.2; P4 Technical Deep
 * Dive, OAM bullet.] */
void orc_pool_vnorm(const orc_tensor* v, int B, int N, int H, int D, int bs,
                    double* out /* [B][H][nb] */) {
    int nb = (N + bs - 1) / bs;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < nb; ++i) {
                int lo = i * bs, hi = (i + 1) * bs < N ? (i + 1) * bs : N;
                double acc = 0.0;
                for (int t = lo; t < hi; ++t) {
                    double ss = 0.0;
                    for (int c = 0; c < D; ++c) {
                        double e = load_elem(v, b, t, h, c);
                        ss += e * e;
                    }
                    acc += sqrt(ss);
                }
                out[((int64_t)b * H + h) * nb + i] = acc / (double)(hi - lo);
            }
}

/* ---------------------------------------------------------------- a2: block scores */

/* S[b,h,i,j] for the causal block grid; j > i is -inf.  Query head h reads the pooled keys
 * of kv head h / (Hq/Hkv).  [P1 §3.2 and §二.2.1: additive metric, no softmax, no gather;
 * one GEMM of the pooled representations gives every block score.] */
void orc_score(const double* qbar /* [B][Hq][nb][D] */, const double* kbar /* [B][Hkv][nb][D] */,
               const double* vbar /* [B][Hkv][nb] */, int B, int Hq, int Hkv, int nb, int D,
               double tau, int metric, double* S /* [B][Hq][nb][nb] */) {
    int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            for (int i = 0; i < nb; ++i)
                for (int j = 0; j < nb; ++j) {
                    double* dst = &S[(((int64_t)b * Hq + h) * nb + i) * nb + j];
                    if (j > i) {
                        *dst = -INFINITY;
                        continue;
                    }
                    const double* qv = &qbar[(((int64_t)b * Hq + h) * nb + i) * D];
                    const double* kv = &kbar[(((int64_t)b * Hkv + hk) * nb + j) * D];
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];
                    double s = tau * dot;
                    double amp = vbar[((int64_t)b * Hkv + hk) * nb + j];
                    if (metric == ORC_METRIC_OAM)
                        s = s + log(amp); /* log(0) = -inf: a zero-amplitude block never wins */
                    else if (metric == ORC_METRIC_OAM_MUL)
                        s = s * amp;
                    *dst = s;
                }
        }
}

/* Group-shared selection (an extension: the pages select per query head and say nothing about
 * grouped-query attention).  The query-side representation of KV-head group hk is the mean of
 * its G = Hq / Hkv query heads' pooled Q:  gbar[b,hk,i,:] = (1/G) sum_{g<G} qbar[b, hk*G+g, i, :].
 * orc_score on gbar (with Hq := Hkv) then gives the group's score rows. */
void orc_group_mean(const double* qbar /* [B][Hq][nb][D] */, int B, int Hq, int Hkv, int nb, int D,
                    double* gbar /* [B][Hkv][nb][D] */) {
    int G = Hq / Hkv;
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int i = 0; i < nb; ++i)
                for (int c = 0; c < D; ++c) {
                    double acc = 0.0;
                    for (int g = 0; g < G; ++g) acc += qbar[(((int64_t)b * Hq + hk * G + g) * nb + i) * D + c];
                    gbar[(((int64_t)b * Hkv + hk) * nb + i) * D + c] = acc / G;
                }
}

/* ---------------------------------------------------------------- a3: TPD budget */

typedef struct {
    uint32_t frac;
    int32_t row;
} orc_rem;

static int rem_cmp(const void* a, const void* b) {
    const orc_rem* x = (const orc_rem*)a;
    const orc_rem* y = (const orc_rem*)b;
    if (x->frac != y->frac) return x->frac > y->frac ? -1 : 1; /* larger fraction first */
    return x->row < y->row ? -1 : (x->row > y->row ? 1 : 0);    /* then the earlier row */
}

/* Token Position Decay budget for a causal grid of nb query blocks.  [P1 §3.1: TPD
 * re-distributes a fixed budget and does not raise it; P4 Technical Deep Dive: a
 * position-dependent top-k that gives initial positions a larger share.]
 *
 * Row i has n_i = i+1 causal blocks and must keep m_i blocks (1 for row 0, else the sink
 * block 0 and the diagonal block).  The total is K* = round(density * sum n_i), clamped to
 * [sum m_i, sum n_i].  The real-valued share of row i is
 *     t_i(c) = min(n_i, max(m_i, c * n_i^(1-beta))),
 * i.e. a keep ratio decaying like (i+1)^-beta.  The constant c is found by 64 bisection
 * steps on [0, nb] against the fixed-point total sum floor(t_i(c) * 2^32) >= K* * 2^32;
 * whole blocks are floor(t_i), and the R = K* - sum floor(t_i) leftover blocks go to the rows
 * with the largest fractional parts (earlier row first on ties) that are not full yet.
 * Only beta = 0 (uniform) and beta = 1/2 are accepted: for them n^(1-beta) is exact or a
 * correctly rounded sqrt.  Returns K*, or -1 for invalid arguments. */
int64_t orc_tpd_budget(int32_t nb, double density, double beta, int32_t* k_out) {
    if (nb <= 0 || nb > 32768 || !(density > 0.0) || !(density <= 1.0)) return -1;
    if (!(beta == 0.0 || beta == 0.5)) return -1;
    int64_t T = (int64_t)nb * (nb + 1) / 2;
    int64_t sum_m = 2 * (int64_t)nb - 1;
    double kd = floor(density * (double)T + 0.5);
    int64_t Kstar = (int64_t)kd;
    if (Kstar < sum_m) Kstar = sum_m;
    if (Kstar > T) Kstar = T;

    double* w = (double*)malloc(sizeof(double) * nb);
    int64_t* F = (int64_t*)malloc(sizeof(int64_t) * nb);
    orc_rem* rem = (orc_rem*)malloc(sizeof(orc_rem) * nb);
    for (int i = 0; i < nb; ++i) w[i] = beta == 0.5 ? sqrt((double)(i + 1)) : (double)(i + 1);

    const double two32 = 4294967296.0;
    const int64_t target = Kstar * ((int64_t)1 << 32);
    double lo = 0.0, hi = (double)nb;
    for (int it = 0; it < 64; ++it) {
        double mid = (lo + hi) * 0.5;
        int64_t total = 0;
        for (int i = 0; i < nb; ++i) {
            double n = (double)(i + 1), m = i == 0 ? 1.0 : 2.0;
            double t = mid * w[i];
            if (t < m) t = m;
            if (t > n) t = n;
            total += (int64_t)floor(t * two32);
        }
        if (total >= target)
            hi = mid;
        else
            lo = mid;
    }
    int64_t whole = 0;
    int nrem = 0;
    for (int i = 0; i < nb; ++i) {
        double n = (double)(i + 1), m = i == 0 ? 1.0 : 2.0;
        double t = hi * w[i];
        if (t < m) t = m;
        if (t > n) t = n;
        F[i] = (int64_t)floor(t * two32);
        k_out[i] = (int32_t)(F[i] >> 32);
        whole += k_out[i];
        if (k_out[i] < i + 1) {
            rem[nrem].frac = (uint32_t)(F[i] & 0xFFFFFFFFll);
            rem[nrem].row = i;
            ++nrem;
        }
    }
    int64_t R = Kstar - whole;
    qsort(rem, nrem, sizeof(orc_rem), rem_cmp);
    for (int64_t r = 0; r < R && r < nrem; ++r) k_out[rem[r].row] += 1;
    free(w);
    free(F);
    free(rem);
    return Kstar;
}

/* ---------------------------------------------------------------- a4: per-row top-k */

typedef struct {
    double s;
    int32_t j;
} orc_cand;

static int cand_cmp(const void* a, const void* b) {
    const orc_cand* x = (const orc_cand*)a;
    const orc_cand* y = (const orc_cand*)b;
    if (x->s > y->s) return -1; /* higher score first */
    if (x->s < y->s) return 1;
    return x->j < y->j ? -1 : (x->j > y->j ? 1 : 0); /* equal scores: smaller j first */
}

static int int_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return x < y ? -1 : (x > y ? 1 : 0);
}

/* Keep list of query block i: the sink block 0 and the diagonal block i, plus the k_i - 2
 * best-scoring blocks among 1..i-1 (NaN scores count as -inf; equal scores prefer the
 * smaller j), returned in ascending order.  Row 0 keeps only block 0.  [P1 §3.2 selection
 * by the metric within the budget.  Keeping the sink block 0 and the diagonal block in every
 * row is a reading: the pages do not print the rule.] */
void orc_select_row(const double* srow /* S[i][0..i] */, int32_t i, int32_t k_i, int32_t* out) {
    if (i == 0) {
        out[0] = 0;
        return;
    }
    int32_t n_c = i - 1;
    orc_cand* c = (orc_cand*)malloc(sizeof(orc_cand) * (n_c > 0 ? n_c : 1));
    for (int32_t j = 1; j < i; ++j) {
        double s = srow[j];
        c[j - 1].s = isnan(s) ? -INFINITY : s;
        c[j - 1].j = j;
    }
    qsort(c, n_c, sizeof(orc_cand), cand_cmp);
    int32_t take = k_i - 2, n = 0;
    out[n++] = 0;
    for (int32_t r = 0; r < take; ++r) out[n++] = c[r].j;
    out[n++] = i;
    qsort(out, n, sizeof(int32_t), int_cmp);
    free(c);
}

/* Budget + selection for a batch of causal score matrices.  row_ptr[b][i] is the offset of
 * row i's list inside col_idx[b][h][*] (the same for every head of sequence b, since the
 * budget depends only on nb_b); col_idx has maxK entries per (b, h).  Returns 0 on success. */
int orc_select(const double* S /* [B][Hq][nbs][nbs] */, int B, int Hq, const int32_t* nb_per_seq,
               int nbs, double density, double beta, int32_t* row_ptr /* [B][nbs+1] */,
               int32_t* col_idx /* [B][Hq][maxK] */, int64_t maxK) {
    for (int b = 0; b < B; ++b) {
        int nb = nb_per_seq[b];
        if (nb > nbs) return -1;
        int32_t* k = (int32_t*)malloc(sizeof(int32_t) * nb);
        int64_t tot = orc_tpd_budget(nb, density, beta, k);
        if (tot < 0 || tot > maxK) {
            free(k);
            return -1;
        }
        int32_t* rp = &row_ptr[(int64_t)b * (nbs + 1)];
        rp[0] = 0;
        for (int i = 0; i < nb; ++i) rp[i + 1] = rp[i] + k[i];
        for (int i = nb; i < nbs; ++i) rp[i + 1] = rp[nb];
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
        for (int h = 0; h < Hq; ++h)
            for (int i = 0; i < nb; ++i) {
                const double* srow = &S[(((int64_t)b * Hq + h) * nbs + i) * nbs];
                orc_select_row(srow, i, k[i], &col_idx[((int64_t)b * Hq + h) * maxK + rp[i]]);
            }
        free(k);
    }
    return 0;
}

/* ---------------------------------------------------------------- a5: attention */

/* Output and log-sum-exp of individual query rows under the block-sparse causal mask.
 * For query token t of head h: the allowed keys are A(t) = {s <= t : block(s) is in the
 * keep list of (b, h, block(t))}; every other key has score -inf, so
 *     O = sum_{s in A(t)} softmax_s(tau * q_t . k_s) v_s,   lse = ln sum_{s in A(t)} e^{tau q.k}.
 * [P1 §二.2.2: a skipped block is mathematically a block of -inf scores, so softmax is exact.]
 * rows holds n_rows triples (b, h, t).  The mask is built explicitly per row.
 * amp (if not NULL) receives, per output element, the same softmax average of |v_s|:
 *     amp = sum_{s in A(t)} softmax_s(tau * q_t . k_s) |v_s|,
 * the magnitude a rounding of each weight by a relative eps can move O by at most eps * amp
 * (used by the tests to bound the rounding of the weights to a 16-bit operand type). */
void orc_attention_rows(const orc_tensor* q, const orc_tensor* k, const orc_tensor* v, int N,
                        int Hq, int Hkv, int D, int bs, const int32_t* row_ptr, int rp_stride,
                        const int32_t* col_idx, int64_t maxK, double tau, const int64_t* rows,
                        int64_t n_rows, double* out /* [n_rows][D] */, double* lse /* [n_rows] */,
                        double* amp /* nullable [n_rows][D] */) {
    int G = Hq / Hkv;
#pragma omp parallel
    {
        unsigned char* allowed = (unsigned char*)malloc((size_t)N);
        double* logit = (double*)malloc(sizeof(double) * (size_t)N);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            int64_t hk = h / G;
            int64_t i = t / bs;
            const int32_t* rp = &row_ptr[b * rp_stride];
            const int32_t* list = &col_idx[(b * Hq + h) * maxK + rp[i]];
            int32_t len = rp[i + 1] - rp[i];
            memset(allowed, 0, (size_t)N);
            for (int32_t n = 0; n < len; ++n) {
                int64_t j = list[n];
                for (int64_t s = j * bs; s < (j + 1) * bs && s < N; ++s)
                    if (s <= t) allowed[s] = 1;
            }
            for (int c = 0; c < D; ++c) qrow[c] = load_elem(q, b, t, h, c);
            double m = -INFINITY;
            for (int64_t s = 0; s < N; ++s) {
                if (!allowed[s]) {
                    logit[s] = -INFINITY;
                    continue;
                }
                double dot = 0.0;
                for (int c = 0; c < D; ++c) dot += qrow[c] * load_elem(k, b, s, hk, c);
                logit[s] = tau * dot;
                if (logit[s] > m) m = logit[s];
            }
            double z = 0.0;
            double* o = &out[r * D];
            double* a = amp ? &amp[r * D] : NULL;
            for (int c = 0; c < D; ++c) o[c] = 0.0;
            if (a)
                for (int c = 0; c < D; ++c) a[c] = 0.0;
            for (int64_t s = 0; s < N; ++s) {
                if (!allowed[s]) continue;
                double w = exp(logit[s] - m);
                z += w;
                for (int c = 0; c < D; ++c) o[c] += w * load_elem(v, b, s, hk, c);
                if (a)
                    for (int c = 0; c < D; ++c) a[c] += w * fabs(load_elem(v, b, s, hk, c));
            }
            for (int c = 0; c < D; ++c) o[c] /= z;
            if (a)
                for (int c = 0; c < D; ++c) a[c] /= z;
            if (lse) lse[r] = m + log(z);
        }
        free(allowed);
        free(logit);
        free(qrow);
    }
}

/* Attention with the threshold skip of [P5] ("BLASST: Dynamic BLocked Attention Sparsity via
 * Softmax Thresholding", §2.1 基于运行最大值的剪枝) on top of the kept-block lists.  For query
 * token t the list's blocks are visited in stored order while a running maximum m of the logits
 * seen so far is kept: for block j, with m~ the largest logit tau * q_t . k_s over its allowed
 * keys s <= t, the block is skipped when m is finite and m~ - m < ln(lambda); otherwise its keys
 * join the softmax and m = max(m, m~).  A skipped block contributes nothing.  O and lse are
 * those of the softmax over the keys of the blocks that were not skipped.  skipped (nullable)
 * receives, per row, the number of list blocks skipped.  ln_lambda = -inf skips nothing. */
void orc_attention_rows_skip(const orc_tensor* q, const orc_tensor* k, const orc_tensor* v, int N,
                             int Hq, int Hkv, int D, int bs, const int32_t* row_ptr, int rp_stride,
                             const int32_t* col_idx, int64_t maxK, double tau, double ln_lambda,
                             const int64_t* rows, int64_t n_rows, double* out /* [n_rows][D] */,
                             double* lse /* [n_rows] */, int32_t* skipped /* nullable [n_rows] */) {
    int G = Hq / Hkv;
#pragma omp parallel
    {
        unsigned char* allowed = (unsigned char*)malloc((size_t)N);
        double* logit = (double*)malloc(sizeof(double) * (size_t)N);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            int64_t hk = h / G;
            int64_t i = t / bs;
            const int32_t* rp = &row_ptr[b * rp_stride];
            const int32_t* list = &col_idx[(b * Hq + h) * maxK + rp[i]];
            int32_t len = rp[i + 1] - rp[i];
            for (int c = 0; c < D; ++c) qrow[c] = load_elem(q, b, t, h, c);
            memset(allowed, 0, (size_t)N);
            double m = -INFINITY;
            int32_t n_skip = 0;
            for (int32_t n = 0; n < len; ++n) {
                int64_t j = list[n];
                double mb = -INFINITY;
                for (int64_t s = j * bs; s < (j + 1) * bs && s < N && s <= t; ++s) {
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qrow[c] * load_elem(k, b, s, hk, c);
                    logit[s] = tau * dot;
                    if (logit[s] > mb) mb = logit[s];
                }
                if (m > -INFINITY && mb - m < ln_lambda) {
                    ++n_skip;
                    continue;
                }
                for (int64_t s = j * bs; s < (j + 1) * bs && s < N && s <= t; ++s) allowed[s] = 1;
                if (mb > m) m = mb;
            }
            double z = 0.0;
            double* o = &out[r * D];
            for (int c = 0; c < D; ++c) o[c] = 0.0;
            for (int64_t s = 0; s <= t; ++s) {
                if (!allowed[s]) continue;
                double w = exp(logit[s] - m);
                z += w;
                for (int c = 0; c < D; ++c) o[c] += w * load_elem(v, b, s, hk, c);
            }
            for (int c = 0; c < D; ++c) o[c] /= z;
            if (lse) lse[r] = m + log(z);
            if (skipped) skipped[r] = n_skip;
        }
        free(allowed);
        free(logit);
        free(qrow);
    }
}

/* The same attention with the selection given as a block mask instead of lists
 * [P1 §二.2.2: HPC-BSA receives the selection as a block mask; a skipped block is a block of
 * -inf scores].  mask is [B][Hq][nb][mask_stride] bytes; the allowed keys of query token t
 * (block i) of head h are A(t) = {s <= t : mask[b][h][i][block(s)] != 0}.  A row with A(t)
 * empty has no softmax; its output is taken as O = 0 and lse = -inf (the convention of
 * softmax over an empty set used by attention kernels).  The mask is read per key.
 * amp as in orc_attention_rows (0 for an empty row). */
void orc_attention_rows_mask(const orc_tensor* q, const orc_tensor* k, const orc_tensor* v, int N,
                             int Hq, int Hkv, int D, int bs, const uint8_t* mask, int64_t mask_stride,
                             double tau, const int64_t* rows, int64_t n_rows, double* out /* [n_rows][D] */,
                             double* lse /* [n_rows] */, double* amp /* nullable [n_rows][D] */) {
    int G = Hq / Hkv;
    int64_t nb = (N + bs - 1) / bs;
#pragma omp parallel
    {
        double* logit = (double*)malloc(sizeof(double) * (size_t)N);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            int64_t hk = h / G;
            const uint8_t* mrow = &mask[((b * Hq + h) * nb + t / bs) * mask_stride];
            for (int c = 0; c < D; ++c) qrow[c] = load_elem(q, b, t, h, c);
            double m = -INFINITY;
            int any = 0;
            for (int64_t s = 0; s <= t; ++s) {
                if (mrow[s / bs] == 0) continue;
                double dot = 0.0;
                for (int c = 0; c < D; ++c) dot += qrow[c] * load_elem(k, b, s, hk, c);
                logit[s] = tau * dot;
                if (logit[s] > m) m = logit[s];
                any = 1;
            }
            double* o = &out[r * D];
            double* a = amp ? &amp[r * D] : NULL;
            for (int c = 0; c < D; ++c) o[c] = 0.0;
            if (a)
                for (int c = 0; c < D; ++c) a[c] = 0.0;
            if (!any) {
                if (lse) lse[r] = -INFINITY;
                continue;
            }
            double z = 0.0;
            for (int64_t s = 0; s <= t; ++s) {
                if (mrow[s / bs] == 0) continue;
                double w = exp(logit[s] - m);
                z += w;
                for (int c = 0; c < D; ++c) o[c] += w * load_elem(v, b, s, hk, c);
                if (a)
                    for (int c = 0; c < D; ++c) a[c] += w * fabs(load_elem(v, b, s, hk, c));
            }
            for (int c = 0; c < D; ++c) o[c] /= z;
            if (a)
                for (int c = 0; c < D; ++c) a[c] /= z;
            if (lse) lse[r] = m + log(z);
        }
        free(logit);
        free(qrow);
    }
}

/* Effective FLOP of block-sparse causal attention: 4 * D * (number of unmasked (t, s) token
 * pairs inside the kept blocks), summed over query heads.  Counts exactly with a ragged tail. */
double orc_effective_flop(int N, int Hq, int D, int bs, const int32_t* row_ptr, int rp_stride,
                          const int32_t* col_idx, int64_t maxK, int b) {
    int nb = (N + bs - 1) / bs;
    double pairs = 0.0;
    const int32_t* rp = &row_ptr[(int64_t)b * rp_stride];
    for (int h = 0; h < Hq; ++h)
        for (int i = 0; i < nb; ++i) {
            int64_t tlo = (int64_t)i * bs, thi = tlo + bs < N ? tlo + bs : N;
            for (int32_t n = rp[i]; n < rp[i + 1]; ++n) {
                int64_t j = col_idx[((int64_t)b * Hq + h) * maxK + n];
                int64_t slo = j * bs, shi = slo + bs < N ? slo + bs : N;
                for (int64_t t = tlo; t < thi; ++t) {
                    int64_t hi = shi - 1 < t ? shi - 1 : t;
                    if (hi >= slo) pairs += (double)(hi - slo + 1);
                }
            }
        }
    return 4.0 * D * pairs;
}

/* Number of host threads the parallel loops above use from now on (for timing the oracle on
 * one core or on all of them; no effect on any result). */
void orc_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
