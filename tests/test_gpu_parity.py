"""CUDA path (through the C ABI) vs the fp64 CPU oracle, on the same seeded inputs.

Tolerances: scores 1e-5 relative to max(|S|, the dot product's magnitude scale); lists
bit-exact when both sides rank the same fp32 scores, and equal up to near-ties against the
oracle's own fp64 scores; BF16 outputs max-abs 2e-2 and rel-L2 1e-2; FP8 outputs rel-L2 5e-2.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(params=["ws3", "ws2", "serial"])
def variant(request, monkeypatch):
    """Attention kernel: every variant the library can run (ws3 is the default)."""
    monkeypatch.setenv("BSA_ATTN_VARIANT", request.param)
    return request.param


def _inputs(w, N=None, storage=None, seed_offset=0):
    d = inputs.make_inputs(w, device=DEV, N=N, storage=storage, seed_offset=seed_offset)
    return d["q"], d["k"], d["v"], d["q_scale"], d["k_scale"], d["v_scale"]


# ----------------------------------------------------------------------------- a1 + a2 scores

SCORE_CASES = [
    # (workload, N, storage, metric)
    (inputs.tiny(), None, "fp32", 0),
    (inputs.tiny(), None, "bf16", 0),
    (inputs.gqa_8k(), None, "bf16", 0),
    (inputs.gqa_8k(), None, "bf16", 1),
    (inputs.gqa_8k(), None, "bf16", 2),
    (inputs.gqa_8k(), 3000, "bf16", 0),        # ragged tail (3000 = 23 * 128 + 56)
    (inputs.gqa_8k(), 2048, "fp8", 0),
    (inputs.Workload("d64", 2, 4, 2, 1000, 64, 64, "bf16", 0.25, "stem", 7), None, "bf16", 0),
    (inputs.gqa_8k(), 32768 + 300, "bf16", 0),  # nb = 259: several 128 x 128 score tiles + a ragged one
]


@pytest.fixture(params=["tc", "simt"])
def score_variant(request, monkeypatch):
    """Score GEMM: tcgen05 3xTF32 (default) or the fp32 FMA kernel."""
    if request.param == "simt":
        monkeypatch.setenv("BSA_SCORE_VARIANT", "simt")
    else:
        monkeypatch.delenv("BSA_SCORE_VARIANT", raising=False)
    return request.param


@pytest.mark.parametrize("w,N,storage,metric", SCORE_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_scores_match_oracle(orc, score_variant, w, N, storage, metric):
    q, k, v, sq, sk, sv = _inputs(w, N, storage)
    B, N, Hq, d = q.shape
    tau = H.default_tau(d)
    nb = (N + w.block - 1) // w.block
    S = bsa.stem_score(q, k, v, w.block, metric=metric, nb_stride=nb + 3, q_scale=sq, k_scale=sk, v_scale=sv)
    torch.cuda.synchronize()
    qb, kb, vb = H.oracle_pool(orc, q, k, v, w.block, sq, sk, sv)
    So = orc.score(qb, kb, vb, tau, metric)
    H.assert_scores_close(S[..., :nb, :nb], So, H.score_scale(qb, kb, vb, tau, metric), nb)


def test_fp8_nan_code_pools_to_nan(orc):
    """An E4M3 NaN code in Q makes that block's pooled row, hence its scores, NaN (as in the
    oracle); every other score is unaffected."""
    w = inputs.gqa_8k()
    q, k, v, sq, sk, sv = _inputs(w, 2048, "fp8")
    q.view(torch.uint8)[0, 700, 3, 17] = 0x7F  # token 700 -> query block 5, head 3
    S = bsa.stem_score(q, k, v, w.block, q_scale=sq, k_scale=sk, v_scale=sv)
    torch.cuda.synchronize()
    qb, kb, vb = H.oracle_pool(orc, q, k, v, w.block, sq, sk, sv)
    assert np.isnan(qb[0, 3, 5, 17])
    So = orc.score(qb, kb, vb, H.default_tau(q.shape[-1]), 0)
    nb = S.shape[-1]
    g = S[0, 3, 5, :6].double().cpu().numpy()
    assert np.all(np.isnan(g)) and np.all(np.isnan(So[0, 3, 5, :6]))
    ok = np.ones(S.shape, bool)
    ok[0, 3, 5, :] = False
    Sg = S.double().cpu().numpy()
    tri = np.broadcast_to(np.tril(np.ones((nb, nb), bool)), S.shape) & ok
    assert np.all(np.isfinite(Sg[tri]) == np.isfinite(So[tri]))


# ----------------------------------------------------------------------------- a3 + a4 select


def _check_lists_equal(rp_g, ci_g, rp_o, ci_o, nbs, Hq):
    rp_g = rp_g.cpu().numpy()
    ci_g = ci_g.cpu().numpy()
    assert np.array_equal(rp_g, rp_o)
    for b in range(rp_o.shape[0]):
        tot = rp_o[b, -1]
        assert np.array_equal(ci_g[b, :, :tot], ci_o[b, :, :tot])


@pytest.mark.parametrize("density", [0.1, 0.2, 0.25, 0.5, 0.8, 1.0])
@pytest.mark.parametrize("decay", [0.5, 0.0])
def test_select_bitexact_on_gpu_scores(orc, density, decay):
    w = inputs.gqa_8k()
    q, k, v, *_ = _inputs(w)
    S = bsa.stem_score(q, k, v, w.block)
    nb = S.shape[-1]
    rp, ci = bsa.stem_select(S, [nb], density, decay)
    torch.cuda.synchronize()
    rp_o, ci_o = orc.select(S.double().cpu().numpy(), [nb], density, decay, maxK=ci.shape[-1])
    _check_lists_equal(rp, ci, rp_o, ci_o, nb, w.Hq)


def test_select_ties_nan_and_varlen(orc):
    """Exact ties, NaN, -0/+0 and -inf scores; three sequences of different lengths."""
    g = torch.Generator().manual_seed(5)
    B, Hq, nbs = 3, 5, 70
    S = torch.round(torch.randn(B, Hq, nbs, nbs, generator=g) * 2) / 2      # many exact ties
    S[0, 0, 40, 3:9] = float("nan")
    S[1, 2, 50, 10:20] = -0.0
    S[1, 2, 50, 20:30] = 0.0
    S[2, 4, 33, 1:5] = float("-inf")
    S = S.to(DEV)
    nbp = [70, 7, 41]
    for density in (0.2, 0.6):
        rp, ci = bsa.stem_select(S, nbp, density)
        torch.cuda.synchronize()
        rp_o, ci_o = orc.select(S.double().cpu().numpy(), nbp, density, maxK=ci.shape[-1])
        _check_lists_equal(rp, ci, rp_o, ci_o, nbs, Hq)


def test_budget_kernel_all_nb(orc):
    """row_ptr of the device budget == the oracle's budget for every nb in 1..2048."""
    for density, decay in [(0.25, 0.5), (0.1, 0.5), (0.8, 0.0)]:
        for start in range(1, 2049, 128):
            nbp = list(range(start, min(start + 128, 2049)))
            nbs = max(nbp)
            S = torch.zeros(len(nbp), 1, nbs, nbs, device=DEV)
            rp, _ = bsa.stem_select(S, nbp, density, decay)
            rp = rp.cpu().numpy()
            for b, nb in enumerate(nbp):
                k, tot = orc.tpd_budget(nb, density, decay)
                assert np.array_equal(np.diff(rp[b, : nb + 1]), k), (nb, density, decay)
                assert rp[b, nbs] == tot


def test_lists_vs_oracle_scores_up_to_near_ties(orc):
    """GPU lists (from GPU fp32 scores) vs oracle lists (from fp64 scores): any difference must
    sit at a near-tie of the k-th threshold."""
    w = inputs.gqa_8k()
    q, k, v, *_ = _inputs(w)
    S = bsa.stem_score(q, k, v, w.block)
    nb = S.shape[-1]
    rp, ci = bsa.stem_select(S, [nb], 0.25)
    torch.cuda.synchronize()
    qb, kb, vb = H.oracle_pool(orc, q, k, v, w.block)
    So = orc.score(qb, kb, vb, H.default_tau(w.d), 0)
    rp_o, ci_o = orc.select(So, [nb], 0.25, maxK=ci.shape[-1])
    rp, ci = rp.cpu().numpy(), ci.cpu().numpy()
    assert np.array_equal(rp, rp_o)
    mism = 0
    for h in range(w.Hq):
        for i in range(nb):
            a = set(ci[0, h, rp[0, i]:rp[0, i + 1]].tolist())
            o = set(ci_o[0, h, rp[0, i]:rp[0, i + 1]].tolist())
            if a == o:
                continue
            mism += 1
            row = So[0, h, i, : i + 1]
            kept_o = [j for j in o if 0 < j < i]
            thr = min(row[kept_o]) if kept_o else np.inf
            for j in a ^ o:
                tol = 1e-5 * max(abs(row[j]), abs(thr), 1e-3 * np.max(np.abs(row[np.isfinite(row)])))
                assert abs(row[j] - thr) <= tol, (h, i, j, row[j], thr)
    assert mism <= nb * w.Hq // 50


# ----------------------------------------------------------------------------- a5 attention


def _lists(q, k, v, block, density, sq=1.0, sk=1.0, sv=1.0):
    S = bsa.stem_score(q, k, v, block, q_scale=sq, k_scale=sk, v_scale=sv)
    return bsa.stem_select(S, [S.shape[-1]] * q.shape[0], density)


ATTN_CASES = [
    # (name, workload, N, storage, full rows?)
    ("tiny-bf16", inputs.tiny(), None, "bf16", True),
    ("d128-bs128-ragged", inputs.Workload("r", 1, 4, 2, 1000, 128, 128, "bf16", 0.3, "stem", 11), None, "bf16", True),
    ("d64-bs128", inputs.Workload("r", 2, 4, 1, 777, 64, 128, "bf16", 0.4, "normal", 12), None, "bf16", True),
    ("d128-bs64", inputs.Workload("r", 1, 2, 2, 1100, 128, 64, "bf16", 0.3, "stem", 13), None, "bf16", True),
    ("gqa-8k", inputs.gqa_8k(), None, "bf16", False),
    ("sweep-32k-rho10", inputs.sweep_32k(0.1), None, "bf16", False),
    ("sweep-32k-rho80", inputs.sweep_32k(0.8), None, "bf16", False),
]


@pytest.mark.parametrize("name,w,N,storage,full", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attention_bf16_matches_oracle(orc, variant, name, w, N, storage, full):
    q, k, v, *_ = _inputs(w, N, storage)
    B, N, Hq, d = q.shape
    rp, ci = _lists(q, k, v, w.block, w.density)
    out, lse = bsa.bsa_prefill(q, k, v, w.block, rp, ci, return_lse=True)
    bsa.bsa_check_device_error()
    rows = H.all_rows(B, Hq, N) if full else H.sample_rows(B, Hq, N, w.block)
    ref, ref_lse, amp = H.oracle_attention(orc, q, k, v, w.block, rp, ci, H.default_tau(d), rows)
    got = H.gather_rows(out, rows)
    H.assert_bf16_close(got, ref, amp)
    got_lse = np.array([lse[b, h, t].item() for b, h, t in rows]) if not full else \
        lse.permute(0, 1, 2).cpu().numpy().reshape(-1)
    assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS


def test_attention_fp8_matches_oracle(orc, variant):
    w = inputs.Workload("fp8-small", 1, 8, 2, 1280, 128, 128, "fp8", 0.3, "stem", 14)
    q, k, v, sq, sk, sv = _inputs(w)
    B, N, Hq, d = q.shape
    rp, ci = _lists(q, k, v, w.block, w.density, sq, sk, sv)
    out = bsa.bsa_prefill(q, k, v, w.block, rp, ci, q_scale=sq, k_scale=sk, v_scale=sv)
    bsa.bsa_check_device_error()
    rows = H.all_rows(B, Hq, N)
    ref, _, _ = H.oracle_attention(orc, q, k, v, w.block, rp, ci, H.default_tau(d), rows, sq, sk, sv)
    got = H.gather_rows(out, rows)
    assert H.rel_l2(got, ref) <= H.FP8_REL_L2


def test_density_one_is_dense_causal(orc, variant):
    w = inputs.Workload("dense", 1, 4, 2, 640, 128, 128, "bf16", 1.0, "stem", 15)
    q, k, v, *_ = _inputs(w)
    rp, ci = _lists(q, k, v, w.block, 1.0)
    out = bsa.bsa_prefill(q, k, v, w.block, rp, ci)
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    qt, kt = q.double().transpose(1, 2), k.double().repeat_interleave(G, 2).transpose(1, 2)
    vt = v.double().repeat_interleave(G, 2).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True).transpose(1, 2)
    amp = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt.abs(), is_causal=True).transpose(1, 2)
    H.assert_bf16_close(out.double().cpu().numpy(), ref.cpu().numpy(), amp.cpu().numpy())


def test_skipped_blocks_do_not_matter(variant):
    """K/V of blocks outside query block i's list may hold anything (1e4, NaN): the outputs of
    block i's rows are bit-identical."""
    w = inputs.Workload("skip", 1, 1, 1, 1024, 128, 128, "bf16", 0.2, "normal", 16)
    q, k, v, *_ = _inputs(w)
    rp, ci = _lists(q, k, v, w.block, 0.2)
    out1 = bsa.bsa_prefill(q, k, v, w.block, rp, ci)
    i = 7
    kept = set(ci[0, 0, rp[0, i]:rp[0, i + 1]].cpu().tolist())
    assert len(kept) < i + 1
    k2, v2 = k.clone(), v.clone()
    for j in range(i + 1):
        if j not in kept:
            k2[:, j * 128:(j + 1) * 128] = 1e4
            v2[:, j * 128:(j + 1) * 128] = float("nan")
    out2 = bsa.bsa_prefill(q, k2, v2, w.block, rp, ci)
    torch.cuda.synchronize()
    assert torch.equal(out1[:, i * 128:(i + 1) * 128], out2[:, i * 128:(i + 1) * 128])


def test_paged_equals_contiguous(variant):
    w = inputs.paged_varlen(seqlens=(1000, 3000, 128, 2177))
    d = inputs.make_paged(w, device=DEV)
    outs, rps, cis = [], [], []
    nbs = max((n + 127) // 128 for n in d["seqlens"])
    Sfull = torch.full((len(d["seqlens"]), w.Hq, nbs, nbs), float("nan"), device=DEV)
    for b, n in enumerate(d["seqlens"]):
        qb = d["q"][d["cu_seqlens"][b]:d["cu_seqlens"][b + 1]].unsqueeze(0)
        bsa.stem_score(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), 128, scores=Sfull[b:b + 1],
                       nb_stride=nbs)
    nbp = [(n + 127) // 128 for n in d["seqlens"]]
    rp, ci = bsa.stem_select(Sfull, nbp, 0.25)
    cu = d["cu_seqlens"].to(DEV)
    outp = bsa.bsa_prefill_paged(d["q"], cu, d["seqlens"], d["k_cache"], d["v_cache"], d["page_table"], 128, rp, ci)
    bsa.bsa_check_device_error()
    for b, n in enumerate(d["seqlens"]):
        qb = d["q"][d["cu_seqlens"][b]:d["cu_seqlens"][b + 1]].unsqueeze(0)
        ref = bsa.bsa_prefill(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), 128, rp[b:b + 1],
                              ci[b:b + 1])
        assert torch.equal(outp[d["cu_seqlens"][b]:d["cu_seqlens"][b + 1]], ref[0]), b


def test_invalid_page_entry_is_flagged(variant):
    """A page-table entry outside [0, num_pages) for a page inside its sequence is read as zeros
    and reported as BSA_ERR_INVALID_PAGE (no out-of-range access)."""
    w = inputs.paged_varlen(seqlens=(1000, 300))
    d = inputs.make_paged(w, device=DEV)
    nbp = [(n + 127) // 128 for n in d["seqlens"]]
    nbs = max(nbp)
    S = torch.full((len(nbp), w.Hq, nbs, nbs), float("nan"), device=DEV)
    for b in range(len(nbp)):
        qb = d["q"][d["cu_seqlens"][b]:d["cu_seqlens"][b + 1]].unsqueeze(0)
        bsa.stem_score(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), 128, scores=S[b:b + 1],
                       nb_stride=nbs)
    rp, ci = bsa.stem_select(S, nbp, 0.25)
    cu = d["cu_seqlens"].to(DEV)
    bsa.bsa_check_device_error()
    pt = d["page_table"].clone()
    pt[0, 3] = d["num_pages"] + 7  # tokens 192..255 of sequence 0 (the diagonal block of query block 1)
    bsa.bsa_prefill_paged(d["q"], cu, d["seqlens"], d["k_cache"], d["v_cache"], pt, 128, rp, ci)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_check_device_error()
    assert ei.value.status == 7
    pt[0, 3] = -2
    bsa.bsa_prefill_paged(d["q"], cu, d["seqlens"], d["k_cache"], d["v_cache"], pt, 128, rp, ci)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_check_device_error()
    assert ei.value.status == 7
    bsa.bsa_check_device_error()  # cleared


def test_invalid_list_entry_is_flagged(variant):
    w = inputs.Workload("bad", 1, 2, 1, 512, 128, 128, "bf16", 0.5, "normal", 17)
    q, k, v, *_ = _inputs(w)
    rp, ci = _lists(q, k, v, w.block, 0.5)
    ci = ci.clone()
    ci[0, 1, rp[0, 2].item()] = 3          # row i=2 pointing at block 3 > i
    bsa.bsa_prefill(q, k, v, w.block, rp, ci)
    with pytest.raises(bsa.BsaError, match="INVALID_LIST"):
        bsa.bsa_check_device_error()
    bsa.bsa_check_device_error()           # the word was cleared


def test_variants_agree_at_full_size_sample(orc, monkeypatch):
    """The serial kernel and the default kernel on the 8K GQA workload agree in rel-L2 over the
    whole output, and on sampled rows within twice the BF16 bound (each is within the bound
    of the oracle; the per-row checks against the oracle are above)."""
    w = inputs.gqa_8k()
    q, k, v, *_ = _inputs(w)
    rp, ci = _lists(q, k, v, w.block, w.density)
    monkeypatch.setenv("BSA_ATTN_VARIANT", "serial")
    a = bsa.bsa_prefill(q, k, v, w.block, rp, ci)
    monkeypatch.setenv("BSA_ATTN_VARIANT", "ws3")
    b = bsa.bsa_prefill(q, k, v, w.block, rp, ci)
    bsa.bsa_check_device_error()
    assert H.rel_l2(b.double().cpu().numpy(), a.double().cpu().numpy()) <= H.BF16_REL_L2
    rows = H.sample_rows(1, w.Hq, w.N, w.block, n_heads=4, n_rand=32, seed=9)
    _, _, amp = H.oracle_attention(orc, q, k, v, w.block, rp, ci, H.default_tau(w.d), rows)
    ga, gb = H.gather_rows(a, rows), H.gather_rows(b, rows)
    assert np.all(np.abs(ga - gb) <= H.bf16_bound(ga, amp) + H.bf16_bound(gb, amp))
