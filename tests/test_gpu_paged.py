"""Paged KV cache: every paged attention instantiation against the fp64 oracle.

[cn486 §二.2.2 BSA算子优化: the operator reads KV straight from the serving engine's paged
cache, natively in FP8.]  The cache holds 64-token pages placed by a seeded permutation of a
pool with spare pages filled with NaN, so a stray read shows up in the output.

- FP8 e4m3 pages with per-tensor K / V scales (the FP8 paged kernel): sampled rows against
  the oracle (rel-L2 5e-2) and the whole output bit-identical to the contiguous FP8 call on
  the same data.
- BF16 pages at head_dim 64 and at block 64: sampled rows against the oracle (the BF16 bound),
  LSE against the oracle.
- group-shared lists on the page pool (bsa_prefill_paged_group): FP8 through the GQA-packed
  kernel and BF16 through the per-head kernels, sampled rows against the oracle with each
  group's list given to every head of the group; the FP8 output bit-identical to the
  contiguous bsa_prefill_group call on the same data.
"""
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
    monkeypatch.setenv("BSA_ATTN_VARIANT", request.param)
    return request.param


def _paged_lists(d, w, kw):
    """Scores of every sequence from its dense K/V view, then the TPD lists."""
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    bs = w.block
    nbp = [(n + bs - 1) // bs for n in seqlens]
    nbs = max(nbp)
    S = torch.full((len(seqlens), w.Hq, nbs, nbs), float("nan"), device=DEV)
    for b in range(len(seqlens)):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        bsa.stem_score(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), bs, scores=S[b:b + 1],
                       nb_stride=nbs, **kw)
    return bsa.stem_select(S, nbp, w.density)


PAGED_CASES = [
    # (name, workload)
    ("fp8-d128-b128", inputs.Workload("paged-fp8", 4, 8, 2, 3000, 128, 128, "fp8", 0.25, "stem", 31,
                                      seqlens=[1000, 3000, 128, 2177], page_size=64)),
    ("bf16-d64-b128", inputs.Workload("paged-d64", 3, 8, 2, 2500, 64, 128, "bf16", 0.3, "stem", 32,
                                      seqlens=[700, 2500, 1290], page_size=64)),
    ("bf16-d128-b64", inputs.Workload("paged-b64", 3, 8, 2, 2100, 128, 64, "bf16", 0.3, "stem", 33,
                                      seqlens=[2100, 65, 1337], page_size=64)),
    ("bf16-d64-b64", inputs.Workload("paged-d64-b64", 2, 4, 1, 1500, 64, 64, "bf16", 0.3, "normal", 34,
                                     seqlens=[1500, 333], page_size=64)),
]


@pytest.mark.parametrize("name,w", PAGED_CASES, ids=[c[0] for c in PAGED_CASES])
def test_paged_matches_oracle(orc, variant, name, w):
    d = inputs.make_paged(w, device=DEV)
    fp8 = w.dtype == "fp8"
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"]) if fp8 else {}
    rp, ci = _paged_lists(d, w, kw)
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    out, lse = bsa.bsa_prefill_paged(d["q"], cu.to(DEV), seqlens, d["k_cache"], d["v_cache"], d["page_table"],
                                     w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()
    assert not torch.isnan(out.float()).any(), "a stray read of a NaN spare page reached the output"
    tau = H.default_tau(w.d)
    for b, n in enumerate(seqlens):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        rows = H.sample_rows(1, w.Hq, n, w.block, n_heads=3, n_rand=24, seed=40 + b)
        sc = (d["q_scale"], d["k_scale"], d["v_scale"]) if fp8 else ()
        ref, ref_lse, amp = H.oracle_attention(orc, qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0),
                                               w.block, rp[b:b + 1], ci[b:b + 1], tau, rows, *sc)
        got = H.gather_rows(out[cu[b]:cu[b + 1]].unsqueeze(0), rows)
        if fp8:
            assert H.rel_l2(got, ref) <= H.FP8_REL_L2, b
        else:
            H.assert_bf16_close(got, ref, amp)
        got_lse = np.array([lse[b, h, t].item() for _, h, t in rows])
        assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS, b


def test_fp8_paged_equals_contiguous():
    """The FP8 paged kernel and the contiguous FP8 kernel read the same codes and scales: their
    outputs and LSE are bit-identical for every sequence."""
    w = PAGED_CASES[0][1]
    d = inputs.make_paged(w, device=DEV)
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"])
    rp, ci = _paged_lists(d, w, kw)
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    out, lse = bsa.bsa_prefill_paged(d["q"], cu.to(DEV), seqlens, d["k_cache"], d["v_cache"], d["page_table"],
                                     w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()
    for b, n in enumerate(seqlens):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        ref, ref_lse = bsa.bsa_prefill(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), w.block,
                                       rp[b:b + 1], ci[b:b + 1], return_lse=True, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out[cu[b]:cu[b + 1]].view(torch.int16), ref[0].view(torch.int16)), b
        assert torch.equal(lse[b, :, :n], ref_lse[0]), b


def _paged_group_lists(d, w, kw):
    """Group scores of every sequence from its dense K/V view, then the TPD lists [B, Hkv, max_k]."""
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    bs = w.block
    nbp = [(n + bs - 1) // bs for n in seqlens]
    nbs = max(nbp)
    S = torch.full((len(seqlens), w.Hkv, nbs, nbs), float("nan"), device=DEV)
    for b in range(len(seqlens)):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        bsa.stem_score_group(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), bs, scores=S[b:b + 1],
                             nb_stride=nbs, **kw)
    return bsa.stem_select(S, nbp, w.density)


PAGED_GROUP_CASES = [
    # (name, workload): FP8 with an even group runs the GQA-packed kernel; BF16 the per-head one
    ("fp8-g4", inputs.Workload("paged-grp-fp8", 4, 8, 2, 3000, 128, 128, "fp8", 0.25, "stem", 35,
                               seqlens=[1000, 3000, 128, 2177], page_size=64)),
    ("bf16-g4", inputs.Workload("paged-grp-bf16", 3, 8, 2, 2500, 128, 128, "bf16", 0.3, "stem", 36,
                                seqlens=[700, 2500, 1290], page_size=64)),
]


@pytest.mark.parametrize("name,w", PAGED_GROUP_CASES, ids=[c[0] for c in PAGED_GROUP_CASES])
def test_paged_group_matches_oracle(orc, monkeypatch, name, w):
    monkeypatch.delenv("BSA_ATTN_VARIANT", raising=False)
    d = inputs.make_paged(w, device=DEV)
    fp8 = w.dtype == "fp8"
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"]) if fp8 else {}
    rp, ci = _paged_group_lists(d, w, kw)
    assert ci.shape[1] == w.Hkv
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    out, lse = bsa.bsa_prefill_paged_group(d["q"], cu.to(DEV), seqlens, d["k_cache"], d["v_cache"],
                                           d["page_table"], w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()
    assert not torch.isnan(out.float()).any(), "a stray read of a NaN spare page reached the output"
    tau = H.default_tau(w.d)
    ci_h = ci.repeat_interleave(w.Hq // w.Hkv, dim=1).contiguous()
    for b, n in enumerate(seqlens):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        rows = H.sample_rows(1, w.Hq, n, w.block, n_heads=3, n_rand=24, seed=60 + b)
        sc = (d["q_scale"], d["k_scale"], d["v_scale"]) if fp8 else ()
        ref, ref_lse, amp = H.oracle_attention(orc, qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0),
                                               w.block, rp[b:b + 1], ci_h[b:b + 1], tau, rows, *sc)
        got = H.gather_rows(out[cu[b]:cu[b + 1]].unsqueeze(0), rows)
        if fp8:
            assert H.rel_l2(got, ref) <= H.FP8_REL_L2, b
        else:
            H.assert_bf16_close(got, ref, amp)
        got_lse = np.array([lse[b, h, t].item() for _, h, t in rows])
        assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS, b


def test_fp8_paged_group_equals_contiguous(monkeypatch):
    """The GQA-packed kernel on the page pool and on contiguous K/V read the same codes and
    scales: outputs and LSE bit-identical for every sequence; the per-head kernel on the same
    shared lists agrees as well."""
    monkeypatch.delenv("BSA_ATTN_VARIANT", raising=False)
    w = PAGED_GROUP_CASES[0][1]
    d = inputs.make_paged(w, device=DEV)
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"])
    rp, ci = _paged_group_lists(d, w, kw)
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    out, lse = bsa.bsa_prefill_paged_group(d["q"], cu.to(DEV), seqlens, d["k_cache"], d["v_cache"],
                                           d["page_table"], w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()
    for b, n in enumerate(seqlens):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        ref, ref_lse = bsa.bsa_prefill_group(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), w.block,
                                             rp[b:b + 1], ci[b:b + 1], return_lse=True, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out[cu[b]:cu[b + 1]].view(torch.int16), ref[0].view(torch.int16)), b
        assert torch.equal(lse[b, :, :n], ref_lse[0]), b
    monkeypatch.setenv("BSA_ATTN_VARIANT", "ws3")
    per_head = bsa.bsa_prefill_paged_group(d["q"], cu.to(DEV), seqlens, d["k_cache"], d["v_cache"],
                                           d["page_table"], w.block, rp, ci, **kw)
    bsa.bsa_check_device_error()
    assert torch.equal(per_head.view(torch.int16), out.view(torch.int16))
