"""Group-shared selection and GQA-packed attention (stem_score_group, stem_select on group
scores, bsa_prefill_group) against the fp64 oracle.

The pages select per query head; one list per KV-head group (the query side being the mean of
the group's pooled queries) is this library's extension.  Checks:
- group scores against the oracle's group mean + score, 1e-5 relative (scaled);
- lists bit-exact against the oracle's budget + top-k on the GPU's own fp32 group scores;
- attention against the oracle with each group's list given to every head of the group: FP8
  (the GQA-packed kernel) rel-L2 5e-2, BF16 (the per-head kernels on shared lists) the BF16 bound;
- the packed kernel bit-identical to the per-head kernel run on the same (expanded) lists;
- an odd group size (no pairing) and full size (fp8-128k).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(w, N=None):
    d = inputs.make_inputs(w, device=DEV, N=N)
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"]) if w.dtype == "fp8" else {}
    return d["q"], d["k"], d["v"], kw


def _expand(ci, G):
    """[B, Hkv, max_k] group lists -> [B, Hq, max_k]: every head of a group gets its list."""
    return ci.repeat_interleave(G, dim=1).contiguous()


def _oracle_group_scores(orc, q, k, v, block, kw, metric=0):
    qb, kb, vb = H.oracle_pool(orc, q, k, v, block, kw.get("q_scale", 1.0), kw.get("k_scale", 1.0),
                               kw.get("v_scale", 1.0))
    gb = orc.group_mean(qb, k.shape[2])
    tau = H.default_tau(q.shape[-1])
    return orc.score(gb, kb, vb, tau, metric), H.score_scale(gb, kb, vb, tau, metric)


GROUP_CASES = [
    # (name, workload)
    ("fp8-g8", inputs.Workload("grp-fp8", 1, 16, 2, 2000, 128, 128, "fp8", 0.3, "stem", 51)),
    ("bf16-g4-B2", inputs.Workload("grp-bf16", 2, 8, 2, 1500, 128, 128, "bf16", 0.3, "stem", 52)),
    ("bf16-d64-b64-g3", inputs.Workload("grp-odd", 1, 6, 2, 900, 64, 64, "bf16", 0.3, "normal", 53)),
    ("fp8-g1", inputs.Workload("grp-mha", 1, 4, 4, 1100, 128, 128, "fp8", 0.3, "stem", 54)),
]


@pytest.mark.parametrize("name,w", GROUP_CASES, ids=[c[0] for c in GROUP_CASES])
@pytest.mark.parametrize("metric", [0, 1])
def test_group_scores_and_lists(orc, name, w, metric):
    q, k, v, kw = _inputs(w)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    S = bsa.stem_score_group(q, k, v, w.block, metric=metric, **kw)
    nb = S.shape[-1]
    assert S.shape == (B, Hkv, nb, nb)
    rp, ci = bsa.stem_select(S, [nb] * B, w.density)
    torch.cuda.synchronize()
    So, scale = _oracle_group_scores(orc, q, k, v, w.block, kw, metric)
    H.assert_scores_close(S, So, scale, nb)
    rp_o, ci_o = orc.select(S.double().cpu().numpy(), [nb] * B, w.density, 0.5, maxK=ci.shape[-1])
    assert np.array_equal(rp.cpu().numpy(), rp_o)
    for b in range(B):
        tot = rp_o[b, -1]
        assert np.array_equal(ci.cpu().numpy()[b, :, :tot], ci_o[b, :, :tot])


@pytest.mark.parametrize("name,w", GROUP_CASES, ids=[c[0] for c in GROUP_CASES])
def test_group_attention_matches_oracle(orc, name, w):
    q, k, v, kw = _inputs(w)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    S = bsa.stem_score_group(q, k, v, w.block, **kw)
    rp, ci = bsa.stem_select(S, [S.shape[-1]] * B, w.density)
    out, lse = bsa.bsa_prefill_group(q, k, v, w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()
    rows = H.all_rows(B, Hq, N)
    sc = (kw["q_scale"], kw["k_scale"], kw["v_scale"]) if kw else ()
    ref, ref_lse, amp = H.oracle_attention(orc, q, k, v, w.block, rp, _expand(ci, Hq // Hkv), H.default_tau(D),
                                           rows, *sc)
    got = H.gather_rows(out, rows)
    if w.dtype == "fp8":
        assert H.rel_l2(got, ref) <= H.FP8_REL_L2
    else:
        H.assert_bf16_close(got, ref, amp)
    got_lse = lse.cpu().numpy().reshape(-1)
    assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS


def test_packed_kernel_equals_per_head_kernel(monkeypatch):
    """The GQA-packed kernel computes each head exactly as the per-head kernel does on the same
    list: outputs and LSE bit-identical."""
    w = inputs.Workload("grp-fp8-eq", 2, 16, 4, 3000, 128, 128, "fp8", 0.25, "stem", 55)
    q, k, v, kw = _inputs(w)
    B, N, Hq, D = q.shape
    S = bsa.stem_score_group(q, k, v, w.block, **kw)
    rp, ci = bsa.stem_select(S, [S.shape[-1]] * B, w.density)
    monkeypatch.delenv("BSA_ATTN_VARIANT", raising=False)
    packed, lse_p = bsa.bsa_prefill_group(q, k, v, w.block, rp, ci, return_lse=True, **kw)
    per_head, lse_h = bsa.bsa_prefill(q, k, v, w.block, rp, _expand(ci, Hq // k.shape[2]), return_lse=True, **kw)
    bsa.bsa_check_device_error()
    assert torch.equal(packed.view(torch.int16), per_head.view(torch.int16))
    assert torch.equal(lse_p, lse_h)
    # the per-head kernels reading the shared lists directly agree too
    for var in ("ws3", "serial"):
        monkeypatch.setenv("BSA_ATTN_VARIANT", var)
        o = bsa.bsa_prefill_group(q, k, v, w.block, rp, ci, **kw)
        bsa.bsa_check_device_error()
        assert H.rel_l2(o.float().cpu().numpy(), per_head.float().cpu().numpy()) <= 1e-2, var


def test_group_fp8_128k(orc):
    """Full size (128K tokens, 64 / 8 heads, FP8): every list row bit-exact against the oracle's
    select on the GPU's group scores, sampled output rows against the oracle."""
    w = inputs.fp8_128k()
    q, k, v, kw = _inputs(w)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    S = bsa.stem_score_group(q, k, v, w.block, **kw)
    nb = S.shape[-1]
    rp, ci = bsa.stem_select(S, [nb] * B, w.density)
    out = bsa.bsa_prefill_group(q, k, v, w.block, rp, ci, **kw)
    bsa.bsa_check_device_error()
    rp_o, ci_o = orc.select(S.double().cpu().numpy(), [nb] * B, w.density, 0.5, maxK=ci.shape[-1])
    del S
    assert np.array_equal(rp.cpu().numpy(), rp_o)
    tot = rp_o[0, -1]
    assert np.array_equal(ci.cpu().numpy()[0, :, :tot], ci_o[0, :, :tot])
    rows = H.sample_rows(B, Hq, N, w.block, n_heads=4, n_rand=32, seed=5)
    ref, _, _ = H.oracle_attention(orc, q, k, v, w.block, rp, _expand(ci, Hq // Hkv), H.default_tau(D), rows,
                                   kw["q_scale"], kw["k_scale"], kw["v_scale"])
    assert H.rel_l2(H.gather_rows(out, rows), ref) <= H.FP8_REL_L2
