"""Threshold skip on top of the kept-block lists (bsa_prefill_skip) against the fp64 oracle.

["BLASST: Dynamic BLocked Attention Sparsity via Softmax Thresholding", §2.1: a block whose local
maximum trails the running maximum by more than ln(lambda) is skipped.]
- lambda = 0, and lambda = 1e-38 (it only drops blocks whose weights are below fp32's range):
  bit-identical to bsa_prefill;
- lambda = 1e-3 / 1e-2: sampled rows against the oracle's restatement of the rule (FP8 rel-L2
  bound; BF16 at head_dim 64 the BF16 bound), and the skip counters against the oracle's count
  of skipped (row, block) pairs on the same rows' sequence;
- shapes the skip does not run are refused.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _setup(w):
    d = inputs.make_inputs(w, device=DEV)
    q, k, v = d["q"], d["k"], d["v"]
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"]) if w.dtype == "fp8" else {}
    S = bsa.stem_score(q, k, v, w.block, **kw)
    rp, ci = bsa.stem_select(S, [S.shape[-1]] * q.shape[0], w.density)
    return q, k, v, kw, rp, ci


CASES = [
    ("fp8", inputs.Workload("skip-fp8", 1, 8, 2, 3000, 128, 128, "fp8", 0.4, "stem", 61)),
    ("bf16-d64", inputs.Workload("skip-bf16", 2, 4, 2, 1500, 64, 128, "bf16", 0.4, "stem", 62)),
]


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_no_skip_is_bit_identical(name, w):
    """lambda = 0 runs the plain kernel (the counters stay untouched); lambda = 1e-38 only drops
    blocks whose weights are below 1e-38 of the row's largest (the outlier channels make such
    gaps real), which cannot change an fp32 sum: both are bit-identical to bsa_prefill."""
    q, k, v, kw, rp, ci = _setup(w)
    ref, ref_lse = bsa.bsa_prefill(q, k, v, w.block, rp, ci, return_lse=True, **kw)
    for lam in (0.0, 1e-38):
        stats = torch.zeros(4, dtype=torch.int64, device=DEV)
        out, lse = bsa.bsa_prefill_skip(q, k, v, w.block, rp, ci, lam, return_lse=True, skip_stats=stats, **kw)
        bsa.bsa_check_device_error()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), lam
        assert torch.equal(lse, ref_lse), lam
        st = stats.cpu().tolist()
        if lam == 0.0:
            assert st == [0, 0, 0, 0]
        else:
            assert st[0] > 0 and st[1] <= st[0] // 100 and st[3] <= st[2], st


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("lam", [1e-3, 1e-2])
def test_skip_matches_oracle(orc, name, w, lam):
    q, k, v, kw, rp, ci = _setup(w)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    out, lse = bsa.bsa_prefill_skip(q, k, v, w.block, rp, ci, lam, return_lse=True, skip_stats=stats, **kw)
    bsa.bsa_check_device_error()
    st = stats.cpu().tolist()
    rows = H.all_rows(B, Hq, N)
    sc = (kw["q_scale"], kw["k_scale"], kw["v_scale"]) if kw else (1.0, 1.0, 1.0)
    ref, ref_lse, skipped = orc.attention_rows_skip(
        orc.view(q.cpu(), sc[0]), orc.view(k.cpu(), sc[1]), orc.view(v.cpu(), sc[2]), N, Hq, Hkv, D, w.block,
        rp.cpu().numpy(), ci.cpu().numpy(), H.default_tau(D), lam, rows)
    got = H.gather_rows(out, rows)
    if w.dtype == "fp8":
        assert H.rel_l2(got, ref) <= H.FP8_REL_L2
    else:
        _, _, amp = H.oracle_attention(orc, q, k, v, w.block, rp, ci, H.default_tau(D), rows)
        H.assert_bf16_close(got, ref, amp)
    assert np.max(np.abs(lse.cpu().numpy().reshape(-1) - ref_lse)) <= H.LSE_ABS
    # counters: every (row, kept block) pair of the real rows is visited once; the skipped count
    # agrees with the oracle's up to decisions within a rounding of the threshold
    visited = sum(int(rp[b, (t // w.block) + 1] - rp[b, t // w.block]) for b, _, t in rows)
    assert st[0] == visited
    assert skipped.sum() > 0
    assert abs(st[1] - int(skipped.sum())) <= max(2, int(1e-3 * visited)), (st, int(skipped.sum()))
    assert 0 <= st[3] <= st[2]


def test_skip_refuses_unsupported_shapes():
    w = inputs.Workload("skip-bf16-128", 1, 4, 2, 512, 128, 128, "bf16", 0.5, "stem", 63)
    q, k, v, kw, rp, ci = _setup(w)
    with pytest.raises(bsa.BsaError, match="UNSUPPORTED"):
        bsa.bsa_prefill_skip(q, k, v, w.block, rp, ci, 1e-3)
    with pytest.raises(bsa.BsaError, match="INVALID_ARG"):
        bsa.bsa_prefill_skip(q, k, v, w.block, rp, ci, 1.5)
