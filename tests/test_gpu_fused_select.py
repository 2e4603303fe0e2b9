"""stem_score_select: score and select without the score matrix.

[cn486 §二.2.1 Stem算子优化: budget generation and selection are fused, with no large
intermediates.]  The call scores one chunk of KV-head groups at a time and selects from it, so
its lists must equal, bit for bit, those of stem_score followed by stem_select on the same
inputs (the same per-tile products, the same per-row selection):
- several shapes, metrics, densities and both TPD decays, B = 2, ragged tails;
- the full 128K FP8 workload (eight chunks of one KV-head group each);
- the lists also bit-exact against the oracle's select on the unfused path's scores.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = [
    ("bf16-gqa-ragged", inputs.Workload("fs1", 2, 8, 2, 3000, 128, 128, "bf16", 0.25, "stem", 71), 0, 0.5),
    ("fp8-sam", inputs.Workload("fs2", 1, 16, 4, 4096, 128, 128, "fp8", 0.2, "stem", 72), 1, 0.5),
    ("bf16-d64-b64-uniform", inputs.Workload("fs3", 2, 4, 4, 1000, 64, 64, "bf16", 0.5, "normal", 73), 0, 0.0),
    ("fp32-oam-mul", inputs.Workload("fs4", 1, 4, 1, 777, 64, 128, "fp32", 0.3, "normal", 74), 2, 0.5),
]


def _unfused(q, k, v, w, metric, decay, kw):
    S = bsa.stem_score(q, k, v, w.block, metric=metric, **kw)
    rp, ci = bsa.stem_select(S, [S.shape[-1]] * q.shape[0], w.density, decay)
    return S, rp, ci


@pytest.mark.parametrize("name,w,metric,decay", CASES, ids=[c[0] for c in CASES])
def test_fused_equals_unfused(orc, name, w, metric, decay):
    d = inputs.make_inputs(w, device=DEV)
    q, k, v = d["q"], d["k"], d["v"]
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"]) if w.dtype == "fp8" else {}
    S, rp, ci = _unfused(q, k, v, w, metric, decay, kw)
    frp, fci = bsa.stem_score_select(q, k, v, w.block, w.density, decay, metric=metric, max_k=ci.shape[-1], **kw)
    bsa.bsa_check_device_error()
    assert torch.equal(frp, rp)
    tot = int(rp[0, -1])
    assert torch.equal(fci[..., :tot], ci[..., :tot])
    nb = S.shape[-1]
    rp_o, ci_o = orc.select(S.double().cpu().numpy(), [nb] * q.shape[0], w.density, decay, maxK=ci.shape[-1])
    assert np.array_equal(frp.cpu().numpy(), rp_o)
    assert np.array_equal(fci.cpu().numpy()[..., :tot], ci_o[..., :tot])


def test_fused_equals_unfused_fp8_128k():
    w = inputs.fp8_128k()
    d = inputs.make_inputs(w, device=DEV)
    q, k, v = d["q"], d["k"], d["v"]
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"])
    S, rp, ci = _unfused(q, k, v, w, 0, 0.5, kw)
    del S
    frp, fci = bsa.stem_score_select(q, k, v, w.block, w.density, **kw)
    bsa.bsa_check_device_error()
    assert torch.equal(frp, rp)
    assert torch.equal(fci, ci)
    # the workspace holds the pooled means and at most 128 MiB of scores, not the score matrix
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    nb = N // w.block
    pooled = bsa.bsa_score_workspace_bytes(B, Hq, Hkv, nb, D)
    fused = bsa.bsa_score_select_workspace_bytes(B, Hq, Hkv, N, w.block, D)
    assert pooled < fused <= pooled + (128 << 20) + 256
    assert fused < pooled + 4 * B * Hq * nb * nb
