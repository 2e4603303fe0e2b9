"""The longest sequence the library takes: one 256K-token sequence (2048 query blocks, the
maximum per sequence), 32 query / 8 KV heads, d = 128, block 128, density 25% (75% sparsity).

[cn486 §二.3 Benchmark: the operator stays stable from 8K to 256K at 75% sparsity.]  Both
storage types of the attention kernels run, through the calls the benchmark times:
- lists: every row bit-exact against the oracle's budget + top-k on the GPU's own fp32 scores;
- attention: sampled query rows (block boundaries, the last tokens, random tokens of three
  heads) against the fp64 oracle on the GPU's lists; LSE against the oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("storage", ["fp8", "bf16"])
def test_256k_single_sequence(orc, storage):
    w = inputs.Workload("single-256k", 1, 32, 8, 262144, 128, 128, storage, 0.25, "stem", 4)
    d = inputs.make_inputs(w, device=DEV)
    q, k, v = d["q"], d["k"], d["v"]
    fp8 = storage == "fp8"
    kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"], v_scale=d["v_scale"]) if fp8 else {}
    B, N, Hq, D = q.shape
    S = bsa.stem_score(q, k, v, w.block, **kw)
    nb = S.shape[-1]
    assert nb == 2048
    rp, ci = bsa.stem_select(S, [nb], w.density)
    out, lse = bsa.bsa_prefill(q, k, v, w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()

    rp_o, ci_o = orc.select(S.double().cpu().numpy(), [nb], w.density, 0.5, maxK=ci.shape[-1])
    del S
    assert np.array_equal(rp.cpu().numpy(), rp_o)
    tot = rp_o[0, -1]
    assert np.array_equal(ci.cpu().numpy()[0, :, :tot], ci_o[0, :, :tot])

    rows = H.sample_rows(B, Hq, N, w.block, n_heads=3, n_rand=24, seed=21)
    sc = (d["q_scale"], d["k_scale"], d["v_scale"]) if fp8 else ()
    ref, ref_lse, amp = H.oracle_attention(orc, q, k, v, w.block, rp, ci, H.default_tau(D), rows, *sc)
    got = H.gather_rows(out, rows)
    if fp8:
        assert H.rel_l2(got, ref) <= H.FP8_REL_L2
    else:
        H.assert_bf16_close(got, ref, amp)
    got_lse = np.array([lse[b, h, t].item() for b, h, t in rows])
    assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS
