"""Parity at the full long-context FP8 size (B=1, N=131072, 64 query / 8 KV heads, d=128,
block 128, density 0.25), through the same calls and kernels the benchmark times.

- Lists: every row bit-exact against the oracle's budget + top-k run on the GPU's own fp32
  scores (the same precision decides the same integers).
- Scores: the whole causal triangle against the oracle's fp64 pooling and score.
- Attention: sampled query rows (block boundaries, the last tokens, random tokens of four
  heads) against the fp64 oracle on the GPU's lists; FP8 rel-L2 bound, LSE abs bound.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_fp8_128k_lists_scores_and_sampled_outputs(orc):
    w = inputs.fp8_128k()
    d = inputs.make_inputs(w, device=DEV)
    q, k, v = d["q"], d["k"], d["v"]
    sq, sk, sv = d["q_scale"], d["k_scale"], d["v_scale"]
    kw = dict(q_scale=sq, k_scale=sk, v_scale=sv)
    B, N, Hq, D = q.shape
    tau = H.default_tau(D)

    S = bsa.stem_score(q, k, v, w.block, **kw)
    nb = S.shape[-1]
    rp, ci = bsa.stem_select(S, [nb] * B, w.density)
    out, lse = bsa.bsa_prefill(q, k, v, w.block, rp, ci, return_lse=True, **kw)
    bsa.bsa_check_device_error()

    # lists, every row
    S_host = S.double().cpu().numpy()
    rp_o, ci_o = orc.select(S_host, [nb] * B, w.density, 0.5, maxK=ci.shape[-1])
    rp_g, ci_g = rp.cpu().numpy(), ci.cpu().numpy()
    assert np.array_equal(rp_g, rp_o)
    tot = rp_o[0, -1]
    assert np.array_equal(ci_g[0, :, :tot], ci_o[0, :, :tot])

    # scores, whole causal triangle
    qb, kb, vb = H.oracle_pool(orc, q, k, v, w.block, sq, sk, sv)
    So = orc.score(qb, kb, vb, tau, 0)
    H.assert_scores_close(S, So, H.score_scale(qb, kb, vb, tau, 0), nb)
    del S_host, So

    # attention, sampled rows
    rows = H.sample_rows(B, Hq, N, w.block, n_heads=4, n_rand=40, seed=3)
    ref, ref_lse, _ = H.oracle_attention(orc, q, k, v, w.block, rp, ci, tau, rows, sq, sk, sv)
    got = H.gather_rows(out, rows)
    assert H.rel_l2(got, ref) <= H.FP8_REL_L2
    got_lse = np.array([lse[b, h, t].item() for b, h, t in rows])
    assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS


def test_paged_varlen_full_size(orc):
    """B=4 sequences of 16K/32K/64K/128K tokens, 32 query / 8 KV heads, BF16 KV in 64-token
    pages placed by a seeded permutation (spare pages hold NaN).  Per sequence: lists bit-exact
    against the oracle's select on the GPU's scores, and sampled output rows and LSE against
    the fp64 oracle on the GPU's lists."""
    w = inputs.paged_varlen()
    d = inputs.make_paged(w, device=DEV)
    seqlens, cu = d["seqlens"], d["cu_seqlens"]
    B, Hq, Hkv, D, bs = len(seqlens), w.Hq, w.Hkv, w.d, w.block
    nbp = [(n + bs - 1) // bs for n in seqlens]
    nbs = max(nbp)
    S = torch.full((B, Hq, nbs, nbs), float("nan"), device=DEV)
    for b in range(B):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        bsa.stem_score(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), bs, scores=S[b:b + 1],
                       nb_stride=nbs)
    rp, ci = bsa.stem_select(S, nbp, w.density)
    out, lse = bsa.bsa_prefill_paged(d["q"], cu.to(DEV), seqlens, d["k_cache"], d["v_cache"], d["page_table"], bs,
                                     rp, ci, return_lse=True)
    bsa.bsa_check_device_error()

    rp_o, ci_o = orc.select(S.double().cpu().numpy(), nbp, w.density, 0.5, maxK=ci.shape[-1])
    rp_g, ci_g = rp.cpu().numpy(), ci.cpu().numpy()
    assert np.array_equal(rp_g, rp_o)
    for b in range(B):
        tot = rp_o[b, -1]
        assert np.array_equal(ci_g[b, :, :tot], ci_o[b, :, :tot]), b

    tau = H.default_tau(D)
    for b, n in enumerate(seqlens):
        qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
        rows = H.sample_rows(1, Hq, n, bs, n_heads=2, n_rand=16, seed=11 + b)
        ref, ref_lse, amp = H.oracle_attention(orc, qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0),
                                               bs, rp[b:b + 1], ci[b:b + 1], tau, rows)
        ob = out[cu[b]:cu[b + 1]].unsqueeze(0)
        H.assert_bf16_close(H.gather_rows(ob, rows), ref, amp)
        got_lse = np.array([lse[b, h, t].item() for _, h, t in rows])
        assert np.max(np.abs(got_lse - ref_lse)) <= H.LSE_ABS, b
