"""bsa_prefill_mask / bsa_mask_to_lists (selection given as a block mask) through the C ABI.

Against the fp64 oracle's mask attention (same tolerances as the list path: BF16 max-abs
2e-2 + four half-ulps and rel-L2 1e-2, FP8 rel-L2 5e-2, LSE 1e-3); rows whose mask keeps
nothing must be exactly 0 with LSE -inf; the lists built from a mask are compared exactly with
a brute-force nonzero(); a mask written from stem_select's lists must give the bsa_prefill
output bit for bit.
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


def _inputs(w):
    d = inputs.make_inputs(w, device=DEV)
    return d["q"], d["k"], d["v"], d["q_scale"], d["k_scale"], d["v_scale"]


def _random_mask(B, Hq, nb, p, seed, empty=(), full=()):
    """Random kept blocks (values 1..255 where kept, anything above the diagonal), in a
    block_mask_buffer.  `empty` rows keep nothing at j <= i (above the diagonal stays random)."""
    g = torch.Generator().manual_seed(seed)
    m = torch.randint(1, 256, (B, Hq, nb, nb), generator=g, dtype=torch.int32)
    m = torch.where(torch.rand(B, Hq, nb, nb, generator=g) < p, m, torch.zeros_like(m)).to(torch.uint8)
    for b, h, i in empty:
        m[b, h, i, :i + 1] = 0
    for b, h, i in full:
        m[b, h, i, :] = 1
    buf = bsa.block_mask_buffer(B, Hq, nb, device=DEV)
    buf.copy_(m.to(DEV))
    return buf


def _oracle(orc, q, k, v, block, mask, rows, sq=1.0, sk=1.0, sv=1.0):
    B, N, Hq, d = q.shape
    return orc.attention_rows_mask(orc.view(q.cpu(), sq), orc.view(k.cpu(), sk), orc.view(v.cpu(), sv), N, Hq,
                                   k.shape[2], d, block, mask.cpu().numpy(), H.default_tau(d), rows, with_amp=True)


def _empty_rows(mask, N, block):
    """(b, h, t) rows whose mask row keeps no block j <= i."""
    m = mask.cpu().numpy()
    B, Hq, nb, _ = m.shape
    keep = np.array([[[m[b, h, i, :i + 1].any() for i in range(nb)] for h in range(Hq)] for b in range(B)])
    return {(b, h, t) for b in range(B) for h in range(Hq) for t in range(N) if not keep[b, h, t // block]}


MASK_CASES = [
    ("bf16-d128-b128-ragged", inputs.Workload("m1", 1, 8, 2, 1000, 128, 128, "bf16", 0.3, "stem", 41)),
    ("bf16-d64-b64-B2", inputs.Workload("m2", 2, 4, 2, 700, 64, 64, "bf16", 0.3, "normal", 42)),
    ("bf16-d128-b64", inputs.Workload("m3", 1, 4, 1, 600, 128, 64, "bf16", 0.3, "stem", 43)),
]


@pytest.mark.parametrize("name,w", MASK_CASES, ids=[c[0] for c in MASK_CASES])
def test_mask_bf16_matches_oracle(orc, variant, name, w):
    q, k, v, *_ = _inputs(w)
    B, N, Hq, d = q.shape
    nb = (N + w.block - 1) // w.block
    mask = _random_mask(B, Hq, nb, 0.35, 100 + nb, empty=[(0, 1, 2), (B - 1, Hq - 1, nb - 1), (0, 0, 0)],
                        full=[(0, 0, nb - 1)])
    out, lse = bsa.bsa_prefill_mask(q, k, v, w.block, mask, return_lse=True)
    bsa.bsa_check_device_error()
    rows = H.all_rows(B, Hq, N)
    ref, ref_lse, amp = _oracle(orc, q, k, v, w.block, mask, rows)
    got = H.gather_rows(out, rows)
    H.assert_bf16_close(got, ref, amp)
    got_lse = lse.cpu().numpy().reshape(-1)            # [B, Hq, N] in (b, h, t) order, as rows
    empty = np.array([tuple(r) in _empty_rows(mask, N, w.block) for r in rows])
    assert empty.any() and not empty.all()
    assert np.all(got[empty] == 0.0) and np.all(np.isneginf(got_lse[empty]))
    assert np.all(np.isneginf(ref_lse[empty]))
    assert np.max(np.abs(got_lse[~empty] - ref_lse[~empty])) <= H.LSE_ABS


def test_mask_fp8_matches_oracle(orc, variant):
    w = inputs.Workload("m-fp8", 1, 8, 2, 1280, 128, 128, "fp8", 0.3, "stem", 44)
    q, k, v, sq, sk, sv = _inputs(w)
    B, N, Hq, d = q.shape
    nb = N // w.block
    mask = _random_mask(B, Hq, nb, 0.3, 7, empty=[(0, 3, 4)])
    out = bsa.bsa_prefill_mask(q, k, v, w.block, mask, q_scale=sq, k_scale=sk, v_scale=sv)
    bsa.bsa_check_device_error()
    rows = H.all_rows(B, Hq, N)
    ref, _, _ = _oracle(orc, q, k, v, w.block, mask, rows, sq, sk, sv)
    got = H.gather_rows(out, rows)
    assert H.rel_l2(got, ref) <= H.FP8_REL_L2
    empty = np.array([tuple(r) in _empty_rows(mask, N, w.block) for r in rows])
    assert empty.any() and np.all(got[empty] == 0.0)


def test_mask_to_lists_is_exact():
    """Integer work: the per-head lists equal numpy's nonzero() of each causal mask row."""
    B, Hq, nb = 2, 3, 300
    mask = _random_mask(B, Hq, nb, 0.2, 9, empty=[(0, 0, 5), (1, 2, 299)], full=[(1, 1, 17)])
    rp, ci = bsa.bsa_mask_to_lists(mask)
    torch.cuda.synchronize()
    m, rp, ci = mask.cpu().numpy(), rp.cpu().numpy(), ci.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            assert rp[b, h, 0] == 0
            for i in range(nb):
                want = np.nonzero(m[b, h, i, :i + 1])[0]
                assert rp[b, h, i + 1] - rp[b, h, i] == len(want), (b, h, i)
                assert np.array_equal(ci[b, h, rp[b, h, i]:rp[b, h, i + 1]], want), (b, h, i)


def test_mask_from_stem_lists_is_bit_identical(variant):
    """The mask holding exactly stem_select's lists gives bsa_prefill's output and LSE bit for bit
    (the lists the mask kernel builds are the same, in the same order)."""
    w = inputs.Workload("m-lists", 1, 8, 2, 2000, 128, 128, "bf16", 0.25, "stem", 45)
    q, k, v, *_ = _inputs(w)
    B, N, Hq, d = q.shape
    S = bsa.stem_score(q, k, v, w.block)
    nb = S.shape[-1]
    rp, ci = bsa.stem_select(S, [nb], w.density)
    ref, ref_lse = bsa.bsa_prefill(q, k, v, w.block, rp, ci, return_lse=True)
    mask = bsa.block_mask_buffer(B, Hq, nb, device=DEV)
    rpc, cic = rp.cpu(), ci.cpu()
    m = torch.zeros(B, Hq, nb, nb, dtype=torch.uint8)
    for h in range(Hq):
        for i in range(nb):
            m[0, h, i, cic[0, h, rpc[0, i]:rpc[0, i + 1]].long()] = 1
    mask.copy_(m.to(DEV))
    got, got_lse = bsa.bsa_prefill_mask(q, k, v, w.block, mask, return_lse=True)
    bsa.bsa_check_device_error()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(got_lse, ref_lse)
