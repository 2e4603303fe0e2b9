"""Pins of the fp64 CPU oracle against things other than itself.

Each test fixes one oracle function to the mathematics or to a library routine: brute force
on tiny inputs, closed forms, exhaustive decoding, the library dense causal attention, and a
hand-worked budget fixture.  Every test plants nothing in the CUDA path; the mutation tests
at the bottom plant mistakes in Python restatements that are fed to the same checks, to
show the checks catch them.
"""
import json
import math
from pathlib import Path

import numpy as np
import pytest
import torch

from block_sparse_attention_42_b200 import inputs

GOLDEN = Path(__file__).resolve().parent / "golden"


# ----------------------------------------------------------------------------- decoding


def test_e4m3_decode_exhaustive(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([orc.decode_e4m3(c) for c in range(256)])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_bf16_decode_exhaustive(orc):
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    x = orc.view(bits.view(torch.bfloat16).reshape(1, 65536, 1, 1))
    got = orc.decode(x, 1, 65536, 1, 1).reshape(-1)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_fp8_scale_applied(orc):
    x = torch.tensor([1.0, -2.0, 0.5, 448.0]).to(torch.float8_e4m3fn).reshape(1, 4, 1, 1)
    got = orc.decode(orc.view(x, scale=0.25), 1, 4, 1, 1).reshape(-1)
    assert got.tolist() == [0.25, -0.5, 0.125, 112.0]


# ----------------------------------------------------------------------------- pool + score


def _brute_scores(q, k, v, bs, tau, metric):
    """Mean over every (query token, key token) pair of the block pair of tau * q.k, plus the
    log of the mean value norm -- written as loops over token pairs, no pooling."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    nb = (N + bs - 1) // bs
    S = np.full((B, Hq, nb, nb), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for i in range(nb):
                for j in range(i + 1):
                    tot, cnt = 0.0, 0
                    for t in range(i * bs, min(N, (i + 1) * bs)):
                        for s in range(j * bs, min(N, (j + 1) * bs)):
                            tot += tau * float(np.dot(q[b, t, h], k[b, s, hk]))
                            cnt += 1
                    val = tot / cnt
                    norms = [np.sqrt(np.sum(v[b, s, hk] ** 2)) for s in range(j * bs, min(N, (j + 1) * bs))]
                    amp = sum(norms) / len(norms)
                    if metric == 0:
                        val += math.log(amp)
                    elif metric == 2:
                        val *= amp
                    S[b, h, i, j] = val
    return S


@pytest.mark.parametrize("metric", [0, 1, 2])
def test_pooled_score_equals_token_pair_mean(orc, metric):
    rng = np.random.default_rng(7)
    B, N, Hq, Hkv, D, bs = 2, 37, 4, 2, 8, 8   # ragged tail (37 = 4*8 + 5), GQA G=2
    q = rng.standard_normal((B, N, Hq, D))
    k = rng.standard_normal((B, N, Hkv, D))
    v = rng.standard_normal((B, N, Hkv, D)) * np.exp(rng.standard_normal((B, N, Hkv, 1)))
    tau = 1 / math.sqrt(D)
    qb = orc.pool_mean(orc.view(q), B, N, Hq, D, bs)
    kb = orc.pool_mean(orc.view(k), B, N, Hkv, D, bs)
    vb = orc.pool_vnorm(orc.view(v), B, N, Hkv, D, bs)
    S = orc.score(qb, kb, vb, tau, metric)
    ref = _brute_scores(q, k, v, bs, tau, metric)
    assert np.array_equal(np.isinf(S), np.isinf(ref))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(S[fin], ref[fin], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("metric", [0, 1, 2])
def test_group_score_is_mean_of_head_scores_and_of_token_pairs(orc, metric):
    """Group-shared selection: the group's score row equals (a) the mean of its G heads' score
    rows and (b) the brute-force mean over the group's heads and all token pairs of the block
    pair (+ the value term).  A wrong head-to-group mapping or a sum for the mean fails both."""
    rng = np.random.default_rng(11)
    B, N, Hq, Hkv, D, bs = 2, 29, 6, 2, 8, 8   # G = 3, ragged tail
    q = rng.standard_normal((B, N, Hq, D))
    k = rng.standard_normal((B, N, Hkv, D))
    v = rng.standard_normal((B, N, Hkv, D)) * np.exp(rng.standard_normal((B, N, Hkv, 1)))
    tau = 1 / math.sqrt(D)
    qb = orc.pool_mean(orc.view(q), B, N, Hq, D, bs)
    kb = orc.pool_mean(orc.view(k), B, N, Hkv, D, bs)
    vb = orc.pool_vnorm(orc.view(v), B, N, Hkv, D, bs)
    Sg = orc.score(orc.group_mean(qb, Hkv), kb, vb, tau, metric)          # [B, Hkv, nb, nb]
    Sh = orc.score(qb, kb, vb, tau, metric)                                # [B, Hq, nb, nb]
    G = Hq // Hkv
    nb = Sg.shape[-1]
    fin = np.isfinite(Sg)
    for hk in range(Hkv):
        mean_rows = Sh[:, hk * G:(hk + 1) * G].mean(axis=1)
        np.testing.assert_allclose(Sg[:, hk][fin[:, hk]], mean_rows[fin[:, hk]], rtol=1e-12, atol=1e-12)
    # brute force over heads x token pairs
    for b in range(B):
        for hk in range(Hkv):
            for i in range(nb):
                for j in range(i + 1):
                    tot, cnt = 0.0, 0
                    for h in range(hk * G, (hk + 1) * G):
                        for t in range(i * bs, min(N, (i + 1) * bs)):
                            for s_ in range(j * bs, min(N, (j + 1) * bs)):
                                tot += tau * float(np.dot(q[b, t, h], k[b, s_, hk]))
                                cnt += 1
                    val = tot / cnt
                    amp = vb[b, hk, j]
                    val = val + math.log(amp) if metric == 0 else (val * amp if metric == 2 else val)
                    assert Sg[b, hk, i, j] == pytest.approx(val, rel=1e-11, abs=1e-11)
    assert np.all(np.isneginf(Sg[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]]))
    # G = 1: the group mean is the identity
    assert np.array_equal(orc.group_mean(qb, Hq), qb)


def test_vnorm_closed_forms(orc):
    D, bs = 16, 4
    v = np.zeros((1, 8, 2, D))
    v[0, :4, 0, :] = -3.0                       # constant rows: norm = 3 sqrt(D)
    v[0, 4:, 0, 5] = np.arange(1, 5)            # one-hot rows: norms 1..4, mean 2.5
    v[0, :, 1, :] = 0.0                         # zero amplitude
    vb = orc.pool_vnorm(orc.view(v), 1, 8, 2, D, bs)
    assert vb[0, 0, 0] == pytest.approx(3 * math.sqrt(D), rel=1e-15)
    assert vb[0, 0, 1] == pytest.approx(2.5, rel=1e-15)
    assert vb[0, 1, 0] == 0.0
    # zero amplitude makes the OAM score -inf, so such a block can never be preferred
    S = orc.score(np.ones((1, 2, 2, D)), np.ones((1, 2, 2, D)), vb, 1.0, 0)
    assert S[0, 1, 1, 0] == -np.inf and S[0, 0, 1, 0] == pytest.approx(D + math.log(3 * math.sqrt(D)))


# ----------------------------------------------------------------------------- TPD budget


def test_tpd_hand_worked_fixture(orc):
    g = json.loads((GOLDEN / "tpd_nb8_rho050.json").read_text())
    k, tot = orc.tpd_budget(g["nb"], g["density"], g["decay"])
    assert tot == g["total"]
    assert k.tolist() == g["k"]


@pytest.mark.parametrize("nb,density,total", [(16, 0.25, 34), (64, 0.25, 520), (256, 0.10, 3290),
                                              (256, 0.20, 6579), (256, 0.25, 8224), (256, 0.50, 16448),
                                              (256, 0.80, 26317), (256, 1.0, 32896), (1024, 0.25, 131200),
                                              (16, 0.10, 31)])
def test_tpd_totals(orc, nb, density, total):
    k, tot = orc.tpd_budget(nb, density, 0.5)
    assert tot == total and int(k.sum()) == total


def _exact_share_solution(nb, Kstar, beta):
    """Independent solve of sum_i min(n_i, max(m_i, c*w_i)) = K* by walking the breakpoints
    of the piecewise-linear total (no bisection, no fixed point)."""
    n = np.arange(1, nb + 1, dtype=np.float64)
    m = np.where(n == 1, 1.0, 2.0)
    w = np.sqrt(n) if beta == 0.5 else n
    bps = np.unique(np.concatenate([m / w, n / w, [0.0]]))
    tot = lambda c: np.minimum(n, np.maximum(m, c * w)).sum()
    for lo, hi in zip(bps[:-1], bps[1:]):
        if tot(lo) <= Kstar <= tot(hi):
            if tot(hi) == tot(lo):
                return lo
            mid = 0.5 * (lo + hi)
            active = (m < mid * w) & (mid * w < n)
            slope = w[active].sum()
            return lo + (Kstar - tot(lo)) / slope
    return bps[-1]


@pytest.mark.parametrize("nb", [1, 2, 3, 7, 16, 64, 100, 257, 1024])
@pytest.mark.parametrize("density", [0.05, 0.1, 0.25, 0.5, 0.8, 1.0])
@pytest.mark.parametrize("beta", [0.0, 0.5])
def test_tpd_invariants_and_apportionment(orc, nb, density, beta):
    k, tot = orc.tpd_budget(nb, density, beta)
    n = np.arange(1, nb + 1)
    m = np.where(n == 1, 1, 2)
    T = nb * (nb + 1) // 2
    Kstar = min(max(math.floor(density * T + 0.5), int(m.sum())), T)
    assert tot == Kstar and int(k.sum()) == Kstar
    assert np.all(k >= m) and np.all(k <= n)
    if density == 1.0:
        assert np.array_equal(k, n)
    # each row gets floor or ceil of its exact real-valued share (largest-remainder rounding)
    c = _exact_share_solution(nb, Kstar, beta)
    w = np.sqrt(n) if beta == 0.5 else n
    t = np.minimum(n, np.maximum(m, c * w))
    assert np.all(k >= np.floor(t - 1e-9)) and np.all(k <= np.ceil(t + 1e-9))
    # the real-valued keep ratio never increases with position
    ratio = t / n
    assert np.all(np.diff(ratio) <= 1e-12)


def test_tpd_rejects_bad_args(orc):
    for args in [(0, 0.5, 0.5), (8, 0.0, 0.5), (8, 1.5, 0.5), (8, 0.5, 0.3), (8, float("nan"), 0.5)]:
        with pytest.raises(ValueError):
            orc.tpd_budget(*args)


# ----------------------------------------------------------------------------- selection


def _brute_row(srow, i, k_i):
    if i == 0:
        return [0]
    cands = [(-(-np.inf if np.isnan(srow[j]) else srow[j]), j) for j in range(1, i)]
    cands.sort()
    keep = sorted([0, i] + [j for _, j in cands[: k_i - 2]])
    return keep


def test_select_row_brute_force(orc):
    rng = np.random.default_rng(3)
    for trial in range(300):
        i = int(rng.integers(0, 40))
        srow = rng.standard_normal(i + 1)
        if trial % 3 == 0 and i > 2:   # inject ties, NaN, signed zeros, -inf
            srow[rng.integers(1, i, size=3)] = 0.5
            srow[rng.integers(1, i)] = np.nan
            srow[rng.integers(1, i)] = -0.0
            srow[rng.integers(1, i)] = 0.0
            srow[rng.integers(1, i)] = -np.inf
        k_i = 1 if i == 0 else int(rng.integers(2, i + 2))
        got = orc.select_row(srow, i, k_i).tolist()
        assert got == _brute_row(srow, i, k_i)
        assert got == sorted(set(got)) and got[0] == 0 and got[-1] == i


def test_select_kept_dominate_dropped(orc):
    rng = np.random.default_rng(11)
    B, Hq, nb = 2, 3, 24
    S = rng.standard_normal((B, Hq, nb, nb))
    S[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] = -np.inf
    row_ptr, col_idx = orc.select(S, [nb, 17], 0.3)
    for b, nbb in enumerate([nb, 17]):
        k, _ = orc.tpd_budget(nbb, 0.3)
        assert np.array_equal(np.diff(row_ptr[b, : nbb + 1]), k)
        for h in range(Hq):
            for i in range(nbb):
                lst = col_idx[b, h, row_ptr[b, i]:row_ptr[b, i + 1]]
                mid = [j for j in lst if 0 < j < i]
                dropped = [j for j in range(1, i) if j not in lst]
                if mid and dropped:
                    assert min(S[b, h, i, mid]) >= max(S[b, h, i, dropped])


# ----------------------------------------------------------------------------- attention


def _dense_lists(B, Hq, nb):
    k = np.arange(1, nb + 1, dtype=np.int32)
    rp = np.concatenate([[0], np.cumsum(k)]).astype(np.int32)
    ci = np.concatenate([np.arange(i + 1) for i in range(nb)]).astype(np.int32)
    return np.tile(rp, (B, 1)), np.tile(ci, (B, Hq, 1))


def _all_rows(B, Hq, N):
    return np.array([(b, h, t) for b in range(B) for h in range(Hq) for t in range(N)], np.int64)


def test_density_one_equals_library_causal_sdpa(orc):
    w = inputs.Workload("pin", 2, 4, 2, 45, 16, 8, "fp32", 1.0, "stem", 99)
    d = inputs.make_inputs(w)
    q, k, v = d["q"].double(), d["k"].double(), d["v"].double()
    B, N, Hq, Hkv, D, bs = 2, 45, 4, 2, 16, 8
    nb = (N + bs - 1) // bs
    rp, ci = _dense_lists(B, Hq, nb)
    tau = 1 / math.sqrt(D)
    out, lse = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, rp, ci, tau,
                                  _all_rows(B, Hq, N))
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.repeat_interleave(G, 2).transpose(1, 2), v.repeat_interleave(G, 2).transpose(1, 2),
        is_causal=True, scale=tau).transpose(1, 2)          # [B, N, Hq, D]
    ref = ref.permute(0, 2, 1, 3).reshape(-1, D).numpy()     # rows ordered (b, h, t)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    logits = torch.einsum("bthd,bshd->bhts", q, k.repeat_interleave(G, 2)) * tau
    mask = torch.ones(N, N, dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), -1).reshape(-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_sparse_equals_library_masked_sdpa(orc):
    w = inputs.Workload("pin", 1, 2, 1, 50, 8, 8, "fp32", 0.3, "normal", 98)
    d = inputs.make_inputs(w)
    q, k, v = d["q"].double(), d["k"].double(), d["v"].double()
    B, N, Hq, Hkv, D, bs = 1, 50, 2, 1, 8, 8
    nb = (N + bs - 1) // bs
    rng = np.random.default_rng(5)
    S = rng.standard_normal((B, Hq, nb, nb))
    rp, ci = orc.select(S, [nb], 0.3)
    tau = 0.37
    out, _ = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, rp, ci, tau,
                                _all_rows(B, Hq, N))
    for h in range(Hq):
        mask = torch.zeros(N, N, dtype=torch.bool)
        for i in range(nb):
            for j in ci[0, h, rp[0, i]:rp[0, i + 1]]:
                mask[i * bs:(i + 1) * bs, j * bs:(j + 1) * bs] = True
        mask &= torch.ones(N, N, dtype=torch.bool).tril()
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, :, h], k[:, :, 0], v[:, :, 0], attn_mask=mask, scale=tau)[0]
        np.testing.assert_allclose(out[h * N:(h + 1) * N], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_skipped_blocks_are_irrelevant(orc):
    w = inputs.Workload("pin", 1, 1, 1, 64, 8, 8, "fp32", 0.3, "normal", 97)
    d = inputs.make_inputs(w)
    q, k, v = d["q"].double(), d["k"].double().clone(), d["v"].double().clone()
    nb = 8
    S = np.random.default_rng(1).standard_normal((1, 1, nb, nb))
    rp, ci = orc.select(S, [nb], 0.3)
    rows = np.array([(0, 0, 63)], np.int64)              # last query row, block 7
    base, _ = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), 64, 1, 1, 8, 8, rp, ci, 0.5, rows)
    kept = set(ci[0, 0, rp[0, 7]:rp[0, 8]].tolist())
    for j in range(nb):
        if j not in kept:
            k[0, j * 8:(j + 1) * 8] = 1e4
            v[0, j * 8:(j + 1) * 8] = float("nan")
    pert, _ = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), 64, 1, 1, 8, 8, rp, ci, 0.5, rows)
    assert np.array_equal(base, pert)


def test_amp_equals_library_sdpa_on_absolute_values(orc):
    """The amp output (softmax average of |v| per output element) equals the library's SDPA
    run with |V| as the values, under the same block-sparse causal mask; and it bounds |O|."""
    w = inputs.Workload("pin", 1, 2, 1, 50, 8, 8, "fp32", 0.3, "stem", 95)
    d = inputs.make_inputs(w)
    q, k, v = d["q"].double(), d["k"].double(), d["v"].double()
    B, N, Hq, Hkv, D, bs = 1, 50, 2, 1, 8, 8
    nb = (N + bs - 1) // bs
    S = np.random.default_rng(6).standard_normal((B, Hq, nb, nb))
    rp, ci = orc.select(S, [nb], 0.3)
    tau = 0.41
    out, _, amp = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, rp, ci, tau,
                                     _all_rows(B, Hq, N), with_amp=True)
    for h in range(Hq):
        mask = torch.zeros(N, N, dtype=torch.bool)
        for i in range(nb):
            for j in ci[0, h, rp[0, i]:rp[0, i + 1]]:
                mask[i * bs:(i + 1) * bs, j * bs:(j + 1) * bs] = True
        mask &= torch.ones(N, N, dtype=torch.bool).tril()
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, :, h], k[:, :, 0], v[:, :, 0].abs(), attn_mask=mask, scale=tau)[0]
        np.testing.assert_allclose(amp[h * N:(h + 1) * N], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(np.abs(out) <= amp * (1 + 1e-12))
    # the block-mask form gives the same amp for the same selection
    mask = np.zeros((B, Hq, nb, nb), np.uint8)
    for h in range(Hq):
        for i in range(nb):
            mask[0, h, i, ci[0, h, rp[0, i]:rp[0, i + 1]]] = 1
    _, _, amp_m = orc.attention_rows_mask(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, mask, tau,
                                          _all_rows(B, Hq, N), with_amp=True)
    np.testing.assert_allclose(amp_m, amp, rtol=1e-13, atol=0)


def test_single_key_closed_form(orc):
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 16, 1, 4)); k = rng.standard_normal((1, 16, 1, 4)); v = rng.standard_normal((1, 16, 1, 4))
    rp, ci = _dense_lists(1, 1, 2)
    out, lse = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), 16, 1, 1, 4, 8, rp, ci, 0.7,
                                  np.array([(0, 0, 0)], np.int64))
    assert np.array_equal(out[0], v[0, 0, 0])             # one allowed key: weight exactly 1
    assert lse[0] == pytest.approx(0.7 * float(q[0, 0, 0] @ k[0, 0, 0]), rel=1e-15)
    _, _, amp = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), 16, 1, 1, 4, 8, rp, ci, 0.7,
                                   np.array([(0, 0, 0)], np.int64), with_amp=True)
    assert np.array_equal(amp[0], np.abs(v[0, 0, 0]))


# ----------------------------------------------------------------------------- threshold skip


def test_skip_with_lambda_zero_is_plain_attention(orc):
    w = inputs.Workload("pin", 1, 4, 2, 96, 16, 8, "fp32", 0.4, "stem", 94)
    d = inputs.make_inputs(w)
    q, k, v = d["q"].double(), d["k"].double(), d["v"].double()
    B, N, Hq, Hkv, D, bs = 1, 96, 4, 2, 16, 8
    nb = N // bs
    S = np.random.default_rng(8).standard_normal((B, Hq, nb, nb))
    rp, ci = orc.select(S, [nb], 0.4)
    rows = _all_rows(B, Hq, N)
    ref, ref_lse = orc.attention_rows(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, rp, ci, 0.3, rows)
    out, lse, skipped = orc.attention_rows_skip(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, rp, ci,
                                                0.3, 0.0, rows)
    assert np.array_equal(out, ref) and np.array_equal(lse, ref_lse) and not skipped.any()
    # the number of skipped blocks never falls as lambda grows
    prev = np.zeros_like(skipped)
    for lam in (1e-6, 1e-3, 1e-1, 0.5, 1.0):
        _, _, sk = orc.attention_rows_skip(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, rp, ci, 0.3,
                                           lam, rows)
        assert np.all(sk >= prev)
        prev = sk
    assert prev.any()


def test_skip_closed_form():
    """Two blocks of 8 keys.  Block 0's keys all give the logit 10, block 1's keys the logit 0.
    Row t in block 1 visits block 0 then block 1: block 1's max trails by 10, so it is skipped
    for lambda = e^-9 (O = mean of block 0's values) and kept for lambda = e^-11 (O = the two
    blocks weighted e^10 : 1 per key)."""
    import oracle as orc
    N, D, bs = 16, 4, 8
    q = np.zeros((1, N, 1, D)); q[0, :, 0, 0] = 1.0
    k = np.zeros((1, N, 1, D)); k[0, :8, 0, 0] = 10.0
    v = np.random.default_rng(3).standard_normal((1, N, 1, D))
    rp = np.array([[0, 1, 3]], np.int32)
    ci = np.array([[[0, 0, 1]]], np.int32)
    for t in (8, 11, 15):
        rows = np.array([(0, 0, t)], np.int64)
        o, lse, sk = orc.attention_rows_skip(orc.view(q), orc.view(k), orc.view(v), N, 1, 1, D, bs, rp, ci, 1.0,
                                             math.exp(-9.0), rows)
        assert sk[0] == 1
        np.testing.assert_allclose(o[0], v[0, :8, 0].mean(axis=0), rtol=1e-13, atol=1e-14)
        assert lse[0] == pytest.approx(10.0 + math.log(8.0), rel=1e-15)
        o, lse, sk = orc.attention_rows_skip(orc.view(q), orc.view(k), orc.view(v), N, 1, 1, D, bs, rp, ci, 1.0,
                                             math.exp(-11.0), rows)
        n1 = t - 7
        wts = np.array([math.exp(10.0)] * 8 + [1.0] * n1)
        ref = (wts[:, None] * v[0, :t + 1, 0]).sum(axis=0) / wts.sum()
        assert sk[0] == 0
        np.testing.assert_allclose(o[0], ref, rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------- block-mask input


def test_mask_all_ones_equals_library_causal_sdpa(orc):
    """An all-ones block mask (above the diagonal too) is dense causal attention."""
    w = inputs.Workload("pin", 2, 4, 2, 45, 16, 8, "fp32", 1.0, "stem", 96)
    d = inputs.make_inputs(w)
    q, k, v = d["q"].double(), d["k"].double(), d["v"].double()
    B, N, Hq, Hkv, D, bs = 2, 45, 4, 2, 16, 8
    nb = (N + bs - 1) // bs
    mask = np.ones((B, Hq, nb, 16), np.uint8)
    tau = 1 / math.sqrt(D)
    out, lse = orc.attention_rows_mask(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, mask, tau,
                                       _all_rows(B, Hq, N))
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.repeat_interleave(G, 2).transpose(1, 2), v.repeat_interleave(G, 2).transpose(1, 2),
        is_causal=True, scale=tau).transpose(1, 2)
    ref = ref.permute(0, 2, 1, 3).reshape(-1, D).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    logits = torch.einsum("bthd,bshd->bhts", q, k.repeat_interleave(G, 2)) * tau
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~causal, float("-inf")), -1).reshape(-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_mask_diagonal_only_equals_sdpa_within_the_block(orc):
    """Only the diagonal block kept: each block is causal attention over its own keys."""
    rng = np.random.default_rng(11)
    B, N, Hq, Hkv, D, bs = 1, 37, 2, 1, 8, 8
    nb = (N + bs - 1) // bs
    q = rng.standard_normal((B, N, Hq, D)); k = rng.standard_normal((B, N, Hkv, D)); v = rng.standard_normal((B, N, Hkv, D))
    mask = np.zeros((B, Hq, nb, 16), np.uint8)
    for i in range(nb):
        mask[:, :, i, i] = 1
    tau = 0.41
    out, _ = orc.attention_rows_mask(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, mask, tau,
                                     _all_rows(B, Hq, N))
    out = out.reshape(Hq, N, D)
    for h in range(Hq):
        for i in range(nb):
            lo, hi = i * bs, min(N, (i + 1) * bs)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[0, lo:hi, h]), torch.from_numpy(k[0, lo:hi, 0]), torch.from_numpy(v[0, lo:hi, 0]),
                is_causal=True, scale=tau)
            np.testing.assert_allclose(out[h, lo:hi], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_mask_empty_row_and_upper_triangle(orc):
    """A row keeping nothing gives O = 0, LSE = -inf; entries above the diagonal change nothing."""
    rng = np.random.default_rng(12)
    B, N, Hq, Hkv, D, bs = 1, 32, 1, 1, 4, 8
    nb = 4
    q = rng.standard_normal((B, N, Hq, D)); k = rng.standard_normal((B, N, Hkv, D)); v = rng.standard_normal((B, N, Hkv, D))
    mask = np.zeros((B, Hq, nb, 16), np.uint8)
    mask[0, 0, 2, :3] = [1, 0, 1]                            # row 2: blocks 0 and 2
    rows = _all_rows(B, Hq, N)
    out, lse = orc.attention_rows_mask(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, mask, 0.5, rows)
    empty = [t for t in range(N) if t // bs != 2]
    assert np.all(out[empty] == 0.0) and np.all(np.isneginf(lse[empty]))
    upper = mask.copy()
    upper[0, 0, 0, 1:] = 7                                   # above the diagonal
    upper[0, 0, 2, 3] = 1
    out2, lse2 = orc.attention_rows_mask(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, upper, 0.5, rows)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    # row 2 against the library with the token mask written out
    tm = torch.zeros(bs, N, dtype=torch.bool)
    tm[:, 0:8] = True
    tm[:, 16:24] = True
    tm &= torch.ones(N, N, dtype=torch.bool).tril()[16:24]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0, 16:24, 0]), torch.from_numpy(k[0, :, 0]), torch.from_numpy(v[0, :, 0]),
        attn_mask=tm, scale=0.5)
    np.testing.assert_allclose(out[16:24], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_mask_per_head_equals_library_masked_sdpa(orc):
    """Random, different masks per query head (GQA): each head against the library's SDPA with
    the token mask written out; rows that keep nothing are 0 / -inf."""
    rng = np.random.default_rng(13)
    B, N, Hq, Hkv, D, bs = 1, 45, 4, 2, 8, 8
    nb = (N + bs - 1) // bs
    q = rng.standard_normal((B, N, Hq, D)); k = rng.standard_normal((B, N, Hkv, D)); v = rng.standard_normal((B, N, Hkv, D))
    mask = (rng.random((B, Hq, nb, 16)) < 0.4).astype(np.uint8)
    mask[0, 1, 3, :] = 0                                     # an empty row
    tau = 0.29
    out, lse = orc.attention_rows_mask(orc.view(q), orc.view(k), orc.view(v), N, Hq, Hkv, D, bs, mask, tau,
                                       _all_rows(B, Hq, N))
    out, lse = out.reshape(Hq, N, D), lse.reshape(Hq, N)
    G = Hq // Hkv
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    for h in range(Hq):
        tm = torch.zeros(N, N, dtype=torch.bool)
        for i in range(nb):
            for j in range(nb):
                if mask[0, h, i, j]:
                    tm[i * bs:(i + 1) * bs, j * bs:(j + 1) * bs] = True
        tm &= causal
        live = tm.any(-1).numpy()
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, :, h]), torch.from_numpy(k[0, :, h // G]), torch.from_numpy(v[0, :, h // G]),
            attn_mask=tm, scale=tau).numpy()
        np.testing.assert_allclose(out[h][live], ref[live], rtol=1e-12, atol=1e-12)
        assert np.all(out[h][~live] == 0.0) and np.all(np.isneginf(lse[h][~live]))
    assert np.all(np.isneginf(lse[1, 24:32])) and np.all(out[1, 24:32] == 0.0)   # the emptied row


def test_effective_flop_counts_pairs(orc):
    for N, bs in [(64, 8), (61, 8), (128, 64)]:
        nb = (N + bs - 1) // bs
        rp, ci = _dense_lists(1, 3, nb)
        assert orc.effective_flop(N, 3, 16, bs, rp, ci) == 4 * 16 * 3 * N * (N + 1) / 2


# ----------------------------------------------------------------------------- mutation checks


def test_checks_catch_planted_mistakes(orc):
    """Plausible slips (a transposed head mapping, a dropped log term, a sum instead of a mean)
    planted in a Python restatement must fail the same brute-force comparison."""
    rng = np.random.default_rng(9)
    B, N, Hq, Hkv, D, bs = 1, 24, 4, 2, 4, 8
    q = rng.standard_normal((B, N, Hq, D)); k = rng.standard_normal((B, N, Hkv, D))
    v = rng.standard_normal((B, N, Hkv, D)) * 3
    tau = 0.5
    ref = _brute_scores(q, k, v, bs, tau, 0)
    nb = N // bs
    qb = q.reshape(B, nb, bs, Hq, D).mean(2).transpose(0, 2, 1, 3)
    kb = k.reshape(B, nb, bs, Hkv, D).mean(2).transpose(0, 2, 1, 3)
    vb = np.sqrt((v ** 2).sum(-1)).reshape(B, nb, bs, Hkv).mean(2).transpose(0, 2, 1)

    def scores(head_map, use_log, qpool):
        S = np.full((B, Hq, nb, nb), -np.inf)
        for h in range(Hq):
            hk = head_map(h)
            for i in range(nb):
                for j in range(i + 1):
                    S[0, h, i, j] = tau * qpool[0, h, i] @ kb[0, hk, j] + (math.log(vb[0, hk, j]) if use_log else 0)
        return S

    good = scores(lambda h: h // 2, True, qb)
    fin = np.isfinite(ref)
    assert np.allclose(good[fin], ref[fin], rtol=1e-12)
    for bad in [scores(lambda h: h % 2, True, qb), scores(lambda h: h // 2, False, qb),
                scores(lambda h: h // 2, True, qb * bs)]:
        assert not np.allclose(bad[fin], ref[fin], rtol=1e-6)


def test_mask_checks_catch_planted_mistakes():
    """Slips a block-mask attention could make (the KV head's mask instead of the query head's,
    the key's block as the mask row, no causal cut inside the diagonal block) planted in a
    Python restatement fail the library-SDPA comparison that pins the oracle's mask function."""
    rng = np.random.default_rng(14)
    B, N, Hq, Hkv, D, bs = 1, 24, 4, 2, 4, 8
    nb = N // bs
    G = Hq // Hkv
    q = rng.standard_normal((N, Hq, D)); k = rng.standard_normal((N, Hkv, D)); v = rng.standard_normal((N, Hkv, D))
    mask = (rng.random((Hq, nb, nb)) < 0.5).astype(np.uint8)
    for i in range(nb):
        mask[:, i, 0] = 1                                    # every row keeps something
    tau = 0.6

    def attend(head_for_mask, row_of, causal):
        out = np.zeros((Hq, N, D))
        for h in range(Hq):
            for t in range(N):
                keys = [s for s in range(N) if mask[head_for_mask(h), row_of(t, s), s // bs]
                        and (s <= t if causal else s // bs <= t // bs)]
                lg = np.array([tau * q[t, h] @ k[s, h // G] for s in keys])
                w = np.exp(lg - lg.max())
                out[h, t] = (w[:, None] * v[keys, h // G]).sum(0) / w.sum()
        return out

    ref = np.zeros((Hq, N, D))
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    for h in range(Hq):
        tm = torch.from_numpy(np.kron(mask[h], np.ones((bs, bs), np.uint8)).astype(bool)) & causal
        ref[h] = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, h]), torch.from_numpy(k[:, h // G]), torch.from_numpy(v[:, h // G]),
            attn_mask=tm, scale=tau).numpy()
    good = attend(lambda h: h, lambda t, s: t // bs, True)
    np.testing.assert_allclose(good, ref, rtol=1e-12, atol=1e-12)
    for bad in [attend(lambda h: h // G, lambda t, s: t // bs, True),      # KV head's mask
                attend(lambda h: h, lambda t, s: s // bs, True),           # key block as the row
                attend(lambda h: h, lambda t, s: t // bs, False)]:         # no causal cut
        assert not np.allclose(bad, ref, rtol=1e-6, atol=1e-9)
