"""Shared helpers of the parity tests: run the oracle on the same inputs the CUDA path sees
and compare with the tolerances the tests state."""
from __future__ import annotations

import math

import numpy as np
import torch

# Tolerances:
SCORE_REL = 1e-5          # scores: |gpu - oracle| <= 1e-5 * max(|oracle|, condition scale)
BF16_MAX_ABS = 2e-2       # BF16 attention output: |g - o| <= 2e-2 beyond the two BF16 roundings below
BF16_P_EPS = 2.0 ** -8    # relative error of the weights: P as a BF16 operand (2^-9) + the logits (2^-9)
BF16_REL_L2 = 1e-2
FP8_REL_L2 = 5e-2         # FP8 attention output
LSE_ABS = 1e-3            # natural-log LSE (fp32 log2/ex2 approximations, bf16-free)


def oracle_pool(orc, q, k, v, block, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    qb = orc.pool_mean(orc.view(q.cpu(), q_scale), B, N, Hq, d, block)
    kb = orc.pool_mean(orc.view(k.cpu(), k_scale), B, N, Hkv, d, block)
    vb = orc.pool_vnorm(orc.view(v.cpu(), v_scale), B, N, Hkv, d, block)
    return qb, kb, vb


def score_scale(qb, kb, vb, tau, metric):
    """Per-entry magnitude scale of the score computation: |tau| |Qbar_i| |Kbar_j| (+ |ln vbar_j|)."""
    Hq, Hkv = qb.shape[1], kb.shape[1]
    G = Hq // Hkv
    qn = np.linalg.norm(qb, axis=-1)                                  # [B,Hq,nb]
    kn = np.repeat(np.linalg.norm(kb, axis=-1), G, axis=1)            # [B,Hq,nb]
    vbr = np.repeat(vb, G, axis=1)
    sc = abs(tau) * qn[..., :, None] * kn[..., None, :]
    with np.errstate(divide="ignore"):
        if metric == 0:
            sc = sc + np.abs(np.log(vbr))[..., None, :]
        elif metric == 2:
            sc = sc * vbr[..., None, :]
    return sc


def assert_scores_close(gpu, ora, scale, nb):
    """Lower triangle: same finite/-inf pattern and |gpu - oracle| <= SCORE_REL * max(|o|, scale)."""
    g = gpu[..., :nb, :nb].double().cpu().numpy()
    o = ora[..., :nb, :nb]
    tri = np.broadcast_to(np.tril(np.ones((nb, nb), bool)), o.shape)
    fin = np.isfinite(o) & tri
    assert np.array_equal(np.isfinite(g) & tri, fin), "finite pattern differs"
    assert np.all(np.isneginf(g[np.isneginf(o) & tri])), "-inf entries differ"
    err = np.abs(g[fin] - o[fin])
    lim = (SCORE_REL * np.maximum(np.abs(o), scale[..., :nb, :nb]))[fin] + 1e-30
    worst = float(np.max(err / lim)) if err.size else 0.0
    assert worst <= 1.0, f"score error {worst:.3f} x tolerance"


def bf16_half_ulp(x):
    """Half the spacing of BF16 numbers at |x|: the largest error of rounding a real to BF16
    (8 significant bits: spacing 2^(e-7) in [2^e, 2^(e+1)))."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def bf16_bound(got, amp):
    """Per-element bound on |BF16 output - exact output|: the 2e-2 absolute target, plus what a
    BF16 tensor-core attention does to the exact result beyond it:
      * the weights: if every weight p_s moves by at most eps of itself, O moves by at most
        eps * sum_s p_s |v_s| / l = eps * amp (amp from the oracle).  The PV product takes P
        rounded to BF16 (eps = 2^-9), and the logits come from an fp32 tensor-core product
        Q K^T that the oracle computes exactly; at the large logits of the outlier channels that
        moves the weights by about as much again (measured on the 8K GQA workload: the largest
        (|g - o| - half ulp) / amp is 3.44e-3, for every kernel), so eps = 2^-8;
      * O is stored in BF16: at most half an ulp of the stored value."""
    return BF16_MAX_ABS + bf16_half_ulp(got) + BF16_P_EPS * np.asarray(amp, np.float64)


def assert_bf16_close(got, ref, amp):
    """Elementwise |got - ref| <= bf16_bound(got, amp) and rel-L2 <= 1e-2.  Returns the plain
    max-abs error, and the plain max-abs over outputs with |ref| <= 1, for reporting."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    excess = err - bf16_bound(got, amp)
    assert np.all(excess <= 0), f"BF16 bound exceeded by {float(np.max(excess)):.3e}"
    assert rel_l2(got, ref) <= BF16_REL_L2, rel_l2(got, ref)
    small = np.abs(ref) <= 1.0
    return float(err.max()) if err.size else 0.0, float(err[small].max()) if small.any() else 0.0


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def sample_rows(B, Hq, N, block, n_heads=4, n_rand=48, seed=0, heads=None):
    """(b, h, t) rows: block boundaries, the ragged tail, and random tokens."""
    rng = np.random.default_rng(seed)
    heads = heads if heads is not None else sorted(set(rng.choice(Hq, size=min(n_heads, Hq), replace=False).tolist()))
    toks = {0, 1, block - 1, min(block, N - 1), N - 1, N - 2, (N // block) * block - 1}
    toks |= set(rng.integers(0, N, size=n_rand).tolist())
    toks = sorted(t for t in toks if 0 <= t < N)
    return np.array([(b, h, t) for b in range(B) for h in heads for t in toks], np.int64)


def all_rows(B, Hq, N):
    return np.array([(b, h, t) for b in range(B) for h in range(Hq) for t in range(N)], np.int64)


def oracle_attention(orc, q, k, v, block, row_ptr, col_idx, tau, rows, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """(O, LSE, amp) of the oracle for the given (b, h, t) rows; amp is the softmax average of
    |v| that bounds the effect of rounding the weights (bf16_bound)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    return orc.attention_rows(orc.view(q.cpu(), q_scale), orc.view(k.cpu(), k_scale), orc.view(v.cpu(), v_scale),
                              N, Hq, Hkv, d, block, row_ptr.cpu().numpy(), col_idx.cpu().numpy(), tau, rows,
                              with_amp=True)


def gather_rows(out, rows):
    """out [B, N, Hq, d] -> [n_rows, d] in the (b, h, t) order of rows."""
    o = out.float().cpu()
    return np.stack([o[b, t, h].numpy() for b, h, t in rows])


def default_tau(d):
    return 1.0 / math.sqrt(d)
