"""Seeded synthetic workloads for the Stem block-sparse prefill path.

This module only draws and stores inputs; it holds none of the method's arithmetic, and
both the CUDA library's tests/bench and the CPU oracle take their inputs from here.

Recipe (the pages run their operator benchmark on synthetic shapes; no dataset is used):
  * Q, K, V start as N(0, 1) in fp32 from a ``torch.Generator`` seeded with
    ``42 + 1000 * config + sub`` (sub = 0 Q, 1 K, 2 V, 3 outlier channels, 4 sink direction,
    5 value log-norms, 6 page placement).
  * "stem" distribution (the GQA prefill workload): per kv head, 4 seeded outlier channels
    are scaled by 8 in Q and K; a seeded unit direction u per kv head is added to every
    query (2u) and to the first 64 keys (2 sqrt(d) u), which lifts the expected sink logit
    by about 4 at scale 1/sqrt(d); every value row is scaled by exp(eta), eta ~ N(0, 1) per
    (token, kv head), so value amplitudes are log-normal and OAM and score-only selection
    differ.
  * "blocky" distribution (only for the selection-quality record): keys carry a per-block
    topic; each query block attends to a seeded set of key blocks whose values have a per-block
    log-normal amplitude.  Per KV head, every key block j gets a seeded unit direction u_j and
    every key of the block adds a * u_j; every query head h and query block i get a seeded set
    J(h, i) = {0, i} plus up to 12 earlier blocks, and every query of block i adds a * u_j for j in
    J(h, i), with a = sqrt(4 sqrt(d)) so a matched key lifts the logit by about 4 at scale
    1/sqrt(d); every value row of block j is scaled by exp(eta_j), eta_j ~ N(0, 1) per (block, KV
    head).  Attention then falls on whole blocks, more of them than a 25% budget keeps, with
    different value amplitudes: the case the scoring metrics are meant to separate.
  * BF16 inputs are the fp32 draws rounded to nearest even; FP8 inputs are e4m3 codes of
    x / s with a per-tensor scale s = amax / 448 (torch's round-to-nearest-even cast).
  * Paged KV: 64-token pages, the pages of every sequence placed by a seeded permutation of
    a pool with 10% spare pages; spare pages hold NaN so a stray read shows up.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

FP8_MAX = 448.0


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int                      # per-sequence length (max length for varlen)
    d: int
    block: int
    dtype: str                  # "fp32" | "bf16" | "fp8"
    density: float
    dist: str                   # "normal" | "stem" | "blocky"
    config_id: int
    seqlens: list = field(default_factory=list)  # varlen lengths (paged workloads)
    page_size: int = 0          # > 0: paged KV cache

    @property
    def nb(self) -> int:
        return (self.N + self.block - 1) // self.block

    def seed(self, sub: int) -> int:
        return 42 + 1000 * self.config_id + sub


# The five workloads of the benchmark plan, in order (index == config id).
def tiny(density=0.25) -> Workload:
    return Workload("tiny-1k", 1, 1, 1, 1024, 64, 64, "fp32", density, "normal", 0)


def gqa_8k(density=0.25) -> Workload:
    return Workload("gqa-8k", 1, 32, 8, 8192, 128, 128, "bf16", density, "stem", 1)


def sweep_32k(density=0.25) -> Workload:
    return Workload("sweep-32k", 1, 32, 8, 32768, 128, 128, "bf16", density, "stem", 2)


def fp8_128k(density=0.25) -> Workload:
    return Workload("fp8-128k", 1, 64, 8, 131072, 128, 128, "fp8", density, "stem", 3)


def paged_varlen(density=0.25, seqlens=(16384, 32768, 65536, 131072)) -> Workload:
    seqlens = list(seqlens)
    return Workload("paged-varlen", len(seqlens), 32, 8, max(seqlens), 128, 128, "bf16", density,
                    "stem", 4, seqlens=seqlens, page_size=64)


def blocky_8k(density=0.25) -> Workload:
    """The 8K GQA shape with block-structured attention (the selection-quality record only)."""
    return Workload("blocky-8k", 1, 32, 8, 8192, 128, 128, "bf16", density, "blocky", 5)


def fp8_32k(density=0.25) -> Workload:
    """The FP8 workload at 32K tokens: a profiling case that still exceeds L2 (Q is 268 MB)."""
    return Workload("fp8-32k", 1, 64, 8, 32768, 128, 128, "fp8", density, "stem", 3)


WORKLOADS = {"tiny-1k": tiny, "gqa-8k": gqa_8k, "sweep-32k": sweep_32k, "fp8-128k": fp8_128k,
             "paged-varlen": paged_varlen, "fp8-32k": fp8_32k, "blocky-8k": blocky_8k}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def draw_fp32(w: Workload, B: int, N: int, device="cpu", seed_offset: int = 0):
    """fp32 Q [B,N,Hq,d], K, V [B,N,Hkv,d] following the workload's distribution."""
    d, Hq, Hkv = w.d, w.Hq, w.Hkv
    G = Hq // Hkv
    dev = torch.device(device)
    q = torch.randn(B, N, Hq, d, generator=_gen(dev, w.seed(0) + seed_offset), device=dev)
    k = torch.randn(B, N, Hkv, d, generator=_gen(dev, w.seed(1) + seed_offset), device=dev)
    v = torch.randn(B, N, Hkv, d, generator=_gen(dev, w.seed(2) + seed_offset), device=dev)
    if w.dist == "stem":
        gc = _gen(torch.device("cpu"), w.seed(3) + seed_offset)
        for hk in range(Hkv):
            ch = torch.randperm(d, generator=gc)[:4].to(dev)
            k[:, :, hk, ch] *= 8.0
            q[:, :, hk * G:(hk + 1) * G, ch] *= 8.0
        u = torch.randn(Hkv, d, generator=_gen(torch.device("cpu"), w.seed(4) + seed_offset))
        u = (u / u.norm(dim=-1, keepdim=True)).to(dev)
        q += 2.0 * u.repeat_interleave(G, dim=0)
        k[:, :64] += 2.0 * math.sqrt(d) * u
        eta = torch.randn(B, N, Hkv, 1, generator=_gen(dev, w.seed(5) + seed_offset), device=dev)
        v *= torch.exp(eta)
    elif w.dist == "blocky":
        nb = (N + w.block - 1) // w.block
        gc = _gen(torch.device("cpu"), w.seed(3) + seed_offset)
        u = torch.randn(B, Hkv, nb, d, generator=gc)
        u = u / u.norm(dim=-1, keepdim=True)
        amp = math.sqrt(4.0 * math.sqrt(d))
        sel = torch.zeros(B, Hq, nb, nb)
        for b in range(B):
            for h in range(Hq):
                for i in range(nb):
                    sel[b, h, i, 0] = 1.0
                    sel[b, h, i, i] = 1.0
                    if i > 1:
                        pick = torch.randperm(i - 1, generator=gc)[:12] + 1
                        sel[b, h, i, pick] = 1.0
        blk = torch.arange(N) // w.block
        ku = u.permute(0, 2, 1, 3)[:, blk]                                        # [B, N, Hkv, d]
        qtop = torch.einsum("bhij,bhjd->bhid", sel, u.repeat_interleave(G, dim=1))  # [B, Hq, nb, d]
        k += (amp * ku).to(dev)
        q += (amp * qtop.permute(0, 2, 1, 3)[:, blk]).to(dev)
        eta = torch.randn(B, nb, Hkv, generator=gc)
        v *= torch.exp(eta[:, blk]).unsqueeze(-1).to(dev)
    return q, k, v


def to_storage(x: torch.Tensor, dtype: str):
    """Round an fp32 tensor to the storage dtype.  Returns (tensor, per-tensor scale)."""
    if dtype == "fp32":
        return x.contiguous(), 1.0
    if dtype == "bf16":
        return x.to(torch.bfloat16).contiguous(), 1.0
    if dtype == "fp8":
        amax = float(x.abs().max())
        s = amax / FP8_MAX if amax > 0 else 1.0
        return (x / s).to(torch.float8_e4m3fn).contiguous(), s
    raise ValueError(dtype)


def make_inputs(w: Workload, device="cpu", N: int | None = None, storage: str | None = None,
                seed_offset: int = 0):
    """Dense-layout inputs [B, N, H, d] in the workload's storage dtype (or ``storage``)."""
    N = w.N if N is None else N
    storage = storage or w.dtype
    q, k, v = draw_fp32(w, w.B, N, device, seed_offset)
    (q, sq), (k, sk), (v, sv) = to_storage(q, storage), to_storage(k, storage), to_storage(v, storage)
    return dict(q=q, k=k, v=v, q_scale=sq, k_scale=sk, v_scale=sv, N=N)


def make_paged(w: Workload, device="cpu", seqlens=None, storage: str | None = None):
    """Varlen inputs with a paged KV cache.

    Returns packed Q [sum N, Hq, d] with cu_seqlens, per-sequence dense K/V views (for the
    scoring step), the page pool K/V [num_pages, page_size, Hkv, d] and page_table
    [B, max_pages] (int32, -1 where unused)."""
    seqlens = list(w.seqlens if seqlens is None else seqlens)
    storage = storage or w.dtype
    P = w.page_size
    B = len(seqlens)
    qs, ks, vs = [], [], []
    for b, n in enumerate(seqlens):
        q, k, v = draw_fp32(w, 1, n, device, seed_offset=17 * b)
        qs.append(q[0]); ks.append(k[0]); vs.append(v[0])
    q = torch.cat(qs, 0)
    # One per-tensor scale over all sequences, as a serving cache would have.
    kall, vall = torch.cat(ks, 0), torch.cat(vs, 0)
    q, sq = to_storage(q, storage)
    kq, sk = to_storage(kall, storage)
    vq, sv = to_storage(vall, storage)
    cu = [0]
    for n in seqlens:
        cu.append(cu[-1] + n)
    pages_per = [(n + P - 1) // P for n in seqlens]
    used = sum(pages_per)
    num_pages = used + max(1, used // 10)
    max_pages = max(pages_per)
    perm = torch.randperm(num_pages, generator=_gen(torch.device("cpu"), w.seed(6)))
    page_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    kc = torch.empty(num_pages, P, w.Hkv, w.d, dtype=kq.dtype, device=device)
    vc = torch.empty_like(kc)
    nan_fill = float("nan")
    if kq.dtype == torch.float8_e4m3fn:
        kc.view(torch.uint8).fill_(0x7F)   # e4m3 NaN
        vc.view(torch.uint8).fill_(0x7F)
    else:
        kc.fill_(nan_fill)
        vc.fill_(nan_fill)
    k_seq, v_seq = [], []
    kflat, vflat = kc.view(num_pages * P, w.Hkv, w.d), vc.view(num_pages * P, w.Hkv, w.d)
    off = 0
    for b, n in enumerate(seqlens):
        kb, vb = kq[cu[b]:cu[b + 1]], vq[cu[b]:cu[b + 1]]
        k_seq.append(kb); v_seq.append(vb)
        phys = perm[off:off + pages_per[b]].to(torch.int32)
        page_table[b, :pages_per[b]] = phys
        slots = (phys.to(torch.int64)[:, None] * P + torch.arange(P)[None, :]).reshape(-1)
        slots = slots.to(device)
        kflat[slots[:n]] = kb
        vflat[slots[:n]] = vb
        if n < slots.numel():   # tail slots of a partial last page hold finite zeros
            kflat[slots[n:]] = 0
            vflat[slots[n:]] = 0
        off += pages_per[b]
    return dict(q=q, cu_seqlens=torch.tensor(cu, dtype=torch.int32), seqlens=seqlens,
                k_seq=k_seq, v_seq=v_seq, k_cache=kc, v_cache=vc,
                page_table=page_table.to(device), num_pages=num_pages, max_pages=max_pages,
                q_scale=sq, k_scale=sk, v_scale=sv)
