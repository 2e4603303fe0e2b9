"""Benchmark of the Stem block-sparse prefill hot path on B200.

One step = the whole path on one batch of synthetic input resident in HBM:
  stem_score (pool + score GEMM) -> stem_select (TPD budget + top-k) -> bsa_prefill.
Default workload: 128K tokens, 64 query / 8 KV heads, head_dim 128, block 128, FP8 e4m3 Q/K/V
with per-tensor scales, BF16 output, TPD density 25% (decay 1/2).

value = effective attention TFLOP/s of the whole step (4 * d * unmasked token pairs inside
the kept blocks, summed over heads and ranks, divided by the max-over-ranks step time).

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]
Under torchrun every rank runs an independent problem (seed offset = rank): weak scaling,
no data-path collective.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "bsa_prefill ms + effective TFLOPS @128K, 25% density, 1×B200; select ms"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="fp8-128k")
    p.add_argument("--density", type=float, default=0.25)
    p.add_argument("--no-dense", action="store_true", help="skip the density-1 ideal-line measurement")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-split", type=int, default=1,
                   help="query-head chunks per KV-head group in the pipelined end-to-end step (1 measured "
                        "fastest at fp8-128k: 56.0 ms vs 57.3 / 62.3 for 2 / 4)")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    p.add_argument("--no-mask", action="store_true", help="skip the block-mask input measurement")
    p.add_argument("--no-sweeps", action="store_true",
                   help="skip the density, length and paged-varlen sweeps of bsa_prefill")
    p.add_argument("--sweep-reps", type=int, default=3, help="timed calls per sweep point")
    p.add_argument("--no-skip", action="store_true", help="skip the threshold-skip (bsa_prefill_skip) measurement")
    p.add_argument("--no-fused", action="store_true", help="skip the stem_score_select measurement")
    p.add_argument("--no-group", action="store_true",
                   help="skip the group-shared selection + GQA-packed attention measurement")
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers


def effective_flop(row_ptr: torch.Tensor, col_idx: torch.Tensor, seqlens, block: int, d: int) -> float:
    """4 * d * (unmasked token pairs inside kept blocks), summed over sequences and heads.
    Off-diagonal kept block: |I_i| * |I_j| pairs; diagonal block: |I_i| (|I_i| + 1) / 2."""
    rp = row_ptr.cpu().numpy().astype(np.int64)
    ci = col_idx.cpu().numpy().astype(np.int64)
    total = 0.0
    for b, N in enumerate(seqlens):
        nb = (N + block - 1) // block
        sizes = np.minimum(block, N - np.arange(nb) * block)           # tokens per block
        rows = np.repeat(np.arange(nb), np.diff(rp[b, : nb + 1]))      # query block of each entry
        cols = ci[b, :, : rp[b, nb]]                                   # [Hq, K]
        qs = sizes[rows][None, :]
        ks = sizes[cols]
        diag = cols == rows[None, :]
        pairs = np.where(diag, qs * (qs + 1) // 2, qs * ks)
        total += float(pairs.sum())
    return 4.0 * d * total


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, power, throttle reasons)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def reduce_max(x: float, world: int, device) -> float:
    """Max over ranks of a per-rank timing (the only collective: not on the data path)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(eff_flop_per_rank: float, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank runs its own problem of the same size."""
    return eff_flop_per_rank * world / (ms_per_step * 1e-3) / 1e12


# DRAM bytes per token moved by one bsa_prefill launch (dram__bytes_read.sum +
# dram__bytes_write.sum of one ncu capture on the fp8-32k workload, divided by its 32768
# tokens).  Q, K, V are read and O written once per token, so the traffic of a launch is
# linear in B x N.  Keyed by attention kernel and (dtype, Hq, Hkv, d) of the capture; any
# other kernel or shape reports null.
TRAFFIC_PER_TOKEN = {
    ("ws3", "fp8", 64, 8, 128): (358.912512e6 + 485.153280e6) / 32768,
}
ATTN_DEFAULT = "ws3"  # the kernel bsa_prefill runs when BSA_ATTN_VARIANT is unset


def attn_traffic(fp8: bool, B: int, N: int, Hq: int, Hkv: int, D: int):
    kern = os.environ.get("BSA_ATTN_VARIANT") or ATTN_DEFAULT
    per = TRAFFIC_PER_TOKEN.get((kern, "fp8" if fp8 else "bf16", Hq, Hkv, D))
    return None if per is None else per * B * N


def mufu_roofline(res, device):
    """exp2 throughput of bsa_prefill against the MUFU peak (bound 'alu')."""
    props = torch.cuda.get_device_properties(device)
    sms = props.multi_processor_count
    mhz = (res.get("clocks") or {}).get("sm_mhz") or 1965.0
    blk = res["w"].block
    n_exp = float(res["kstar"]) * res["Hq"] * res["B"] * blk * blk  # kept blocks x block^2 per head
    achieved = n_exp / (res["attn_ms_mean"] * 1e-3) / 1e12
    peak = 16.0 * sms * mhz * 1e6 / 1e12
    return {"bound": "alu", "unit": "Texp2/s", "achieved": achieved, "peak": peak, "frac": achieved / peak,
            "peak_source": f"16 exp2/clk/SM (MUFU, measured) x {sms} SMs x {mhz:.0f} MHz sampled",
            "kernel": "bsa_prefill"}


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        j = json.loads(p.read_text())
        return j, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------------------------- sweeps

SWEEP_DENSITIES = (0.10, 0.20, 0.25, 0.50, 0.80, 1.00)
SWEEP_LENGTHS = (8192, 16384, 32768, 65536, 131072, 262144)


def _time_calls(fn, reps, stream):
    """Mean ms of `reps` back-to-back calls (CUDA events on the launching stream), after one
    untimed call."""
    fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def density_sweep(bsa, q, k, v, scores, block, seqlens, reps, stream, scale_kw):
    """bsa_prefill over TPD lists at each density of SWEEP_DENSITIES, same inputs and scores:
    ms, effective TFLOP/s and the ideal-line ratio ms / (dense ms x rho_eff), where rho_eff is
    the ratio of effective FLOP to the density-1 (dense causal) FLOP."""
    B, N, Hq, D = q.shape
    nbp = [(n + block - 1) // block for n in seqlens]
    out = torch.empty(B, N, Hq, D, dtype=torch.bfloat16, device=q.device)
    pts = []
    for rho in SWEEP_DENSITIES:
        rp, ci = bsa.stem_select(scores, nbp, rho, 0.5)
        ms = _time_calls(lambda: bsa.bsa_prefill(q, k, v, block, rp, ci, out=out, **scale_kw), reps, stream)
        flop = effective_flop(rp, ci, seqlens, block, D)
        pts.append({"density": rho, "ms": ms, "effective_flop": flop,
                    "effective_tflops": flop / (ms * 1e-3) / 1e12})
        del rp, ci
    dense = pts[-1]
    for pt in pts:
        pt["rho_eff"] = pt["effective_flop"] / dense["effective_flop"]
        pt["ideal_line_ratio"] = pt["ms"] / (dense["ms"] * pt["rho_eff"])
    bsa.bsa_check_device_error(q.device)
    return pts


def run_sweeps(args, device, main):
    """The pages' operator claims as measurements: latency linear in density (skip overhead),
    stable throughput from 8K to 256K tokens at 75% sparsity, contiguous and paged KV, and the
    paged varlen batch."""
    import block_sparse_attention_42_b200 as bsa
    from block_sparse_attention_42_b200 import inputs
    stream = torch.cuda.current_stream(device)
    reps = max(1, args.sweep_reps)
    res = {"reps_per_point": reps}
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        # (a) density sweep on the benchmark workload (same inputs and scores as the step) ...
        res["density_sweep"] = {main["name"]: density_sweep(bsa, main["q"], main["k"], main["v"], main["scores"],
                                                             main["block"], main["seqlens"], reps, stream,
                                                             main["scale_kw"])}
        # ... and on the BF16 32K workload
        w = inputs.sweep_32k()
        d = inputs.make_inputs(w, device=device)
        S = bsa.stem_score(d["q"], d["k"], d["v"], w.block)
        res["density_sweep"][w.name] = density_sweep(bsa, d["q"], d["k"], d["v"], S, w.block, [w.N] * w.B, reps,
                                                      stream, {})
        del d, S
        # (b) length sweep: one sequence, 32 query / 8 KV heads, BF16, density 25%, the KV both
        # contiguous and in 64-token pages placed by a seeded permutation
        lens = []
        for n in SWEEP_LENGTHS:
            wl = inputs.Workload(f"single-{n // 1024}k", 1, 32, 8, n, 128, 128, "bf16", 0.25, "stem", 4,
                                 seqlens=[n], page_size=64)
            d = inputs.make_paged(wl, device=device)
            q1, k1, v1 = d["q"].unsqueeze(0), d["k_seq"][0].unsqueeze(0), d["v_seq"][0].unsqueeze(0)
            S = bsa.stem_score(q1, k1, v1, wl.block)
            nb = S.shape[-1]
            rp, ci = bsa.stem_select(S, [nb], wl.density)
            del S
            flop = effective_flop(rp, ci, [n], wl.block, wl.d)
            out = torch.empty_like(q1, dtype=torch.bfloat16)
            ms_c = _time_calls(lambda: bsa.bsa_prefill(q1, k1, v1, wl.block, rp, ci, out=out), reps, stream)
            cu = d["cu_seqlens"].to(device)
            outp = torch.empty_like(d["q"], dtype=torch.bfloat16)
            ms_p = _time_calls(lambda: bsa.bsa_prefill_paged(d["q"], cu, [n], d["k_cache"], d["v_cache"],
                                                             d["page_table"], wl.block, rp, ci, out=outp),
                               reps, stream)
            same = bool(torch.equal(out[0].view(torch.int16), outp.view(torch.int16)))
            lens.append({"N": n, "effective_flop": flop, "contiguous_ms": ms_c,
                         "contiguous_tflops": flop / (ms_c * 1e-3) / 1e12, "paged_ms": ms_p,
                         "paged_tflops": flop / (ms_p * 1e-3) / 1e12, "paged_equals_contiguous": same})
            del d, q1, k1, v1, rp, ci, out, outp
        bsa.bsa_check_device_error(device)
        res["length_sweep"] = {"config": "B1, 32/8 heads, d128, block 128, bf16, density 0.25 (75% sparsity)",
                               "points": lens}
        # (c) the paged varlen batch: 16K / 32K / 64K / 128K tokens, 32/8 heads, BF16 pages
        wv = inputs.paged_varlen()
        d = inputs.make_paged(wv, device=device)
        seqlens, cu = d["seqlens"], d["cu_seqlens"]
        nbp = [(n + wv.block - 1) // wv.block for n in seqlens]
        nbs = max(nbp)
        S = torch.full((len(seqlens), wv.Hq, nbs, nbs), float("nan"), device=device)
        for b in range(len(seqlens)):
            qb = d["q"][cu[b]:cu[b + 1]].unsqueeze(0)
            bsa.stem_score(qb, d["k_seq"][b].unsqueeze(0), d["v_seq"][b].unsqueeze(0), wv.block,
                           scores=S[b:b + 1], nb_stride=nbs)
        rp, ci = bsa.stem_select(S, nbp, wv.density)
        del S
        cud = cu.to(device)
        outp = torch.empty_like(d["q"], dtype=torch.bfloat16)
        ms = _time_calls(lambda: bsa.bsa_prefill_paged(d["q"], cud, seqlens, d["k_cache"], d["v_cache"],
                                                       d["page_table"], wv.block, rp, ci, out=outp), reps, stream)
        flop = effective_flop(rp, ci, seqlens, wv.block, wv.d)
        res["paged_varlen"] = {"workload": wv.name, "seqlens": seqlens, "Hq": wv.Hq, "Hkv": wv.Hkv, "dtype": "bf16",
                               "density": wv.density, "ms": ms, "effective_flop": flop,
                               "effective_tflops": flop / (ms * 1e-3) / 1e12}
        bsa.bsa_check_device_error(device)
        del d, outp, rp, ci
    res["clocks"] = clk.summary()
    return res


# ----------------------------------------------------------------------------- our arm


def run_ours(args, rank, world, device):
    import block_sparse_attention_42_b200 as bsa
    from block_sparse_attention_42_b200 import inputs

    w = inputs.WORKLOADS[args.workload](args.density)
    if w.page_size:
        raise SystemExit("the paged workload is a parity/test case; bench runs contiguous workloads")
    fp8 = w.dtype == "fp8"
    d = inputs.make_inputs(w, device=device, seed_offset=rank)
    q, k, v = d["q"], d["k"], d["v"]
    sq, sk, sv = d["q_scale"], d["k_scale"], d["v_scale"]
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    nb = (N + w.block - 1) // w.block
    scale_kw = dict(q_scale=sq, k_scale=sk, v_scale=sv)

    # Buffers allocated once; the step writes into them.
    scores = torch.empty(B, Hq, nb, nb, dtype=torch.float32, device=device)
    ws = torch.empty(bsa.bsa_score_workspace_bytes(B, Hq, Hkv, nb, D), dtype=torch.uint8, device=device)
    _, kstar = bsa.bsa_tpd_budget(nb, w.density, 0.5)
    row_ptr = torch.empty(B, nb + 1, dtype=torch.int32, device=device)
    col_idx = torch.empty(B, Hq, kstar, dtype=torch.int32, device=device)
    out = torch.empty(B, N, Hq, D, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def step(record=None):
        if record is not None:
            record[0].record(stream)
        bsa.stem_score(q, k, v, w.block, scores=scores, workspace=ws, **scale_kw)
        if record is not None:
            record[3].record(stream)
        bsa.stem_select(scores, [nb] * B, w.density, 0.5, row_ptr=row_ptr, col_idx=col_idx, max_k=kstar)
        if record is not None:
            record[1].record(stream)
        bsa.bsa_prefill(q, k, v, w.block, row_ptr, col_idx, out=out, **scale_kw)
        if record is not None:
            record[2].record(stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(device)
    bsa.bsa_check_device_error(device)
    eff = effective_flop(row_ptr, col_idx, [N] * B, w.block, D)

    # Timed region: K steps, per-step events on the launching stream.
    per = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        ev[0].record(stream)
        for s in range(args.steps):
            step(per[s])
        ev[1].record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    total_ms = ev[0].elapsed_time(ev[1])
    select_ms = [per[s][0].elapsed_time(per[s][1]) for s in range(args.steps)]
    attn_ms = [per[s][1].elapsed_time(per[s][2]) for s in range(args.steps)]
    score_call_ms = [per[s][0].elapsed_time(per[s][3]) for s in range(args.steps)]
    select_call_ms = [per[s][3].elapsed_time(per[s][1]) for s in range(args.steps)]
    max_ms = reduce_max(total_ms, world, device)
    bsa.bsa_check_device_error(device)

    res = dict(total_ms=max_ms, ms_per_step=max_ms / args.steps, eff_flop=eff,
               select_ms=statistics.median(select_ms), attn_ms=statistics.median(attn_ms),
               score_call_ms=statistics.median(score_call_ms), select_call_ms=statistics.median(select_call_ms),
               attn_ms_mean=sum(attn_ms) / len(attn_ms), clocks=clk.summary(), w=w, N=N, B=B, Hq=Hq, Hkv=Hkv,
               D=D, nb=nb, kstar=kstar, fp8=fp8)

    # Ideal line: the same kernel at density 1 (dense causal), measured on the same inputs.
    if not args.no_dense and rank == 0:
        dense_rp = torch.empty(B, nb + 1, dtype=torch.int32, device=device)
        dense_ci = torch.empty(B, Hq, nb * (nb + 1) // 2, dtype=torch.int32, device=device)
        bsa.stem_select(scores, [nb] * B, 1.0, 0.5, row_ptr=dense_rp, col_idx=dense_ci)
        dense_out = torch.empty_like(out)
        bsa.bsa_prefill(q, k, v, w.block, dense_rp, dense_ci, out=dense_out, **scale_kw)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 2
        e0.record(stream)
        for _ in range(reps):
            bsa.bsa_prefill(q, k, v, w.block, dense_rp, dense_ci, out=dense_out, **scale_kw)
        e1.record(stream)
        torch.cuda.synchronize(device)
        res["dense_ms"] = e0.elapsed_time(e1) / reps
        res["dense_flop"] = effective_flop(dense_rp, dense_ci, [N] * B, w.block, D)
        del dense_out, dense_ci

    # Block-mask input (bsa_prefill_mask): the step's lists written as a [B, Hq, nb, nb] uint8
    # mask (setup, untimed), then the mask -> lists kernel alone and the whole call, timed with
    # events like the step.  Its output is the list path's bit for bit (tests/test_gpu_mask.py).
    if not args.no_mask and rank == 0:
        mask = bsa.block_mask_buffer(B, Hq, nb, device=device)
        counts = (row_ptr[:, 1:] - row_ptr[:, :-1]).long()
        for b in range(B):
            rows = torch.repeat_interleave(torch.arange(nb, device=device), counts[b])
            heads = torch.arange(Hq, device=device)[:, None].expand(Hq, rows.numel())
            mask[b][heads, rows[None].expand(Hq, -1), col_idx[b, :, :rows.numel()].long()] = 1
        mws = torch.empty(bsa.bsa_mask_workspace_bytes(B, Hq, nb), dtype=torch.uint8, device=device)
        lrp = torch.empty(B, Hq, nb + 1, dtype=torch.int32, device=device)
        lci = torch.empty(B, Hq, nb * (nb + 1) // 2, dtype=torch.int32, device=device)
        mout = torch.empty_like(out)
        bsa.bsa_mask_to_lists(mask, row_ptr=lrp, col_idx=lci)
        bsa.bsa_prefill_mask(q, k, v, w.block, mask, out=mout, workspace=mws, **scale_kw)
        torch.cuda.synchronize(device)
        bsa.bsa_check_device_error(device)
        same = bool(torch.equal(mout.view(torch.int16), out.view(torch.int16)))
        reps = 3
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        for _ in range(reps):
            bsa.bsa_mask_to_lists(mask, row_ptr=lrp, col_idx=lci)
        e1.record(stream)
        for _ in range(reps):
            bsa.bsa_prefill_mask(q, k, v, w.block, mask, out=mout, workspace=mws, **scale_kw)
        e2.record(stream)
        torch.cuda.synchronize(device)
        lists_ms = e0.elapsed_time(e1) / reps
        # Algorithmic bytes of mask -> lists: each causal mask byte read once, the lists
        # (sum of kept blocks) and row_ptr written once.
        kept = int(counts.sum().item()) * Hq
        mbytes = B * Hq * nb * (nb + 1) // 2 + 4 * kept + 4 * B * Hq * (nb + 1)
        res["mask"] = {"prefill_mask_ms": e1.elapsed_time(e2) / reps, "mask_to_lists_ms": lists_ms,
                       "mask_to_lists_gbs": mbytes / (lists_ms * 1e-3) / 1e9, "algorithmic_bytes": mbytes,
                       "output_equals_list_path": same}
        del mask, mws, lrp, lci, mout

    # End to end through the public API with host buffers: H2D of Q/K/V from pinned memory,
    # the step, D2H of the output, all inside the timed region.  The step is pipelined over
    # chunks of query heads (e2e_split chunks per KV-head group; every head is an independent
    # problem with its own lists): one stream uploads chunk c+1 (with its group's K/V the first
    # time), another runs score -> select -> prefill of chunk c and a third downloads chunk
    # c-1's output, so the PCIe transfers (both directions) overlap the kernels.  Host and
    # device buffers are per chunk (K/V per group) and contiguous.
    if not args.no_e2e:
        G = Hkv
        gq = Hq // G
        F = max(1, min(args.e2e_split, gq))
        while gq % F:
            F -= 1
        cq = gq // F                       # query heads per chunk
        NC = G * F                          # chunks: F per KV-head group, K/V uploaded with the first
        slq = [slice(c * cq, (c + 1) * cq) for c in range(NC)]
        hq = [q[:, :, slq[c]].contiguous().cpu().pin_memory() for c in range(NC)]
        hk = [k[:, :, g:g + 1].contiguous().cpu().pin_memory() for g in range(G)]
        hv = [v[:, :, g:g + 1].contiguous().cpu().pin_memory() for g in range(G)]
        hout = [torch.empty((B, N, cq, D), dtype=out.dtype, pin_memory=True) for _ in range(NC)]
        dq = [torch.empty_like(x, device=device) for x in hq]
        dk = [torch.empty_like(x, device=device) for x in hk]
        dv = [torch.empty_like(x, device=device) for x in hv]
        dout = [torch.empty((B, N, cq, D), dtype=out.dtype, device=device) for _ in range(NC)]
        g_scores = torch.empty(B, cq, nb, nb, dtype=torch.float32, device=device)
        g_ws = torch.empty(bsa.bsa_score_workspace_bytes(B, cq, 1, nb, D), dtype=torch.uint8, device=device)
        g_rp = torch.empty(B, nb + 1, dtype=torch.int32, device=device)
        g_ci = torch.empty(B, cq, kstar, dtype=torch.int32, device=device)
        s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(NC)]
        ev_cmp = [torch.cuda.Event() for _ in range(NC)]
        ev_out = [torch.cuda.Event() for _ in range(NC)]
        started = [False]

        def e2e_step():
            for c in range(NC):
                g = c // F
                with torch.cuda.stream(s_in):
                    if started[0]:
                        s_in.wait_event(ev_cmp[c])  # the previous step's kernels of chunk c are done with its inputs
                        if c % F == 0:
                            s_in.wait_event(ev_cmp[c + F - 1])  # ... and every chunk of group g with its K/V
                    dq[c].copy_(hq[c], non_blocking=True)
                    if c % F == 0:
                        dk[g].copy_(hk[g], non_blocking=True)
                        dv[g].copy_(hv[g], non_blocking=True)
                    ev_in[c].record(s_in)
            for c in range(NC):
                g = c // F
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[c])
                    if started[0]:
                        s_cmp.wait_event(ev_out[c])  # the previous step's download of dout[c] is done
                    bsa.stem_score(dq[c], dk[g], dv[g], w.block, scores=g_scores, workspace=g_ws, **scale_kw)
                    bsa.stem_select(g_scores, [nb] * B, w.density, 0.5, row_ptr=g_rp, col_idx=g_ci, max_k=kstar)
                    bsa.bsa_prefill(dq[c], dk[g], dv[g], w.block, g_rp, g_ci, out=dout[c], **scale_kw)
                    ev_cmp[c].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[c])
                    hout[c].copy_(dout[c], non_blocking=True)
                    ev_out[c].record(s_out)
            started[0] = True

        main = torch.cuda.current_stream(device)
        e2e_step()
        torch.cuda.synchronize(device)
        # the pipelined output equals the full-size call's
        for c in (0, NC - 1):
            assert torch.equal(hout[c], out[:, :, slq[c]].cpu()), "pipelined e2e output differs from the full call"
        n_e2e = max(1, args.steps)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(main)
        for _ in range(n_e2e):
            e2e_step()
        for st in (s_in, s_cmp, s_out):
            main.wait_stream(st)
        e1.record(main)
        torch.cuda.synchronize(device)
        res["e2e_ms"] = reduce_max(e0.elapsed_time(e1) / n_e2e, world, device)
        res["e2e_steps"] = n_e2e
        res["h2d_bytes"] = sum(x.numel() * x.element_size() for x in (q, k, v))
        res["d2h_bytes"] = out.numel() * out.element_size()
        res["e2e_pipeline"] = f"{NC} chunks ({G} KV-head groups x {F}), H2D / kernels / D2H on three streams"
        del hq, hk, hv, hout, dq, dk, dv, dout, g_scores, g_ws, g_rp, g_ci

    # Group-shared selection (one list per KV-head group) and the GQA-packed attention kernel on
    # the same inputs: the whole path timed like the step, plus the attention call alone.
    if not args.no_group and rank == 0:
        G = Hq // Hkv
        g_scores = torch.empty(B, Hkv, nb, nb, dtype=torch.float32, device=device)
        g_ws = torch.empty(bsa.bsa_score_group_workspace_bytes(B, Hq, Hkv, nb, D), dtype=torch.uint8, device=device)
        g_rp = torch.empty(B, nb + 1, dtype=torch.int32, device=device)
        g_ci = torch.empty(B, Hkv, kstar, dtype=torch.int32, device=device)
        g_out = torch.empty_like(out)

        def g_select():
            bsa.stem_score_group(q, k, v, w.block, scores=g_scores, workspace=g_ws, **scale_kw)
            bsa.stem_select(g_scores, [nb] * B, w.density, 0.5, row_ptr=g_rp, col_idx=g_ci, max_k=kstar)

        def g_attn():
            bsa.bsa_prefill_group(q, k, v, w.block, g_rp, g_ci, out=g_out, **scale_kw)

        reps = max(3, min(args.steps, 10))
        sel_ms = _time_calls(g_select, reps, stream)
        attn_g_ms = _time_calls(g_attn, reps, stream)
        bsa.bsa_check_device_error(device)
        g_flop = G * effective_flop(g_rp, g_ci, [N] * B, w.block, D)
        res["group"] = {"what": "stem_score_group + stem_select (one list per KV-head group) and bsa_prefill_group "
                                "(two query heads per CTA, each kept K/V block loaded once for both)",
                        "select_ms": sel_ms, "bsa_prefill_group_ms": attn_g_ms, "effective_flop": g_flop,
                        "effective_tflops": g_flop / (attn_g_ms * 1e-3) / 1e12,
                        "per_head_bsa_prefill_ms": res["attn_ms"], "reps": reps}
        # The same K/V in a pool of 64-token pages placed by a seeded permutation (the serving
        # engine's cache layout), through bsa_prefill_paged_group: same lists, same kernel.
        if B == 1 and N % 64 == 0:
            npg = N // 64
            perm = torch.randperm(npg, generator=torch.Generator().manual_seed(7)).to(device)
            k_pool = torch.empty(npg, 64, Hkv, D, dtype=k.dtype, device=device)
            v_pool = torch.empty_like(k_pool)
            k_pool[perm] = k[0].reshape(npg, 64, Hkv, D)
            v_pool[perm] = v[0].reshape(npg, 64, Hkv, D)
            page_table = perm.to(torch.int32).view(1, npg)
            cu = torch.tensor([0, N], dtype=torch.int32, device=device)
            g_outp = torch.empty(N, Hq, D, dtype=torch.bfloat16, device=device)

            def g_attn_paged():
                bsa.bsa_prefill_paged_group(q[0], cu, [N], k_pool, v_pool, page_table, w.block, g_rp, g_ci,
                                            out=g_outp, **scale_kw)

            paged_ms = _time_calls(g_attn_paged, reps, stream)
            bsa.bsa_check_device_error(device)
            res["group"].update({"paged_group_ms": paged_ms,
                                 "paged_group_tflops": g_flop / (paged_ms * 1e-3) / 1e12,
                                 "paged_equals_contiguous": bool(torch.equal(g_outp.view(torch.int16),
                                                                             g_out[0].view(torch.int16))),
                                 "paged_layout": f"{npg} pages of 64 tokens, seeded permutation"})
            del k_pool, v_pool, g_outp
        del g_scores, g_ws, g_rp, g_ci, g_out

    # Score + select in one call without the score matrix: same lists, timed like select_ms.
    if not args.no_fused and rank == 0:
        f_ws = torch.empty(bsa.bsa_score_select_workspace_bytes(B, Hq, Hkv, N, w.block, D), dtype=torch.uint8,
                           device=device)
        f_rp = torch.empty(B, nb + 1, dtype=torch.int32, device=device)
        f_ci = torch.empty(B, Hq, kstar, dtype=torch.int32, device=device)

        def fused():
            bsa.stem_score_select(q, k, v, w.block, w.density, 0.5, row_ptr=f_rp, col_idx=f_ci, max_k=kstar,
                                  workspace=f_ws, **scale_kw)

        f_ms = _time_calls(fused, max(3, min(args.steps, 10)), stream)
        bsa.bsa_check_device_error(device)
        same = bool(torch.equal(f_rp, row_ptr) and torch.equal(f_ci, col_idx))
        res["fused_select"] = {"what": "stem_score_select: pool, budget, then per chunk of KV-head groups the score "
                                       "GEMM into a scratch of at most 128 MiB and the top-k from it; no score matrix",
                               "ms": f_ms, "unfused_select_ms": res["select_ms"], "lists_equal_unfused": same,
                               "workspace_bytes": f_ws.numel(),
                               "unfused_bytes": scores.numel() * 4 + ws.numel()}
        del f_ws, f_rp, f_ci

    # Threshold skip on top of the step's lists: speed and the kernel's own skip counters.
    if not args.no_skip and rank == 0 and (fp8 or D == 64 or w.block == 64):
        pts = []
        reps = max(3, min(args.steps, 10))
        for lam in (1e-4, 1e-3, 1e-2):
            stats = torch.zeros(4, dtype=torch.int64, device=device)
            s_out = torch.empty_like(out)
            bsa.bsa_prefill_skip(q, k, v, w.block, row_ptr, col_idx, lam, out=s_out, skip_stats=stats, **scale_kw)
            torch.cuda.synchronize(device)
            st = stats.cpu().tolist()
            ms = _time_calls(lambda: bsa.bsa_prefill_skip(q, k, v, w.block, row_ptr, col_idx, lam, out=s_out,
                                                          **scale_kw), reps, stream)
            diff = (s_out.float() - out.float())
            pts.append({"lambda": lam, "ms": ms, "speedup_vs_bsa_prefill": res["attn_ms"] / ms,
                        "row_block_skip_rate": st[1] / max(st[0], 1),
                        "tile_block_product_skip_rate": st[3] / max(st[2], 1),
                        "rel_l2_vs_no_skip": float(diff.norm() / out.float().norm())})
            del s_out, stats
        bsa.bsa_check_device_error(device)
        res["skip"] = {"what": "bsa_prefill_skip: a row drops a kept block whose max trails its running max by more "
                               "than ln(lambda); a warp whose rows all drop it skips the exponentials, a query block "
                               "whose rows all drop it skips the P.V product", "reps": reps, "points": pts}

    if not args.no_sweeps and rank == 0:
        res["sweeps"] = run_sweeps(args, device, dict(name=w.name, q=q, k=k, v=v, scores=scores, block=w.block,
                                                      seqlens=[N] * B, scale_kw=scale_kw))

    res["cpu"] = None
    if not args.no_cpu and rank == 0:
        res["cpu"] = cpu_baseline(q, k, v, sq, sk, sv, row_ptr, col_idx, w, budget_s=12.0)
    return res


def _oracle_sample_rows(w, N, Hq, n_rows, seed=0):
    rng = np.random.default_rng(seed)
    heads = rng.integers(0, Hq, size=n_rows)
    toks = rng.integers(0, N, size=n_rows)
    return np.stack([np.zeros(n_rows, np.int64), heads, toks], 1).astype(np.int64)


def cpu_baseline(q, k, v, sq, sk, sv, row_ptr, col_idx, w, budget_s=12.0):
    """The CPU oracle as it stands, on the host cores:
    - attention: randomly sampled query rows of the same workload and lists (all host threads,
      then one thread), effective TFLOP/s of those rows;
    - the select path exactly (pool + score + TPD budget + top-k over the whole workload), on all
      host threads and on one."""
    import oracle
    oracle.build()
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    B, N, Hq, D = qh.shape
    Hkv = kh.shape[2]
    nb = (N + w.block - 1) // w.block
    tau = 1.0 / math.sqrt(D)
    qv, kv, vv = oracle.view(qh, sq), oracle.view(kh, sk), oracle.view(vh, sv)
    cores = len(os.sched_getaffinity(0))

    def row_flop(rows):
        f = 0.0
        for b, h, t in rows:
            i = t // w.block
            for j in ci[b, h, rp[b, i]:rp[b, i + 1]]:
                lo = j * w.block
                hi = min(N, lo + w.block) - 1
                hi = min(hi, t)
                if hi >= lo:
                    f += hi - lo + 1
        return 4.0 * D * f

    def attention_sample(budget):
        n, flop, secs, seed = 16, 0.0, 0.0, 0
        while secs < budget:
            rows = _oracle_sample_rows(w, N, Hq, n, seed)
            t0 = time.perf_counter()
            oracle.attention_rows(qv, kv, vv, N, Hq, Hkv, D, w.block, rp, ci, tau, rows)
            secs += time.perf_counter() - t0
            flop += row_flop(rows)
            seed += 1
            n = min(4096, n * 2)
        return flop, secs

    def select_path():
        t0 = time.perf_counter()
        qb = oracle.pool_mean(qv, B, N, Hq, D, w.block)
        kb = oracle.pool_mean(kv, B, N, Hkv, D, w.block)
        vb = oracle.pool_vnorm(vv, B, N, Hkv, D, w.block)
        S = oracle.score(qb, kb, vb, tau, 0)
        oracle.select(S, [nb] * B, w.density, 0.5)
        return time.perf_counter() - t0

    oracle.set_threads(cores)
    flop, secs = attention_sample(budget_s)
    sel_s = select_path()
    oracle.set_threads(1)
    flop1, secs1 = attention_sample(budget_s / 3)
    sel1_s = select_path()
    oracle.set_threads(cores)
    return {"value": flop / secs / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle attention on {int(flop / 4 / D)} sampled (query, key) pairs of random "
                      f"query rows of the same workload and lists, {secs:.1f} s on {cores} threads",
            "one_core": {"value": flop1 / secs1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                         "sample": f"the same, {int(flop1 / 4 / D)} pairs, {secs1:.1f} s on one thread"},
            "select_path": {"what": "pool + score + TPD budget + top-k over the whole workload (exact, not sampled)",
                            "ms": 1e3 * sel_s, "cores": cores, "ms_one_core": 1e3 * sel1_s}}


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step is a bounded sample (query rows) of the
    same workload, on the host cores; rank 0 only."""
    from block_sparse_attention_42_b200 import inputs
    import oracle
    oracle.build()
    w = inputs.WORKLOADS[args.workload](args.density)
    dev = "cuda:0" if torch.cuda.is_available() else "cpu"
    d = inputs.make_inputs(w, device=dev)
    q, k, v = d["q"].cpu(), d["k"].cpu(), d["v"].cpu()
    sq, sk, sv = d["q_scale"], d["k_scale"], d["v_scale"]
    del d
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    nb = (N + w.block - 1) // w.block
    tau = 1.0 / math.sqrt(D)
    qv, kv, vv = oracle.view(q, sq), oracle.view(k, sk), oracle.view(v, sv)
    # Lists from the oracle's own select path (setup, untimed).
    qb = oracle.pool_mean(qv, B, N, Hq, D, w.block)
    kb = oracle.pool_mean(kv, B, N, Hkv, D, w.block)
    vb = oracle.pool_vnorm(vv, B, N, Hkv, D, w.block)
    S = oracle.score(qb, kb, vb, tau, 0)
    rp, ci = oracle.select(S, [nb] * B, w.density, 0.5)
    del S

    def one_step(seed):
        rows = _oracle_sample_rows(w, N, Hq, 64, seed)
        t0 = time.perf_counter()
        oracle.attention_rows(qv, kv, vv, N, Hq, Hkv, D, w.block, rp, ci, tau, rows)
        dt = time.perf_counter() - t0
        pairs = 0
        for b, h, t in rows:
            i = t // w.block
            for j in ci[b, h, rp[b, i]:rp[b, i + 1]]:
                lo = j * w.block
                hi = min(min(N, lo + w.block) - 1, t)
                pairs += max(0, hi - lo + 1)
        return dt, 4.0 * D * pairs

    for s in range(args.warmup):
        one_step(1000 + s)
    tot_t, tot_f = 0.0, 0.0
    for s in range(args.steps):
        dt, f = one_step(s)
        tot_t += dt
        tot_f += f
    cores = len(os.sched_getaffinity(0))
    val = tot_f / tot_t / 1e12
    sample = f"fp64 oracle attention, 64 random query rows per step of {w.name}; lists from the oracle's own select"
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "N": N, "Hq": Hq, "Hkv": Hkv, "d": D, "block": w.block,
                       "density": w.density},
            "impl": "reference",
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": val, "unit": "TFLOP/s"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, rank, world)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    res = run_ours(args, rank, world, device)
    if rank == 0:
        pk, src = peaks()
        fp8 = res["fp8"]
        peak = (pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * (2.0 if fp8 else 1.0))
        attn_ach = res["eff_flop"] / (res["attn_ms_mean"] * 1e-3) / 1e12
        value = whole_job_tflops(res["eff_flop"], world, res["ms_per_step"])
        w = res["w"]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": res["B"], "N": res["N"], "Hq": res["Hq"], "Hkv": res["Hkv"],
                       "d": res["D"], "block": w.block, "density": w.density, "tpd_decay": 0.5,
                       "kept_blocks_per_head": res["kstar"], "l2": "inputs larger than L2 (Q alone > 126 MB)",
                       "parallelism": f"independent problem per rank x{world}"},
            "bsa_prefill_ms": res["attn_ms"], "select_ms": res["select_ms"],
            "bsa_prefill_effective_tflops": attn_ach,
            "effective_flop_per_step": res["eff_flop"],
            "roofline": {"bound": "tensor", "kernel": "bsa_prefill", "achieved": attn_ach, "peak": peak,
                         "unit": "TFLOP/s", "frac": attn_ach / peak,
                         "peak_source": f"{src} bf16 {'sustained' if 'bf16_tflops_sustained' in pk else 'burst'}"
                                        f"{' x2 (fp8/bf16 nominal ratio)' if fp8 else ''}",
                         "traffic": attn_traffic(fp8, res["B"], res["N"], res["Hq"], res["Hkv"], res["D"]),
                         "traffic_source": "ncu dram bytes of the fp8-32k capture, scaled by tokens",
                         # the same against the burst GEMM figure (measured near the maximum clock,
                         # where this kernel runs; the sustained figure was measured power-capped)
                         "peak_burst": pk["bf16_tflops"] * (2.0 if fp8 else 1.0),
                         "frac_of_burst_peak": attn_ach / (pk["bf16_tflops"] * (2.0 if fp8 else 1.0))},
            # The bound that binds for E4M3 attention: the exponentials.  Every kept 128-key
            # block needs block x block exp2 per query row tile; the MUFU unit does 16 per clock
            # per SM (measured with a throughput probe on this machine), so the peak is
            # 16 x SMs x the median SM clock sampled during the timed steps.
            "roofline_mufu": mufu_roofline(res, device),
            # pool, score, TPD budget, one select launch per row-length class present
            # (query blocks in [0, 256), [256, 512), [512, 1024), [1024, 2048)), attention
            "gpu_launches": (4 + sum(1 for lo in (0, 256, 512, 1024) if res["nb"] > lo)) * args.steps,
            "clocks": res["clocks"],
        }
        if "dense_ms" in res:
            rho_eff = res["eff_flop"] / res["dense_flop"]
            line["dense_ms"] = res["dense_ms"]
            line["ideal_line_ratio"] = res["attn_ms_mean"] / (res["dense_ms"] * rho_eff)
            line["rho_eff"] = rho_eff
        if "e2e_ms" in res:
            line["e2e"] = {"value": whole_job_tflops(res["eff_flop"], world, res["e2e_ms"]), "unit": "TFLOP/s",
                           "h2d_bytes_per_step": res["h2d_bytes"], "d2h_bytes_per_step": res["d2h_bytes"],
                           "ms_per_step": res["e2e_ms"], "steps": res["e2e_steps"],
                           "pipeline": res.get("e2e_pipeline")}
        # The selection path's HBM rates.  stem_score = pool + score GEMM: its bytes are the
        # pool's (Q, K, V read once), so the rate is a lower bound on the pool kernel's.
        # stem_select = TPD budget + top-k: the causal scores read once, the lists written.
        elt = 1 if fp8 else 2
        n_tok = res["B"] * res["N"]
        pool_bytes = n_tok * (res["Hq"] + 2 * res["Hkv"]) * res["D"] * elt
        causal = res["B"] * res["nb"] * (res["nb"] + 1) // 2
        sel_bytes = 4 * res["Hq"] * causal + 4 * res["Hq"] * res["B"] * res["kstar"]
        line["select_path"] = {
            "stem_score_ms": res["score_call_ms"], "stem_select_ms": res["select_call_ms"],
            "pool_bytes": pool_bytes, "pool_gbs_lower_bound": pool_bytes / (res["score_call_ms"] * 1e-3) / 1e9,
            "select_bytes": sel_bytes, "select_gbs": sel_bytes / (res["select_call_ms"] * 1e-3) / 1e9,
            "hbm_peak_gbs": pk["hbm_gbs"]}
        if "sweeps" in res:
            line["sweeps"] = res["sweeps"]
        if "group" in res:
            line["group_shared"] = res["group"]
        if "skip" in res:
            line["threshold_skip"] = res["skip"]
        if "fused_select" in res:
            line["fused_select"] = res["fused_select"]
        if "mask" in res:
            m = dict(res["mask"])
            m["mask_to_lists_roofline"] = {"bound": "hbm", "achieved": m.pop("mask_to_lists_gbs"),
                                           "peak": pk["hbm_gbs"], "unit": "GB/s"}
            m["mask_to_lists_roofline"]["frac"] = m["mask_to_lists_roofline"]["achieved"] / pk["hbm_gbs"]
            line["mask_input"] = m
        if res["cpu"] is not None:
            line["cpu_baseline"] = res["cpu"]
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
