"""Writes oam_sam_gqa8k.json: how much of dense attention the block selection of each
scoring metric keeps at density 25%, computed by the fp64 oracle alone, on two 8K GQA input
distributions: the benchmark's ("stem": Gaussian tokens, outlier channels, a sink, log-normal
value norms per token) and a block-structured one ("blocky": attention falls on whole key
blocks with per-block value amplitudes).

The Stem write-up (cn486, section 3.2 OAM) argues that weighting the routing score by the value
amplitude selects blocks that matter more for the output than the score alone (SAM); the
setupai write-up ("Technical Deep Dive", OAM bullet) says the same.  This is a record of that
comparison on synthetic inputs with log-normal value norms, not a pass/fail check.

For each metric (OAM log-add, SAM, OAM_MUL) the oracle pools, scores and selects (TPD, decay
1/2), then computes attention on sampled query rows; the dense reference is the same rows at
density 1.  Recorded per metric:
  - rel_l2: ||O_sparse - O_dense|| / ||O_dense|| over the sampled rows;
  - mass_kept_mean / mass_kept_p05: exp(LSE_sparse - LSE_dense) per row, the share of the
    dense softmax mass that falls in the kept blocks (mean and 5th percentile).

    python tests/golden/oam_sam_record.py          # rewrites the JSON next to this script
"""
from __future__ import annotations

import json
import math
import sys
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
ROOT = HERE.parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

OUT = HERE / "oam_sam_gqa8k.json"
METRICS = {"OAM": 0, "SAM": 1, "OAM_MUL": 2}


def sample_rows(B, Hq, N, n_per_head, seed):
    rng = np.random.default_rng(seed)
    rows = [(b, h, int(t)) for b in range(B) for h in range(Hq)
            for t in rng.integers(0, N, size=n_per_head)]
    return np.array(rows, np.int64)


def compute(w, n_per_head: int = 48, seed: int = 7) -> dict:
    import oracle
    from block_sparse_attention_42_b200 import inputs
    oracle.build()
    d = inputs.make_inputs(w)
    q, k, v = d["q"], d["k"], d["v"]
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    nb = (N + w.block - 1) // w.block
    tau = 1.0 / math.sqrt(D)
    qv, kv, vv = oracle.view(q), oracle.view(k), oracle.view(v)
    qb = oracle.pool_mean(qv, B, N, Hq, D, w.block)
    kb = oracle.pool_mean(kv, B, N, Hkv, D, w.block)
    vb = oracle.pool_vnorm(vv, B, N, Hkv, D, w.block)
    rows = sample_rows(B, Hq, N, n_per_head, seed)
    rp_d, ci_d = oracle.select(oracle.score(qb, kb, vb, tau, 0), [nb] * B, 1.0, 0.5)
    o_dense, lse_dense = oracle.attention_rows(qv, kv, vv, N, Hq, Hkv, D, w.block, rp_d, ci_d, tau, rows)
    rec = {"workload": w.name, "distribution": w.dist, "B": B, "N": N, "Hq": Hq, "Hkv": Hkv, "d": D, "block": w.block,
           "density": w.density, "tpd_decay": 0.5, "rows": int(rows.shape[0]), "row_seed": seed,
           "metrics": {}}
    for name, metric in METRICS.items():
        S = oracle.score(qb, kb, vb, tau, metric)
        rp, ci = oracle.select(S, [nb] * B, w.density, 0.5)
        o, lse = oracle.attention_rows(qv, kv, vv, N, Hq, Hkv, D, w.block, rp, ci, tau, rows)
        mass = np.exp(lse - lse_dense)
        rec["metrics"][name] = {
            "rel_l2": float(np.linalg.norm(o - o_dense) / np.linalg.norm(o_dense)),
            "mass_kept_mean": float(mass.mean()),
            "mass_kept_p05": float(np.quantile(mass, 0.05)),
        }
    return rec


def compute_all() -> dict:
    from block_sparse_attention_42_b200 import inputs
    return {"stem": compute(inputs.gqa_8k()), "blocky": compute(inputs.blocky_8k())}


def main():
    rec = compute_all()
    rec["what"] = ("share of dense attention kept by each scoring metric's block selection (fp64 oracle; "
                   "a record, not a pass/fail check)")
    rec["source"] = ("Stem write-up (cn486), section 3.2 OAM: routing probability x value amplitude selects "
                     "blocks that matter more for the output than the score alone; setupai, Technical Deep Dive")
    rec["script"] = "tests/golden/oam_sam_record.py (calls only oracle/ and the input generator)"
    OUT.write_text(json.dumps(rec, indent=2) + "\n")
    print(json.dumps({k: v["metrics"] for k, v in rec.items() if isinstance(v, dict)}, indent=2))


if __name__ == "__main__":
    main()
