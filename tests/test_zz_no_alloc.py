"""stem_score_noalloc: the allocation-free variant of stem_score.

Some callers cannot allocate device memory (a plain C program that links only this
library, or a runtime whose memory pool owns all of HBM); this entry point keeps the pooled
block representations in a fixed 32 MiB array inside the library instead of a caller
workspace.  These tests call it through the C ABI and check it against stem_score on two
calls in a row (different inputs, so stale scratch contents would show up), and that a
problem too large for the fixed scratch is refused with a clear error.

The file is named to be collected last: a failure here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import binding, inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_noalloc_matches_stem_score_twice(orc):
    cases = [(inputs.gqa_8k(), 8192, "bf16", 0), (inputs.Workload("na", 2, 4, 2, 1000, 64, 64, "bf16", 0.25,
                                                                    "stem", 31), None, "bf16", 1)]
    for w, N, storage, metric in cases:
        d = inputs.make_inputs(w, device=DEV, N=N, storage=storage)
        q, k, v = d["q"], d["k"], d["v"]
        nb = (q.shape[1] + w.block - 1) // w.block
        ref = bsa.stem_score(q, k, v, w.block, metric=metric)
        got = binding.stem_score_noalloc(q, k, v, w.block, metric=metric)
        torch.cuda.synchronize()
        qb, kb, vb = H.oracle_pool(orc, q, k, v, w.block)
        scale = H.score_scale(qb, kb, vb, H.default_tau(w.d), metric)
        # same tolerance as the stem_score parity tests, against stem_score's own output
        H.assert_scores_close(got, ref.double().cpu().numpy(), scale, nb)


def test_noalloc_rejects_oversized_problem():
    w = inputs.fp8_128k()
    q = torch.empty(1, 65536, 64, 128, dtype=torch.float8_e4m3fn, device=DEV)
    kv = torch.empty(1, 65536, 8, 128, dtype=torch.float8_e4m3fn, device=DEV)
    with pytest.raises(bsa.BsaError, match="UNSUPPORTED.*fixed scratch"):
        binding.stem_score_noalloc(q, kv, kv, 128, q_scale=0.1, k_scale=0.1, v_scale=0.1)
