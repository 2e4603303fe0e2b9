"""The shared timeout path of the pipeline waits, exercised on the GPU without a fault: a
test-only kernel waits on an mbarrier that nothing arrives at, with a 50 ms limit.  It must
record BSA_ERR_TIMEOUT in the device error word, free its tensor memory and leave the context
usable (an attention call right after it runs and matches the oracle)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_wait_that_never_completes_reports_timeout_and_frees_tmem(orc):
    torch.cuda.set_device(DEV)
    bsa.bsa_check_device_error()  # start from a clear error word
    bsa.bsa_selftest_wait_timeout(50_000_000)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_check_device_error()
    assert ei.value.status == 6  # BSA_ERR_TIMEOUT
    bsa.bsa_check_device_error()  # reading the word cleared it

    # The context is intact and the tensor memory was returned: a full attention call works.
    w = inputs.tiny()
    d = inputs.make_inputs(w, device=DEV, storage="bf16")
    q, k, v = d["q"], d["k"], d["v"]
    B, N, Hq, dh = q.shape
    S = bsa.stem_score(q, k, v, w.block)
    rp, ci = bsa.stem_select(S, [S.shape[-1]], w.density)
    out = bsa.bsa_prefill(q, k, v, w.block, rp, ci)
    bsa.bsa_check_device_error()
    rows = H.sample_rows(B, Hq, N, w.block)
    ref, _, amp = H.oracle_attention(orc, q, k, v, w.block, rp, ci, H.default_tau(dh), rows)
    H.assert_bf16_close(H.gather_rows(out, rows), ref, amp)
