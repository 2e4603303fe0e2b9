"""bsa_validate_lists: the debug list check through the C ABI.  Lists from stem_select and from
bsa_mask_to_lists pass; each corruption the attention kernels would not all catch (entries out
of order, a repeated entry) and the ones they do (an entry past i, a bad row pointer) are
reported as BSA_ERR_INVALID_LIST by bsa_check_device_error, through the device error word."""
import pytest
import torch

import block_sparse_attention_42_b200 as bsa
from block_sparse_attention_42_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _stem_lists():
    w = inputs.Workload("val", 2, 4, 2, 4000, 128, 128, "bf16", 0.3, "stem", 51)
    d = inputs.make_inputs(w, device=DEV)
    S = bsa.stem_score(d["q"], d["k"], d["v"], w.block)
    nb = S.shape[-1]
    rp, ci = bsa.stem_select(S, [nb, nb], w.density)
    return rp, ci, nb


def _expect_invalid(rp, ci, nbs, allow_empty=False):
    bsa.bsa_validate_lists(rp, ci, nbs, allow_empty)
    with pytest.raises(bsa.BsaError, match="INVALID_LIST"):
        bsa.bsa_check_device_error()
    bsa.bsa_check_device_error()            # the word was cleared


def test_valid_lists_pass():
    rp, ci, nb = _stem_lists()
    bsa.bsa_validate_lists(rp, ci, [nb, nb])
    bsa.bsa_check_device_error()
    mask = bsa.block_mask_buffer(2, 4, nb, device=DEV)
    mask[..., :] = (torch.rand(2, 4, nb, nb, device=DEV) < 0.3).to(torch.uint8)
    mask[0, 1, 3, :4] = 0                  # an empty row
    mrp, mci = bsa.bsa_mask_to_lists(mask)
    bsa.bsa_validate_lists(mrp, mci, [nb, nb], allow_empty=True)
    bsa.bsa_check_device_error()
    _expect_invalid(mrp, mci, [nb, nb], allow_empty=False)   # the empty row is not allowed here


@pytest.mark.parametrize("kind", ["swap", "repeat", "past_diagonal", "negative", "row_ptr"])
def test_corruptions_are_flagged(kind):
    rp, ci, nb = _stem_lists()
    ci = ci.clone()
    rp = rp.clone()
    b, h = 1, 2
    i = int(torch.argmax((rp[b, 1:nb + 1] - rp[b, :nb]).cpu()).item())   # the longest row
    lo, hi = rp[b, i].item(), rp[b, i + 1].item()
    assert hi - lo >= 3
    if kind == "swap":
        a0, a1 = ci[b, h, lo + 1].item(), ci[b, h, lo + 2].item()
        ci[b, h, lo + 1], ci[b, h, lo + 2] = a1, a0
    elif kind == "repeat":
        ci[b, h, lo + 2] = ci[b, h, lo + 1]
    elif kind == "past_diagonal":
        ci[b, h, hi - 1] = i + 1
    elif kind == "negative":
        ci[b, h, lo] = -1
    else:
        rp[b, i + 1] = lo - 1               # row i ends before it starts
    _expect_invalid(rp, ci, [nb, nb])
