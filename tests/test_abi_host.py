"""Host-side checks of the C ABI that need no GPU: the library loads, exports every symbol
include/bsa.h declares, its host TPD budget equals the oracle's bit for bit, and argument
errors come back as status codes before anything touches the device."""
import ctypes
import re
from pathlib import Path

import numpy as np
import pytest
import torch

ROOT = Path(__file__).resolve().parent.parent


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_42_b200 import binding, build
    build.build()
    return binding.lib()


def _declared_functions():
    text = (ROOT / "include" / "bsa.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"if", "sizeof"})


def test_exports_every_declared_symbol(lib):
    from block_sparse_attention_42_b200 import binding
    names = _declared_functions()
    assert set(names) == set(binding.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_host_budget_equals_oracle_exhaustive(lib, orc):
    from block_sparse_attention_42_b200 import binding
    for decay in (0.5, 0.0):
        for density in (0.1, 0.2, 0.25, 0.5, 0.8, 1.0):
            for nb in range(1, 2049) if decay == 0.5 and density == 0.25 else range(1, 2049, 37):
                k, tot = binding.bsa_tpd_budget(nb, density, decay)
                ko, toto = orc.tpd_budget(nb, density, decay)
                assert tot == toto and np.array_equal(k.numpy(), ko), (nb, density, decay)
                # k_out = NULL: the total alone
                assert binding.tpd_kstar(nb, density, decay) == toto, (nb, density, decay)


def test_host_budget_rejects_bad_args(lib):
    k = (ctypes.c_int32 * 8)()
    assert lib.bsa_tpd_budget(0, 0.5, 0.5, k) == -1
    assert lib.bsa_tpd_budget(8, 0.0, 0.5, k) == -1
    assert lib.bsa_tpd_budget(8, 0.5, 0.25, k) == -1
    assert lib.bsa_tpd_budget(0, 0.5, 0.5, None) == -1
    assert lib.bsa_tpd_budget(8, 1.5, 0.5, None) == -1


def test_mask_workspace_bytes(lib):
    # row_ptr [B*Hq][nb+1] (256-byte aligned) then col_idx [B*Hq][nb(nb+1)/2], int32
    for B, Hq, nb in [(1, 8, 8), (2, 64, 1024), (4, 32, 2048), (1, 1, 1)]:
        rp = 4 * B * Hq * (nb + 1)
        assert lib.bsa_mask_workspace_bytes(B, Hq, nb) == (rp + 255) // 256 * 256 + 4 * B * Hq * nb * (nb + 1) // 2
    assert lib.bsa_mask_workspace_bytes(1, 8, 2049) == 0
    assert lib.bsa_mask_workspace_bytes(0, 8, 8) == 0


def _t(ptr=0x10000, dtype=0, st=1024, sh=128, sb=1 << 20, scale=1.0):
    from block_sparse_attention_42_b200.binding import BsaTensor
    return BsaTensor(ptr, dtype, scale, sb, st, sh)


def test_argument_errors_return_status(lib):
    P = ctypes.c_void_p
    ws = P(0x20000)
    sc = P(0x30000)
    # null q
    assert lib.stem_score(_t(ptr=0), _t(), _t(), 1, 1024, 8, 8, 128, 128, 0, 0.0, sc, 8, ws, 1 << 30, None) == 1
    # misaligned base pointer
    assert lib.stem_score(_t(ptr=0x10008), _t(), _t(), 1, 1024, 8, 8, 128, 128, 0, 0.0, sc, 8, ws, 1 << 30, None) == 1
    # stride not a multiple of 16 bytes
    assert lib.stem_score(_t(st=1023), _t(), _t(), 1, 1024, 8, 8, 128, 128, 0, 0.0, sc, 8, ws, 1 << 30, None) == 1
    # Hq % Hkv != 0
    assert lib.stem_score(_t(), _t(), _t(), 1, 1024, 6, 4, 128, 128, 0, 0.0, sc, 8, ws, 1 << 30, None) == 1
    # unsupported head_dim / block
    assert lib.stem_score(_t(), _t(), _t(), 1, 1024, 8, 8, 96, 128, 0, 0.0, sc, 8, ws, 1 << 30, None) == 2
    assert lib.stem_score(_t(), _t(), _t(), 1, 1024, 8, 8, 128, 32, 0, 0.0, sc, 8, ws, 1 << 30, None) == 2
    # workspace too small
    assert lib.stem_score(_t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, 0, 0.0, sc, 8, ws, 16, None) == 4
    # nb_stride too small
    assert lib.stem_score(_t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, 0, 0.0, sc, 4, ws, 1 << 30, None) == 1
    nbp = (ctypes.c_int32 * 1)(8)
    # density out of range, decay unsupported, max_k too small
    assert lib.stem_select(sc, 1, 8, nbp, 8, 0.0, 0.5, P(0x40000), P(0x50000), 100, None) == 1
    assert lib.stem_select(sc, 1, 8, nbp, 8, 0.5, 0.3, P(0x40000), P(0x50000), 100, None) == 2
    assert lib.stem_select(sc, 1, 8, nbp, 8, 0.5, 0.5, P(0x40000), P(0x50000), 3, None) == 1
    # attention: FP8 needs d=128/block=128; out must be BF16; null lists
    f8 = dict(dtype=1, scale=0.5)
    assert lib.bsa_prefill(_t(**f8), _t(**f8), _t(**f8), _t(), 1, 1024, 8, 8, 64, 128, P(1), 9, P(1), 36, 0.0,
                           None, None) == 2
    assert lib.bsa_prefill(_t(), _t(), _t(), _t(dtype=2), 1, 1024, 8, 8, 128, 128, P(1), 9, P(1), 36, 0.0,
                           None, None) == 2
    assert lib.bsa_prefill(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, None, 9, P(1), 36, 0.0, None, None) == 1
    # FP8 with a non-positive scale
    assert lib.bsa_prefill(_t(dtype=1, scale=0.0), _t(**f8), _t(**f8), _t(), 1, 1024, 8, 8, 128, 128, P(1), 9,
                           P(1), 36, 0.0, None, None) == 1
    # paged: page size must be 64
    sl = (ctypes.c_int32 * 1)(1024)
    assert lib.bsa_prefill_paged(_t(), _t(), P(1), sl, 1, _t(), _t(), 100, 32, P(1), 16, 8, 8, 128, 128, P(1), 9,
                                 P(1), 36, 0.0, None, None) == 2
    assert lib.bsa_prefill_paged_group(_t(), _t(), P(1), sl, 1, _t(), _t(), 100, 32, P(1), 16, 8, 8, 128, 128, P(1),
                                       9, P(1), 36, 0.0, None, None) == 2
    assert lib.bsa_prefill_paged_group(_t(), _t(), None, sl, 1, _t(), _t(), 100, 64, P(1), 16, 8, 8, 128, 128, P(1),
                                       9, P(1), 36, 0.0, None, None) == 1
    # block-mask input: stride a multiple of 16 and >= nb, a 16-byte aligned mask, room for the
    # lists; nb at most 2048
    ws_need = lib.bsa_mask_workspace_bytes(1, 8, 8)
    assert lib.bsa_prefill_mask(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, P(0x60000), 10, 0.0, None, ws,
                                1 << 30, None) == 1
    assert lib.bsa_prefill_mask(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, P(0x60000), 0, 0.0, None, ws,
                                1 << 30, None) == 1
    assert lib.bsa_prefill_mask(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, P(0x60008), 16, 0.0, None, ws,
                                1 << 30, None) == 1
    assert lib.bsa_prefill_mask(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, None, 16, 0.0, None, ws,
                                1 << 30, None) == 1
    assert lib.bsa_prefill_mask(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, P(0x60000), 16, 0.0, None, ws,
                                ws_need - 1, None) == 4
    assert lib.bsa_prefill_mask(_t(), _t(), _t(), _t(), 1, 1024, 8, 8, 128, 128, P(0x60000), 16, 0.0, None, None,
                                1 << 30, None) == 4
    assert lib.bsa_mask_to_lists(P(0x60000), 16, 1, 8, 8, P(0x40000), P(0x50000), 35, None) == 1   # max_k < 36
    assert lib.bsa_mask_to_lists(P(0x60000), 16, 1, 8, 8, None, P(0x50000), 36, None) == 1
    assert lib.bsa_mask_to_lists(P(0x60000), 2064, 1, 8, 2049, P(0x40000), P(0x50000), 1 << 22, None) == 2
    assert lib.bsa_mask_to_lists(P(0x60000), 2048, 256, 65535, 2048, P(0x40000), P(0x50000), 1 << 22, None) == 2
    # list validation: null pointers, B / nb out of range, strides too small for nb
    nb8 = (ctypes.c_int32 * 2)(8, 8)
    assert lib.bsa_validate_lists(None, 9, 0, P(0x50000), 36, 1, 8, nb8, 0, None) == 1
    assert lib.bsa_validate_lists(P(0x40000), 9, 0, P(0x50000), 36, 0, 8, nb8, 0, None) == 2
    assert lib.bsa_validate_lists(P(0x40000), 9, 0, P(0x50000), 36, 1, 8, (ctypes.c_int32 * 1)(2049), 0, None) == 2
    assert lib.bsa_validate_lists(P(0x40000), 8, 0, P(0x50000), 36, 1, 8, nb8, 0, None) == 1   # stride < nb + 1
    assert lib.bsa_validate_lists(P(0x40000), 9 * 7, 9, P(0x50000), 36, 1, 8, nb8, 1, None) == 1  # < Hq * 9
    assert lib.bsa_validate_lists(P(0x40000), 9, 0, P(0x50000), 0, 1, 8, nb8, 0, None) == 1   # max_k < 1
    # allocation-free scoring: a size stem_score refuses for another reason gets stem_score's own
    # error, even when the problem would also be too large for the fixed scratch
    big = 1 << 20
    assert lib.stem_score_noalloc(_t(), _t(), _t(), 1, big, 64, 8, 96, 128, 0, 0.0, sc, 8192, None) == 2
    assert "head_dim" in lib.bsa_last_error().decode()
    assert lib.stem_score_noalloc(_t(), _t(), _t(), 1, big, 64, 8, 128, 1, 0, 0.0, sc, 1 << 20, None) == 2
    assert "block" in lib.bsa_last_error().decode()
    assert lib.stem_score_noalloc(_t(), _t(), _t(), 1, big, 64, 12, 128, 128, 0, 0.0, sc, 8192, None) == 1
    assert lib.stem_score_noalloc(_t(), _t(), _t(), 1, big, 64, 8, 128, 128, 0, 0.0, sc, 8192, None) == 2
    assert "fixed scratch" in lib.bsa_last_error().decode()
    # wait-timeout self-test: the limit must lie in [1 us, 1 s]
    assert lib.bsa_selftest_wait_timeout(ctypes.c_uint64(0), None) == 1
    assert lib.bsa_selftest_wait_timeout(ctypes.c_uint64(2_000_000_000), None) == 1
    assert lib.bsa_last_error().decode() != ""


def test_block_mask_buffer_and_argument_checks():
    """The binding's mask marshalling: padded rows, bool accepted, bad layouts refused (CPU tensors;
    nothing is launched)."""
    from block_sparse_attention_42_b200 import binding
    for nb in (1, 15, 16, 17, 1000):
        m = binding.block_mask_buffer(2, 3, nb)
        assert m.shape == (2, 3, nb, nb) and m.dtype == torch.uint8
        assert m.stride(2) % 16 == 0 and m.stride(2) >= nb and m.stride(3) == 1
        ptr, ms = binding._mask_arg(m, 2, 3, nb)
        assert ms == m.stride(2) and ptr.value == m.data_ptr()
    mb = binding.block_mask_buffer(1, 2, 20, dtype=torch.bool)
    assert binding._mask_arg(mb, 1, 2, 20)[1] == 32
    with pytest.raises(TypeError):
        binding._mask_arg(torch.zeros(1, 2, 20, 32, dtype=torch.int32), 1, 2, 20)
    with pytest.raises(ValueError):
        binding._mask_arg(torch.zeros(1, 2, 19, 32, dtype=torch.uint8), 1, 2, 20)      # wrong nb
    with pytest.raises(ValueError):
        binding._mask_arg(torch.zeros(1, 2, 20, 32, dtype=torch.uint8)[..., ::2], 1, 2, 20)  # strided columns
    with pytest.raises(ValueError):
        binding._mask_arg(torch.zeros(1, 20, 2, 32, dtype=torch.uint8).transpose(1, 2), 1, 2, 20)  # heads not outer


def test_group_wrappers_refuse_per_head_lists():
    """bsa_prefill_group and bsa_prefill_paged_group take one list per KV-head group
    (col_idx [B, Hkv, max_k]); per-head lists are refused before anything is launched (CPU
    tensors)."""
    from block_sparse_attention_42_b200 import binding
    B, N, Hq, Hkv, d = 1, 256, 8, 2, 128
    q = torch.zeros(B, N, Hq, d, dtype=torch.bfloat16)
    k = torch.zeros(B, N, Hkv, d, dtype=torch.bfloat16)
    rp = torch.zeros(B, 3, dtype=torch.int32)
    per_head = torch.zeros(B, Hq, 3, dtype=torch.int32)
    with pytest.raises(ValueError):
        binding.bsa_prefill_group(q, k, k, 128, rp, per_head)
    kc = torch.zeros(4, 64, Hkv, d, dtype=torch.bfloat16)
    pt = torch.arange(4, dtype=torch.int32).view(1, 4)
    cu = torch.tensor([0, N], dtype=torch.int32)
    with pytest.raises(ValueError):
        binding.bsa_prefill_paged_group(q[0], cu, [N], kc, kc, pt, 128, rp, per_head)
