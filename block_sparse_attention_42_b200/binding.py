"""Thin ctypes binding of libbsa.so: the same entry points as include/bsa.h.

Argument marshalling only: torch tensors become pointers, strides and the current CUDA
stream; every step of the path runs in the library's kernels.  PyTorch allocates outputs
and workspaces when the caller passes none.  There is no fallback: if libbsa.so is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libbsa.so"
_lib = None

BSA_BF16, BSA_FP8_E4M3, BSA_FP32 = 0, 1, 2
BSA_METRIC_OAM, BSA_METRIC_SAM, BSA_METRIC_OAM_MUL = 0, 1, 2
STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_CUDA",
          4: "BSA_ERR_WORKSPACE", 5: "BSA_ERR_INVALID_LIST", 6: "BSA_ERR_TIMEOUT", 7: "BSA_ERR_INVALID_PAGE"}

# Every symbol include/bsa.h declares.
EXPORTS = ["bsa_tpd_budget", "bsa_score_workspace_bytes", "stem_score", "stem_select", "bsa_prefill",
           "bsa_prefill_paged", "bsa_last_error", "bsa_check_device_error", "stem_score_noalloc",
           "bsa_selftest_wait_timeout", "bsa_mask_workspace_bytes", "bsa_mask_to_lists", "bsa_prefill_mask",
           "bsa_validate_lists", "bsa_score_group_workspace_bytes", "stem_score_group", "bsa_prefill_group",
           "bsa_prefill_skip", "bsa_score_select_workspace_bytes", "stem_score_select", "bsa_prefill_paged_group"]


class BsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class BsaTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("stride_b", ctypes.c_int64), ("stride_t", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


def lib():
    """Loads libbsa.so (raises if it is missing: there is no CPU or library fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise ImportError(f"{_LIB_PATH.name} is not built; run block_sparse_attention_42_b200.build.build()")
    L = ctypes.CDLL(str(_LIB_PATH))
    P, i32, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    T = BsaTensor
    L.bsa_tpd_budget.argtypes = [i32, f64, f64, P]
    L.bsa_tpd_budget.restype = i64
    L.bsa_score_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.bsa_score_workspace_bytes.restype = ctypes.c_size_t
    L.stem_score.argtypes = [T, T, T, i32, i32, i32, i32, i32, i32, i32, f32, P, i32, P, ctypes.c_size_t, P]
    L.stem_score_group.argtypes = L.stem_score.argtypes
    L.stem_score_select.argtypes = [T, T, T, i32, i32, i32, i32, i32, i32, i32, f32, f64, f64, P, P, i64, P,
                                    ctypes.c_size_t, P]
    L.bsa_score_select_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    L.bsa_score_select_workspace_bytes.restype = ctypes.c_size_t
    L.bsa_score_group_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.bsa_score_group_workspace_bytes.restype = ctypes.c_size_t
    L.stem_score_noalloc.argtypes = [T, T, T, i32, i32, i32, i32, i32, i32, i32, f32, P, i32, P]
    L.stem_select.argtypes = [P, i32, i32, P, i32, f64, f64, P, P, i64, P]
    L.bsa_prefill.argtypes = [T, T, T, T, i32, i32, i32, i32, i32, i32, P, i32, P, i64, f32, P, P]
    L.bsa_prefill_group.argtypes = L.bsa_prefill.argtypes
    L.bsa_prefill_skip.argtypes = [T, T, T, T, i32, i32, i32, i32, i32, i32, P, i32, P, i64, f32, f64, P, P, P]
    L.bsa_prefill_paged.argtypes = [T, T, P, P, i32, T, T, i32, i32, P, i32, i32, i32, i32, i32, P, i32, P, i64,
                                    f32, P, P]
    L.bsa_prefill_paged_group.argtypes = L.bsa_prefill_paged.argtypes
    L.bsa_mask_workspace_bytes.argtypes = [i32, i32, i32]
    L.bsa_mask_workspace_bytes.restype = ctypes.c_size_t
    L.bsa_mask_to_lists.argtypes = [P, i64, i32, i32, i32, P, P, i64, P]
    L.bsa_prefill_mask.argtypes = [T, T, T, T, i32, i32, i32, i32, i32, i32, P, i64, f32, P, P, ctypes.c_size_t, P]
    L.bsa_validate_lists.argtypes = [P, i64, i64, P, i64, i32, i32, P, i32, P]
    L.bsa_last_error.restype = ctypes.c_char_p
    L.bsa_check_device_error.argtypes = [P]
    L.bsa_selftest_wait_timeout.argtypes = [ctypes.c_uint64, P]
    for name in ["stem_score", "stem_score_select", "stem_score_group", "bsa_prefill_group", "bsa_prefill_skip", "stem_score_noalloc", "stem_select", "bsa_prefill", "bsa_prefill_paged", "bsa_prefill_paged_group", "bsa_check_device_error",
                 "bsa_selftest_wait_timeout", "bsa_mask_to_lists", "bsa_prefill_mask", "bsa_validate_lists"]:
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        raise BsaError(status, lib().bsa_last_error().decode())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return {torch.bfloat16: BSA_BF16, torch.float8_e4m3fn: BSA_FP8_E4M3, torch.float32: BSA_FP32}[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def tensor_arg(t: torch.Tensor, scale: float = 1.0) -> BsaTensor:
    """[B, N, H, d] (or packed [T, H, d]) tensor -> bsa_tensor_t.  The last dim must be contiguous."""
    if t.stride(-1) != 1:
        raise ValueError("the head_dim dimension must be contiguous")
    if t.dim() == 4:
        sb, st, sh = t.stride()[:3]
    elif t.dim() == 3:
        sb, (st, sh) = 0, t.stride()[:2]
    else:
        raise ValueError("expected a 4-D [B, N, H, d] or 3-D [T, H, d] tensor")
    return BsaTensor(t.data_ptr(), _dtype_code(t), float(scale), sb, st, sh)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def bsa_tpd_budget(nb: int, density: float, tpd_decay: float = 0.5):
    """Host TPD budget: (k [nb] int32 tensor, total)."""
    k = torch.zeros(max(nb, 1), dtype=torch.int32)
    tot = lib().bsa_tpd_budget(nb, float(density), float(tpd_decay), ctypes.c_void_p(k.data_ptr()))
    if tot < 0:
        raise BsaError(1, "invalid TPD arguments")
    return k[:nb], int(tot)


def tpd_kstar(nb: int, density: float, tpd_decay: float = 0.5) -> int:
    """K*, the TPD budget total of a sequence of nb blocks (bsa_tpd_budget with k_out = NULL)."""
    tot = lib().bsa_tpd_budget(nb, float(density), float(tpd_decay), None)
    if tot < 0:
        raise BsaError(1, "invalid TPD arguments")
    return int(tot)


def bsa_score_workspace_bytes(B, Hq, Hkv, nb, d) -> int:
    return int(lib().bsa_score_workspace_bytes(B, Hq, Hkv, nb, d))


def stem_score(q, k, v, block: int, metric: int = BSA_METRIC_OAM, softmax_scale: float = 0.0, scores=None,
               nb_stride: int | None = None, workspace=None, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """OAM block scores [B, Hq, nb_stride, nb_stride] fp32 (causal lower triangle valid)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    nb = (N + block - 1) // block
    nbs = nb if nb_stride is None else nb_stride
    if scores is None:
        scores = torch.empty(B, Hq, nbs, nbs, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(bsa_score_workspace_bytes(B, Hq, Hkv, nb, d), dtype=torch.uint8, device=q.device)
    st = lib().stem_score(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale), B, N, Hq, Hkv, d,
                          block, metric, float(softmax_scale), _ptr(scores), nbs, _ptr(workspace),
                          workspace.numel(), _stream(q))
    _check(st)
    return scores


def bsa_score_group_workspace_bytes(B, Hq, Hkv, nb, d) -> int:
    return int(lib().bsa_score_group_workspace_bytes(B, Hq, Hkv, nb, d))


def stem_score_group(q, k, v, block: int, metric: int = BSA_METRIC_OAM, softmax_scale: float = 0.0, scores=None,
                     nb_stride: int | None = None, workspace=None, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """Group-shared block scores [B, Hkv, nb_stride, nb_stride] fp32: one row per KV-head group,
    from the mean of the group's query heads' pooled Q (causal lower triangle valid)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    nb = (N + block - 1) // block
    nbs = nb if nb_stride is None else nb_stride
    if scores is None:
        scores = torch.empty(B, Hkv, nbs, nbs, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(bsa_score_group_workspace_bytes(B, Hq, Hkv, nb, d), dtype=torch.uint8,
                                device=q.device)
    st = lib().stem_score_group(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale), B, N, Hq,
                                Hkv, d, block, metric, float(softmax_scale), _ptr(scores), nbs, _ptr(workspace),
                                workspace.numel(), _stream(q))
    _check(st)
    return scores


def bsa_score_select_workspace_bytes(B, Hq, Hkv, N, block, d) -> int:
    return int(lib().bsa_score_select_workspace_bytes(B, Hq, Hkv, N, block, d))


def stem_score_select(q, k, v, block: int, density: float, tpd_decay: float = 0.5, metric: int = BSA_METRIC_OAM,
                      softmax_scale: float = 0.0, row_ptr=None, col_idx=None, max_k: int | None = None,
                      workspace=None, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """Score + TPD select without the score matrix: (row_ptr [B, nb+1], col_idx [B, Hq, max_k])."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    nb = (N + block - 1) // block
    if max_k is None:
        max_k = tpd_kstar(nb, density, tpd_decay)
    if row_ptr is None:
        row_ptr = torch.empty(B, nb + 1, dtype=torch.int32, device=q.device)
    if col_idx is None:
        col_idx = torch.empty(B, Hq, max_k, dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = torch.empty(bsa_score_select_workspace_bytes(B, Hq, Hkv, N, block, d), dtype=torch.uint8,
                                device=q.device)
    st = lib().stem_score_select(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale), B, N, Hq,
                                 Hkv, d, block, metric, float(softmax_scale), float(density), float(tpd_decay),
                                 _ptr(row_ptr), _ptr(col_idx), int(max_k), _ptr(workspace), workspace.numel(),
                                 _stream(q))
    _check(st)
    return row_ptr, col_idx


def stem_score_noalloc(q, k, v, block: int, metric: int = BSA_METRIC_OAM, softmax_scale: float = 0.0,
                       scores=None, nb_stride: int | None = None, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """stem_score with the library's fixed 32 MiB scratch instead of a workspace (for callers
    that cannot allocate device memory).  Calls that overlap on the GPU race on that scratch."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    nb = (N + block - 1) // block
    nbs = nb if nb_stride is None else nb_stride
    if scores is None:
        scores = torch.empty(B, Hq, nbs, nbs, dtype=torch.float32, device=q.device)
    st = lib().stem_score_noalloc(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale), B, N,
                                  Hq, Hkv, d, block, metric, float(softmax_scale), _ptr(scores), nbs, _stream(q))
    _check(st)
    return scores


def stem_select(scores, nb_per_seq, density: float, tpd_decay: float = 0.5, row_ptr=None, col_idx=None,
                max_k: int | None = None):
    """TPD budget + top-k: (row_ptr [B, nbs+1], col_idx [B, Hq, max_k]) int32 device tensors."""
    B, Hq, nbs, _ = scores.shape
    nbp = torch.tensor(list(nb_per_seq), dtype=torch.int32)
    if max_k is None:
        max_k = max(tpd_kstar(int(n), density, tpd_decay) for n in nbp)
    if row_ptr is None:
        row_ptr = torch.empty(B, nbs + 1, dtype=torch.int32, device=scores.device)
    if col_idx is None:
        col_idx = torch.empty(B, Hq, max_k, dtype=torch.int32, device=scores.device)
    st = lib().stem_select(_ptr(scores), B, Hq, ctypes.c_void_p(nbp.data_ptr()), nbs, float(density),
                           float(tpd_decay), _ptr(row_ptr), _ptr(col_idx), int(max_k), _stream(scores))
    _check(st)
    return row_ptr, col_idx


def bsa_prefill(q, k, v, block: int, row_ptr, col_idx, softmax_scale: float = 0.0, out=None, lse=None,
                return_lse: bool = False, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """Block-sparse causal prefill.  q [B,N,Hq,d], k/v [B,N,Hkv,d]; returns out (BF16)[, lse]."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty(B, N, Hq, d, dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    st = lib().bsa_prefill(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale), tensor_arg(out),
                           B, N, Hq, Hkv, d, block, _ptr(row_ptr), row_ptr.shape[-1], _ptr(col_idx),
                           col_idx.shape[-1], float(softmax_scale), _ptr(lse), _stream(q))
    _check(st)
    return (out, lse) if return_lse else out


def bsa_prefill_skip(q, k, v, block: int, row_ptr, col_idx, skip_lambda: float, softmax_scale: float = 0.0,
                     out=None, lse=None, return_lse: bool = False, q_scale=1.0, k_scale=1.0, v_scale=1.0,
                     skip_stats=None):
    """bsa_prefill with the threshold skip: a row drops a kept block whose max trails its running
    max by more than ln(skip_lambda) (0 drops nothing).  skip_stats: optional int64 device tensor
    of 4 counters (see bsa.h), incremented by the call."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty(B, N, Hq, d, dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    st = lib().bsa_prefill_skip(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale),
                                tensor_arg(out), B, N, Hq, Hkv, d, block, _ptr(row_ptr), row_ptr.shape[-1],
                                _ptr(col_idx), col_idx.shape[-1], float(softmax_scale), float(skip_lambda),
                                _ptr(lse), _ptr(skip_stats), _stream(q))
    _check(st)
    return (out, lse) if return_lse else out


def bsa_prefill_group(q, k, v, block: int, row_ptr, col_idx, softmax_scale: float = 0.0, out=None, lse=None,
                      return_lse: bool = False, q_scale=1.0, k_scale=1.0, v_scale=1.0):
    """Block-sparse causal prefill with one list per KV-head group: col_idx [B, Hkv, max_k] (from
    stem_select on stem_score_group's scores), shared by the group's query heads."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if col_idx.shape[1] != Hkv:
        raise ValueError("col_idx must be [B, Hkv, max_k]: one list per KV-head group")
    if out is None:
        out = torch.empty(B, N, Hq, d, dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    st = lib().bsa_prefill_group(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale),
                                 tensor_arg(out), B, N, Hq, Hkv, d, block, _ptr(row_ptr), row_ptr.shape[-1],
                                 _ptr(col_idx), col_idx.shape[-1], float(softmax_scale), _ptr(lse), _stream(q))
    _check(st)
    return (out, lse) if return_lse else out


def block_mask_buffer(B: int, Hq: int, nb: int, device=None, dtype=torch.uint8) -> torch.Tensor:
    """A zeroed [B, Hq, nb, nb] block mask whose rows start every multiple of 16 bytes, as
    bsa_prefill_mask needs (a view into a [B, Hq, nb, 16 * ceil(nb / 16)] buffer)."""
    ms = 16 * ((nb + 15) // 16)
    return torch.zeros(B, Hq, nb, ms, dtype=dtype, device=device)[..., :nb]


def _mask_arg(block_mask: torch.Tensor, B: int, Hq: int, nb: int):
    """(pointer, row stride) of a [B, Hq, nb, >= nb] uint8 / bool mask with unit last stride."""
    if block_mask.dtype == torch.bool:
        block_mask = block_mask.view(torch.uint8)
    if block_mask.dtype != torch.uint8:
        raise TypeError("block_mask must be uint8 or bool")
    if block_mask.dim() != 4 or tuple(block_mask.shape[:3]) != (B, Hq, nb) or block_mask.shape[3] < nb:
        raise ValueError(f"block_mask must be [B={B}, Hq={Hq}, nb={nb}, >= nb]")
    ms = block_mask.stride(2)
    if block_mask.stride(3) != 1 or block_mask.stride(1) != nb * ms or block_mask.stride(0) != Hq * nb * ms:
        raise ValueError("block_mask must be dense apart from row padding (see block_mask_buffer)")
    return ctypes.c_void_p(block_mask.data_ptr()), ms


def bsa_mask_workspace_bytes(B: int, Hq: int, nb: int) -> int:
    return int(lib().bsa_mask_workspace_bytes(B, Hq, nb))


def bsa_mask_to_lists(block_mask: torch.Tensor, row_ptr=None, col_idx=None):
    """Per-head lists of a block mask: (row_ptr [B, Hq, nb+1], col_idx [B, Hq, nb(nb+1)/2]) int32."""
    B, Hq, nb = block_mask.shape[:3]
    ptr, ms = _mask_arg(block_mask, B, Hq, nb)
    cap = nb * (nb + 1) // 2
    if row_ptr is None:
        row_ptr = torch.empty(B, Hq, nb + 1, dtype=torch.int32, device=block_mask.device)
    if col_idx is None:
        col_idx = torch.empty(B, Hq, cap, dtype=torch.int32, device=block_mask.device)
    _check(lib().bsa_mask_to_lists(ptr, ms, B, Hq, nb, _ptr(row_ptr), _ptr(col_idx), col_idx.shape[-1],
                                   _stream(block_mask)))
    return row_ptr, col_idx


def bsa_prefill_mask(q, k, v, block: int, block_mask, softmax_scale: float = 0.0, out=None, lse=None,
                     return_lse: bool = False, q_scale=1.0, k_scale=1.0, v_scale=1.0, workspace=None):
    """Block-sparse causal prefill from a block mask [B, Hq, nb, >= nb] (uint8 / bool)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    nb = (N + block - 1) // block
    ptr, ms = _mask_arg(block_mask, B, Hq, nb)
    if out is None:
        out = torch.empty(B, N, Hq, d, dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(bsa_mask_workspace_bytes(B, Hq, nb), 1), dtype=torch.uint8, device=q.device)
    st = lib().bsa_prefill_mask(tensor_arg(q, q_scale), tensor_arg(k, k_scale), tensor_arg(v, v_scale), tensor_arg(out),
                                B, N, Hq, Hkv, d, block, ptr, ms, float(softmax_scale), _ptr(lse),
                                _ptr(workspace), workspace.numel(), _stream(q))
    _check(st)
    return (out, lse) if return_lse else out


def bsa_validate_lists(row_ptr, col_idx, nb_per_seq, allow_empty: bool = False):
    """Debug check of a list set: row_ptr [B, nbs+1] (one per sequence, as stem_select writes) or
    [B, Hq, nb+1] (per head, as bsa_mask_to_lists writes); col_idx [B, Hq, max_k].  A violation
    shows up in bsa_check_device_error (BSA_ERR_INVALID_LIST)."""
    B, Hq, max_k = col_idx.shape
    if row_ptr.dim() == 2:
        rs, hs = row_ptr.stride(0), 0
    elif row_ptr.dim() == 3:
        rs, hs = row_ptr.stride(0), row_ptr.stride(1)
    else:
        raise ValueError("row_ptr must be [B, nbs+1] or [B, Hq, nb+1]")
    if row_ptr.stride(-1) != 1:
        raise ValueError("row_ptr rows must be contiguous")
    nbp = torch.tensor([int(n) for n in nb_per_seq], dtype=torch.int32)
    _check(lib().bsa_validate_lists(_ptr(row_ptr), rs, hs, _ptr(col_idx), max_k, B, Hq,
                                    ctypes.c_void_p(nbp.data_ptr()), 1 if allow_empty else 0, _stream(col_idx)))


def bsa_prefill_paged(q, cu_seqlens, seqlens, k_cache, v_cache, page_table, block: int, row_ptr, col_idx,
                      softmax_scale: float = 0.0, out=None, lse=None, return_lse: bool = False, q_scale=1.0,
                      k_scale=1.0, v_scale=1.0, _group: bool = False):
    """Paged-KV variant: q packed [sum N, Hq, d]; k_cache/v_cache [num_pages, page_size, Hkv, d]."""
    T, Hq, d = q.shape
    num_pages, page_size, Hkv, _ = k_cache.shape
    seqlens = [int(s) for s in seqlens]
    B = len(seqlens)
    sl = torch.tensor(seqlens, dtype=torch.int32)
    if out is None:
        out = torch.empty(T, Hq, d, dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, max(seqlens), dtype=torch.float32, device=q.device)
    kc, vc = tensor_arg(k_cache, k_scale), tensor_arg(v_cache, v_scale)
    fn = lib().bsa_prefill_paged_group if _group else lib().bsa_prefill_paged
    st = fn(tensor_arg(q, q_scale), tensor_arg(out), _ptr(cu_seqlens), ctypes.c_void_p(sl.data_ptr()), B, kc, vc,
            num_pages, page_size, _ptr(page_table), page_table.shape[-1], Hq, Hkv, d, block, _ptr(row_ptr),
            row_ptr.shape[-1], _ptr(col_idx), col_idx.shape[-1], float(softmax_scale), _ptr(lse), _stream(q))
    _check(st)
    return (out, lse) if return_lse else out


def bsa_prefill_paged_group(q, cu_seqlens, seqlens, k_cache, v_cache, page_table, block: int, row_ptr, col_idx,
                            softmax_scale: float = 0.0, out=None, lse=None, return_lse: bool = False, q_scale=1.0,
                            k_scale=1.0, v_scale=1.0):
    """bsa_prefill_paged with one list per KV-head group: col_idx [B, Hkv, max_k] (from stem_select
    on stem_score_group's scores), shared by the group's query heads."""
    if col_idx.shape[1] != k_cache.shape[2]:
        raise ValueError("col_idx must be [B, Hkv, max_k]: one list per KV-head group")
    return bsa_prefill_paged(q, cu_seqlens, seqlens, k_cache, v_cache, page_table, block, row_ptr, col_idx,
                             softmax_scale, out, lse, return_lse, q_scale, k_scale, v_scale, _group=True)


def bsa_check_device_error(device=None):
    """Synchronises the current stream and raises if a kernel recorded an error."""
    s = torch.cuda.current_stream(device)
    _check(lib().bsa_check_device_error(ctypes.c_void_p(s.cuda_stream)))


def bsa_selftest_wait_timeout(limit_ns: int = 50_000_000, device=None):
    """Launches the library's wait-timeout self-test kernel on the current stream (see bsa.h);
    a following bsa_check_device_error() raises BsaError with status BSA_ERR_TIMEOUT."""
    s = torch.cuda.current_stream(device)
    _check(lib().bsa_selftest_wait_timeout(int(limit_ns), ctypes.c_void_p(s.cuda_stream)))


def nb_of(N: int, block: int) -> int:
    return (N + block - 1) // block


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
