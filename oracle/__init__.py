"""Plain fp64 CPU oracle for the Stem block-sparse prefill path (ctypes over oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, the smoke check in ``__graft_entry__`` and the CPU
baseline leg of ``bench.py`` may use this package; the product library never does.  It
shares no code with the CUDA path; inputs reach both sides from
``block_sparse_attention_42_b200.inputs``.

Every function is a thin marshalling layer: the arithmetic lives in ``oracle.c`` and each
C function there cites the page and section it follows.  ``build()`` compiles the C file
with gcc (fp64, no FMA contraction, OpenMP).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

F32, BF16, E4M3, F64 = 0, 1, 2, 3
METRIC_OAM, METRIC_SAM, METRIC_OAM_MUL = 0, 1, 2


def build(force: bool = False) -> Path:
    """Compile oracle.c into liboracle.so (skipped when the .so is newer than the source)."""
    if not force and _LIB_PATH.exists() and _LIB_PATH.stat().st_mtime >= _SRC.stat().st_mtime:
        return _LIB_PATH
    tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp")
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", "-o", str(tmp), str(_SRC), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OrcTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("scale", ctypes.c_double), ("sb", ctypes.c_int64), ("st", ctypes.c_int64),
                ("sh", ctypes.c_int64)]


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(str(_LIB_PATH))
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    T = ctypes.POINTER(OrcTensor)
    lib.orc_decode_bf16.argtypes = [ctypes.c_uint16]
    lib.orc_decode_bf16.restype = f64
    lib.orc_decode_e4m3.argtypes = [ctypes.c_uint8]
    lib.orc_decode_e4m3.restype = f64
    lib.orc_decode_tensor.argtypes = [T, i64, i64, i64, i64, P]
    lib.orc_pool_mean.argtypes = [T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    lib.orc_pool_vnorm.argtypes = [T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    lib.orc_score.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, f64, ctypes.c_int, P]
    lib.orc_tpd_budget.argtypes = [i32, f64, f64, P]
    lib.orc_tpd_budget.restype = i64
    lib.orc_select_row.argtypes = [P, i32, i32, P]
    lib.orc_select.argtypes = [P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, f64, f64, P, P, i64]
    lib.orc_select.restype = ctypes.c_int
    lib.orc_attention_rows.argtypes = [T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, P, ctypes.c_int, P, i64, f64, P, i64, P, P, P]
    lib.orc_attention_rows_mask.argtypes = [T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, P, i64, f64, P, i64, P, P, P]
    lib.orc_effective_flop.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P,
                                       ctypes.c_int, P, i64, ctypes.c_int]
    lib.orc_effective_flop.restype = f64
    lib.orc_set_threads.argtypes = [ctypes.c_int]
    lib.orc_attention_rows_skip.argtypes = [T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, P, ctypes.c_int, P, i64, f64, f64, P, i64, P, P, P]
    lib.orc_group_mean.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class View:
    """A host array viewed as [B, N, H, D] with element strides; keeps the buffer alive."""

    def __init__(self, arr: np.ndarray, dtype: int, strides, scale: float = 1.0):
        self.arr = arr
        self.struct = OrcTensor(arr.ctypes.data, dtype, 0, float(scale), *[int(s) for s in strides])


def view(t, scale: float = 1.0) -> View:
    """Wrap a CPU tensor/array of shape [B, N, H, D] (last dim contiguous).

    torch bf16 / float8_e4m3fn tensors are passed as their raw bits; the oracle decodes them
    itself (``orc_decode_bf16`` / ``orc_decode_e4m3``)."""
    import torch

    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        assert t.dim() == 4 and t.stride(3) == 1
        strides = t.stride()[:3]
        if t.dtype == torch.bfloat16:
            arr, code = t.view(torch.int16).numpy(), BF16
        elif t.dtype == torch.float8_e4m3fn:
            arr, code = t.view(torch.uint8).numpy(), E4M3
        elif t.dtype == torch.float32:
            arr, code = t.numpy(), F32
        elif t.dtype == torch.float64:
            arr, code = t.numpy(), F64
        else:
            raise TypeError(t.dtype)
        # numpy keeps torch's strides; the base pointer is the tensor's data pointer.
        return View(arr, code, strides, scale)
    a = np.asarray(t)
    code = {np.dtype(np.float32): F32, np.dtype(np.float64): F64}[a.dtype]
    return View(a, code, [s // a.itemsize for s in a.strides[:3]], scale)


def decode_bf16(bits: int) -> float:
    return _load().orc_decode_bf16(bits)


def decode_e4m3(code: int) -> float:
    return _load().orc_decode_e4m3(code)


def decode(x: View, B: int, N: int, H: int, D: int) -> np.ndarray:
    out = np.empty((B, N, H, D), np.float64)
    _load().orc_decode_tensor(ctypes.byref(x.struct), B, N, H, D, _ptr(out))
    return out


def pool_mean(x: View, B, N, H, D, bs) -> np.ndarray:
    nb = (N + bs - 1) // bs
    out = np.empty((B, H, nb, D), np.float64)
    _load().orc_pool_mean(ctypes.byref(x.struct), B, N, H, D, bs, _ptr(out))
    return out


def pool_vnorm(v: View, B, N, H, D, bs) -> np.ndarray:
    nb = (N + bs - 1) // bs
    out = np.empty((B, H, nb), np.float64)
    _load().orc_pool_vnorm(ctypes.byref(v.struct), B, N, H, D, bs, _ptr(out))
    return out


def group_mean(qbar, Hkv: int) -> np.ndarray:
    """[B, Hq, nb, D] pooled queries -> [B, Hkv, nb, D] mean over each KV-head group's heads."""
    qbar = _c(qbar, np.float64)
    B, Hq, nb, D = qbar.shape
    out = np.empty((B, Hkv, nb, D), np.float64)
    _load().orc_group_mean(_ptr(qbar), B, Hq, Hkv, nb, D, _ptr(out))
    return out


def score(qbar, kbar, vbar, tau: float, metric: int = METRIC_OAM) -> np.ndarray:
    qbar, kbar, vbar = _c(qbar, np.float64), _c(kbar, np.float64), _c(vbar, np.float64)
    B, Hq, nb, D = qbar.shape
    Hkv = kbar.shape[1]
    S = np.empty((B, Hq, nb, nb), np.float64)
    _load().orc_score(_ptr(qbar), _ptr(kbar), _ptr(vbar), B, Hq, Hkv, nb, D, float(tau), metric, _ptr(S))
    return S


def tpd_budget(nb: int, density: float, decay: float = 0.5):
    """Returns (k [nb] int32, K*) or raises ValueError for invalid arguments."""
    k = np.zeros(max(nb, 1), np.int32)
    tot = _load().orc_tpd_budget(nb, float(density), float(decay), _ptr(k))
    if tot < 0:
        raise ValueError("invalid TPD arguments")
    return k[:nb], int(tot)


def select_row(srow, i: int, k_i: int) -> np.ndarray:
    srow = _c(srow, np.float64)
    out = np.zeros(max(k_i, 1), np.int32)
    _load().orc_select_row(_ptr(srow), i, k_i, _ptr(out))
    return out[:k_i]


def select(S, nb_per_seq, density: float, decay: float = 0.5, maxK: int | None = None):
    """Budget + top-k for [B, Hq, nbs, nbs] scores.  Returns (row_ptr [B, nbs+1], col_idx [B, Hq, maxK])."""
    S = _c(S, np.float64)
    B, Hq, nbs, _ = S.shape
    nbp = _c(nb_per_seq, np.int32)
    if maxK is None:
        maxK = max(tpd_budget(int(n), density, decay)[1] for n in nbp)
    row_ptr = np.zeros((B, nbs + 1), np.int32)
    col_idx = np.full((B, Hq, maxK), -1, np.int32)
    rc = _load().orc_select(_ptr(S), B, Hq, _ptr(nbp), nbs, float(density), float(decay),
                            _ptr(row_ptr), _ptr(col_idx), int(maxK))
    if rc != 0:
        raise ValueError("invalid select arguments")
    return row_ptr, col_idx


def attention_rows(q: View, k: View, v: View, N, Hq, Hkv, D, bs, row_ptr, col_idx, tau, rows,
                   with_amp: bool = False):
    """O and LSE (natural log) of the requested (b, h, t) query rows, fp64.  With with_amp,
    also the softmax average of |v| per output element (see orc_attention_rows)."""
    row_ptr = _c(row_ptr, np.int32)
    col_idx = _c(col_idx, np.int32)
    rows = _c(rows, np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    amp = np.empty((n, D), np.float64) if with_amp else None
    _load().orc_attention_rows(ctypes.byref(q.struct), ctypes.byref(k.struct), ctypes.byref(v.struct),
                               N, Hq, Hkv, D, bs, _ptr(row_ptr), row_ptr.shape[-1], _ptr(col_idx),
                               col_idx.shape[-1], float(tau), _ptr(rows), n, _ptr(out), _ptr(lse),
                               None if amp is None else _ptr(amp))
    return (out, lse, amp) if with_amp else (out, lse)


def attention_rows_skip(q: View, k: View, v: View, N, Hq, Hkv, D, bs, row_ptr, col_idx, tau, lam: float, rows):
    """O, LSE and the number of skipped list blocks of the requested (b, h, t) rows under the
    threshold skip with parameter lam (0 skips nothing), fp64."""
    row_ptr = _c(row_ptr, np.int32)
    col_idx = _c(col_idx, np.int32)
    rows = _c(rows, np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    skipped = np.empty((n,), np.int32)
    ln_lam = float(np.log(lam)) if lam > 0 else -np.inf
    _load().orc_attention_rows_skip(ctypes.byref(q.struct), ctypes.byref(k.struct), ctypes.byref(v.struct),
                                    N, Hq, Hkv, D, bs, _ptr(row_ptr), row_ptr.shape[-1], _ptr(col_idx),
                                    col_idx.shape[-1], float(tau), ln_lam, _ptr(rows), n, _ptr(out), _ptr(lse),
                                    _ptr(skipped))
    return out, lse, skipped


def attention_rows_mask(q: View, k: View, v: View, N, Hq, Hkv, D, bs, mask, tau, rows,
                        with_amp: bool = False):
    """O and LSE of the requested (b, h, t) rows with the selection as a block mask
    [B, Hq, nb, >= nb] (uint8; nonzero = kept), fp64.  Empty rows: O = 0, LSE = -inf.
    With with_amp, also the softmax average of |v| per output element."""
    mask = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    rows = _c(rows, np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    amp = np.empty((n, D), np.float64) if with_amp else None
    _load().orc_attention_rows_mask(ctypes.byref(q.struct), ctypes.byref(k.struct), ctypes.byref(v.struct),
                                    N, Hq, Hkv, D, bs, _ptr(mask), mask.shape[-1], float(tau), _ptr(rows), n,
                                    _ptr(out), _ptr(lse), None if amp is None else _ptr(amp))
    return (out, lse, amp) if with_amp else (out, lse)


def effective_flop(N, Hq, D, bs, row_ptr, col_idx, b: int = 0) -> float:
    row_ptr = _c(row_ptr, np.int32)
    col_idx = _c(col_idx, np.int32)
    return _load().orc_effective_flop(N, Hq, D, bs, _ptr(row_ptr), row_ptr.shape[-1], _ptr(col_idx),
                                      col_idx.shape[-1], b)


def set_threads(n: int) -> None:
    """Host threads of the oracle's parallel loops from now on (timing only; results do not
    depend on it)."""
    _load().orc_set_threads(int(n))
