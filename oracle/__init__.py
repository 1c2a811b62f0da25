"""TEST INFRASTRUCTURE: the fp64 CPU oracle for sparse-mask scaled dot-product attention.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The library (``sparse_mask_scaled_b200``)
never does, and nothing here imports the library: the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this file
only loads it and marshals numpy arrays. See ``oracle.c`` for which passage of
the pages each step follows.

Inputs: numpy arrays. ``uint16`` arrays are read as bf16 bit patterns,
``float32``/``float64`` arrays as their values; every input is widened to fp64
exactly. Additive mask/bias arrays are 4-D and broadcast to ``[B, H, n, n]``
(size-1 dimensions get stride 0).

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
(the gradients in ``tests/test_oracle_bwd_pins.py``: central finite differences
of the forward, closed forms for one nonzero per row, zero row sums of the score
gradient)
against facts fixed by the pages or by mathematics (dense softmax through
scipy, one nonzero per row, row sums, the streaming form against the two-pass
form, -inf mask entries against dropping them, shift invariance, uniform scores,
constant V, brute-force and closed-form mask counts, the worked key-padding mask
of the AlphaFold2 flash-attention thread, large-magnitude bias).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_F64, _F32, _BF16 = 0, 1, 2
KINDS = {"sliding": 1, "varwin": 2, "bsg": 3, "coo": 4, "dense": 5}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP, IEEE math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_sdpa.restype = I32
        lib.oracle_sdpa.argtypes = [I32, I64, I64, I64, I64, P, P, P, I32, I64, P, P, D,
                                    P, I32, P, P, I32, P, P, I64, P, P, I32]
        lib.oracle_row_weights.restype = I32
        lib.oracle_row_weights.argtypes = [I64, I64, I64, I64, P, P, P, I32, I64, P, P, D,
                                           P, I32, P, P, I32, P, I64, P]
        lib.oracle_sdpa_bwd.restype = I32
        lib.oracle_sdpa_bwd.argtypes = [I64, I64, I64, I64, P, P, P, I32, I64, P, P, D,
                                        P, I32, P, P, I32, P, P, I32, P, P, P, P, P, I64]
        lib.oracle_mask_csr.restype = I64
        lib.oracle_mask_csr.argtypes = [I32, I64, I64, I64, I64, I64, I64, P, P, P, I32, P, P]
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _elem(a: np.ndarray):
    """Contiguous array plus its oracle element-type code."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, _BF16
    if a.dtype == np.float32:
        return a, _F32
    return np.ascontiguousarray(a, dtype=np.float64), _F64


def _addend(a: Optional[np.ndarray], B: int, H: int, n: int):
    if a is None:
        return None, _F64, np.zeros(4, np.int64)
    if a.ndim != 4:
        raise ValueError("mask/bias must be 4-D")
    for got, full in zip(a.shape, (B, H, n, n)):
        if got not in (1, full):
            raise ValueError(f"shape {a.shape} does not broadcast to {(B, H, n, n)}")
    arr, t = _elem(a)
    strides = np.array([0 if arr.shape[x] == 1 else arr.strides[x] // arr.itemsize
                        for x in range(4)], dtype=np.int64)
    return arr, t, strides


def masked_sdpa(q: np.ndarray, k: np.ndarray, v: np.ndarray, row_ptr: np.ndarray,
                col_idx: np.ndarray, num_masks: int, scale: float,
                add_mask: Optional[np.ndarray] = None, bias: Optional[np.ndarray] = None,
                rows: Optional[Sequence[int]] = None, variant: str = "two_pass",
                threads: int = 0):
    """Attention over a CSR mask. q, k, v: [B, H, n, d]. row_ptr: [num_masks*n + 1].

    Returns (out, lse): out [B, H, n, d] and lse [B, H, n] in fp64, or, when
    ``rows`` lists flat row ids ``(b*H + h)*n + i``, out [len(rows), d] and
    lse [len(rows)].
    """
    B, H, n, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    qa, t = _elem(q)
    ka, tk = _elem(k)
    va, tv = _elem(v)
    assert t == tk == tv
    rp = np.ascontiguousarray(row_ptr, dtype=np.int64)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    assert rp.shape == (num_masks * n + 1,)
    ma, mt, ms = _addend(add_mask, B, H, n)
    ba, bt, bs = _addend(bias, B, H, n)
    if rows is None:
        rr, nr = None, B * H * n
    else:
        rr = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rr.size
    out = np.zeros((nr, d), np.float64)
    lse = np.zeros(nr, np.float64)
    rc = _load().oracle_sdpa({"two_pass": 0, "online": 1}[variant], B, H, n, d,
                             _ptr(qa), _ptr(ka), _ptr(va), t, num_masks, _ptr(rp), _ptr(ci),
                             float(scale), _ptr(ma), mt, _ptr(ms), _ptr(ba), bt, _ptr(bs),
                             _ptr(rr), nr, _ptr(out), _ptr(lse), int(threads))
    if rc != 0:
        raise ValueError("oracle_sdpa: bad argument")
    if rows is None:
        return out.reshape(B, H, n, d), lse.reshape(B, H, n)
    return out, lse


def row_weights(q, k, v, row_ptr, col_idx, num_masks, scale, flat_row,
                add_mask=None, bias=None) -> np.ndarray:
    """Softmax weights of one row in CSR order (two-pass definition)."""
    B, H, n, d = q.shape
    qa, t = _elem(q)
    ka, _ = _elem(k)
    va, _ = _elem(v)
    rp = np.ascontiguousarray(row_ptr, dtype=np.int64)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    ma, mt, ms = _addend(add_mask, B, H, n)
    ba, bt, bs = _addend(bias, B, H, n)
    i = flat_row % n
    b = flat_row // (H * n)
    r = (0 if num_masks == 1 else b) * n + i
    w = np.zeros(max(1, int(rp[r + 1] - rp[r])), np.float64)
    _load().oracle_row_weights(B, H, n, d, _ptr(qa), _ptr(ka), _ptr(va), t, num_masks,
                               _ptr(rp), _ptr(ci), float(scale), _ptr(ma), mt, _ptr(ms),
                               _ptr(ba), bt, _ptr(bs), int(flat_row), _ptr(w))
    return w[: int(rp[r + 1] - rp[r])]


def masked_sdpa_bwd(q, k, v, row_ptr, col_idx, num_masks, scale, dout, add_mask=None, bias=None,
                    want_dbias: bool = False):
    """Gradients (dq, dk, dv [B, H, n, d] fp64, and dbias with the bias's shape or
    None) of sum(dout * out) for the attention of ``masked_sdpa``."""
    B, H, n, d = q.shape
    qa, t = _elem(q)
    ka, tk = _elem(k)
    va, tv = _elem(v)
    assert t == tk == tv
    da, dt = _elem(dout)
    assert da.shape == q.shape
    rp = np.ascontiguousarray(row_ptr, dtype=np.int64)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    ma, mt, ms = _addend(add_mask, B, H, n)
    ba, bt, bs = _addend(bias, B, H, n)
    dq = np.zeros((B, H, n, d), np.float64)
    dk = np.zeros_like(dq)
    dv = np.zeros_like(dq)
    dbias, dbs, nb = None, None, 0
    if want_dbias:
        assert bias is not None
        dbias = np.zeros(bias.shape, np.float64)
        dbs = np.array([0 if dbias.shape[x] == 1 else dbias.strides[x] // 8 for x in range(4)], np.int64)
        nb = dbias.size
    rc = _load().oracle_sdpa_bwd(B, H, n, d, _ptr(qa), _ptr(ka), _ptr(va), t, num_masks, _ptr(rp),
                                 _ptr(ci), float(scale), _ptr(ma), mt, _ptr(ms), _ptr(ba), bt,
                                 _ptr(bs), _ptr(da), dt, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbias),
                                 _ptr(dbs), nb)
    if rc != 0:
        raise ValueError("oracle_sdpa_bwd: bad argument")
    return dq, dk, dv, dbias


def mask_csr(kind: str, n: int, num_masks: int = 1, *, window: int = 0, block: int = 0,
             stride: int = 0, n_global: int = 0, half_widths: Optional[np.ndarray] = None,
             cand_row_ptr: Optional[np.ndarray] = None, cand_cols: Optional[np.ndarray] = None,
             add_diagonal: bool = False):
    """Brute-force CSR (row_ptr int64 [num_masks*n + 1], col_idx int32) of a pattern."""
    lib = _load()
    hw = None if half_widths is None else np.ascontiguousarray(half_widths, dtype=np.int32).ravel()
    crp = None if cand_row_ptr is None else np.ascontiguousarray(cand_row_ptr, dtype=np.int64)
    cc = None if cand_cols is None else np.ascontiguousarray(cand_cols, dtype=np.int32)
    if kind == "varwin":
        assert hw is not None and hw.size == num_masks * n
    if kind == "coo":
        assert crp is not None and crp.size == num_masks * n + 1 and cc is not None
    row_ptr = np.zeros(num_masks * n + 1, np.int64)
    args = (KINDS[kind], n, num_masks, window, block, stride, n_global, _ptr(hw), _ptr(crp),
            _ptr(cc), int(bool(add_diagonal)), _ptr(row_ptr))
    nnz = lib.oracle_mask_csr(*args, None)
    if nnz < 0:
        raise ValueError("oracle_mask_csr: bad argument")
    col_idx = np.zeros(max(1, nnz), np.int32)
    lib.oracle_mask_csr(*args, _ptr(col_idx))
    return row_ptr, col_idx[:nnz]


def mask_from_params(mp) -> tuple:
    """Brute-force CSR for a ``workloads.MaskParams``."""
    return mask_csr(mp.kind, mp.n, mp.num_masks, window=mp.window, block=mp.block,
                    stride=mp.stride, n_global=mp.n_global, half_widths=mp.half_widths,
                    cand_row_ptr=mp.cand_row_ptr, cand_cols=mp.cand_cols,
                    add_diagonal=mp.add_diagonal)
