"""Python binding of libspattn, the sparse-mask scaled dot-product attention
library for B200 (sm_100a) declared in ``include/spattn.h``.

This module only marshals arguments: torch tensors become ``spattn_tensor``
descriptors (pointer, dtype, shape, strides) and Python numbers become C
integers/floats. Every step of the computation runs in libspattn's CUDA kernels;
there is no fallback. Importing the module fails if ``libspattn.so`` has not been
built (``python sparse_mask_scaled_b200/_build.py``).

PyTorch provides device memory and streams only.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspattn.so")

# spattn_status
SPATTN_OK = 0
SPATTN_ERR_INVALID_ARG = 1
SPATTN_ERR_UNSUPPORTED = 2
SPATTN_ERR_BAD_CSR = 3
SPATTN_ERR_CUDA = 4
SPATTN_ERR_TIMEOUT = 5
SPATTN_ERR_OOM = 6
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "BAD_CSR", 4: "CUDA",
                5: "TIMEOUT", 6: "OOM"}

# spattn_dtype
SPATTN_BF16 = 0
SPATTN_F32 = 1

# spattn_mask_kind
SPATTN_MASK_CSR = 0
SPATTN_MASK_SLIDING = 1
SPATTN_MASK_VARWIN = 2
SPATTN_MASK_BLOCK_STRIDED_GLOBAL = 3
SPATTN_MASK_COO = 4
SPATTN_MASK_DENSE = 5
MASK_KINDS = {"csr": 0, "sliding": 1, "varwin": 2, "bsg": 3, "coo": 4, "dense": 5}


class SpattnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"spattn {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class spattn_tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("shape", ctypes.c_int64 * 4),
                ("stride", ctypes.c_int64 * 4)]


SPATTN_MASK_ASYNC = 1


class spattn_mask_spec(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("n", ctypes.c_int32), ("num_masks", ctypes.c_int32),
                ("window", ctypes.c_int32), ("block", ctypes.c_int32), ("stride", ctypes.c_int32),
                ("n_global", ctypes.c_int32), ("add_diagonal", ctypes.c_int32),
                ("half_widths", ctypes.c_void_p), ("in_row_ptr", ctypes.c_void_p),
                ("in_col_idx", ctypes.c_void_p), ("in_nnz", ctypes.c_int64),
                ("tile_min_nnz", ctypes.c_int32), ("flags", ctypes.c_uint32)]


_P = ctypes.c_void_p
_TP = ctypes.POINTER(spattn_tensor)
# name -> (restype, argtypes); one entry per function of include/spattn.h
SIGNATURES = {
    "spattn_create_csr_mask": (ctypes.c_int, [ctypes.POINTER(spattn_mask_spec), _P,
                                              ctypes.POINTER(_P)]),
    "spattn_mask_info": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(_P),
                                        ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_int64)]),
    "spattn_mask_copy_csr": (ctypes.c_int, [_P, _P, _P, _P]),
    "spattn_mask_copy_long_rows": (ctypes.c_int, [_P, _P, _P]),
    "spattn_mask_csr": (ctypes.c_int, [_P, ctypes.POINTER(_P), ctypes.POINTER(_P),
                                       ctypes.POINTER(ctypes.c_int64)]),
    "spattn_mask_plan_info": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int64),
                                             ctypes.POINTER(ctypes.c_int64),
                                             ctypes.POINTER(ctypes.c_int64)]),
    "spattn_mask_copy_plan": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P]),
    "spattn_mask_tile_count": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int64)]),
    "spattn_destroy_mask": (ctypes.c_int, [_P]),
    "spattn_fwd": (ctypes.c_int, [_TP, _TP, _TP, _P, _P, ctypes.c_int32, ctypes.c_int64, _TP, _TP,
                                  ctypes.c_float, _TP, _P, _P]),
    "spattn_fwd_mask": (ctypes.c_int, [_TP, _TP, _TP, _P, _TP, _TP, ctypes.c_float, _TP, _P, _P]),
    "spattn_fwd_noalloc": (ctypes.c_int, [_TP, _TP, _TP, _P, _P, ctypes.c_int32, ctypes.c_int64, _TP,
                                          _TP, ctypes.c_float, _TP, _P, _P]),
    "spattn_last_error": (ctypes.c_char_p, []),
    "spattn_device_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "spattn_check_device_error": (ctypes.c_int, [_P]),
    "spattn_fwd_mask_kpad": (ctypes.c_int, [_TP, _TP, _TP, _P, _P, _TP, _TP, ctypes.c_float, _TP, _P,
                                            _P]),
    "spattn_fwd_unfused": (ctypes.c_int, [_TP, _TP, _TP, _P, _P, ctypes.c_int32, ctypes.c_int64, _TP,
                                          _TP, ctypes.c_float, _TP, _P, _P]),
    "spattn_bwd_mask": (ctypes.c_int, [_TP, _TP, _TP, _P, _TP, _TP, ctypes.c_float, _TP, _P, _TP, _TP,
                                       _TP, _TP, _TP, _P]),
    "spattn_version": (ctypes.c_int, []),
    "spattn_launch_count": (ctypes.c_uint64, []),
    "spattn_alloc_count": (ctypes.c_uint64, []),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python sparse_mask_scaled_b200/_build.py`"
                          " (the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        if not hasattr(lib, name):
            raise ImportError(f"{LIB_PATH} does not export {name}: it is older than the sources,"
                              " rebuild it with `python sparse_mask_scaled_b200/_build.py`")
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def _check(status: int):
    if status != SPATTN_OK:
        raise SpattnError(status, LIB.spattn_last_error().decode())


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def tensor_desc(t) -> spattn_tensor:
    """Describe a 4-D torch tensor (bf16 or fp32) for the C ABI."""
    import torch
    if t.dim() != 4:
        raise ValueError("spattn tensors are 4-D")
    code = {torch.bfloat16: SPATTN_BF16, torch.float32: SPATTN_F32}.get(t.dtype)
    if code is None:
        raise ValueError(f"unsupported dtype {t.dtype}")
    d = spattn_tensor()
    d.data = t.data_ptr()
    d.dtype = code
    d.reserved = 0
    for x in range(4):
        d.shape[x] = t.shape[x]
        d.stride[x] = t.stride(x)
    return d


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


class Mask:
    """A mask built on the device by ``spattn_create_csr_mask`` (owns its memory).

    Sizes are read from the library on first use: for an asynchronous build that
    waits for it, and ``n_mixed_rows`` of an interval mask writes its explicit
    plan first."""

    def __init__(self, handle: int, n: int, num_masks: int):
        self.handle = handle
        self.n, self.num_masks = n, num_masks
        self._sizes = None
        self._plan_sizes = None
        self._mixed = None

    def _info(self):
        if self._sizes is None:
            nnz, nl = ctypes.c_int64(), ctypes.c_int64()
            _check(LIB.spattn_mask_info(self.handle, None, None, ctypes.byref(nnz), None, None,
                                        ctypes.byref(nl)))
            self._sizes = (nnz.value, nl.value)
        return self._sizes

    def _plan_info(self):
        if self._plan_sizes is None:
            nt, rn = ctypes.c_int64(), ctypes.c_int64()
            _check(LIB.spattn_mask_plan_info(self.handle, ctypes.byref(nt), ctypes.byref(rn), None))
            self._plan_sizes = (nt.value, rn.value)
        return self._plan_sizes

    @property
    def nnz(self) -> int:
        return self._info()[0]

    @property
    def n_long(self) -> int:
        return self._info()[1]

    @property
    def n_tiles(self) -> int:
        return self._plan_info()[0]

    @property
    def residual_nnz(self) -> int:
        return self._plan_info()[1]

    @property
    def tc_tiles(self) -> int:
        """128 x 128 tensor-core tiles one bf16 forward computes per (b, h),
        summed over the masks (spattn_mask_tile_count)."""
        t = ctypes.c_int64()
        _check(LIB.spattn_mask_tile_count(self.handle, ctypes.byref(t)))
        return t.value

    @property
    def n_mixed_rows(self) -> int:
        if self._mixed is None:
            nm = ctypes.c_int64()
            _check(LIB.spattn_mask_plan_info(self.handle, None, None, ctypes.byref(nm)))
            self._mixed = nm.value
        return self._mixed

    def csr(self, stream=None):
        """Copies of (row_ptr, col_idx) as int32 torch tensors on the current device."""
        import torch
        rp = torch.empty(self.num_masks * self.n + 1, dtype=torch.int32, device="cuda")
        ci = torch.empty(max(1, self.nnz), dtype=torch.int32, device="cuda")
        _check(LIB.spattn_mask_copy_csr(self.handle, rp.data_ptr(), ci.data_ptr(), _stream(stream)))
        return rp, ci[: self.nnz]

    def long_rows(self, stream=None):
        """The rows with more than 1024 nonzeros (mask-row ids m*n + i), sorted,
        as an int32 CUDA tensor."""
        import torch
        out = torch.empty(max(1, self.n_long), dtype=torch.int32, device="cuda")
        _check(LIB.spattn_mask_copy_long_rows(self.handle, out.data_ptr(), _stream(stream)))
        return torch.sort(out[: self.n_long]).values

    def plan(self, stream=None):
        """Copies of the tile plan (block_tile_off, tile_info, tile_bits,
        residual row_ptr, residual col_idx) as int32 CUDA tensors, or None."""
        import torch
        if self.n_tiles == 0:
            return None
        nqb = (self.n + 127) // 128
        bto = torch.empty(self.num_masks * nqb + 1, dtype=torch.int32, device="cuda")
        info = torch.empty(max(1, self.n_tiles), dtype=torch.int32, device="cuda")
        bits = torch.empty(max(1, self.n_tiles * 128 * 4), dtype=torch.int32, device="cuda")
        rrp = torch.empty(self.num_masks * self.n + 1, dtype=torch.int32, device="cuda")
        rci = torch.empty(max(1, self.residual_nnz), dtype=torch.int32, device="cuda")
        _check(LIB.spattn_mask_copy_plan(self.handle, bto.data_ptr(), info.data_ptr(), bits.data_ptr(),
                                         rrp.data_ptr(), rci.data_ptr(), _stream(stream)))
        return bto, info[: self.n_tiles], bits[: self.n_tiles * 512], rrp, rci[: self.residual_nnz]

    def close(self):
        if self.handle:
            _check(LIB.spattn_destroy_mask(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def spattn_create_csr_mask(kind, n: int, num_masks: int = 1, *, window: int = 0, block: int = 0,
                           stride: int = 0, n_global: int = 0, add_diagonal: bool = False,
                           half_widths=None, in_row_ptr=None, in_col_idx=None,
                           tile_min_nnz: int = 0, asynchronous: bool = False,
                           stream=None) -> Mask:
    """Build a CSR mask on the device. ``kind``: a name of MASK_KINDS or its code.
    Array arguments are int32 CUDA tensors. ``asynchronous``: SPATTN_MASK_ASYNC
    (interval masks are built without a host synchronisation)."""
    spec = spattn_mask_spec()
    spec.kind = MASK_KINDS[kind] if isinstance(kind, str) else int(kind)
    spec.n, spec.num_masks = n, num_masks
    spec.window, spec.block, spec.stride, spec.n_global = window, block, stride, n_global
    spec.add_diagonal = 1 if add_diagonal else 0
    spec.half_widths = _ptr(half_widths)
    spec.in_row_ptr = _ptr(in_row_ptr)
    spec.in_col_idx = _ptr(in_col_idx)
    spec.in_nnz = 0 if in_col_idx is None else int(in_col_idx.numel())
    spec.tile_min_nnz = int(tile_min_nnz)
    spec.flags = SPATTN_MASK_ASYNC if asynchronous else 0
    h = _P()
    _check(LIB.spattn_create_csr_mask(ctypes.byref(spec), _stream(stream), ctypes.byref(h)))
    return Mask(h.value, n, num_masks)


def _outputs(q, out, lse, want_lse):
    import torch
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[0] * q.shape[1] * q.shape[2], dtype=torch.float32,
                          device=q.device)
    return out, lse


def spattn_fwd(q, k, v, row_ptr, col_idx, num_masks: int = 1, add_mask=None, bias=None,
               scale: Optional[float] = None, out=None, lse=None, want_lse: bool = True,
               stream=None) -> Tuple[object, object]:
    """Masked attention over a raw device CSR (int32 row_ptr / col_idx tensors).
    Returns (out [B,H,n,d], lse [B*H*n] or None)."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    out, lse = _outputs(q, out, lse, want_lse)
    dq, dk, dv, do = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    dm = tensor_desc(add_mask) if add_mask is not None else None
    db = tensor_desc(bias) if bias is not None else None
    _check(LIB.spattn_fwd(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), _ptr(row_ptr),
                          _ptr(col_idx), int(num_masks), int(col_idx.numel()),
                          ctypes.byref(dm) if dm is not None else None,
                          ctypes.byref(db) if db is not None else None, float(scale),
                          ctypes.byref(do), _ptr(lse), _stream(stream)))
    return out, lse


def spattn_fwd_mask(q, k, v, mask: Mask, add_mask=None, bias=None, scale: Optional[float] = None,
                    out=None, lse=None, want_lse: bool = True, stream=None):
    """Masked attention over a mask built by spattn_create_csr_mask."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    out, lse = _outputs(q, out, lse, want_lse)
    dq, dk, dv, do = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    dm = tensor_desc(add_mask) if add_mask is not None else None
    db = tensor_desc(bias) if bias is not None else None
    _check(LIB.spattn_fwd_mask(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), mask.handle,
                               ctypes.byref(dm) if dm is not None else None,
                               ctypes.byref(db) if db is not None else None, float(scale),
                               ctypes.byref(do), _ptr(lse), _stream(stream)))
    return out, lse


def spattn_fwd_noalloc(q, k, v, row_ptr, col_idx, num_masks: int = 1, add_mask=None, bias=None,
                       scale: Optional[float] = None, out=None, lse=None, stream=None):
    """spattn_fwd without any device allocation inside the call: its scratch is
    a fixed array in the library (num_masks * n <= NOALLOC_MAX_ROWS). For
    callers that cannot allocate device memory while they run. ``out`` and
    ``lse`` must be passed in (this wrapper allocates nothing either)."""
    if out is None or lse is None:
        raise ValueError("spattn_fwd_noalloc needs caller-provided out and lse")
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    dq, dk, dv, do = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    dm = tensor_desc(add_mask) if add_mask is not None else None
    db = tensor_desc(bias) if bias is not None else None
    _check(LIB.spattn_fwd_noalloc(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv),
                                  _ptr(row_ptr), _ptr(col_idx), int(num_masks), int(col_idx.numel()),
                                  ctypes.byref(dm) if dm is not None else None,
                                  ctypes.byref(db) if db is not None else None, float(scale),
                                  ctypes.byref(do), _ptr(lse), _stream(stream)))
    return out, lse


NOALLOC_MAX_ROWS = 262143


def spattn_device_error(stream=None) -> int:
    """Synchronise the stream; return (and clear) the kernels' error flag bits."""
    flags = ctypes.c_uint32()
    st = LIB.spattn_device_error(_stream(stream), ctypes.byref(flags))
    if st not in (SPATTN_OK, SPATTN_ERR_BAD_CSR):
        _check(st)
    return flags.value


def spattn_check_device_error(stream=None) -> int:
    """Synchronise the stream, clear the kernels' error flags and return the
    status they map to (SPATTN_OK, SPATTN_ERR_TIMEOUT or SPATTN_ERR_BAD_CSR);
    raises only when the synchronisation itself fails."""
    st = LIB.spattn_check_device_error(_stream(stream))
    if st not in (SPATTN_OK, SPATTN_ERR_BAD_CSR, SPATTN_ERR_TIMEOUT):
        _check(st)
    return st


def spattn_mask_csr(mask: "Mask"):
    """The mask's own CSR through ``spattn_mask_csr``: (row_ptr address,
    col_idx address, nnz_total); the arrays belong to the mask."""
    rp, ci, nz = _P(), _P(), ctypes.c_int64()
    _check(LIB.spattn_mask_csr(mask.handle, ctypes.byref(rp), ctypes.byref(ci), ctypes.byref(nz)))
    return rp.value, ci.value, nz.value


def spattn_last_error() -> str:
    return LIB.spattn_last_error().decode()


def spattn_fwd_mask_kpad(q, k, v, mask: "Mask", seqlen_k, add_mask=None, bias=None,
                         scale: Optional[float] = None, out=None, lse=None, want_lse: bool = True,
                         stream=None) -> Tuple[object, object]:
    """``spattn_fwd_mask`` with key padding as lengths: ``seqlen_k`` is an int32
    CUDA tensor [B]; keys j >= seqlen_k[b] are left out."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    out, lse = _outputs(q, out, lse, want_lse)
    dq, dk, dv, do = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    dm = tensor_desc(add_mask) if add_mask is not None else None
    db = tensor_desc(bias) if bias is not None else None
    _check(LIB.spattn_fwd_mask_kpad(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), mask.handle,
                                    _ptr(seqlen_k), ctypes.byref(dm) if dm is not None else None,
                                    ctypes.byref(db) if db is not None else None, float(scale),
                                    ctypes.byref(do), _ptr(lse), _stream(stream)))
    return out, lse


def spattn_fwd_unfused(q, k, v, row_ptr, col_idx, num_masks: int = 1, add_mask=None, bias=None,
                       scale: Optional[float] = None, out=None, lse=None, want_lse: bool = True,
                       stream=None) -> Tuple[object, object]:
    """The forward as three separate stages (SDDMM, softmax, SpMM) with an
    nnz-sized fp32 score buffer; same arguments as ``spattn_fwd``."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    out, lse = _outputs(q, out, lse, want_lse)
    dq, dk, dv, do = tensor_desc(q), tensor_desc(k), tensor_desc(v), tensor_desc(out)
    dm = tensor_desc(add_mask) if add_mask is not None else None
    db = tensor_desc(bias) if bias is not None else None
    _check(LIB.spattn_fwd_unfused(ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), _ptr(row_ptr),
                                  _ptr(col_idx), int(num_masks), int(col_idx.numel()),
                                  ctypes.byref(dm) if dm is not None else None,
                                  ctypes.byref(db) if db is not None else None, float(scale),
                                  ctypes.byref(do), _ptr(lse), _stream(stream)))
    return out, lse


def spattn_bwd_mask(q, k, v, mask: "Mask", out, lse, dout, add_mask=None, bias=None,
                    scale: Optional[float] = None, want_dbias: bool = False, dq=None, dk=None, dv=None,
                    dbias=None, stream=None):
    """Gradients of sum(dout * out) for the forward over ``mask``: returns
    (dq, dk, dv, dbias or None); dbias is float32 with the bias's shape."""
    import torch
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    if want_dbias and dbias is None:
        dbias = torch.empty(bias.shape, dtype=torch.float32, device=bias.device)
    ds = [tensor_desc(x) for x in (q, k, v, out, dout, dq, dk, dv)]
    dm = tensor_desc(add_mask) if add_mask is not None else None
    db = tensor_desc(bias) if bias is not None else None
    ddb = tensor_desc(dbias) if dbias is not None else None
    _check(LIB.spattn_bwd_mask(ctypes.byref(ds[0]), ctypes.byref(ds[1]), ctypes.byref(ds[2]), mask.handle,
                               ctypes.byref(dm) if dm is not None else None,
                               ctypes.byref(db) if db is not None else None, float(scale),
                               ctypes.byref(ds[3]), _ptr(lse), ctypes.byref(ds[4]), ctypes.byref(ds[5]),
                               ctypes.byref(ds[6]), ctypes.byref(ds[7]),
                               ctypes.byref(ddb) if ddb is not None else None, _stream(stream)))
    return dq, dk, dv, dbias


def spattn_version() -> int:
    return LIB.spattn_version()


def spattn_launch_count() -> int:
    """Kernels the library has enqueued since it was loaded (all threads, devices)."""
    return int(LIB.spattn_launch_count())


def spattn_alloc_count() -> int:
    """Memory allocations the library has made since it was loaded (pool blocks,
    device and mapped host memory; all threads, devices)."""
    return int(LIB.spattn_alloc_count())
