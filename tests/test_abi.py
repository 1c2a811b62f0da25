"""The C ABI, checked without a GPU: every function include/*.h declares is
exported by libspattn.so and bound under the same name in Python, and argument
validation rejects bad calls before touching the device."""
import ctypes
import glob
import os
import re

import pytest

import sparse_mask_scaled_b200 as sp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?\w+\s*\**\s*(spattn_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ("spattn_create_csr_mask", "spattn_fwd", "spattn_fwd_mask", "spattn_destroy_mask"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(sp.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_python_binding_covers_every_symbol():
    names = _declared_functions()
    assert set(names) == set(sp.SIGNATURES)
    for n in names:
        if n in ("spattn_mask_info", "spattn_mask_copy_csr", "spattn_destroy_mask",
                 "spattn_mask_plan_info", "spattn_mask_copy_plan", "spattn_mask_tile_count",
                 "spattn_mask_copy_long_rows"):
            continue        # reached through sp.Mask
        assert callable(getattr(sp, n)), n


def test_struct_layouts_match_the_header():
    # spattn_tensor: pointer, 2 x int32, 4 x int64, 4 x int64
    assert ctypes.sizeof(sp.spattn_tensor) == 8 + 8 + 32 + 32
    assert sp.spattn_tensor.shape.offset == 16
    # spattn_mask_spec: 8 x int32, 3 pointers, int64, 2 x int32
    assert ctypes.sizeof(sp.spattn_mask_spec) == 32 + 24 + 8 + 8
    assert sp.spattn_mask_spec.half_widths.offset == 32
    assert sp.spattn_mask_spec.tile_min_nnz.offset == 64


def test_version():
    assert sp.spattn_version() >= 100


# ------------------------------------------------------------ host validation
def _desc(shape, dtype=sp.SPATTN_BF16, data=0x100000, strides=None, es=2):
    t = sp.spattn_tensor()
    t.data = data
    t.dtype = dtype
    t.reserved = 0
    if strides is None:
        strides, acc = [0] * 4, 1
        for x in range(3, -1, -1):
            strides[x] = acc
            acc *= shape[x]
    for x in range(4):
        t.shape[x] = shape[x]
        t.stride[x] = strides[x]
    return t


def _fwd(q, k=None, v=None, out=None, num_masks=1, mask=None, bias=None, nnz=10, row_ptr=0x200000,
         col_idx=0x300000):
    k = k or q
    v = v or q
    out = out or q
    st = sp.LIB.spattn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), row_ptr, col_idx,
                           num_masks, nnz, ctypes.byref(mask) if mask else None,
                           ctypes.byref(bias) if bias else None, 0.125, ctypes.byref(out), None, None)
    return st, sp.spattn_last_error()


S = (2, 3, 16, 64)


@pytest.mark.parametrize("d", [16, 48, 96, 256])
def test_unsupported_head_dim(d):
    st, msg = _fwd(_desc((2, 3, 16, d)))
    assert st == sp.SPATTN_ERR_UNSUPPORTED and "head dim" in msg


def test_shape_mismatch_is_invalid():
    st, msg = _fwd(_desc(S), k=_desc((2, 3, 17, 64)))
    assert st == sp.SPATTN_ERR_INVALID_ARG and "k shape" in msg


def test_dtype_mismatch_is_invalid():
    st, _ = _fwd(_desc(S), v=_desc(S, dtype=sp.SPATTN_F32))
    assert st == sp.SPATTN_ERR_INVALID_ARG


def test_misaligned_base_is_unsupported():
    st, msg = _fwd(_desc(S, data=0x100008))
    assert st == sp.SPATTN_ERR_UNSUPPORTED and "aligned" in msg


def test_row_stride_not_16_bytes_is_unsupported():
    st, msg = _fwd(_desc(S, strides=[3 * 16 * 68, 16 * 68, 68 + 1, 1]))
    assert st == sp.SPATTN_ERR_UNSUPPORTED


def test_inner_stride_must_be_one():
    st, msg = _fwd(_desc(S, strides=[3 * 16 * 64 * 2, 16 * 64 * 2, 64 * 2, 2]))
    assert st == sp.SPATTN_ERR_UNSUPPORTED and "stride 1" in msg


def test_num_masks_must_be_one_or_batch():
    st, msg = _fwd(_desc(S), num_masks=3)
    assert st == sp.SPATTN_ERR_INVALID_ARG and "num_masks" in msg


def test_negative_nnz_is_invalid():
    st, _ = _fwd(_desc(S), nnz=-1)
    assert st == sp.SPATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("shape,ok", [((2, 1, 1, 16), True), ((1, 3, 16, 16), True),
                                      ((2, 3, 16, 16), True), ((1, 1, 16, 1), True),
                                      ((2, 2, 16, 16), False), ((2, 1, 1, 15), False)])
def test_mask_and_bias_broadcast_rules(shape, ok):
    # shapes accepted per the AlphaFold2 mask/bias rules, generalised to any
    # broadcast over [B, H, n, n]; validation fails before any device work, so
    # an accepted shape is reported by the next check (null row_ptr here).
    m = _desc(shape, data=0x400000)
    st, msg = _fwd(_desc(S), mask=m, row_ptr=None)
    if ok:
        assert st == sp.SPATTN_ERR_INVALID_ARG and "row_ptr" in msg
    else:
        assert st == sp.SPATTN_ERR_INVALID_ARG and "broadcast" in msg
    st, msg = _fwd(_desc(S), bias=m, row_ptr=None)
    assert ("row_ptr" in msg) == ok


def _create(**kw):
    spec = sp.spattn_mask_spec()
    spec.kind = kw.get("kind", sp.SPATTN_MASK_SLIDING)
    spec.n = kw.get("n", 16)
    spec.num_masks = kw.get("num_masks", 1)
    spec.window = kw.get("window", 2)
    spec.block = kw.get("block", 0)
    spec.stride = kw.get("stride", 0)
    spec.n_global = kw.get("n_global", 0)
    spec.half_widths = kw.get("half_widths", None)
    spec.in_row_ptr = kw.get("in_row_ptr", None)
    spec.in_col_idx = kw.get("in_col_idx", None)
    spec.in_nnz = kw.get("in_nnz", 0)
    h = ctypes.c_void_p(1234)
    st = sp.LIB.spattn_create_csr_mask(ctypes.byref(spec), None, ctypes.byref(h))
    return st, h.value, sp.spattn_last_error()


@pytest.mark.parametrize("kw,frag", [(dict(kind=9), "kind"), (dict(n=0), "n must"),
                                     (dict(num_masks=0), "num_masks"), (dict(window=-1), "window"),
                                     (dict(kind=sp.SPATTN_MASK_VARWIN), "half_widths"),
                                     (dict(kind=sp.SPATTN_MASK_BLOCK_STRIDED_GLOBAL, block=-2), ">= 0"),
                                     (dict(kind=sp.SPATTN_MASK_COO), "in_row_ptr"),
                                     (dict(kind=sp.SPATTN_MASK_CSR, in_row_ptr=0x1000, in_nnz=5), "in_col_idx")])
def test_mask_spec_validation(kw, frag):
    st, h, msg = _create(**kw)
    assert st == sp.SPATTN_ERR_INVALID_ARG and frag in msg
    assert h is None            # *out cleared on error


def test_null_mask_handle():
    assert sp.LIB.spattn_destroy_mask(None) == sp.SPATTN_OK
    assert sp.LIB.spattn_mask_info(None, None, None, None, None, None, None) == sp.SPATTN_ERR_INVALID_ARG


def test_rejected_calls_launch_nothing():
    before = sp.spattn_launch_count()
    _fwd(_desc((2, 3, 16, 48)))
    _create(kind=9)
    _fwd(_desc(S), num_masks=3)
    assert sp.spattn_launch_count() == before
