"""The persistent tile kernel (k_fwd_pp) against the fp64 oracle (needs a B200).

Block + strided + global masks whose parameters allow it (block dividing 128,
stride 0 or 128, at most 128 global tokens, n a multiple of 128) are kept in
closed form: the forward derives every tile and every row's bits from the
parameters and runs the regular query blocks and the residue-permuted blocks
of the strided entries in one launch, a regular block starting each of its rows
from the published partial state of the row's permuted part. These tests cover the parameter corners of that plan (no global tokens, no
block part, no strided part, permuted blocks shorter than a tile, more than one
permuted tile per residue, one mask per batch element), d = 64 and 128, the
fallbacks that go through the CSR-built copy of the mask (fp32 inputs, an
additive term, key lengths), interval masks (dense, sliding, variable window)
on the same kernel at d = 128 (and, with SPATTN_DEBUG_PP_INTERVAL=1, at
d = 32 and 64, where the default is the four-CTAs-per-SM tile kernel) -- with
additive mask and bias layouts staged through shared memory, key lengths, and
the layouts that fall back to the per-block kernels --, the entry points
spattn_mask_csr and spattn_check_device_error, and the bounded waits: with a
wait limit of zero cycles every wait gives up, the call reports
SPATTN_ERR_TIMEOUT, and the next call is exact again (the kernel released its
tensor memory and left no state).
"""
import ctypes
import math
import os

import numpy as np
import pytest

import oracle
import workloads
from helpers import assert_close, build_mask, device_inputs, to_f64, torch_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp


def _bsg(n, block, stride, ng, nm=1):
    return workloads.MaskParams("bsg", n, nm, block=block, stride=stride, n_global=ng)


def _inputs(rng, B, H, n, d, dtype=workloads.BF16, std=0.5):
    return [workloads.make_tensor(rng.standard_normal((B, H, n, d)) * std, dtype) for _ in range(3)]


def _rows_sample(rng, B, H, n, count):
    """Flat row ids (b*H + h)*n + i: every row of query block 0 and of the
    first residue's permuted rows, plus a random sample."""
    fixed = [i for i in range(min(n, 128))] + [k * 128 for k in range(n // 128)]
    rows = set()
    for bh in range(B * H):
        rows.update(bh * n + i for i in fixed)
    rows.update(rng.choice(B * H * n, size=min(count, B * H * n), replace=False).tolist())
    return np.array(sorted(rows), np.int64)


def _check(mp, B, H, d, seed=0, sample=None, what="", dtype=workloads.BF16):
    rng = np.random.default_rng(seed)
    n = mp.n
    q, k, v = _inputs(rng, B, H, n, d, dtype)
    rp, ci = oracle.mask_from_params(mp)
    scale = 1.0 / math.sqrt(d)
    rows = None if sample is None else _rows_sample(rng, B, H, n, sample)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, mp.num_masks, scale, rows=rows)
    with build_mask(mp) as m:
        assert m.nnz == rp[-1]
        assert m.n_long == int(np.sum(np.diff(rp) > 1024))
        out, lse = sp.spattn_fwd_mask(torch_tensor(q), torch_tensor(k), torch_tensor(v), m, scale=scale)
        torch.cuda.synchronize()
    got = to_f64(out).reshape(-1, d)
    gl = to_f64(lse)
    if rows is not None:
        got, gl = got[rows], gl[rows]
    assert_close(got, gl, out_ref.reshape(-1, d), lse_ref.reshape(-1), dtype, what)
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("n,block,stride,ng,d,B,H,nm", [
    (2048, 64, 128, 32, 128, 1, 2, 1),     # the block + strided + global workload's pattern, reduced
    (2048, 64, 128, 32, 64, 1, 2, 1),      # d = 64
    (384, 64, 128, 32, 128, 2, 1, 2),      # three positions per residue; one mask per batch element
    (1024, 32, 128, 0, 128, 1, 2, 1),      # no global tokens
    (1024, 0, 128, 16, 64, 1, 1, 1),       # no block part
    (1024, 128, 0, 8, 128, 1, 2, 1),       # no strided part
    (1280, 16, 128, 128, 128, 1, 1, 1),    # 128 global rows: query block 0 entirely global
    (256, 1, 128, 1, 128, 2, 2, 1),        # two positions per residue
])
def test_closed_form_matches_oracle(n, block, stride, ng, d, B, H, nm):
    _check(_bsg(n, block, stride, ng, nm), B, H, d, seed=n + block + ng,
           what=f"closed form n={n} block={block} S={stride} ng={ng} d={d}")


def test_closed_form_two_permuted_tiles_per_residue():
    """n = 32768: 256 positions per residue, so every permuted block walks two
    key tiles and each residue has two permuted blocks; sampled rows."""
    _check(_bsg(32768, 64, 128, 32), 1, 1, 128, seed=7, sample=3000, what="n=32768")


def test_closed_form_repeated_calls_and_layouts():
    """Two calls in a row (the per-call counts start from zero again), no lse,
    and an output written through a strided (non-contiguous) view."""
    mp = _bsg(1024, 64, 128, 32)
    B, H, d, n = 2, 2, 128, 1024
    rp, ci = oracle.mask_from_params(mp)
    with build_mask(mp) as m:
        for seed in (1, 2):
            rng = np.random.default_rng(seed)
            q, k, v = _inputs(rng, B, H, n, d)
            out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, 1 / math.sqrt(d))
            big = torch.zeros((B, n, H, d), dtype=torch.bfloat16, device="cuda")
            out = big.permute(0, 2, 1, 3)                 # [B, H, n, d] view, row stride H*d
            sp.spattn_fwd_mask(torch_tensor(q), torch_tensor(k), torch_tensor(v), m, out=out, want_lse=False)
            lse = torch.empty(B * H * n, dtype=torch.float32, device="cuda")
            out2, _ = sp.spattn_fwd_mask(torch_tensor(q), torch_tensor(k), torch_tensor(v), m, lse=lse)
            torch.cuda.synchronize()
            assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1),
                         workloads.BF16, f"strided out, call {seed}")
            assert torch.equal(out.contiguous(), out2)     # same bits either way
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("case", ["f32", "mask", "kpad"])
def test_closed_form_fallbacks(case):
    """Inputs the closed-form kernel does not take run over the mask's
    CSR-built copy, with the same results."""
    n, B, H, d = 1024, 2, 1, 64
    mp = _bsg(n, 64, 128, 32)
    rng = np.random.default_rng(11)
    dtype = workloads.F32 if case == "f32" else workloads.BF16
    q, k, v = _inputs(rng, B, H, n, d, dtype)
    rp, ci = oracle.mask_from_params(mp)
    am = None
    lengths = None
    if case == "mask":
        am = workloads.make_tensor(np.where(rng.random((B, 1, 1, n)) < 0.1, -np.inf, 0.0), workloads.BF16)
    if case == "kpad":
        lengths = np.array([700, 1024], np.int64)
        am = workloads.make_tensor(np.where(np.arange(n)[None, None, None, :] >= lengths[:, None, None, None],
                                            -np.inf, 0.0), workloads.BF16)
    scale = 1 / math.sqrt(d)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, scale,
                                          add_mask=None if am is None else am.raw)
    with build_mask(mp) as m:
        if case == "kpad":
            sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
            out, lse = sp.spattn_fwd_mask_kpad(torch_tensor(q), torch_tensor(k), torch_tensor(v), m, sl,
                                               scale=scale)
        else:
            out, lse = sp.spattn_fwd_mask(torch_tensor(q), torch_tensor(k), torch_tensor(v), m,
                                          add_mask=None if am is None else torch_tensor(am), scale=scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1), dtype,
                 f"fallback {case}")
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("n,B,H", [(1000, 1, 2), (512, 2, 2)])
def test_dense_interval_mask_d128(n, B, H):
    """An all-ones mask at d = 128 on the persistent kernel (ragged last tiles
    when n is not a multiple of 128)."""
    mp = workloads.MaskParams("dense", n, 1)
    _check(mp, B, H, 128, seed=n, what=f"dense d=128 n={n}")


@pytest.mark.parametrize("route", ["default", "persistent"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("layout", ["row_mask", "bias_only", "pad_mask_and_bias", "row_mask_and_bias",
                                    "f32_bias", "head_mask"])
@pytest.mark.parametrize("kind,n", [("dense", 256), ("sliding", 384), ("dense", 200)])
def test_interval_mask_with_additive_terms(d, layout, kind, n, route, monkeypatch):
    """Additive mask and bias on interval masks at d <= 64: by default on the
    four-CTAs-per-SM tile kernel (its build that stages the row-varying term by
    TMA for the bf16 layouts, the one that prefetches it into registers for the
    fp32 bias); with SPATTN_DEBUG_PP_INTERVAL=1 on the
    persistent kernel, where bf16 terms with keys contiguous and 16-byte rows
    are staged through shared memory tile by tile (row-varying, shared by all
    rows, per head) and an fp32 term, or rows that are not 16-byte multiples
    (n = 200: 400-byte rows are, n odd would not), take the per-block kernel;
    every route must equal the oracle."""
    if route == "persistent":
        monkeypatch.setenv("SPATTN_DEBUG_PP_INTERVAL", "1")
    rng = np.random.default_rng(7 + d + n)
    B, H = 2, 3
    mp = workloads.MaskParams(kind, n, 1, window=40 if kind == "sliding" else 0)
    q, k, v = _inputs(rng, B, H, n, d, std=1.0)
    row_mask = workloads.make_tensor(np.where(rng.random((B, 1, n, n)) < 0.1, -np.inf,
                                              rng.standard_normal((B, 1, n, n))), workloads.BF16)
    pad_mask = workloads.make_tensor(np.where(rng.random((B, 1, 1, n)) < 0.2, -np.inf, 0.0), workloads.BF16)
    head_mask = workloads.make_tensor(np.where(rng.random((1, H, 1, n)) < 0.2, -np.inf, 0.0), workloads.BF16)
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)), workloads.BF16)
    bias32 = workloads.make_tensor(rng.standard_normal((1, H, n, n)), workloads.F32)
    am, b = {"row_mask": (row_mask, None), "bias_only": (None, bias), "pad_mask_and_bias": (pad_mask, bias),
             "row_mask_and_bias": (row_mask, bias), "f32_bias": (pad_mask, bias32),
             "head_mask": (head_mask, bias)}[layout]
    rp, ci = oracle.mask_from_params(mp)
    scale = 1 / math.sqrt(d)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, scale,
                                          add_mask=None if am is None else am.raw,
                                          bias=None if b is None else b.raw)
    with build_mask(mp) as m:
        out, lse = sp.spattn_fwd_mask(torch_tensor(q), torch_tensor(k), torch_tensor(v), m,
                                      add_mask=None if am is None else torch_tensor(am),
                                      bias=None if b is None else torch_tensor(b), scale=scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1),
                 workloads.BF16, f"{kind} n={n} d={d} {layout}")
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("d,route", [(32, "default"), (32, "persistent"), (64, "default"), (64, "persistent"),
                                     (128, "default")])
def test_key_lengths_with_bias_on_the_persistent_kernel(d, route, monkeypatch):
    """Key lengths on tile edges with a pair bias (on the persistent kernel,
    d <= 64 stages the bias; at d = 128 the bias takes the per-block kernel),
    against the oracle with the equivalent additive key-padding mask."""
    if route == "persistent":
        monkeypatch.setenv("SPATTN_DEBUG_PP_INTERVAL", "1")
    lengths = [0, 1, 127, 128, 129, 255, 256, 200]
    B, H, n = len(lengths), 2, 256
    rng = np.random.default_rng(30 + d)
    q, k, v = _inputs(rng, B, H, n, d, std=1.0)
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)), workloads.BF16)
    pad = np.zeros((B, 1, 1, n))
    for bb, L in enumerate(lengths):
        pad[bb, 0, 0, L:] = -np.inf
    rp, ci = oracle.mask_csr("dense", n)
    scale = 1 / math.sqrt(d)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, scale, add_mask=pad, bias=bias.raw)
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    with sp.spattn_create_csr_mask("dense", n, 1, asynchronous=True) as m:
        out, lse = sp.spattn_fwd_mask_kpad(torch_tensor(q), torch_tensor(k), torch_tensor(v), m, sl,
                                           bias=torch_tensor(bias), scale=scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1),
                 workloads.BF16, f"lengths + bias d={d}")
    assert sp.spattn_device_error() == 0


def test_variable_window_d128():
    """A variable-window mask at d = 128: tiles on the persistent kernel, the
    window edges outside them gathered first and merged in its epilogue."""
    wl = workloads.make(1, B=2, H=2, n=1000, d=128)
    q, k, v, _, _ = device_inputs(wl)
    rp, ci = oracle.mask_from_params(wl.mask)
    out_ref, lse_ref = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale)
    with build_mask(wl.mask) as m:
        out, lse = sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, 128), to_f64(lse), out_ref.reshape(-1, 128), lse_ref.reshape(-1),
                 workloads.BF16, "varwin d=128")
    assert sp.spattn_device_error() == 0


class _DeviceArray:
    """An int32 device array owned by the library, viewed by torch without a copy."""

    def __init__(self, ptr, count):
        self.__cuda_array_interface__ = {"shape": (count,), "typestr": "<i4", "data": (ptr, False),
                                         "version": 2}


def test_mask_csr_and_check_device_error_entry_points():
    """spattn_mask_csr hands out the mask's own device CSR (equal to the
    oracle's); spattn_check_device_error reports a skipped out-of-range column
    as SPATTN_ERR_BAD_CSR once, then SPATTN_OK."""
    mp = _bsg(512, 64, 128, 32)
    rp_ref, ci_ref = oracle.mask_from_params(mp)
    with build_mask(mp) as m:
        rp_ptr, ci_ptr = ctypes.c_void_p(), ctypes.c_void_p()
        nnz = ctypes.c_int64()
        st = sp.LIB.spattn_mask_csr(m.handle, ctypes.byref(rp_ptr), ctypes.byref(ci_ptr), ctypes.byref(nnz))
        assert st == sp.SPATTN_OK, sp.spattn_last_error()
        assert nnz.value == rp_ref[-1]
        torch.cuda.synchronize()
        rp = torch.as_tensor(_DeviceArray(rp_ptr.value, rp_ref.size), device="cuda")
        ci = torch.as_tensor(_DeviceArray(ci_ptr.value, int(nnz.value)), device="cuda")
        assert np.array_equal(rp.cpu().numpy(), rp_ref)
        assert np.array_equal(ci.cpu().numpy(), ci_ref)
    stream = torch.cuda.current_stream().cuda_stream
    assert sp.LIB.spattn_check_device_error(stream) == sp.SPATTN_OK
    n, d = 64, 32
    q = torch.randn((1, 1, n, d), device="cuda").to(torch.bfloat16)
    bad_rp = torch.tensor([0] + [1] * n, dtype=torch.int32, device="cuda")
    bad_ci = torch.tensor([n + 5], dtype=torch.int32, device="cuda")   # outside [0, n): skipped, flagged
    sp.spattn_fwd(q, q, q, bad_rp, bad_ci, 1)
    assert sp.LIB.spattn_check_device_error(stream) == sp.SPATTN_ERR_BAD_CSR
    assert sp.LIB.spattn_check_device_error(stream) == sp.SPATTN_OK        # read and cleared


def test_expired_waits_report_timeout_and_leave_no_state(monkeypatch):
    """With the wait limit at zero cycles every bounded wait in the persistent
    kernel gives up at once: the CTAs drain what they issued, free their
    tensor memory and raise the timeout flag (no arrival is held back, so
    everything issued completes). The next call, with the normal limit, is
    exact again."""
    mp = _bsg(1024, 64, 128, 32)
    B, H, d, n = 1, 2, 128, 1024
    rng = np.random.default_rng(5)
    q, k, v = _inputs(rng, B, H, n, d)
    rp, ci = oracle.mask_from_params(mp)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, 1 / math.sqrt(d))
    dq, dk, dv = torch_tensor(q), torch_tensor(k), torch_tensor(v)
    stream = torch.cuda.current_stream().cuda_stream
    assert sp.LIB.spattn_check_device_error(stream) == sp.SPATTN_OK
    with build_mask(mp) as m:
        monkeypatch.setenv("SPATTN_DEBUG_WAIT_CYCLES", "0")
        sp.spattn_fwd_mask(dq, dk, dv, m)
        assert sp.LIB.spattn_check_device_error(stream) == sp.SPATTN_ERR_TIMEOUT
        monkeypatch.delenv("SPATTN_DEBUG_WAIT_CYCLES")
        out, lse = sp.spattn_fwd_mask(dq, dk, dv, m)
        assert sp.LIB.spattn_check_device_error(stream) == sp.SPATTN_OK
    assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1),
                 workloads.BF16, "after the expired call")
