"""Backward pass (spattn_bwd_mask) against the oracle's gradients
(oracle.masked_sdpa_bwd, pinned by finite differences): dq, dk, dv and the
bias gradient for the five workload kinds at reduced sizes (several tiles,
ragged n, rows and columns above 1024 entries, one mask per batch element),
masks with empty and fully -inf rows, and fp32 inputs.

Tolerance, relative to the largest reference magnitude of each gradient
(G = max |g_ref|): bf16 inputs max-abs <= 1e-2 G and mean-abs <= 1e-3 G -- the
gradients are rounded to bf16 (2^-9 relative) and D_i = <dout_i, out_i> uses
the forward's bf16-rounded out, each a few 2^-9 of G; fp32 inputs 1e-4 G."""
import math

import numpy as np
import pytest

import oracle
import workloads
from helpers import build_mask, device_inputs, to_f64, torch_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp

GTOL = {workloads.BF16: (1e-2, 1e-3), workloads.F32: (1e-4, 1e-5)}


def grad_close(g, ref, dtype, what):
    tmax, tmean = GTOL[dtype]
    G = max(float(np.abs(ref).max()), 1e-30)
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    assert err.max() <= tmax * G, f"{what}: max-abs {err.max():.3g} > {tmax} * {G:.3g}"
    assert err.mean() <= tmean * G, f"{what}: mean-abs {err.mean():.3g} > {tmean} * {G:.3g}"


def _run(wl, m, rp, ci, want_dbias=False, seed=0):
    q, k, v, am, bias = device_inputs(wl)
    rng = np.random.default_rng(seed)
    dout_t = workloads.make_tensor(rng.standard_normal(q.shape), wl.dtype)
    dout = torch_tensor(dout_t)
    out, lse = sp.spattn_fwd_mask(q, k, v, m, add_mask=am, bias=bias, scale=wl.scale)
    dq, dk, dv, db = sp.spattn_bwd_mask(q, k, v, m, out, lse, dout, add_mask=am, bias=bias, scale=wl.scale,
                                        want_dbias=want_dbias)
    torch.cuda.synchronize()
    ref = oracle.masked_sdpa_bwd(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale,
                                 dout_t.raw, add_mask=None if wl.add_mask is None else wl.add_mask.raw,
                                 bias=None if wl.bias is None else wl.bias.raw, want_dbias=want_dbias)
    for name, g, r in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
        grad_close(to_f64(g), r, wl.dtype, name)
    if want_dbias:
        grad_close(db.double().cpu().numpy(), ref[3], wl.dtype, "dbias")
    assert sp.spattn_device_error() == 0
    return dq, dk, dv, db


@pytest.mark.parametrize("cfg,kw", [
    (0, dict()),                               # sliding window, fp32
    (1, dict(B=2, H=2, n=300)),                # variable window, one mask per batch element
    (2, dict(B=2, H=2, n=500)),                # random CSR
    (3, dict(B=1, H=2, n=1100)),               # block + strided + global: rows and columns > 1024
    (4, dict(B=3, H=2, n=200)),                # Evoformer: key padding + pair bias (and its gradient)
])
def test_backward_matches_oracle(cfg, kw):
    wl = workloads.make(cfg, **kw)
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask) as m:
        _run(wl, m, rp, ci, want_dbias=wl.bias is not None, seed=cfg)


@pytest.mark.parametrize("asynchronous", [False, True])
def test_backward_over_interval_mask_built_asynchronously(asynchronous):
    wl = workloads.make(1, B=1, H=3, n=640)
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask, asynchronous=asynchronous) as m:
        a = _run(wl, m, rp, ci, seed=7)
        b = _run(wl, m, rp, ci, seed=7)        # the transpose is reused; the result repeats exactly
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype,bias_shape", [(workloads.F32, "BHnn"), (workloads.BF16, "BHnn"),
                                              (workloads.BF16, "1Hnn"), (workloads.F32, "11nn"),
                                              (workloads.BF16, "111n")])
def test_backward_empty_and_masked_rows_and_bias_shapes(dtype, bias_shape):
    rng = np.random.default_rng(8)
    B, H, n, d = 2, 2, 150, 64
    rows, rp = [], [0]
    for i in range(n):
        c = np.nonzero(rng.random(n) < 0.3)[0]
        if i % 17 == 0:
            c = c[:0]                          # empty rows
        rows.append(c)
        rp.append(rp[-1] + c.size)
    rp = np.array(rp, np.int64)
    ci = np.concatenate(rows).astype(np.int32)
    q, k, v, dout = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), dtype) for _ in range(4))
    mask = np.zeros((B, 1, n, n))
    mask[:, :, 5, :] = -np.inf                 # a row whose scores are all -inf
    am = workloads.make_tensor(mask, dtype)
    shape = tuple({"B": B, "H": H, "n": n, "1": 1}[x] for x in bias_shape)
    bias = workloads.make_tensor(rng.standard_normal(shape), dtype)
    scale = 1 / math.sqrt(d)
    with sp.spattn_create_csr_mask("csr", n, 1, in_row_ptr=torch.from_numpy(rp.astype(np.int32)).cuda(),
                                   in_col_idx=torch.from_numpy(ci).cuda()) as m:
        dq_, dk_, dv_ = (torch_tensor(x) for x in (q, k, v))
        out, lse = sp.spattn_fwd_mask(dq_, dk_, dv_, m, add_mask=torch_tensor(am), bias=torch_tensor(bias),
                                      scale=scale)
        g = sp.spattn_bwd_mask(dq_, dk_, dv_, m, out, lse, torch_tensor(dout), add_mask=torch_tensor(am),
                               bias=torch_tensor(bias), scale=scale, want_dbias=True)
        torch.cuda.synchronize()
    ref = oracle.masked_sdpa_bwd(q.raw, k.raw, v.raw, rp, ci, 1, scale, dout.raw, add_mask=am.raw,
                                 bias=bias.raw, want_dbias=True)
    for name, x, r in (("dq", g[0], ref[0]), ("dk", g[1], ref[1]), ("dv", g[2], ref[2])):
        grad_close(to_f64(x), r, dtype, name)
    grad_close(g[3].double().cpu().numpy(), ref[3], dtype, "dbias")
    dq_h = to_f64(g[0])
    assert np.all(dq_h[:, :, 5] == 0) and np.all(dq_h[:, :, ::17] == 0)
    assert sp.spattn_device_error() == 0


def test_backward_argument_checks():
    wl = workloads.make(0)
    q, k, v, _, _ = device_inputs(wl)
    with build_mask(wl.mask) as m:
        out, lse = sp.spattn_fwd_mask(q, k, v, m)
        with pytest.raises(sp.SpattnError):     # dbias without bias
            sp.spattn_bwd_mask(q, k, v, m, out, lse, torch.zeros_like(q),
                               dbias=torch.zeros((1, 1, 1, wl.n), device="cuda"))
        with pytest.raises(sp.SpattnError):     # lse missing
            sp.spattn_bwd_mask(q, k, v, m, out, None, torch.zeros_like(q))
