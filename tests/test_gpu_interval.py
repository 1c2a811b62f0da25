"""Interval masks (sliding window, variable window, dense): every row is one run
of columns [lo, hi), so the mask keeps the runs and its tile selection, the
forward pass derives columns and tile bits from them, and the CSR is written
only on request. Built with or without waiting for the device, they must give
the oracle's result; the CSR written on request must be the brute-force mask;
an asynchronous build reports a negative half-width through the device error
flag and leaves that row empty."""
import math

import numpy as np
import pytest

import oracle
import workloads
from helpers import assert_close, build_mask, device_inputs, to_f64, torch_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp


def _oracle(wl, rp, ci):
    out, lse = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale,
                                  add_mask=None if wl.add_mask is None else wl.add_mask.raw,
                                  bias=None if wl.bias is None else wl.bias.raw)
    return out.reshape(-1, wl.d), lse.reshape(-1)


CASES = [
    (1, dict(B=2, H=2, n=1100), 0),        # variable window: every touched tile selected
    (1, dict(B=2, H=2, n=1100), 9000),     # variable window: window edges gathered, rows mixed
    (0, dict(), 0),                        # sliding window, fp32: gather only
    (0, dict(B=1, H=2, n=700), 2000),      # sliding window, fp32, ragged n
    (4, dict(B=3, H=2, n=256), 0),         # dense with key-padding mask and pair bias
    (4, dict(B=2, H=2, n=200), 20000),     # dense, nothing selected: gather only
]


@pytest.mark.parametrize("cfg,kw,thr", CASES)
@pytest.mark.parametrize("asynchronous", [False, True])
def test_interval_forward_matches_oracle(cfg, kw, thr, asynchronous):
    wl = workloads.make(cfg, **kw)
    rp, ci = oracle.mask_from_params(wl.mask)
    out_ref, lse_ref = _oracle(wl, rp, ci)
    q, k, v, am, bias = device_inputs(wl)
    with build_mask(wl.mask, tile_min_nnz=thr, asynchronous=asynchronous) as m:
        # the first call may run before the build's totals are known
        out, lse = sp.spattn_fwd_mask(q, k, v, m, add_mask=am, bias=bias, scale=wl.scale)
        torch.cuda.synchronize()
        out2, lse2 = sp.spattn_fwd_mask(q, k, v, m, add_mask=am, bias=bias, scale=wl.scale)
        torch.cuda.synchronize()
        assert m.nnz == rp[-1]
        assert m.n_long == int(np.sum(np.diff(rp) > 1024))
        grp, gci = m.csr()
        assert np.array_equal(grp.cpu().numpy(), rp) and np.array_equal(gci.cpu().numpy(), ci)
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref, lse_ref, wl.dtype,
                 f"cfg{cfg} thr={thr} async={asynchronous}")
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    assert sp.spattn_device_error() == 0


def test_asynchronous_build_is_one_kernel_and_no_wait():
    wl = workloads.make(1, B=2, H=2, n=1024)
    q, k, v, _, _ = device_inputs(wl)
    hw = torch.from_numpy(np.ascontiguousarray(wl.mask.half_widths, np.int32).ravel()).cuda()
    torch.cuda.synchronize()
    c0 = sp.spattn_launch_count()
    m = sp.spattn_create_csr_mask("varwin", wl.n, wl.mask.num_masks, half_widths=hw, asynchronous=True)
    assert sp.spattn_launch_count() - c0 == 1
    c1 = sp.spattn_launch_count()
    sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
    assert sp.spattn_launch_count() - c1 in (1, 2)    # tensor-core kernel, gather when unknown
    m.close()
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype,thr", [(workloads.F32, -1), (workloads.BF16, -1), (workloads.BF16, 16385),
                                       (workloads.BF16, 9000)])
def test_long_interval_rows(dtype, thr):
    """Rows of up to 3001 entries: above 1024 the eight warps of a block share a row."""
    n, w, B, H, d = 3000, 1500, 1, 2, 64
    rng = np.random.default_rng(11)
    q, k, v = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), dtype) for _ in range(3))
    mp = workloads.MaskParams("sliding", n, 1, window=w)
    rp, ci = oracle.mask_from_params(mp)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, 1 / math.sqrt(d))
    with build_mask(mp, tile_min_nnz=thr, asynchronous=True) as m:
        out, lse = sp.spattn_fwd_mask(torch_tensor(q), torch_tensor(k), torch_tensor(v), m,
                                      scale=1 / math.sqrt(d))
        torch.cuda.synchronize()
        assert np.array_equal(m.long_rows().cpu().numpy(), np.nonzero(np.diff(rp) > 1024)[0])
    assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1),
                 dtype, f"long rows thr={thr}")
    assert sp.spattn_device_error() == 0


def test_negative_half_width():
    """A negative half-width: the synchronous build rejects the mask; the
    asynchronous one leaves that row empty (out 0, lse -inf) and raises the
    device error flag, and every other row is exact."""
    wl = workloads.make(1, B=1, H=2, n=600)
    hw = np.ascontiguousarray(wl.mask.half_widths, np.int32).ravel().copy()
    bad = [0, 257, 599]
    hw[bad] = -3
    dhw = torch.from_numpy(hw).cuda()
    with pytest.raises(sp.SpattnError) as e:
        sp.spattn_create_csr_mask("varwin", wl.n, 1, half_widths=dhw)
    assert e.value.status == sp.SPATTN_ERR_BAD_CSR
    assert sp.spattn_device_error() == 0
    n = wl.n
    rows = []
    for i in range(n):
        rows.append(np.arange(max(0, i - hw[i]), min(n, i + hw[i] + 1)) if hw[i] >= 0 else np.zeros(0, int))
    rp = np.concatenate([[0], np.cumsum([r.size for r in rows])]).astype(np.int64)
    ci = np.concatenate(rows).astype(np.int32)
    out_ref, lse_ref = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, 1, wl.scale)
    q, k, v, _, _ = device_inputs(wl)
    with sp.spattn_create_csr_mask("varwin", wl.n, 1, half_widths=dhw, asynchronous=True) as m:
        out, lse = sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
        torch.cuda.synchronize()
        assert m.nnz == rp[-1]
    assert sp.spattn_device_error() & 1
    assert sp.spattn_device_error() == 0           # read and cleared
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref.reshape(-1, wl.d), lse_ref.reshape(-1),
                 wl.dtype, "negative half-width")
    lse_h = lse.cpu().numpy().reshape(2, n)
    assert np.all(np.isneginf(lse_h[:, bad]))


def test_oversized_interval_mask_takes_the_csr_builder():
    """More than 65,536 query blocks: the interval mask is built as a CSR (the
    explicit interval plan); its plan must equal the one the general CSR path
    builds from the same CSR."""
    n, nm, w = 256, 32769, 3
    with sp.spattn_create_csr_mask("sliding", n, nm, window=w) as a:
        rp, ci = a.csr()
        pa = a.plan()
        assert a.nnz == int(rp[-1].item())
        with sp.spattn_create_csr_mask("csr", n, nm, in_row_ptr=rp, in_col_idx=ci) as b:
            pb = b.plan()
            assert (a.n_tiles, a.residual_nnz, a.n_mixed_rows) == (b.n_tiles, b.residual_nnz, b.n_mixed_rows)
    for x, y in zip(pa, pb):
        assert torch.equal(x, y)
    # the pattern, checked on its first and last masks
    want = oracle.mask_from_params(workloads.MaskParams("sliding", n, 1, window=w))
    rph = rp.cpu().numpy().astype(np.int64)
    per = int(want[0][-1])
    assert np.array_equal(rph[: n + 1], want[0]) and rph[-1] == per * nm
    assert np.array_equal(ci[:per].cpu().numpy(), want[1]) and np.array_equal(ci[-per:].cpu().numpy(), want[1])
