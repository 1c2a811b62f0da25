"""Key padding given as lengths (spattn_fwd_mask_kpad): keys j >= seqlen_k[b]
are left out, which must equal the oracle with the additive key-padding mask
[B, 1, 1, n] (0 / -inf) -- the AlphaFold2 thread's mask -- on every path:
tensor-core tiles (d = 32, 64, 128; lengths at 0, inside and on tile edges),
interval masks with their gather kernel, gathered CSR rows and fp32 inputs."""
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


def _pad_mask(lengths, n):
    m = np.zeros((len(lengths), 1, 1, n))
    for b, L in enumerate(lengths):
        m[b, 0, 0, max(0, min(n, L)):] = -np.inf
    return m


def _check(wl_q, wl_k, wl_v, rp, ci, nm, n, d, dtype, lengths, mask_handle, bias=None, what=""):
    scale = 1 / math.sqrt(d)
    out_ref, lse_ref = oracle.masked_sdpa(wl_q.raw, wl_k.raw, wl_v.raw, rp, ci, nm, scale,
                                          add_mask=_pad_mask(lengths, n),
                                          bias=None if bias is None else bias.raw)
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out, lse = sp.spattn_fwd_mask_kpad(torch_tensor(wl_q), torch_tensor(wl_k), torch_tensor(wl_v), mask_handle,
                                       sl, bias=None if bias is None else torch_tensor(bias), scale=scale)
    torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1), dtype, what)
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("d", [32, 64, 128])
def test_dense_mask_lengths_on_tile_edges(d):
    lengths = [0, 1, 127, 128, 129, 255, 256]
    B, H, n = len(lengths), 2, 256
    rng = np.random.default_rng(d)
    q, k, v = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), workloads.BF16) for _ in range(3))
    rp, ci = oracle.mask_csr("dense", n)
    with sp.spattn_create_csr_mask("dense", n, 1) as m:
        assert m.n_tiles == 4
        _check(q, k, v, rp, ci, 1, n, d, workloads.BF16, lengths, m, what=f"dense d={d}")


def test_evoformer_with_lengths_and_bias():
    wl = workloads.make(4, B=5, H=2, n=256)
    keep = wl.add_mask.f64()[:, 0, 0, :] == 0
    lengths = [int(np.argmin(row)) if not row.all() else len(row) for row in keep]
    assert np.all(keep[np.arange(5)[:, None], np.arange(256)[None, :]] ==
                  (np.arange(256)[None, :] < np.array(lengths)[:, None]))
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask) as m:
        _check(wl.q, wl.k, wl.v, rp, ci, 1, wl.n, wl.d, wl.dtype, lengths, m, bias=wl.bias, what="evoformer")


def test_split_query_block_with_lengths():
    """d = 128, block + strided + global: query block 0's tile list is split into
    chunks; with 500 keys the second chunk has no tile left and only hands an
    empty partial state to the merge."""
    wl = workloads.make(3, B=2, H=2, n=2048)
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask) as m:
        _check(wl.q, wl.k, wl.v, rp, ci, wl.mask.num_masks, wl.n, wl.d, wl.dtype, [500, 1900], m,
               what="bsg d=128")


@pytest.mark.parametrize("thr", [0, 9000])
def test_variable_window_with_lengths(thr):
    wl = workloads.make(1, B=3, H=2, n=900)
    rng = np.random.default_rng(thr)
    lengths = [int(x) for x in rng.integers(300, 901, size=3)]
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask, tile_min_nnz=thr, asynchronous=True) as m:
        _check(wl.q, wl.k, wl.v, rp, ci, wl.mask.num_masks, wl.n, wl.d, wl.dtype, lengths, m,
               what=f"varwin thr={thr}")


@pytest.mark.parametrize("cfg,kw", [(2, dict(B=2, H=2, n=700)), (0, dict(B=2, H=2, n=300))])
def test_gathered_rows_with_lengths(cfg, kw):
    wl = workloads.make(cfg, **kw)
    lengths = [wl.n // 3, wl.n - 5]
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask) as m:
        _check(wl.q, wl.k, wl.v, rp, ci, wl.mask.num_masks, wl.n, wl.d, wl.dtype, lengths, m, what=f"cfg{cfg}")
