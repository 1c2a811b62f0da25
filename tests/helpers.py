"""Test helpers: move seeded workloads to the GPU, build masks through the C ABI,
and compare the CUDA path with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np

import workloads

# Tolerances for out and lse (bf16 inputs with fp32 accumulation: max-abs 2e-2,
# mean-abs 2e-3 on out; fp32 inputs: 1e-4 on out). lse is returned in fp32, so
# its bound is an absolute part plus lse_rel * |lse| (about four fp32 ulps):
# with scores of magnitude 1e4 (a large additive bias) one ulp of lse is ~2e-3.
TOL = {
    workloads.BF16: dict(out_max=2e-2, out_mean=2e-3, lse_max=1e-3, lse_rel=5e-7),
    workloads.F32: dict(out_max=1e-4, out_mean=1e-4, lse_max=1e-5, lse_rel=5e-7),
}


def torch_tensor(t: workloads.Tensor, device="cuda"):
    import torch
    if t.dtype == workloads.BF16:
        x = torch.from_numpy(np.ascontiguousarray(t.raw).view(np.int16)).view(torch.bfloat16)
    else:
        x = torch.from_numpy(np.ascontiguousarray(t.raw))
    return x.to(device)


def device_inputs(wl: workloads.Workload, device="cuda"):
    q, k, v = (torch_tensor(x, device) for x in (wl.q, wl.k, wl.v))
    m = torch_tensor(wl.add_mask, device) if wl.add_mask is not None else None
    b = torch_tensor(wl.bias, device) if wl.bias is not None else None
    return q, k, v, m, b


def build_mask(mp: workloads.MaskParams, stream=None, tile_min_nnz=0, asynchronous=False):
    """The CUDA mask builder, from the same parameters the oracle builds from."""
    import torch
    import sparse_mask_scaled_b200 as sp
    kw = dict(window=mp.window, block=mp.block, stride=mp.stride, n_global=mp.n_global,
              add_diagonal=mp.add_diagonal, stream=stream, tile_min_nnz=tile_min_nnz,
              asynchronous=asynchronous)
    if mp.kind == "varwin":
        kw["half_widths"] = torch.from_numpy(np.ascontiguousarray(mp.half_widths, np.int32).ravel()).cuda()
    if mp.kind == "coo":
        kw["in_row_ptr"] = torch.from_numpy(mp.cand_row_ptr.astype(np.int32)).cuda()
        kw["in_col_idx"] = torch.from_numpy(mp.cand_cols.astype(np.int32)).cuda()
    return sp.spattn_create_csr_mask(mp.kind, mp.n, mp.num_masks, **kw)


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, dtype, what=""):
    """out_gpu: [rows, d] float64 numpy (already converted), lse_gpu: [rows]."""
    tol = TOL[dtype]
    err = np.abs(out_gpu - out_ref)
    assert np.all(np.isfinite(out_gpu)), f"{what}: non-finite output"
    assert err.max() <= tol["out_max"], f"{what}: out max-abs {err.max():.3g}"
    assert err.mean() <= tol["out_mean"], f"{what}: out mean-abs {err.mean():.3g}"
    # -inf exactly where the oracle has -inf (degenerate rows), close elsewhere
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ninf_ref), f"{what}: lse -inf pattern"
    if (~ninf_ref).any():
        le = np.abs(lse_gpu[~ninf_ref] - lse_ref[~ninf_ref])
        bound = tol["lse_max"] + tol["lse_rel"] * np.abs(lse_ref[~ninf_ref])
        assert np.all(le <= bound), f"{what}: lse max-abs {le.max():.3g} (bound {bound.min():.3g}..)"
    return float(err.max()), float(err.mean())


def to_f64(x):
    import torch
    return x.detach().to(torch.float64).cpu().numpy()
