"""The tile plan and the tensor-core (tcgen05) path, against the oracle.

Plan (integer work, bit-exact): a 128 x 128 tile is selected exactly when it
holds at least tile_min_nnz nonzeros, its per-row bits list exactly its CSR
entries, it is flagged dense exactly when all 128 x 128 entries are present,
and the selected tiles' entries plus the residual CSR are the whole CSR.

Forward (bf16 inputs): masks whose entries all sit in tiles, masks mixing tile
and residual entries in the same rows, ragged n, head dims 32/64/128, additive
mask and bias -- within the bf16 tolerance of the oracle.
"""
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


def _tile_counts(rp, ci, n, nm):
    nqb = (n + 127) // 128
    cnt = np.zeros((nm * nqb, nqb), np.int64)
    for r in range(nm * n):
        m, i = divmod(r, n)
        cols = ci[rp[r]:rp[r + 1]]
        np.add.at(cnt[m * nqb + i // 128], cols // 128, 1)
    return cnt


def _check_plan(mask, rp, ci, n, nm, thr):
    plan = mask.plan()
    cnt = _tile_counts(rp, ci, n, nm)
    sel = cnt >= thr
    if not sel.any():
        assert plan is None and mask.n_tiles == 0
        return
    bto, info, bits, rrp, rci = (x.cpu().numpy() for x in plan)
    nqb = (n + 127) // 128
    assert mask.n_tiles == int(sel.sum())
    assert np.array_equal(np.diff(bto), sel.sum(axis=1))
    covered = set()
    for x in range(nm * nqb):
        kts = (info[bto[x]:bto[x + 1]] & 0x7fffffff)
        assert np.array_equal(kts, np.nonzero(sel[x])[0])
        m, qb = divmod(x, nqb)
        for t in range(bto[x], bto[x + 1]):
            kt = info[t] & 0x7fffffff
            dense = info[t] < 0
            assert dense == (cnt[x, kt] == 128 * 128)
            w = bits[t * 512:(t + 1) * 512].view(np.uint32).reshape(128, 4)
            if dense:      # all entries present; bits are not stored
                assert not w.any()
                covered.update((m * n + qb * 128 + rr, kt * 128 + c) for rr in range(128) for c in range(128))
                continue
            for rr in range(128):
                i = qb * 128 + rr
                word = w[rr]
                on = [c for c in range(128) if (word[c >> 5] >> (c & 31)) & 1]
                if i >= n:
                    assert not on
                    continue
                cols = ci[rp[m * n + i]:rp[m * n + i + 1]]
                want = [c - kt * 128 for c in cols if c // 128 == kt]
                assert on == want
                covered.update((m * n + i, kt * 128 + c) for c in on)
    residual = set()
    for r in range(nm * n):
        row = rci[rrp[r]:rrp[r + 1]]
        assert np.all(np.diff(row) > 0)
        residual.update((r, int(c)) for c in row)
    full = {(r, int(c)) for r in range(nm * n) for c in ci[rp[r]:rp[r + 1]]}
    assert covered.isdisjoint(residual)
    assert covered | residual == full
    assert mask.residual_nnz == len(residual)


@pytest.mark.parametrize("cfg,kw,thr", [
    (1, dict(B=2, H=1, n=700), 0),          # variable window, ragged n, default threshold
    (3, dict(B=1, H=1, n=1000), 0),         # block + strided + global
    (4, dict(B=2, H=1, n=256), 0),          # dense
    (2, dict(B=2, H=1, n=1000), 600),       # random: some tiles selected, rest residual
    (1, dict(B=2, H=1, n=900), 9000),       # variable window (interval plan): window edges residual
    (0, dict(B=1, H=1, n=333), 2000),       # sliding window (interval plan), ragged n
])
def test_plan_partitions_the_csr(cfg, kw, thr):
    wl = workloads.make(cfg, **kw)
    rp, ci = oracle.mask_from_params(wl.mask)
    mp = wl.mask
    with build_mask(mp) if thr == 0 else _mask_with_thr(mp, thr) as m:
        _check_plan(m, rp, ci, mp.n, mp.num_masks, 512 if thr == 0 else thr)


def _mask_with_thr(mp, thr):
    return sp.spattn_create_csr_mask(
        mp.kind, mp.n, mp.num_masks, window=mp.window, block=mp.block, stride=mp.stride,
        n_global=mp.n_global, add_diagonal=mp.add_diagonal,
        half_widths=(torch.from_numpy(np.ascontiguousarray(mp.half_widths, np.int32).ravel()).cuda()
                     if mp.kind == "varwin" else None),
        in_row_ptr=(torch.from_numpy(mp.cand_row_ptr.astype(np.int32)).cuda() if mp.kind == "coo" else None),
        in_col_idx=(torch.from_numpy(mp.cand_cols.astype(np.int32)).cuda() if mp.kind == "coo" else None),
        tile_min_nnz=thr)


def _user_csr_mask(rp, ci, n, thr):
    return sp.spattn_create_csr_mask("csr", n, (rp.size - 1) // n,
                                     in_row_ptr=torch.from_numpy(rp.astype(np.int32)).cuda(),
                                     in_col_idx=torch.from_numpy(ci.astype(np.int32)).cuda(),
                                     tile_min_nnz=thr)


def _run_both(q, k, v, rp, ci, nm, n, d, thr, mask=None, bias=None, scale=None, what=""):
    scale = 1 / math.sqrt(d) if scale is None else scale
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, nm, scale,
                                          add_mask=None if mask is None else mask.raw,
                                          bias=None if bias is None else bias.raw)
    dq, dk, dv = torch_tensor(q), torch_tensor(k), torch_tensor(v)
    dm = torch_tensor(mask) if mask is not None else None
    db = torch_tensor(bias) if bias is not None else None
    res = {}
    for t in (thr, -1):                         # tensor-core plan, then gather only
        with _user_csr_mask(rp, ci, n, t) as m:
            if t != -1:
                assert m.n_tiles > 0
            out, lse = sp.spattn_fwd_mask(dq, dk, dv, m, add_mask=dm, bias=db, scale=scale)
            torch.cuda.synchronize()
            res[t] = (out, lse, m.n_tiles, m.n_mixed_rows)
        assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d),
                     lse_ref.reshape(-1), workloads.BF16, f"{what} thr={t}")
    assert sp.spattn_device_error() == 0
    return res


def _rand_csr(rng, n, nm, p, dense_blocks=()):
    rows, rp = [], [0]
    for r in range(nm * n):
        i = r % n
        on = rng.random(n) < p
        for (a, b) in dense_blocks:             # fully dense 128 x 128 areas
            if a * 128 <= i < (a + 1) * 128:
                on[b * 128:(b + 1) * 128] = True
        c = np.nonzero(on)[0].astype(np.int32)
        rows.append(c)
        rp.append(rp[-1] + c.size)
    return np.array(rp, np.int64), np.concatenate(rows).astype(np.int32)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_tensor_core_tiles_with_mixed_rows(d):
    """Dense tiles, partly filled tiles, and residual entries in the same rows."""
    rng = np.random.default_rng(d)
    B, H, n = 2, 2, 600
    rp, ci = _rand_csr(rng, n, 1, 0.03, dense_blocks=[(0, 0), (1, 1), (2, 3), (4, 4)])
    q, k, v = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), workloads.BF16) for _ in range(3))
    res = _run_both(q, k, v, rp, ci, 1, n, d, 1000, what=f"mixed d={d}")
    assert res[1000][3] > 0                     # there are mixed rows


@pytest.mark.parametrize("d", [32, 64, 128])
def test_tensor_core_all_entries_in_tiles(d):
    rng = np.random.default_rng(100 + d)
    B, H, n = 1, 3, 389
    rp, ci = _rand_csr(rng, n, 1, 0.25)
    q, k, v = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), workloads.BF16) for _ in range(3))
    res = _run_both(q, k, v, rp, ci, 1, n, d, 1, what=f"all-tiles d={d}")
    assert res[1][3] == 0


def test_tensor_core_with_mask_bias_and_per_batch_csr():
    rng = np.random.default_rng(7)
    B, H, n, d = 3, 2, 300, 64
    rp, ci = _rand_csr(rng, n, B, 0.2, dense_blocks=[(0, 0), (2, 2)])
    q, k, v = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), workloads.BF16) for _ in range(3))
    mask = workloads.make_tensor(np.where(rng.random((B, 1, 1, n)) < 0.1, -np.inf, 0.0), workloads.BF16)
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)), workloads.BF16)
    _run_both(q, k, v, rp, ci, B, n, d, 500, mask=mask, bias=bias, what="mask+bias")


def test_tensor_core_large_bias_and_empty_rows():
    rng = np.random.default_rng(8)
    B, H, n, d = 1, 2, 256, 64
    rp, ci = _rand_csr(rng, n, 1, 0.5)
    # empty some rows inside tensor-core blocks
    keep = np.ones(n, bool)
    keep[[3, 77, 200]] = False
    rows, rps = [], [0]
    for i in range(n):
        c = ci[rp[i]:rp[i + 1]] if keep[i] else np.zeros(0, np.int32)
        rows.append(c)
        rps.append(rps[-1] + c.size)
    rp, ci = np.array(rps, np.int64), np.concatenate(rows).astype(np.int32)
    q, k, v = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), workloads.BF16) for _ in range(3))
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)) * 1e4, workloads.F32)
    _run_both(q, k, v, rp, ci, 1, n, d, 1, bias=bias, what="bias 1e4 + empty rows")


def test_evoformer_workload_on_tensor_cores():
    wl = workloads.make(4, B=8, H=4, n=256)
    q, k, v, am, bias = device_inputs(wl)
    rp, ci = oracle.mask_from_params(wl.mask)
    out_ref, lse_ref = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, 1, wl.scale,
                                          add_mask=wl.add_mask.raw, bias=wl.bias.raw)
    with build_mask(wl.mask) as m:
        assert m.n_tiles == 4 and m.residual_nnz == 0
        out, lse = sp.spattn_fwd_mask(q, k, v, m, add_mask=am, bias=bias, scale=wl.scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref.reshape(-1, wl.d),
                 lse_ref.reshape(-1), wl.dtype, "evoformer")
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("thr", [0, 9000, 12000])
def test_variable_window_interval_plan_forward(thr):
    """Variable window masks use the interval plan; high thresholds leave the
    window edges to the gather kernel, so rows mix both paths."""
    wl = workloads.make(1, B=2, H=3, n=1100)
    q, k, v, _, _ = device_inputs(wl)
    rp, ci = oracle.mask_from_params(wl.mask)
    out_ref, lse_ref = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale)
    with _mask_with_thr(wl.mask, thr) as m:
        if thr == 9000:
            assert m.n_tiles > 0 and m.n_mixed_rows > 0
        out, lse = sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref.reshape(-1, wl.d),
                 lse_ref.reshape(-1), wl.dtype, f"varwin thr={thr}")
    assert sp.spattn_device_error() == 0


def _check_interval_plan(mask, rp, ci, n, nm, thr):
    """Vectorised plan check for masks whose rows are single runs [lo, hi):
    selected tiles, dense flags, every bit of every stored tile, and the
    residual CSR (the run minus the selected tiles, ascending)."""
    rows = nm * n
    ln = np.diff(rp)
    lo = np.where(ln > 0, ci[np.minimum(rp[:-1], max(ci.size - 1, 0))], 0).astype(np.int64)
    hi = lo + ln
    assert np.array_equal(ci, np.concatenate([np.arange(a, b) for a, b in zip(lo, hi)]))
    nqb = (n + 127) // 128
    r = np.arange(rows)
    blk = (r // n) * nqb + (r % n) // 128
    span = int(ln.max()) // 128 + 2
    cnt = np.zeros((nm * nqb, nqb), np.int64)
    parts = []
    for j in range(span):
        kt = lo // 128 + j
        ov = np.minimum(hi, kt * 128 + 128) - np.maximum(lo, kt * 128)
        ok = (ov > 0) & (kt < nqb)
        np.add.at(cnt, (blk[ok], kt[ok]), ov[ok])
        parts.append((kt, np.where(ok, ov, 0)))
    sel = cnt >= thr
    plan = mask.plan()
    assert mask.n_tiles == int(sel.sum())
    bto, info, bits, rrp, rci = (x.cpu().numpy() for x in plan)
    assert np.array_equal(np.diff(bto), sel.sum(axis=1))
    tb, tk = np.nonzero(sel)                      # tiles in (block, key tile) order
    assert np.array_equal(info & 0x7fffffff, tk)
    dense = info < 0
    assert np.array_equal(dense, cnt[tb, tk] == 128 * 128)
    # bits: row rr of tile t holds [lo, hi) clipped to the tile
    got = np.unpackbits(bits.view(np.uint8).reshape(-1, 128, 16), axis=2, bitorder="little").astype(bool)
    qrow = (tb % nqb)[:, None] * 128 + np.arange(128)[None, :]            # [T, 128]
    valid = qrow < n
    grow = np.where(valid, (tb // nqb)[:, None] * n + qrow, 0)
    a = np.clip(lo[grow] - tk[:, None] * 128, 0, 128)
    b = np.clip(hi[grow] - tk[:, None] * 128, 0, 128)
    c = np.arange(128)[None, None, :]
    want = (c >= a[:, :, None]) & (c < b[:, :, None]) & valid[:, :, None] & ~dense[:, None, None]
    assert np.array_equal(got, want)
    # residual: what the selected tiles leave of each run
    res = ln.copy()
    for kt, ov in parts:
        res -= np.where(sel[blk, np.minimum(kt, nqb - 1)], ov, 0)
    assert np.array_equal(np.diff(rrp), res)
    assert mask.residual_nnz == int(res.sum())
    rrow = np.repeat(r, res)
    assert np.all((rci >= lo[rrow]) & (rci < hi[rrow]))
    assert not sel[blk[rrow], rci // 128].any()
    same = rrow[1:] == rrow[:-1]
    assert np.all(np.diff(rci)[same] > 0)


@pytest.mark.parametrize("n,thr,asynchronous", [(32000, 9000, False), (33000, 9000, True), (33000, 0, True)])
def test_interval_plan_at_scale(n, thr, asynchronous):
    """Two variable-window masks of n = 32,000 or 33,000 rows each (500 or 516 query blocks):
    the tile selection, every tile bit and the residual CSR that the interval
    mask writes on request, and the forward on sampled rows."""
    wl = workloads.make(1, B=2, H=1, n=n)
    rp, ci = oracle.mask_from_params(wl.mask)
    with build_mask(wl.mask, tile_min_nnz=thr, asynchronous=asynchronous) as m:
        grp, gci = m.csr()
        assert np.array_equal(grp.cpu().numpy(), rp) and np.array_equal(gci.cpu().numpy(), ci)
        _check_interval_plan(m, rp, ci, n, wl.mask.num_masks, 512 if thr == 0 else thr)
        q, k, v, _, _ = device_inputs(wl)
        out, lse = sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
        torch.cuda.synchronize()
    rng = np.random.default_rng(n)
    rows = np.unique(np.concatenate([rng.integers(0, 2 * n, 400), [0, n - 1, n, 2 * n - 1]]))
    out_ref, lse_ref = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks,
                                          wl.scale, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    assert_close(to_f64(out.reshape(-1, wl.d)[idx]), to_f64(lse[idx]), out_ref, lse_ref, wl.dtype,
                 f"varwin n={n} thr={thr}")
    assert sp.spattn_device_error() == 0
