"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Bit-exact: the CSR the device builder writes (against the oracle's brute-force
masks) and the row -> lse mapping (-inf exactly where the oracle has it).
Floating point: bf16 inputs max-abs 2e-2 / mean-abs 2e-3 on out, fp32 inputs
1e-4; see helpers.TOL.
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from helpers import assert_close, build_mask, device_inputs, to_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp


# reduced shapes of the five workloads: several tiles, ragged tails, and (cfg 3)
# rows long enough for the block-per-row kernel
SMALL = {
    0: dict(),                                 # full size already small
    1: dict(B=2, H=2, n=1024),
    2: dict(B=2, H=2, n=1000),
    3: dict(B=1, H=2, n=2048),
    4: dict(B=6, H=3, n=256),
}


def _oracle_csr(mp):
    return oracle.mask_from_params(mp)


def _gpu_csr(mask):
    rp, ci = mask.csr()
    torch.cuda.synchronize()
    return rp.cpu().numpy().astype(np.int64), ci.cpu().numpy()


def _run_oracle(wl, rp, ci, rows=None, threads=0):
    return oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale,
                              add_mask=None if wl.add_mask is None else wl.add_mask.raw,
                              bias=None if wl.bias is None else wl.bias.raw, rows=rows,
                              threads=threads)


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_mask_builder_matches_brute_force(cfg):
    wl = workloads.make(cfg, **SMALL[cfg])
    rp_ref, ci_ref = _oracle_csr(wl.mask)
    with build_mask(wl.mask) as m:
        rp, ci = _gpu_csr(m)
        assert m.nnz == rp_ref[-1]
        assert m.n_long == int(np.sum(np.diff(rp_ref) > 1024))
        # the schedule's long rows are exactly the rows above 1024 nonzeros
        assert np.array_equal(m.long_rows().cpu().numpy(), np.nonzero(np.diff(rp_ref) > 1024)[0])
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(ci, ci_ref)


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_fused_forward_matches_oracle(cfg):
    wl = workloads.make(cfg, **SMALL[cfg])
    q, k, v, am, bias = device_inputs(wl)
    rp_ref, ci_ref = _oracle_csr(wl.mask)
    out_ref, lse_ref = _run_oracle(wl, rp_ref, ci_ref)
    with build_mask(wl.mask) as m:
        out, lse = sp.spattn_fwd_mask(q, k, v, m, add_mask=am, bias=bias, scale=wl.scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref.reshape(-1, wl.d),
                 lse_ref.reshape(-1), wl.dtype, f"cfg{cfg} mask path")
    # the raw-CSR entry point on the same CSR, with each row's columns shuffled
    rng = np.random.default_rng(cfg)
    ci_shuf = ci_ref.copy()
    for r in range(rp_ref.size - 1):
        seg = ci_shuf[rp_ref[r]:rp_ref[r + 1]]
        rng.shuffle(seg)
    out2, lse2 = sp.spattn_fwd(q, k, v, torch.from_numpy(rp_ref.astype(np.int32)).cuda(),
                               torch.from_numpy(ci_shuf).cuda(), wl.mask.num_masks,
                               add_mask=am, bias=bias, scale=wl.scale)
    torch.cuda.synchronize()
    assert_close(to_f64(out2).reshape(-1, wl.d), to_f64(lse2), out_ref.reshape(-1, wl.d),
                 lse_ref.reshape(-1), wl.dtype, f"cfg{cfg} raw path")
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("n", [1100, 2048])
def test_split_query_block_d128(n):
    """Query block 0 of the block + strided + global mask lists every key tile
    (its global rows attend to all keys); the d = 128 tile kernel splits such a
    block into chunks of eight tiles, one thread block each, and merges their
    partial states (n = 1100: chunks of 8 and 1 tiles)."""
    wl = workloads.make(3, B=1, H=2, n=n)
    q, k, v, am, bias = device_inputs(wl)
    rp_ref, ci_ref = _oracle_csr(wl.mask)
    out_ref, lse_ref = _run_oracle(wl, rp_ref, ci_ref)
    with build_mask(wl.mask) as m:
        out, lse = sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref.reshape(-1, wl.d),
                 lse_ref.reshape(-1), wl.dtype, f"split block n={n}")
    assert sp.spattn_device_error() == 0


@pytest.mark.parametrize("stride,n", [(64, 8192), (128, 2048)])
def test_strided_entries_as_permuted_tiles(stride, n):
    """Block + strided + global masks keep their strided entries as a residue-
    permuted mask of dense tiles, run as a second tile pass and merged by
    log-sum-exp. With n / stride a multiple of 128 (stride 64, n = 8192) the
    d = 128 tile kernel reads the permuted rows in place through five-dimensional
    maps; otherwise (stride 128, n = 2048) they are copied in permuted order."""
    import dataclasses
    wl = workloads.make(3, B=1, H=2, n=n)
    wl = dataclasses.replace(wl, mask=workloads.MaskParams("bsg", n, 1, block=64, stride=stride, n_global=32))
    q, k, v, am, bias = device_inputs(wl)
    rp_ref, ci_ref = _oracle_csr(wl.mask)
    out_ref, lse_ref = _run_oracle(wl, rp_ref, ci_ref)
    with build_mask(wl.mask) as m:
        out, lse = sp.spattn_fwd_mask(q, k, v, m, scale=wl.scale)
        torch.cuda.synchronize()
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), out_ref.reshape(-1, wl.d),
                 lse_ref.reshape(-1), wl.dtype, f"strided tiles S={stride} n={n}")
    assert sp.spattn_device_error() == 0


# ------------------------------------------------------------------ edge cases
def _rand_csr(rng, n, num_masks, p, empty=(), dup=False):
    rows, rp = [], [0]
    for r in range(num_masks * n):
        on = rng.random(n) < p
        on[r % n] = True
        if r in empty:
            on[:] = False
        c = np.nonzero(on)[0].astype(np.int32)
        if dup and c.size:
            c = np.concatenate([c, c[: max(1, c.size // 3)]])
        rows.append(c)
        rp.append(rp[-1] + c.size)
    return np.array(rp, np.int64), np.concatenate(rows).astype(np.int32)


def _inputs(rng, B, H, n, d, dtype, std=1.0):
    return [workloads.make_tensor(rng.standard_normal((B, H, n, d)) * std, dtype) for _ in range(3)]


def _dev(t):
    from helpers import torch_tensor
    return torch_tensor(t)


def _check_raw(B, H, n, d, dtype, rp, ci, nm, mask=None, bias=None, scale=None, seed=0,
               tensors=None, what=""):
    rng = np.random.default_rng(seed)
    q, k, v = tensors or _inputs(rng, B, H, n, d, dtype)
    scale = 1 / math.sqrt(d) if scale is None else scale
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, nm, scale,
                                          add_mask=None if mask is None else mask.raw,
                                          bias=None if bias is None else bias.raw)
    out, lse = sp.spattn_fwd(_dev(q), _dev(k), _dev(v), torch.from_numpy(rp.astype(np.int32)).cuda(),
                             torch.from_numpy(ci).cuda(), nm,
                             add_mask=None if mask is None else _dev(mask),
                             bias=None if bias is None else _dev(bias), scale=scale)
    torch.cuda.synchronize()
    return assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d),
                        lse_ref.reshape(-1), dtype, what)


@pytest.mark.parametrize("dtype", [workloads.BF16, workloads.F32])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("n", [127, 255, 257])
def test_odd_lengths_with_mask_and_bias(dtype, d, n):
    """Odd sequence lengths with mask and bias (the AlphaFold2 thread reports a
    misaligned-address failure there)."""
    rng = np.random.default_rng(n * d)
    B, H = 2, 2
    rp, ci = _rand_csr(rng, n, B, 0.2)
    mask = workloads.make_tensor(np.where(rng.random((B, 1, 1, n)) < 0.1, -np.inf, 0.0), workloads.BF16)
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)), dtype)
    _check_raw(B, H, n, d, dtype, rp, ci, B, mask, bias, seed=n + d, what=f"n={n} d={d}")


@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("layout", ["row_mask", "bias_only", "pad_mask_and_bias", "row_mask_and_bias",
                                    "f32_bias"])
def test_tile_addend_layouts(d, layout):
    """The tensor-core kernel takes one addend that varies by row from registers
    fetched a tile ahead (bf16, unit column stride, aligned rows) and loads the
    other when it is used; every combination must give the same result."""
    rng = np.random.default_rng(7 + d)
    B, H, n = 2, 3, 256
    rp, ci = _rand_csr(rng, n, 1, 0.6)
    row_mask = workloads.make_tensor(np.where(rng.random((B, 1, n, n)) < 0.1, -np.inf,
                                              rng.standard_normal((B, 1, n, n))), workloads.BF16)
    pad_mask = workloads.make_tensor(np.where(rng.random((B, 1, 1, n)) < 0.2, -np.inf, 0.0), workloads.BF16)
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)), workloads.BF16)
    bias32 = workloads.make_tensor(rng.standard_normal((1, H, n, n)), workloads.F32)
    mask, b = {"row_mask": (row_mask, None), "bias_only": (None, bias),
               "pad_mask_and_bias": (pad_mask, bias), "row_mask_and_bias": (row_mask, bias),
               "f32_bias": (pad_mask, bias32)}[layout]
    _check_raw(B, H, n, d, workloads.BF16, rp, ci, 1, mask, b, seed=d, what=f"{layout} d={d}")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.3])
def test_tile_scale_sign(d, scale):
    """The tensor-core kernels keep raw scores until the exponent when the scale
    is positive; a negative or zero scale takes the scaled-scores path. Both must
    follow the definition (a zero scale gives every listed entry the same weight)."""
    rng = np.random.default_rng(11 + d)
    B, H, n = 1, 2, 256
    rp, ci = _rand_csr(rng, n, 1, 0.5)
    _check_raw(B, H, n, d, workloads.BF16, rp, ci, 1, scale=scale, seed=d, what=f"scale={scale} d={d}")


def test_empty_and_fully_masked_rows():
    rng = np.random.default_rng(1)
    B, H, n, d = 2, 2, 96, 64
    rp, ci = _rand_csr(rng, n, 1, 0.1, empty=(0, 5, 95))
    m = np.zeros((1, 1, n, n))
    for i in (7, 8, 50):          # every entry of these rows -inf
        m[0, 0, i, :] = -np.inf
    mask = workloads.make_tensor(m, workloads.F32)
    _check_raw(B, H, n, d, workloads.BF16, rp, ci, 1, mask, what="empty rows")


def test_worked_key_padding_fixture_on_gpu():
    from conftest import load_golden
    g = load_golden("mas_mask.txt")
    for key in ("mas_mask", "mas_mask_T"):
        m = g[key]
        B, n = m.shape
        # the fixture's sequences are short; place them at the start of n = 32 keys
        N = 32
        full = np.full((B, 1, 1, N), -np.inf)
        full[:, 0, 0, :n] = m
        rp = np.arange(0, N * N + 1, N, dtype=np.int64)
        ci = np.tile(np.arange(N, dtype=np.int32), N)
        _check_raw(B, 2, N, 32, workloads.F32, rp, ci, 1,
                   workloads.make_tensor(full, workloads.F32), what=key)


def test_large_magnitude_bias():
    rng = np.random.default_rng(2)
    B, H, n, d = 1, 4, 200, 64
    rp, ci = _rand_csr(rng, n, 1, 0.3)
    bias = workloads.make_tensor(rng.standard_normal((1, H, n, n)) * 1e4, workloads.F32)
    _check_raw(B, H, n, d, workloads.BF16, rp, ci, 1, bias=bias, what="bias 1e4")


def test_duplicate_columns_count_per_occurrence():
    rng = np.random.default_rng(3)
    B, H, n, d = 2, 2, 150, 32
    rp, ci = _rand_csr(rng, n, B, 0.2, dup=True)
    _check_raw(B, H, n, d, workloads.F32, rp, ci, B, what="duplicates")


@pytest.mark.parametrize("shape", [(2, 1, 1, 300), (1, 3, 300, 300), (2, 3, 300, 300), (1, 1, 300, 1)])
def test_mask_broadcast_shapes(shape):
    rng = np.random.default_rng(4)
    B, H, n, d = 2, 3, 300, 64
    rp, ci = _rand_csr(rng, n, 1, 0.05)
    vals = np.where(rng.random(shape) < 0.2, -np.inf, rng.standard_normal(shape))
    mask = workloads.make_tensor(vals, workloads.BF16)
    _check_raw(B, H, n, d, workloads.BF16, rp, ci, 1, mask, what=str(shape))
    _check_raw(B, H, n, d, workloads.BF16, rp, ci, 1, bias=mask, what="bias " + str(shape))


@pytest.mark.parametrize("dtype,d", [(workloads.BF16, 64), (workloads.F32, 128), (workloads.BF16, 128)])
def test_long_rows_take_the_block_kernel(dtype, d):
    """Rows above 1024 nonzeros (dense n = 3000, plus a few short rows)."""
    rng = np.random.default_rng(5)
    B, H, n = 1, 3, 3000
    rp, ci = _rand_csr(rng, n, 1, 0.35)         # ~1050 per row: mixed long and short
    lens = np.diff(rp)
    assert (lens > 1024).any() and (lens <= 1024).any()
    _check_raw(B, H, n, d, dtype, rp, ci, 1, what="long rows")


def test_one_nonzero_per_row_is_exact():
    rng = np.random.default_rng(6)
    B, H, n, d = 2, 2, 500, 64
    perm = np.concatenate([rng.permutation(n) for _ in range(B)]).astype(np.int32)
    rp = np.arange(B * n + 1, dtype=np.int64)
    q, k, v = _inputs(rng, B, H, n, d, workloads.BF16)
    out, _ = sp.spattn_fwd(_dev(q), _dev(k), _dev(v), torch.from_numpy(rp.astype(np.int32)).cuda(),
                           torch.from_numpy(perm).cuda(), B)
    torch.cuda.synchronize()
    got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    for b in range(B):
        assert np.array_equal(got[b], v.raw[b][:, perm[b * n:(b + 1) * n]])


def test_strided_views():
    """q/k/v/out as non-contiguous views ([B, n, H, d] storage seen as [B, H, n, d])."""
    rng = np.random.default_rng(7)
    B, H, n, d = 2, 4, 200, 64
    rp, ci = _rand_csr(rng, n, 1, 0.1)
    q, k, v = _inputs(rng, B, H, n, d, workloads.BF16)
    out_ref, lse_ref = oracle.masked_sdpa(q.raw, k.raw, v.raw, rp, ci, 1, 0.125)

    def view(t):
        x = _dev(t).permute(0, 2, 1, 3).contiguous()     # [B, n, H, d] storage
        return x.permute(0, 2, 1, 3)                      # [B, H, n, d] view
    qv, kv, vv = view(q), view(k), view(v)
    out = torch.empty((B, n, H, d), dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)
    assert not qv.is_contiguous()
    o, lse = sp.spattn_fwd(qv, kv, vv, torch.from_numpy(rp.astype(np.int32)).cuda(),
                           torch.from_numpy(ci).cuda(), 1, scale=0.125, out=out)
    torch.cuda.synchronize()
    assert_close(to_f64(o).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d),
                 lse_ref.reshape(-1), workloads.BF16, "strided")


def test_bad_column_is_skipped_and_flagged():
    rng = np.random.default_rng(8)
    B, H, n, d = 1, 2, 64, 32
    rp, ci = _rand_csr(rng, n, 1, 0.2)
    bad = ci.copy()
    bad[3] = n + 5            # out of range: skipped by the kernel's bounds check
    bad[10] = -2
    q, k, v = _inputs(rng, B, H, n, d, workloads.F32)
    sp.spattn_device_error()  # clear
    sp.spattn_fwd(_dev(q), _dev(k), _dev(v), torch.from_numpy(rp.astype(np.int32)).cuda(),
                  torch.from_numpy(bad).cuda(), 1)
    assert sp.spattn_device_error() & 1
    assert sp.spattn_device_error() == 0     # cleared


def test_deterministic():
    wl = workloads.make(2, B=2, H=2, n=800)
    q, k, v, _, _ = device_inputs(wl)
    with build_mask(wl.mask) as m:
        a = sp.spattn_fwd_mask(q, k, v, m)
        b = sp.spattn_fwd_mask(q, k, v, m)
        torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bad_user_csr_is_rejected():
    n = 16
    rp = torch.tensor(list(range(0, 2 * n + 1, 2)), dtype=torch.int32, device="cuda")
    ci = torch.tensor([1, 0] * n, dtype=torch.int32, device="cuda")      # unsorted rows
    with pytest.raises(sp.SpattnError) as e:
        sp.spattn_create_csr_mask("csr", n, in_row_ptr=rp, in_col_idx=ci)
    assert e.value.status == sp.SPATTN_ERR_BAD_CSR
    ci2 = torch.tensor([0, n] * n, dtype=torch.int32, device="cuda")     # column out of range
    with pytest.raises(sp.SpattnError):
        sp.spattn_create_csr_mask("csr", n, in_row_ptr=rp, in_col_idx=ci2)
    ok = torch.tensor([0, 1] * n, dtype=torch.int32, device="cuda")
    with sp.spattn_create_csr_mask("csr", n, in_row_ptr=rp, in_col_idx=ok) as m:
        r2, c2 = m.csr()
        assert torch.equal(r2, rp) and torch.equal(c2, ok)


def test_coo_builder_duplicates_and_long_rows():
    """COO candidates with repeats, rows above the warp sort limit (n-bit map path)."""
    rng = np.random.default_rng(9)
    n, nm = 3000, 2
    rps, cols = [0], []
    for r in range(nm * n):
        cnt = 1500 if r % 97 == 0 else int(rng.integers(0, 40))
        c = rng.integers(0, n, size=cnt)
        cols.append(c)
        rps.append(rps[-1] + c.size)
    mp = workloads.MaskParams("coo", n, nm, cand_row_ptr=np.array(rps, np.int64),
                              cand_cols=np.concatenate(cols).astype(np.int32), add_diagonal=True)
    rp_ref, ci_ref = oracle.mask_from_params(mp)
    with build_mask(mp) as m:
        rp, ci = _gpu_csr(m)
    assert np.array_equal(rp, rp_ref) and np.array_equal(ci, ci_ref)


@pytest.mark.parametrize("kind,kw", [("sliding", dict(window=0)), ("sliding", dict(window=5000)),
                                     ("bsg", dict(block=0, stride=7, n_global=0)),
                                     ("bsg", dict(block=33, stride=0, n_global=40)),
                                     ("dense", {})])
def test_builder_parameter_corners(kind, kw):
    n = 1500
    mp = workloads.MaskParams(kind, n, 1, **kw)
    rp_ref, ci_ref = oracle.mask_from_params(mp)
    with build_mask(mp) as m:
        rp, ci = _gpu_csr(m)
    assert np.array_equal(rp, rp_ref) and np.array_equal(ci, ci_ref)


@pytest.mark.parametrize("n,nm", [(16, 1), (32768, 2), (35000, 2)])
def test_user_csr_both_build_paths(n, nm):
    """User CSR through both phase-1 paths (one launch up to 65,536 rows, the
    multi-launch scan above): the copy is exact, long rows are listed, and a
    broken row_ptr or an unsorted row is still rejected."""
    rng = np.random.default_rng(n)
    lens = rng.integers(0, 12, size=nm * n)
    lens[:: max(1, (nm * n) // 3)] = min(n, 1100)            # a few long rows
    rows = [np.sort(rng.choice(n, size=int(c), replace=False)) for c in lens]
    rp = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    drp, dci = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
    with sp.spattn_create_csr_mask("csr", n, nm, in_row_ptr=drp, in_col_idx=dci) as m:
        r2, c2 = m.csr()
        assert m.nnz == int(rp[-1])
        assert m.n_long == int(np.sum(lens > 1024))
        assert np.array_equal(m.long_rows().cpu().numpy(), np.nonzero(lens > 1024)[0])
        assert torch.equal(r2, drp) and torch.equal(c2, dci)
    bad = rp.copy()
    bad[nm * n // 2] = bad[nm * n // 2 + 1] + 1                 # decreasing row_ptr
    with pytest.raises(sp.SpattnError) as e:
        sp.spattn_create_csr_mask("csr", n, nm, in_row_ptr=torch.from_numpy(bad).cuda(), in_col_idx=dci)
    assert e.value.status == sp.SPATTN_ERR_BAD_CSR
    j = int(np.argmax(lens >= 2))
    uns = ci.copy()
    uns[rp[j]], uns[rp[j] + 1] = uns[rp[j] + 1], uns[rp[j]]     # swap two columns of a row
    with pytest.raises(sp.SpattnError) as e:
        sp.spattn_create_csr_mask("csr", n, nm, in_row_ptr=drp, in_col_idx=torch.from_numpy(uns).cuda())
    assert e.value.status == sp.SPATTN_ERR_BAD_CSR
