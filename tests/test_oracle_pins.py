"""Pins for the fp64 oracle (CPU only).

Each test ties the oracle to something other than itself: a library routine in
a special case where the method reduces to it (dense softmax attention through
scipy), closed forms, invariants of the softmax, brute force on tiny inputs,
and the worked mask printed in the AlphaFold2 flash-attention thread.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
import workloads
from conftest import load_golden


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _dense_csr(n, num_masks=1):
    row_ptr = np.arange(0, num_masks * n * n + 1, n, dtype=np.int64)
    col_idx = np.tile(np.arange(n, dtype=np.int32), num_masks * n)
    return row_ptr, col_idx


def _random_csr(rng, n, num_masks, p, keep_diag=True, empty_rows=()):
    rows, rp = [], [0]
    for r in range(num_masks * n):
        i = r % n
        on = rng.random(n) < p
        if keep_diag:
            on[i] = True
        if r in empty_rows:
            on[:] = False
        cols = np.nonzero(on)[0].astype(np.int32)
        rows.append(cols)
        rp.append(rp[-1] + cols.size)
    return np.array(rp, np.int64), (np.concatenate(rows) if rows else np.zeros(0, np.int32)).astype(np.int32)


def _dense_reference(q, k, v, scale, add=0.0):
    """softmax(scale * Q K^T + add) V and logsumexp, through scipy."""
    s = scale * np.einsum("bhid,bhjd->bhij", q, k) + add
    return softmax(s, axis=-1) @ v, logsumexp(s, axis=-1)


# ---------------------------------------------------------------- P1 dense equivalence
@pytest.mark.parametrize("with_mask,with_bias", [(False, False), (True, False), (False, True), (True, True)])
def test_all_ones_mask_is_dense_softmax_attention(with_mask, with_bias):
    rng = np.random.default_rng(1)
    B, H, n, d = 2, 3, 37, 16
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    scale = 1 / math.sqrt(d)
    mask = bias = None
    add = 0.0
    if with_mask:   # key padding, shape [B, 1, 1, n] (AlphaFold2 mask rule)
        mask = np.zeros((B, 1, 1, n))
        mask[0, 0, 0, 30:] = -np.inf
        mask[1, 0, 0, ::3] = -np.inf
        add = add + mask
    if with_bias:   # pair bias, shape [1, H, n, n] (AlphaFold2 bias rule)
        bias = _rand(rng, 1, H, n, n)
        add = add + bias
    rp, ci = _dense_csr(n)
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, 1, scale, mask, bias)
    ref_out, ref_lse = _dense_reference(q, k, v, scale, add)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-13)


def test_full_mask_and_bias_broadcast_shapes():
    """A full [B, H, n, n] mask and a [1, H, 1, n] bias broadcast like numpy."""
    rng = np.random.default_rng(2)
    B, H, n, d = 2, 2, 11, 8
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    # finite, nonzero additive values as well as -inf, so that a scale wrongly
    # applied to the mask changes the result
    mask = np.where(rng.random((B, H, n, n)) < 0.3, -np.inf, 2.0 * _rand(rng, B, H, n, n))
    for b in range(B):
        for h in range(H):
            for i in range(n):
                mask[b, h, i, i] = 0.5
    bias = _rand(rng, 1, H, 1, n)
    rp, ci = _dense_csr(n)
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.7, mask, bias)
    ref_out, ref_lse = _dense_reference(q, k, v, 0.7, mask + bias)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- P2 one nonzero per row
def test_one_nonzero_per_row_returns_that_v_row_exactly():
    rng = np.random.default_rng(3)
    B, H, n, d = 2, 2, 29, 12
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    perms = [rng.permutation(n) for _ in range(B)]
    rp = np.arange(B * n + 1, dtype=np.int64)
    ci = np.concatenate(perms).astype(np.int32)
    scale = 0.3
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, B, scale)
    for b in range(B):
        for h in range(H):
            assert np.array_equal(out[b, h], v[b, h, perms[b]])      # weight exp(0)/1 = 1
            s = [scale * math.fsum(q[b, h, i] * k[b, h, perms[b][i]]) for i in range(n)]
            np.testing.assert_allclose(lse[b, h], s, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- P3 row sums
def test_softmax_weights_are_a_distribution():
    rng = np.random.default_rng(4)
    B, H, n, d = 1, 2, 40, 8
    q, k, v = _rand(rng, B, H, n, d) * 3, _rand(rng, B, H, n, d) * 3, _rand(rng, B, H, n, d)
    rp, ci = _random_csr(rng, n, 1, 0.3)
    for flat in range(0, B * H * n, 7):
        w = oracle.row_weights(q, k, v, rp, ci, 1, 0.5, flat)
        assert np.all(w >= 0)
        assert abs(w.sum() - 1.0) < 1e-14
    # weights follow exp(score) ratios
    flat = 5
    w = oracle.row_weights(q, k, v, rp, ci, 1, 0.5, flat)
    cols = ci[rp[5]:rp[6]]
    s = np.array([0.5 * math.fsum(q[0, 0, 5] * k[0, 0, j]) for j in cols])
    np.testing.assert_allclose(w, softmax(s), rtol=1e-12)


# ---------------------------------------------------------------- P4 streaming = two-pass
@pytest.mark.parametrize("seed", [5, 6])
def test_running_max_sum_equals_two_pass(seed):
    rng = np.random.default_rng(seed)
    B, H, n, d = 2, 3, 53, 16
    q, k, v = _rand(rng, B, H, n, d) * 4, _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    rp, ci = _random_csr(rng, n, B, 0.25, keep_diag=False, empty_rows=(3, n + 7))
    mask = np.where(rng.random((B, 1, 1, n)) < 0.2, -np.inf, 0.0)
    bias = _rand(rng, 1, H, n, n) * 5
    a = oracle.masked_sdpa(q, k, v, rp, ci, B, 0.25, mask, bias, variant="two_pass")
    b = oracle.masked_sdpa(q, k, v, rp, ci, B, 0.25, mask, bias, variant="online")
    np.testing.assert_allclose(b[0], a[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b[1], a[1], rtol=1e-12, atol=1e-13)
    assert np.array_equal(np.isneginf(a[1]), np.isneginf(b[1]))
    # the empty rows: out 0, lse -inf
    assert np.all(a[0][0, :, 3] == 0) and np.all(np.isneginf(a[1][0, :, 3]))
    assert np.all(a[0][1, :, 7] == 0) and np.all(np.isneginf(a[1][1, :, 7]))


# ---------------------------------------------------------------- P5 -inf mask = drop
def test_minus_inf_mask_equals_dropping_the_entry():
    rng = np.random.default_rng(7)
    B, H, n, d = 2, 2, 31, 8
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    rp, ci = _random_csr(rng, n, 1, 0.4)
    drop = rng.random(ci.size) < 0.3
    mask = np.zeros((1, 1, n, n))
    kept_rows, kept_rp = [], [0]
    for i in range(n):
        cols = ci[rp[i]:rp[i + 1]]
        dr = drop[rp[i]:rp[i + 1]]
        mask[0, 0, i, cols[dr]] = -np.inf
        kept_rows.append(cols[~dr])
        kept_rp.append(kept_rp[-1] + int((~dr).sum()))
    rp2, ci2 = np.array(kept_rp, np.int64), np.concatenate(kept_rows).astype(np.int32)
    bias = _rand(rng, 1, H, n, n)
    for variant in ("two_pass", "online"):
        a = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.4, mask, bias, variant=variant)
        b = oracle.masked_sdpa(q, k, v, rp2, ci2, 1, 0.4, None, bias, variant=variant)
        assert np.array_equal(a[0], b[0])
        assert np.array_equal(a[1], b[1])


# ---------------------------------------------------------------- P6 shift invariance
def test_row_constant_shift_moves_lse_only():
    rng = np.random.default_rng(8)
    B, H, n, d = 1, 2, 33, 8
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    rp, ci = _random_csr(rng, n, 1, 0.3)
    c = _rand(rng, 1, 1, n, 1) * 10
    a = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.5)
    b = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.5, bias=c)
    np.testing.assert_allclose(b[0], a[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b[1], a[1] + c[0, 0, :, 0][None, None, :], rtol=1e-13, atol=1e-12)


# ---------------------------------------------------------------- P7 uniform scores
def test_zero_queries_give_the_mean_of_v_and_log_count():
    rng = np.random.default_rng(9)
    B, H, n, d = 2, 2, 27, 8
    q = np.zeros((B, H, n, d))
    k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    rp, ci = _random_csr(rng, n, B, 0.35)
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, B, 0.9)
    for b in range(B):
        for h in range(H):
            for i in range(n):
                cols = ci[rp[b * n + i]:rp[b * n + i + 1]]
                np.testing.assert_allclose(out[b, h, i], v[b, h, cols].mean(axis=0), rtol=1e-13, atol=1e-14)
                assert abs(lse[b, h, i] - math.log(cols.size)) < 1e-14


# ---------------------------------------------------------------- P8 constant V
def test_constant_v_rows_pass_through():
    rng = np.random.default_rng(10)
    B, H, n, d = 1, 3, 25, 8
    q, k = _rand(rng, B, H, n, d) * 2, _rand(rng, B, H, n, d) * 2
    c = _rand(rng, d)
    v = np.broadcast_to(c, (B, H, n, d)).copy()
    rp, ci = _random_csr(rng, n, 1, 0.5)
    out, _ = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.5, bias=_rand(rng, 1, H, n, n))
    np.testing.assert_allclose(out, np.broadcast_to(c, out.shape), rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------- P9 mask builder
@pytest.mark.parametrize("n,w", [(128, 16), (64, 0), (50, 49), (300, 7)])
def test_sliding_window_closed_form_count(n, w):
    rp, ci = oracle.mask_csr("sliding", n, window=w)
    w_eff = min(w, n - 1)
    assert rp[-1] == n * (2 * w_eff + 1) - w_eff * (w_eff + 1)
    if (n, w) == (128, 16):
        assert rp[-1] == 3952


def _as_dense(rp, ci, n, m=0):
    a = np.zeros((n, n), bool)
    for i in range(n):
        a[i, ci[rp[m * n + i]:rp[m * n + i + 1]]] = True
    return a


def _sorted_unique_rows(rp, ci):
    for r in range(rp.size - 1):
        row = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(row) > 0)


@pytest.mark.parametrize("kind,kw", [("sliding", dict(window=5)), ("bsg", dict(block=8, stride=16, n_global=3)),
                                     ("dense", {})])
def test_symmetric_patterns_give_symmetric_masks(kind, kw):
    n = 97
    rp, ci = oracle.mask_csr(kind, n, **kw)
    _sorted_unique_rows(rp, ci)
    a = _as_dense(rp, ci, n)
    assert np.array_equal(a, a.T)


def test_variable_window_rows_are_clipped_intervals():
    rng = np.random.default_rng(11)
    n, nm = 200, 3
    hw = rng.integers(0, 60, size=(nm, n)).astype(np.int32)
    rp, ci = oracle.mask_csr("varwin", n, nm, half_widths=hw)
    _sorted_unique_rows(rp, ci)
    for m in range(nm):
        for i in range(n):
            lo, hi = max(0, i - hw[m, i]), min(n - 1, i + hw[m, i])
            assert np.array_equal(ci[rp[m * n + i]:rp[m * n + i + 1]], np.arange(lo, hi + 1))


def test_block_strided_global_small_against_set_union():
    n, blk, st, ng = 150, 16, 24, 5
    rp, ci = oracle.mask_csr("bsg", n, block=blk, stride=st, n_global=ng)
    for i in range(n):
        want = set(range(ng)) | set(range((i // blk) * blk, min(n, (i // blk + 1) * blk)))
        want |= set(range(i % st, n, st))
        if i < ng:
            want = set(range(n))
        assert list(ci[rp[i]:rp[i + 1]]) == sorted(want)


@pytest.mark.slow
def test_block_strided_global_full_size_count():
    """Block 64, stride 128, 32 global tokens at n = 16384: inclusion-exclusion
    per row gives 32*16384 + sum over i >= 32 of
    (32 + 64 + 128 - 32*[i < 64] - [i mod 128 < 32] - 1) = 4,165,696."""
    n = 16384
    i = np.arange(32, n)
    count = 32 * n + int(np.sum(223 - 32 * (i < 64) - (i % 128 < 32)))
    assert count == 4_165_696
    rp, _ = oracle.mask_csr("bsg", n, block=64, stride=128, n_global=32)
    assert rp[-1] == count
    lens = np.diff(rp)
    assert lens.min() == 191 and lens.max() == n


def test_coo_candidates_merge_duplicates_and_add_diagonal():
    rng = np.random.default_rng(12)
    n, nm = 40, 2
    rp_c, cols = [0], []
    for r in range(nm * n):
        c = rng.integers(0, n, size=rng.integers(0, 12))
        c = np.concatenate([c, c[: c.size // 2]])          # duplicates
        cols.append(c)
        rp_c.append(rp_c[-1] + c.size)
    crp, cc = np.array(rp_c, np.int64), np.concatenate(cols).astype(np.int32)
    rp, ci = oracle.mask_csr("coo", n, nm, cand_row_ptr=crp, cand_cols=cc, add_diagonal=True)
    for r in range(nm * n):
        want = np.unique(np.concatenate([cc[crp[r]:crp[r + 1]], [r % n]]))
        assert np.array_equal(ci[rp[r]:rp[r + 1]], want)
    rp0, ci0 = oracle.mask_csr("coo", n, nm, cand_row_ptr=crp, cand_cols=cc, add_diagonal=False)
    for r in range(nm * n):
        assert np.array_equal(ci0[rp0[r]:rp0[r + 1]], np.unique(cc[crp[r]:crp[r + 1]]))


def test_random_workload_row_lengths():
    wl = workloads.make(2, B=2, H=1, n=512)
    rp, ci = oracle.mask_from_params(wl.mask)
    lens = np.diff(rp)
    want = np.diff(wl.mask.cand_row_ptr) + 1      # k_i distinct off-diagonal draws + the diagonal
    assert np.array_equal(lens, want)
    for r in range(0, 2 * 512, 37):
        assert (r % 512) in ci[rp[r]:rp[r + 1]]


# ---------------------------------------------------------------- P10 worked fixture
def test_worked_key_padding_mask_from_the_alphafold2_thread():
    g = load_golden("mas_mask.txt")
    rng = np.random.default_rng(13)
    for key in ("mas_mask", "mas_mask_T"):
        m = g[key]                       # [sequences, keys]
        B, n = m.shape
        H, d = 2, 4
        q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
        add = m[:, None, None, :]        # [B, 1, 1, n]: one key-padding row per sequence
        rp, ci = _dense_csr(n)
        out, lse = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.5, add_mask=add)
        # dropping the -inf keys from a per-sequence CSR gives the same bits
        rows, rps = [], [0]
        for b in range(B):
            keep = np.nonzero(np.isfinite(m[b]))[0].astype(np.int32)
            for _ in range(n):
                rows.append(keep)
                rps.append(rps[-1] + keep.size)
        out2, lse2 = oracle.masked_sdpa(q, k, v, np.array(rps, np.int64), np.concatenate(rows), B, 0.5)
        assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
        for b in range(B):
            if np.all(np.isneginf(m[b])):       # fully masked sequence: out 0, lse -inf
                assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            else:
                ref_out, ref_lse = _dense_reference(q[b:b + 1], k[b:b + 1], v[b:b + 1], 0.5, add[b:b + 1])
                np.testing.assert_allclose(out[b:b + 1], ref_out, rtol=1e-12, atol=1e-13)
                np.testing.assert_allclose(lse[b:b + 1], ref_lse, rtol=1e-12, atol=1e-13)
    assert g["mas_mask_T"].shape == (6, 2)
    assert np.array_equal(g["mas_mask_T"], g["mas_mask"].T)


# ---------------------------------------------------------------- P11 large bias
def test_large_magnitude_bias_stays_finite_and_exact():
    rng = np.random.default_rng(14)
    B, H, n, d = 1, 2, 24, 8
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    bias = _rand(rng, 1, H, n, n) * 1e4
    rp, ci = _dense_csr(n)
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, 1, 0.2, bias=bias)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    ref_out, ref_lse = _dense_reference(q, k, v, 0.2, bias)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)


# ---------------------------------------------------------------- input widening
def test_bf16_and_f32_inputs_are_read_exactly():
    rng = np.random.default_rng(15)
    B, H, n, d = 1, 1, 16, 8
    t = [workloads.make_tensor(_rand(rng, B, H, n, d), workloads.BF16) for _ in range(3)]
    rp, ci = _random_csr(rng, n, 1, 0.5)
    a = oracle.masked_sdpa(t[0].raw, t[1].raw, t[2].raw, rp, ci, 1, 0.5)
    b = oracle.masked_sdpa(t[0].f64(), t[1].f64(), t[2].f64(), rp, ci, 1, 0.5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # the bf16 bit patterns decode to the values numpy's float32 gives them
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0xFF80, 0x0001], np.uint16)
    np.testing.assert_array_equal(workloads.bf16_bits_to_f64(bits),
                                  [1.0, -1.0, 3.140625, -np.inf, 2.0 ** -133])


def test_row_subset_matches_full_run():
    rng = np.random.default_rng(16)
    B, H, n, d = 2, 2, 30, 8
    q, k, v = _rand(rng, B, H, n, d), _rand(rng, B, H, n, d), _rand(rng, B, H, n, d)
    rp, ci = _random_csr(rng, n, B, 0.3)
    full_out, full_lse = oracle.masked_sdpa(q, k, v, rp, ci, B, 0.5)
    rows = [0, 5, 31, 77, B * H * n - 1]
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, B, 0.5, rows=rows)
    np.testing.assert_array_equal(out, full_out.reshape(-1, d)[rows])
    np.testing.assert_array_equal(lse, full_lse.reshape(-1)[rows])
