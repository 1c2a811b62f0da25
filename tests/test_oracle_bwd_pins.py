"""Pins of the oracle's gradients (oracle.masked_sdpa_bwd), independent of the
gradient code itself: central finite differences of the fp64 forward oracle
for every input element (q, k, v and the bias, broadcast dimensions included),
closed forms (one nonzero per row: out_i = v_j exactly, so dq = dk = 0 and dv
sums the upstream rows), the zero row sums of the score gradient, and rows
that contribute nothing (no nonzeros, or every score -inf)."""
import numpy as np
import pytest

import oracle


def _rand_csr(rng, n, nm, p, empty_rows=()):
    rp, cols = [0], []
    for r in range(nm * n):
        c = np.nonzero(rng.random(n) < p)[0]
        if r in empty_rows:
            c = c[:0]
        cols.append(c)
        rp.append(rp[-1] + c.size)
    return np.array(rp, np.int64), np.concatenate(cols).astype(np.int32)


def _loss(q, k, v, rp, ci, nm, scale, dout, mask, bias):
    out, _ = oracle.masked_sdpa(q, k, v, rp, ci, nm, scale, add_mask=mask, bias=bias)
    return float(np.sum(out * dout))


def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + h
        fp = f()
        x[idx] = old - h
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


@pytest.mark.parametrize("nm,bias_shape", [(1, (1, 2, 7, 7)), (2, (2, 1, 7, 7)), (1, (1, 1, 1, 7))])
def test_gradients_match_finite_differences(nm, bias_shape):
    rng = np.random.default_rng(3)
    B, H, n, d = 2, 2, 7, 3
    q, k, v, dout = (rng.standard_normal((B, H, n, d)) for _ in range(4))
    bias = rng.standard_normal(bias_shape)
    mask = np.where(rng.random((B, 1, 1, n)) < 0.2, -np.inf, 0.0)
    rp, ci = _rand_csr(rng, n, nm, 0.6, empty_rows=(3,))
    scale = 0.7
    dq, dk, dv, db = oracle.masked_sdpa_bwd(q, k, v, rp, ci, nm, scale, dout, add_mask=mask, bias=bias,
                                            want_dbias=True)
    f = lambda: _loss(q, k, v, rp, ci, nm, scale, dout, mask, bias)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("bias", bias, db)):
        fd = _fd(f, x)
        assert np.allclose(g, fd, atol=2e-7, rtol=1e-6), f"d{name}: max diff {np.abs(g - fd).max():.3g}"


def test_one_nonzero_per_row_closed_form():
    rng = np.random.default_rng(4)
    B, H, n, d = 1, 2, 9, 4
    q, k, v, dout = (rng.standard_normal((B, H, n, d)) for _ in range(4))
    cols = rng.integers(0, n, size=n).astype(np.int32)
    rp = np.arange(n + 1, dtype=np.int64)
    dq, dk, dv, _ = oracle.masked_sdpa_bwd(q, k, v, rp, cols, 1, 0.5, dout)
    assert np.all(dq == 0) and np.all(dk == 0)
    want = np.zeros_like(dv)
    for i in range(n):
        want[:, :, cols[i]] += dout[:, :, i]
    assert np.array_equal(dv, want)


def test_score_gradient_rows_sum_to_zero():
    rng = np.random.default_rng(5)
    B, H, n, d = 1, 1, 12, 5
    q, k, v, dout = (rng.standard_normal((B, H, n, d)) for _ in range(4))
    bias = rng.standard_normal((1, 1, n, n))
    rp, ci = _rand_csr(rng, n, 1, 0.5)
    _, _, _, db = oracle.masked_sdpa_bwd(q, k, v, rp, ci, 1, 0.3, dout, bias=bias, want_dbias=True)
    assert np.allclose(db[0, 0].sum(axis=1), 0.0, atol=1e-12)
    # entries outside the mask get no gradient
    off = np.ones((n, n), bool)
    for i in range(n):
        off[i, ci[rp[i]:rp[i + 1]]] = False
    assert np.all(db[0, 0][off] == 0)


def test_rows_that_contribute_nothing():
    rng = np.random.default_rng(6)
    B, H, n, d = 1, 1, 6, 3
    q, k, v, dout = (rng.standard_normal((B, H, n, d)) for _ in range(4))
    rp, ci = _rand_csr(rng, n, 1, 0.7, empty_rows=(2,))
    mask = np.zeros((1, 1, n, n))
    mask[0, 0, 4, :] = -np.inf                 # row 4: every score -inf
    dq, dk, dv, _ = oracle.masked_sdpa_bwd(q, k, v, rp, ci, 1, 1.0, dout, add_mask=mask)
    assert np.all(dq[0, 0, 2] == 0) and np.all(dq[0, 0, 4] == 0)
    # the same gradients as with rows 2 and 4 removed from the mask
    rp2, ci2 = [0], []
    for i in range(n):
        c = ci[rp[i]:rp[i + 1]] if i not in (2, 4) else ci[:0]
        ci2.append(c)
        rp2.append(rp2[-1] + c.size)
    g2 = oracle.masked_sdpa_bwd(q, k, v, np.array(rp2), np.concatenate(ci2), 1, 1.0, dout)
    for a, b in zip((dq, dk, dv), g2[:3]):
        assert np.array_equal(a, b)
