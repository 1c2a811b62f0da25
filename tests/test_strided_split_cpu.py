"""The decomposition behind the strided tiles of block + strided + global masks,
checked with the oracle on the CPU (no GPU code involved).

The library moves a mask's strided entries (j = i mod S) into a second mask in
residue-permuted order -- row or key i at position perm(i) = (i mod S) n/S +
i div S -- runs attention over both parts (the permuted one over Q, K, V with
rows permuted) and merges each row's two results through their log-sum-exps.
This must equal attention over the whole mask: the softmax over a union of
disjoint entry sets, renormalised."""
import numpy as np
import pytest

import oracle
import workloads


def _perm(n, S):
    i = np.arange(n)
    return (i % S) * (n // S) + i // S


def _split(rp, ci, n, S):
    """Rows of the mask (one mask) split into strided entries, in permuted
    order, and the rest."""
    p = _perm(n, S)
    s_rows, r_rows = [[] for _ in range(n)], []
    for i in range(n):
        row = ci[rp[i]:rp[i + 1]]
        strided = row[row % S == i % S]
        s_rows[p[i]] = sorted(p[strided].tolist())
        r_rows.append(row[row % S != i % S])
    def csr(rows):
        ptr = np.zeros(n + 1, np.int64)
        ptr[1:] = np.cumsum([len(r) for r in rows])
        cols = np.concatenate([np.asarray(r, np.int32) for r in rows]) if ptr[-1] else np.zeros(0, np.int32)
        return ptr, cols
    return csr(s_rows), csr(r_rows)


@pytest.mark.parametrize("S,n", [(8, 64), (16, 128)])
def test_strided_split_and_lse_merge_equal_the_whole(S, n):
    rng = np.random.default_rng(S)
    B, H, d = 1, 2, 16
    mp = workloads.MaskParams("bsg", n, 1, block=8, stride=S, n_global=3)
    rp, ci = oracle.mask_from_params(mp)
    q, k, v = (rng.standard_normal((B, H, n, d)) for _ in range(3))
    scale = 1 / np.sqrt(d)
    out, lse = oracle.masked_sdpa(q, k, v, rp, ci, 1, scale)

    (srp, sci), (grp, gci) = _split(rp, ci, n, S)
    assert srp[-1] + grp[-1] == rp[-1]
    p = _perm(n, S)
    inv = np.argsort(p)
    qp, kp, vp = (np.empty_like(x) for x in (q, k, v))
    for x, xp in ((q, qp), (k, kp), (v, vp)):
        xp[:, :, p, :] = x  # row i at position perm(i)
    o2, l2 = oracle.masked_sdpa(qp, kp, vp, srp, sci, 1, scale)
    o1, l1 = oracle.masked_sdpa(q, k, v, grp, gci, 1, scale)
    o2, l2 = o2[:, :, p, :], l2[:, :, p]  # back to row order (row i was at perm(i))
    L = np.logaddexp(l1, l2)
    w1 = np.where(np.isfinite(L), np.exp(l1 - L), 0.0)
    w2 = np.where(np.isfinite(L), np.exp(l2 - L), 0.0)
    merged = o1 * w1[..., None] + o2 * w2[..., None]
    assert np.allclose(merged, out, atol=1e-12)
    assert np.allclose(L, lse, atol=1e-12)
    assert np.array_equal(inv[p], np.arange(n))  # perm is a permutation


def test_strided_entries_are_dense_blocks_in_permuted_order():
    """In permuted order the pure stride pattern (no blocks, no global tokens)
    is n/S x n/S dense blocks on the diagonal: what makes them tensor-core tiles."""
    n, S = 256, 16
    G = n // S
    mp = workloads.MaskParams("bsg", n, 1, block=0, stride=S, n_global=0)
    rp, ci = oracle.mask_from_params(mp)
    (srp, sci), (grp, gci) = _split(rp, ci, n, S)
    assert grp[-1] == 0
    for pi in range(n):
        r = pi // G
        assert np.array_equal(sci[srp[pi]:srp[pi + 1]], np.arange(r * G, (r + 1) * G))
