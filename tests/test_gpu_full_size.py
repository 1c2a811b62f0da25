"""The five workloads at full size, in the launch configuration the benchmark
times (mask built on the device, then the mask-handle forward): the whole CSR is
compared bit-exactly with the oracle's brute-force mask, and the outputs of
every row of two (b, h) heads (the first and the last), plus a sample of other
rows (random rows, the first and last rows of every (b, h), the rows of the
block-per-row kernel), with the oracle's values for those rows."""
import numpy as np
import pytest

import oracle
import workloads
from helpers import assert_close, build_mask, device_inputs, to_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp


def _sample_rows(wl, rp, count, seed):
    rng = np.random.default_rng(seed)
    B, H, n = wl.B, wl.H, wl.n
    total = B * H * n
    rows = set(rng.integers(0, total, size=count).tolist())
    for bh in (0, B * H - 1):                      # two whole heads
        rows.update(range(bh * n, (bh + 1) * n))
    for bh in range(0, B * H, max(1, (B * H) // 8)):
        rows.update([bh * n, bh * n + n - 1])
    lens = np.diff(rp)
    long_rows = np.nonzero(lens > 1024)[0]
    for r in long_rows[:4]:
        m, i = divmod(int(r), n)
        b = m if wl.mask.num_masks > 1 else 0
        for h in (0, H - 1):
            rows.add((b * H + h) * n + i)
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_full_size_workload(cfg):
    wl = workloads.make(cfg)
    rp_ref, ci_ref = oracle.mask_from_params(wl.mask)
    q, k, v, am, bias = device_inputs(wl)
    with build_mask(wl.mask) as m:
        rp, ci = m.csr()
        out, lse = sp.spattn_fwd_mask(q, k, v, m, add_mask=am, bias=bias, scale=wl.scale)
        torch.cuda.synchronize()
        assert m.nnz == rp_ref[-1]
        assert m.n_long == int(np.sum(np.diff(rp_ref) > 1024))
    assert np.array_equal(rp.cpu().numpy(), rp_ref)
    assert np.array_equal(ci.cpu().numpy(), ci_ref)
    rows = _sample_rows(wl, rp_ref, 600, cfg)
    out_ref, lse_ref = oracle.masked_sdpa(
        wl.q.raw, wl.k.raw, wl.v.raw, rp_ref, ci_ref, wl.mask.num_masks, wl.scale,
        add_mask=None if wl.add_mask is None else wl.add_mask.raw,
        bias=None if wl.bias is None else wl.bias.raw, rows=rows)
    got = to_f64(out.reshape(-1, wl.d)[torch.from_numpy(rows).cuda()])
    got_lse = to_f64(lse[torch.from_numpy(rows).cuda()])
    assert_close(got, got_lse, out_ref, lse_ref, wl.dtype, f"cfg{cfg} full size")
    # properties that hold for every row: finite output, finite lse (every row
    # of these masks keeps at least one finite score)
    assert torch.isfinite(out).all()
    assert torch.isfinite(lse).all()
    assert sp.spattn_device_error() == 0
