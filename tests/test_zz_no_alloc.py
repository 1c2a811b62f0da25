"""The allocation-free forward (spattn_fwd_noalloc) against spattn_fwd.

spattn_fwd_noalloc exists for callers that may not allocate device memory
while they run (a host program or plug-in whose memory manager owns the whole
device budget, or code that must not meet an allocation failure mid-work). It
keeps its scratch -- the list of rows above 1024 nonzeros and its counter -- in
a fixed array inside the library instead of taking it from the memory pool.

This file is collected last on purpose. It calls the entry point through the C
ABI twice in a row, on two different masks, so that the second call would see
the first call's leftovers if the shared array were not cleared, and compares
each result with the fp64 oracle and with spattn_fwd's under the tolerances of
the other tests. The library counts every allocation it makes
(spattn_alloc_count): the count must not move across the two calls, while the
same work through spattn_fwd does allocate. It also passes when run alone in a
fresh process (the first call does the per-device set-up).
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import workloads
from helpers import assert_close, to_f64, torch_tensor

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp


def _csr(rng, n, num_masks, p_short, long_rows):
    rows, rp = [], [0]
    for r in range(num_masks * n):
        p = 0.6 if (r % n) in long_rows else p_short
        on = rng.random(n) < p
        on[r % n] = True
        c = np.nonzero(on)[0].astype(np.int32)
        rows.append(c)
        rp.append(rp[-1] + c.size)
    return (torch.from_numpy(np.array(rp, np.int32)).cuda(),
            torch.from_numpy(np.concatenate(rows)).cuda())


def _call_noalloc(q, k, v, rp, ci, nm, mask, out, lse, scale):
    d = [sp.tensor_desc(x) for x in (q, k, v, out)]
    dm = sp.tensor_desc(mask) if mask is not None else None
    st = sp.LIB.spattn_fwd_noalloc(ctypes.byref(d[0]), ctypes.byref(d[1]), ctypes.byref(d[2]),
                                   rp.data_ptr(), ci.data_ptr(), nm, ci.numel(),
                                   ctypes.byref(dm) if dm is not None else None, None, scale,
                                   ctypes.byref(d[3]), lse.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert st == sp.SPATTN_OK, sp.spattn_last_error()


def test_noalloc_matches_oracle_and_spattn_fwd_on_two_calls_in_a_row():
    rng = np.random.default_rng(2024)
    cases = [
        # (B, H, n, d, dtype, rows made long (> 1024 nonzeros), num_masks)
        (2, 3, 2500, 64, workloads.BF16, set(range(0, 2500, 50)), 2),
        (1, 2, 1800, 128, workloads.F32, {3, 4, 5}, 1),
    ]
    prepared = []
    for B, H, n, d, dtype, long_rows, nm in cases:
        tq, tk, tv = (workloads.make_tensor(rng.standard_normal((B, H, n, d)), dtype) for _ in range(3))
        tm = workloads.make_tensor(np.where(rng.random((B, 1, 1, n)) < 0.05, -np.inf, 0.0), workloads.BF16)
        rp, ci = _csr(rng, n, nm, 0.02, long_rows)
        assert int((rp[1:] - rp[:-1] > 1024).sum()) == len(long_rows) * nm
        scale = 1.0 / math.sqrt(d)
        out_ref, lse_ref = oracle.masked_sdpa(tq.raw, tk.raw, tv.raw, rp.cpu().numpy().astype(np.int64),
                                              ci.cpu().numpy(), nm, scale, add_mask=tm.raw)
        q, k, v, mask = (torch_tensor(x) for x in (tq, tk, tv, tm))
        a0 = sp.spattn_alloc_count()
        fwd_out, fwd_lse = sp.spattn_fwd(q, k, v, rp, ci, nm, add_mask=mask, scale=scale)
        assert sp.spattn_alloc_count() > a0          # the pool path does allocate (scratch)
        out = torch.empty_like(q)
        lse = torch.empty(B * H * n, dtype=torch.float32, device="cuda")
        prepared.append((q, k, v, rp, ci, nm, mask, out, lse, scale, d, dtype, out_ref, lse_ref,
                         fwd_out, fwd_lse))
    torch.cuda.synchronize()
    a1 = sp.spattn_alloc_count()
    for (q, k, v, rp, ci, nm, mask, out, lse, scale, *_rest) in prepared:   # two calls in a row
        _call_noalloc(q, k, v, rp, ci, nm, mask, out, lse, scale)
    torch.cuda.synchronize()
    assert sp.spattn_alloc_count() == a1, "spattn_fwd_noalloc allocated memory"
    for (q, k, v, rp, ci, nm, mask, out, lse, scale, d, dtype, out_ref, lse_ref, fwd_out, fwd_lse) in prepared:
        assert_close(to_f64(out).reshape(-1, d), to_f64(lse), out_ref.reshape(-1, d), lse_ref.reshape(-1),
                     dtype, "noalloc vs oracle")
        assert_close(to_f64(out).reshape(-1, d), to_f64(lse), to_f64(fwd_out).reshape(-1, d),
                     to_f64(fwd_lse), dtype, "noalloc vs spattn_fwd")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, H, d = 2, 1, 32
    n = sp.NOALLOC_MAX_ROWS // 2 + 1            # num_masks * n = MAX + 1 with num_masks = 2
    q = torch.empty((B, H, n, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty(B * H * n, dtype=torch.float32, device="cuda")
    rp = torch.zeros(2 * n + 1, dtype=torch.int32, device="cuda")
    ci = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(sp.SpattnError) as e:
        sp.spattn_fwd_noalloc(q, q, q, rp, ci, 2, out=out, lse=lse)
    assert e.value.status == sp.SPATTN_ERR_UNSUPPORTED and "scratch" in str(e.value)
