"""The unfused three-stage forward (spattn_fwd_unfused: SDDMM -> softmax -> SpMM
with an nnz-sized score buffer) against the oracle, on the same inputs and
tolerances as the fused path (helpers.TOL)."""
import numpy as np
import pytest

import oracle
import workloads
from helpers import assert_close, device_inputs, to_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_mask_scaled_b200 as sp


@pytest.mark.parametrize("cfg,kw", [(0, dict()), (1, dict(B=2, H=2, n=700)), (2, dict(B=2, H=2, n=900)),
                                    (3, dict(B=1, H=2, n=1100)), (4, dict(B=3, H=2, n=256))])
def test_unfused_matches_oracle(cfg, kw):
    wl = workloads.make(cfg, **kw)
    rp, ci = oracle.mask_from_params(wl.mask)
    q, k, v, am, bias = device_inputs(wl)
    drp = torch.from_numpy(rp.astype(np.int32)).cuda()
    dci = torch.from_numpy(ci).cuda()
    out, lse = sp.spattn_fwd_unfused(q, k, v, drp, dci, wl.mask.num_masks, add_mask=am, bias=bias,
                                     scale=wl.scale)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale,
                                          add_mask=None if wl.add_mask is None else wl.add_mask.raw,
                                          bias=None if wl.bias is None else wl.bias.raw)
    assert_close(to_f64(out).reshape(-1, wl.d), to_f64(lse), ref_out.reshape(-1, wl.d), ref_lse.reshape(-1),
                 wl.dtype, f"unfused cfg{cfg}")
    assert sp.spattn_device_error() == 0
