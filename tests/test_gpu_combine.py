"""hyb_combine on the GPU against the oracle's FP64 log-sum-exp merge."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S", [1, 2, 7, 64, 257])
def test_combine_matches_oracle(S):
    import torch
    from int8_paged_kv_hybrid_b200 import hyb_combine
    rng = np.random.default_rng(S)
    B, H, D = 3, 5, 128
    o = rng.standard_normal((B * H, S, D)).astype(np.float32)
    lse = (rng.standard_normal((B * H, S)) * 4).astype(np.float32)
    if S > 1:
        lse[0, 1] = -np.inf          # an empty split
        lse[1, :] = -np.inf          # an all-empty row
    ref, ref_lse = oracle.combine(o.astype(np.float64), lse.astype(np.float64))
    out = torch.empty((B, H, D), dtype=torch.float16, device="cuda")
    lo = torch.empty((B, H), dtype=torch.float32, device="cuda")
    hyb_combine(B, H, D, S, torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), out, lo)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().reshape(B * H, D)
    gl = lo.cpu().numpy().reshape(-1)
    assert np.abs(got - ref).max() <= 2e-3
    fin = np.isfinite(ref_lse)
    assert np.abs(gl[fin] - ref_lse[fin]).max() <= 1e-4
    assert np.all(np.isneginf(gl[~fin]))


def test_combine_rejects_bad_arguments():
    import torch
    from int8_paged_kv_hybrid_b200 import HybError, hyb_combine
    o = torch.zeros((1, 1, 2, 128), device="cuda")
    l = torch.zeros((1, 1, 2), device="cuda")
    out = torch.empty((1, 1, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(HybError):
        hyb_combine(1, 1, 64, 2, o, l, out)
    with pytest.raises(HybError):
        hyb_combine(1, 1, 128, 0, o, l, out)
