"""The bounded-wait timeout path of the decode kernel, exercised safely: the
pipeline's wait limit is cut to a few SM cycles (hyb_set_wait_limit), so the
first wait for a stage's bulk copy gives up long before the copy lands.  The
kernel must record HYB_STATUS_TIMEOUT, let its copies in flight land (that
drain wait keeps the full ~1 s limit), and return with zero output and -inf
log-sum-exp for the rows it gave up on; with the default limit restored the
next call is correct again.  Nothing here faults or hangs: every copy is
valid and every wait is bounded."""
import numpy as np
import pytest

from harness import assert_decode_close, decode_both, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


# splits far longer than the 3-stage copy ring, so that most items are
# issued during the loop and waited for shortly after (one CTA per split);
# split_tokens -4: per-sequence splits on the persistent kernel, whose
# producer then hands out the remaining units with no items
@pytest.mark.parametrize("split", [64 * 40, 64 * 128, -4])
def test_wait_limit_times_out_then_recovers(split):
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    w = synth.custom_workload("timeout", [3000, 1200, 700], 32, 8, seed=17, schedule="chunk")
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    L = int(w.lens.max())
    q = torch.from_numpy(synth.query(w)).cuda()
    assert cache.status() == 0
    try:
        _lib.hyb_set_wait_limit(4)
        lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
        out = cache.decode(q, w.softmax_scale, L, split, lse=lse)
        torch.cuda.synchronize()
    finally:
        _lib.hyb_set_wait_limit(0)
    assert cache.status(clear=True) == _lib.HYB_STATUS_TIMEOUT
    o = out.float()
    assert torch.isfinite(o).all()
    # rows whose splits all gave up are exactly zero with lse -inf; a split
    # whose copies had already landed may still contribute to its row.  In
    # the one-CTA-per-split kernel some rows always give up whole; in the
    # persistent kernel (split < 0) the producer issues a unit's first copies
    # before its consumers reach it, so whether every unit of a row finds
    # data missing within the limit depends on timing
    gave_up = torch.isneginf(lse)
    if split > 0:
        assert gave_up.any()
    if gave_up.any():
        assert float(o[gave_up].abs().max()) == 0.0
    # the cache is untouched and the next call, with the default limit, is right
    got, lse2, ref, ref_lse = decode_both(w, cache, ora, split_tokens=split)
    assert_decode_close(w, got, lse2, ref, ref_lse, what="after timeout split=%d" % split)
    assert cache.status() == 0


@pytest.mark.parametrize("split", [64 * 40, -4])
def test_wait_limit_in_fused_step(split):
    """The fused step with the short limit: the status reports the timeout and
    every barrier of the fused append is still passed by all warps (the call
    returns); after restoring the limit the library keeps working."""
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    w = synth.custom_workload("timeout_step", [2000, 513], 32, 8, seed=19, schedule="chunk")
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    L = int(w.lens.max()) + 1
    rng = np.random.default_rng(3)
    n = torch.ones(w.batch, dtype=torch.int32, device="cuda")
    k = torch.from_numpy(rng.standard_normal((w.batch, 1, 8, 128)).astype(np.float16)).cuda()
    v = torch.from_numpy(rng.standard_normal((w.batch, 1, 8, 128)).astype(np.float16)).cuda()
    q = torch.from_numpy(synth.query(w)).cuda()
    try:
        _lib.hyb_set_wait_limit(4)
        cache.step(n, k, v, q, w.softmax_scale, L, split)
        torch.cuda.synchronize()
    finally:
        _lib.hyb_set_wait_limit(0)
    assert cache.status(clear=True) == _lib.HYB_STATUS_TIMEOUT
    out = cache.decode(q, w.softmax_scale, L, split)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert cache.status() == 0
