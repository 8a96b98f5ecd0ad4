"""hyb_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory when they run it (a fixed budget handed out at start-up, an
allocator owned by the host application, a decode loop where an allocation
could block or fail).  Its scratch is a static buffer inside the library, so
it must give the same result as hyb_decode_attn with a caller workspace,
call after call (the buffer keeps the previous call's contents).

This file is collected last on purpose; it builds its own inputs so that it
also passes alone in a fresh process."""
import numpy as np
import pytest

from harness import MAX_ABS, assert_decode_close, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    # 64-token splits: ~30 splits per long sequence, more than a cluster holds,
    # so the split merge goes through the scratch buffer
    w = synth.custom_workload("noalloc", [2000, 900, 33, 0, 1500], 32, 8, seed=21, max_step=64)
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    L = int(w.lens.max())
    split = 64
    need = _lib.hyb_decode_workspace_bytes(cache.desc, L, split)
    assert 0 < need <= _lib.hyb_noalloc_scratch_limit()
    q = torch.from_numpy(synth.query(w)).cuda()
    ref = cache.decode(q, w.softmax_scale, L, split).float()
    for call in range(2):
        out = torch.empty_like(ref, dtype=torch.float16)
        lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
        _lib.hyb_decode_attn_noalloc(cache.desc, q, w.softmax_scale, L, split, out, lse)
        torch.cuda.synchronize()
        err = float((out.float() - ref).abs().max())
        assert err <= MAX_ABS, (call, err)
        assert torch.isfinite(lse[:3]).all() and torch.isneginf(lse[3]).all()
    assert cache.status() == 0


def test_noalloc_matches_oracle_and_alternates_merge_paths():
    """Against the FP64 oracle within the accuracy bar, and call after call
    with plans that alternate between a split merge inside a thread-block
    cluster (the scratch is not used) and merges through the scratch buffer
    (one level, and two levels above 16 splits), so that each call finds the
    buffer as the previous, different call left it."""
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    w = synth.custom_workload("noalloc_ora", [3100, 700, 1, 2300], 32, 8, seed=8, max_step=64)
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    L = int(w.lens.max())
    qn = synth.query(w)
    q = torch.from_numpy(qn).cuda()
    ref, ref_lse = ora.decode(qn, w.softmax_scale)
    uses = {}
    for split in (0, 64, 1024, 128, 0, 64, 3072, 64):
        need = _lib.hyb_decode_workspace_bytes(cache.desc, L, split)
        assert need <= _lib.hyb_noalloc_scratch_limit()
        _, ns = _lib.hyb_decode_plan(cache.desc, L, split)
        uses[need > 0] = True
        out = torch.empty((w.batch, w.num_q_heads, 128), dtype=torch.float16, device="cuda")
        lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
        _lib.hyb_decode_attn_noalloc(cache.desc, q, w.softmax_scale, L, split, out, lse)
        torch.cuda.synchronize()
        assert_decode_close(w, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse,
                            what="noalloc split=%d (%d splits)" % (split, ns))
    assert uses.get(True) and uses.get(False), "both merge paths must be exercised"
    assert cache.status() == 0


def test_noalloc_rejects_problems_beyond_its_buffer():
    import torch
    from int8_paged_kv_hybrid_b200 import HybError, _lib
    # many rows x many splits: more scratch than the static buffer holds
    w = synth.custom_workload("noalloc_big", [8000] * 8, 64, 8, seed=3, schedule="one")
    cache, _ = make_pair(w, gpu=True)
    L = int(w.lens.max())
    assert _lib.hyb_decode_workspace_bytes(cache.desc, L, 64) > _lib.hyb_noalloc_scratch_limit()
    q = torch.zeros((w.batch, w.num_q_heads, 128), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(HybError) as ei:
        _lib.hyb_decode_attn_noalloc(cache.desc, q, 1.0, L, 64, out)
    assert ei.value.code == _lib.HYB_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.strerror(_lib.HYB_ERR_SCRATCH_LIMIT)
