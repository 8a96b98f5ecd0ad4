"""hyb_kv_migrate (INT8 <-> INT4 tier migration in place) against the oracle:
the whole cache bit-exact after every migration, decode attention within the
accuracy bar, and appends that continue after it bit-exact too."""
import numpy as np
import pytest

from harness import assert_cache_equal, assert_decode_close, decode_both, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def _both_migrate(w, cache, ora, target, max_delta=None):
    import torch
    ora.migrate(target)
    cache.migrate(torch.from_numpy(np.asarray(target, np.int32)).cuda(), max_delta)
    w.n_int4 = np.asarray(target, np.int32)


@pytest.mark.parametrize("hq,hkv", [(32, 8), (28, 4), (8, 8)])
def test_migrate_bit_exact_then_decode_and_append(hq, hkv):
    lens = [0, 20, 33, 97, 130, 700, 1500, 2047]
    nb = [synth.cold_blocks_for(L) for L in lens]
    # widen the table so that appends can continue after the migrations
    w = synth.custom_workload("mig", lens, hq, hkv, seed=hq + hkv, max_step=64, pool_extra=0,
                              n_int4=[n // 4 for n in nb])
    extra = 5
    bt = np.full((w.batch, w.max_blocks + extra), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(nb[b], synth.cold_blocks_for(lens[b] + 200)):
            bt[b, j] = nxt
            nxt += 1
    w.block_table, w.num_phys_blocks = bt, nxt
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    assert_cache_equal(w, cache, ora, "before")
    # demote most blocks, including the partial tail and blocks not sealed yet
    _both_migrate(w, cache, ora, [min(n + 2, w.max_blocks) for n in nb])
    assert_cache_equal(w, cache, ora, "after demotion")
    got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=0)
    assert_decode_close(w, got, lse, ref, ref_lse, what="after demotion")
    # promote some back, leave others, demote one more
    tgt = [max(0, n // 2) if b % 3 else min(n + 1, w.max_blocks) for b, n in enumerate(nb)]
    _both_migrate(w, cache, ora, tgt)
    assert_cache_equal(w, cache, ora, "after mixed move")
    got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=128)
    assert_decode_close(w, got, lse, ref, ref_lse, what="after mixed move")
    # appends continue: new blocks get the width their tier says
    import torch
    rng = np.random.default_rng(3)
    for st in range(4):
        n = rng.integers(0, 40, size=w.batch).astype(np.int32)
        k = rng.standard_normal((w.batch, 40, w.num_kv_heads, 128)).astype(np.float16)
        v = rng.standard_normal((w.batch, 40, w.num_kv_heads, 128)).astype(np.float16)
        ora.append(n, k, v)
        cache.append(torch.from_numpy(n).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    w.lens = ora.lens()
    assert_cache_equal(w, cache, ora, "after appends")
    got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=0)
    assert_decode_close(w, got, lse, ref, ref_lse, what="after appends")
    assert cache.status() == 0


def test_migrate_full_size_qwen_mixed():
    """The Qwen2-7B mixed-length workload (INT4 for the oldest quarter):
    demote to half of every sequence's blocks, then promote all back."""
    w = synth.make_workload(5)
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    nb = w.cold_blocks()
    _both_migrate(w, cache, ora, nb // 2)
    assert_cache_equal(w, cache, ora, "demoted to half")
    pairs = [(b, 0) for b in range(0, w.batch, 9)] + [(b, w.num_q_heads - 1) for b in range(4, w.batch, 9)]
    got, lse, ref, ref_lse = decode_both(w, cache, ora, pairs=pairs)
    assert_decode_close(w, got, lse, ref, ref_lse, pairs=pairs, what="demoted to half")
    _both_migrate(w, cache, ora, np.zeros(w.batch, np.int32))
    assert_cache_equal(w, cache, ora, "promoted back")


def test_migrate_rejects_bad_targets():
    """A target beyond the table or farther than max_delta leaves that
    sequence unchanged and sets HYB_STATUS_BAD_TIER; the others move."""
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    lens = [500, 800, 300]
    w = synth.custom_workload("migbad", lens, 8, 2, seed=4, schedule="chunk")
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    before = cache.cold.clone()
    cache.migrate(torch.tensor([w.max_blocks + 1, 0, 0], dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert cache.status(clear=True) == _lib.HYB_STATUS_BAD_TIER
    assert torch.equal(cache.cold, before) and cache.n_int4.tolist() == [0, 0, 0]
    # max_delta 2: sequence 1 asks for 5 blocks and is refused, 0 and 2 move
    tgt = [2, 5, 1]
    cache.migrate(torch.tensor(tgt, dtype=torch.int32).cuda(), max_delta=2)
    torch.cuda.synchronize()
    assert cache.status(clear=True) == _lib.HYB_STATUS_BAD_TIER
    assert cache.n_int4.tolist() == [2, 0, 1]
    ora.migrate(np.array([2, 0, 1], np.int32))
    w.n_int4 = np.array([2, 0, 1], np.int32)
    assert_cache_equal(w, cache, ora, "partial move")
