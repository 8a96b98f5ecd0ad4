"""Drive the GPU library and the CPU oracle through the same call sequence."""
import numpy as np

import oracle
from int8_paged_kv_hybrid_b200 import synth

# accuracy bar of the decode attention output versus the FP64 oracle
MAX_ABS = 2e-3
MAX_REL_L2 = 1e-3


def make_pair(w, quant_bits=8, gpu=True):
    ora = oracle.OracleCache(w.batch, w.num_kv_heads, w.num_q_heads, w.max_blocks, quant_bits,
                             hot=w.hot_tokens, block=w.block_size)
    if w.n_int4 is not None:
        ora.set_n_int4(w.n_int4)
    cache = None
    if gpu:
        from int8_paged_kv_hybrid_b200 import HybridKVCache
        cache = HybridKVCache(w.batch, w.num_kv_heads, w.num_q_heads, w.num_phys_blocks, w.max_blocks,
                              quant_bits=quant_bits, block_table=w.block_table, n_int4=w.n_int4,
                              hot_tokens=w.hot_tokens, block_size=w.block_size)
    return cache, ora


def replay(w, cache, ora, steps=None, check_every=None):
    """Run the workload's append schedule on both sides.  If check_every is set,
    compare the whole cache bit for bit every that many calls."""
    import torch
    sched = w.schedule if steps is None else w.schedule[:steps]
    for si, n in enumerate(sched):
        k, v = synth.step_tokens(w, si, n)
        ora.append(n, k, v)
        if cache is not None:
            cache.append(torch.from_numpy(np.ascontiguousarray(n)).cuda(),
                         torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            if check_every and (si + 1) % check_every == 0:
                assert_cache_equal(w, cache, ora, where="after call %d" % si)


def assert_cache_equal(w, cache, ora, where=""):
    import torch
    torch.cuda.synchronize()
    ex = ora.export(w.block_table, w.num_phys_blocks)
    cold = cache.cold.cpu().numpy()
    sc = cache.scales.cpu().numpy()
    hot = cache.hot.cpu().numpy()
    sl = cache.seq_lens.cpu().numpy()
    assert np.array_equal(sl, ex["seq_lens"]), (where, sl, ex["seq_lens"])
    want = ex["cold"]
    if ora.quant_bits != 0:
        # the upper half of an INT4 block's tiles holds no code (unspecified)
        cold = cold.copy()
        want = want.copy()
        bt = np.asarray(w.block_table)
        for b in range(w.batch):
            for i in range(bt.shape[1]):
                if bt[b, i] >= 0 and ora.block_q(b, i) == 7:
                    cold[bt[b, i], :, :, 4096:] = 0
                    want[bt[b, i], :, :, 4096:] = 0
    if not np.array_equal(cold, want):
        bad = np.argwhere(cold != want)
        raise AssertionError("%s: %d cold bytes differ, first at %s (gpu %d, oracle %d)" % (
            where, len(bad), tuple(bad[0]), cold[tuple(bad[0])], want[tuple(bad[0])]))
    if not np.array_equal(sc.view(np.uint32), ex["scales"].view(np.uint32)):
        bad = np.argwhere(sc.view(np.uint32) != ex["scales"].view(np.uint32))
        raise AssertionError("%s: %d scales differ, first at %s (gpu %r, oracle %r)" % (
            where, len(bad), tuple(bad[0]), sc[tuple(bad[0])], ex["scales"][tuple(bad[0])]))
    assert np.array_equal(hot.view(np.uint16), ex["hot"].view(np.uint16)), where
    assert cache.status() == 0


def decode_both(w, cache, ora, split_tokens=None, pairs=None, q=None):
    """GPU decode (all rows) and oracle decode (all rows or `pairs`)."""
    import torch
    if q is None:
        q = synth.query(w)
    st = w.split_tokens if split_tokens is None else split_tokens
    qt = torch.from_numpy(q).cuda()
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
    out = cache.decode(qt, w.softmax_scale, int(w.lens.max()), st, lse=lse)
    torch.cuda.synchronize()
    ref, ref_lse = ora.decode(q, w.softmax_scale, pairs=pairs)
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse


def errors(got, ref, pairs=None):
    """(max-abs, max per-row relative L2) over the rows the oracle computed."""
    if pairs is None:
        g = got.reshape(-1, got.shape[-1])
        r = ref.reshape(-1, ref.shape[-1])
    else:
        g = np.stack([got[b, h] for b, h in pairs])
        r = np.stack([ref[b, h] for b, h in pairs])
    mabs = float(np.abs(g - r).max())
    nr = np.linalg.norm(r, axis=1)
    rel = np.linalg.norm(g - r, axis=1) / np.where(nr > 0, nr, 1.0)
    return mabs, float(rel.max())


def assert_decode_close(w, got, lse, ref, ref_lse, pairs=None, what=""):
    mabs, rel = errors(got, ref, pairs)
    assert mabs <= MAX_ABS and rel <= MAX_REL_L2, "%s: max-abs %.3g rel-L2 %.3g" % (what, mabs, rel)
    rows = [(b, h) for b in range(w.batch) for h in range(w.num_q_heads)] if pairs is None else pairs
    for b, h in rows:
        if np.isinf(ref_lse[b, h]):
            assert np.isneginf(lse[b, h])
        else:
            assert abs(lse[b, h] - ref_lse[b, h]) <= 1e-3 * max(1.0, abs(ref_lse[b, h])), (b, h)
    return mabs, rel
