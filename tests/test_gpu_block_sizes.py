"""block_size 128 and 32 on the GPU against the oracle.  A 128-token block is
two 64-token sub-blocks sharing one scale pair; a 32-token block uses the
first half of one 64-slot tile pair.  Appends bit-exact (including a grown
scale re-quantizing the first sub-block), decode within the accuracy bar,
fused steps whose seals grow the block's scale, tier migration, sparse L2
decode."""
import numpy as np
import pytest

from harness import assert_cache_equal, assert_decode_close, decode_both, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu

LENS = [0, 1, 31, 32, 33, 95, 96, 97, 159, 160, 161, 500, 1300]


def _widen(w, extra_tokens):
    need = [synth.cold_blocks_for(int(L) + extra_tokens, w.hot_tokens, w.block_size) for L in w.lens]
    bt = np.full((w.batch, max(max(need), w.max_blocks)), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(synth.cold_blocks_for(int(w.lens[b]), w.hot_tokens, w.block_size), need[b]):
            bt[b, j] = nxt
            nxt += 1
    w.block_table, w.num_phys_blocks = bt, nxt


BLOCKS = [128, 32]


@pytest.mark.parametrize("blk", BLOCKS)
@pytest.mark.parametrize("qbits,int4", [(8, False), (8, True), (4, False), (0, False)])
def test_appends_bit_exact(qbits, int4, blk):
    nb = [synth.cold_blocks_for(L, 32, blk) for L in LENS]
    w = synth.custom_workload("b%d" % blk, LENS, 8, 2, seed=qbits + 10 * int4, max_step=70, block=blk,
                              n_int4=[n // 2 for n in nb] if int4 else None)
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora, check_every=1)
    assert_cache_equal(w, cache, ora, "final")


@pytest.mark.parametrize("blk", BLOCKS)
@pytest.mark.parametrize("qbits,hq,hkv", [(8, 32, 8), (4, 28, 4), (0, 8, 2)])
@pytest.mark.parametrize("split", [0, 128, 256])
def test_decode_parity(qbits, hq, hkv, split, blk):
    nb = [synth.cold_blocks_for(L, 32, blk) for L in LENS]
    w = synth.custom_workload("b%dd" % blk, LENS, hq, hkv, seed=hq + split, max_step=64, block=blk,
                              n_int4=[n // 3 for n in nb] if qbits == 8 else None)
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora)
    got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=split)
    assert_decode_close(w, got, lse, ref, ref_lse, what="block %d qbits=%d split=%d" % (blk, qbits, split))
    assert cache.status() == 0


@pytest.mark.parametrize("blk", BLOCKS)
@pytest.mark.parametrize("qbits,split", [(8, 0), (8, 128), (4, 0), (0, 0)])
def test_fused_steps(qbits, split, blk):
    """90 one-token steps; some tokens carry a K four times larger or a V
    outlier channel, so that seals into the second sub-block grow the block's
    K or V scale (outputs stay of unit size, so the absolute bar applies)."""
    import torch
    w = synth.custom_workload("b%ds" % blk, LENS, 8, 2, seed=5 + qbits, max_step=64, pool_extra=0, block=blk)
    _widen(w, 100)
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora)
    rng = np.random.default_rng(21)
    L_max = int(ora.lens().max()) + 90
    ws = cache.step_workspace(L_max, split)
    for st in range(90):
        n = np.ones(w.batch, np.int32)
        k = rng.standard_normal((w.batch, 1, 2, 128)) * (4.0 if st % 7 == 3 else 1.0)
        v = rng.standard_normal((w.batch, 1, 2, 128))
        if st % 7 == 5:
            v[:, :, :, 0] = 6.0
        k, v = k.astype(np.float16), v.astype(np.float16)
        q = rng.standard_normal((w.batch, 8, 128)).astype(np.float16)
        ora.append(n, k, v)
        lse = torch.empty((w.batch, 8), dtype=torch.float32, device="cuda")
        out = cache.step(torch.from_numpy(n).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                         torch.from_numpy(q).cuda(), w.softmax_scale, L_max, split, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        w.lens = ora.lens()
        assert_cache_equal(w, cache, ora, "step %d" % st)
        ref, ref_lse = ora.decode(q, w.softmax_scale)
        assert_decode_close(w, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse,
                            what="step %d" % st)


@pytest.mark.parametrize("blk", BLOCKS)
def test_migration(blk):
    import torch
    lens = [97, 300, 700, 1300]
    nb = [synth.cold_blocks_for(L, 32, blk) for L in lens]
    w = synth.custom_workload("b%dm" % blk, lens, 32, 8, seed=8, max_step=64, block=blk, n_int4=[1, 0, 2, 3])
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    for tgt in ([n for n in nb], [0, 1, 1, 2], [min(n + 1, w.max_blocks) for n in nb]):
        ora.migrate(np.asarray(tgt, np.int32))
        cache.migrate(torch.tensor(tgt, dtype=torch.int32, device="cuda"))
        w.n_int4 = np.asarray(tgt, np.int32)
        assert_cache_equal(w, cache, ora, "after move to %s" % tgt)
        got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=0)
        assert_decode_close(w, got, lse, ref, ref_lse, what="after move to %s" % tgt)


@pytest.mark.parametrize("blk", BLOCKS)
@pytest.mark.parametrize("k", [0, 5, 64, 1024])
def test_sparse_l2(k, blk):
    import torch
    lens = [300, 1300, 2100]
    nb = [synth.cold_blocks_for(L, 32, blk) for L in lens]
    w = synth.custom_workload("b%dp" % blk, lens, 28, 4, seed=k, max_step=64, block=blk,
                              n_int4=[(2 * n) // 3 for n in nb])
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    q = synth.query(w)
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
    out = cache.decode_sparse(torch.from_numpy(q).cuda(), w.softmax_scale, int(w.lens.max()), k, 0, lse=lse)
    torch.cuda.synchronize()
    ref, ref_lse = ora.decode(q, w.softmax_scale, top_k=k)
    assert_decode_close(w, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse,
                        what="block %d sparse k=%d" % (blk, k))
