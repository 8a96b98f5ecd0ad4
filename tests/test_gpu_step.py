"""hyb_decode_step (append of one token per sequence + attention, one launch)
against the oracle: the cache after every step bit-exact (codes, scales, hot
ring, seq_lens) and the attention output within the accuracy bar."""
import numpy as np
import pytest

from harness import assert_cache_equal, assert_decode_close, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def _run_steps(w, cache, ora, n_steps, split, seed, n_pattern=None, qbits=8):
    """n_steps fused steps of one token per sequence (or n_pattern[step])."""
    import torch
    rng = np.random.default_rng(seed)
    lens = ora.lens().astype(np.int64)
    L_max = int(lens.max()) + n_steps
    ws = cache.step_workspace(L_max, split)
    for st in range(n_steps):
        n = np.ones(w.batch, np.int32) if n_pattern is None else n_pattern[st].astype(np.int32)
        k = rng.standard_normal((w.batch, 1, w.num_kv_heads, 128)).astype(np.float16)
        v = rng.standard_normal((w.batch, 1, w.num_kv_heads, 128)).astype(np.float16)
        q = rng.standard_normal((w.batch, w.num_q_heads, 128)).astype(np.float16)
        ora.append(n, k, v)
        lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
        out = cache.step(torch.from_numpy(n).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                         torch.from_numpy(q).cuda(), w.softmax_scale, L_max, split, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        w.lens = ora.lens()
        assert_cache_equal(w, cache, ora, "step %d" % st)
        ref, ref_lse = ora.decode(q, w.softmax_scale)
        assert_decode_close(w, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref,
                            ref_lse, what="step %d" % st)
    return ws


@pytest.mark.parametrize("hq,hkv,split", [(8, 8, 0), (32, 8, 128), (28, 4, 64), (16, 2, 0), (32, 8, -4),
                                           (16, 2, -9), (32, 8, -20), (28, 4, -24)])
def test_steps_bit_exact_and_close(hq, hkv, split):
    """Lengths around every edge: empty, below / at the hot size, first seal,
    block boundaries, several splits (cluster and workspace merges)."""
    lens = [0, 1, 31, 32, 33, 63, 95, 96, 97, 159, 160, 500, 1200]
    w = synth.custom_workload("step", lens, hq, hkv, seed=hq + 7 * hkv, max_step=64, pool_extra=0)
    # room for the steps: widen the block table
    extra = 3
    bt = np.full((w.batch, w.max_blocks + extra), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(synth.cold_blocks_for(int(w.lens[b])), synth.cold_blocks_for(int(w.lens[b]) + 70)):
            bt[b, j] = nxt
            nxt += 1
    w.block_table = bt
    w.num_phys_blocks = nxt
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    _run_steps(w, cache, ora, 70, split, seed=11)


@pytest.mark.parametrize("hq,hkv,split", [(8, 2, 0), (32, 8, 128)])
def test_steps_fp16_cold(hq, hkv, split):
    """quantization_bits 0: the sealed token's FP16 rows move into the staged
    half block and the cache; 70 steps cross both halves of a block."""
    lens = [0, 1, 31, 32, 33, 63, 64, 65, 95, 96, 97, 500, 1200]
    w = synth.custom_workload("step16", lens, hq, hkv, seed=hq + hkv, max_step=64, pool_extra=0)
    nb = [synth.cold_blocks_for(L + 70) for L in lens]
    bt = np.full((w.batch, max(nb)), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(synth.cold_blocks_for(int(w.lens[b])), nb[b]):
            bt[b, j] = nxt
            nxt += 1
    w.block_table = bt
    w.num_phys_blocks = nxt
    cache, ora = make_pair(w, quant_bits=0)
    replay(w, cache, ora)
    _run_steps(w, cache, ora, 70, split, seed=17, qbits=0)


@pytest.mark.parametrize("hot,qbits,hq,hkv,split", [(16, 8, 8, 2, 0), (64, 8, 32, 8, 0), (128, 8, 8, 2, 64),
                                                    (64, 0, 8, 2, 0), (128, 4, 28, 4, 0)])
def test_steps_hot_sizes(hot, qbits, hq, hkv, split):
    """hot_tokens 16 / 64 / 128: the evicted token (position L - hot, read in
    the prologue) is sealed at the tail block's item, the new token written
    at the hot item holding ring slot L % hot."""
    lens = [0, 1, hot - 1, hot, hot + 1, hot + 63, hot + 64, 500]
    w = synth.custom_workload("steph%d" % hot, lens, hq, hkv, seed=hot + qbits, max_step=64, pool_extra=0,
                              hot=hot)
    nb = [synth.cold_blocks_for(L + 70, hot) for L in lens]
    bt = np.full((w.batch, max(max(nb), w.max_blocks)), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(synth.cold_blocks_for(int(w.lens[b]), hot), nb[b]):
            bt[b, j] = nxt
            nxt += 1
    w.block_table = bt
    w.num_phys_blocks = nxt
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora)
    _run_steps(w, cache, ora, 70, split, seed=hot, qbits=qbits)


@pytest.mark.parametrize("qbits,int4", [(4, False), (8, True)])
def test_steps_int4(qbits, int4):
    lens = [40, 130, 600]
    nb = [synth.cold_blocks_for(L + 40) for L in lens]
    w = synth.custom_workload("step4", lens, 28, 4, seed=5, schedule="chunk",
                              n_int4=[max(1, n // 2) for n in nb] if int4 else None)
    bt = np.full((w.batch, max(nb)), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(synth.cold_blocks_for(int(w.lens[b])), nb[b]):
            bt[b, j] = nxt
            nxt += 1
    w.block_table = bt
    w.num_phys_blocks = nxt
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora)
    _run_steps(w, cache, ora, 40, 0, seed=3, qbits=qbits)


def test_mixed_and_invalid_n_new():
    """Sequences that do not append this step (0), and an invalid count (2):
    that sequence is attended unchanged and the status says so."""
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    lens = [100, 200, 300]
    w = synth.custom_workload("mixed", lens, 8, 2, seed=9, schedule="chunk")
    bt = np.full((w.batch, w.max_blocks + 1), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    for b in range(w.batch):
        bt[b, synth.cold_blocks_for(lens[b])] = w.num_phys_blocks + b
    w.block_table = bt
    w.num_phys_blocks += w.batch
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    pattern = [np.array([1, 0, 1])] * 3 + [np.array([0, 1, 0])]
    _run_steps(w, cache, ora, 4, 0, seed=1, n_pattern=pattern)
    assert cache.status() == 0
    before = cache.seq_lens.cpu().numpy().copy()
    n = torch.tensor([2, 1, 0], dtype=torch.int32, device="cuda")
    k = torch.zeros((3, 1, 2, 128), dtype=torch.float16, device="cuda")
    q = torch.from_numpy(synth.query(w)).cuda()
    cache.step(n, k, k, q, w.softmax_scale, int(before.max()) + 1, 0)
    torch.cuda.synchronize()
    assert cache.status(clear=True) == _lib.HYB_STATUS_BAD_N_NEW
    assert list(cache.seq_lens.cpu().numpy()) == [before[0], before[1] + 1, before[2]]


def test_step_into_unallocated_block():
    """The token that leaves the hot ring belongs to a block the table does
    not give (-1): HYB_STATUS_BAD_BLOCK, nothing written to the cold pool for
    that sequence (as hyb_kv_append skips such a block), the new token still
    in the ring and seq_lens advanced; the other sequence is unaffected."""
    import torch
    from int8_paged_kv_hybrid_b200 import _lib
    lens = [96, 200]  # sequence 0: its next sealed token opens block 1, not allocated
    w = synth.custom_workload("unalloc", lens, 8, 2, seed=13, schedule="chunk")
    assert w.block_table[0, 1] == -1
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    cold0 = cache.cold.clone()
    rng = np.random.default_rng(2)
    n = np.ones(2, np.int32)
    k = rng.standard_normal((2, 1, 2, 128)).astype(np.float16)
    v = rng.standard_normal((2, 1, 2, 128)).astype(np.float16)
    q = rng.standard_normal((2, 8, 128)).astype(np.float16)
    lse = torch.empty((2, 8), dtype=torch.float32, device="cuda")
    out = cache.step(torch.from_numpy(n).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                     torch.from_numpy(q).cuda(), w.softmax_scale, 201, 0, lse=lse)
    torch.cuda.synchronize()
    assert cache.status(clear=True) == _lib.HYB_STATUS_BAD_BLOCK
    assert cache.seq_lens.tolist() == [97, 201]
    assert torch.isfinite(out.float()).all()
    # sequence 0: ring slot 96 % 32 = 0 holds the new token; its blocks are untouched
    hot = cache.hot.cpu().numpy()
    assert np.array_equal(hot[0, :, 0, 0], k[0, 0]) and np.array_equal(hot[0, :, 0, 1], v[0, 0])
    phys0 = [int(p) for p in w.block_table[0] if p >= 0]
    assert torch.equal(cache.cold[phys0], cold0[phys0])
    # sequence 1 matches the oracle
    ora.append(n, k, v)
    ref, ref_lse = ora.decode(q, w.softmax_scale, pairs=[(1, hh) for hh in range(8)])
    w.lens = ora.lens()
    assert_decode_close(w, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse,
                        pairs=[(1, hh) for hh in range(8)], what="sequence 1")
