"""hyb_decode_attn_sparse (top-k of the INT4 "L2" block tokens per query head)
on the GPU against the oracle's ora_decode_topk: the same selection (the key
is exact integer / FP32 arithmetic on both sides) and the output within the
accuracy bar of the dense path."""
import numpy as np
import pytest

from harness import assert_decode_close, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def _decode_sparse(w, cache, ora, top_k, split=0, q=None):
    import torch
    if q is None:
        q = synth.query(w)
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
    out = cache.decode_sparse(torch.from_numpy(q).cuda(), w.softmax_scale, int(w.lens.max()), top_k, split,
                              lse=lse)
    torch.cuda.synchronize()
    ref, ref_lse = ora.decode(q, w.softmax_scale, top_k=top_k)
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse


@pytest.mark.parametrize("qbits,hq,hkv", [(8, 32, 8), (8, 28, 4), (4, 8, 2)])
@pytest.mark.parametrize("split", [0, 64])
def test_sparse_parity(qbits, hq, hkv, split):
    lens = [0, 1, 40, 97, 300, 700, 2100]
    nb = [synth.cold_blocks_for(L) for L in lens]
    w = synth.custom_workload("sparse", lens, hq, hkv, seed=qbits * 5 + hq + split, max_step=64,
                              n_int4=[(2 * n) // 3 for n in nb] if qbits == 8 else None)
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora)
    for k in (0, 1, 7, 32, 128, 1024):
        got, lse, ref, ref_lse = _decode_sparse(w, cache, ora, k, split)
        assert_decode_close(w, got, lse, ref, ref_lse, what="top_k=%d qbits=%d split=%d" % (k, qbits, split))
    assert cache.status() == 0


def test_sparse_all_ties_keep_oldest():
    """Zero K on the L2 tokens: every key is 0 and the oldest top_k are kept."""
    lens = [400, 333]
    w = synth.custom_workload("ties", lens, 8, 2, seed=3, schedule="chunk", n_int4=[3, 2])
    cache, ora = make_pair(w, quant_bits=8)
    import torch
    for si, n in enumerate(w.schedule):
        k, v = synth.step_tokens(w, si, n)
        start = [sum(int(x[b]) for x in w.schedule[:si]) for b in range(w.batch)]
        for b in range(w.batch):
            for j in range(int(n[b])):
                if start[b] + j < 192:
                    k[b, j] = 0
        ora.append(n, k, v)
        cache.append(torch.from_numpy(np.ascontiguousarray(n)).cuda(), torch.from_numpy(k).cuda(),
                     torch.from_numpy(v).cuda())
    for k in (5, 64, 100):
        got, lse, ref, ref_lse = _decode_sparse(w, cache, ora, k)
        assert_decode_close(w, got, lse, ref, ref_lse, what="ties top_k=%d" % k)


def test_sparse_long_context_rule():
    """A 32K-token sequence with half its cold blocks INT4: top_k from the
    page's rule (min(128, ctx // 256) = 128), two sequences, 512-token splits."""
    from int8_paged_kv_hybrid_b200 import hyb_sparse_top_k
    lens = [32768, 20000]
    nb = [synth.cold_blocks_for(L) for L in lens]
    w = synth.custom_workload("long", lens, 32, 8, seed=11, schedule="chunk", chunk=1024,
                              n_int4=[n // 2 for n in nb])
    cache, ora = make_pair(w, quant_bits=8)
    replay(w, cache, ora)
    k = hyb_sparse_top_k(32768)
    assert k == 128
    pairs = [(b, h) for b in range(2) for h in (0, 5, 17, 31)]
    import torch
    q = synth.query(w)
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
    out = cache.decode_sparse(torch.from_numpy(q).cuda(), w.softmax_scale, 32768, k, 512, lse=lse)
    torch.cuda.synchronize()
    ref, ref_lse = ora.decode(q, w.softmax_scale, pairs=pairs, top_k=k)
    assert_decode_close(w, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy(), ref, ref_lse,
                        pairs=pairs, what="32K top_k=128")
