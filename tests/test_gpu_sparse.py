"""hyb_decode_attn_sparse (top-k of the INT4 "L2" block tokens per query head)
on the GPU against the oracle.

The oracle keeps the top_k L2 tokens by their exact FP64 attention logit.
The GPU ranks by a key computed in lower precision, so where two logits are
closer than the key's error bound either choice is correct.  The tests
therefore check that the GPU's selection (read back from the workspace) is a
valid top-k -- the right count, distinct L2 positions, and no unselected
token whose exact logit beats a selected one's by more than the two tokens'
key error bounds -- and that the output matches the oracle's attention over
that same selection within the accuracy bar of the dense path.

Key error bound (the GPU key, in logit units): q is taken in 16-bit fixed
point, qi_c = rint(q_c * 32767 / M) with M = max|q|, so q_c = (qi_c + d_c) *
M / 32767 with |d_c| <= 0.5 plus the FP32 rounding of q_c * (32767 / M)
(below 32767 * 2^-24 < 0.002).  The integer dot product of qi with the codes
is exact; the key is (float)dot * K-scale, two FP32 roundings (2^-24 each,
relative).  Hence |key * M / 32767 * softmax_scale - logit_j| <= |scale| *
(M / 32767) * 0.502 * Kscale_j * sum_c |code_j,c| + 2^-22 * |logit_j|.
"""
import numpy as np
import pytest

from harness import assert_decode_close, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def _key_err(ora, q, scale, b, h, n2):
    """Per L2 position of (b, h): the bound on |GPU key - exact logit|."""
    g = ora.hq // ora.hkv
    hk = h // g
    M = float(np.abs(q[b, h].astype(np.float64)).max())
    err = np.zeros(n2)
    blk = ora.block
    for i in range((n2 + blk - 1) // blk):
        _, codes, sc = ora.get_block(b, i)
        kc = codes[hk, 0].astype(np.int64)  # [block][d]
        sa = np.abs(kc).sum(axis=1).astype(np.float64)
        lo, hi = i * blk, min(n2, (i + 1) * blk)
        err[lo:hi] = abs(scale) * (M / 32767.0) * 0.502 * float(sc[hk, 0]) * sa[:hi - lo]
    return err


def _l2_count(w, ora, b):
    L = int(ora.lens()[b])
    cold = max(0, L - w.hot_tokens)
    n4 = (1 << 30) if ora.quant_bits == 4 else (0 if w.n_int4 is None else int(w.n_int4[b]))
    return min(cold, n4 * w.block_size)


def check_sparse(w, cache, ora, top_k, split=0, q=None, max_seq_len=None, pairs=None, what=""):
    """Run the sparse call; check the selection's validity and the output
    against the oracle's attention over the GPU's own selection."""
    import torch
    if q is None:
        q = synth.query(w)
    L = int(w.lens.max()) if max_seq_len is None else max_seq_len
    ws = cache.sparse_workspace(L, split)
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
    out = cache.decode_sparse(torch.from_numpy(q).cuda(), w.softmax_scale, L, top_k, split, lse=lse,
                              workspace=ws)
    torch.cuda.synchronize()
    selv = cache.sparse_selection(ws, L, split).cpu().numpy()
    rows = [(b, h) for b in range(w.batch) for h in range(w.num_q_heads)] if pairs is None else pairs
    sel = [[] for _ in range(w.batch * w.num_q_heads)]
    for b, h in rows:
        n2 = _l2_count(w, ora, b)
        cnt = min(top_k, n2)
        got = selv[b, h, :cnt].astype(np.int64) if cnt > 0 else np.zeros(0, np.int64)
        assert np.all(np.diff(got) > 0) and (cnt == 0 or (got[0] >= 0 and got[-1] < n2)), (what, b, h, got)
        sel[b * w.num_q_heads + h] = got.tolist()
        if 0 < cnt < n2:
            s = ora.l2_scores(q, w.softmax_scale, b, h)
            e = _key_err(ora, q, w.softmax_scale, b, h, n2) + 2.0 ** -22 * np.abs(s)
            kept = np.zeros(n2, bool)
            kept[got] = True
            worst_kept = float((s[kept] + e[kept]).min())
            best_left = float((s[~kept] - e[~kept]).max())
            assert worst_kept >= best_left, (
                "%s (b=%d h=%d): an unselected L2 token's logit beats a selected one's by more than the "
                "key error bounds (%.9g < %.9g)" % (what, b, h, worst_kept, best_left))
    ref, ref_lse = ora.decode(q, w.softmax_scale, sel=sel, pairs=pairs)
    got = out.float().cpu().numpy().astype(np.float64)
    assert_decode_close(w, got, lse.cpu().numpy(), ref, ref_lse, pairs=pairs, what=what)
    return sel


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
        check_sparse(w, cache, ora, k, split, what="top_k=%d qbits=%d split=%d" % (k, qbits, split))
    assert cache.status() == 0


def test_sparse_negative_scale():
    """A negative softmax scale: the top logits are the most negative dot products."""
    lens = [500, 900]
    nb = [synth.cold_blocks_for(L) for L in lens]
    w = synth.custom_workload("negscale", lens, 8, 2, seed=77, softmax_scale=-0.09, schedule="chunk",
                              n_int4=[n // 2 for n in nb])
    cache, ora = make_pair(w, quant_bits=8)
    replay(w, cache, ora)
    for k in (3, 50):
        check_sparse(w, cache, ora, k, what="negative scale top_k=%d" % k)


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
        sel = check_sparse(w, cache, ora, k, what="ties top_k=%d" % k)
        # exact ties (all keys 0) resolve to the oldest positions on both sides
        for r in range(w.batch * w.num_q_heads):
            assert sel[r] == list(range(min(k, _l2_count(w, ora, r // w.num_q_heads)))), r
        ref, ref_lse = ora.decode(synth.query(w), w.softmax_scale, top_k=k)
        ref2, _ = ora.decode(synth.query(w), w.softmax_scale, sel=sel)
        assert np.array_equal(ref, ref2)


def test_sparse_near_ties():
    """L2 K built so that many logits nearly tie (K = c * q with c on a coarse
    grid plus tiny noise): the selection must stay valid within the bound."""
    import torch
    lens = [700, 1200]
    nb = [synth.cold_blocks_for(L) for L in lens]
    w = synth.custom_workload("neartie", lens, 4, 1, seed=5, schedule="chunk", n_int4=[n // 2 for n in nb])
    cache, ora = make_pair(w, quant_bits=8)
    q = synth.query(w)
    rng = np.random.default_rng(9)
    for si, n in enumerate(w.schedule):
        k, v = synth.step_tokens(w, si, n)
        for b in range(w.batch):
            for j in range(int(n[b])):
                c = rng.integers(-3, 4) / 4.0
                k[b, j, 0] = (c * q[b, 0].astype(np.float32) + 1e-3 * rng.standard_normal(128)).astype(np.float16)
        ora.append(n, k, v)
        cache.append(torch.from_numpy(np.ascontiguousarray(n)).cuda(), torch.from_numpy(k).cuda(),
                     torch.from_numpy(v).cuda())
    for k in (10, 100, 250):
        check_sparse(w, cache, ora, k, q=q, what="near ties top_k=%d" % k)


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
    check_sparse(w, cache, ora, k, split=512, max_seq_len=32768, pairs=pairs, what="32K top_k=128")
