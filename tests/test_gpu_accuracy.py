"""Accuracy of hyb_decode_attn against the FP64 oracle in the regimes that
stress the arithmetic (max-abs <= 2e-3, per-row relative L2 <= 1e-3):

* an attention sink: one early token about 12 nats above a long diffuse tail,
  so that most of the softmax mass sits in thousands of tokens far below the
  running maximum -- with the largest legal split (128 blocks = 8192 tokens
  per CTA) and with the automatic plan;
* a query with one channel 100x the others, which stretches the fixed-point
  range of q.

The weights are quantized relative to the maximum of their own 16-token
group, so a token's weight keeps 16 bits of precision relative to its
neighbours whatever the running maximum is; q carries 24 bits relative to
its largest channel."""
import numpy as np
import pytest

from harness import assert_decode_close, decode_both, make_pair
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def _replay_patched(w, cache, ora, patch):
    """Replay the workload's appends with patch(si, start, k, v) editing each
    call's FP16 inputs in place (start[b] = the call's first position)."""
    import torch
    pos = np.zeros(w.batch, np.int64)
    for si, n in enumerate(w.schedule):
        k, v = synth.step_tokens(w, si, n)
        patch(si, pos.copy(), k, v)
        ora.append(n, k, v)
        cache.append(torch.from_numpy(np.ascontiguousarray(n)).cuda(), torch.from_numpy(k).cuda(),
                     torch.from_numpy(v).cuda())
        pos += n


def _group_query(w, seed):
    """q with every query head of a kv-head group equal (so one sink key
    dominates all of them): [batch][Hq][128] FP16."""
    rng = np.random.default_rng(seed)
    g = w.num_q_heads // w.num_kv_heads
    base = rng.standard_normal((w.batch, w.num_kv_heads, 128)).astype(np.float16)
    return np.repeat(base, g, axis=1)


@pytest.mark.parametrize("L", [8192, 32768])
@pytest.mark.parametrize("split", [8192, 0])
def test_attention_sink(L, split):
    lens = [L, L // 2 + 77]
    w = synth.custom_workload("sink", lens, 8, 2, seed=L // 64 + split // 64, schedule="chunk", chunk=1024)
    q = _group_query(w, 5)
    qf = q.astype(np.float64)

    def patch(si, start, k, v):
        for b in range(w.batch):
            if start[b] == 0 and k.shape[1] > 0:
                for hk in range(w.num_kv_heads):
                    qq = qf[b, hk * (w.num_q_heads // w.num_kv_heads)]
                    c = 12.0 / (w.softmax_scale * float(qq @ qq))
                    k[b, 0, hk] = (c * qq).astype(np.float16)
    cache, ora = make_pair(w)
    _replay_patched(w, cache, ora, patch)
    got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=split, q=q)
    # the sink holds a large share of the mass, but not all of it: the tail matters
    z0 = ref_lse[0, 0]
    assert np.isfinite(z0)
    mabs, rel = assert_decode_close(w, got, lse, ref, ref_lse, what="sink L=%d split=%d" % (L, split))
    print("sink L=%d split=%d: max-abs %.3g rel-L2 %.3g" % (L, split, mabs, rel))


@pytest.mark.parametrize("split", [0, 1024])
def test_query_outlier_channel(split):
    lens = [8192, 3000, 100]
    w = synth.custom_workload("qout", lens, 32, 8, seed=13 + split, schedule="chunk", chunk=1024)
    cache, ora = make_pair(w)
    _replay_patched(w, cache, ora, lambda *a: None)
    q = synth.query(w).astype(np.float32)
    q[:, :, 37] *= 100.0
    q = q.astype(np.float16)
    got, lse, ref, ref_lse = decode_both(w, cache, ora, split_tokens=split, q=q)
    mabs, rel = assert_decode_close(w, got, lse, ref, ref_lse, what="q outlier split=%d" % split)
    print("q outlier split=%d: max-abs %.3g rel-L2 %.3g" % (split, mabs, rel))
