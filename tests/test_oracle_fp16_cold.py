"""Pins of the oracle's FP16 cold zone (quantization_bits 0).

Source: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 5.2
(quantization_bits 0 switches quantization off and keeps the cold zone in
FP16) and section 4.2 (one softmax over hot and cold keys).  With nothing
quantized the decode result is plain softmax attention over the FP16 inputs,
so the pins rebuild K and V from the appended arrays alone (not through the
oracle's storage) and compare against dense brute force; the export is
checked slot by slot against the same inputs.
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from golden_cases import HOT, D

BLOCK = 64


def _fill(oc, rng, total, hkv, max_step=70):
    B = len(total)
    cur = np.zeros(B, np.int64)
    hk, hv = [[] for _ in range(B)], [[] for _ in range(B)]
    while (cur < total).any():
        n = np.minimum(rng.integers(1, max_step + 1, size=B), total - cur)
        mx = max(1, int(n.max()))
        k = rng.standard_normal((B, mx, hkv, D)).astype(np.float16)
        v = rng.standard_normal((B, mx, hkv, D)).astype(np.float16)
        oc.append(n.astype(np.int32), k, v)
        for b in range(B):
            hk[b].append(k[b, :n[b]])
            hv[b].append(v[b, :n[b]])
        cur += n
    return ([np.concatenate(x, 0) if x else np.zeros((0, hkv, D), np.float16) for x in hk],
            [np.concatenate(x, 0) if x else np.zeros((0, hkv, D), np.float16) for x in hv])


@pytest.mark.parametrize("hkv,g", [(1, 1), (2, 4), (1, 8)])
def test_fp16_cold_is_plain_attention(hkv, g):
    rng = np.random.default_rng(300 + hkv * 10 + g)
    total = np.array([200, 1, 32, 33, 97, 0, 96, 160])
    B = len(total)
    oc = oracle.OracleCache(B, hkv, hkv * g, max_blocks_per_seq=3, quant_bits=0)
    ks, vs = _fill(oc, rng, total, hkv)
    q = rng.standard_normal((B, hkv * g, D)).astype(np.float16)
    scale = 1.0 / np.sqrt(D)
    out, lse = oc.decode(q, scale, nthreads=2)
    for b in range(B):
        L = int(total[b])
        if L == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        K, V = ks[b].astype(np.float64), vs[b].astype(np.float64)
        for h in range(hkv * g):
            z = scale * (K[:, h // g, :] @ q[b, h].astype(np.float64))
            assert np.abs(out[b, h] - softmax(z) @ V[:, h // g, :]).max() < 1e-12
            assert abs(lse[b, h] - logsumexp(z)) < 1e-12


def test_fp16_blocks_hold_the_inputs_and_export_in_ring_layout():
    rng = np.random.default_rng(41)
    total = np.array([160, 97, 20])
    B, hkv = 3, 2
    oc = oracle.OracleCache(B, hkv, 8, max_blocks_per_seq=3, quant_bits=0)
    ks, vs = _fill(oc, rng, total, hkv)
    for b in range(B):
        cold = max(0, int(total[b]) - HOT)
        for i in range(3):
            ok, vals = oc.get_block_fp16(b, i)
            n = min(BLOCK, max(0, cold - i * BLOCK))
            assert ok == (n > 0)
            if not ok:
                continue
            for t in range(n):
                p = i * BLOCK + t
                assert np.array_equal(vals[:, 0, t], ks[b][p]) and np.array_equal(vals[:, 1, t], vs[b][p])
            assert not vals[:, :, n:].any()  # unsealed slots stay 0
        assert oc.get_block(b, 0)[0] == 0  # no INT8/INT4 view of an FP16 block
    table = np.array([[5, 0, 3], [1, 4, -1], [-1, -1, -1]], np.int32)
    ex = oc.export(table, 6)
    cold, lens = ex["cold"], ex["seq_lens"]
    assert cold.shape == (6, hkv, 4, BLOCK * D)
    c16 = cold.reshape(6, hkv, BLOCK, 2, D * 2).view(np.float16)  # [phys][h][slot][K|V][d]
    for b in range(B):
        L = int(total[b])
        assert lens[b] == L
        for p in range(max(0, L - HOT)):
            phys = table[b, p // BLOCK]
            assert np.array_equal(c16[phys, :, p % BLOCK, 0], ks[b][p])
            assert np.array_equal(c16[phys, :, p % BLOCK, 1], vs[b][p])
    # physical block 2 is referenced by nobody: left zero
    assert not cold[2].any()


def test_fp16_cold_rejects_migration_and_tiers():
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=2, quant_bits=0)
    k = np.ones((1, 100, 1, D), np.float16)
    oc.append(np.array([100], np.int32), k, k)
    with pytest.raises(Exception):
        oc.migrate(np.array([1], np.int32))
