"""Pins of the oracle's sparse L2 decode (top-k of the INT4-block tokens).

Source: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 2.2 (the
L2 cold blocks keep only the KV of the top-k attention scores) and section
5.3 (sparse_top_k, default 32; rule min(128, context_length // 256)).  Pins:
the dense result when k covers every L2 token or there is no L2 block;
planted tokens whose scores stand far above the rest are exactly the ones
kept (checked against dense brute force over that set, rebuilt from the
stored codes); equal scores keep the oldest positions; k = 0 drops the L2
tokens; the page's rule at its worked value (32K context -> 128).
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from golden_cases import D

BLOCK = 64


def _dense_kv(oc, b, L):
    """K, V [L][hkv][D] float64 rebuilt from the oracle's storage."""
    K = np.zeros((L, oc.hkv, D))
    V = np.zeros((L, oc.hkv, D))
    ring = oc.ring(b).astype(np.float64)
    cold = max(0, L - oc.hot)
    for p in range(L):
        if p >= cold:
            K[p], V[p] = ring[:, p % oc.hot, 0], ring[:, p % oc.hot, 1]
        else:
            _, codes, sc = oc.get_block(b, p // BLOCK)
            K[p] = codes[:, 0, p % BLOCK] * sc[:, 0:1].astype(np.float64)
            V[p] = codes[:, 1, p % BLOCK] * sc[:, 1:2].astype(np.float64)
    return K, V


def _attend(q, K, V, keep, scale, kv):
    z = scale * (K[keep, kv, :] @ q.astype(np.float64))
    return softmax(z) @ V[keep, kv, :], logsumexp(z)


def _cache(L, n4, hkv=1, hq=1, qbits=8, seed=0, kfn=None, vscale=1.0):
    rng = np.random.default_rng(seed)
    nb = (max(0, L - 32) + BLOCK - 1) // BLOCK
    oc = oracle.OracleCache(1, hkv, hq, max_blocks_per_seq=max(1, nb), quant_bits=qbits)
    if qbits == 8:
        oc.set_n_int4(np.array([n4], np.int32))
    k = rng.standard_normal((1, L, hkv, D)).astype(np.float16)
    if kfn is not None:
        k = kfn(k, rng).astype(np.float16)
    v = (rng.standard_normal((1, L, hkv, D)) * vscale).astype(np.float16)
    oc.append(np.array([L], np.int32), k, v)
    return oc


@pytest.mark.parametrize("qbits,n4", [(8, 2), (4, 0)])
def test_k_covering_all_l2_tokens_is_dense(qbits, n4):
    L = 300
    oc = _cache(L, n4, hkv=2, hq=8, qbits=qbits, seed=1)
    q = np.random.default_rng(2).standard_normal((1, 8, D)).astype(np.float16)
    dense, ld = oc.decode(q, 0.088)
    n_l2 = min(L - 32, (n4 if qbits == 8 else 99) * BLOCK)
    for k in (n_l2, n_l2 + 5, 1000):
        out, lse = oc.decode(q, 0.088, top_k=k)
        assert np.abs(out - dense).max() < 1e-12 and np.abs(lse - ld).max() < 1e-12


def test_no_l2_blocks_is_dense_for_any_k():
    oc = _cache(400, 0, hkv=1, hq=4, seed=3)
    q = np.random.default_rng(4).standard_normal((1, 4, D)).astype(np.float16)
    dense, ld = oc.decode(q, 0.088)
    for k in (0, 1, 32):
        out, lse = oc.decode(q, 0.088, top_k=k)
        assert np.abs(out - dense).max() < 1e-12 and np.abs(lse - ld).max() < 1e-12


def test_planted_tokens_are_the_ones_kept():
    """Six L2 tokens get K = 0.3 * q (scores well above the rest); all other L2 keys
    are small noise.  top_k = 6 keeps exactly those six, and the output is
    dense attention over them plus every non-L2 token."""
    L, n4 = 400, 4  # L2 = positions 0..255
    q = np.random.default_rng(5).standard_normal((1, 1, D)).astype(np.float16)
    planted = [3, 64, 100, 191, 200, 255]

    def kfn(k, rng):
        k = k * 0.05
        for p in planted:
            k[0, p, 0] = 0.3 * q[0, 0]
        return k
    oc = _cache(L, n4, seed=6, kfn=kfn)
    K, V = _dense_kv(oc, 0, L)
    keep = planted + list(range(256, L))
    want, wl = _attend(q[0, 0], K, V, keep, 0.088, 0)
    out, lse = oc.decode(q, 0.088, top_k=6)
    assert np.abs(out[0, 0] - want).max() < 1e-12 and abs(lse[0, 0] - wl) < 1e-12
    # and it differs from the dense result (the other L2 tokens matter)
    dense, _ = oc.decode(q, 0.088)
    assert np.abs(dense[0, 0] - want).max() > 1e-4


def test_equal_scores_keep_the_oldest_positions():
    """K = 0 on every L2 token: all L2 scores are 0, so top_k keeps positions
    0..k-1 (the older position wins a tie)."""
    L, n4, k = 300, 2, 10

    def kfn(kk, rng):
        kk[0, :128] = 0.0
        return kk
    oc = _cache(L, n4, seed=7, kfn=kfn)
    q = np.random.default_rng(8).standard_normal((1, 1, D)).astype(np.float16)
    K, V = _dense_kv(oc, 0, L)
    want, wl = _attend(q[0, 0], K, V, list(range(k)) + list(range(128, L)), 0.088, 0)
    out, lse = oc.decode(q, 0.088, top_k=k)
    assert np.abs(out[0, 0] - want).max() < 1e-12 and abs(lse[0, 0] - wl) < 1e-12
    # top_k = 0: no L2 token at all
    want0, wl0 = _attend(q[0, 0], K, V, list(range(128, L)), 0.088, 0)
    out0, lse0 = oc.decode(q, 0.088, top_k=0)
    assert np.abs(out0[0, 0] - want0).max() < 1e-12 and abs(lse0[0, 0] - wl0) < 1e-12


def test_sparse_top_k_rule():
    """Section 5.3: k = min(128, context_length // 256); 32K context -> 128."""
    assert oracle.sparse_top_k(32768) == 128
    assert oracle.sparse_top_k(8192) == 32
    assert oracle.sparse_top_k(255) == 0
    assert oracle.sparse_top_k(10 ** 7) == 128
