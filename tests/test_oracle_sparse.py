"""Pins of the oracle's sparse L2 decode (top-k of the INT4-block tokens).

Source: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 2.2 (the
L2 cold blocks keep only the KV of the top-k attention scores) and section
5.3 (sparse_top_k, default 32; rule min(128, context_length // 256)).  The
score of a token is its FP64 attention logit.  Pins: a hand-worked selection
whose scores are exact in FP64, with a near-tie that 16-bit fixed-point q
would resolve differently (tests/golden/sparse_select.txt); brute force on
small random caches (numpy logits on K rebuilt from the stored codes, ranked
by numpy); the dense result when k covers every L2 token or there is no L2
block;
planted tokens whose scores stand far above the rest are exactly the ones
kept (checked against dense brute force over that set, rebuilt from the
stored codes); equal scores keep the oldest positions; k = 0 drops the L2
tokens; the page's rule at its worked value (32K context -> 128).
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from golden_cases import D, GOLDEN

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


def _fixture():
    cfg, q, ktok, scores, sel = {}, {}, {}, {}, {}
    with open(GOLDEN + "/sparse_select.txt", encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].split()
            if not line:
                continue
            if line[0] == "config":
                cfg = {k: int(v) for k, v in (x.split("=") for x in line[1:])}
            elif line[0] == "q":
                q = {int(a): float(b) for a, b in (x.split("=") for x in line[1:])}
            elif line[0] == "ktok":
                ktok[int(line[1])] = {int(a): float(b) for a, b in (x.split("=") for x in line[2:])}
            elif line[0] == "score":
                scores[int(line[1])] = float(line[2])
            elif line[0] == "select":
                sel[int(line[1])] = [int(x) for x in line[2:]]
    return cfg, q, ktok, scores, sel


def test_golden_selection():
    """The hand-worked fixture: exact FP64 scores, the kept sets for every
    listed top_k (near-ties decided by the 2^-20 term, exact ties by age)."""
    cfg, qd, ktok, scores, sel = _fixture()
    L, n4 = cfg["L"], cfg["n_int4"]
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=2, quant_bits=8)
    oc.set_n_int4(np.array([n4], np.int32))
    k = np.zeros((1, L, 1, D), np.float32)
    for p, vals in ktok.items():
        for ch, val in vals.items():
            k[0, p, 0, ch] = val
    v = np.random.default_rng(21).standard_normal((1, L, 1, D)).astype(np.float16)
    oc.append(np.array([L], np.int32), k.astype(np.float16), v)
    q = np.zeros((1, 1, D), np.float32)
    for ch, val in qd.items():
        q[0, 0, ch] = val
    q = q.astype(np.float16)
    assert float(q[0, 0, 1]) == 2.0 ** -20  # exact in FP16
    got = oc.l2_scores(q, 1.0, 0, 0)
    assert got.shape == (64,)
    for p in range(64):
        assert got[p] == scores.get(p, 0.0), (p, got[p])
    K, V = _dense_kv(oc, 0, L)
    for kk, want in sel.items():
        keep = want + list(range(64, L))
        ref, ref_l = _attend(q[0, 0], K, V, keep, 1.0, 0)
        out, lse = oc.decode(q, 1.0, top_k=kk)
        assert np.abs(out[0, 0] - ref).max() < 1e-12 and abs(lse[0, 0] - ref_l) < 1e-12, kk
        # the same rows through an explicit selection
        out2, lse2 = oc.decode(q, 1.0, sel=[want])
        assert np.array_equal(out2, out) and np.array_equal(lse2, lse), kk
    # a wrong set (the fixed-point answer for top_k = 2) gives another output
    wrong, _ = _attend(q[0, 0], K, V, [5, 9] + list(range(64, L)), 1.0, 0)
    out, _ = oc.decode(q, 1.0, top_k=2)
    assert np.abs(out[0, 0] - wrong).max() > 1e-3


@pytest.mark.parametrize("seed,qbits,hkv,hq,scale", [(0, 8, 1, 2, 0.088), (1, 8, 2, 8, 1.0), (2, 4, 1, 4, 0.3),
                                                     (3, 8, 1, 1, -0.5)])
def test_selection_matches_brute_force(seed, qbits, hkv, hq, scale):
    """Random caches: the kept set is numpy's top_k of numpy logits on K
    rebuilt position by position (ties, which random data does not produce,
    would go to the older position), for several top_k; the output is dense
    softmax attention over that set."""
    L = 350
    n4 = 3
    oc = _cache(L, n4, hkv=hkv, hq=hq, qbits=qbits, seed=10 + seed)
    q = np.random.default_rng(40 + seed).standard_normal((1, hq, D)).astype(np.float16)
    K, V = _dense_kv(oc, 0, L)
    n2 = min(L - 32, (n4 if qbits == 8 else 99) * BLOCK)
    g = hq // hkv
    for kk in (0, 1, 5, 40, n2 - 1):
        out, lse = oc.decode(q, scale, top_k=kk)
        for h in range(hq):
            z = scale * (K[:n2, h // g, :] @ q[0, h].astype(np.float64))
            order = np.lexsort((np.arange(n2), -z))
            keep = sorted(order[:kk].tolist()) + list(range(n2, L))
            want, wl = _attend(q[0, h], K, V, keep, scale, h // g)
            assert np.abs(out[0, h] - want).max() < 1e-12 and abs(lse[0, h] - wl) < 1e-12, (kk, h)
            sc = oc.l2_scores(q, scale, 0, h)
            assert np.allclose(sc, z, rtol=0, atol=1e-12)


def test_selection_rejects_bad_sets():
    oc = _cache(300, 2, seed=9)
    q = np.random.default_rng(3).standard_normal((1, 1, D)).astype(np.float16)
    for bad in ([200], [3, 3], [-1]):
        with pytest.raises(ValueError):
            oc.decode(q, 0.1, sel=[bad])
