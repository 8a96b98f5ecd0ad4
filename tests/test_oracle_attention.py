"""Pins of the oracle's FP64 decode attention and LSE combine.

Source: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 4.2
(hot zone attended in FP16, cold zone dequantized, one output per query) and
section 2.1 (the hot zone is the most recent 32 tokens).  Pins: dense
brute-force softmax attention (scipy) on explicit K/V arrays rebuilt by the
test from positions, closed-form special cases (one-hot softmax, constant V,
all-hot context, GQA head mapping) and the split/merge identity of softmax.
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from golden_cases import HOT, D


def _fill(oc, rng, total, hkv, max_step=70, kscale=1.0, vscale=1.0):
    B = len(total)
    cur = np.zeros(B, np.int64)
    hk, hv = [[] for _ in range(B)], [[] for _ in range(B)]
    while (cur < total).any():
        n = np.minimum(rng.integers(1, max_step + 1, size=B), total - cur)
        mx = max(1, int(n.max()))
        k = (rng.standard_normal((B, mx, hkv, D)) * kscale).astype(np.float16)
        v = (rng.standard_normal((B, mx, hkv, D)) * vscale).astype(np.float16)
        oc.append(n.astype(np.int32), k, v)
        for b in range(B):
            hk[b].append(k[b, :n[b]])
            hv[b].append(v[b, :n[b]])
        cur += n
    return [np.concatenate(x, 0) for x in hk], [np.concatenate(x, 0) for x in hv]


def _dense_kv(oc, b, L):
    """Rebuild K, V [L][hkv][D] (float64) position by position: the newest
    oc.hot from the hot ring (slot p % hot), older ones as code * scale of
    block p//64, slot p%64."""
    K = np.zeros((L, oc.hkv, D))
    V = np.zeros((L, oc.hkv, D))
    ring = oc.ring(b).astype(np.float64)
    H = oc.hot
    cold = max(0, L - H)
    blocks = {}
    for p in range(L):
        if p >= cold:
            K[p] = ring[:, p % H, 0]
            V[p] = ring[:, p % H, 1]
        else:
            i = p // oc.block
            if i not in blocks:
                blocks[i] = oc.get_block(b, i)
            _, codes, sc = blocks[i]
            K[p] = codes[:, 0, p % oc.block].astype(np.float64) * sc[:, 0:1].astype(np.float64)
            V[p] = codes[:, 1, p % oc.block].astype(np.float64) * sc[:, 1:2].astype(np.float64)
    return K, V


def _brute(q, K, V, scale, g):
    hq = q.shape[0]
    out = np.zeros((hq, D))
    lse = np.zeros(hq)
    for h in range(hq):
        z = scale * (K[:, h // g, :] @ q[h].astype(np.float64))
        out[h] = softmax(z) @ V[:, h // g, :]
        lse[h] = logsumexp(z)
    return out, lse


@pytest.mark.parametrize("hkv,g,qbits", [(1, 1, 8), (2, 4, 8), (1, 4, 4), (2, 1, 8)])
def test_brute_force_tiny(hkv, g, qbits):
    rng = np.random.default_rng(100 + hkv * 10 + g + qbits)
    total = np.array([200, 1, 32, 33, 97, 0])
    B = len(total)
    oc = oracle.OracleCache(B, hkv, hkv * g, max_blocks_per_seq=4, quant_bits=qbits)
    oc.set_n_int4(np.array([1, 0, 0, 0, 1, 0], np.int32))
    _fill(oc, rng, total, hkv)
    q = rng.standard_normal((B, hkv * g, D)).astype(np.float16)
    scale = 1.0 / np.sqrt(D)
    out, lse = oc.decode(q, scale, nthreads=2)
    for b in range(B):
        L = int(total[b])
        if L == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        K, V = _dense_kv(oc, b, L)
        o2, l2 = _brute(q[b], K, V, scale, g)
        assert np.abs(out[b] - o2).max() < 1e-12
        assert np.abs(lse[b] - l2).max() < 1e-12


@pytest.mark.parametrize("hot", [16, 64, 128])
def test_brute_force_other_hot_sizes(hot):
    """hot_tokens 16 / 64 / 128 (the contract's other powers of two): the
    newest `hot` tokens stay FP16, the rest is sealed into blocks."""
    rng = np.random.default_rng(200 + hot)
    total = np.array([300, 1, hot - 1, hot, hot + 1, hot + 64, 0])
    B, hkv, g = len(total), 2, 4
    oc = oracle.OracleCache(B, hkv, hkv * g, max_blocks_per_seq=5, hot=hot)
    ks, vs = _fill(oc, rng, total, hkv)
    q = rng.standard_normal((B, hkv * g, D)).astype(np.float16)
    scale = 1.0 / np.sqrt(D)
    out, lse = oc.decode(q, scale, nthreads=2)
    for b in range(B):
        L = int(total[b])
        if L == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        # the hot ring holds exactly the newest min(L, hot) inputs
        ring = oc.ring(b)
        for p in range(max(0, L - hot), L):
            assert np.array_equal(ring[:, p % hot, 0], ks[b][p]) and np.array_equal(ring[:, p % hot, 1], vs[b][p])
        # sealed blocks: one per started 64 tokens of the cold range
        nb = (max(0, L - hot) + 63) // 64
        assert [oc.get_block(b, i)[0] != 0 for i in range(5)] == [i < nb for i in range(5)]
        K, V = _dense_kv(oc, b, L)
        if L <= hot:  # nothing quantized: plain attention on the inputs
            assert np.array_equal(K, ks[b].astype(np.float64)) and np.array_equal(V, vs[b].astype(np.float64))
        o2, l2 = _brute(q[b], K, V, scale, g)
        assert np.abs(out[b] - o2).max() < 1e-12
        assert np.abs(lse[b] - l2).max() < 1e-12


@pytest.mark.parametrize("qbits,blk", [(8, 128), (4, 128), (8, 32), (4, 32)])
def test_brute_force_other_block_sizes(qbits, blk):
    """block_size 128 / 32: one scale per block of sealed tokens (the textbook
    absmax quantizer over the whole group when it is sealed in one call),
    attention equal to dense brute force."""
    rng = np.random.default_rng(300 + qbits + blk)
    total = np.array([32 + blk, 32 + 300, 5, 0])
    B, hkv, g = len(total), 2, 4
    oc = oracle.OracleCache(B, hkv, hkv * g, max_blocks_per_seq=300 // blk + 1, quant_bits=qbits, block=blk)
    k = rng.standard_normal((B, 332, hkv, D)).astype(np.float16)
    v = rng.standard_normal((B, 332, hkv, D)).astype(np.float16)
    oc.append(total.astype(np.int32), k, v)
    Q = 127 if qbits == 8 else 7
    # sequence 0: exactly one full block, sealed in one call
    _, codes, sc = oc.get_block(0, 0)
    for h in range(hkv):
        for kv, x in ((0, k), (1, v)):
            grp = x[0, :blk, h].astype(np.float32)
            s = np.float32(np.abs(grp).max()) / np.float32(Q)
            assert sc[h, kv] == s
            want = np.clip(np.rint(grp / s), -Q, Q)
            assert np.array_equal(codes[h, kv, :blk], want)
    q = rng.standard_normal((B, hkv * g, D)).astype(np.float16)
    out, lse = oc.decode(q, 0.088, nthreads=2)
    for b in range(B):
        L = int(total[b])
        if L == 0:
            continue
        K, V = _dense_kv(oc, b, L)
        o2, l2 = _brute(q[b], K, V, 0.088, g)
        assert np.abs(out[b] - o2).max() < 1e-12 and np.abs(lse[b] - l2).max() < 1e-12


def test_pairs_subset_matches_full():
    rng = np.random.default_rng(5)
    total = np.array([150, 90])
    oc = oracle.OracleCache(2, 2, 8, max_blocks_per_seq=2)
    _fill(oc, rng, total, 2)
    q = rng.standard_normal((2, 8, D)).astype(np.float16)
    full, lf = oc.decode(q, 0.3)
    part, lp = oc.decode(q, 0.3, pairs=[(1, 5), (0, 0)])
    assert np.array_equal(part[1, 5], full[1, 5]) and np.array_equal(part[0, 0], full[0, 0])
    assert lp[1, 5] == lf[1, 5]
    assert np.isnan(part[0, 1]).all()


def test_all_hot_equals_unquantized_attention():
    """L <= 32: nothing is quantized; the result is plain softmax attention on
    the FP16 inputs (section 3.1: the hot zone is never quantized)."""
    rng = np.random.default_rng(9)
    for L in (1, 5, 31, 32):
        k = rng.standard_normal((1, L, 2, D)).astype(np.float16)
        v = rng.standard_normal((1, L, 2, D)).astype(np.float16)
        oc = oracle.OracleCache(1, 2, 8, max_blocks_per_seq=1)
        oc.append(np.array([L], np.int32), k, v)
        q = rng.standard_normal((1, 8, D)).astype(np.float16)
        out, lse = oc.decode(q, 0.125)
        o2, l2 = _brute(q[0], k[0].astype(np.float64), v[0].astype(np.float64), 0.125, 4)
        assert np.abs(out[0] - o2).max() < 1e-13
        assert np.abs(lse[0] - l2).max() < 1e-13


def test_one_hot_softmax_returns_chosen_row():
    """K_j = 8 e_j (one channel per position), q = 20 e_j*: the logit of j* is
    160 above all others, so the output is V_j* (dequantized if cold) to
    within e^-160."""
    L = 100
    k = np.zeros((1, L, 1, D), np.float16)
    for j in range(L):
        k[0, j, 0, j] = 8.0
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, L, 1, D)).astype(np.float16)
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=2)
    oc.append(np.array([L], np.int32), k, v)
    Kd, Vd = _dense_kv(oc, 0, L)
    for jstar in (3, 50, 67, 80, 99):   # cold block 0, cold block 1, hot
        q = np.zeros((1, 1, D), np.float16)
        q[0, 0, jstar] = 20.0
        out, lse = oc.decode(q, 1.0)
        assert np.abs(out[0, 0] - Vd[jstar, 0]).max() < 1e-12
        assert abs(lse[0, 0] - 20.0 * Kd[jstar, 0, jstar]) < 1e-9


def test_constant_v_returns_constant():
    """Every V row equal to u with u = k * 0.125, k integer in [-127, 127]
    and max|k| = 127: each block's scale is exactly 0.125 and its codes
    exactly k, so the output is u in FP64 whatever the logits."""
    rng = np.random.default_rng(4)
    kint = rng.integers(-127, 128, size=D)
    kint[7] = 127
    u = (kint * 0.125).astype(np.float16)
    L = 300
    kk = rng.standard_normal((1, L, 1, D)).astype(np.float16)
    vv = np.broadcast_to(u, (1, L, 1, D)).astype(np.float16)
    oc = oracle.OracleCache(1, 1, 4, max_blocks_per_seq=5)
    cur = 0
    for n in (33, 1, 64, 100, 2, 100):
        oc.append(np.array([n], np.int32), kk[:, cur:cur + n], vv[:, cur:cur + n])
        cur += n
    assert cur == L
    q = rng.standard_normal((1, 4, D)).astype(np.float16)
    out, _ = oc.decode(q, 1.0)
    assert np.abs(out[0] - u.astype(np.float64)[None, :]).max() < 1e-12


def test_gqa_head_mapping():
    """Query head h reads kv head h // (Hq/Hkv): with kv head 0's V = 15.875
    and kv head 1's V = -15.875 everywhere (127 * 0.125, so cold blocks hold
    them exactly), q heads 0-3 give 15.875 and heads 4-7 give -15.875."""
    L = 150
    rng = np.random.default_rng(6)
    k = rng.standard_normal((1, L, 2, D)).astype(np.float16)
    v = np.zeros((1, L, 2, D), np.float16)
    v[:, :, 0] = 15.875
    v[:, :, 1] = -15.875
    oc = oracle.OracleCache(1, 2, 8, max_blocks_per_seq=2)
    oc.append(np.array([L], np.int32), k, v)
    q = rng.standard_normal((1, 8, D)).astype(np.float16)
    out, _ = oc.decode(q, 0.1)
    assert np.abs(out[0, :4] - 15.875).max() < 1e-12
    assert np.abs(out[0, 4:] + 15.875).max() < 1e-12


def test_mha_is_gqa_with_one_group():
    """Hq = Hkv: replicating each kv head 4x as its own kv head gives the same
    output as GQA with g = 4."""
    rng = np.random.default_rng(8)
    L = 130
    k = rng.standard_normal((1, L, 2, D)).astype(np.float16)
    v = rng.standard_normal((1, L, 2, D)).astype(np.float16)
    gqa = oracle.OracleCache(1, 2, 8, max_blocks_per_seq=2)
    gqa.append(np.array([L], np.int32), k, v)
    mha = oracle.OracleCache(1, 8, 8, max_blocks_per_seq=2)
    mha.append(np.array([L], np.int32), np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2))
    q = rng.standard_normal((1, 8, D)).astype(np.float16)
    o1, l1 = gqa.decode(q, 0.2)
    o2, l2 = mha.decode(q, 0.2)
    assert np.abs(o1 - o2).max() < 1e-14 and np.abs(l1 - l2).max() < 1e-12


def test_combine_split_identity():
    """Softmax over a set equals the LSE-weighted merge of softmaxes over a
    partition of it (with empty parts at lse = -inf)."""
    rng = np.random.default_rng(12)
    rows, L = 5, 257
    z = rng.standard_normal((rows, L)) * 3
    V = rng.standard_normal((L, D))
    full = softmax(z, axis=1) @ V
    full_lse = logsumexp(z, axis=1)
    cuts = [0, 10, 10, 128, 200, 257]       # one empty split
    S = len(cuts) - 1
    o_part = np.zeros((rows, S, D))
    l_part = np.full((rows, S), -np.inf)
    for s in range(S):
        a, b = cuts[s], cuts[s + 1]
        if b > a:
            o_part[:, s] = softmax(z[:, a:b], axis=1) @ V[a:b]
            l_part[:, s] = logsumexp(z[:, a:b], axis=1)
    out, lse = oracle.combine(o_part, l_part)
    assert np.abs(out - full).max() < 1e-13
    assert np.abs(lse - full_lse).max() < 1e-12
    # a single split is the identity; all-empty gives zeros and -inf
    o1, l1 = oracle.combine(o_part[:, 3:4], l_part[:, 3:4])
    assert np.array_equal(o1, o_part[:, 3]) and np.array_equal(l1, l_part[:, 3])
    o0, l0 = oracle.combine(np.zeros((2, 3, D)), np.full((2, 3), -np.inf))
    assert not o0.any() and np.isneginf(l0).all()
