"""Pins of the oracle's quantizer / append against values fixed outside it.

Source of the rule: web page "DeepSeek V4混合式KV Cache推理优化实战解析",
sections 2.1, 3.1, 3.2, 4.2.  The pins are hand-worked fixtures
(tests/golden/), the textbook absmax quantizer written with numpy for the
special case of blocks sealed whole in one call, and invariants.
"""
import numpy as np
import pytest

import oracle
from golden_cases import HOT, D, parse_cases, token_arrays
from int8_paged_kv_hybrid_b200 import synth


def _run_case(case, check_bytes=False):
    qb = case["quant_bits"]
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=2, quant_bits=qb)
    pos = 0
    for op, arg in case["ops"]:
        if op == "append":
            k, v = token_arrays(case, pos, arg)
            oc.append(np.array([arg], np.int32), k, v)
            pos += arg
        else:
            q, codes, sc = oc.get_block(0, int(arg["block"]))
            assert q == (127 if qb == 8 else 7)
            kv = {"K": 0, "V": 1}[arg["kv"]]
            if "scale" in arg:
                assert sc[0, kv] == np.float32(float(arg["scale"])), (arg, sc)
            if arg["codes"] is not None:
                slot = int(arg["slot"])
                for ch in range(D):
                    want = arg["codes"].get(ch, 0)
                    assert codes[0, kv, slot, ch] == want, (arg, ch, codes[0, kv, slot, :12])
    return oc


@pytest.mark.parametrize("name", ["int8_first_write", "int4_first_write"])
def test_golden_first_write(name):
    _run_case(parse_cases("quant_first_write.txt")[name])


def test_golden_requant_growth():
    _run_case(parse_cases("quant_requant.txt")["int8_requant"])


@pytest.mark.parametrize("name", ["int8_first_write", "int4_first_write"])
def test_golden_physical_bytes(name):
    """Export writes the documented byte layout (hand-derived offsets)."""
    case = parse_cases("quant_first_write.txt")[name]
    oc = _run_case(case)
    phys = 1
    bt = np.array([[phys, 0]], np.int32)
    ex = oc.export(bt, num_phys=2)
    for kv, off, val in parse_cases("physical_format.txt")[name]["bytes"]:
        assert ex["cold"][phys, 0, kv, off] == val, (kv, off, hex(ex["cold"][phys, 0, kv, off]))
    # scales land at [phys][head][K|V]
    q, _, sc = oc.get_block(0, 0)
    assert np.array_equal(ex["scales"][phys, 0], sc[0])
    assert not ex["cold"][0].any()


def _textbook_quant(x, q):
    """Symmetric absmax quantization of one whole block (numpy, FP32)."""
    x = x.astype(np.float32)
    a = np.float32(np.abs(x).max())
    s = np.float32(a / np.float32(q))
    if s == 0:
        return np.zeros(x.shape, np.int8), s
    c = np.clip(np.rint(x / s), -q, q).astype(np.int8)
    return c, s


@pytest.mark.parametrize("qbits", [8, 4])
def test_whole_block_matches_textbook(qbits):
    """One append of 32 + 64*nb tokens seals nb whole blocks in single groups:
    each must equal textbook absmax quantization of its 64 tokens."""
    rng = np.random.default_rng(7)
    nb, hkv = 3, 2
    n = HOT + 64 * nb
    k = (rng.standard_normal((1, n, hkv, D)) * 3).astype(np.float16)
    v = (rng.standard_normal((1, n, hkv, D)) * 0.1).astype(np.float16)
    k[0, 5, 1, 17] = 40.0  # an outlier that sets one block's scale
    oc = oracle.OracleCache(1, hkv, hkv, max_blocks_per_seq=nb, quant_bits=qbits)
    oc.append(np.array([n], np.int32), k, v)
    qmax = 127 if qbits == 8 else 7
    for i in range(nb):
        q, codes, sc = oc.get_block(0, i)
        assert q == qmax
        for h in range(hkv):
            for kv, src in ((0, k), (1, v)):
                want_c, want_s = _textbook_quant(src[0, 64 * i:64 * (i + 1), h, :], qmax)
                assert sc[h, kv] == want_s
                assert np.array_equal(codes[h, kv], want_c)
    # the newest 32 stay in the hot ring, FP16 bits unchanged, slot = pos % 32
    ring = oc.ring(0)
    for p in range(n - HOT, n):
        assert np.array_equal(ring[:, p % HOT, 0].view(np.uint16), k[0, p].view(np.uint16))
        assert np.array_equal(ring[:, p % HOT, 1].view(np.uint16), v[0, p].view(np.uint16))


def test_invariants_random_schedule():
    """Random append schedules (1..70 tokens per call): codes stay in [-Q, Q];
    the sealed positions reproduce their inputs within half a step of the
    block's final scale plus the accumulated re-quantization error; every
    block that was written in one group hits +-Q at its absmax element."""
    rng = np.random.default_rng(11)
    hkv, hq, B = 2, 4, 3
    total = np.array([300, 77, 33])
    oc = oracle.OracleCache(B, hkv, hq, max_blocks_per_seq=5, quant_bits=8)
    oc.set_n_int4(np.array([1, 0, 0], np.int32))
    hist_k = [[] for _ in range(B)]
    cur = np.zeros(B, np.int64)
    while (cur < total).any():
        n = np.minimum(rng.integers(1, 71, size=B), total - cur)
        mx = int(n.max())
        k = (rng.standard_normal((B, mx, hkv, D))).astype(np.float16)
        v = (rng.standard_normal((B, mx, hkv, D))).astype(np.float16)
        oc.append(n.astype(np.int32), k, v)
        for b in range(B):
            hist_k[b].append(k[b, :n[b]])
        cur += n
    assert np.array_equal(oc.lens(), total.astype(np.int32))
    for b in range(B):
        allk = np.concatenate(hist_k[b], axis=0)
        cold = max(0, int(total[b]) - HOT)
        for i in range((cold + 63) // 64):
            q, codes, sc = oc.get_block(b, i)
            qmax = 7 if (b == 0 and i < 1) else 127
            assert q == qmax
            assert np.abs(codes.astype(int)).max() <= qmax
            sealed = min(64, cold - 64 * i)
            for h in range(hkv):
                x = allk[64 * i:64 * i + sealed, h, :].astype(np.float64)
                deq = codes[h, 0, :sealed].astype(np.float64) * float(sc[h, 0])
                # each re-quantization adds at most half a step of the then
                # current scale, which never exceeds the final one
                assert np.abs(deq - x).max() <= float(sc[h, 0]) * (0.5 * 64) + 1e-6
                assert np.abs(deq - x).max() <= 0.5 * np.abs(x).max() + 1e-6


def test_eviction_reads_ring_before_overwrite():
    """With L_old = 40 and one new token, position 8 leaves the hot zone from
    ring slot 8, which the new position 40 then reuses."""
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=2, quant_bits=8)
    n1 = 40
    k = np.zeros((1, n1, 1, D), np.float16)
    for p in range(n1):
        k[0, p, 0, :] = p  # every channel equals the position
    oc.append(np.array([n1], np.int32), k, k)
    _, codes, sc = oc.get_block(0, 0)
    # positions 0..7 sealed in one group: absmax 7 -> scale 7/127; code(p) = RNE(p*127/7)
    s = np.float32(7.0) / np.float32(127)
    for p in range(8):
        want = int(np.rint(np.float32(p) / s))
        assert codes[0, 0, p, 0] == want
    k2 = np.full((1, 1, 1, D), 99.0, np.float16)
    oc.append(np.array([1], np.int32), k2, k2)
    _, codes, sc = oc.get_block(0, 0)
    # position 8 (value 8) sealed: scale grows to 8/127; old codes re-quantized
    assert sc[0, 0] == np.float32(8.0) / np.float32(127)
    assert codes[0, 0, 8, 0] == 127
    ring = oc.ring(0)
    assert float(ring[0, 8, 0, 0]) == 99.0          # slot 8 now holds position 40
    assert float(ring[0, 9, 0, 0]) == 9.0           # position 9 still hot


def test_zero_and_rejected_appends():
    oc = oracle.OracleCache(2, 1, 1, max_blocks_per_seq=1, quant_bits=8)
    z = np.zeros((2, 4, 1, D), np.float16)
    oc.append(np.array([0, 4], np.int32), z, z)
    assert list(oc.lens()) == [0, 4]
    with pytest.raises(ValueError):
        oc.append(np.array([5, 0], np.int32), z, z)   # n > max_new
    with pytest.raises(ValueError):
        oc.append(np.array([-1, 0], np.int32), z, z)  # negative
    big = np.zeros((2, 100, 1, D), np.float16)
    with pytest.raises(ValueError):
        oc.append(np.array([0, 93], np.int32), big, big)  # 97 tokens > 32 hot + 64 cold
    assert list(oc.lens()) == [0, 4]                  # rejected calls change nothing


def test_half_conversion_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits[::97]])
    w = want[::97]
    fin = np.isfinite(w)
    assert np.array_equal(got[fin], w[fin])
    assert np.array_equal(np.isnan(got), np.isnan(w))
    assert oracle.half_to_double(0x3C00) == 1.0
    assert oracle.half_to_double(0x0001) == 2.0 ** -24
    assert oracle.half_to_double(0x7BFF) == 65504.0


def test_metadata_block_counts():
    """Cold block count for a 32K context matches the page's 512 (section 5.4)."""
    import os
    from golden_cases import GOLDEN
    for line in open(os.path.join(GOLDEN, "metadata_sizes.txt"), encoding="utf-8"):
        line = line.split("#", 1)[0].split()
        if not line:
            continue
        ctx, bs, nblk, hdr = map(int, line)
        assert -(-ctx // bs) == nblk and nblk * 16 == hdr
        if bs == 64:
            assert synth.cold_blocks_for(ctx) == nblk


def test_export_128_token_blocks_as_two_sub_blocks():
    """block_size 128 in the device format: slot t of a block is slot t % 64
    of sub-block t // 64 (each sub-block a 64-slot K tile + V tile of the
    64-token format); one scale pair per block."""
    rng = np.random.default_rng(12)
    L = 32 + 200
    oc = oracle.OracleCache(1, 2, 2, max_blocks_per_seq=2, quant_bits=8, block=128)
    k = rng.standard_normal((1, L, 2, D)).astype(np.float16)
    v = rng.standard_normal((1, L, 2, D)).astype(np.float16)
    oc.append(np.array([L], np.int32), k, v)
    table = np.array([[3, 1]], np.int32)
    ex = oc.export(table, 4)
    cold = ex["cold"].reshape(4, 2, 2, 2, 64 * D)  # [phys][h][sub-block][K|V][8192]
    for i, phys in enumerate(table[0]):
        _, codes, sc = oc.get_block(0, i)
        assert np.array_equal(ex["scales"][phys], sc)
        n = min(128, L - 32 - 128 * i)
        for t in range(n):
            sb, s = divmod(t, 64)
            kt = cold[phys, :, sb, 0].view(np.int8)
            vt = cold[phys, :, sb, 1].view(np.int8)
            assert np.array_equal(kt[:, s * D:(s + 1) * D], codes[:, 0, t])
            for ch in (0, 5, 77, 127):
                off = ch * 64 + (((s // 16) ^ ((ch // 2) % 4)) * 16) + s % 16
                assert np.array_equal(vt[:, off], codes[:, 1, t, ch])


def test_export_32_token_blocks_in_half_a_tile():
    """block_size 32 in the device format: a block uses slots 0..31 of one
    64-slot K/V tile pair (16 KB per block and kv head); one scale pair per
    32 tokens; slots 32..63 stay untouched."""
    rng = np.random.default_rng(13)
    L = 32 + 80
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=3, quant_bits=8, block=32)
    k = rng.standard_normal((1, L, 1, D)).astype(np.float16)
    v = rng.standard_normal((1, L, 1, D)).astype(np.float16)
    oc.append(np.array([L], np.int32), k, v)
    # one scale per 32 sealed tokens: the textbook absmax quantizer per block
    for i in range(2):
        _, codes, sc = oc.get_block(0, i)
        grp = k[0, 32 * i:32 * i + 32, 0].astype(np.float32)
        assert sc[0, 0] == np.float32(np.abs(grp).max()) / np.float32(127)
    table = np.array([[2, 0, 1]], np.int32)
    ex = oc.export(table, 3)
    cold = ex["cold"].reshape(3, 1, 2, 64 * D)
    for i, phys in enumerate(table[0][:3]):
        _, codes, sc = oc.get_block(0, i)
        n = min(32, L - 32 - 32 * i)
        kt = cold[phys, 0, 0].view(np.int8)
        vt = cold[phys, 0, 1].view(np.int8)
        for t in range(n):
            assert np.array_equal(kt[t * D:(t + 1) * D], codes[0, 0, t])
            for ch in (0, 9, 127):
                assert vt[ch * 64 + (((t // 16) ^ ((ch // 2) % 4)) * 16) + t % 16] == codes[0, 1, t, ch]
        assert not kt[32 * D:].any()  # the tile's upper 32 slots are never written
