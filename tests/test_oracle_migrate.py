"""Pins of the oracle's tier migration and migration policy.

Source: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 3.3 (a
cold block moves between the INT8 "L1" and the INT4 "L2" tier; the adaptive
threshold 3000 * (1 + 0.2 * load_factor) ms with load_factor = geometric mean
of the batch's sequence lengths / 512; promotion below the threshold,
demotion above 1.5 x the threshold) and section 3.2 (the moved block gets a
new scale).  Pins: hand-worked fixtures (tests/golden/), closed forms, the
quantization error bound and invariants.
"""
import math
import os

import numpy as np
import pytest

import oracle
from golden_cases import GOLDEN, D, parse_cases, token_arrays
from int8_paged_kv_hybrid_b200 import synth


def _run_case(case):
    oc = oracle.OracleCache(1, 1, 1, max_blocks_per_seq=2, quant_bits=case["quant_bits"])
    pos = 0
    for op, arg in case["ops"]:
        if op == "append":
            k, v = token_arrays(case, pos, arg)
            oc.append(np.array([arg], np.int32), k, v)
            pos += arg
        elif op == "migrate":
            oc.migrate(np.array([arg], np.int32))
            assert oc.n_int4()[0] == arg
        else:
            q, codes, sc = oc.get_block(0, int(arg["block"]))
            kv = {"K": 0, "V": 1}[arg["kv"]]
            if "q" in arg:
                assert q == int(arg["q"]), (arg, q)
            if "scale" in arg:
                assert sc[0, kv] == np.float32(float(arg["scale"])), (arg, repr(sc[0, kv]))
            if arg["codes"] is not None:
                slot = int(arg["slot"])
                for ch in range(D):
                    want = arg["codes"].get(ch, 0)
                    assert codes[0, kv, slot, ch] == want, (arg, ch, codes[0, kv, slot, :8])


@pytest.mark.parametrize("name", ["int8_demote_promote", "empty_block_changes_tier"])
def test_golden_migration(name):
    _run_case(parse_cases("migrate_requant.txt")[name])


def test_golden_threshold():
    n = 0
    for line in open(os.path.join(GOLDEN, "migration_threshold.txt"), encoding="utf-8"):
        f = line.split("#", 1)[0].split()
        if not f:
            continue
        want, lens = float(f[0]), [int(x) for x in f[1:]]
        got = oracle.migration_threshold_ms(lens)
        assert abs(got - want) <= 1e-9 * want, (lens, got, want)
        n += 1
    assert n >= 8
    # the page's example: the geometric (not arithmetic) mean of its lengths
    assert abs(oracle.migration_threshold_ms([256, 1024, 512, 2048]) - (3000 + 600 * math.sqrt(2))) < 1e-9


def test_decision_boundaries():
    t = 3848.5
    assert oracle.migration_decision(t - 1e-6, t, True) == 1      # L2 block accessed often: up
    assert oracle.migration_decision(t, t, True) == 0             # strictly below
    assert oracle.migration_decision(100.0, t, False) == 0        # L1 stays L1 when hot
    assert oracle.migration_decision(1.5 * t + 1e-6, t, False) == -1
    assert oracle.migration_decision(1.5 * t, t, False) == 0      # strictly above
    assert oracle.migration_decision(1e9, t, True) == 0           # L2 stays L2 when cold


def _random_cache(seed=7, lens=(700, 1500, 33, 0, 130), hkv=2):
    w = synth.custom_workload("mig", list(lens), 2 * hkv, hkv, seed=seed, max_step=64)
    oc = oracle.OracleCache(w.batch, w.num_kv_heads, w.num_q_heads, w.max_blocks)
    for si, n in enumerate(w.schedule):
        k, v = synth.step_tokens(w, si, n)
        oc.append(n, k, v)
    return w, oc


def test_requant_error_bound_and_full_range():
    """Every code moves by at most half a new step, and the block's largest
    value maps to +-Q' (the new scale is the absmax over Q')."""
    w, oc = _random_cache()
    before = {(b, i): oc.get_block(b, i) for b in range(w.batch) for i in range(w.max_blocks)}
    target = np.array([3, 0, 1, 2, 1], np.int32)
    oc.migrate(target)
    for b in range(w.batch):
        nblk = synth.cold_blocks_for(int(w.lens[b]))
        for i in range(w.max_blocks):
            q0, c0, s0 = before[(b, i)]
            q1, c1, s1 = oc.get_block(b, i)
            if i >= nblk:
                assert q0 == 0 and q1 == 0
                continue
            assert q1 == (7 if i < target[b] else 127)
            for h in range(w.num_kv_heads):
                for kv in range(2):
                    v0 = c0[h, kv].astype(np.float64) * np.float64(s0[h, kv])
                    v1 = c1[h, kv].astype(np.float64) * np.float64(s1[h, kv])
                    if q1 == q0:
                        assert np.array_equal(c0[h, kv], c1[h, kv]) and s0[h, kv] == s1[h, kv]
                        continue
                    assert np.abs(c1[h, kv]).max() <= q1
                    if s0[h, kv] > 0:
                        assert np.abs(c1[h, kv]).max() == q1
                        assert np.abs(v1 - v0).max() <= 0.5 * s1[h, kv] * (1 + 1e-5)
                    else:
                        assert s1[h, kv] == 0 and not c1[h, kv].any()
    assert np.array_equal(oc.n_int4(), target)


def test_round_trip_stays_within_int4_error():
    """Demote then promote: the block keeps its INT4 values to within half an
    INT8 step, and attention moves by at most the INT4 quantization noise."""
    w, oc = _random_cache(seed=11, lens=(900,), hkv=1)
    nblk = synth.cold_blocks_for(900)
    q = synth.query(w)
    ref, _ = oc.decode(q, w.softmax_scale)
    oc.migrate(np.array([nblk], np.int32))
    mid = [oc.get_block(0, i) for i in range(nblk)]
    out4, _ = oc.decode(q, w.softmax_scale)
    oc.migrate(np.array([0], np.int32))
    for i in range(nblk):
        q4, c4, s4 = mid[i]
        q8, c8, s8 = oc.get_block(0, i)
        assert q4 == 7 and q8 == 127
        for kv in range(2):
            v4 = c4[0, kv] * np.float64(s4[0, kv])
            v8 = c8[0, kv] * np.float64(s8[0, kv])
            assert np.abs(v8 - v4).max() <= 0.5 * s8[0, kv] * (1 + 1e-5)
    out8, _ = oc.decode(q, w.softmax_scale)
    # INT4 noise is ~18x INT8's: the demoted output differs visibly, the
    # promoted one keeps that difference (the precision is not recovered)
    d4 = np.abs(out4 - ref).max()
    assert 1e-4 < d4 < 0.2
    assert np.abs(out8 - out4).max() < 0.25 * d4


def test_invalid_target_changes_nothing():
    w, oc = _random_cache(lens=(300,), hkv=1)
    b0 = oc.get_block(0, 0)
    with pytest.raises(ValueError):
        oc.migrate(np.array([w.max_blocks + 1], np.int32))
    with pytest.raises(ValueError):
        oc.migrate(np.array([-1], np.int32))
    b1 = oc.get_block(0, 0)
    assert b0[0] == b1[0] and np.array_equal(b0[1], b1[1]) and np.array_equal(b0[2], b1[2])
    assert oc.n_int4()[0] == 0
