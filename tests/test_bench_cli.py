"""bench.py's command line and the JSON fields it derives on the host (no GPU):
every cold-format, hot-size and block-size variant parses, and its
configuration object names the workload by what it is."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from int8_paged_kv_hybrid_b200 import synth  # noqa: E402


@pytest.mark.parametrize("argv", [
    [], ["--quant-bits", "0"], ["--quant-bits", "4"], ["--hot-tokens", "16"], ["--hot-tokens", "128"],
    ["--block-size", "32"], ["--block-size", "128"], ["--sparse-top-k", "-1"], ["--migrate"],
    ["--lean", "--steps", "3", "--warmup", "1"], ["--impl", "reference", "--gpus", "2"],
])
def test_arguments_parse(argv, monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
    a = bench.parse()
    assert a.steps > 0 and a.warmup >= 0


@pytest.mark.parametrize("qb,hot,blk", [(8, 32, 64), (0, 64, 64), (4, 16, 32), (8, 128, 128)])
def test_config_object(qb, hot, blk):
    w = synth.make_workload(2)
    w.hot_tokens, w.block_size = hot, blk
    bench.room_for_growth(w, 0)
    cfg = bench.workload_config(w, 0, 6, qb)
    json.dumps(cfg)
    assert cfg["hot_tokens"] == hot and cfg["block_size"] == blk and cfg["quant_bits"] == qb
    assert "llama3-8b" in cfg["workload"] and "%d-token blocks" % blk in cfg["workload"]
    # every sequence has a physical block for each of its cold blocks
    need = w.cold_blocks()
    assert all((w.block_table[b, :need[b]] >= 0).all() for b in range(w.batch))


def test_split_descriptions():
    """The configuration's split text says what the launched kernel does: runs
    of the split length on the one-CTA-per-split kernels, near-equal splits of
    at most that length per sequence on the persistent one, at least n
    near-equal splits for split_tokens = -n."""
    assert bench.split_desc(0, 384, 6) == "automatic: 6 splits of 384 tokens"
    assert bench.split_desc(512, 512, 5) == "5 splits of 512 tokens"
    d = bench.split_desc(0, 2048, 4, persistent=True)
    assert d.startswith("automatic: ") and "near-equal" in d and "<= 2048 tokens" in d
    d = bench.split_desc(-64, 2048, 65, persistent=True)
    assert "at least 64 near-equal splits" in d and "65 splits" in d


def test_launch_kinds_are_known():
    """Every launch kind the library reports has a kernel name and a launch
    count in the bench, and the persistent ones are told apart by name."""
    from int8_paged_kv_hybrid_b200 import _lib
    for kind in _lib.KERNEL_NAMES.values():
        assert kind in bench.DECODE_KERNELS and kind in bench.DECODE_LAUNCHES
        assert bench.is_persistent(kind) == kind.startswith("persistent")
        cfg = bench.workload_config(synth.make_workload(3), 0, 4, 8, 2048, persistent=bench.is_persistent(kind))
        assert ("near-equal" in cfg["splits"]) == bench.is_persistent(kind)
