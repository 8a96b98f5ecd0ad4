"""The multi-GPU path of bench.py is replicas only (an independent batch per
rank, no data-path collective); its host logic runs here as world-size-2
gloo ranks on the CPU: the slowest rank's time is what every rank reports,
the whole-job rate counts every rank's bytes, ranks get different seeded
inputs of the same shapes, and the reference arm under torchrun prints one
line from rank 0 while the other rank exits cleanly."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from int8_paged_kv_hybrid_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's own time; every rank must end up with the slowest one
        ms = bench.max_over_ranks(1.0 + 2.5 * rank, world)
        # replicas: seeded per rank, same shapes
        w = synth.make_workload(1, seed_offset=1000 * rank)
        q = torch.from_numpy(synth.query(w).astype(np.float32))
        qs = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(qs, q)
        same_data = bool(torch.equal(qs[0], qs[1]))
        out.put((rank, ms, tuple(q.shape), same_data))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_max_time_and_replicas():
    ctx = mp.get_context("spawn")
    port = _free_port()
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [3.5, 3.5]           # max over ranks, on both
    assert res[0][2] == res[1][2]                      # same shapes
    assert res[0][3] is False                          # different inputs per rank


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 34.2 MB per rank in 0.025 ms, 4 ranks: 4 x 34.2e6 B / 25e-6 s
    assert abs(bench.job_throughput(34.2e6, 4, 0.025) - 4 * 34.2e6 / 25e-6 / 1e9) < 1e-9
    assert bench.max_over_ranks(7.0, 1) == 7.0


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "1"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
