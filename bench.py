#!/usr/bin/env python
"""Benchmark of the hybrid_v2 decode path on B200.

One step = one pass of the whole hot path over one batch: hyb_decode_step,
i.e. the append of the step's token (hot-ring write + sealing of the token
that leaves the hot zone, with quantization) fused with split-KV attention
over the hot ring and the INT8 cold blocks and the log-sum-exp merge of its
splits, in one launch.

Default run (the line the driver reads): the headline is the long-context
workload (batch 4, L = 32K, 32K, 128K, 128K, Llama-3-8B attention shapes,
at least 64 splits per sequence), the largest single-GPU configuration; the same run
reports sub-records for the Llama-3-8B batch-8 L=2048 workload, the
variable-length batch of 64 and the Qwen2-7B mixed batch of 128 (each with
its own e2e and CPU baseline), an append-only record (one hyb_kv_append of
U[1,64] tokens per sequence on the variable-length batch) and the oracle's
one-thread time on the single-sequence workload.  Seeded synthetic N(0,1)
data throughout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload 1..5] [--lean] [--migrate] [--sparse-top-k K] ...

Prints one JSON line (rank 0).  With N > 1 (torchrun), every rank runs its
own batch (weak scaling, no data-path collective); times are the max over
ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn KV GB/s (frac of HBM peak) and tokens/s at 1 B200 vs CPU oracle"
UNIT = "GB/s"
HEADLINE = 4              # the largest single-GPU configuration
SUB_WORKLOADS = (2, 3, 5)  # reported in the same run
APPEND_WORKLOAD = 3
PROFILE_JSON = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
# the profiled kernel's sources (their hash tells whether a capture is current)
KERNEL_SOURCES = ["decode_kernel.cuh", "decode_persist.cuh", "decode_dev.cuh", "mma.cuh", "common.cuh",
                  "kernels.cuh"]
FLUSH_BYTES = 512 << 20   # > 126 MB L2
CLEAN_BYTES = 256 << 20   # read after the flush write: L2 holds no dirty line when the timed step starts
L2_NOTE = ("flushed between timed steps: a 512 MB write, then a read of another 256 MB buffer, so that the "
           "flush's dirty lines are written back before the timed step, not inside it")


class L2Flush:
    """Evicts everything from L2 between timed steps: writes a buffer larger
    than L2, then reads another one (the write-backs of the written lines
    happen during that read, outside the timed region)."""

    def __init__(self, torch, dev, enabled=True):
        self.sum = torch.sum
        self.w = torch.empty(FLUSH_BYTES if enabled else 0, dtype=torch.uint8, device=dev)
        self.r = torch.zeros((CLEAN_BYTES // 4) if enabled else 0, dtype=torch.int32, device=dev)
        self.acc = torch.zeros((), dtype=torch.int64, device=dev)

    def __call__(self):
        if self.w.numel():
            self.w.zero_()
            self.sum(self.r, 0, out=self.acc)


DECODE_KERNELS = {"persistent": "hyb::decode_persist_kernel", "split_cta": "hyb::decode_kernel",
                  "cluster": "hyb::decode_kernel (clusters)",
                  "persistent+combine": "hyb::decode_persist_kernel, then hyb::persist_combine_kernel"}
DECODE_LAUNCHES = {"persistent": 1, "split_cta": 1, "cluster": 1, "persistent+combine": 2}


def is_persistent(kind):
    """The launch kind (hyb_decode_launch_info's name) runs the persistent kernel."""
    return kind in ("persistent", "persistent+combine")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--split", type=int, default=0, help="split_tokens (0 = automatic)")
    p.add_argument("--workload", type=int, default=None,
                   help="1..5: measure this workload alone (default: the headline workload 4 plus the "
                        "sub-records of workloads 2, 3 and 5, the append record and the 1-thread oracle)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--migrate", action="store_true",
                   help="time hyb_kv_migrate instead of the decode step: demote a quarter of every "
                        "sequence's cold blocks to INT4 and promote them back (workload default 3)")
    p.add_argument("--quant-bits", type=int, default=8, choices=[8, 4, 0],
                   help="cold blocks: 8 (INT8, the default), 4 (all INT4) or 0 (FP16, quantization off)")
    p.add_argument("--hot-tokens", type=int, default=32, choices=[16, 32, 64, 128],
                   help="hot-zone tokens (32, the default, is the page's value)")
    p.add_argument("--block-size", type=int, default=64, choices=[32, 64, 128],
                   help="tokens per cold block (64, the default, is the page's value)")
    p.add_argument("--sparse-top-k", type=int, default=None,
                   help="time hyb_decode_attn_sparse with this top_k (-1: the page's rule min(128, L // 256)) "
                        "against the dense hyb_decode_attn on the same cache (workload default 4, the older "
                        "half of every sequence's cold blocks INT4)")
    p.add_argument("--lean", action="store_true",
                   help="profiling run: no state restore, L2 flush, e2e or CPU baseline")
    return p.parse_args()


COLD_KIND = {8: "INT8", 4: "INT4", 0: "FP16"}


def split_desc(split, split_len, ns, persistent=False):
    if split < 0:
        return ("per sequence: at least %d near-equal splits of <= 32 blocks (the longest sequence: %d splits "
                "of <= %d tokens)" % (-split, ns, split_len))
    head = "automatic: " if split == 0 else ""
    if persistent:
        # the persistent kernel cuts each sequence into near-equal splits of at most split_len tokens
        return "%seach sequence in near-equal splits of <= %d tokens (the longest: %d)" % (head, split_len, ns)
    return "%s%d splits of %d tokens" % (head, ns, split_len)


def workload_config(w, split, ns, qbits=8, split_len=None, persistent=False):
    lens = w.lens
    cold = COLD_KIND[qbits]
    if qbits == 8 and w.n_int4 is not None:
        cold = "INT8 (oldest quarter INT4)"
    H = w.hot_tokens
    if w.name == synth_name(2):
        what = ("llama3-8b decode attention, 1 layer: batch %d, Hq %d, Hkv %d, d 128, L %d (%d FP16 hot + "
                "%d %s cold in %d-token blocks), %d-block pool"
                % (w.batch, w.num_q_heads, w.num_kv_heads, int(lens[0]), H, int(lens[0]) - H, cold,
                   w.block_size, w.num_phys_blocks))
    else:
        what = ("decode attention, 1 layer: batch %d, Hq %d, Hkv %d, d 128, L %d..%d (mean %.0f), %d FP16 hot "
                "+ %s cold in %d-token blocks, %d-block pool"
                % (w.batch, w.num_q_heads, w.num_kv_heads, int(lens.min()), int(lens.max()), float(lens.mean()),
                   H, cold, w.block_size, w.num_phys_blocks))
    return {"workload": what, "batch": int(w.batch), "seq_len": int(lens.max()),
            "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads, "head_dim": 128, "hot_tokens": H,
            "block_size": w.block_size, "quant_bits": qbits, "split_tokens": split, "n_splits": ns,
            "splits": split_desc(split, split if split_len is None else split_len, ns, persistent),
            "step": "hyb_decode_step: append 1 token/seq + split-KV attention, one launch",
            "l2": L2_NOTE,
            "parallelism": "replicas (independent batch per GPU)"}


def max_over_ranks(x, world, device=None):
    """The largest x over all ranks (each rank passes its own); x itself with
    one rank.  A collective: every rank must call it, in the same order."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_throughput(bytes_per_rank, world, ms):
    """Whole-job GB/s: what every rank processed over the slowest rank's ms."""
    return bytes_per_rank * world / (ms * 1e-3) / 1e9


def synth_name(idx):
    from int8_paged_kv_hybrid_b200 import synth
    return synth.WORKLOAD_NAMES[idx]


def kernel_sha():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "int8_paged_kv_hybrid_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name):
    """(DRAM bytes per decode launch, how it was obtained) for this workload
    from the committed ncu figures (profiles/decode_kernel_traffic.json), if
    they were taken on the current kernel source; else (None, reason)."""
    try:
        with open(PROFILE_JSON, encoding="utf-8") as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None, "no committed ncu figures"
    if d.get("kernel_source_sha") != kernel_sha():
        return None, "committed ncu figures predate the current kernel source"
    rec = d.get("workloads", {}).get(workload_name)
    if not rec:
        return None, "no ncu figure for this workload"
    return float(rec["dram_bytes_per_launch"]), rec.get("how", "ncu")


def cpu_model():
    try:
        with open("/proc/cpuinfo", encoding="utf-8") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 10 ms; stop() summarises
    the samples taken after mark() (the timed region)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.t_mark = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), "--query-gpu=timestamp," + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def mark(self):
        self.t_mark = time.time()

    def stop(self):
        if self.proc is None:
            return None
        t_stop = time.time()
        time.sleep(0.05)
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        import datetime
        rows = []
        for line in text.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]), [x.lower() == "active" for x in f[6:10]]))
            except ValueError:
                continue
        if not rows:
            return None
        # samples taken from the start of the timed region on (nvidia-smi's
        # timestamps are wall-clock local time, as datetime parses them)
        t0 = self.t_mark or 0.0
        timed = [r for r in rows if t0 <= r[0] <= t_stop] or rows[-3:]
        sm = sorted(r[1] for r in timed)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in timed for i in range(4) if r[3][i]})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": rows[0][2], "reasons": reasons,
                "samples_timed": len(timed), "samples": len(rows)}


def room_for_growth(w, extra_tokens):
    """Give every sequence physical blocks for its tokens plus `extra_tokens`
    more: every missing table entry gets a spare pool block (or a new one past
    the pool), the table widened when needed.  For runs that let the cache
    grow, or whose hot or block size needs more blocks than the table has."""
    import numpy as np
    from int8_paged_kv_hybrid_b200 import synth
    need = [synth.cold_blocks_for(int(L) + extra_tokens, w.hot_tokens, w.block_size) for L in w.lens]
    width = max(w.max_blocks, max(need))
    bt = np.full((w.batch, width), -1, np.int32)
    bt[:, :w.max_blocks] = w.block_table
    used = set(int(x) for x in w.block_table[w.block_table >= 0])
    spare = [p for p in range(w.num_phys_blocks) if p not in used]
    nxt = w.num_phys_blocks
    for b in range(w.batch):
        for j in range(need[b]):
            if bt[b, j] < 0:
                if spare:
                    bt[b, j] = spare.pop(0)
                else:
                    bt[b, j] = nxt
                    nxt += 1
    w.block_table = bt
    w.num_phys_blocks = nxt


def build_gpu_state(w, torch, qbits=8, ora=None):
    """The library's cache for workload w, prefilled by the library's own
    appends (64-token calls) to one token short of w.lens; the oracle `ora`,
    if given, replays the very same calls.  Returns (cache, n_last, k_last, v_last, q): the step's inputs."""
    from int8_paged_kv_hybrid_b200 import HybridKVCache, synth
    cache = HybridKVCache(w.batch, w.num_kv_heads, w.num_q_heads, w.num_phys_blocks, w.max_blocks,
                          quant_bits=qbits, block_table=w.block_table,
                          n_int4=w.n_int4 if qbits == 8 else None, hot_tokens=w.hot_tokens,
                          block_size=w.block_size)
    sched = synth._chunk_schedule(w.lens, 64)
    for si, n in enumerate(sched[:-1]):
        k, v = synth.step_tokens(w, si, n, max_new=64)
        cache.append(torch.from_numpy(n).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        if ora is not None:
            ora.append(n, k, v)
    last = len(sched) - 1
    n_last = sched[-1]
    k_last, v_last = synth.step_tokens(w, last, n_last, max_new=1)
    q = synth.query(w)
    torch.cuda.synchronize()
    return cache, n_last, k_last, v_last, q


def new_oracle(w, qbits=8):
    import oracle
    ora = oracle.OracleCache(w.batch, w.num_kv_heads, w.num_q_heads, w.max_blocks + 16, qbits, hot=w.hot_tokens,
                             block=w.block_size)
    if qbits == 8 and w.n_int4 is not None:
        ora.set_n_int4(w.n_int4)
    return ora


def _touched_blocks(w, n_new, lens_new=None):
    """Physical blocks an append of n_new[b] tokens (reaching lens_new[b],
    default w.lens) can write: the blocks holding the positions that leave
    the hot zone."""
    import numpy as np
    lens_new = w.lens if lens_new is None else lens_new
    phys = []
    for b in range(w.batch):
        L_new = int(lens_new[b])
        L_old = L_new - int(n_new[b])
        e0, e1 = max(0, L_old - w.hot_tokens), max(0, L_new - w.hot_tokens)
        for i in range(e0 // w.block_size, (e1 + w.block_size - 1) // w.block_size):
            if e1 > e0:
                phys.append(int(w.block_table[b, i]))
    return np.array(sorted(set(phys)), np.int64)


class StateSnapshot:
    """What a step changes (hot ring, scales, lengths, the blocks it seals
    into), copied once and restored before every timed step, untimed."""

    def __init__(self, cache, touched, torch, dev):
        self.cache = cache
        self.touched = torch.from_numpy(touched).to(dev)
        self.snap = {"hot": cache.hot.clone(), "scales": cache.scales.clone(),
                     "seq_lens": cache.seq_lens.clone(), "cold": cache.cold.index_select(0, self.touched)}

    def restore(self):
        c, sn = self.cache, self.snap
        c.hot.copy_(sn["hot"])
        c.scales.copy_(sn["scales"])
        c.seq_lens.copy_(sn["seq_lens"])
        c.cold.index_copy_(0, self.touched, sn["cold"])


def time_events(n, stream, before, body):
    """n iterations of before() (untimed) then body() between two CUDA events
    on `stream`; returns the event pairs."""
    import torch
    evs = []
    for _ in range(n):
        before()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        body()
        e1.record(stream)
        evs.append((e0, e1))
    return evs


def mean_ms(evs):
    return sum(a.elapsed_time(b) for a, b in evs) / len(evs)


def read_floor(torch, dev, nbytes, stream, side, args, world):
    """Time hyb_stream_read over `nbytes` (rounded up to 16) the way the step is
    timed: a CUDA graph of the one launch, replayed between two events, L2
    flushed before each replay.  The result is the attainable time of any
    kernel that reads that many bytes once: no table lookup, no dependent load,
    no arithmetic, only the launch, the ramp-up and the drain."""
    from int8_paged_kv_hybrid_b200 import hyb_stream_read
    nb = (nbytes + 15) // 16 * 16
    buf = torch.empty(nb, dtype=torch.uint8, device=dev)
    buf.fill_(0x5a)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = L2Flush(torch, dev)
    with torch.cuda.stream(side):
        hyb_stream_read(buf, sink)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        hyb_stream_read(buf, sink, stream=side)
    torch.cuda.synchronize()
    time_events(args.warmup, stream, flush, g.replay)
    evs = time_events(args.steps, stream, flush, g.replay)
    torch.cuda.synchronize()
    del g, buf
    ms = max_over_ranks(mean_ms(evs), world, dev)
    return {"bytes": nb, "ms_per_call": round(ms, 5), "GB/s": round(nb / (ms * 1e-3) / 1e9, 1),
            "what": "hyb_stream_read of the step's algorithmic bytes: one coalesced streaming read with no "
                    "lookup, dependent load or arithmetic, timed like the step (CUDA-graph replay between "
                    "events, L2 flushed before each); the attainable time of any kernel that reads these "
                    "bytes once",
            "gpu_launches": args.steps}


def run_config(args, wl, rank, world, local_rank, clocks=None, cpu=True):
    """One workload: the fused decode step timed on the device (a CUDA graph
    of the hyb_decode_step launch, replayed per step), end to end through the
    C ABI with host buffers, and the oracle on the host cores (rank 0, N=1).
    Returns (record, workload)."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from int8_paged_kv_hybrid_b200 import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.make_workload(wl, seed_offset=1000 * rank)
    if args.hot_tokens != w.hot_tokens or args.block_size != w.block_size:
        # a smaller hot zone seals more blocks; larger blocks use the first
        # entries of the same table
        w.hot_tokens, w.block_size = args.hot_tokens, args.block_size
        room_for_growth(w, 0)
    if args.lean:
        room_for_growth(w, args.warmup + args.steps + 2)  # the lean run lets the cache grow
    L = int(w.lens.max())
    qb = args.quant_bits
    want_cpu = cpu and rank == 0 and world == 1 and not args.no_cpu_baseline and not args.lean
    ora = new_oracle(w, qb) if want_cpu else None
    cache, n_last, k_last, v_last, q = build_gpu_state(w, torch, qb, ora)
    if args.lean:
        L += args.warmup + args.steps  # the lean run lets the cache grow one token per step
    # split_tokens as asked (negative: at least that many splits per sequence)
    # and the plan it gives: the longest sequence's split length, its splits
    split = args.split or w.split_tokens
    split_len, ns = cache.plan(L, split)
    launch_kind, launch_ctas, launch_occ = cache.launch_info(L, split)
    # the step's inputs packed in one pinned host buffer (each part 256-byte
    # aligned), moved in one copy per step
    parts = [np.ascontiguousarray(a) for a in (n_last, k_last, v_last, q)]
    offs, off = [], 0
    for a in parts:
        offs.append(off)
        off += (a.nbytes + 255) // 256 * 256
    h_in = torch.empty(off, dtype=torch.uint8).pin_memory()
    for a, o in zip(parts, offs):
        h_in[o:o + a.nbytes].copy_(torch.from_numpy(a.view(np.uint8).reshape(-1)))
    d_in = h_in.to(dev)
    views = [d_in[o:o + a.nbytes].view(torch.from_numpy(a).dtype).view(a.shape) for a, o in zip(parts, offs)]
    n_d, k_d, v_d, q_d = views
    out = torch.empty((w.batch, w.num_q_heads, 128), dtype=torch.float16, device=dev)
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device=dev)
    ws = cache.step_workspace(L, split)

    snap = None if args.lean else StateSnapshot(cache, _touched_blocks(w, n_last), torch, dev)
    flush = L2Flush(torch, dev, enabled=not args.lean)

    def before():
        if snap is not None:
            snap.restore()
        flush()

    # one eager run (sets kernel attributes, checks the path), then capture the
    # step -- hyb_decode_step: append of the step's token + attention, one
    # launch -- as a CUDA graph on a side stream
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        before()
        cache.step(n_d, k_d, v_d, q_d, w.softmax_scale, L, split, out=out, lse=lse, workspace=ws)
        before()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=side):
        cache.step(n_d, k_d, v_d, q_d, w.softmax_scale, L, split, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    time_events(args.warmup, stream, before, g_step.replay)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark()
    evs = time_events(args.steps, stream, before, g_step.replay)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    ms_step = max_over_ranks(mean_ms(evs), world, dev)
    assert torch.isfinite(out.float()).all() and cache.status() == 0
    if args.lean:
        return {"lean": True, "ms_per_step": ms_step}, w
    del g_step

    # end to end through the C ABI with host buffers: every step copies its
    # inputs (n_new, k_new, v_new, q) from pinned host memory in one
    # cudaMemcpyAsync, calls hyb_decode_step (host checks, planning and the
    # launch, from Python through ctypes) and copies the output back into
    # pinned host memory -- all between the two events
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = int(h_in.numel())
    d2h = h_out.numel() * h_out.element_size()

    def e2e_body():
        d_in.copy_(h_in, non_blocking=True)
        cache.step(n_d, k_d, v_d, q_d, w.softmax_scale, L, split, out=out, lse=lse, workspace=ws)
        h_out.copy_(out, non_blocking=True)

    time_events(args.warmup, stream, before, e2e_body)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e = time_events(args.steps, stream, before, e2e_body)
    torch.cuda.synchronize()
    assert torch.equal(h_out, out.cpu())
    ms_e2e = max_over_ranks(mean_ms(e2e), world, dev)

    # the same, with the three operations captured once as a CUDA graph
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=side):
        e2e_body()
    torch.cuda.synchronize()
    time_events(args.warmup, stream, before, g_e2e.replay)
    e2e_g = time_events(args.steps, stream, before, g_e2e.replay)
    torch.cuda.synchronize()
    del g_e2e
    ms_e2e_g = max_over_ranks(mean_ms(e2e_g), world, dev)

    kvb = synth.kv_bytes(w, quant_bits=qb)
    stepb = kvb + synth.append_bytes(w, n_last, qb)
    floor = read_floor(torch, dev, stepb, stream, side, args, world)
    peak, peak_kind = measured_peaks()
    value = job_throughput(kvb, world, ms_step)
    tokens_s = w.batch * world / (ms_step * 1e-3)
    achieved = stepb / (ms_step * 1e-3) / 1e9
    default_shape = (qb == 8 and args.hot_tokens == 32 and args.block_size == 64 and not args.split)
    traffic, traffic_how = profiled_traffic(w.name) if default_shape else (None, "non-default shape")
    layers = 28 if w.num_q_heads == 28 else 32
    rec = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {8: "int8", 4: "int4", 0: "f16"}[qb],
        "data": "synthetic (seeded N(0,1) FP16 K/V/q; caches built by the library's own appends)",
        "config": workload_config(w, split, ns, qb, split_len, persistent=is_persistent(launch_kind)),
        "tokens_per_s": round(tokens_s, 1),
        "tokens_per_s_model_equiv": round(tokens_s / layers, 1),
        "kv_bytes_per_step": kvb,
        "frac_of_hbm_peak_step": round(value / world / peak, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": None if traffic is None else int(traffic),
                     "traffic_source": traffic_how,
                     "kernel": "%s (fused append + attention; %d CTAs, %d per SM; %d launch(es) per step, "
                               "all inside the timed span)"
                               % (DECODE_KERNELS[launch_kind], launch_ctas, launch_occ, DECODE_LAUNCHES[launch_kind]),
                     "peak_kind": peak_kind,
                     "achieved_bytes": "algorithmic bytes per launch: attention %d + append %d"
                                       % (kvb, stepb - kvb)},
        "e2e": {"value": round(job_throughput(kvb, world, ms_e2e), 1), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 5),
                "path": "per step: cudaMemcpyAsync of the packed inputs from pinned host memory, "
                        "hyb_decode_step through the C ABI (ctypes), cudaMemcpyAsync of the output to "
                        "pinned host memory"},
        "e2e_graph": {"value": round(job_throughput(kvb, world, ms_e2e_g), 1), "unit": UNIT,
                      "ms_per_step": round(ms_e2e_g, 5),
                      "path": "the same three operations captured once as a CUDA graph and replayed"},
        "gpu_launches": DECODE_LAUNCHES[launch_kind] * args.steps,
        "clocks": clk,
    }
    floor["frac"] = round(floor["GB/s"] / peak, 4)
    floor["step_over_floor"] = round(ms_step / floor["ms_per_call"], 3)
    rec["read_floor"] = floor
    if want_cpu:
        sec, n, threads = oracle_step_rate(ora, w, n_last, k_last, v_last, q, 3, 0, budget_s=25.0, qbits=qb)
        rec["cpu_baseline"] = {"value": round(kvb / sec / 1e9, 4), "unit": UNIT, "cores": threads,
                               "kind": "oracle", "cpu_model": cpu_model(),
                               "sample": "%d full steps of the same workload (1-token append + FP64 attention "
                                         "of all rows) on the host, OpenMP over rows" % n}
    del ora
    return rec, w


def run_append(args, rank, world, local_rank):
    """hyb_kv_append alone on the variable-length batch: the cache is built
    to L - n, then one timed call appends n[b] ~ U[1, 64] tokens to every
    sequence (sealing the tokens that leave the hot zone, quantizing them
    into their blocks, and writing the newest tokens into the ring).  The
    state the call changes is restored before every call (untimed) and L2 is
    flushed."""
    import numpy as np
    import torch
    from int8_paged_kv_hybrid_b200 import HybridKVCache, synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.make_workload(APPEND_WORKLOAD, seed_offset=1000 * rank)
    rng = np.random.default_rng([w.seed, 7])
    n_step = np.minimum(rng.integers(1, 65, size=w.batch), w.lens).astype(np.int32)
    start = (w.lens - n_step).astype(np.int64)
    cache = HybridKVCache(w.batch, w.num_kv_heads, w.num_q_heads, w.num_phys_blocks, w.max_blocks,
                          block_table=w.block_table, hot_tokens=w.hot_tokens, block_size=w.block_size)
    sched = synth._chunk_schedule(start, 64)  # prefill to exactly `start` tokens
    for si, n in enumerate(sched):
        k, v = synth.step_tokens(w, si, n, max_new=64)
        cache.append(torch.from_numpy(n).to(dev), torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(cache.seq_lens.cpu().numpy(), start.astype(np.int32))
    k, v = synth.step_tokens(w, 10_000, n_step, max_new=64)
    n_d, k_d, v_d = (torch.from_numpy(x).to(dev) for x in (n_step, k, v))
    snap = StateSnapshot(cache, _touched_blocks(w, n_step), torch, dev)
    flush = L2Flush(torch, dev)

    def before():
        snap.restore()
        flush()

    def body():
        cache.append(n_d, k_d, v_d)

    # device time: the call (its two launches) captured once as a CUDA graph
    # and replayed; e2e: the call itself from Python through the C ABI
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        before()
        body()
        before()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        body()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    time_events(args.warmup, stream, before, g.replay)
    evs = time_events(args.steps, stream, before, g.replay)
    time_events(args.warmup, stream, before, body)
    evs_e = time_events(args.steps, stream, before, body)
    torch.cuda.synchronize()
    del g
    assert cache.status() == 0
    ms = max_over_ranks(mean_ms(evs), world, dev)
    ms_e = max_over_ranks(mean_ms(evs_e), world, dev)
    ab = synth.append_call_bytes(w, start, n_step)
    return {"workload": "hyb_kv_append on the variable-length batch: 64 sequences, L in [256, 8192], one call of "
                        "U[1,64] new tokens per sequence (%d in all), INT8 cold blocks" % int(n_step.sum()),
            "ms_per_call": round(ms, 5), "us_per_call": round(ms * 1e3, 2),
            "GB/s": round(ab / (ms * 1e-3) / 1e9, 1), "algorithmic_bytes": ab,
            "tokens_per_s": round(float(n_step.sum()) / (ms * 1e-3), 1),
            "e2e_us_per_call": round(ms_e * 1e3, 2),
            "timing": "device: CUDA-graph replay of the call (append kernel + length update), events around it, "
                      "L2 flushed and state restored before each; e2e: the call from Python through the C ABI",
            "bytes": "per kv head: new K/V read (512 B/token), ring rows written (512 B each), evicted FP16 rows "
                     "read from the ring (512 B each), sealed codes written (256 B/token), the touched blocks' "
                     "scale pairs read and written (16 B/block)",
            "gpu_launches": 4 * args.steps}


def run_migrate(args):
    """Tier migration on one GPU: per timed step, one hyb_kv_migrate call that
    demotes the next quarter of every sequence's cold blocks (INT8 -> INT4),
    and one that promotes them back, alternating; L2 flushed before each."""
    import numpy as np
    import torch
    from int8_paged_kv_hybrid_b200 import synth
    wl = args.workload if args.workload is not None else 3
    w = synth.make_workload(wl)
    cache, n_last, k_last, v_last, q = build_gpu_state(w, torch)
    cache.append(torch.from_numpy(n_last).cuda(), torch.from_numpy(k_last).cuda(), torch.from_numpy(v_last).cuda())
    nb = w.cold_blocks()
    n0 = np.zeros(w.batch, np.int32) if w.n_int4 is None else w.n_int4.astype(np.int32)
    n1 = np.minimum(nb, n0 + nb // 4).astype(np.int32)
    moved = int((n1 - n0).sum()) * w.num_kv_heads  # (block, kv head) tile pairs per call
    delta = int((n1 - n0).max())
    t_down = torch.from_numpy(n1).cuda()
    t_up = torch.from_numpy(n0).cuda()
    flush = L2Flush(torch, "cuda")
    clocks = ClockSampler(0)
    times = {"demote": [], "promote": []}
    for i in range(2 * (args.warmup + args.steps)):
        kind = "demote" if i % 2 == 0 else "promote"
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        cache.migrate(t_down if kind == "demote" else t_up, delta)
        e1.record()
        if i == 2 * args.warmup:
            torch.cuda.synchronize()
            clocks.mark()
        if i >= 2 * args.warmup:
            times[kind].append((e0, e1))
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert cache.status() == 0
    ms = {k: sum(a.elapsed_time(b) for a, b in v) / len(v) for k, v in times.items()}
    peak, peak_kind = measured_peaks()
    tile = 2 * 8192
    # algorithmic bytes: the old tiles read and the new codes written (plus the
    # 8-byte scale pair read and written)
    alg = {"demote": moved * (tile + tile // 2 + 16), "promote": moved * (tile // 2 + tile + 16)}
    gbs = {k: alg[k] / (ms[k] * 1e-3) / 1e9 for k in ms}
    return {
        "metric": "hyb_kv_migrate GB/s of tiles re-quantized (INT8 -> INT4 demotion; promotion in 'promote')",
        "value": round(gbs["demote"], 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms["demote"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": dict(workload_config(w, 0, 0), migration="quarter of every sequence's cold blocks: "
                       "%d tile pairs per call, max_delta %d" % (moved, delta)),
        "promote": {"value": round(gbs["promote"], 1), "unit": "GB/s", "ms_per_step": round(ms["promote"], 5)},
        "roofline": {"bound": "hbm", "achieved": round(gbs["demote"], 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs["demote"] / peak, 4), "traffic": None, "peak_kind": peak_kind,
                     "kernel": "hyb::migrate_kernel",
                     "achieved_bytes": "per call: %d tile pairs x (16384 read + 8192 written + 16 scale bytes)"
                                       % moved,
                     "promote_frac": round(gbs["promote"] / peak, 4)},
        "bytes_written_demote": moved * (tile // 2 + 8),
        "gpu_launches": 2 * args.steps * 2,
        "clocks": clk,
    }


def run_sparse(args):
    """Sparse L2 attention on one GPU: hyb_decode_attn_sparse and the dense
    hyb_decode_attn on the same cache, alternating, L2 flushed before each."""
    import numpy as np
    import torch
    from int8_paged_kv_hybrid_b200 import hyb_sparse_top_k, synth
    wl = args.workload if args.workload is not None else 4
    w = synth.make_workload(wl)
    if w.n_int4 is None:
        w.n_int4 = (w.cold_blocks() // 2).astype(np.int32)
    cache, n_last, k_last, v_last, q = build_gpu_state(w, torch)
    cache.append(torch.from_numpy(n_last).cuda(), torch.from_numpy(k_last).cuda(), torch.from_numpy(v_last).cuda())
    L = int(w.lens.max())
    top_k = hyb_sparse_top_k(L) if args.sparse_top_k < 0 else args.sparse_top_k
    # the sparse path takes a fixed split length (512 tokens: >= 64 splits
    # for every sequence of the long-context workload)
    split = args.split or (w.split_tokens if w.split_tokens >= 0 else 512)
    qd = torch.from_numpy(q).cuda()
    out = torch.empty((w.batch, w.num_q_heads, 128), dtype=torch.float16, device="cuda")
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device="cuda")
    ws_s = cache.sparse_workspace(L, split)
    ws_d = cache.workspace(L, split)
    flush = L2Flush(torch, "cuda")
    clocks = ClockSampler(0)
    times = {"sparse": [], "dense": []}
    for i in range(2 * (args.warmup + args.steps)):
        kind = "sparse" if i % 2 == 0 else "dense"
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if kind == "sparse":
            cache.decode_sparse(qd, w.softmax_scale, L, top_k, split, out=out, lse=lse, workspace=ws_s)
        else:
            cache.decode(qd, w.softmax_scale, L, split, out=out, lse=lse, workspace=ws_d)
        e1.record()
        if i == 2 * args.warmup:
            torch.cuda.synchronize()
            clocks.mark()
        if i >= 2 * args.warmup:
            times[kind].append((e0, e1))
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert cache.status() == 0 and torch.isfinite(out.float()).all()
    ms = {k: sum(a.elapsed_time(b) for a, b in v) / len(v) for k, v in times.items()}
    # L2 tokens per sequence and the bytes the sparse call must move: the
    # dense bytes minus the L2 V codes (64 B per token and kv head), plus the
    # selected tokens' V codes (64 B per token and query head)
    nb = w.cold_blocks()
    l2 = np.minimum(np.maximum(w.lens - w.hot_tokens, 0), w.n_int4 * 64)
    dense_b = synth.kv_bytes(w)
    sel = np.minimum(l2, top_k)
    sparse_b = dense_b - int(l2.sum()) * w.num_kv_heads * 64 + int(sel.sum()) * w.num_q_heads * 64
    peak, peak_kind = measured_peaks()
    gbs = sparse_b / (ms["sparse"] * 1e-3) / 1e9
    return {
        "metric": "hyb_decode_attn_sparse (top-k of the INT4 L2 tokens) GB/s of the bytes the sparse pass must move",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms["sparse"], 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4", "data": "synthetic",
        "config": dict(workload_config(w, split, 0), top_k=top_k,
                       l2="older half of every sequence's cold blocks INT4: %d L2 tokens in all" % int(l2.sum())),
        "dense": {"ms_per_step": round(ms["dense"], 5), "kv_bytes": dense_b,
                  "GB/s": round(dense_b / (ms["dense"] * 1e-3) / 1e9, 1)},
        "sparse_bytes": sparse_b,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None, "peak_kind": peak_kind,
                     "kernel": "decode_kernel (l2_skip) + l2_score_kernel + l2_topk_kernel"},
        "gpu_launches": 3 * args.steps + args.steps,
        "clocks": clk,
    }


def oracle_step_rate(ora, w, n_last, k_last, v_last, q, steps, warmup, budget_s=None, qbits=8, nthreads=None):
    """Time the CPU oracle (as it stands) on a prefilled copy of the workload:
    per step the 1-token append plus FP64 attention of every (sequence,
    head).  The state grows by one token per step (bounded sample)."""
    threads = nthreads or os.cpu_count() or 1
    times = []
    for i in range(warmup + steps):
        t0 = time.perf_counter()
        ora.append(n_last, k_last, v_last)
        ora.decode(q, w.softmax_scale, nthreads=threads)
        t1 = time.perf_counter()
        if i >= warmup:
            times.append(t1 - t0)
        if budget_s is not None and sum(times) > budget_s and len(times) >= 1:
            break
    return sum(times) / len(times), len(times), threads


def oracle_prefilled(w, qbits=8):
    """The oracle with the workload's prefill replayed (the same arrays the
    library gets) and the step's inputs."""
    from int8_paged_kv_hybrid_b200 import synth
    ora = new_oracle(w, qbits)
    sched = synth._chunk_schedule(w.lens, 64)
    for si, n in enumerate(sched[:-1]):
        k, v = synth.step_tokens(w, si, n, max_new=64)
        ora.append(n, k, v)
    last = len(sched) - 1
    n_last = sched[-1]
    k_last, v_last = synth.step_tokens(w, last, n_last, max_new=1)
    return ora, n_last, k_last, v_last, synth.query(w)


def oracle_one_thread_config1():
    """The oracle on the single-sequence workload (L = 1024, 8 heads) with one
    thread: FP64 attention of all rows, per step."""
    from int8_paged_kv_hybrid_b200 import synth
    w = synth.make_workload(1)
    ora, n_last, k_last, v_last, q = oracle_prefilled(w)
    sec, n, _ = oracle_step_rate(ora, w, n_last, k_last, v_last, q, 20, 2, budget_s=10.0, nthreads=1)
    kvb = synth.kv_bytes(w)
    return {"workload": w.name, "threads": 1, "ms_per_step": round(sec * 1e3, 3),
            "value": round(kvb / sec / 1e9, 4), "unit": UNIT, "steps": n, "cpu_model": cpu_model()}


SUB_KEYS = ("value", "unit", "ms_per_step", "tokens_per_s", "tokens_per_s_model_equiv", "kv_bytes_per_step",
            "frac_of_hbm_peak_step", "e2e", "e2e_graph", "cpu_baseline", "config", "read_floor")


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world == 1 and args.gpus > 1:
        print(json.dumps({"error": "run N > 1 under torchrun"}))
        return 2
    from int8_paged_kv_hybrid_b200 import synth
    wl_main = HEADLINE if args.workload is None else args.workload

    if args.impl == "reference":
        # the CPU oracle on the host cores: rank 0 alone
        if rank != 0:
            return 0
        w = synth.make_workload(wl_main)
        w.hot_tokens, w.block_size = args.hot_tokens, args.block_size
        ora, n_last, k_last, v_last, q = oracle_prefilled(w, args.quant_bits)
        sec, n, threads = oracle_step_rate(ora, w, n_last, k_last, v_last, q, args.steps, args.warmup,
                                           budget_s=120.0, qbits=args.quant_bits)
        kvb = synth.kv_bytes(w, quant_bits=args.quant_bits)
        val = kvb / sec / 1e9
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": UNIT, "n_gpus": world,
            "steps": n, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, w.split_tokens, 0, args.quant_bits),
            "tokens_per_s": round(w.batch / sec, 3),
            "cpu_baseline": {"value": round(val, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": "%d full steps of the workload (append 1 token/seq + FP64 attention "
                                       "of all %d rows), state growing 1 token per step (at most ~120 s)"
                                       % (n, w.batch * w.num_q_heads)},
            "e2e": {"value": round(val, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return 0

    import torch
    if args.migrate:
        if rank == 0:
            print(json.dumps(run_migrate(args)))
        return 0
    if args.sparse_top_k is not None:
        if rank == 0:
            print(json.dumps(run_sparse(args)))
        return 0
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    clocks = ClockSampler(local_rank) if rank == 0 and not args.lean else None
    res, w = run_config(args, wl_main, rank, world, local_rank, clocks=clocks)
    if args.workload is None and not args.lean:
        # every other measured configuration in the same run, then the
        # append-only record and the oracle's one-thread time
        res["configs"] = {}
        for wl in SUB_WORKLOADS:
            sub, ws = run_config(args, wl, rank, world, local_rank)
            res["configs"][ws.name] = {k: sub[k] for k in SUB_KEYS if k in sub}
            res["configs"][ws.name]["roofline_frac"] = sub["roofline"]["frac"]
            res["configs"][ws.name]["traffic"] = sub["roofline"]["traffic"]
            res["gpu_launches"] += sub["gpu_launches"]
        res["append"] = run_append(args, rank, world, local_rank)
        res["gpu_launches"] += res["append"]["gpu_launches"]
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["oracle_one_thread"] = oracle_one_thread_config1()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
