"""Seeded synthetic workloads for the hybrid_v2 decode path.

This module only draws random inputs and lays out block tables and append
schedules; it holds none of the method's arithmetic (no quantization, no
attention).  Tests feed the very same arrays to the GPU library and to the
CPU oracle.

The five workloads follow the shapes the hybrid_v2 page measures on
(Llama-3-8B and Qwen2-7B attention shapes, the 50/30/20 mixed serving load of
its section 2.2) with i.i.d. normal FP16 data; no dataset or trace is used.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

HOT, BLOCK, HEAD_DIM = 32, 64, 128


@dataclasses.dataclass
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    lens: np.ndarray              # final tokens per sequence (int32 [batch])
    softmax_scale: float
    q_std: float                  # q ~ N(0, q_std^2)
    num_phys_blocks: int
    block_table: np.ndarray       # int32 [batch][max_blocks], -1 = unassigned
    n_int4: Optional[np.ndarray]  # int32 [batch] or None
    schedule: List[np.ndarray]    # n_new per append call (int32 [batch])
    max_new: int                  # width of the k_new / v_new staging arrays
    seed: int
    outlier_channels: Optional[np.ndarray] = None  # int [hkv][4] scaled x10 in K
    split_tokens: int = 0
    head_dim: int = HEAD_DIM
    hot_tokens: int = HOT
    block_size: int = BLOCK

    @property
    def max_blocks(self) -> int:
        return self.block_table.shape[1]

    def cold_blocks(self) -> np.ndarray:
        return np.array([cold_blocks_for(int(L), self.hot_tokens, self.block_size) for L in self.lens], np.int64)


# The measured workloads, by what they are.
WORKLOAD_NAMES = {
    1: "one_seq_mha8_L1024",
    2: "llama3_8b_b8_L2048",
    3: "var64_gqa4_L256_8192",
    4: "long_b4_L32k_128k",
    5: "qwen2_7b_b128_mixed_int4",
}


def cold_blocks_for(L: int, hot: int = HOT, block: int = BLOCK) -> int:
    """Cold blocks a sequence of L tokens occupies (the newest `hot` stay hot)."""
    return (max(0, L - hot) + block - 1) // block


def _block_table(rng, nblk: np.ndarray, pool: int) -> np.ndarray:
    need = int(nblk.sum())
    assert need <= pool, (need, pool)
    perm = rng.permutation(pool)[:need].astype(np.int32)
    width = max(1, int(nblk.max()))
    bt = np.full((len(nblk), width), -1, np.int32)
    o = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = perm[o:o + n]
        o += n
    return bt


def _chunk_schedule(lens: np.ndarray, chunk: int) -> List[np.ndarray]:
    """Prefill to L-1 in appends of `chunk` tokens, then one append of 1 token
    per sequence (the decode step)."""
    lens = np.asarray(lens, np.int64)
    cur = np.zeros_like(lens)
    target = np.maximum(lens - 1, 0)
    sched = []
    while (cur < target).any():
        n = np.minimum(chunk, target - cur)
        sched.append(n.astype(np.int32))
        cur += n
    sched.append((lens - cur).astype(np.int32))
    return sched


def _random_step_schedule(rng, lens: np.ndarray, lo: int, hi: int) -> List[np.ndarray]:
    """Appends of U[lo, hi] tokens per sequence per call until every sequence
    reaches its length (sequences that are done append 0)."""
    lens = np.asarray(lens, np.int64)
    cur = np.zeros_like(lens)
    sched = []
    while (cur < lens).any():
        n = rng.integers(lo, hi + 1, size=len(lens))
        n = np.minimum(n, lens - cur)
        sched.append(n.astype(np.int32))
        cur += n
    return sched


def make_workload(idx: int, scale_down: int = 1, seed_offset: int = 0) -> Workload:
    """Workload `idx` in 1..5.  scale_down > 1 shrinks lengths and batch (same
    structure) for quick tests; seed_offset gives an independent replica of
    the same shapes (one per GPU in the multi-GPU benchmark)."""
    seed = 1000 + idx + seed_offset
    rng = np.random.default_rng([seed, 0])
    d = HEAD_DIM
    n_int4 = None
    outl = None
    split = 0
    if idx == 1:
        # one sequence, one layer, MHA 8 heads, L = 1024 (32 hot + 992 cold)
        B, hq, hkv = 1, 8, 8
        lens = np.array([1024 // scale_down], np.int64)
        sm, qstd = 1.0 / math.sqrt(d), 1.0
        nblk = np.array([cold_blocks_for(int(lens[0]))])
        pool = max(1, int(nblk.sum()))
        sched_kind = "chunk"
    elif idx == 2:
        # Llama-3-8B decode, one layer: batch 8, GQA 32/8, L = 2048, pool 4096
        B, hq, hkv = max(1, 8 // scale_down), 32, 8
        lens = np.full(B, 2048 // scale_down, np.int64)
        sm, qstd = 1.0, 1.0 / math.sqrt(d)
        nblk = np.array([cold_blocks_for(int(L)) for L in lens])
        pool = 4096 // scale_down
        sched_kind = "chunk"
    elif idx == 3:
        # variable lengths U[256, 8192], 4 outlier K channels x10 per kv head
        B, hq, hkv = max(2, 64 // scale_down), 32, 8
        lens = rng.integers(256 // scale_down, 8192 // scale_down + 1, size=B)
        sm, qstd = 1.0 / math.sqrt(d), 1.0
        nblk = np.array([cold_blocks_for(int(L)) for L in lens])
        pool = int(math.ceil(1.25 * nblk.sum()))
        outl = np.stack([rng.choice(d, 4, replace=False) for _ in range(hkv)])
        sched_kind = "random"
    elif idx == 4:
        # long context: L = 32K, 32K, 128K, 128K; >= 64 splits per sequence
        B, hq, hkv = 4, 32, 8
        lens = np.array([32768, 32768, 131072, 131072], np.int64) // scale_down
        sm, qstd = 1.0 / math.sqrt(d), 1.0
        nblk = np.array([cold_blocks_for(int(L)) for L in lens])
        pool = int(nblk.sum())
        split = -64  # per-sequence splits: at least 64 for every sequence
        sched_kind = "chunk"
    elif idx == 5:
        # Qwen2-7B mixed serving load, batch 128: 50% L in [64,512],
        # 30% in [4096,8192], 20% in [1024,2048]; oldest 25% cold blocks INT4
        B, hq, hkv = max(4, 128 // scale_down), 28, 4
        n_a = int(round(0.5 * B))
        n_b = int(round(0.3 * B))
        n_c = B - n_a - n_b
        la = rng.integers(64, 512 + 1, size=n_a)
        lb = rng.integers(4096 // scale_down, 8192 // scale_down + 1, size=n_b)
        lc = rng.integers(1024 // scale_down, 2048 // scale_down + 1, size=n_c)
        lens = rng.permutation(np.concatenate([la, lb, lc]))
        sm, qstd = 1.0 / math.sqrt(d), 1.0
        nblk = np.array([cold_blocks_for(int(L)) for L in lens])
        pool = int(math.ceil(1.25 * nblk.sum()))
        n_int4 = (nblk // 4).astype(np.int32)
        sched_kind = "chunk"
    else:
        raise ValueError("workload index must be 1..5")
    lens = np.asarray(lens, np.int64)
    bt = _block_table(rng, nblk, pool)
    if sched_kind == "chunk":
        sched = _chunk_schedule(lens, 64)
        max_new = 64
    else:
        sched = _random_step_schedule(rng, lens, 1, 64)
        max_new = 64
    return Workload(name=WORKLOAD_NAMES[idx], batch=B, num_q_heads=hq, num_kv_heads=hkv,
                    lens=lens.astype(np.int32), softmax_scale=sm, q_std=qstd,
                    num_phys_blocks=pool, block_table=bt, n_int4=n_int4,
                    schedule=sched, max_new=max_new, seed=seed,
                    outlier_channels=outl, split_tokens=split)


def step_tokens(w: Workload, step: int, n_new: np.ndarray, max_new: Optional[int] = None):
    """FP16 K and V for append call `step`: [batch][max_new][hkv][d] each.
    Rows beyond n_new[b] are zero (never read)."""
    mx = w.max_new if max_new is None else max_new
    n_new = np.asarray(n_new, np.int64)
    rng = np.random.default_rng([w.seed, 1, step])
    rows = (w.num_kv_heads, w.head_dim)
    total = int(n_new.sum())
    kd = rng.standard_normal((total,) + rows, dtype=np.float32)
    vd = rng.standard_normal((total,) + rows, dtype=np.float32)
    if w.outlier_channels is not None:
        for h in range(w.num_kv_heads):
            kd[:, h, w.outlier_channels[h]] *= 10.0
    k = np.zeros((w.batch, mx) + rows, np.float16)
    v = np.zeros((w.batch, mx) + rows, np.float16)
    o = 0
    for b, n in enumerate(n_new):
        k[b, :n] = kd[o:o + n]
        v[b, :n] = vd[o:o + n]
        o += n
    return k, v


def query(w: Workload, step: int = 0) -> np.ndarray:
    """FP16 q [batch][hq][d] ~ N(0, q_std^2)."""
    rng = np.random.default_rng([w.seed, 2, step])
    q = rng.standard_normal((w.batch, w.num_q_heads, w.head_dim), dtype=np.float32)
    return (q * w.q_std).astype(np.float16)


def kv_bytes(w: Workload, lens: Optional[np.ndarray] = None, quant_bits: int = 8) -> int:
    """Algorithmic bytes one decode pass must move: cold codes (256 B per
    token and kv head at INT8, 128 B at INT4), two FP32 scales per block and
    kv head, FP16 hot tokens (512 B per token and kv head), the block table
    (4 B per block), q and the FP16 output.  quant_bits 4: every cold block
    INT4; quant_bits 0: FP16 cold tokens (512 B per token and kv head) and no
    scales."""
    lens = w.lens if lens is None else lens
    hkv, d = w.num_kv_heads, w.head_dim
    total = 0
    for b, L in enumerate(lens):
        L = int(L)
        cold = max(0, L - w.hot_tokens)
        hot = L - cold
        nblk = (cold + w.block_size - 1) // w.block_size
        n4 = 0
        if quant_bits == 4:
            n4 = nblk
        elif w.n_int4 is not None and quant_bits == 8:
            n4 = min(int(w.n_int4[b]), nblk)
        # tokens in INT4 blocks (the oldest n4 blocks are always full)
        t4 = min(cold, n4 * w.block_size)
        t8 = cold - t4
        if quant_bits == 0:
            total += hkv * cold * 2 * d * 2        # K + V, FP16
        else:
            total += hkv * (t8 * 2 * d + t4 * d)   # K + V codes
            total += hkv * nblk * 2 * 4            # scales
        total += hkv * hot * 2 * d * 2             # hot K + V FP16
        total += nblk * 4                          # block table entries
    total += w.batch * w.num_q_heads * d * 2 * 2   # q in, out
    return total


def append_call_bytes(w: Workload, lens_old: np.ndarray, n_new: np.ndarray, quant_bits: int = 8) -> int:
    """Algorithmic bytes of one hyb_kv_append call that adds n_new[b] tokens
    to sequences of lens_old[b] tokens: per kv head, the new tokens' FP16 K
    and V read (512 B each), the ring rows written (512 B per new token kept
    hot), the evicted tokens' FP16 rows read from the ring (512 B each, for
    those that were in the cache before the call), their codes written (256 B
    per token at INT8, 128 B at INT4; their 512 B FP16 rows at quant_bits 0)
    and the scale pair of every block they land in read and written (16 B)."""
    H, Bs = w.hot_tokens, w.block_size
    total = 0
    for L0, n in zip(lens_old, n_new):
        L0, n = int(L0), int(n)
        L1 = L0 + n
        e0, e1 = max(0, L0 - H), max(0, L1 - H)
        evicted = e1 - e0
        from_ring = max(0, min(e1, L0) - e0)
        blocks = ((e1 - 1) // Bs - e0 // Bs + 1) if evicted > 0 else 0
        per_token_code = 512 if quant_bits == 0 else (256 if quant_bits == 8 else 128)
        b = n * 512 + min(n, H) * 512 + from_ring * 512 + evicted * per_token_code
        if quant_bits != 0:
            b += blocks * 16
        total += b * w.num_kv_heads
    return total


def custom_workload(name, lens, num_q_heads, num_kv_heads, seed, softmax_scale=None,
                    schedule="random", chunk=64, max_step=64, pool_extra=3, n_int4=None,
                    outliers=False, split_tokens=0, hot=HOT, block=BLOCK) -> Workload:
    """A small workload with the given final lengths (for parity tests).
    schedule: "random" (U[1, max_step] tokens per call), "chunk" (prefill in
    `chunk`-token calls then one 1-token call) or "one" (a single call)."""
    rng = np.random.default_rng([seed, 0])
    lens = np.asarray(lens, np.int64)
    B = len(lens)
    nblk = np.array([cold_blocks_for(int(L), hot, block) for L in lens])
    pool = int(nblk.sum()) + pool_extra
    bt = _block_table(rng, nblk, pool)
    if schedule == "random":
        sched = _random_step_schedule(rng, lens, 1, max_step)
        mx = max_step
    elif schedule == "chunk":
        sched = _chunk_schedule(lens, chunk)
        mx = chunk
    else:
        sched = [lens.astype(np.int32)]
        mx = max(1, int(lens.max()))
    outl = None
    if outliers:
        outl = np.stack([rng.choice(HEAD_DIM, 4, replace=False) for _ in range(num_kv_heads)])
    sm = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(HEAD_DIM)
    return Workload(name=name, batch=B, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                    lens=lens.astype(np.int32), softmax_scale=sm, q_std=1.0,
                    num_phys_blocks=pool, block_table=bt,
                    n_int4=None if n_int4 is None else np.asarray(n_int4, np.int32),
                    schedule=sched, max_new=mx, seed=seed, outlier_channels=outl,
                    split_tokens=split_tokens, hot_tokens=hot, block_size=block)


def append_bytes(w: Workload, n_new: np.ndarray, quant_bits: int = 8) -> int:
    """Algorithmic bytes of appending n_new[b] in {0, 1} tokens beyond what the
    attention pass reads anyway (the evicted token and the tail block are in
    the attention bytes): the new token's FP16 K and V read (512 B per kv
    head) and written to the hot ring (512 B), the sealed token's codes
    written (256 B at INT8, 128 B at INT4, its 512 B FP16 rows at
    quant_bits 0) and the two scales (8 B, none at quant_bits 0), per kv
    head."""
    seal = {8: 256 + 8, 4: 128 + 8, 0: 512}[quant_bits]
    total = 0
    for b, n in enumerate(np.asarray(n_new)):
        if int(n) == 0:
            continue
        L_old = int(w.lens[b]) - int(n)
        per_head = 512 + 512 + (seal if L_old >= w.hot_tokens else 0)
        total += w.num_kv_heads * per_head
    return total
