"""CPU oracle for the hybrid_v2 two-tier KV cache (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this package.  The GPU library (``int8_paged_kv_hybrid_b200``)
never imports it, and it imports nothing from the GPU library.

The arithmetic lives in ``hyb_oracle.c`` (plain C, FP32 quantizer, FP64
attention); this module only builds it with gcc and marshals numpy arrays.
Source of the method: the web page "DeepSeek V4混合式KV Cache推理优化实战解析",
sections 2.1, 3.1, 3.2 and 4.2 (see the header of hyb_oracle.c).

Every function of the oracle is pinned by tests in ``tests/test_oracle_*.py``
(closed forms, hand-worked examples under ``tests/golden/``, brute force on
tiny inputs and invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyb_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhyb_oracle.so")
_lib = None

HOT, BLOCK, HEAD_DIM = 32, 64, 128


def build(force: bool = False) -> str:
    """Compile hyb_oracle.c into libhyb_oracle.so next to it (gcc, no fast-math,
    no FMA contraction, OpenMP for the independent (sequence, head) loop)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i32 = ctypes.c_int
    lib.ora_new.restype = P
    lib.ora_new.argtypes = [i32] * 8
    lib.ora_free.argtypes = [P]
    lib.ora_set_n_int4.argtypes = [P, P]
    lib.ora_len.argtypes = [P, i32]
    lib.ora_len.restype = ctypes.c_int32
    lib.ora_append.argtypes = [P, P, i32, P, P]
    lib.ora_decode.argtypes = [P, P, ctypes.c_double, P, i32, P, P, i32]
    lib.ora_decode_topk.argtypes = [P, P, ctypes.c_double, i32, P, i32, P, P, i32]
    lib.ora_decode_topk.restype = ctypes.c_int32
    lib.ora_decode_sel.argtypes = [P, P, ctypes.c_double, P, i32, P, P, i32, P, P, i32]
    lib.ora_decode_sel.restype = ctypes.c_int32
    lib.ora_l2_scores.argtypes = [P, P, ctypes.c_double, i32, i32, P]
    lib.ora_l2_scores.restype = ctypes.c_int32
    lib.ora_sparse_top_k.argtypes = [ctypes.c_long]
    lib.ora_sparse_top_k.restype = ctypes.c_int32
    lib.ora_combine.argtypes = [i32, i32, i32, P, P, P, P]
    lib.ora_get_block.argtypes = [P, i32, i32, P, P]
    lib.ora_get_block_fp16.argtypes = [P, i32, i32, P]
    lib.ora_get_ring.argtypes = [P, i32, P]
    lib.ora_block_q.argtypes = [P, i32, i32]
    lib.ora_block_q.restype = ctypes.c_int32
    lib.ora_export.argtypes = [P, P, i32, P, P, P, P]
    lib.ora_migrate.argtypes = [P, P]
    lib.ora_n_int4.argtypes = [P, i32]
    lib.ora_n_int4.restype = ctypes.c_int32
    lib.ora_migration_threshold_ms.argtypes = [P, i32]
    lib.ora_migration_threshold_ms.restype = ctypes.c_double
    lib.ora_migration_decision.argtypes = [ctypes.c_double, ctypes.c_double, i32]
    lib.ora_half_to_double.argtypes = [ctypes.c_uint16]
    lib.ora_half_to_double.restype = ctypes.c_double
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def half_to_double(bits: int) -> float:
    return float(_load().ora_half_to_double(ctypes.c_uint16(bits)))


class OracleCache:
    """Logical hybrid_v2 cache on the host: FP16 hot ring + quantized cold blocks."""

    def __init__(self, batch, num_kv_heads, num_q_heads, max_blocks_per_seq,
                 quant_bits=8, head_dim=HEAD_DIM, hot=HOT, block=BLOCK):
        self._lib = _load()
        self.batch, self.hkv, self.hq = batch, num_kv_heads, num_q_heads
        self.d, self.hot, self.block = head_dim, hot, block
        self.max_blocks = max_blocks_per_seq
        self.quant_bits = quant_bits
        self._h = self._lib.ora_new(batch, num_kv_heads, num_q_heads, head_dim,
                                    hot, block, max_blocks_per_seq, quant_bits)
        if not self._h:
            raise ValueError("oracle: invalid cache configuration")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.ora_free(h)
            self._h = None

    def set_n_int4(self, n_int4):
        a = _c(n_int4, np.int32)
        self._lib.ora_set_n_int4(self._h, _ptr(a))

    def append(self, n_new, k_new, v_new):
        """k_new, v_new: float16 [batch][max_new][hkv][d]; n_new: int [batch]."""
        n = _c(n_new, np.int32)
        k = _c(k_new, np.float16)
        v = _c(v_new, np.float16)
        max_new = k.shape[1]
        rc = self._lib.ora_append(self._h, _ptr(n), max_new, _ptr(k.view(np.uint16)),
                                  _ptr(v.view(np.uint16)))
        if rc != 0:
            raise ValueError("oracle append rejected (rc=%d)" % rc)

    def migrate(self, target_n_int4):
        """Move each sequence's INT4 block count to target_n_int4[b],
        re-quantizing the blocks in between (see ora_migrate)."""
        t = _c(target_n_int4, np.int32)
        rc = self._lib.ora_migrate(self._h, _ptr(t))
        if rc != 0:
            raise ValueError("oracle migrate rejected (rc=%d)" % rc)

    def n_int4(self):
        return np.array([self._lib.ora_n_int4(self._h, b) for b in range(self.batch)], np.int32)

    def lens(self):
        return np.array([self._lib.ora_len(self._h, b) for b in range(self.batch)], np.int32)

    def decode(self, q, softmax_scale, pairs=None, nthreads=None, top_k=None, sel=None):
        """q: float16 [batch][hq][d].  Returns (out float64 [batch][hq][d],
        lse float64 [batch][hq]); with `pairs` ([(b, h), ...]) only those rows
        are computed and the others are NaN.  top_k: sparse L2 blocks (each
        head attends only the top_k of its INT4-block tokens by attention
        logit, see ora_decode_topk); None = dense.  sel: a given selection
        instead, a list over rows r = b * hq + h of the L2 positions that row
        attends (see ora_decode_sel)."""
        qq = _c(q, np.float16)
        out = np.full((self.batch, self.hq, self.d), np.nan)
        lse = np.full((self.batch, self.hq), np.nan)
        if pairs is None:
            pp, npairs = None, 0
        else:
            pp = _c(np.asarray(pairs, np.int32).reshape(-1, 2), np.int32)
            npairs = pp.shape[0]
        nt = nthreads or os.cpu_count() or 1
        if sel is not None:
            rows = self.batch * self.hq
            assert len(sel) == rows
            stride = max(1, max(len(x) for x in sel))
            sa = np.zeros((rows, stride), np.int32)
            cnt = np.zeros(rows, np.int32)
            for r, x in enumerate(sel):
                sa[r, :len(x)] = x
                cnt[r] = len(x)
            rc = self._lib.ora_decode_sel(self._h, _ptr(qq.view(np.uint16)), float(softmax_scale), _ptr(sa),
                                          stride, _ptr(cnt), None if pp is None else _ptr(pp), npairs,
                                          _ptr(out), _ptr(lse), nt)
            if rc != 0:
                raise ValueError("oracle decode_sel rejected the selection (rc=%d)" % rc)
            return out, lse
        rc = self._lib.ora_decode_topk(self._h, _ptr(qq.view(np.uint16)), float(softmax_scale),
                                       -1 if top_k is None else int(top_k),
                                       None if pp is None else _ptr(pp), npairs, _ptr(out), _ptr(lse), nt)
        if rc != 0:
            raise MemoryError("oracle decode failed (rc=%d)" % rc)
        return out, lse

    def l2_scores(self, q, softmax_scale, b, h):
        """FP64 attention logits of the L2 tokens of sequence b for query head
        h (the scores the top-k selection ranks), positions 0.. in order."""
        qq = _c(q, np.float16)
        buf = np.zeros(max(1, int(self.lens()[b])), np.float64)
        n = self._lib.ora_l2_scores(self._h, _ptr(qq.view(np.uint16)), float(softmax_scale), int(b), int(h),
                                    _ptr(buf))
        if n < 0:
            raise ValueError("oracle l2_scores rejected (b, h)")
        return buf[:n].copy()

    def get_block(self, b, i):
        """(Q, codes int8 [hkv][2][block][d], scales float32 [hkv][2]); Q = 0 if unsealed."""
        codes = np.zeros((self.hkv, 2, self.block, self.d), np.int8)
        sc = np.zeros((self.hkv, 2), np.float32)
        q = self._lib.ora_get_block(self._h, b, i, _ptr(codes), _ptr(sc))
        return q, codes, sc

    def get_block_fp16(self, b, i):
        """FP16 cold block (quant_bits 0): (sealed?, float16 [hkv][2][block][d])."""
        vals = np.zeros((self.hkv, 2, self.block, self.d), np.uint16)
        ok = self._lib.ora_get_block_fp16(self._h, b, i, _ptr(vals))
        return bool(ok), vals.view(np.float16)

    def block_q(self, b, i):
        """127 (INT8), 7 (INT4), -1 (FP16) once block i of sequence b holds a
        sealed token, else 0."""
        return int(self._lib.ora_block_q(self._h, int(b), int(i)))

    def ring(self, b):
        r = np.zeros((self.hkv, self.hot, 2, self.d), np.uint16)
        self._lib.ora_get_ring(self._h, b, _ptr(r))
        return r.view(np.float16)

    def export(self, block_table, num_phys):
        """Device memory format of the whole cache (see hyb_oracle.c):
        returns dict(cold uint8 [num_phys][hkv][2][8192] ([4][8192] for FP16
        blocks), scales float32
        [num_phys][hkv][2], hot float16 [batch][hkv][hot][2][d], seq_lens int32)."""
        bt = _c(block_table, np.int32)
        assert bt.shape == (self.batch, self.max_blocks)
        # 8 KB parts: K and V tiles per 64-slot sub-block (a 32-token block
        # uses half of one); FP16 blocks: 512 B per token row
        parts = self.block // 16 if self.quant_bits == 0 else 2 * max(1, self.block // 64)
        cold = np.zeros((num_phys, self.hkv, parts, 64 * self.d), np.uint8)
        sc = np.zeros((num_phys, self.hkv, 2), np.float32)
        hot = np.zeros((self.batch, self.hkv, self.hot, 2, self.d), np.uint16)
        sl = np.zeros(self.batch, np.int32)
        rc = self._lib.ora_export(self._h, _ptr(bt), num_phys, _ptr(cold), _ptr(sc),
                                  _ptr(hot), _ptr(sl))
        if rc != 0:
            raise ValueError("oracle export failed (rc=%d)" % rc)
        return dict(cold=cold, scales=sc, hot=hot.view(np.float16), seq_lens=sl)


def sparse_top_k(context_length):
    """The page's sparse_top_k rule (see ora_sparse_top_k)."""
    return int(_load().ora_sparse_top_k(int(context_length)))


def migration_threshold_ms(lens):
    """Adaptive migration threshold in ms (see ora_migration_threshold_ms)."""
    a = _c(np.asarray(lens, np.int32), np.int32)
    return float(_load().ora_migration_threshold_ms(_ptr(a), a.size))


def migration_decision(avg_interval_ms, threshold_ms, is_int4):
    """+1 promote (INT4 -> INT8), -1 demote (INT8 -> INT4), 0 keep."""
    return int(_load().ora_migration_decision(float(avg_interval_ms), float(threshold_ms), 1 if is_int4 else 0))


def combine(o_part, lse_part):
    """LSE merge in FP64.  o_part [rows][S][d], lse_part [rows][S] -> (out [rows][d], lse [rows])."""
    lib = _load()
    o = _c(o_part, np.float64)
    l = _c(lse_part, np.float64)
    rows, s, d = o.shape
    out = np.zeros((rows, d))
    lse = np.zeros(rows)
    lib.ora_combine(rows, s, d, _ptr(o), _ptr(l), _ptr(out), _ptr(lse))
    return out, lse
