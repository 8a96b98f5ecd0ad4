"""ctypes binding of libhybkv.so (the C ABI in include/hyb_kv.h).

Argument marshalling only: every step of the decode path runs in the CUDA
library.  Tensors are PyTorch CUDA tensors (PyTorch provides device memory
and streams); their data pointers go straight to the C functions.  There is
no CPU fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhybkv.so")

HYB_OK = 0
HYB_ERR_INVALID_VALUE = -1
HYB_ERR_UNSUPPORTED = -2
HYB_ERR_WORKSPACE = -3
HYB_ERR_CUDA = -4
HYB_ERR_SCRATCH_LIMIT = -5

HYB_STATUS_OK = 0
HYB_STATUS_BAD_BLOCK = 1
HYB_STATUS_BAD_N_NEW = 2
HYB_STATUS_CAPACITY = 3
HYB_STATUS_SEQ_LEN = 4
HYB_STATUS_TIMEOUT = 5
HYB_STATUS_BAD_TIER = 6

EXPORTED = (
    "hyb_check_desc", "hyb_kv_append", "hyb_decode_plan", "hyb_decode_workspace_bytes",
    "hyb_decode_attn", "hyb_decode_step", "hyb_decode_step_workspace_bytes", "hyb_combine",
    "hyb_read_status", "hyb_strerror",
    "hyb_last_cuda_error", "hyb_version", "hyb_decode_attn_noalloc", "hyb_noalloc_scratch_limit",
    "hyb_kv_migrate", "hyb_migration_threshold_ms", "hyb_migration_decision",
    "hyb_decode_attn_sparse", "hyb_decode_sparse_workspace_bytes", "hyb_decode_sparse_selection",
    "hyb_sparse_top_k", "hyb_set_wait_limit", "hyb_decode_launch_info", "hyb_stream_read",
)


class HybError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (what, strerror(code), code))


class CacheDesc(ctypes.Structure):
    """Mirror of hyb_cache_desc."""
    _fields_ = [
        ("hot_tokens", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("quant_bits", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_phys_blocks", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("hot", ctypes.c_void_p),
        ("cold", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("n_int4_blocks", ctypes.c_void_p),
        ("status", ctypes.c_void_p),
    ]


_lib = None


def load(path: str = LIB_PATH):
    """Load libhybkv.so (building it first if it is missing and nvcc exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        from . import build as _build
        _build.build()
    lib = ctypes.CDLL(path)
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(CacheDesc)
    lib.hyb_check_desc.argtypes = [D]
    lib.hyb_kv_append.argtypes = [D, P, i32, P, P, P]
    lib.hyb_decode_plan.argtypes = [D, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.hyb_decode_workspace_bytes.argtypes = [D, i32, i32]
    lib.hyb_decode_workspace_bytes.restype = sz
    lib.hyb_decode_launch_info.argtypes = [D, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                           ctypes.POINTER(i32)]
    lib.hyb_decode_launch_info.restype = ctypes.c_int
    lib.hyb_decode_attn.argtypes = [D, P, ctypes.c_float, i32, i32, P, sz, P, P, P]
    lib.hyb_decode_attn_sparse.argtypes = [D, P, ctypes.c_float, i32, i32, i32, P, sz, P, P, P]
    lib.hyb_decode_sparse_workspace_bytes.argtypes = [D, i32, i32]
    lib.hyb_decode_sparse_workspace_bytes.restype = sz
    lib.hyb_decode_sparse_selection.argtypes = [D, i32, i32, ctypes.POINTER(ctypes.c_int32)]
    lib.hyb_decode_sparse_selection.restype = sz
    lib.hyb_set_wait_limit.argtypes = [ctypes.c_int64]
    lib.hyb_sparse_top_k.argtypes = [ctypes.c_int64]
    lib.hyb_sparse_top_k.restype = i32
    lib.hyb_decode_step.argtypes = [D, P, P, P, P, ctypes.c_float, i32, i32, P, sz, P, P, P]
    lib.hyb_decode_step_workspace_bytes.argtypes = [D, i32, i32]
    lib.hyb_decode_step_workspace_bytes.restype = sz
    lib.hyb_combine.argtypes = [i32, i32, i32, i32, P, P, P, P, P]
    lib.hyb_decode_attn_noalloc.argtypes = [D, P, ctypes.c_float, i32, i32, P, P, P]
    lib.hyb_decode_attn_noalloc.restype = ctypes.c_int
    lib.hyb_noalloc_scratch_limit.argtypes = []
    lib.hyb_noalloc_scratch_limit.restype = sz
    lib.hyb_kv_migrate.argtypes = [D, P, i32, P]
    lib.hyb_migration_threshold_ms.argtypes = [ctypes.POINTER(i32), i32]
    lib.hyb_migration_threshold_ms.restype = ctypes.c_double
    lib.hyb_migration_decision.argtypes = [ctypes.c_double, ctypes.c_double, i32]
    lib.hyb_migration_decision.restype = ctypes.c_int
    lib.hyb_read_status.argtypes = [D, ctypes.POINTER(i32), i32, P]
    lib.hyb_stream_read.argtypes = [P, sz, P, P]
    lib.hyb_stream_read.restype = ctypes.c_int
    lib.hyb_strerror.argtypes = [ctypes.c_int]
    lib.hyb_strerror.restype = ctypes.c_char_p
    for name in ("hyb_check_desc", "hyb_kv_append", "hyb_decode_plan", "hyb_decode_attn", "hyb_decode_step",
                 "hyb_combine", "hyb_read_status", "hyb_last_cuda_error", "hyb_version", "hyb_kv_migrate"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().hyb_strerror(int(code)).decode()


def _check(rc, what):
    if rc != HYB_OK:
        raise HybError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def hyb_check_desc(desc: CacheDesc) -> int:
    return load().hyb_check_desc(ctypes.byref(desc))


def hyb_kv_append(desc, n_new, max_new, k_new, v_new, stream=None):
    _check(load().hyb_kv_append(ctypes.byref(desc), _ptr(n_new), int(max_new), _ptr(k_new),
                                _ptr(v_new), _stream(stream)), "hyb_kv_append")


def hyb_decode_plan(desc, max_seq_len, split_tokens=0):
    st, ns = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load().hyb_decode_plan(ctypes.byref(desc), int(max_seq_len), int(split_tokens),
                                  ctypes.byref(st), ctypes.byref(ns)), "hyb_decode_plan")
    return st.value, ns.value


KERNEL_NAMES = {0: "split_cta", 1: "cluster", 2: "persistent", 3: "persistent+combine"}


def hyb_decode_launch_info(desc, max_seq_len, split_tokens=0):
    """(kernel name, CTAs of the launch, CTAs per SM) of the decode launch."""
    k, c, o = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(load().hyb_decode_launch_info(ctypes.byref(desc), int(max_seq_len), int(split_tokens), ctypes.byref(k),
                                         ctypes.byref(c), ctypes.byref(o)), "hyb_decode_launch_info")
    return KERNEL_NAMES[k.value], c.value, o.value


def hyb_decode_workspace_bytes(desc, max_seq_len, split_tokens=0) -> int:
    return int(load().hyb_decode_workspace_bytes(ctypes.byref(desc), int(max_seq_len), int(split_tokens)))


def hyb_decode_attn(desc, q, softmax_scale, max_seq_len, split_tokens, workspace, out,
                    lse_out=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyb_decode_attn(ctypes.byref(desc), _ptr(q), float(softmax_scale), int(max_seq_len),
                                  int(split_tokens), _ptr(workspace), ws_bytes, _ptr(out),
                                  _ptr(lse_out), _stream(stream)), "hyb_decode_attn")


def hyb_decode_sparse_workspace_bytes(desc, max_seq_len, split_tokens=0) -> int:
    return int(load().hyb_decode_sparse_workspace_bytes(ctypes.byref(desc), int(max_seq_len), int(split_tokens)))


def hyb_decode_sparse_selection(desc, max_seq_len, split_tokens=0):
    """(byte offset in the sparse workspace, row stride) of the selected L2
    positions; raises on invalid arguments."""
    stride = ctypes.c_int32(0)
    off = int(load().hyb_decode_sparse_selection(ctypes.byref(desc), int(max_seq_len), int(split_tokens),
                                                  ctypes.byref(stride)))
    if off == 0:
        raise HybError(HYB_ERR_INVALID_VALUE, "hyb_decode_sparse_selection")
    return off, stride.value


def hyb_decode_attn_sparse(desc, q, softmax_scale, max_seq_len, split_tokens, top_k, workspace, out,
                           lse_out=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyb_decode_attn_sparse(ctypes.byref(desc), _ptr(q), float(softmax_scale), int(max_seq_len),
                                         int(split_tokens), int(top_k), _ptr(workspace), ws_bytes, _ptr(out),
                                         _ptr(lse_out), _stream(stream)), "hyb_decode_attn_sparse")


def hyb_sparse_top_k(context_length) -> int:
    return int(load().hyb_sparse_top_k(int(context_length)))


def hyb_decode_step_workspace_bytes(desc, max_seq_len, split_tokens=0) -> int:
    return int(load().hyb_decode_step_workspace_bytes(ctypes.byref(desc), int(max_seq_len), int(split_tokens)))


def hyb_decode_step(desc, n_new, k_new, v_new, q, softmax_scale, max_seq_len, split_tokens, workspace,
                    out, lse_out=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyb_decode_step(ctypes.byref(desc), _ptr(n_new), _ptr(k_new), _ptr(v_new), _ptr(q),
                                  float(softmax_scale), int(max_seq_len), int(split_tokens),
                                  _ptr(workspace), ws_bytes, _ptr(out), _ptr(lse_out), _stream(stream)),
           "hyb_decode_step")


def hyb_decode_attn_noalloc(desc, q, softmax_scale, max_seq_len, split_tokens, out, lse_out=None,
                            stream=None):
    """hyb_decode_attn with the library's static scratch buffer instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _check(load().hyb_decode_attn_noalloc(ctypes.byref(desc), _ptr(q), float(softmax_scale),
                                          int(max_seq_len), int(split_tokens), _ptr(out), _ptr(lse_out),
                                          _stream(stream)), "hyb_decode_attn_noalloc")


def hyb_noalloc_scratch_limit() -> int:
    return int(load().hyb_noalloc_scratch_limit())


def hyb_combine(batch, num_q_heads, head_dim, n_splits, o_partial, lse_partial, out,
                lse_out=None, stream=None):
    _check(load().hyb_combine(int(batch), int(num_q_heads), int(head_dim), int(n_splits),
                              _ptr(o_partial), _ptr(lse_partial), _ptr(out), _ptr(lse_out),
                              _stream(stream)), "hyb_combine")


def hyb_kv_migrate(desc, target_n_int4, max_delta, stream=None):
    """target_n_int4: int32 CUDA tensor [batch]; max_delta: host bound on the move."""
    _check(load().hyb_kv_migrate(ctypes.byref(desc), _ptr(target_n_int4), int(max_delta), _stream(stream)),
           "hyb_kv_migrate")


def hyb_migration_threshold_ms(seq_lens) -> float:
    """Adaptive migration threshold (ms) for host sequence lengths."""
    lens = [int(x) for x in seq_lens]
    arr = (ctypes.c_int32 * max(1, len(lens)))(*lens)
    return float(load().hyb_migration_threshold_ms(arr, len(lens)))


def hyb_migration_decision(avg_interval_ms, threshold_ms, block_is_int4) -> int:
    """+1 promote (INT4 -> INT8), -1 demote (INT8 -> INT4), 0 keep."""
    return int(load().hyb_migration_decision(float(avg_interval_ms), float(threshold_ms), 1 if block_is_int4 else 0))


def hyb_read_status(desc, clear=False, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(load().hyb_read_status(ctypes.byref(desc), ctypes.byref(v), 1 if clear else 0,
                                  _stream(stream)), "hyb_read_status")
    return v.value


def hyb_set_wait_limit(cycles: int) -> None:
    """Limit (SM cycles) of the decode pipeline's bounded waits; <= 0 restores the default."""
    _check(load().hyb_set_wait_limit(int(cycles)), "hyb_set_wait_limit")


def hyb_last_cuda_error() -> int:
    return load().hyb_last_cuda_error()


def hyb_stream_read(src, sink, stream=None) -> None:
    """One streaming read of the CUDA tensor `src` (contiguous, 16-byte aligned, nbytes a
    multiple of 16): XORs the XOR of its 32-bit words into the int32 CUDA tensor `sink`."""
    if not src.is_contiguous():
        raise HybError(HYB_ERR_INVALID_VALUE, "hyb_stream_read: src must be contiguous")
    _check(load().hyb_stream_read(_ptr(src), src.numel() * src.element_size(), _ptr(sink),
                                  _stream(stream)), "hyb_stream_read")


def hyb_version() -> int:
    return load().hyb_version()
