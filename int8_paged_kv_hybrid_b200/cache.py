"""HybridKVCache: device buffers of one hybrid_v2 cache plus its descriptor.

PyTorch only allocates the buffers and supplies the stream; appends and
attention go through the C ABI (libhybkv.so).  Layouts are those of
include/hyb_kv.h.
"""
from __future__ import annotations

import math

from . import _lib

HOT, BLOCK, HEAD_DIM = 32, 64, 128
TILE_BYTES = BLOCK * HEAD_DIM


class HybridKVCache:
    def __init__(self, batch, num_kv_heads, num_q_heads, num_phys_blocks, max_blocks_per_seq,
                 quant_bits=8, block_table=None, n_int4=None, device="cuda", hot_tokens=HOT,
                 block_size=BLOCK):
        import torch
        self.batch, self.hkv, self.hq = int(batch), int(num_kv_heads), int(num_q_heads)
        self.num_phys, self.max_blocks = int(num_phys_blocks), int(max_blocks_per_seq)
        self.quant_bits = int(quant_bits)
        self.hot_tokens = int(hot_tokens)
        self.block_size = int(block_size)
        dev = torch.device(device)
        self.device = dev
        self.hot = torch.zeros((self.batch, self.hkv, self.hot_tokens, 2, HEAD_DIM), dtype=torch.float16,
                               device=dev)
        # 8 KB parts per block and kv head: K and V tiles of each 64-token
        # sub-block (a 32-token block uses half of one); FP16 blocks
        # (quant_bits 0) hold 512-byte rows of K then V
        parts = self.block_size // 16 if self.quant_bits == 0 else 2 * max(1, self.block_size // BLOCK)
        self.cold = torch.zeros((self.num_phys, self.hkv, parts, TILE_BYTES), dtype=torch.uint8, device=dev)
        self.scales = torch.zeros((self.num_phys, self.hkv, 2), dtype=torch.float32, device=dev)
        if block_table is None:
            self.block_table = torch.full((self.batch, self.max_blocks), -1, dtype=torch.int32, device=dev)
        else:
            self.block_table = torch.as_tensor(block_table, dtype=torch.int32).to(dev).contiguous()
            assert tuple(self.block_table.shape) == (self.batch, self.max_blocks)
        self.seq_lens = torch.zeros(self.batch, dtype=torch.int32, device=dev)
        self.n_int4 = None
        if n_int4 is not None:
            self.n_int4 = torch.as_tensor(n_int4, dtype=torch.int32).to(dev).contiguous()
        self.status_word = torch.zeros(1, dtype=torch.int32, device=dev)
        self.desc = self._make_desc()
        rc = _lib.hyb_check_desc(self.desc)
        if rc != _lib.HYB_OK:
            raise _lib.HybError(rc, "hyb_check_desc")

    def _make_desc(self):
        d = _lib.CacheDesc()
        d.hot_tokens, d.block_size, d.head_dim = self.hot_tokens, self.block_size, HEAD_DIM
        d.quant_bits = self.quant_bits
        d.num_kv_heads, d.num_q_heads = self.hkv, self.hq
        d.num_phys_blocks, d.max_blocks_per_seq, d.batch = self.num_phys, self.max_blocks, self.batch
        d.reserved = 0
        d.hot = self.hot.data_ptr()
        d.cold = self.cold.data_ptr()
        d.scales = self.scales.data_ptr()
        d.block_table = self.block_table.data_ptr()
        d.seq_lens = self.seq_lens.data_ptr()
        d.n_int4_blocks = None if self.n_int4 is None else self.n_int4.data_ptr()
        d.status = self.status_word.data_ptr()
        return d

    # ---- the three calls ----
    def append(self, n_new, k_new, v_new, stream=None):
        """n_new: int32 CUDA [batch]; k_new, v_new: FP16 CUDA [batch][max_new][Hkv][128]."""
        assert k_new.is_contiguous() and v_new.is_contiguous() and n_new.is_contiguous()
        _lib.hyb_kv_append(self.desc, n_new, k_new.shape[1], k_new, v_new, stream)

    def migrate(self, target_n_int4, max_delta=None, stream=None):
        """Move every sequence's INT4 block count to target_n_int4 (int32
        [batch], host or CUDA), re-quantizing the blocks in between in place
        (hyb_kv_migrate).  max_delta: bound on the move (default: the table width)."""
        import torch
        if self.n_int4 is None:
            self.n_int4 = torch.zeros(self.batch, dtype=torch.int32, device=self.device)
            self.desc = self._make_desc()
        tgt = torch.as_tensor(target_n_int4, dtype=torch.int32).to(self.device).contiguous()
        md = self.max_blocks if max_delta is None else int(max_delta)
        _lib.hyb_kv_migrate(self.desc, tgt, md, stream)

    def plan(self, max_seq_len, split_tokens=0):
        return _lib.hyb_decode_plan(self.desc, max_seq_len, split_tokens)

    def launch_info(self, max_seq_len, split_tokens=0):
        """(kernel, CTAs, CTAs per SM) of the decode launch for these arguments."""
        return _lib.hyb_decode_launch_info(self.desc, max_seq_len, split_tokens)

    def workspace(self, max_seq_len, split_tokens=0):
        import torch
        n = _lib.hyb_decode_workspace_bytes(self.desc, max_seq_len, split_tokens)
        return None if n == 0 else torch.zeros(n, dtype=torch.uint8, device=self.device)

    def decode(self, q, softmax_scale, max_seq_len, split_tokens=0, out=None, lse=None,
               workspace=None, stream=None):
        """q: FP16 CUDA [batch][Hq][128] -> out FP16 [batch][Hq][128] (and lse FP32 [batch][Hq])."""
        import torch
        assert q.is_contiguous()
        if out is None:
            out = torch.empty((self.batch, self.hq, HEAD_DIM), dtype=torch.float16, device=self.device)
        if workspace is None:
            workspace = self.workspace(max_seq_len, split_tokens)
        _lib.hyb_decode_attn(self.desc, q, softmax_scale, max_seq_len, split_tokens, workspace,
                             out, lse, stream)
        return out

    def sparse_workspace(self, max_seq_len, split_tokens=0):
        import torch
        n = _lib.hyb_decode_sparse_workspace_bytes(self.desc, max_seq_len, split_tokens)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=self.device)

    def decode_sparse(self, q, softmax_scale, max_seq_len, top_k, split_tokens=0, out=None, lse=None,
                      workspace=None, stream=None):
        """As decode, but each query head attends only the top_k of the tokens
        in its sequence's INT4 (L2) blocks (hyb_decode_attn_sparse)."""
        import torch
        assert q.is_contiguous()
        if out is None:
            out = torch.empty((self.batch, self.hq, HEAD_DIM), dtype=torch.float16, device=self.device)
        if workspace is None:
            workspace = self.sparse_workspace(max_seq_len, split_tokens)
        _lib.hyb_decode_attn_sparse(self.desc, q, softmax_scale, max_seq_len, split_tokens, top_k, workspace,
                                    out, lse, stream)
        return out

    def sparse_selection(self, workspace, max_seq_len, split_tokens=0):
        """The selected L2 positions the last decode_sparse call with this
        workspace left: int32 CUDA view [batch][Hq][stride] (row (b, h): the
        first min(top_k, L2 tokens of b) entries, ascending)."""
        import torch
        off, stride = _lib.hyb_decode_sparse_selection(self.desc, max_seq_len, split_tokens)
        n = self.batch * self.hq * stride * 4
        return workspace[off:off + n].view(torch.int32).view(self.batch, self.hq, stride)

    def step_workspace(self, max_seq_len, split_tokens=0):
        import torch
        n = _lib.hyb_decode_step_workspace_bytes(self.desc, max_seq_len, split_tokens)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=self.device)

    def step(self, n_new, k_new, v_new, q, softmax_scale, max_seq_len, split_tokens=0, out=None,
             lse=None, workspace=None, stream=None):
        """Fused decode step: append n_new[b] in {0, 1} tokens (k_new, v_new FP16
        [batch][1][Hkv][128]) and attend q; max_seq_len bounds the new lengths."""
        import torch
        assert q.is_contiguous() and k_new.is_contiguous() and v_new.is_contiguous()
        if out is None:
            out = torch.empty((self.batch, self.hq, HEAD_DIM), dtype=torch.float16, device=self.device)
        if workspace is None:
            workspace = self.step_workspace(max_seq_len, split_tokens)
        _lib.hyb_decode_step(self.desc, n_new, k_new, v_new, q, softmax_scale, max_seq_len, split_tokens,
                             workspace, out, lse, stream)
        return out

    def status(self, clear=False, stream=None):
        return _lib.hyb_read_status(self.desc, clear, stream)


def default_softmax_scale(head_dim=HEAD_DIM):
    return 1.0 / math.sqrt(head_dim)
