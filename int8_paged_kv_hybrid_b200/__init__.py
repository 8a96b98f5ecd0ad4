"""B200 (sm_100a) decode attention over the hybrid_v2 two-tier KV cache.

The hot zone keeps the most recent hot_tokens (32 by default) of every
sequence in FP16; older tokens live in 64-token INT8 (or INT4, or FP16) cold
blocks behind a block table.  The library (libhybkv.so, C ABI in
include/hyb_kv.h) provides the append / quantize kernel, the split-KV decode
attention kernel (dense, fused with the append, or sparse over the INT4 "L2"
blocks), the log-sum-exp combine and the INT8 <-> INT4 tier migration.  This
package is its thin Python binding.
"""
from ._lib import (  # noqa: F401
    CacheDesc, HybError, hyb_check_desc, hyb_combine, hyb_decode_attn, hyb_decode_plan, hyb_decode_launch_info,
    hyb_decode_attn_sparse, hyb_decode_sparse_workspace_bytes, hyb_decode_step,
    hyb_decode_step_workspace_bytes, hyb_sparse_top_k,
    hyb_decode_workspace_bytes, hyb_kv_append, hyb_kv_migrate, hyb_last_cuda_error,
    hyb_migration_decision, hyb_migration_threshold_ms, hyb_read_status, hyb_stream_read, hyb_version, load,
    strerror,
)
from .cache import HybridKVCache  # noqa: F401
