"""Host-side checks of the C ABI (no GPU): exported symbols, the hybrid_v2
configuration contract, split planning and workspace sizing."""
import ctypes
import os
import re

import numpy as np
import pytest

import int8_paged_kv_hybrid_b200 as hk
from int8_paged_kv_hybrid_b200 import _lib, synth
from golden_cases import GOLDEN

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn), encoding="utf-8").read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"^[A-Za-z_][\w \*]*?\b(hyb_\w+)\s*\(", text, flags=re.M))
    return names


def test_library_exports_every_declared_symbol():
    lib = hk.load()
    declared = _declared_functions()
    assert {"hyb_kv_append", "hyb_decode_attn", "hyb_combine"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTED) <= declared


def _desc(hot=32, block=64, qbits=8, d=128, hkv=8, hq=32, batch=2, phys=16, maxb=4):
    x = _lib.CacheDesc()
    x.hot_tokens, x.block_size, x.head_dim, x.quant_bits = hot, block, d, qbits
    x.num_kv_heads, x.num_q_heads, x.num_phys_blocks = hkv, hq, phys
    x.max_blocks_per_seq, x.batch, x.reserved = maxb, batch, 0
    base = 0x7f0000000000
    x.hot, x.cold, x.scales = base, base + 0x100000, base + 0x200000
    x.block_table, x.seq_lens, x.status = base + 0x300000, base + 0x310000, base + 0x320000
    x.n_int4_blocks = None
    return x


def test_config_contract_golden():
    """hot_tokens / block_size / quantization_bits per the page (sections 3.1, 5.1)."""
    codes = {"ok": 0, "invalid": _lib.HYB_ERR_INVALID_VALUE, "unsupported": _lib.HYB_ERR_UNSUPPORTED}
    n = 0
    for line in open(os.path.join(GOLDEN, "config_contract.txt"), encoding="utf-8"):
        f = line.split("#", 1)[0].split()
        if not f:
            continue
        hot, block, qbits, want = int(f[0]), int(f[1]), int(f[2]), f[3]
        assert hk.hyb_check_desc(_desc(hot=hot, block=block, qbits=qbits)) == codes[want], f
        n += 1
    assert n >= 10


def test_descriptor_rejections():
    ok = _desc()
    assert hk.hyb_check_desc(ok) == 0
    for field, val, want in [
        ("head_dim", 64, _lib.HYB_ERR_UNSUPPORTED),
        ("num_q_heads", 30, _lib.HYB_ERR_INVALID_VALUE),    # not a multiple of Hkv
        ("num_q_heads", 72, _lib.HYB_ERR_UNSUPPORTED),      # group of 9
        ("batch", 0, _lib.HYB_ERR_INVALID_VALUE),
        ("max_blocks_per_seq", 0, _lib.HYB_ERR_INVALID_VALUE),
        ("reserved", 1, _lib.HYB_ERR_INVALID_VALUE),
        ("hot", 0x7f0000000100, _lib.HYB_ERR_INVALID_VALUE),  # hot zone not 512-byte aligned
        ("cold", 0x7f0000100008, _lib.HYB_ERR_INVALID_VALUE),
        ("status", None, _lib.HYB_ERR_INVALID_VALUE),
    ]:
        d = _desc()
        setattr(d, field, val)
        assert hk.hyb_check_desc(d) == want, (field, val)
    assert hk.load().hyb_check_desc(None) == _lib.HYB_ERR_INVALID_VALUE


def _splits(L, st, hot=32, block=64, qbits=8):
    """Splits of a sequence of L tokens at st tokens per split: the cold
    blocks plus the hot ring's items counted as blocks (capped at a split)."""
    tb = st // block
    nblk = -(-max(0, L - hot) // block)
    ipb = block // 32 if qbits == 0 else (2 if block == 128 else 1)
    dh = -(-min(L, hot) // 32)
    dhb = min(-(-dh // ipb), tb)
    return max(1, -(-(nblk + dhb) // tb))


def test_plan_and_workspace():
    d = _desc(batch=4, maxb=2048, phys=8192)
    st, ns = hk.hyb_decode_plan(d, 131072, 512)
    assert st == 512 and ns == 257      # ceil((2048 cold blocks + 1 hot item) / 8)
    st, ns = hk.hyb_decode_plan(d, 32768, 512)
    assert ns == 65                     # the page's 32K context: >= 64 splits at 512 tokens
    st, ns = hk.hyb_decode_plan(d, 32, 512)
    assert ns == 1 and hk.hyb_decode_workspace_bytes(d, 32, 512) == 0
    ws = hk.hyb_decode_workspace_bytes(d, 131072, 512)
    rows = 4 * 32
    assert ws >= rows * 257 * 128 * 4 + rows * 257 * 4
    for bad in (100, -65536, 64 * 129):
        with pytest.raises(hk.HybError):
            hk.hyb_decode_plan(d, 4096, bad)
    with pytest.raises(hk.HybError):
        hk.hyb_decode_plan(d, 64 * 2048 + 33, 0)  # longer than the block table allows
    # automatic splits: a multiple of 64 tokens, at most 8192
    for L in (33, 1000, 2048, 131072):
        st, ns = hk.hyb_decode_plan(d, L, 0)
        assert st % 64 == 0 and 64 <= st <= 8192 and ns >= 1
        assert ns == _splits(L, st)
    # one wave when every split fits on the GPU at once: 4 x 8 rows, splits of
    # at least 6 blocks (33 items -> 6 splits)
    assert hk.hyb_decode_plan(d, 2048, 0) == (384, 6)


def _per_seq_splits(c, n):
    """Splits of a sequence of c items (cold blocks + 1 for the hot ring) when
    at least n per sequence are asked for: near-equal runs of <= 32 items."""
    if c <= 0:
        return 1
    return min(c, max(n, -(-c // 32)))


def test_plan_per_sequence_splits():
    """split_tokens = -n: every sequence cut into at least n near-equal splits
    (one per item when it has fewer), none longer than 32 blocks."""
    d = _desc(batch=4, maxb=2048, phys=8192)
    st, ns = hk.hyb_decode_plan(d, 131072, -64)
    assert (st, ns) == (32 * 64, 65)    # 2048 cold blocks + the ring = 2049 items
    st, ns = hk.hyb_decode_plan(d, 32768, -64)
    assert (st, ns) == (9 * 64, 64)     # 513 items: runs of 8 or 9
    assert hk.hyb_decode_plan(d, 20, -64) == (64, 1)
    assert hk.hyb_decode_plan(d, 0, -3) == (64, 1)
    for L in (33, 100, 1000, 5000, 131072):
        nblk = -(-max(0, L - 32) // 64)
        assert hk.hyb_decode_plan(d, L, -5)[1] == _per_seq_splits(nblk + 1, 5)
    # the split ranges the kernel uses: every item once, runs of 1..32, at
    # least min(n, c) of them, and never more splits for a shorter sequence
    for n in (1, 3, 64, 200):
        prev = 1
        for c in range(0, 7000, 3):
            S = _per_seq_splits(c, n)
            assert S >= prev
            prev = S
            if c == 0:
                assert S == 1
                continue
            edges = [s * c // S for s in range(S + 1)]
            assert edges[0] == 0 and edges[-1] == c
            assert all(1 <= edges[i + 1] - edges[i] <= 32 for i in range(S))
            assert S >= min(n, c)
    ws = hk.hyb_decode_workspace_bytes(d, 131072, -64)
    assert ws >= 4 * 32 * 65 * 128 * 4
    # caches the persistent kernel does not take (FP16 cold blocks): every
    # sequence takes the longest one's split length
    d0 = _desc(batch=4, maxb=2048, phys=8192, qbits=0)
    st, ns = hk.hyb_decode_plan(d0, 32768, -64)
    assert st == 9 * 64 and ns == _splits(32768, st, qbits=0)
    # the sparse path takes no per-sequence splits
    assert hk.hyb_decode_sparse_workspace_bytes(d, 32768, -64) == 0


def test_launch_info():
    """The kernel a plan launches: per-sequence splits and several waves of
    splits take the persistent kernel, one wave of a few splits the
    one-CTA-per-split kernel; FP16 cold blocks never the persistent one."""
    d = _desc(batch=4, maxb=2048, phys=8192)
    # more than 16 splits per sequence: partials, then a merge launch
    kern, ctas, occ = hk.hyb_decode_launch_info(d, 131072, -64)
    assert kern == "persistent+combine" and 1 <= ctas <= 4 * 8 * 65 and occ >= 0
    kern, ctas, _ = hk.hyb_decode_launch_info(d, 131072, 512)
    assert kern == "persistent+combine" and ctas <= 4 * 8 * 257
    # up to 16: merged inside the launch
    kern, ctas, _ = hk.hyb_decode_launch_info(d, 8192, -8)
    assert kern == "persistent" and hk.hyb_decode_plan(d, 8192, -8)[1] == 8
    kern, ctas, _ = hk.hyb_decode_launch_info(d, 100, 64)
    assert kern == "split_cta" and ctas == 4 * 8 * hk.hyb_decode_plan(d, 100, 64)[1]
    d0 = _desc(batch=4, maxb=2048, phys=8192, qbits=0)
    assert hk.hyb_decode_launch_info(d0, 131072, -64)[0] != "persistent"
    with pytest.raises(hk.HybError):
        hk.hyb_decode_launch_info(d, 4096, 100)


def test_automatic_multiwave_split_length_by_head_group():
    """Several waves of splits on the persistent kernel: the automatic plan's
    longest split is 32 blocks for head groups of up to 4 and 24 above (a
    wider group's block costs about twice the arithmetic, so shorter units
    keep the tail of the launch short)."""
    w3, w5 = synth.make_workload(3), synth.make_workload(5)
    for w, want in ((w3, 32 * 64), (w5, 24 * 64)):
        d = _desc(batch=w.batch, maxb=w.max_blocks, phys=w.num_phys_blocks, hkv=w.num_kv_heads,
                  hq=w.num_q_heads)
        L = int(w.lens.max())
        tokens, ns = hk.hyb_decode_plan(d, L, 0)
        nblk = -(-(L - 32) // 64)
        assert tokens == want and ns == -(-(nblk + 1) // (want // 64)), (w.name, tokens, ns)
        assert hk.hyb_decode_launch_info(d, L, 0)[0] == "persistent"


@pytest.mark.parametrize("block,hot", [(32, 16), (128, 64), (64, 128)])
def test_plan_other_block_and_hot_sizes(block, hot):
    """Splits count blocks of the descriptor's size; the cold range is the
    length minus the hot zone."""
    d = _desc(hot=hot, block=block, batch=4, maxb=4096, phys=8192)
    for L in (hot + 1, 1000, 40000):
        st, ns = hk.hyb_decode_plan(d, L, 0)
        assert st % block == 0 and st >= block and ns == _splits(L, st, hot, block)
    st, ns = hk.hyb_decode_plan(d, 40000, 4 * block)
    assert st == 4 * block and ns == _splits(40000, st, hot, block)
    for bad in (block // 2, 3 * block + 8):
        with pytest.raises(hk.HybError):
            hk.hyb_decode_plan(d, 4096, bad)
    # the block table bounds the length in blocks of this size
    with pytest.raises(hk.HybError):
        hk.hyb_decode_plan(d, block * 4096 + hot + 1, 0)


def test_strerror_covers_codes():
    for c in (0, -1, -2, -3, -4, 100, 101, 102, 103, 104, 105):
        assert hk.strerror(c) and hk.strerror(c) != "unknown code"
    assert hk.strerror(12345) == "unknown code"


def test_kv_bytes_formula():
    """Algorithmic bytes of the Llama-3-8B batch-8 L-2048 workload: 8 x 8
    heads x (2016 cold tokens x 256 B + 32 hot x 512 B + 32 blocks x 8 B) +
    8 x 32 block-table entries x 4 B + q and out (8 x 32 x 128 x 2 B each);
    all-INT4 cold blocks halve the codes, FP16 ones double them and drop the
    scales."""
    w = synth.make_workload(2)
    want = 8 * 8 * (2016 * 256 + 32 * 512 + 32 * 8) + 8 * 32 * 4 + 2 * 8 * 32 * 128 * 2
    assert synth.kv_bytes(w) == want
    assert abs(want / 1e6 - 34.2) < 0.5   # "34.2 MB"
    assert synth.kv_bytes(w, quant_bits=4) == want - 8 * 8 * 2016 * 128
    assert synth.kv_bytes(w, quant_bits=0) == want + 8 * 8 * (2016 * 256 - 32 * 8)
    n = np.ones(8, np.int32)
    assert synth.append_bytes(w, n) == 8 * 8 * (1024 + 264)
    assert synth.append_bytes(w, n, quant_bits=0) == 8 * 8 * (1024 + 512)


def test_workload_shapes():
    w = synth.make_workload(4)
    assert list(w.lens) == [32768, 32768, 131072, 131072] and w.split_tokens == -64
    w5 = synth.make_workload(5)
    assert w5.num_q_heads == 28 and w5.num_kv_heads == 4 and w5.batch == 128
    nb = w5.cold_blocks()
    assert np.array_equal(w5.n_int4, nb // 4)
    w3 = synth.make_workload(3)
    assert w3.lens.min() >= 256 and w3.lens.max() <= 8192 and w3.outlier_channels.shape == (8, 4)
    for w in (synth.make_workload(i) for i in (1, 2, 3, 4, 5)):
        used = w.block_table[w.block_table >= 0]
        assert len(np.unique(used)) == len(used) and used.max() < w.num_phys_blocks
        assert sum(int(s.sum()) for s in w.schedule) == int(w.lens.sum())


def test_migration_policy_matches_fixture_and_oracle():
    """hyb_migration_threshold_ms / hyb_migration_decision (host functions)
    against the page's worked example (tests/golden/migration_threshold.txt)
    and the oracle's restatement on random batches."""
    import oracle
    for line in open(os.path.join(GOLDEN, "migration_threshold.txt"), encoding="utf-8"):
        f = line.split("#", 1)[0].split()
        if f:
            want, lens = float(f[0]), [int(x) for x in f[1:]]
            assert abs(hk.hyb_migration_threshold_ms(lens) - want) <= 1e-9 * want, lens
    rng = np.random.default_rng(5)
    for _ in range(50):
        lens = rng.integers(0, 200000, size=int(rng.integers(1, 64))).tolist()
        t = hk.hyb_migration_threshold_ms(lens)
        assert abs(t - oracle.migration_threshold_ms(lens)) <= 1e-9 * t
        for iai in (0.5 * t, t, 1.2 * t, 1.5 * t, 2.0 * t):
            for int4 in (True, False):
                assert hk.hyb_migration_decision(iai, t, int4) == oracle.migration_decision(iai, t, int4)


def test_sparse_argument_checks():
    """hyb_decode_attn_sparse rejects bad arguments on the host, before any launch."""
    lib = hk.load()
    d = _desc(batch=4, maxb=16, phys=64)
    q = ctypes.c_void_p(0x7f0000400000)
    out = ctypes.c_void_p(0x7f0000500000)
    ws = ctypes.c_void_p(0x7f0000600000)
    need = lib.hyb_decode_sparse_workspace_bytes(ctypes.byref(d), 1000, 0)
    assert need >= 4 * 8 * 4 + 4 * 8 * 1024 * 4  # lse rows + keys [4][8][max_l2 = 1024]
    for top_k in (-1, 1025):
        assert lib.hyb_decode_attn_sparse(ctypes.byref(d), q, ctypes.c_float(0.1), 1000, 0, top_k, ws, need,
                                          out, None, None) == _lib.HYB_ERR_INVALID_VALUE
    assert lib.hyb_decode_attn_sparse(ctypes.byref(d), q, ctypes.c_float(0.1), 1000, 0, 32, ws, need - 1,
                                      out, None, None) == _lib.HYB_ERR_WORKSPACE
    d0 = _desc(batch=4, maxb=16, phys=64, qbits=0)
    assert lib.hyb_decode_attn_sparse(ctypes.byref(d0), q, ctypes.c_float(0.1), 1000, 0, 32, ws, need,
                                      out, None, None) == _lib.HYB_ERR_UNSUPPORTED
    # the page's rule, section 5.3
    assert [hk.hyb_sparse_top_k(x) for x in (32768, 8192, 255, -5, 10 ** 9)] == [128, 32, 0, 0, 128]


def test_migrate_argument_checks():
    """hyb_kv_migrate rejects bad arguments on the host, before any launch."""
    lib = hk.load()
    d = _desc(batch=4, maxb=16, phys=64)
    tgt = ctypes.c_void_p(0x7f0000400000)
    # no per-sequence INT4 counts to move
    assert lib.hyb_kv_migrate(ctypes.byref(d), tgt, 1, None) == _lib.HYB_ERR_INVALID_VALUE
    d.n_int4_blocks = 0x7f0000330000
    assert lib.hyb_kv_migrate(ctypes.byref(d), None, 1, None) == _lib.HYB_ERR_INVALID_VALUE
    assert lib.hyb_kv_migrate(ctypes.byref(d), ctypes.c_void_p(0x7f0000400002), 1, None) == \
        _lib.HYB_ERR_INVALID_VALUE  # misaligned target
    for bad in (-1, 17):
        assert lib.hyb_kv_migrate(ctypes.byref(d), tgt, bad, None) == _lib.HYB_ERR_INVALID_VALUE
    d4 = _desc(batch=4, maxb=16, phys=64, qbits=4)
    d4.n_int4_blocks = 0x7f0000330000
    assert lib.hyb_kv_migrate(ctypes.byref(d4), tgt, 1, None) == _lib.HYB_ERR_UNSUPPORTED
    d0 = _desc(batch=4, maxb=16, phys=64, qbits=0)  # FP16 cold blocks have no tiers
    d0.n_int4_blocks = 0x7f0000330000
    assert lib.hyb_kv_migrate(ctypes.byref(d0), tgt, 1, None) == _lib.HYB_ERR_UNSUPPORTED
    assert "migration" in hk.strerror(100 + _lib.HYB_STATUS_BAD_TIER)


def test_stream_read_argument_checks():
    """hyb_stream_read rejects null, misaligned and ragged arguments on the host; a
    zero-byte read launches nothing."""
    lib = hk.load()
    src, sink = ctypes.c_void_p(0x7f0000400000), ctypes.c_void_p(0x7f0000500000)
    bad = _lib.HYB_ERR_INVALID_VALUE
    assert lib.hyb_stream_read(None, 16, sink, None) == bad
    assert lib.hyb_stream_read(src, 16, None, None) == bad
    assert lib.hyb_stream_read(ctypes.c_void_p(0x7f0000400008), 16, sink, None) == bad  # src not 16-aligned
    assert lib.hyb_stream_read(src, 16, ctypes.c_void_p(0x7f0000500002), None) == bad  # sink not 4-aligned
    assert lib.hyb_stream_read(src, 24, sink, None) == bad  # not a multiple of 16 bytes
    assert lib.hyb_stream_read(src, 0, sink, None) == _lib.HYB_OK
