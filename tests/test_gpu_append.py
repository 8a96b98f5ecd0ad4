"""hyb_kv_append on the GPU: bit-exact against the CPU oracle (codes after
packing, FP32 scales as bits, hot ring, seq_lens) and against the hand-worked
golden values; device-side error handling."""
import numpy as np
import pytest

import oracle
from golden_cases import parse_cases, token_arrays
from harness import assert_cache_equal, make_pair, replay
from int8_paged_kv_hybrid_b200 import synth

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


@pytest.mark.parametrize("fname,name", [("quant_first_write.txt", "int8_first_write"),
                                        ("quant_first_write.txt", "int4_first_write"),
                                        ("quant_requant.txt", "int8_requant")])
def test_golden_values_on_gpu(fname, name):
    """The GPU reproduces the hand-worked codes and scales directly."""
    torch = _torch()
    from int8_paged_kv_hybrid_b200 import HybridKVCache
    case = parse_cases(fname)[name]
    qb = case["quant_bits"]
    phys = 1
    cache = HybridKVCache(1, 1, 1, num_phys_blocks=2, max_blocks_per_seq=2, quant_bits=qb,
                          block_table=np.array([[phys, 0]], np.int32))
    pos = 0
    for op, arg in case["ops"]:
        if op == "append":
            k, v = token_arrays(case, pos, arg)
            cache.append(torch.tensor([arg], dtype=torch.int32, device="cuda"),
                         torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            pos += arg
            continue
        torch.cuda.synchronize()
        kv = {"K": 0, "V": 1}[arg["kv"]]
        if "scale" in arg:
            assert cache.scales[phys, 0, kv].item() == np.float32(float(arg["scale"]))
        if arg["codes"] is not None:
            slot = int(arg["slot"])
            tile = cache.cold[phys, 0, kv].cpu().numpy()
            for ch in range(128):
                want = arg["codes"].get(ch, 0)
                if qb == 8 and kv == 0:
                    got = int(tile[slot * 128 + ch].astype(np.int8))
                elif qb == 8:
                    got = int(tile[ch * 64 + 16 * ((slot // 16) ^ ((ch // 2) % 4)) + slot % 16].astype(np.int8))
                elif kv == 0:
                    byte = tile[slot * 64 + 4 * (ch // 8) + (ch % 8) % 4]
                    nib = (int(byte) >> (4 if ch % 8 >= 4 else 0)) & 0xF
                    got = nib - 16 if nib >= 8 else nib
                else:
                    in_u = slot % 16
                    unit = (slot // 16) ^ ((ch // 4) % 4)
                    byte = tile[ch * 32 + unit * 8 + 4 * (in_u // 8) + (in_u % 8) % 4]
                    nib = (int(byte) >> (4 if in_u % 8 >= 4 else 0)) & 0xF
                    got = nib - 16 if nib >= 8 else nib
                assert got == want, (name, arg, ch, got, want)
    assert cache.status() == 0


@pytest.mark.parametrize("hkv,hq,qbits,int4", [(1, 1, 8, False), (2, 8, 8, True), (2, 2, 4, False),
                                               (4, 28, 8, True), (2, 8, 0, False)])
def test_random_schedule_bit_exact(hkv, hq, qbits, int4):
    """Random 1..70-token appends; the whole cache is compared after every call."""
    lens = [0, 1, 31, 32, 33, 97, 200, 333]
    nb = [synth.cold_blocks_for(L) for L in lens]
    w = synth.custom_workload("rand", lens, hq, hkv, seed=77 + hkv + qbits, max_step=70,
                              n_int4=[n // 2 for n in nb] if int4 else None)
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora, check_every=1)
    assert_cache_equal(w, cache, ora, "final")


@pytest.mark.parametrize("hot,qbits", [(16, 8), (64, 8), (128, 4), (64, 0)])
def test_hot_sizes_bit_exact(hot, qbits):
    """hot_tokens 16 / 64 / 128: ring of that many slots, sealing at L - hot."""
    lens = [0, 1, hot - 1, hot, hot + 1, hot + 63, hot + 64, 400]
    w = synth.custom_workload("hot%d" % hot, lens, 8, 2, seed=hot + qbits, max_step=70, hot=hot)
    cache, ora = make_pair(w, quant_bits=qbits)
    replay(w, cache, ora, check_every=1)
    assert_cache_equal(w, cache, ora, "final")


def test_outliers_and_big_appends_bit_exact():
    """Outlier K channels (x10) and single calls sealing many blocks at once."""
    lens = [1000, 90, 5000]
    w = synth.custom_workload("big", lens, 8, 8, seed=5, schedule="one", outliers=True)
    cache, ora = make_pair(w)
    replay(w, cache, ora)
    assert_cache_equal(w, cache, ora)
    # then a few 1-token decode steps
    torch = _torch()
    for step in range(3):
        n = np.ones(w.batch, np.int32)
        k, v = synth.step_tokens(w, 1000 + step, n, max_new=1)
        ora.append(n, k, v)
        cache.append(torch.from_numpy(n).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    w.lens = w.lens + 3
    # the block table has room: cold blocks of L+3 may need one more block
    assert_cache_equal(w, cache, ora, "after decode steps")


def test_device_errors_set_status_without_fault():
    """n_new > max_new and a sequence outgrowing its table leave the sequence
    untouched; an out-of-range block-table entry skips that block.  The
    first error code sticks."""
    torch = _torch()
    from int8_paged_kv_hybrid_b200 import HybridKVCache, _lib
    bt = np.array([[0, 1], [2, -1], [7, 3]], np.int32)   # -1 and 7 are outside a 4-block pool
    cache = HybridKVCache(3, 1, 1, num_phys_blocks=4, max_blocks_per_seq=2, block_table=bt)
    z = torch.zeros((3, 8, 1, 128), dtype=torch.float16, device="cuda")
    cache.append(torch.tensor([9, 0, 0], dtype=torch.int32, device="cuda"), z, z)
    assert cache.status(clear=True) == _lib.HYB_STATUS_BAD_N_NEW
    assert cache.seq_lens.tolist() == [0, 0, 0]
    big = torch.ones((3, 200, 1, 128), dtype=torch.float16, device="cuda")
    cache.append(torch.tensor([0, 0, 161], dtype=torch.int32, device="cuda"), big, big)  # needs 3 blocks
    assert cache.status(clear=True) == _lib.HYB_STATUS_CAPACITY
    assert cache.seq_lens.tolist() == [0, 0, 0]
    cache.append(torch.tensor([0, 0, 100], dtype=torch.int32, device="cuda"), big, big)
    torch.cuda.synchronize()
    assert cache.status(clear=True) == _lib.HYB_STATUS_BAD_BLOCK   # block 0 -> phys 7
    assert cache.seq_lens.tolist() == [0, 0, 100]
    # block 1 -> phys 3 was still written
    assert cache.scales[3, 0, 0].item() == np.float32(1.0) / np.float32(127.0)
    assert cache.status() == 0
