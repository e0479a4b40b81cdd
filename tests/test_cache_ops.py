"""reshape_and_cache and copy_blocks on the GPU, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import bits_of, prepare, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _flag():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("name", ["tiny", "longtail"])
def test_reshape_and_cache_workloads(pa, orc, name):
    prep = prepare(W.WORKLOADS[name])
    s = prep.case.spec
    kc, vc = prep.k_pool.copy(), prep.v_pool.copy()
    orc.reshape_and_cache(prep.case.new_k, prep.case.new_v, kc, vc, prep.new_slots)
    dk, dv = to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype)
    flag = _flag()
    pa.reshape_and_cache(to_dev(prep.case.new_k, s.dtype), to_dev(prep.case.new_v, s.dtype),
                         dk, dv, to_dev(prep.new_slots), error_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(dk), kc)
    assert np.array_equal(bits_of(dv), vc)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("bs", [128, 256])
def test_reshape_and_copy_large_blocks(pa, orc, bs):
    """Blocks of 128 and 256 tokens (512 KiB per pool at 8 KV heads of 128):
    new rows land bit-exact, and copy_blocks copies whole large blocks."""
    spec = W.WORKLOADS["longtail"].replace(num_seqs=24, new_rows=24, block_size=bs, seed=50 + bs)
    prep = prepare(spec)
    s = prep.case.spec
    kc, vc = prep.k_pool.copy(), prep.v_pool.copy()
    orc.reshape_and_cache(prep.case.new_k, prep.case.new_v, kc, vc, prep.new_slots)
    nb = kc.shape[0]
    pairs = np.stack([np.arange(0, nb // 2, 3), np.arange(nb // 2, nb, 3)[:len(range(0, nb // 2, 3))]],
                     axis=1).astype(np.int32)
    orc.copy_blocks([kc, vc], pairs, int(np.prod(kc.shape[1:])) * 2)
    dk, dv = to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype)
    flag = _flag()
    pa.reshape_and_cache(to_dev(prep.case.new_k, s.dtype), to_dev(prep.case.new_v, s.dtype),
                         dk, dv, to_dev(prep.new_slots), error_flag=flag)
    pa.copy_blocks([dk], [dv], to_dev(pairs), error_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(dk), kc)
    assert np.array_equal(bits_of(dv), vc)
    assert int(flag.item()) == 0


def test_reshape_code_example_and_padding(pa, orc):
    # the code example's shapes: pool (2, 64, 32, 8, 128) fp16, 4 rows to slots 0..3,
    # plus padding tokens (slot -1) and rows taken from a wider strided tensor
    rng = np.random.default_rng(0)
    nb, bs, hkv, d = 64, 32, 8, 128
    kc = rng.integers(0, 65536, (nb, bs, hkv, d), dtype=np.uint16)
    vc = rng.integers(0, 65536, (nb, bs, hkv, d), dtype=np.uint16)
    wide = rng.integers(0, 65536, (6, 3 * hkv * d), dtype=np.uint16)  # qkv-like rows
    k_rows = wide[:, hkv * d:2 * hkv * d].reshape(6, hkv, d)
    v_rows = wide[:, 2 * hkv * d:].reshape(6, hkv, d)
    slots = np.array([0, 1, -1, 2, 3, -1], np.int32)
    ek, ev = kc.copy(), vc.copy()
    orc.reshape_and_cache(k_rows, v_rows, ek, ev, slots)
    dwide = to_dev(wide, "f16")
    dk3 = dwide[:, hkv * d:2 * hkv * d].view(6, hkv, d)
    dv3 = dwide[:, 2 * hkv * d:].view(6, hkv, d)
    dk, dv = to_dev(kc, "f16"), to_dev(vc, "f16")
    pa.reshape_and_cache(dk3, dv3, dk, dv, to_dev(slots))
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(dk), ek) and np.array_equal(bits_of(dv), ev)


def test_reshape_bad_slot_is_flagged_and_skipped(pa):
    nb, bs, hkv, d = 4, 4, 2, 64
    dk = torch.zeros((nb, bs, hkv, d), dtype=torch.bfloat16, device="cuda")
    dv = torch.zeros_like(dk)
    rows = torch.ones((2, hkv, d), dtype=torch.bfloat16, device="cuda")
    flag = _flag()
    pa.reshape_and_cache(rows, rows, dk, dv, torch.tensor([5, nb * bs], dtype=torch.int32,
                                                           device="cuda"), error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_BAD_SLOT
    assert float(dk.sum()) == hkv * d  # only slot 5 written


def test_copy_blocks_shared_prefix_pairs(pa, orc):
    spec = W.WORKLOADS["shared_prefix"].replace(prompts=4, num_seqs=32)
    prep = prepare(spec)
    pairs = prep.cow_pairs
    assert pairs.shape[0] == 4 * 7  # samples 0..6 of each prompt copy, sample 7 writes in place
    layers = 3
    rng = np.random.default_rng(1)
    host = [prep.k_pool.copy(), prep.v_pool.copy()]
    for _ in range(layers - 1):
        host += [rng.integers(0, 65536, prep.k_pool.shape, dtype=np.uint16) for _ in range(2)]
    dev = [to_dev(h, "bf16") for h in host]
    ref = [h.copy() for h in host]
    block_bytes = int(np.prod(prep.k_pool.shape[1:])) * 2
    orc.copy_blocks(ref, pairs, block_bytes)
    flag = _flag()
    pa.copy_blocks(dev[0::2], dev[1::2], to_dev(pairs), error_flag=flag)
    torch.cuda.synchronize()
    for d_, r in zip(dev, ref):
        assert np.array_equal(bits_of(d_), r)
    assert int(flag.item()) == 0


def test_copy_blocks_odd_sizes_and_bad_ids(pa, orc):
    rng = np.random.default_rng(3)
    nb, bs, hkv, d = 10, 3, 1, 5       # 30-byte blocks: the byte-wise path
    host = [rng.integers(0, 65536, (nb, bs, hkv, d), dtype=np.uint16) for _ in range(2)]
    pairs = np.array([[1, 4], [2, 7], [3, 99]], np.int32)
    ref = [h.copy() for h in host]
    orc.copy_blocks(ref, pairs[:2], bs * hkv * d * 2)
    dev = [to_dev(h, "f16") for h in host]
    flag = _flag()
    pa.copy_blocks([dev[0]], [dev[1]], to_dev(pairs), error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_BAD_SLOT
    for d_, r in zip(dev, ref):
        assert np.array_equal(bits_of(d_), r)
