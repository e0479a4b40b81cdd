"""The benchmark's byte accounting on hand-built cases (CPU): the bytes a step
must read, with and without shared prompt blocks, and the KV memory held.
Expected values are counted by hand in each test."""
import numpy as np

import bench
import pa_workloads as W


def _spec(**kw):
    base = dict(name="t", num_seqs=2, num_q_heads=32, num_kv_heads=8, head_dim=128,
                block_size=16, dtype="bf16", seed=0)
    base.update(kw)
    return W.Spec(**base)


ROW = 2 * 8 * 128 * 2  # K and V bytes of one token at Hkv 8, D 128, 16-bit


def test_kv_bytes_counts_every_token():
    spec = _spec()
    assert bench.kv_bytes(spec, np.array([100, 37])) == 137 * ROW
    assert bench.kv_bytes(spec.replace(kv_dtype="fp8_e4m3"), np.array([10])) == 10 * ROW // 2


def test_unique_bytes_count_shared_slots_once():
    # block size 4: both sequences start with physical block 5 (full), then
    # seq 0 holds 2 tokens of block 1 and seq 1 holds 3 tokens of block 2
    spec = _spec(block_size=4)
    wl = {"lens": np.array([6, 7]), "tables": np.array([[5, 1], [5, 2]])}
    assert bench.unique_kv_bytes(spec, wl) == (4 + 2 + 3) * ROW


def test_packed_bytes_read_a_shared_prefix_once():
    # group 4: windows of 8 sequences; a window of 2 falls back to one pair.
    # The pair shares 5 full blocks (80 tokens, 5 tiles >= 4): read once.
    spec = _spec()
    wl = {"lens": np.array([100, 90]), "shared_blocks": np.array([5, 0])}
    assert bench.packed_kv_bytes(spec, wl) == (100 + 90 - 80) * ROW
    # fewer than 4 shared tiles (3 blocks = 48 tokens): no pack
    wl = {"lens": np.array([100, 90]), "shared_blocks": np.array([3, 0])}
    assert bench.packed_kv_bytes(spec, wl) == 190 * ROW


def test_packed_bytes_whole_window():
    # 8 sequences that all share 10 full blocks (160 tokens): one pack of 8
    spec = _spec(num_seqs=8)
    lens = np.array([200, 190, 170, 165, 300, 161, 180, 175])
    wl = {"lens": lens, "shared_blocks": np.array([10] * 7 + [0])}
    assert bench.packed_kv_bytes(spec, wl) == (int(lens.sum()) - 7 * 160) * ROW
    # sequences 2 and 3 share only 2 blocks: the window breaks into aligned
    # pairs; (0,1), (4,5), (6,7) share 10 blocks each, (2,3) too few to pack
    sb = np.array([10, 10, 2, 10, 10, 10, 10, 0])
    wl = {"lens": lens, "shared_blocks": sb}
    assert bench.packed_kv_bytes(spec, wl) == (int(lens.sum()) - 3 * 160) * ROW


def test_kv_memory_counts_blocks_held_once():
    spec = _spec(block_size=4)
    wl = {"lens": np.array([6, 7]), "tables": np.array([[5, 1], [5, 2]])}
    m = bench.kv_memory(spec, wl)
    assert m["blocks_held"] == 3 and m["blocks_if_unshared"] == 4
    assert m["tokens"] == 13
    assert m["max_waste_tokens_per_seq"] == 2  # seq 0: 8 slots for 6 tokens
    assert abs(m["sharing_saving"] - 0.25) < 1e-12
