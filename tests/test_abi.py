"""The C-ABI library on the CPU: it loads, exports every entry point the header
declares, and rejects bad arguments on the host before any launch.  Also the
native block manager against the reference block manager, table for table."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedattn.h")


@pytest.fixture(scope="module")
def pa():
    import importlib.util
    path = os.path.join(ROOT, "paged_kv_cache_343_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_pa_build", path)
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()  # compiles the library if missing, before the package loads it
    import paged_kv_cache_343_b200 as pa
    return pa


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(pa):
    names = _declared()
    assert "pa_decode_attention" in names and "pa_reshape_and_cache" in names
    assert "pa_copy_blocks" in names
    lib = ctypes.CDLL(pa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(pa):
    assert pa.lib.pa_status_string(0) == b"PA_OK"
    assert pa.lib.pa_status_string(1) == b"PA_ERR_INVALID_ARG"
    assert pa.version() >= 100


def test_host_validation_without_gpu(pa):
    lib = pa.lib
    # null pointers are refused before anything touches the device
    st = lib.pa_decode_attention(None, 1, None, None, None, None, 1, None, 4, 16, 4, 2, 64, 8,
                                 4, 0.125, 1, 0, None, 0, None, None)
    assert st == 1
    st = lib.pa_reshape_and_cache(None, None, 128, 128, None, None, None, 4, 8, 4, 2, 64, 0, 0,
                                  None, None, None, None)
    assert st == 1
    # unknown cache types are refused; fp8 without its scales is an invalid call
    st = lib.pa_reshape_and_cache(None, None, 128, 128, None, None, None, 4, 8, 4, 2, 64, 0, 7,
                                  None, None, None, None)
    assert st == 2
    st = lib.pa_reshape_and_cache(None, None, 128, 128, None, None, None, 4, 8, 4, 2, 64, 0, 1,
                                  None, None, None, None)
    assert st == 1
    st = lib.pa_decode_attention_fp8(None, 1, None, 1, None, None, None, None, None, 1, None, 4,
                                     16, 4, 2, 128, 8, 16, 0.1, 0, None, 0, None, None)
    assert st == 1
    # zero work is a no-op
    assert lib.pa_decode_attention(None, 1, None, None, None, None, 1, None, 0, 16, 4, 2, 64, 8,
                                   4, 0.125, 1, 0, None, 0, None, None) == 0
    assert lib.pa_copy_blocks(None, None, 1, None, 0, 8, 1024, None, None) == 0
    # bad sizes
    assert lib.pa_copy_blocks(None, None, 1, None, 3, 0, 1024, None, None) == 1
    # the read-bandwidth stream: ragged sizes, unaligned buffers, no sink, bad grids
    fake = 1 << 20  # a 16-byte aligned address that is never dereferenced
    assert lib.pa_stream_read(fake, 100, fake, 4, None) == 1
    assert lib.pa_stream_read(fake + 8, 1024, fake, 4, None) == 1
    assert lib.pa_stream_read(fake, 1024, None, 4, None) == 1
    assert lib.pa_stream_read(fake, 1024, fake, 0, None) == 1
    assert lib.pa_stream_read(fake, 1024, fake, 65536, None) == 1
    assert lib.pa_stream_read(fake, -16, fake, 4, None) == 1


def test_workspace_shape_checks_without_gpu(pa):
    out = ctypes.c_size_t(0)
    lib = pa.lib
    # Hq not a multiple of Hkv
    assert lib.pa_decode_workspace_bytes(4, 6, 4, 128, 16, 512, 0, ctypes.byref(out)) == 1
    # unsupported head_dim / block size / group
    assert lib.pa_decode_workspace_bytes(4, 8, 2, 96, 16, 512, 0, ctypes.byref(out)) == 2
    assert lib.pa_decode_workspace_bytes(4, 8, 2, 128, 12, 512, 0, ctypes.byref(out)) == 2
    assert lib.pa_decode_workspace_bytes(4, 32, 2, 128, 16, 512, 0, ctypes.byref(out)) == 2
    # partition not block aligned
    assert lib.pa_decode_workspace_bytes(4, 8, 2, 128, 32, 512, 48, ctypes.byref(out)) == 1


def _ops_trace(seed, num_blocks=64, bs=4):
    rng = np.random.default_rng(seed)
    order = rng.permutation(num_blocks).astype(np.int32)
    ops = [("add", 0, 7), ("add", 1, 4), ("fork", 0, 2), ("fork", 0, 3)]
    for _ in range(40):
        ops.append(("append", int(rng.integers(0, 4)), None))
    ops += [("free", 1, None), ("add", 4, 9), ("fork", 2, 5)]
    for _ in range(20):
        ops.append(("append", int(rng.choice([0, 2, 3, 4, 5])), None))
    return order, ops


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_native_block_manager_matches_reference(pa, seed):
    from oracle.blockmgr import RefBlockManager
    order, ops = _ops_trace(seed)
    ref = RefBlockManager(64, 4, order)
    nat = pa.BlockManager(64, 4, order)
    live = set()
    for op, a, b in ops:
        if op == "add":
            ref.add_sequence(a, b); nat.add_sequence(a, b); live.add(a)
        elif op == "fork":
            ref.fork(a, b); nat.fork(a, b); live.add(b)
        elif op == "free":
            ref.free_sequence(a); nat.free_sequence(a); live.discard(a)
        else:
            assert ref.append_slot(a) == nat.append_slot(a)
        for s in live:
            assert ref.block_table(s) == nat.block_table(s)
            assert ref.lengths[s] == nat.seq_len(s)
        ref.check_invariants()
    assert [ref.refcount[i] for i in range(64)] == [nat.refcount(i) for i in range(64)]
    assert len(ref.free) == nat.num_free()


def test_native_block_manager_errors(pa):
    bm = pa.BlockManager(2, 4)
    bm.add_sequence(0, 8)
    with pytest.raises(pa.PagedAttnError) as e:
        bm.append_slot(0)
    assert e.value.name == "PA_ERR_OUT_OF_BLOCKS"
    with pytest.raises(pa.PagedAttnError) as e:
        bm.append_slot(7)
    assert e.value.name == "PA_ERR_NOT_FOUND"
    with pytest.raises(pa.PagedAttnError):
        pa.BlockManager(3, 4, [0, 0, 1])  # not a permutation


def test_native_shared_blocks_counts(pa):
    """pa_bm_shared_blocks on forked sequences: the prompt's full blocks are
    shared until a copy-on-write replaces the partial one."""
    bm = pa.BlockManager(64, 4)
    bm.add_sequence(0, 10)          # blocks a, b, c(partial)
    bm.fork(0, 1)
    bm.fork(0, 2)
    bm.add_sequence(3, 9)
    bm.append_slot(1)               # copy-on-write of the partial block
    assert bm.shared_blocks([0, 1, 2, 3]).tolist() == [2, 2, 0, 0]
    assert bm.shared_blocks([0, 2]).tolist() == [3, 0]
    assert bm.shared_blocks([]).tolist() == []
    with pytest.raises(pa.PagedAttnError) as e:
        bm.shared_blocks([0, 9])
    assert e.value.name == "PA_ERR_NOT_FOUND"


def test_shared_prefix_host_validation(pa):
    lib = pa.lib
    # a null shared_blocks is an invalid call; zero work is a no-op
    st = lib.pa_decode_attention_shared_prefix(None, 1, None, None, None, None, 1, None, None, 4,
                                               16, 4, 2, 64, 8, 4, 0.125, 1, 0, None, 0, None,
                                               None)
    assert st == 1
    assert lib.pa_decode_attention_shared_prefix(None, 1, None, None, None, None, 1, None, None,
                                                 0, 16, 4, 2, 64, 8, 4, 0.125, 1, 0, None, 0,
                                                 None, None) == 0


def test_binding_refuses_mismatched_head_dim(pa):
    """Pools whose head_dim differs from the query's are refused before any
    pointer reaches the library (the C entry points take head_dim from one
    side only)."""
    import torch
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    k = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    tables = torch.zeros(2, 8, dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    for fn in (pa.decode_attention, pa.decode_attention_noalloc):
        with pytest.raises(ValueError):
            fn(torch.empty_like(q), q, k, k, tables, lens, 16, 0.1)
    with pytest.raises(ValueError):
        pa.reshape_and_cache(torch.zeros(3, 2, 128, dtype=torch.bfloat16),
                             torch.zeros(3, 2, 128, dtype=torch.bfloat16), k, k,
                             torch.zeros(3, dtype=torch.int32))


def test_binding_refuses_unsupported_dtypes(pa):
    """An output or query type the library has no code for is a ValueError
    raised by the binding, before any call into the library."""
    import torch
    q = torch.zeros(2, 8, 64, dtype=torch.bfloat16)
    k = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    tables = torch.zeros(2, 8, dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="unsupported dtype"):
        pa.decode_attention(torch.empty(q.shape, dtype=torch.float64), q, k, k, tables, lens,
                            16, 0.1)
    q64 = q.double()
    with pytest.raises(ValueError):
        pa.decode_attention(torch.empty_like(q64), q64, k.double(), k.double(), tables, lens,
                            16, 0.1)


def test_noalloc_binding_refuses_before_any_library_call(pa):
    """decode_attention_noalloc makes decode_attention's checks (CPU tensors:
    a refusal here is raised before any pointer reaches the library): a uint8
    code pool under a 16-bit query, a query of another 16-bit type, K and V of
    different strides, a strided half of an interleaved pool (the entry point
    has no strided form), 64-bit tables or lengths, a non-contiguous query."""
    import torch
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    out = torch.empty_like(q)
    k = torch.zeros(4, 16, 2, 128, dtype=torch.bfloat16)
    tables = torch.zeros(2, 8, dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    f = pa.decode_attention_noalloc
    codes = torch.zeros(4, 16, 2, 128, dtype=torch.uint8)
    with pytest.raises(ValueError):
        f(out, q, codes, codes, tables, lens, 16, 0.1)
    with pytest.raises(ValueError):
        f(out, q, k.half(), k.half(), tables, lens, 16, 0.1)
    kv = torch.zeros(4, 2, 16, 2, 128, dtype=torch.bfloat16)  # per-block interleaved K/V
    with pytest.raises(ValueError, match="contiguous"):
        f(out, q, kv[:, 0], kv[:, 1], tables, lens, 16, 0.1)
    with pytest.raises(ValueError):
        f(out, q, k, k.transpose(1, 2).contiguous().transpose(1, 2), tables, lens, 16, 0.1)
    with pytest.raises(ValueError):
        f(out, q, k, k, tables.long(), lens, 16, 0.1)
    with pytest.raises(ValueError):
        f(out, q, k, k, tables, lens.long(), 16, 0.1)
    qt = torch.zeros(8, 2, 128, dtype=torch.bfloat16).transpose(0, 1)
    with pytest.raises(ValueError):
        f(torch.empty(2, 8, 128, dtype=torch.bfloat16), qt, k, k, tables, lens, 16, 0.1)
    with pytest.raises(ValueError, match="unsupported dtype"):
        f(torch.empty(q.shape, dtype=torch.float64), q, k, k, tables, lens, 16, 0.1)


def _sampling_trace(bm, seed, prompts=3, samples=4, prompt_len=10):
    """Prompts forked into samples (parallel sampling), as both managers see it."""
    sid = 0
    for _ in range(prompts):
        bm.add_sequence(sid, prompt_len + seed)
        for s in range(1, samples):
            bm.fork(sid, sid + s)
        sid += samples
    return list(range(sid))


@pytest.mark.parametrize("seed", [0, 1, 3])
def test_native_append_slots_matches_one_by_one(pa, seed):
    """pa_bm_append_slots over a batch gives the slots and copy-on-write pairs
    of pa_bm_append_slot called in the same order, and of the reference
    manager, step after step (block boundaries and copies included)."""
    from oracle.blockmgr import RefBlockManager
    rng = np.random.default_rng(seed)
    order = rng.permutation(96).astype(np.int32)
    batch_bm, one_bm, ref = (pa.BlockManager(96, 4, order), pa.BlockManager(96, 4, order),
                             RefBlockManager(96, 4, order))
    seqs = [_sampling_trace(m, seed) for m in (batch_bm, one_bm, ref)][0]
    for step in range(7):
        batch = [int(x) for x in rng.permutation(seqs)[:int(rng.integers(1, len(seqs) + 1))]]
        slots, pairs = batch_bm.append_slots(batch)
        want_slots, want_pairs = [], []
        for s in batch:
            slot, cow = one_bm.append_slot(s)
            rslot, rcow = ref.append_slot(s)
            assert (slot, cow) == (rslot, rcow)
            want_slots.append(slot)
            if cow is not None:
                want_pairs.append(cow)
        assert slots.tolist() == want_slots
        assert [tuple(p) for p in pairs.tolist()] == want_pairs
        for s in seqs:
            assert batch_bm.block_table(s) == ref.block_table(s)
        ref.check_invariants()
    assert [batch_bm.refcount(i) for i in range(96)] == [ref.refcount[i] for i in range(96)]


def test_native_append_slots_all_or_nothing(pa):
    """A batch the free list cannot cover fails with PA_ERR_OUT_OF_BLOCKS and
    changes nothing; an unknown or repeated sequence is refused up front."""
    bm = pa.BlockManager(5, 4)
    bm.add_sequence(0, 6)          # blocks 0, 1 (2 of 4 slots used in 1)
    bm.fork(0, 1)
    bm.fork(0, 2)                  # block 1 shared three ways, partially filled
    bm.add_sequence(3, 4)          # block 2, full
    # seq 0 and seq 1 each copy the shared block, seq 3 needs a new block:
    # three blocks, two free
    before = ([bm.block_table(s) for s in range(4)], [bm.refcount(i) for i in range(5)],
              bm.num_free())
    with pytest.raises(pa.PagedAttnError) as e:
        bm.append_slots([0, 1, 3])
    assert e.value.name == "PA_ERR_OUT_OF_BLOCKS"
    assert ([bm.block_table(s) for s in range(4)], [bm.refcount(i) for i in range(5)],
            bm.num_free()) == before
    # the last holder writes in place: seqs 0, 1 copy, seq 2 does not
    slots, pairs = bm.append_slots([0, 1, 2])
    assert pairs.tolist() == [[1, 3], [1, 4]]
    assert slots.tolist() == [3 * 4 + 2, 4 * 4 + 2, 1 * 4 + 2]
    assert bm.num_free() == 0
    for bad, name in (([7], "PA_ERR_NOT_FOUND"), ([0, 0], "PA_ERR_INVALID_ARG")):
        with pytest.raises(pa.PagedAttnError) as e:
            bm.append_slots(bad)
        assert e.value.name == name
    assert bm.append_slots([])[0].numel() == 0


def test_native_fill_tables(pa):
    bm = pa.BlockManager(32, 4, np.arange(31, -1, -1).astype(np.int32))
    bm.add_sequence(5, 9)
    bm.add_sequence(9, 0)
    bm.add_sequence(2, 4)
    tables, lens = bm.fill_tables([9, 5, 2], 4)
    assert tables.tolist() == [[-1, -1, -1, -1], [31, 30, 29, -1], [28, -1, -1, -1]]
    assert lens.tolist() == [0, 9, 4]
    with pytest.raises(pa.PagedAttnError) as e:
        bm.fill_tables([5], 2)      # three blocks do not fit in two columns
    assert e.value.name == "PA_ERR_INVALID_ARG"
    with pytest.raises(pa.PagedAttnError) as e:
        bm.fill_tables([5, 4], 4)
    assert e.value.name == "PA_ERR_NOT_FOUND"


def test_native_stats_by_hand(pa):
    """Counted by hand: block size 4, a 6-token prompt forked twice, then one
    token for each of the three sequences (two copy the shared partial block)."""
    bm = pa.BlockManager(16, 4)
    bm.add_sequence(0, 6)
    bm.fork(0, 1)
    bm.fork(0, 2)
    st = bm.stats()
    assert (st["held_blocks"], st["logical_blocks"], st["tokens"]) == (2, 6, 18)
    assert (st["stored_slots"], st["waste_slots"], st["max_waste_per_seq"]) == (6, 2, 2)
    bm.append_slots([0, 1, 2])
    st = bm.stats()
    # blocks: 0 shared (4 tokens), 1 (seq 2, 3 tokens), 2 and 3 (copies, 3 each)
    assert (st["held_blocks"], st["free_blocks"], st["logical_blocks"]) == (4, 12, 6)
    assert (st["tokens"], st["stored_slots"], st["waste_slots"]) == (21, 13, 3)
    assert st["max_waste_per_seq"] == 1 and st["num_seqs"] == 3
    assert abs(st["occupancy"] - 13 / 16) < 1e-12
    assert abs(st["sharing_saving"] - (1 - 4 / 6)) < 1e-12


def test_native_stats_agree_with_the_bench_accounting(pa):
    """On a parallel-sampling workload the native counts equal the benchmark's
    own count from the tables (blocks held once, blocks without sharing,
    tokens, largest waste per sequence)."""
    import bench
    import pa_workloads as W
    spec = W.WORKLOADS["shared_prefix"].replace(prompts=4, num_seqs=32, seed=5)
    case = W.draw(spec)
    bm = pa.BlockManager(case.num_blocks, spec.block_size, case.free_order)
    sid = 0
    for _ in range(spec.prompts):
        bm.add_sequence(sid, spec.prompt_len)
        for s in range(1, spec.samples):
            bm.fork(sid, sid + s)
        sid += spec.samples
    for _ in range(int(case.extra_tokens.max())):
        live = [b for b in range(spec.num_seqs)
                if bm.seq_len(b) < spec.prompt_len + int(case.extra_tokens[b])]
        bm.append_slots(live)
    seqs = list(range(spec.num_seqs))
    width = max(len(bm.block_table(b)) for b in seqs)
    tables, lens = bm.fill_tables(seqs, width)
    mem = bench.kv_memory(spec, {"lens": lens.numpy(), "tables": tables.numpy()})
    st = bm.stats()
    assert st["held_blocks"] == mem["blocks_held"]
    assert st["logical_blocks"] == mem["blocks_if_unshared"]
    assert st["tokens"] == mem["tokens"]
    assert st["max_waste_per_seq"] == mem["max_waste_tokens_per_seq"]
    assert abs(st["sharing_saving"] - mem["sharing_saving"]) < 1e-4


@pytest.mark.parametrize("seed", [0, 2])
def test_native_append_tokens_matches_the_reference_manager(pa, seed):
    """pa_bm_append_tokens: counts[i] tokens of seqs[i] in order give the
    slots and copies of the reference manager appending them one by one, and
    q_start is the running sum of the counts (zero counts included)."""
    from oracle.blockmgr import RefBlockManager
    rng = np.random.default_rng(10 + seed)
    order = rng.permutation(160).astype(np.int32)
    nat, ref = pa.BlockManager(160, 4, order), RefBlockManager(160, 4, order)
    seqs = [_sampling_trace(m, seed, prompts=2, samples=3, prompt_len=9) for m in (nat, ref)][0]
    for step in range(5):
        batch = [int(x) for x in rng.permutation(seqs)]
        counts = [int(c) for c in rng.integers(0, 6, len(batch))]
        slots, q_start, pairs = nat.append_tokens(batch, counts)
        want_slots, want_pairs = [], []
        for s, c in zip(batch, counts):
            for _ in range(c):
                slot, cow = ref.append_slot(s)
                want_slots.append(slot)
                if cow is not None:
                    want_pairs.append(cow)
        assert slots.tolist() == want_slots
        assert [tuple(p) for p in pairs.tolist()] == want_pairs
        assert q_start.tolist() == [0] + list(np.cumsum(counts))
        for s in seqs:
            assert nat.block_table(s) == ref.block_table(s)
        ref.check_invariants()


def test_native_append_tokens_all_or_nothing(pa):
    bm = pa.BlockManager(4, 4)
    bm.add_sequence(0, 6)           # blocks 0, 1
    bm.fork(0, 1)                   # block 1 shared and partial
    before = ([bm.block_table(s) for s in range(2)], bm.num_free())
    # seq 0: a copy of block 1 plus one new block for positions 8..9 -> 2;
    # seq 1: then the last holder of block 1, writes in place, and needs a new
    # block for positions 8..11 -> 1; three blocks, two free
    with pytest.raises(pa.PagedAttnError) as e:
        bm.append_tokens([0, 1], [4, 6])
    assert e.value.name == "PA_ERR_OUT_OF_BLOCKS"
    assert ([bm.block_table(s) for s in range(2)], bm.num_free()) == before
    with pytest.raises(pa.PagedAttnError) as e:
        bm.append_tokens([0], [-1])
    assert e.value.name == "PA_ERR_INVALID_ARG"
    slots, q_start, pairs = bm.append_tokens([0, 1], [4, 2])
    assert q_start.tolist() == [0, 4, 6] and pairs.tolist() == [[1, 2]]
    assert slots.tolist() == [2 * 4 + 2, 2 * 4 + 3, 3 * 4 + 0, 3 * 4 + 1, 1 * 4 + 2, 1 * 4 + 3]
    assert bm.num_free() == 0


def test_native_blocks_needed_predicts_the_appends(pa):
    """pa_bm_blocks_needed changes nothing and equals the free blocks the
    following append call takes, copies of shared partial blocks included."""
    rng = np.random.default_rng(4)
    bm = pa.BlockManager(400, 4, rng.permutation(400).astype(np.int32))
    seqs = _sampling_trace(bm, 1, prompts=3, samples=4, prompt_len=9)
    for step in range(6):
        batch = [int(x) for x in rng.permutation(seqs)]
        if step % 2:
            counts = [int(c) for c in rng.integers(0, 7, len(batch))]
            tables = [bm.block_table(s) for s in seqs]
            need = bm.blocks_needed(batch, counts)
            assert [bm.block_table(s) for s in seqs] == tables
            free = bm.num_free()
            bm.append_tokens(batch, counts)
        else:
            need = bm.blocks_needed(batch)
            free = bm.num_free()
            bm.append_slots(batch)
        assert free - bm.num_free() == need
    with pytest.raises(pa.PagedAttnError) as e:
        bm.blocks_needed([0, 0])
    assert e.value.name == "PA_ERR_INVALID_ARG"


def _prompt(seed, n):
    return [int(x) for x in np.random.default_rng(seed).integers(0, 32000, n)]


def test_prefix_cache_shares_the_full_blocks_of_a_common_prompt(pa):
    """Two requests with one 40-token prompt at block size 16: the second
    shares the two full blocks (32 cached tokens) and gets its own partial
    block; a third prompt sharing only the first 16 tokens shares one block."""
    bm = pa.BlockManager(32, 16)
    p = _prompt(1, 40)
    assert bm.add_sequence_with_prefix(0, p) == 0
    assert bm.add_sequence_with_prefix(1, p) == 32
    t0, t1 = bm.block_table(0), bm.block_table(1)
    assert t1[:2] == t0[:2] and t1[2] != t0[2]
    assert [bm.refcount(b) for b in t0] == [2, 2, 1]
    q = p[:16] + _prompt(2, 20)
    assert bm.add_sequence_with_prefix(2, q) == 16
    assert bm.block_table(2)[0] == t0[0] and bm.refcount(t0[0]) == 3
    assert bm.stats()["cached_blocks"] == 3      # t0[0], t0[1] and seq 2's second block
    assert bm.seq_len(1) == 40


def test_prefix_cache_match_is_exact_and_chained(pa):
    """A block matches only when its tokens and every token before it match:
    the same second block after a different first block is not shared, nor is
    a block that differs in one token."""
    bm = pa.BlockManager(32, 4)
    a, b = _prompt(3, 4), _prompt(4, 4)
    y = _prompt(5, 4)
    assert bm.add_sequence_with_prefix(0, a + y) == 0
    assert bm.add_sequence_with_prefix(1, b + y) == 0            # y after b: no match
    assert bm.add_sequence_with_prefix(2, a + y[:3] + [y[3] + 1]) == 4
    assert bm.add_sequence_with_prefix(3, a + y + [7]) == 8      # both full blocks, then 1 token
    assert bm.block_table(3)[:2] == bm.block_table(0)


def test_prefix_cache_entries_leave_with_their_blocks(pa):
    bm = pa.BlockManager(8, 4)
    p = _prompt(6, 12)
    bm.add_sequence_with_prefix(0, p)
    bm.add_sequence_with_prefix(1, p)
    bm.free_sequence(0)                       # blocks still held by seq 1
    assert bm.add_sequence_with_prefix(2, p) == 12
    bm.free_sequence(1)
    bm.free_sequence(2)
    assert bm.stats()["cached_blocks"] == 0 and bm.num_free() == 8
    assert bm.add_sequence_with_prefix(3, p) == 0


def test_prefix_cache_all_or_nothing_and_appends(pa):
    """A request whose uncached blocks do not fit changes nothing; appending
    after a prompt that ends on a block boundary never writes a shared
    block (a new block is taken, no copy)."""
    bm = pa.BlockManager(5, 4)
    p = _prompt(7, 8)
    bm.add_sequence_with_prefix(0, p)         # 2 blocks, both cached
    bm.add_sequence(9, 8)                     # 2 more: 1 free
    with pytest.raises(pa.PagedAttnError) as e:
        bm.add_sequence_with_prefix(1, p[:4] + _prompt(8, 8))   # 1 shared + 2 new
    assert e.value.name == "PA_ERR_OUT_OF_BLOCKS"
    assert bm.num_free() == 1 and bm.stats()["cached_blocks"] == 2
    assert bm.add_sequence_with_prefix(1, p) == 8   # all shared, nothing new
    slot, cow = bm.append_slot(1)
    assert cow is None and bm.num_free() == 0
    assert bm.block_table(1)[:2] == bm.block_table(0)
    assert slot // 4 == bm.block_table(1)[2]


def test_c_abi_from_plain_c(pa, tmp_path):
    """The header compiles as C99 with warnings as errors, and a C program
    linked against the library sees the declared host-side behaviour."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_check"
    lib_dir = os.path.dirname(pa.LIB_PATH)
    build = subprocess.run(
        [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
         os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", lib_dir, "-lpagedattn",
         "-Wl,-rpath," + lib_dir, "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert "all checks held" in run.stdout


def test_import_fails_loudly_without_the_library(tmp_path):
    """The binding has no fallback: a copy of the package without its
    library refuses to import, naming the missing file."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "paged_kv_cache_343_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "paged_kv_cache_343_b200", "__init__.py"), pkg / "__init__.py")
    run = subprocess.run([sys.executable, "-c", "import paged_kv_cache_343_b200"],
                         cwd=tmp_path, capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, PYTHONPATH=str(tmp_path)))
    assert run.returncode != 0
    assert "libpagedattn.so is missing" in run.stderr


def test_order_by_prefix_groups_the_samples_of_a_prompt(pa):
    """Samples of three prompts listed in a shuffled order: after
    pa_bm_order_by_prefix each prompt's samples are neighbours, so the
    shared-blocks counts of the reordered batch show the sharing."""
    bm = pa.BlockManager(256, 4, np.random.default_rng(0).permutation(256).astype(np.int32))
    sid = 0
    owner = {}
    for prompt, length in enumerate((22, 9, 30)):
        bm.add_sequence(sid, length)
        owner[sid] = prompt
        for k in range(1, 4):
            bm.fork(sid, sid + k)
            owner[sid + k] = prompt
        sid += 4
    batch = [int(x) for x in np.random.default_rng(1).permutation(sid)]
    order = bm.order_by_prefix(batch)
    assert sorted(order) == list(range(sid))
    seqs = [batch[i] for i in order]
    groups = [owner[s] for s in seqs]
    for g0 in range(0, sid, 4):           # each run of four is one prompt's samples
        assert len(set(groups[g0:g0 + 4])) == 1
        run = seqs[g0:g0 + 4]
        shared = bm.shared_blocks(run).tolist()
        full = -(-bm.seq_len(run[0]) // 4)
        assert shared == [full] * 3 + [0]
    # ties keep the given order
    assert [s for s in seqs if owner[s] == owner[seqs[0]]] == \
        [s for s in batch if owner[s] == owner[seqs[0]]]
    with pytest.raises(pa.PagedAttnError) as e:
        bm.order_by_prefix([0, 999])
    assert e.value.name == "PA_ERR_NOT_FOUND"
