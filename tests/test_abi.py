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
