"""pa_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (framework plugins that must not call cudaMalloc,
callers without an allocator, loops that cannot afford cudaMalloc/cudaFree's
device synchronisation).  Its scratch is the library's static per-device
array; this file checks, through the C ABI, that two calls in a row match the
regular entry point (which takes a caller-allocated workspace) and that a
shape needing more scratch than the array holds is refused.  Kept in its own
file, collected last."""
import ctypes

import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import as_f64, prepare, to_dev

pytestmark = pytest.mark.gpu

TOL_STORED = 2e-3
TOL_F32 = 1e-4


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _args(prep):
    s = prep.case.spec
    q = to_dev(prep.case.q, s.dtype)
    return dict(query=q, key_cache=to_dev(prep.k_pool, s.dtype),
                value_cache=to_dev(prep.v_pool, s.dtype), block_tables=to_dev(prep.tables),
                seq_lens=to_dev(prep.seq_lens), max_seq_len=int(prep.seq_lens.max()),
                scale=W.scale_of(s), partition_size=s.partition_size)


def _noalloc_via_cabi(pa, out, a):
    """Direct ctypes call of the C entry point (no Python-side allocation)."""
    q, k = a["query"], a["key_cache"]
    B, hq, d = q.shape
    nb, bs, hkv, _ = k.shape
    code = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2}
    st = pa.lib.pa_decode_attention_noalloc(
        ctypes.c_void_p(out.data_ptr()), code[out.dtype], ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(a["value_cache"].data_ptr()),
        ctypes.c_void_p(a["block_tables"].data_ptr()), a["block_tables"].stride(0),
        ctypes.c_void_p(a["seq_lens"].data_ptr()), B, a["max_seq_len"], hq, hkv, d, nb, bs,
        a["scale"], code[q.dtype], a["partition_size"], None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("out_dtype", [None, torch.float32])
def test_noalloc_matches_workspace_entry_point_twice(pa, orc, out_dtype):
    # two different workloads back to back: the second call must not see
    # anything the first one left in the shared static scratch
    preps = [prepare(W.WORKLOADS["llama8b"].replace(num_seqs=6, len_lo=300, len_hi=1200, seed=31)),
             prepare(W.WORKLOADS["longtail"].replace(num_seqs=48, new_rows=0, seed=32))]
    tol = TOL_F32 if out_dtype == torch.float32 else TOL_STORED
    for prep in preps:
        a = _args(prep)
        ref = torch.empty(a["query"].shape, dtype=out_dtype or a["query"].dtype, device="cuda")
        pa.decode_attention(ref, **a)
        got = torch.full_like(ref, float("nan"))
        assert _noalloc_via_cabi(pa, got, a) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert float((got.float() - ref.float()).abs().max()) <= tol
        # and against the oracle
        s = prep.case.spec
        oref = orc.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                          W.scale_of(s), s.dtype, nthreads=4)
        assert float(np.max(np.abs(as_f64(got) - oref))) <= max(tol, TOL_STORED if out_dtype is None else tol)


def test_noalloc_through_the_binding(pa, orc):
    """The Python wrapper's path (its checks, then the same C entry point)
    gives the regular entry point's result on a reduced llama8b batch."""
    prep = prepare(W.WORKLOADS["llama8b"].replace(num_seqs=5, len_lo=100, len_hi=900, seed=33))
    a = _args(prep)
    ref = torch.empty_like(a["query"])
    pa.decode_attention(ref, **a)
    got = torch.full_like(ref, float("nan"))
    pa.decode_attention_noalloc(got, **a)
    torch.cuda.synchronize()
    assert float((got.float() - ref.float()).abs().max()) <= TOL_STORED
    s = prep.case.spec
    oref = orc.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                      W.scale_of(s), s.dtype, nthreads=4)
    assert float(np.max(np.abs(as_f64(got) - oref))) <= TOL_STORED


def test_noalloc_refuses_shapes_beyond_its_scratch(pa):
    # 4096 sequences of up to 32768 tokens in 16-token partitions needs far more
    # than the static array; the call must refuse before launching anything
    need = pa.decode_workspace_bytes(4096, 32, 8, 128, 16, 32768, 16)
    assert need > pa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((4096, 32, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((8, 16, 8, 128), dtype=torch.bfloat16, device="cuda")
    a = dict(query=q, key_cache=k, value_cache=k,
             block_tables=torch.zeros((4096, 2048), dtype=torch.int32, device="cuda"),
             seq_lens=torch.zeros(4096, dtype=torch.int32, device="cuda"), max_seq_len=32768,
             scale=0.1, partition_size=16)
    out = torch.empty_like(q)
    assert _noalloc_via_cabi(pa, out, a) == 6  # PA_ERR_TOO_LARGE
    assert pa.lib.pa_status_string(6) == b"PA_ERR_TOO_LARGE"
