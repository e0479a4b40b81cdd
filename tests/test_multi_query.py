"""Several new tokens per sequence (pa_decode_attention_multi_query) on the GPU
against the fp64 oracle (orc_decode_multi): query i of a sequence's last n
tokens attends positions 0 .. L - n + i.  Pools are NaN-poisoned outside the
sequences' tokens; stored outputs within the fp32-path error plus half a
storage ulp, fp32 outputs within 1e-4."""
import os

import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import TOL_F32, as_f64, prepare, stored_within, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _case(hq=32, hkv=8, d=128, bs=16, dtype="bf16", B=6, lo=300, hi=900, qmax=4,
          qlens=None, seed=3001):
    spec = W.Spec("mq", B, hq, hkv, d, bs, dtype, seed=seed, len_dist="uniform",
                  len_lo=lo, len_hi=hi)
    prep = prepare(spec)
    g = torch.Generator().manual_seed(seed + 17)
    if qlens is None:
        qlens = torch.randint(1, qmax + 1, (B,), generator=g).numpy()
    qlens = np.asarray(qlens, dtype=np.int32)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = W.randn_bits((int(qs[-1]), hq, d), dtype, g)
    return spec, prep, q, qs, int(qlens.max())


def _run(pa, spec, prep, q, qs, qmax, out_dtype, psize=0, flag=None):
    dq = to_dev(q, spec.dtype)
    out = torch.empty(dq.shape, dtype=out_dtype, device="cuda")
    pa.decode_attention_multi_query(out, dq, to_dev(qs), to_dev(prep.k_pool, spec.dtype),
                                    to_dev(prep.v_pool, spec.dtype), to_dev(prep.tables),
                                    to_dev(prep.seq_lens), int(prep.seq_lens.max()), qmax,
                                    W.scale_of(spec), partition_size=psize, error_flag=flag)
    torch.cuda.synchronize()
    return out


def _check(pa, orc, spec, prep, q, qs, qmax, psize=0):
    ref = orc.decode_multi(q, qs, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                           W.scale_of(spec), spec.dtype)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(pa, spec, prep, q, qs, qmax, TORCH_DTYPE[spec.dtype], psize, flag)
    assert stored_within(out, ref, spec.dtype)
    out32 = _run(pa, spec, prep, q, qs, qmax, torch.float32, psize)
    o = as_f64(out32)
    assert np.all(np.isfinite(o))
    assert float(np.max(np.abs(o - ref))) <= TOL_F32
    assert int(flag.item()) == 0
    return o, ref


TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.mark.parametrize("hq,hkv,d,bs,dtype,qmax", [
    (32, 8, 128, 16, "bf16", 4),    # group 4: 16 columns per KV head
    (32, 8, 128, 16, "bf16", 8),    # group 4: 32 columns (two warps per head)
    (32, 8, 128, 16, "f16", 13),    # more than 8 tokens: chunks of 8
    (64, 8, 128, 32, "bf16", 4),    # group 8
    (8, 8, 128, 16, "bf16", 32),    # group 1: 32 tokens in one chunk
    (16, 8, 64, 4, "f16", 6),       # group 2, head_dim 64, 4-token blocks
])
def test_multi_query_matches_oracle(pa, orc, hq, hkv, d, bs, dtype, qmax):
    spec, prep, q, qs, m = _case(hq=hq, hkv=hkv, d=d, bs=bs, dtype=dtype, qmax=qmax)
    _check(pa, orc, spec, prep, q, qs, m)


@pytest.mark.parametrize("psize", [16, 64])
def test_multi_query_partitions(pa, orc, psize):
    spec, prep, q, qs, m = _case(qmax=8, seed=3002)
    _check(pa, orc, spec, prep, q, qs, m, psize=psize)


def test_multi_query_many_sequences(pa, orc):
    """64 sequences of 1..300 tokens, up to 4 new tokens each."""
    spec, prep, q, qs, m = _case(B=64, lo=4, hi=300, qmax=4, seed=3003)
    _check(pa, orc, spec, prep, q, qs, m)


def test_multi_query_more_chunks_than_the_plans_shared_table(pa, orc):
    """3000 sequences of 1..8 new tokens at group 8 (chunks of 4 query rows):
    about 4500 entries, more than the 4096 whose prefix sums the plan keeps in
    shared memory."""
    spec, prep, q, qs, m = _case(hq=16, hkv=2, d=64, bs=16, B=3000, lo=1, hi=60, qmax=8,
                                 seed=3007)
    qlens = np.diff(qs)
    assert int(np.sum((qlens + 3) // 4)) > 4096
    _check(pa, orc, spec, prep, q, qs, m)


def test_multi_query_edges(pa, orc):
    """No new token for one sequence, more new tokens than the sequence holds
    for another (its first queries see nothing: zeros), a single token."""
    spec, prep, q, qs, m = _case(B=4, lo=2, hi=40, qlens=[0, 6, 1, 3], seed=3004)
    L = prep.seq_lens
    assert L[1] >= 1
    o, ref = _check(pa, orc, spec, prep, q, qs, m)
    if L[1] < 6:  # queries before the sequence's first token attend nothing
        assert np.all(o[qs[1]:qs[1] + 6 - int(L[1])] == 0.0)


def test_one_query_each_is_the_decode_step(pa, orc):
    """One new token per sequence: the same numbers as decode_attention."""
    spec, prep, q, qs, m = _case(qlens=[1] * 6, seed=3005)
    dq = to_dev(q, spec.dtype)
    a = as_f64(_run(pa, spec, prep, q, qs, 1, torch.float32))
    out = torch.empty(dq.shape, dtype=torch.float32, device="cuda")
    pa.decode_attention(out, dq, to_dev(prep.k_pool, spec.dtype), to_dev(prep.v_pool, spec.dtype),
                        to_dev(prep.tables), to_dev(prep.seq_lens), int(prep.seq_lens.max()),
                        W.scale_of(spec))
    torch.cuda.synchronize()
    assert float(np.max(np.abs(a - as_f64(out)))) <= 2 * TOL_F32


def test_bad_query_ranges_are_flagged(pa):
    """q_start leaving [0, rows) is flagged; nothing is written out of bounds
    (the output tensor is followed by a guard that must stay untouched)."""
    spec, prep, q, qs, m = _case(B=3, qlens=[2, 2, 2], seed=3006)
    bad = qs.copy()
    bad[3] = 9  # the last sequence claims rows past the 6 that exist
    dq = to_dev(q, spec.dtype)
    buf = torch.zeros((dq.shape[0] + 4,) + tuple(dq.shape[1:]), dtype=torch.float32,
                      device="cuda")
    guard = buf[dq.shape[0]:]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.decode_attention_multi_query(buf[:dq.shape[0]], dq, to_dev(bad),
                                    to_dev(prep.k_pool, spec.dtype),
                                    to_dev(prep.v_pool, spec.dtype), to_dev(prep.tables),
                                    to_dev(prep.seq_lens), int(prep.seq_lens.max()), 3,
                                    W.scale_of(spec), error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_BAD_SEQLEN
    assert torch.count_nonzero(guard).item() == 0


@pytest.mark.slow
def test_full_size_four_new_tokens(pa, orc):
    """The benchmark's multi-query workload (llama8b shape, 4 new tokens per
    sequence) in its launch configuration, every query row compared."""
    spec = W.WORKLOADS["llama8b_mq4"]
    prep = prepare(spec.replace(q_len=1))  # pools, tables and lengths of the shape
    g = torch.Generator().manual_seed(spec.seed + 11)
    qlens = np.full(spec.num_seqs, spec.q_len, np.int32)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = W.randn_bits((int(qs[-1]), spec.num_q_heads, spec.head_dim), spec.dtype, g)
    out = as_f64(_run(pa, spec, prep, q, qs, spec.q_len, torch.float32))
    assert np.all(np.isfinite(out))
    ref = orc.decode_multi(q, qs, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                           W.scale_of(spec), spec.dtype,
                           nthreads=max(1, len(os.sched_getaffinity(0))))
    assert float(np.max(np.abs(out - ref))) <= TOL_F32
