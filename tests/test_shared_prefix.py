"""Shared-prefix decode (parallel samples of one prompt read the prompt's
blocks once per pack) on the GPU against the fp64 oracle.

The oracle attends every sequence over its own block table; packing is only a
different order of the same reads, so the bar is the plain decode's: stored
outputs within the fp32-path error plus half a storage ulp, fp32 outputs
within 1e-4.  Pools are NaN-poisoned in every slot that holds no token."""
import os

import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import (TOL_F32, as_f64, pools_after_appends, prepare, shared_blocks_of,
                     stored_within, to_dev)

pytestmark = pytest.mark.gpu

NTHREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _spec(**kw):
    base = W.WORKLOADS["shared_prefix"]
    prompts = kw.pop("prompts", 2)
    samples = kw.pop("samples", 8)
    return base.replace(prompts=prompts, samples=samples, num_seqs=prompts * samples, **kw)


def _inputs(prep):
    s = prep.case.spec
    k, v = pools_after_appends(prep)
    sb = shared_blocks_of(prep.tables, prep.seq_lens, s.block_size)
    return k, v, sb


def _ref(orc, prep, k, v, seqs=None):
    s = prep.case.spec
    q, tables, lens = prep.case.q, prep.tables, prep.seq_lens
    if seqs is not None:
        q, tables, lens = q[seqs], tables[seqs], lens[seqs]
    return orc.decode(q, k, v, tables, lens, W.scale_of(s), s.dtype, nthreads=NTHREADS)


def _run_shared(pa, prep, k, v, sb, out_dtype=None, partition_size=0, flag=None):
    s = prep.case.spec
    q = to_dev(prep.case.q, s.dtype)
    out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device="cuda")
    lens = prep.seq_lens
    pa.decode_attention_shared_prefix(out, q, to_dev(k, s.dtype), to_dev(v, s.dtype),
                                      to_dev(prep.tables), to_dev(lens.astype(np.int32)),
                                      to_dev(sb.astype(np.int32)), int(lens.max()),
                                      W.scale_of(s), partition_size=partition_size,
                                      error_flag=flag)
    torch.cuda.synchronize()
    return out


def _run_plain(pa, prep, k, v, out_dtype=None, partition_size=0):
    s = prep.case.spec
    q = to_dev(prep.case.q, s.dtype)
    out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device="cuda")
    lens = prep.seq_lens
    pa.decode_attention(out, q, to_dev(k, s.dtype), to_dev(v, s.dtype), to_dev(prep.tables),
                        to_dev(lens.astype(np.int32)), int(lens.max()), W.scale_of(s),
                        partition_size=partition_size)
    torch.cuda.synchronize()
    return out


def _check(pa, orc, spec, partition_size=0, expect_packs=True):
    prep = prepare(spec)
    k, v, sb = _inputs(prep)
    if expect_packs:
        assert sb.max() * spec.block_size >= 64, "the case should share a packable prefix"
    ref = _ref(orc, prep, k, v)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run_shared(pa, prep, k, v, sb, partition_size=partition_size, flag=flag)
    assert stored_within(out, ref, spec.dtype)
    out32 = _run_shared(pa, prep, k, v, sb, out_dtype=torch.float32,
                        partition_size=partition_size)
    o = as_f64(out32)
    assert np.all(np.isfinite(o))
    assert float(np.max(np.abs(o - ref))) <= TOL_F32
    assert int(flag.item()) == 0
    return prep, k, v, sb, out32


def test_reduced_shared_prefix_matches_oracle(pa, orc):
    """The benchmark's shape (8 samples of a 2047-token prompt, 4 query heads
    per KV head: packs of 8) at 2 prompts."""
    _check(pa, orc, _spec())


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", [
    (8, 8, 128, 16, "bf16"),    # 1 query head per KV head: packs of 8
    (16, 8, 128, 16, "f16"),    # 2: packs of 4
    (24, 8, 64, 16, "bf16"),    # 3: packs of 2, six of eight columns
    (32, 8, 128, 4, "bf16"),    # 4 with 4-token blocks
    (32, 8, 128, 32, "f16"),    # 4 with 32-token blocks
    (64, 8, 128, 16, "bf16"),   # 8: no room to pack, plain path with the larger workspace
    (4, 1, 64, 8, "f16"),       # one KV head
])
def test_group_shapes(pa, orc, hq, hkv, d, bs, dtype):
    spec = _spec(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs, dtype=dtype,
                 prompt_len=700, extra_lo=1, extra_hi=60)
    _check(pa, orc, spec)


def test_many_prompts(pa, orc):
    """6 prompts x 8 samples (48 sequences): the plan walks the few cut points
    of each entry and the combine runs a warp per head."""
    _check(pa, orc, _spec(prompts=6, prompt_len=300, extra_hi=40))


@pytest.mark.parametrize("psize", [16, 64, 512])
def test_partitions(pa, orc, psize):
    _check(pa, orc, _spec(prompt_len=900, extra_hi=80), partition_size=psize)


def test_samples_not_aligned_to_packs(pa, orc):
    """3 samples per prompt: windows of 2 straddle prompts and stay unpacked."""
    _check(pa, orc, _spec(prompts=5, samples=3, prompt_len=500, extra_hi=40))


def test_prefix_ends_on_a_tile(pa, orc):
    """A 256-token prompt and samples with 0..2 extra tokens: some sequences
    are attended entirely through their pack (their own entry has no tiles)."""
    _check(pa, orc, _spec(prompts=3, samples=4, prompt_len=256, extra_lo=0, extra_hi=2))


def test_every_tile_in_a_pack(pa, orc):
    """A 256-token prompt and no extra tokens: every tile of every sequence is
    attended through its pack, so the sequences' own tiles (the second part
    of the tile line) are empty."""
    _check(pa, orc, _spec(prompts=3, samples=8, prompt_len=256, extra_lo=0, extra_hi=0))


def test_short_prompt_is_not_packed(pa, orc):
    _check(pa, orc, _spec(prompts=3, samples=4, prompt_len=40, extra_hi=30),
           expect_packs=False)


def test_no_sharing_matches_the_plain_path(pa, orc):
    """shared_blocks all 0: no packs, every sequence attended alone.  The
    entry point runs its own launch shape (fewer heads per CTA, wider warps),
    so the partials are cut elsewhere: equal to the plain path and the oracle
    within the fp32 bound, not bit for bit."""
    prep = prepare(_spec(prompt_len=600, extra_hi=50))
    k, v, sb = _inputs(prep)
    ref = _ref(orc, prep, k, v)
    a = as_f64(_run_shared(pa, prep, k, v, np.zeros_like(sb), out_dtype=torch.float32))
    b = as_f64(_run_plain(pa, prep, k, v, out_dtype=torch.float32))
    assert float(np.max(np.abs(a - ref))) <= TOL_F32
    assert float(np.max(np.abs(a - b))) <= 2 * TOL_F32


def test_packed_matches_plain_path(pa, orc):
    prep = prepare(_spec(prompt_len=1200, extra_hi=100))
    k, v, sb = _inputs(prep)
    a = as_f64(_run_shared(pa, prep, k, v, sb, out_dtype=torch.float32))
    b = as_f64(_run_plain(pa, prep, k, v, out_dtype=torch.float32))
    assert float(np.max(np.abs(a - b))) <= 2 * TOL_F32


def test_false_sharing_claim_is_flagged(pa, orc):
    """shared_blocks that promise blocks the tables do not share: the kernel
    reads the first member's blocks for the pack and flags BAD_SHARE; nothing
    non-finite comes out."""
    prep = prepare(W.WORKLOADS["llama8b"].replace(num_seqs=6, len_lo=512, len_hi=900))
    k, v = prep.k_pool, prep.v_pool
    sb = np.full(prep.case.spec.num_seqs, 1000, dtype=np.int32)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run_shared(pa, prep, k, v, sb, flag=flag)
    assert int(flag.item()) & pa.DEVERR_BAD_SHARE
    assert torch.isfinite(out.float()).all()


def test_native_block_manager_counts(pa):
    """BlockManager.shared_blocks against the tables it hands out."""
    spec = _spec(prompts=3, samples=4, prompt_len=300, extra_hi=40)
    case = W.draw(spec)
    bm = pa.BlockManager(case.num_blocks, spec.block_size, case.free_order)
    sid = 0
    for _ in range(spec.prompts):
        bm.add_sequence(sid, spec.prompt_len)
        for s in range(1, spec.samples):
            bm.fork(sid, sid + s)
        sid += spec.samples
    for b in range(spec.num_seqs):
        for _ in range(int(case.extra_tokens[b])):
            bm.append_slot(b)
    seqs = list(range(spec.num_seqs))
    width = max(len(bm.block_table(b)) for b in seqs)
    tables = bm.tables(seqs, width).numpy()
    lens = np.array([bm.seq_len(b) for b in seqs], dtype=np.int32)
    assert np.array_equal(bm.shared_blocks(seqs).numpy(),
                          shared_blocks_of(tables, lens, spec.block_size))


@pytest.mark.slow
def test_full_size_shared_prefix(pa, orc):
    """The benchmark's workload (32 prompts x 8 samples), every sequence compared."""
    spec = W.WORKLOADS["shared_prefix"]
    prep = prepare(spec)
    k, v, sb = _inputs(prep)
    ref = _ref(orc, prep, k, v)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run_shared(pa, prep, k, v, sb, flag=flag)
    o = as_f64(out)
    assert np.all(np.isfinite(o))
    assert float(np.max(np.abs(o - ref))) <= 2e-3
    assert int(flag.item()) == 0
