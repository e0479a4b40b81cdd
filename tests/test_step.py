"""The decode with its split plan made on the host, and the whole decode step
from host buffers through the C entry point pa_decode_step.

- decode_attention_planned (plan from pa_decode_plan, copied to the device)
  gives bit for bit the output of decode_attention, whose plan kernel makes
  the same plan on the device: the same segments mean the same arithmetic.
- A plan made for other lengths or another shape is flagged on the device
  (PA_DEVERR_BAD_SEQLEN / PA_DEVERR_BAD_PLAN) and never read out of bounds.
- pa_decode_step, run for several steps of growing sequences (copy-on-write
  of shared partial blocks on the first append of forked samples), matches
  the fp64 oracle step for step, and leaves pools bit-identical to the
  oracle's writes and copies."""
import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import as_f64, prepare, stored_within, to_dev
from oracle.blockmgr import RefBlockManager

pytestmark = pytest.mark.gpu

TOL_STORED = 2e-3
TOL_F32 = 1e-4


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _dev_args(prep):
    s = prep.case.spec
    return dict(query=to_dev(prep.case.q, s.dtype), key_cache=to_dev(prep.k_pool, s.dtype),
                value_cache=to_dev(prep.v_pool, s.dtype), block_tables=to_dev(prep.tables),
                seq_lens=to_dev(prep.seq_lens), max_seq_len=int(prep.seq_lens.max()),
                scale=W.scale_of(s), partition_size=s.partition_size)


def _planned(pa, prep, a, out, lens_for_plan=None, flag=None):
    s = prep.case.spec
    lens = prep.seq_lens if lens_for_plan is None else lens_for_plan
    plan, _ = pa.decode_plan(torch.from_numpy(np.ascontiguousarray(lens, np.int32)),
                             s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size,
                             a["max_seq_len"], a["partition_size"])
    dplan = plan.to("cuda")
    pa.decode_attention_planned(out, a["query"], a["key_cache"], a["value_cache"],
                                a["block_tables"], a["seq_lens"], a["max_seq_len"], a["scale"],
                                dplan, partition_size=a["partition_size"], error_flag=flag)
    return dplan


SPECS = {
    "tiny": W.WORKLOADS["tiny"],
    "llama8b": W.WORKLOADS["llama8b"].replace(num_seqs=12, len_lo=300, len_hi=2500, seed=41),
    "longtail": W.WORKLOADS["longtail"].replace(num_seqs=96, new_rows=0, seed=42),
    "longctx": W.WORKLOADS["longctx"].replace(num_seqs=2, fixed_lens=(9000, 9000), seed=43),
    "zeros": W.Spec("zeros", 7, 8, 2, 64, 8, "f16", seed=44, len_dist="fixed",
                    fixed_lens=(0, 5, 0, 130, 17, 0, 1)),
}


@pytest.mark.parametrize("name", sorted(SPECS))
@pytest.mark.parametrize("out_dtype", [None, torch.float32])
def test_planned_equals_device_planned_bitwise(pa, orc, name, out_dtype):
    prep = prepare(SPECS[name].replace(new_rows=0))
    a = _dev_args(prep)
    ref = torch.empty(a["query"].shape, dtype=out_dtype or a["query"].dtype, device="cuda")
    pa.decode_attention(ref, **a)
    got = torch.full_like(ref, float("nan"))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    _planned(pa, prep, a, got, flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    assert torch.equal(got.view(torch.int16) if got.element_size() == 2 else got.view(torch.int32),
                       ref.view(torch.int16) if ref.element_size() == 2 else ref.view(torch.int32))
    s = prep.case.spec
    oref = orc.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                      W.scale_of(s), s.dtype, nthreads=8)
    if out_dtype == torch.float32:
        assert float(np.max(np.abs(as_f64(got) - oref))) <= TOL_F32
    else:
        assert stored_within(got, oref, s.dtype)


def test_plan_from_other_lengths_is_flagged_not_read(pa):
    """The device lengths of two sequences differ from the plan's: those two
    are flagged and attended as empty; the others keep their exact result."""
    prep = prepare(SPECS["llama8b"].replace(new_rows=0))
    a = _dev_args(prep)
    ref = torch.empty(a["query"].shape, dtype=torch.float32, device="cuda")
    pa.decode_attention(ref, **a)
    lens = prep.seq_lens.copy()
    lens[3] += 40    # more tiles in the plan than the device length has
    lens[7] = 16     # fewer tiles
    got = torch.full_like(ref, float("nan"))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    _planned(pa, prep, a, got, lens_for_plan=lens, flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_BAD_SEQLEN
    assert torch.isfinite(got).all()
    keep = [b for b in range(lens.size) if b not in (3, 7)]
    # the other sequences' segments may be cut differently: same result to rounding
    assert float((got[keep] - ref[keep]).abs().max()) <= TOL_F32


def test_plan_for_another_shape_computes_nothing(pa):
    prep = prepare(SPECS["llama8b"].replace(new_rows=0))
    a = _dev_args(prep)
    s = prep.case.spec
    plan, _ = pa.decode_plan(torch.from_numpy(prep.seq_lens[:-1].copy()), s.num_q_heads,
                             s.num_kv_heads, s.head_dim, s.block_size, a["max_seq_len"])
    got = torch.full(a["query"].shape, float("nan"), dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.decode_attention_planned(got, a["query"], a["key_cache"], a["value_cache"],
                                a["block_tables"], a["seq_lens"], a["max_seq_len"], a["scale"],
                                plan.to("cuda"), error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == pa.DEVERR_BAD_PLAN
    assert torch.isnan(got).all()  # untouched


def _run_steps(pa, orc, bm, k_pool, v_pool, seqs, steps, hq, hkv, d, bs, dtype, seed,
               out_dtype=None, partition_size=0, max_len_cap=None):
    """Drives `steps` decode steps of `seqs` through DecodeStep (one slot per
    step parity) and the oracle side by side."""
    td = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    B = len(seqs)
    nb = k_pool.shape[0]
    final_max = max(len(bm.block_table(b)) * bs for b in seqs) + steps * bs + bs
    width = -(-final_max // bs)
    max_len = max_len_cap or final_max
    kd, vd = to_dev(k_pool, dtype), to_dev(v_pool, dtype)
    k_ref, v_ref = k_pool.copy(), v_pool.copy()
    runner = pa.DecodeStep(kd, vd, B, hq, width, max_len, d ** -0.5, partition_size,
                           out_dtype=out_dtype, max_cow=B, slots=2)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = torch.Generator().manual_seed(seed)
    tol = TOL_F32 if out_dtype == torch.float32 else None
    ncopies = 0
    for step in range(steps):
        slot = step % 2
        n0 = len(bm.copies)
        slots = np.array([bm.append_slot(b)[0] for b in seqs], np.int32)
        cow = np.array(bm.copies[n0:], np.int32).reshape(-1, 2)
        ncopies += cow.shape[0]
        tables = np.full((B, width), -1, np.int32)
        for i, b in enumerate(seqs):
            t = bm.block_table(b)
            tables[i, :len(t)] = t
        lens = np.array([bm.lengths[b] for b in seqs], np.int32)
        q = W.randn_bits((B, hq, d), dtype, g)
        nk = W.randn_bits((B, hkv, d), dtype, g)
        nv = W.randn_bits((B, hkv, d), dtype, g)
        h = runner.host(slot)
        h["q"].copy_(torch.from_numpy(q).view(torch.int16).view(td))
        h["new_k"].copy_(torch.from_numpy(nk).view(torch.int16).view(td))
        h["new_v"].copy_(torch.from_numpy(nv).view(torch.int16).view(td))
        h["slots"].copy_(torch.from_numpy(slots))
        h["tables"].copy_(torch.from_numpy(tables))
        h["lens"].copy_(torch.from_numpy(lens))
        if cow.size:
            h["cow"][:cow.shape[0]].copy_(torch.from_numpy(cow))
        runner.submit(slot, cow.shape[0], error_flag=flag)
        # the oracle's step meanwhile
        if cow.size:
            orc.copy_blocks([k_ref, v_ref], cow, int(np.prod(k_ref.shape[1:])) * 2)
        orc.reshape_and_cache(nk, nv, k_ref, v_ref, slots)
        oref = orc.decode(q, k_ref, v_ref, tables, lens, d ** -0.5, dtype, nthreads=8)
        out = runner.wait(slot)
        assert int(flag.item()) == 0
        if tol is not None:
            assert float(np.max(np.abs(as_f64(out) - oref))) <= tol
        else:
            assert stored_within(out, oref, dtype)
    torch.cuda.synchronize()
    kb = kd.cpu().view(torch.int16).numpy().view(np.uint16)
    vb = vd.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(kb, k_ref) and np.array_equal(vb, v_ref)
    return ncopies


@pytest.mark.parametrize("out_dtype", [None, torch.float32])
def test_decode_step_plain_batch_several_steps(pa, orc, out_dtype):
    rng = np.random.default_rng(5)
    B, hq, hkv, d, bs = 20, 32, 8, 128, 16
    lens = rng.integers(1, 1500, B)
    nb = int(sum(-(-int(L) // bs) + 2 for L in lens) * 1.2)
    bm = RefBlockManager(nb, bs, rng.permutation(nb).astype(np.int32))
    for b in range(B):
        bm.add_sequence(b, int(lens[b]))
    g = torch.Generator().manual_seed(6)
    k_pool = W.randn_bits((nb, bs, hkv, d), "bf16", g)
    v_pool = W.randn_bits((nb, bs, hkv, d), "bf16", g)
    assert _run_steps(pa, orc, bm, k_pool, v_pool, list(range(B)), 3, hq, hkv, d, bs, "bf16",
                      seed=7, out_dtype=out_dtype) == 0


def test_decode_step_forked_samples_copy_on_write(pa, orc):
    """Prompts of 37 tokens forked into 4 samples each: the first step copies
    the shared partial block for all but the last sample of each prompt
    (pa_copy_blocks inside the step), later steps write in place."""
    prompts, samples, plen = 3, 4, 37
    hq, hkv, d, bs = 8, 2, 64, 16
    nb = 64
    bm = RefBlockManager(nb, bs, np.random.default_rng(8).permutation(nb).astype(np.int32))
    sid = 0
    for _ in range(prompts):
        bm.add_sequence(sid, plen)
        for s in range(1, samples):
            bm.fork(sid, sid + s)
        sid += samples
    g = torch.Generator().manual_seed(9)
    k_pool = W.randn_bits((nb, bs, hkv, d), "f16", g)
    v_pool = W.randn_bits((nb, bs, hkv, d), "f16", g)
    copies = _run_steps(pa, orc, bm, k_pool, v_pool, list(range(sid)), 3, hq, hkv, d, bs, "f16",
                        seed=10)
    assert copies == prompts * (samples - 1)


def test_decode_step_long_context_partitions(pa, orc):
    """Two 5000-token sequences in 512-token partitions: many partials per
    sequence, merged by the combine inside the step."""
    B, hq, hkv, d, bs = 2, 64, 8, 128, 32
    nb = 2 * (5000 // bs + 4)
    bm = RefBlockManager(nb, bs, np.random.default_rng(11).permutation(nb).astype(np.int32))
    for b in range(B):
        bm.add_sequence(b, 5000)
    g = torch.Generator().manual_seed(12)
    k_pool = W.randn_bits((nb, bs, hkv, d), "bf16", g)
    v_pool = W.randn_bits((nb, bs, hkv, d), "bf16", g)
    _run_steps(pa, orc, bm, k_pool, v_pool, [0, 1], 2, hq, hkv, d, bs, "bf16", seed=13,
               out_dtype=torch.float32, partition_size=512)


def test_decode_step_refuses_lengths_beyond_max_before_any_copy(pa):
    k = torch.zeros((8, 16, 2, 64), dtype=torch.float16, device="cuda")
    runner = pa.DecodeStep(k, k.clone(), 2, 4, 4, 64, 0.125)
    h = runner.host(0)
    h["lens"].copy_(torch.tensor([10, 65], dtype=torch.int32))
    with pytest.raises(pa.PagedAttnError, match="INVALID_ARG"):
        runner.submit(0)


@pytest.mark.slow
def test_decode_step_full_size_llama8b(pa, orc):
    """The benchmark's end-to-end configuration: the llama8b batch (64
    sequences, lengths U[512, 4096]) through pa_decode_step from pinned host
    buffers, each sequence appending its current token; every sequence of the
    output compared with the oracle, and the pools' new rows bit-exact."""
    import os
    spec = W.WORKLOADS["llama8b"]
    case = W.draw(spec)
    bs, B = spec.block_size, spec.num_seqs
    bm = RefBlockManager(case.num_blocks, bs, case.free_order)
    lens = case.seq_lens.astype(np.int32)
    for b in range(B):
        bm.add_sequence(b, int(lens[b]) - 1)
    slots = np.array([bm.append_slot(b)[0] for b in range(B)], np.int32)
    width = max(len(bm.block_table(b)) for b in range(B))
    tables = np.full((B, width), -1, np.int32)
    for b in range(B):
        t = bm.block_table(b)
        tables[b, :len(t)] = t
    g = torch.Generator().manual_seed(spec.seed + 7)
    nk = W.randn_bits((B, spec.num_kv_heads, spec.head_dim), spec.dtype, g)
    nv = W.randn_bits((B, spec.num_kv_heads, spec.head_dim), spec.dtype, g)
    td = torch.bfloat16
    kd, vd = to_dev(case.k_pool, spec.dtype), to_dev(case.v_pool, spec.dtype)
    runner = pa.DecodeStep(kd, vd, B, spec.num_q_heads, width, int(lens.max()), W.scale_of(spec))
    h = runner.host(0)
    h["q"].copy_(torch.from_numpy(case.q).view(torch.int16).view(td))
    h["new_k"].copy_(torch.from_numpy(nk).view(torch.int16).view(td))
    h["new_v"].copy_(torch.from_numpy(nv).view(torch.int16).view(td))
    h["slots"].copy_(torch.from_numpy(slots))
    h["tables"].copy_(torch.from_numpy(tables))
    h["lens"].copy_(torch.from_numpy(lens))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    runner.submit(0, error_flag=flag)
    k_ref, v_ref = case.k_pool.copy(), case.v_pool.copy()
    orc.reshape_and_cache(nk, nv, k_ref, v_ref, slots)
    ref = orc.decode(case.q, k_ref, v_ref, tables, lens, W.scale_of(spec), spec.dtype,
                     nthreads=max(1, len(os.sched_getaffinity(0))))
    out = runner.wait(0)
    assert int(flag.item()) == 0
    assert stored_within(out, ref, spec.dtype)
    assert float(np.max(np.abs(as_f64(out) - ref))) <= TOL_STORED
    blocks = np.unique(slots // bs)
    kb = kd[torch.from_numpy(blocks).cuda()].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(kb, k_ref[blocks])
