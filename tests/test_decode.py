"""Paged decode attention on the GPU against the fp64 oracle.

Tolerances: outputs stored in the 16-bit input type must be within 2e-3
max-abs of the oracle (fp16/bf16 storage, fp32 accumulation); the fp32-output
mode, which removes the final storage rounding, must be within 1e-4.  Pools are
NaN-poisoned in every slot that holds no token, so any read past a sequence's
end or of a block outside its table shows up as NaN."""
import os

import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import as_f64, prepare, stored_within, to_dev

pytestmark = pytest.mark.gpu

TOL_STORED = 2e-3
TOL_F32 = 1e-4
NTHREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _run(pa, prep, lens=None, out_dtype=None, partition_size=None, k=None, v=None, tables=None,
         flag=None):
    s = prep.case.spec
    lens = prep.seq_lens if lens is None else lens
    q = to_dev(prep.case.q, s.dtype)
    dk = to_dev(prep.k_pool, s.dtype) if k is None else k
    dv = to_dev(prep.v_pool, s.dtype) if v is None else v
    tb = to_dev(prep.tables if tables is None else tables)
    out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device="cuda")
    ps = s.partition_size if partition_size is None else partition_size
    pa.decode_attention(out, q, dk, dv, tb, to_dev(lens.astype(np.int32)), int(lens.max()),
                        W.scale_of(s), partition_size=ps, error_flag=flag)
    torch.cuda.synchronize()
    return out


def _oracle(orc, prep, lens=None, k=None, v=None, tables=None, seqs=None):
    s = prep.case.spec
    lens = prep.seq_lens if lens is None else lens
    tables = prep.tables if tables is None else tables
    q = prep.case.q
    if seqs is not None:
        q, tables, lens = q[seqs], tables[seqs], lens[seqs]
    return orc.decode(q, prep.k_pool if k is None else k, prep.v_pool if v is None else v,
                      tables, lens, W.scale_of(s), s.dtype, nthreads=NTHREADS)


def _maxerr(out, ref, seqs=None):
    o = as_f64(out)
    if seqs is not None:
        o = o[seqs]
    assert np.all(np.isfinite(o)), "non-finite output"
    return float(np.max(np.abs(o - ref)))


def _stored_within(out, ref, dtype):
    return stored_within(out, ref, dtype, TOL_F32)


def _reduced(name):
    base = W.WORKLOADS[name]
    if name == "llama8b":
        return base.replace(num_seqs=6, len_lo=512, len_hi=1100)
    if name == "longtail":
        return base.replace(num_seqs=40, new_rows=40)
    if name == "longctx":
        return base.replace(num_seqs=2, fixed_lens=(4096, 4096))
    if name == "shared_prefix":
        return base.replace(prompts=2, num_seqs=16)
    return base


@pytest.mark.parametrize("name", ["tiny", "llama8b", "longtail", "longctx", "shared_prefix"])
def test_decode_reduced(pa, orc, name):
    """Every workload's shape at a size the oracle runs in seconds (several tiles
    per sequence, ragged last tiles), stored and fp32 outputs."""
    prep = prepare(_reduced(name))
    s = prep.case.spec
    k, v = prep.k_pool, prep.v_pool
    if prep.cow_pairs is not None:
        # the decode step sees the pool after copy-on-write and the appends
        import oracle
        k, v = k.copy(), v.copy()
        oracle.copy_blocks([k, v], prep.cow_pairs, int(np.prod(k.shape[1:])) * 2)
        oracle.reshape_and_cache(prep.case.new_k, prep.case.new_v, k, v, prep.new_slots)
    ref = _oracle(orc, prep, k=k, v=v)
    dk, dv = to_dev(k, s.dtype), to_dev(v, s.dtype)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(pa, prep, k=dk, v=dv, flag=flag)
    assert _maxerr(out, ref) <= TOL_STORED
    out32 = _run(pa, prep, k=dk, v=dv, out_dtype=torch.float32)
    assert _maxerr(out32, ref) <= TOL_F32
    assert int(flag.item()) == 0


def test_tiny_write_then_attend(pa, orc):
    """Tiny workload: reshape_and_cache of the 4 new tokens at their next slots
    (the 16-token sequence first gets a fifth block), then attention over
    lengths + 1 reads them back."""
    prep = prepare(W.WORKLOADS["tiny"])
    s = prep.case.spec
    k, v = prep.k_pool.copy(), prep.v_pool.copy()
    orc.reshape_and_cache(prep.case.new_k, prep.case.new_v, k, v, prep.new_slots)
    lens1 = prep.seq_lens + 1
    ref = _oracle(orc, prep, lens=lens1, k=k, v=v)
    dk, dv = to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype)
    pa.reshape_and_cache(to_dev(prep.case.new_k, s.dtype), to_dev(prep.case.new_v, s.dtype),
                         dk, dv, to_dev(prep.new_slots))
    out = _run(pa, prep, lens=lens1, k=dk, v=dv, out_dtype=torch.float32)
    assert _maxerr(out, ref) <= TOL_F32
    # the 16-token sequence's new token sits in a fifth block
    assert prep.tables[2, 4] >= 0


@pytest.mark.parametrize("psize", [0, 16, 32, 64, 512, 4096])
def test_partition_sizes_agree(pa, orc, psize):
    spec = W.WORKLOADS["llama8b"].replace(num_seqs=5, len_lo=1, len_hi=1500, seed=77)
    prep = prepare(spec)
    ref = _oracle(orc, prep)
    out32 = _run(pa, prep, out_dtype=torch.float32, partition_size=psize)
    assert _maxerr(out32, ref) <= TOL_F32


@pytest.mark.parametrize("bs,dtype,hq,hkv,d", [
    (4, "bf16", 8, 2, 128), (8, "f16", 16, 4, 64), (32, "f16", 8, 8, 128),
    (64, "bf16", 16, 2, 128), (128, "bf16", 4, 1, 64), (16, "f16", 24, 8, 128),
    (16, "bf16", 64, 8, 128), (256, "bf16", 32, 8, 128), (256, "f16", 8, 2, 64),
])
def test_shapes(pa, orc, bs, dtype, hq, hkv, d):
    spec = W.Spec("shape", 7, hq, hkv, d, bs, dtype, seed=bs * 7 + hq, len_dist="uniform",
                  len_lo=1, len_hi=700)
    prep = prepare(spec)
    ref = _oracle(orc, prep)
    out32 = _run(pa, prep, out_dtype=torch.float32)
    assert _maxerr(out32, ref) <= TOL_F32
    # lengths down to 1 give |out| near 1-2, where one storage ulp of bf16 alone
    # exceeds 2e-3: the stored check is the fp32 bound plus half an ulp
    out = _run(pa, prep)
    assert _stored_within(out, ref, dtype)


@pytest.mark.parametrize("psize", [0, 64])
def test_batch_of_64_short_sequences(pa, orc, psize):
    """64 sequences of 1..400 tokens: without partitions the plan walks each
    sequence's few cut points and the combine runs a warp per head; with
    64-token partitions (about ten partials per sequence) it counts them in
    closed form and the combine splits each head's partials across warps."""
    spec = W.WORKLOADS["llama8b"].replace(len_lo=1, len_hi=400, seed=2001)
    prep = prepare(spec)
    ref = _oracle(orc, prep)
    out = _run(pa, prep, partition_size=psize)
    # short sequences: |out| reaches a few units, where bf16 storage alone
    # rounds by more than 2e-3; the fp32 output carries the tight bound
    assert _stored_within(out, ref, spec.dtype)
    out32 = _run(pa, prep, out_dtype=torch.float32, partition_size=psize)
    assert _maxerr(out32, ref) <= TOL_F32


def test_empty_and_single_token_sequences(pa, orc):
    spec = W.Spec("edge", 6, 8, 2, 128, 16, "bf16", seed=5, len_dist="fixed",
                  fixed_lens=(0, 1, 16, 17, 0, 33))
    prep = prepare(spec)
    ref = _oracle(orc, prep)
    out32 = _run(pa, prep, out_dtype=torch.float32)
    o = as_f64(out32)
    assert np.all(o[0] == 0) and np.all(o[4] == 0)
    assert _maxerr(out32, ref) <= TOL_F32
    # seq_len 1: the output is that token's value row, exactly (fp32 out)
    vrow = prep.v_pool[prep.tables[1, 0], 0]  # [Hkv, D] bits
    import oracle
    vv = oracle.bf16_to_double(vrow)
    for h in range(8):
        assert np.array_equal(o[1, h], vv[h // 4])


def test_placement_invariance_bitwise(pa):
    """Relabelling physical blocks (data and tables together) leaves the GPU
    output bit-identical: the summation order does not depend on placement."""
    spec = W.WORKLOADS["llama8b"].replace(num_seqs=4, len_lo=100, len_hi=900, seed=9)
    prep = prepare(spec)
    out_a = _run(pa, prep, out_dtype=torch.float32)
    nb = prep.case.num_blocks
    perm = np.random.default_rng(4).permutation(nb)
    kp, vp = np.empty_like(prep.k_pool), np.empty_like(prep.v_pool)
    kp[perm], vp[perm] = prep.k_pool, prep.v_pool
    tp = np.where(prep.tables >= 0, perm[np.maximum(prep.tables, 0)], -1).astype(np.int32)
    out_b = _run(pa, prep, out_dtype=torch.float32, k=to_dev(kp, "bf16"), v=to_dev(vp, "bf16"),
                 tables=tp)
    assert torch.equal(out_a, out_b)


def test_repeat_runs_bitwise_identical(pa):
    spec = W.WORKLOADS["longtail"].replace(num_seqs=64, new_rows=0, seed=3)
    prep = prepare(spec)
    a = _run(pa, prep)
    b = _run(pa, prep)
    assert torch.equal(a, b)


def test_bad_block_id_flagged_and_skipped(pa, orc):
    spec = W.WORKLOADS["llama8b"].replace(num_seqs=3, len_lo=64, len_hi=64, seed=12)
    prep = prepare(spec)
    tables = prep.tables.copy()
    tables[1, 2] = prep.case.num_blocks + 5       # tokens 32..47 of sequence 1 are unreachable
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(pa, prep, out_dtype=torch.float32, tables=tables, flag=flag)
    assert int(flag.item()) & pa.DEVERR_BAD_BLOCK
    # the other sequences are unaffected
    ref = _oracle(orc, prep)
    o = as_f64(out)
    assert np.max(np.abs(o[[0, 2]] - ref[[0, 2]])) <= TOL_F32
    # sequence 1 equals attention over its 48 reachable tokens
    import oracle
    keep = [t for t in range(64) if not (32 <= t < 48)]
    t1 = prep.tables[1]
    blk = np.array([t1[t // 16] for t in keep])
    off = np.array([t % 16 for t in keep])
    k = np.ascontiguousarray(prep.k_pool[blk, off][:, None])   # [48, 1, Hkv, D]: block size 1
    v = np.ascontiguousarray(prep.v_pool[blk, off][:, None])
    ref1 = oracle.decode(prep.case.q[1:2], k, v, np.arange(48, dtype=np.int32)[None],
                         np.array([48], np.int32), W.scale_of(spec), "bf16")
    assert np.max(np.abs(o[1] - ref1[0])) <= TOL_F32


def test_seq_len_above_max_is_flagged(pa):
    spec = W.WORKLOADS["llama8b"].replace(num_seqs=2, len_lo=40, len_hi=40, seed=13)
    prep = prepare(spec)
    s = prep.case.spec
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = to_dev(prep.case.q, s.dtype)
    out = torch.empty_like(q)
    pa.decode_attention(out, q, to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype),
                        to_dev(prep.tables), to_dev(prep.seq_lens), 32, W.scale_of(s),
                        error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_BAD_SEQLEN
    assert torch.isfinite(out.float()).all()


# --------------------------------------------------------------------------
# full sizes, in the launch configuration the benchmark times
@pytest.mark.parametrize("psize", [0, 16])
def test_more_sequences_than_the_plans_shared_table(pa, orc, psize):
    """4500 short sequences: more than the 4096 entries whose tile prefix sums
    the plan keeps in shared memory, so the plan and the CTAs locate tiles
    through the prefix sums in the workspace; with 16-token partitions every
    tile is its own partial."""
    spec = W.Spec("many", 4500, 8, 2, 64, 16, "bf16", seed=91, len_dist="uniform", len_lo=1,
                  len_hi=40)
    prep = prepare(spec)
    ref = _oracle(orc, prep)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out32 = _run(pa, prep, out_dtype=torch.float32, partition_size=psize, flag=flag)
    assert _maxerr(out32, ref) <= TOL_F32
    assert int(flag.item()) == 0


# --------------------------------------------------------------------------
@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama8b", "longtail", "longctx", "shared_prefix"])
def test_decode_full_size(pa, orc, name):
    prep = prepare(W.WORKLOADS[name])
    s = prep.case.spec
    k, v = prep.k_pool, prep.v_pool
    if prep.cow_pairs is not None:
        import oracle
        k, v = k.copy(), v.copy()
        oracle.copy_blocks([k, v], prep.cow_pairs, int(np.prod(k.shape[1:])) * 2)
        oracle.reshape_and_cache(prep.case.new_k, prep.case.new_v, k, v, prep.new_slots)
    # every sequence of the batch, element by element
    ref = _oracle(orc, prep, k=k, v=v)
    dk, dv = to_dev(k, s.dtype), to_dev(v, s.dtype)
    out = _run(pa, prep, k=dk, v=dv)
    assert _maxerr(out, ref) <= TOL_STORED
    assert torch.isfinite(out.float()).all()


def test_copy_on_write_step_end_to_end(pa, orc):
    """Parallel sampling with a shared prompt, all on the GPU: the native block
    manager plans the step (same tables, slots and copy pairs as the reference
    manager), copy_blocks makes the copies, reshape_and_cache writes every
    sample's new tokens, decode attends -- against the oracle doing the same
    three steps.  Invariants: shared full prompt blocks are untouched, at most one
    copy per sequence, copy targets are distinct, refcounts match the tables."""
    import oracle
    spec = W.WORKLOADS["shared_prefix"].replace(prompts=3, num_seqs=24, seed=71)
    prep = prepare(spec)
    s = prep.case.spec
    bm_ref = prep.extra["bm"]
    # the native manager, driven by the same operations
    bm = pa.BlockManager(prep.case.num_blocks, s.block_size, prep.case.free_order)
    sid = 0
    for _ in range(s.prompts):
        bm.add_sequence(sid, s.prompt_len)
        for k in range(1, s.samples):
            bm.fork(sid, sid + k)
        sid += s.samples
    slots, cow = [], []
    for b in range(s.num_seqs):
        for _ in range(int(prep.case.extra_tokens[b])):
            slot, c = bm.append_slot(b)
            slots.append(slot)
            if c is not None:
                cow.append(c)
    assert slots == prep.new_slots.tolist()
    assert cow == [tuple(x) for x in prep.cow_pairs.tolist()]
    for b in range(s.num_seqs):
        assert bm.block_table(b) == bm_ref.block_table(b)
    assert all(bm.refcount(i) == bm_ref.refcount[i] for i in range(prep.case.num_blocks))
    # invariants of the plan
    dst = [d for _, d in cow]
    assert len(set(dst)) == len(dst)
    assert len(cow) <= s.num_seqs and len(cow) == s.prompts * (s.samples - 1)
    full_prompt_blocks = sorted({blk for b in range(0, s.num_seqs, s.samples)
                                 for blk in bm_ref.block_table(b)[: s.prompt_len // s.block_size]})
    for blk in full_prompt_blocks:
        assert bm.refcount(blk) == s.samples
    # oracle chain
    k, v = prep.k_pool.copy(), prep.v_pool.copy()
    block_bytes = int(np.prod(k.shape[1:])) * 2
    oracle.copy_blocks([k, v], prep.cow_pairs, block_bytes)
    oracle.reshape_and_cache(prep.case.new_k, prep.case.new_v, k, v, prep.new_slots)
    ref = _oracle(orc, prep, k=k, v=v)
    # GPU chain
    dk, dv = to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.copy_blocks([dk], [dv], to_dev(prep.cow_pairs), error_flag=flag)
    pa.reshape_and_cache(to_dev(prep.case.new_k, s.dtype), to_dev(prep.case.new_v, s.dtype),
                         dk, dv, to_dev(prep.new_slots), error_flag=flag)
    out = _run(pa, prep, k=dk, v=dv, out_dtype=torch.float32, flag=flag)
    assert int(flag.item()) == 0
    from harness import bits_of
    assert np.array_equal(bits_of(dk), k) and np.array_equal(bits_of(dv), v)
    # shared full blocks are bit-identical to their initial contents
    assert np.array_equal(bits_of(dk)[full_prompt_blocks], prep.k_pool[full_prompt_blocks])
    assert np.array_equal(bits_of(dv)[full_prompt_blocks], prep.v_pool[full_prompt_blocks])
    assert _maxerr(out, ref) <= TOL_F32


def test_end_to_end_step_from_host_buffers(pa, orc):
    """DecodeStep called directly (pa_decode_step on one stream): pinned host
    inputs -> plan on the host, reshape_and_cache + decode -> pinned host
    output, three steps in a row with new inputs each step."""
    spec = W.WORKLOADS["llama8b"].replace(num_seqs=5, len_lo=40, len_hi=600, seed=41)
    prep = prepare(spec)
    s = prep.case.spec
    B = s.num_seqs
    bm = prep.extra["bm"]
    dk, dv = to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype)
    k_ref, v_ref = prep.k_pool.copy(), prep.v_pool.copy()
    width = prep.tables.shape[1] + 4
    step = pa.DecodeStep(dk, dv, B, s.num_q_heads, width, int(prep.seq_lens.max()) + 8,
                         W.scale_of(s))
    td = {"bf16": torch.bfloat16, "f16": torch.float16}[s.dtype]
    h = step.host(0)
    g = torch.Generator().manual_seed(3)
    for it in range(3):
        slots = np.array([bm.append_slot(b)[0] for b in range(B)], np.int32)
        lens = np.array([bm.lengths[b] for b in range(B)], np.int32)
        tables = np.full((B, width), -1, np.int32)
        for b in range(B):
            t = bm.block_table(b)
            tables[b, :len(t)] = t
        q = W.randn_bits((B, s.num_q_heads, s.head_dim), s.dtype, g)
        nk = W.randn_bits((B, s.num_kv_heads, s.head_dim), s.dtype, g)
        nv = W.randn_bits((B, s.num_kv_heads, s.head_dim), s.dtype, g)
        for name, src in (("q", q), ("new_k", nk), ("new_v", nv)):
            h[name].copy_(torch.from_numpy(src).view(torch.int16).view(td))
        h["slots"].copy_(torch.from_numpy(slots))
        h["tables"].copy_(torch.from_numpy(tables))
        h["lens"].copy_(torch.from_numpy(lens))
        out = step()
        orc.reshape_and_cache(nk, nv, k_ref, v_ref, slots)
        ref = orc.decode(q, k_ref, v_ref, tables, lens, W.scale_of(s), s.dtype, nthreads=4)
        assert np.max(np.abs(out.double().numpy() - ref)) <= TOL_STORED


def test_end_to_end_pipelined_slots(pa, orc):
    """DecodeStep with two slots: the host fills one slot while the other
    step is in flight (submit step i + 1, then wait for step i); every step
    appends one token per sequence and attends the token the step before it
    wrote (the kernels of both slots run in submission order), and each output
    matches the oracle on the pools as they stand after that step's writes."""
    spec = W.WORKLOADS["llama8b"].replace(num_seqs=5, len_lo=40, len_hi=600, seed=42)
    prep = prepare(spec)
    s = prep.case.spec
    B = s.num_seqs
    bm = prep.extra["bm"]
    dk, dv = to_dev(prep.k_pool, s.dtype), to_dev(prep.v_pool, s.dtype)
    k_ref, v_ref = prep.k_pool.copy(), prep.v_pool.copy()
    width = prep.tables.shape[1] + 4
    step = pa.DecodeStep(dk, dv, B, s.num_q_heads, width, int(prep.seq_lens.max()) + 8,
                         W.scale_of(s), slots=2)
    td = {"bf16": torch.bfloat16, "f16": torch.float16}[s.dtype]
    g = torch.Generator().manual_seed(5)
    refs = {}

    def fill(slot, it):
        slots = np.array([bm.append_slot(b)[0] for b in range(B)], np.int32)
        lens = np.array([bm.lengths[b] for b in range(B)], np.int32)
        tables = np.full((B, width), -1, np.int32)
        for b in range(B):
            t = bm.block_table(b)
            tables[b, :len(t)] = t
        q = W.randn_bits((B, s.num_q_heads, s.head_dim), s.dtype, g)
        nk = W.randn_bits((B, s.num_kv_heads, s.head_dim), s.dtype, g)
        nv = W.randn_bits((B, s.num_kv_heads, s.head_dim), s.dtype, g)
        h = step.host(slot)
        for name, src in (("q", q), ("new_k", nk), ("new_v", nv)):
            h[name].copy_(torch.from_numpy(src).view(torch.int16).view(td))
        h["slots"].copy_(torch.from_numpy(slots))
        h["tables"].copy_(torch.from_numpy(tables))
        h["lens"].copy_(torch.from_numpy(lens))
        orc.reshape_and_cache(nk, nv, k_ref, v_ref, slots)
        refs[it] = orc.decode(q, k_ref, v_ref, tables, lens, W.scale_of(s), s.dtype, nthreads=4)

    steps = 5
    fill(0, 0)
    step.submit(0)
    for it in range(1, steps):
        fill(it % 2, it)
        step.submit(it % 2)
        out = step.wait((it - 1) % 2)
        assert np.max(np.abs(out.double().numpy() - refs[it - 1])) <= TOL_STORED
    out = step.wait((steps - 1) % 2)
    assert np.max(np.abs(out.double().numpy() - refs[steps - 1])) <= TOL_STORED
