"""The multi-GPU path on the CPU: two gloo ranks.

The decode step shards over sequences with no exchange: each rank decodes its
own sequences and the batch result is the concatenation.  Here two ranks run
the oracle on their halves of one batch and the gathered result must equal the
single-process result bit for bit; the benchmark's per-rank seeding and
max/sum-over-ranks reductions are exercised with the same process group."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import bench
        import oracle
        import pa_workloads as W
        from harness import prepare
        spec = W.WORKLOADS["longtail"].replace(num_seqs=12, new_rows=0, seed=5)
        prep = prepare(spec)
        mine = np.arange(rank, spec.num_seqs, world)
        out = oracle.decode(prep.case.q[mine], prep.k_pool, prep.v_pool, prep.tables[mine],
                            prep.seq_lens[mine], W.scale_of(spec), spec.dtype)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, out))
        # reductions used by the benchmark
        mx = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        sm = bench.sum_over_ranks(1.0 + rank, world, torch.device("cpu"))
        seeds = [bench.rank_spec(spec, r, world).seed for r in range(world)]
        if rank == 0:
            full = oracle.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables,
                                 prep.seq_lens, W.scale_of(spec), spec.dtype)
            merged = np.empty_like(full)
            for idx, part in gathered:
                merged[idx] = part
            q.put(("ok", bool(np.array_equal(merged, full)), mx, sm, seeds))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put(("error", repr(e), None, None, None))
        raise


def test_two_rank_sharded_decode_equals_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    status, same, mx, sm, seeds = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
    assert status == "ok", same
    assert same
    assert mx == 11.0 and sm == 3.0
    assert len(set(seeds)) == 2
    assert all(p.exitcode == 0 for p in procs)
