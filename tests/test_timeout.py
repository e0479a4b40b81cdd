"""Bounded pipeline waits, exercised on purpose: with a 1 ns limit on the
consuming warps' waits for landed stages, those waits run out, the kernel
flags PA_DEVERR_TIMEOUT and returns (the loading warp keeps its 2 s limit,
including its final wait for every copy it issued, so no copy is in flight
when a CTA exits).  The same call with the default limit then gives the
exact result: the context stays usable.  No fault, trap or endless loop is
involved; the longest wait is the loading warp's 2 s."""
import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import as_f64, prepare, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def test_consumer_wait_timeout_is_flagged_and_the_context_survives(pa, orc):
    prep = prepare(W.WORKLOADS["llama8b"].replace(num_seqs=16, len_lo=1000, len_hi=3000,
                                                  seed=81))
    s = prep.case.spec
    args = (to_dev(prep.case.q, s.dtype), to_dev(prep.k_pool, s.dtype),
            to_dev(prep.v_pool, s.dtype), to_dev(prep.tables), to_dev(prep.seq_lens),
            int(prep.seq_lens.max()), W.scale_of(s))
    out = torch.empty(args[0].shape, dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.set_consumer_wait_limit_ns(1)
    try:
        pa.decode_attention(out, *args, error_flag=flag)
        torch.cuda.synchronize()
    finally:
        pa.set_consumer_wait_limit_ns(0)
    assert int(flag.item()) & pa.DEVERR_TIMEOUT
    # the default limit again: no flag, and the oracle's result
    flag.zero_()
    pa.decode_attention(out, *args, error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    ref = orc.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                     W.scale_of(s), s.dtype, nthreads=8)
    assert float(np.max(np.abs(as_f64(out) - ref))) <= 1e-4
