"""Prefix caching end to end on the CPU: the native block manager's tables
with the fp64 oracle's cache writes and attention.

A second request with the same prompt shares the first request's full
blocks ("PagedAttention", "Sharing and copy-on-write": requests that begin
with one system prompt can hold the same blocks) and only writes the rows of
its uncached tokens; attending those tokens over the shared blocks with the
multi-query rule gives exactly what the first request computes for the same
tokens over its own blocks.  Both sides are the oracle, so the check is
bit-exact: it pins that sharing blocks changes nothing in what is attended."""
import numpy as np
import pytest
import torch

import pa_workloads as W


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _rows(n, hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    return W.randn_bits((n, hkv, d), "bf16", g)


@pytest.mark.parametrize("L,bs", [(37, 8), (70, 16), (5, 4), (64, 16)])
def test_uncached_tail_over_shared_blocks_equals_the_full_prompt(pa, orc, L, bs):
    hq, hkv, d = 8, 2, 64
    nb = 64
    bm = pa.BlockManager(nb, bs)
    prompt = [int(t) for t in np.random.default_rng(L).integers(0, 5000, L)]
    k_pool = np.full((nb, bs, hkv, d), W.NAN_BITS["bf16"], np.uint16)
    v_pool = k_pool.copy()
    # the prompt's key / value rows (the same tokens give the same rows)
    k_rows, v_rows = _rows(L, hkv, d, 1), _rows(L, hkv, d, 2)

    def slots_of(seq, first):
        t = bm.block_table(seq)
        return np.array([t[p // bs] * bs + p % bs for p in range(first, L)], np.int32)

    assert bm.add_sequence_with_prefix(0, prompt) == 0
    orc.reshape_and_cache(k_rows, v_rows, k_pool, v_pool, slots_of(0, 0))
    cached = bm.add_sequence_with_prefix(1, prompt)
    assert cached == (L // bs) * bs
    before = k_pool.copy()
    orc.reshape_and_cache(k_rows[cached:], v_rows[cached:], k_pool, v_pool, slots_of(1, cached))
    # the shared blocks were not written again
    shared = bm.block_table(1)[:cached // bs]
    assert np.array_equal(k_pool[shared], before[shared])

    # queries: the uncached tokens of request 1, and the same tokens of request 0
    n = L - cached
    if n == 0:  # the prompt ends on a block boundary: every token is shared
        assert bm.block_table(1) == bm.block_table(0)
        return
    q = W.randn_bits((n, hq, d), "bf16", torch.Generator().manual_seed(3))
    tables, lens = bm.fill_tables([0, 1], -(-L // bs))
    qs = np.array([0, n], np.int32)
    scale = d ** -0.5
    via_shared = orc.decode_multi(q, qs, k_pool, v_pool, tables.numpy()[1:], lens.numpy()[1:],
                                  scale, "bf16")
    via_own = orc.decode_multi(q, qs, k_pool, v_pool, tables.numpy()[:1], lens.numpy()[:1],
                               scale, "bf16")
    assert np.all(np.isfinite(via_shared))
    assert np.array_equal(via_shared, via_own)


def test_two_requests_added_in_one_step_share_rows_written_once(pa, orc):
    """Two requests with one prompt added back to back, before any row is
    written: the second hits the first's full blocks (a block enters the cache
    when it is allocated), so the first request's write alone fills the rows
    both attend; the second writes only its uncached tail.  Freeing the first
    leaves the shared blocks held by the second, still cached."""
    L, bs, hq, hkv, d, nb = 45, 8, 4, 2, 64, 32
    bm = pa.BlockManager(nb, bs)
    prompt = [int(t) for t in np.random.default_rng(7).integers(0, 5000, L)]
    assert bm.add_sequence_with_prefix(0, prompt) == 0
    cached = bm.add_sequence_with_prefix(1, prompt)
    assert cached == (L // bs) * bs
    t0, t1 = bm.block_table(0), bm.block_table(1)
    assert t1[:cached // bs] == t0[:cached // bs] and t1[-1] != t0[-1]
    k_pool = np.full((nb, bs, hkv, d), W.NAN_BITS["bf16"], np.uint16)
    v_pool = k_pool.copy()
    k_rows, v_rows = _rows(L, hkv, d, 1), _rows(L, hkv, d, 2)
    s0 = np.array([t0[p // bs] * bs + p % bs for p in range(L)], np.int32)
    s1 = np.array([t1[p // bs] * bs + p % bs for p in range(cached, L)], np.int32)
    orc.reshape_and_cache(k_rows, v_rows, k_pool, v_pool, s0)
    orc.reshape_and_cache(k_rows[cached:], v_rows[cached:], k_pool, v_pool, s1)
    n = L - cached
    q = W.randn_bits((n, hq, d), "bf16", torch.Generator().manual_seed(3))
    tables, lens = bm.fill_tables([0, 1], -(-L // bs))
    qs = np.array([0, n], np.int32)
    a = orc.decode_multi(q, qs, k_pool, v_pool, tables.numpy()[1:], lens.numpy()[1:], 0.125, "bf16")
    b = orc.decode_multi(q, qs, k_pool, v_pool, tables.numpy()[:1], lens.numpy()[:1], 0.125, "bf16")
    assert np.all(np.isfinite(a)) and np.array_equal(a, b)
    bm.free_sequence(0)
    for blk in t1[:cached // bs]:
        assert bm.refcount(blk) == 1
    assert bm.stats()["cached_blocks"] == cached // bs
    assert bm.add_sequence_with_prefix(2, prompt) == cached
