"""Pins for the oracle: what the pages and the mathematics fix, CPU only.

Each test checks the oracle against something other than itself: the pages'
worked example and code example (tests/golden/), the standard library's IEEE
codecs, a pure-Python fsum brute force, torch's float64 attention on an
identity block table, closed forms and placement invariance.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import pa_workloads as W
from oracle import brute
from oracle.blockmgr import RefBlockManager

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(x, dtype):
    td = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    return torch.as_tensor(x, dtype=torch.float64).to(td).view(torch.int16).numpy().view(np.uint16)


def _to_f64(bits, dtype):
    td = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(td).to(torch.float64).numpy()


# --------------------------------------------------------------------------
# 16-bit decoders against library codecs, every bit pattern
# --------------------------------------------------------------------------
def test_half_decoder_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint16)
    mine = orc.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, mine[0x8000]) == -1.0


def test_bf16_decoder_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint16)
    mine = orc.bf16_to_double(bits)
    ref = _to_f64(bits, "bf16")
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


# --------------------------------------------------------------------------
# Slot arithmetic: the worked example (block size 4, 22 tokens)
# --------------------------------------------------------------------------
def test_worked_example_slots(orc):
    g = _load_golden("worked_example_bs4.json")
    bs = g["block_size"]
    phys = g["physical_blocks_in_logical_order"]
    table = np.array([phys], dtype=np.int32)
    n = g["num_tokens"]
    slots = orc.slot_mapping(table, np.zeros(n, np.int32), np.arange(n, dtype=np.int32), bs)
    for blk, toks in zip(phys, g["tokens_per_block_in_logical_order"]):
        for off, t in enumerate(toks):
            assert slots[t] // bs == blk
            assert slots[t] % bs == off
    # the figure's last block holds two tokens
    assert len(g["tokens_per_block_in_logical_order"][-1]) == n - (len(phys) - 1) * bs
    # every token gets its own slot
    assert len(set(slots.tolist())) == n


def test_worked_example_decode_reads_listed_blocks(orc):
    """Attention over the figure's table reads exactly the listed blocks: a
    pool that holds distinct values only there gives the brute-force result,
    and poisoning any unlisted block or the tail of block 0 changes nothing."""
    g = _load_golden("worked_example_bs4.json")
    bs, n = g["block_size"], g["num_tokens"]
    phys = g["physical_blocks_in_logical_order"]
    rng = np.random.default_rng(3)
    nb, hkv, hq, d = 12, 1, 2, 8
    kc = _bits(rng.standard_normal((nb, bs, hkv, d)), "f16")
    vc = _bits(rng.standard_normal((nb, bs, hkv, d)), "f16")
    q = _bits(rng.standard_normal((1, hq, d)), "f16")
    table = np.array([phys], dtype=np.int32)
    lens = np.array([n], dtype=np.int32)
    out = orc.decode(q, kc, vc, table, lens, 0.3, "f16")
    kp, vp = kc.copy(), vc.copy()
    for b in range(nb):
        if b not in phys:
            kp[b] = W.NAN_BITS["f16"]
            vp[b] = W.NAN_BITS["f16"]
    kp[0, 2:] = W.NAN_BITS["f16"]  # block 0 holds tokens 20, 21 only
    vp[0, 2:] = W.NAN_BITS["f16"]
    out_p = orc.decode(q, kp, vp, table, lens, 0.3, "f16")
    assert np.array_equal(out, out_p)
    ref = brute.decode_attention(q.tolist(), kc.tolist(), vc.tolist(), table.tolist(),
                                 lens.tolist(), 0.3, "f16")
    assert np.max(np.abs(out - np.array(ref))) <= 1e-12


# --------------------------------------------------------------------------
# reshape_and_cache: the code example, and the definition via numpy indexing
# --------------------------------------------------------------------------
def test_code_example_write(orc):
    g = _load_golden("code_example_write.json")
    _, nb, bs, hkv, d = g["kv_cache_shape"]
    rng = np.random.default_rng(5)
    kc = _bits(rng.standard_normal((nb, bs, hkv, d)), "f16")
    vc = _bits(rng.standard_normal((nb, bs, hkv, d)), "f16")
    k0, v0 = kc.copy(), vc.copy()
    nk = _bits(rng.standard_normal(g["new_rows_shape"]), "f16")
    nv = _bits(rng.standard_normal(g["new_rows_shape"]), "f16")
    orc.reshape_and_cache(nk, nv, kc, vc, np.array(g["slot_mapping"], np.int32))
    changed = np.zeros((nb, bs), bool)
    for row, (blk, off) in enumerate(g["expected_block_and_offset_of_row"]):
        assert np.array_equal(kc[blk, off], nk[row])
        assert np.array_equal(vc[blk, off], nv[row])
        changed[blk, off] = True
    assert np.array_equal(kc[~changed], k0[~changed])
    assert np.array_equal(vc[~changed], v0[~changed])


@pytest.mark.parametrize("bs", [4, 16, 32])
def test_reshape_matches_fancy_index(orc, bs):
    rng = np.random.default_rng(bs)
    nb, hkv, d, T = 20, 4, 64, 37
    kc = rng.integers(0, 65536, (nb, bs, hkv, d), dtype=np.uint16)
    vc = rng.integers(0, 65536, (nb, bs, hkv, d), dtype=np.uint16)
    nk = rng.integers(0, 65536, (T, hkv, d), dtype=np.uint16)  # NaN/denormal bits included
    nv = rng.integers(0, 65536, (T, hkv, d), dtype=np.uint16)
    slots = rng.permutation(nb * bs)[:T].astype(np.int32)
    slots[::5] = -1  # padding tokens
    ek, ev = kc.copy().reshape(nb * bs, hkv, d), vc.copy().reshape(nb * bs, hkv, d)
    keep = slots >= 0
    ek[slots[keep]] = nk[keep]
    ev[slots[keep]] = nv[keep]
    orc.reshape_and_cache(nk, nv, kc, vc, slots)
    assert np.array_equal(kc.reshape(nb * bs, hkv, d), ek)
    assert np.array_equal(vc.reshape(nb * bs, hkv, d), ev)


def test_copy_blocks_bytes(orc):
    rng = np.random.default_rng(7)
    nb, bs, hkv, d, layers = 16, 8, 2, 64, 3
    caches = [rng.integers(0, 65536, (nb, bs, hkv, d), dtype=np.uint16) for _ in range(2 * layers)]
    ref = [c.copy() for c in caches]
    pairs = np.array([[1, 9], [4, 2], [1, 15]], np.int32)
    for c in ref:
        for s, t in pairs:
            c[t] = c[s]
    block_bytes = bs * hkv * d * 2
    orc.copy_blocks(caches, pairs, block_bytes)
    for a, b in zip(caches, ref):
        assert np.array_equal(a, b)


# --------------------------------------------------------------------------
# decode attention
# --------------------------------------------------------------------------
def _tiny_case(seed=11, B=3, hq=4, hkv=2, d=16, bs=4, nb=24, lens=(1, 7, 13), dtype="f16"):
    rng = np.random.default_rng(seed)
    kc = _bits(rng.standard_normal((nb, bs, hkv, d)), dtype)
    vc = _bits(rng.standard_normal((nb, bs, hkv, d)), dtype)
    q = _bits(rng.standard_normal((B, hq, d)), dtype)
    perm = rng.permutation(nb).astype(np.int32)
    maxb = max(-(-L // bs) for L in lens)
    table = np.full((B, maxb + 1), -1, np.int32)
    k = 0
    for b, L in enumerate(lens):
        nblk = -(-L // bs)
        table[b, :nblk] = perm[k:k + nblk]
        k += nblk
    return q, kc, vc, table, np.array(lens, np.int32)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_decode_vs_brute(orc, dtype):
    q, kc, vc, table, lens = _tiny_case(dtype=dtype)
    out = orc.decode(q, kc, vc, table, lens, 0.25, dtype)
    ref = np.array(brute.decode_attention(q.tolist(), kc.tolist(), vc.tolist(),
                                          table.tolist(), lens.tolist(), 0.25, dtype))
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_decode_tiny_workload_vs_brute(orc):
    case = W.draw(W.WORKLOADS["tiny"])
    s = case.spec
    bm = RefBlockManager(case.num_blocks, s.block_size, case.free_order)
    for b, L in enumerate(case.seq_lens):
        bm.add_sequence(b, int(L))
    table = np.full((s.num_seqs, 6), -1, np.int32)
    for b in range(s.num_seqs):
        t = bm.block_table(b)
        table[b, :len(t)] = t
    out = orc.decode(case.q, case.k_pool, case.v_pool, table, case.seq_lens, W.scale_of(s), s.dtype)
    ref = np.array(brute.decode_attention(case.q.tolist(), case.k_pool.tolist(),
                                          case.v_pool.tolist(), table.tolist(),
                                          case.seq_lens.tolist(), W.scale_of(s), s.dtype))
    assert np.max(np.abs(out - ref)) <= 1e-12


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2)])
def test_identity_table_vs_torch_sdpa(orc, hq, hkv):
    """A block table 0, 1, 2, ... over a contiguous buffer is plain attention."""
    rng = np.random.default_rng(hq * 10 + hkv)
    B, d, bs, L = 2, 32, 8, 45
    nblk = -(-L // bs)
    nb = B * nblk
    kc = _bits(rng.standard_normal((nb, bs, hkv, d)), "bf16")
    vc = _bits(rng.standard_normal((nb, bs, hkv, d)), "bf16")
    q = _bits(rng.standard_normal((B, hq, d)), "bf16")
    table = np.arange(nb, dtype=np.int32).reshape(B, nblk)
    lens = np.array([L, L - 9], np.int32)
    scale = 1.0 / math.sqrt(d)
    out = orc.decode(q, kc, vc, table, lens, scale, "bf16")
    K = torch.from_numpy(_to_f64(kc, "bf16")).reshape(B, nblk * bs, hkv, d)
    V = torch.from_numpy(_to_f64(vc, "bf16")).reshape(B, nblk * bs, hkv, d)
    Q = torch.from_numpy(_to_f64(q, "bf16"))
    for b in range(B):
        Lb = int(lens[b])
        kb = K[b, :Lb].permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)  # [Hq, L, d]
        vb = V[b, :Lb].permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q[b][:, None, :], kb, vb, scale=scale)[:, 0, :]
        assert np.max(np.abs(out[b] - ref.numpy())) <= 1e-12


def test_closed_forms(orc):
    rng = np.random.default_rng(21)
    nb, bs, hkv, d, hq = 8, 4, 1, 16, 2
    kc = _bits(rng.standard_normal((nb, bs, hkv, d)), "f16")
    vc = _bits(rng.standard_normal((nb, bs, hkv, d)), "f16")
    q = _bits(rng.standard_normal((1, hq, d)), "f16")
    table = np.array([[5, 2, 7]], np.int32)
    V = _to_f64(vc, "f16")
    # seq_len 1: the output is the single value row, exactly
    out = orc.decode(q, kc, vc, table, np.array([1], np.int32), 0.5, "f16")
    assert np.array_equal(out[0, 0], V[5, 0, 0]) and np.array_equal(out[0, 1], V[5, 0, 0])
    # q = 0: uniform weights, the output is the mean of the value rows
    qz = np.zeros_like(q)
    L = 10
    out = orc.decode(qz, kc, vc, table, np.array([L], np.int32), 0.5, "f16")
    rows = np.stack([V[table[0, t // bs], t % bs, 0] for t in range(L)])
    assert np.max(np.abs(out[0, 0] - rows.mean(0))) <= 1e-12
    # all value rows equal: the output is that row whatever the weights
    ve = vc.copy()
    ve[:] = vc[5, 0, 0]
    out = orc.decode(q, kc, ve, table, np.array([L], np.int32), 0.5, "f16")
    assert np.max(np.abs(out[0] - V[5, 0, 0][None, :])) <= 1e-12
    # one key aligned with a large query: the output is that key's value row
    kk = np.zeros_like(kc)
    kk[7, 1, 0, 3] = _bits(8.0, "f16")
    qq = np.zeros_like(q)
    qq[0, :, 3] = _bits(64.0, "f16")
    out = orc.decode(qq, kk, vc, table, np.array([L], np.int32), 1.0 / 8, "f16")
    assert np.max(np.abs(out[0] - V[7, 1, 0][None, :])) <= 1e-20


def test_empty_sequence_is_zero(orc):
    q, kc, vc, table, lens = _tiny_case(lens=(0, 9, 0))
    out = orc.decode(q, kc, vc, table, np.array([0, 9, 0], np.int32), 0.3, "f16")
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isfinite(out[1]))


def test_permutation_invariance(orc):
    """Relabelling physical blocks (data and tables together) changes nothing."""
    q, kc, vc, table, lens = _tiny_case(seed=4, lens=(5, 17, 11), nb=30)
    out = orc.decode(q, kc, vc, table, lens, 0.4, "f16")
    rng = np.random.default_rng(99)
    perm = rng.permutation(kc.shape[0])          # new id of old block i is perm[i]
    kp, vp = np.empty_like(kc), np.empty_like(vc)
    kp[perm], vp[perm] = kc, vc
    tp = np.where(table >= 0, perm[np.maximum(table, 0)], -1).astype(np.int32)
    out_p = orc.decode(q, kp, vp, tp, lens, 0.4, "f16")
    assert np.array_equal(out, out_p)


def test_threads_do_not_change_result(orc):
    q, kc, vc, table, lens = _tiny_case(seed=8, B=3, lens=(13, 2, 9))
    a = orc.decode(q, kc, vc, table, lens, 0.4, "f16", nthreads=1)
    b = orc.decode(q, kc, vc, table, lens, 0.4, "f16", nthreads=3)
    assert np.array_equal(a, b)


def test_planted_gqa_mistake_is_caught(orc):
    """A plausible slip (query head h reading KV head h % Hkv instead of
    h // group) disagrees with the identity-table library attention."""
    rng = np.random.default_rng(2)
    B, d, bs, L, hq, hkv = 1, 16, 4, 12, 4, 2
    kc = _bits(rng.standard_normal((3, bs, hkv, d)), "f16")
    vc = _bits(rng.standard_normal((3, bs, hkv, d)), "f16")
    q = _bits(rng.standard_normal((B, hq, d)), "f16")
    table = np.arange(3, dtype=np.int32)[None]
    good = orc.decode(q, kc, vc, table, np.array([L], np.int32), 0.25, "f16")
    # the wrong mapping, emulated by permuting the query heads fed to the oracle
    wrong_q = q[:, [0, 2, 1, 3]]
    bad = orc.decode(wrong_q, kc, vc, table, np.array([L], np.int32), 0.25, "f16")[:, [0, 2, 1, 3]]
    assert np.max(np.abs(good - bad)) > 1e-3


# --------------------------------------------------------------------------
# several query tokens per sequence (causal over the paged tokens)
# --------------------------------------------------------------------------
def _multi_case(seed, lens, qlens, hq=4, hkv=2, d=16, bs=4, dtype="f16"):
    rng = np.random.default_rng(seed)
    B = len(lens)
    nblk = [-(-L // bs) for L in lens]
    nb = sum(nblk) + 3
    kc = _bits(rng.standard_normal((nb, bs, hkv, d)), dtype)
    vc = _bits(rng.standard_normal((nb, bs, hkv, d)), dtype)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = _bits(rng.standard_normal((int(qs[-1]), hq, d)), dtype)
    perm = rng.permutation(nb).astype(np.int32)
    table = np.full((B, max(nblk) + 1), -1, np.int32)
    k = 0
    for b in range(B):
        table[b, :nblk[b]] = perm[k:k + nblk[b]]
        k += nblk[b]
    return q, qs, kc, vc, table, np.array(lens, np.int32)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_multi_query_vs_brute(orc, dtype):
    q, qs, kc, vc, table, lens = _multi_case(5, (9, 14, 3, 6), (3, 5, 3, 1), dtype=dtype)
    out = orc.decode_multi(q, qs, kc, vc, table, lens, 0.3, dtype)
    ref = np.array(brute.decode_attention_multi(q.tolist(), qs.tolist(), kc.tolist(), vc.tolist(),
                                                table.tolist(), lens.tolist(), 0.3, dtype))
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_multi_query_identity_table_vs_torch_sdpa(orc):
    """With the block table 0, 1, 2, ... the pool is a contiguous sequence, and
    the n new tokens are the last n queries of causal attention: torch's
    float64 scaled_dot_product_attention with the matching boolean mask (query
    i of n sees key positions <= L - n + i)."""
    rng = np.random.default_rng(9)
    hq, hkv, d, bs, L, n = 8, 2, 32, 8, 41, 6
    nblk = -(-L // bs)
    kc = _bits(rng.standard_normal((nblk, bs, hkv, d)), "bf16")
    vc = _bits(rng.standard_normal((nblk, bs, hkv, d)), "bf16")
    q = _bits(rng.standard_normal((n, hq, d)), "bf16")
    table = np.arange(nblk, dtype=np.int32)[None]
    scale = 1.0 / math.sqrt(d)
    out = orc.decode_multi(q, np.array([0, n], np.int32), kc, vc, table,
                           np.array([L], np.int32), scale, "bf16")
    K = torch.from_numpy(_to_f64(kc, "bf16")).reshape(nblk * bs, hkv, d)[:L]
    V = torch.from_numpy(_to_f64(vc, "bf16")).reshape(nblk * bs, hkv, d)[:L]
    Q = torch.from_numpy(_to_f64(q, "bf16")).permute(1, 0, 2)            # [Hq, n, d]
    kb = K.permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)          # [Hq, L, d]
    vb = V.permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    pos = torch.arange(L)[None, :]
    allowed = pos <= (L - n + torch.arange(n))[:, None]                  # [n, L]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, kb, vb, attn_mask=allowed,
                                                           scale=scale)
    assert np.max(np.abs(out - ref.permute(1, 0, 2).numpy())) <= 1e-12


def test_multi_query_single_token_is_decode(orc):
    """One query token per sequence is the decode step (every token seen)."""
    q, qs, kc, vc, table, lens = _multi_case(6, (9, 14, 1, 6), (1, 1, 1, 1))
    a = orc.decode_multi(q, qs, kc, vc, table, lens, 0.3, "f16")
    b = orc.decode(q, kc, vc, table, lens, 0.3, "f16")
    assert np.array_equal(a, b)


def test_multi_query_last_token_sees_everything(orc):
    """The last of a sequence's new tokens attends the whole sequence: its row
    equals the one-token decode of that sequence; the first new token equals
    the decode of the sequence cut just after it."""
    q, qs, kc, vc, table, lens = _multi_case(7, (12, 20), (4, 6))
    out = orc.decode_multi(q, qs, kc, vc, table, lens, 0.3, "f16")
    last = qs[1:] - 1
    full = orc.decode(q[last], kc, vc, table, lens, 0.3, "f16")
    assert np.max(np.abs(out[last] - full)) <= 1e-15
    first = qs[:-1]
    cut = lens - (qs[1:] - qs[:-1]) + 1
    part = orc.decode(q[first], kc, vc, table, cut, 0.3, "f16")
    assert np.max(np.abs(out[first] - part)) <= 1e-15


def test_planted_causal_off_by_one_is_caught(orc):
    """A plausible slip in the causal limit (query i seeing one token more or
    one less) disagrees with the masked library attention: emulated by
    handing the oracle one more (or one fewer) token than the sequence has."""
    q, qs, kc, vc, table, lens = _multi_case(8, (11,), (4,), hq=2, hkv=2)
    good = orc.decode_multi(q, qs, kc, vc, table, lens, 0.5, "f16")
    for delta in (-1, 1):
        bad = orc.decode_multi(q, qs, kc, vc, table, lens + delta, 0.5, "f16")
        assert np.max(np.abs(good - bad)) > 1e-3


def test_multi_query_more_queries_than_tokens(orc):
    """q_len > seq_len: the leading queries see nothing and give zeros."""
    q, qs, kc, vc, table, lens = _multi_case(4, (3,), (5,))
    out = orc.decode_multi(q, qs, kc, vc, table, lens, 0.3, "f16")
    assert np.all(out[:2] == 0.0)
    assert np.all(np.abs(out[2:]).sum(axis=(1, 2)) > 0)


# --------------------------------------------------------------------------
# fp8 (E4M3) cache pieces
# --------------------------------------------------------------------------
def test_e4m3_decoder_all_codes(orc):
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3_to_double(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.nanmax(mine) == 448.0 and np.min(mine[mine > 0]) == 2.0 ** -9


def test_e4m3_encoder_matches_library_in_range(orc):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * 50,
        rng.standard_normal(1000).astype(np.float32) * 0.01,       # subnormal range
        orc.e4m3_to_double(np.arange(0, 0x7e, dtype=np.uint8)).astype(np.float32),  # exact codes
        ((orc.e4m3_to_double(np.arange(0, 0x7d, dtype=np.uint8)) +
          orc.e4m3_to_double(np.arange(1, 0x7e, dtype=np.uint8))) / 2).astype(np.float32),  # ties
        np.array([0.0, -0.0, 447.9, -447.9, 416.0, 432.0], np.float32),
    ])
    x = np.concatenate([x, -x])
    mine = orc.float_to_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def test_e4m3_encoder_saturates(orc):
    x = np.array([448.0, 449.0, 500.0, 1e6, np.inf, -1e6, -np.inf], np.float32)
    assert orc.float_to_e4m3(x).tolist() == [0x7e, 0x7e, 0x7e, 0x7e, 0x7e, 0xfe, 0xfe]


def test_fp8_write_and_decode_pins(orc):
    """The fp8 write stores e4m3(x / scale); decode over a cache of codes equals
    the 16-bit decode over the dequantised values (codes * scale), and a single
    token returns its dequantised value row."""
    rng = np.random.default_rng(4)
    nb, bs, hkv, d, hq = 6, 4, 2, 16, 4
    B, T = 2, 9
    rows_k = _bits(rng.standard_normal((T, hkv, d)) * 3, "bf16")
    rows_v = _bits(rng.standard_normal((T, hkv, d)) * 3, "bf16")
    kc = np.zeros((nb, bs, hkv, d), np.uint8)
    vc = np.zeros((nb, bs, hkv, d), np.uint8)
    slots = np.array([5, 4, 6, 7, 12, 13, 14, 0, 1], np.int32)
    orc.reshape_and_cache_fp8(rows_k, rows_v, kc, vc, slots, "bf16", 0.5, 2.0)
    exp_k = orc.float_to_e4m3((_to_f64(rows_k, "bf16").astype(np.float32) / np.float32(0.5)))
    assert np.array_equal(kc.reshape(nb * bs, hkv, d)[slots], exp_k)
    exp_v = orc.float_to_e4m3((_to_f64(rows_v, "bf16").astype(np.float32) / np.float32(2.0)))
    assert np.array_equal(vc.reshape(nb * bs, hkv, d)[slots], exp_v)
    q = _bits(rng.standard_normal((B, hq, d)), "bf16")
    table = np.array([[1, 3, 0], [0, 2, 1]], np.int32)
    lens = np.array([9, 1], np.int32)
    out = orc.decode_fp8(q, kc, vc, 0.5, 2.0, table, lens, 0.3, "bf16")
    # same attention with the dequantised cache, through the 16-bit oracle in
    # float64 terms: build it with torch SDPA on gathered values
    Kd = orc.e4m3_to_double(kc) * 0.5
    Vd = orc.e4m3_to_double(vc) * 2.0
    Q = _to_f64(q, "bf16")
    for b in range(B):
        L = int(lens[b])
        ks = np.stack([Kd[table[b, t // bs], t % bs] for t in range(L)])  # [L, hkv, d]
        vs = np.stack([Vd[table[b, t // bs], t % bs] for t in range(L)])
        kk = torch.from_numpy(ks).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
        vv = torch.from_numpy(vs).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[b])[:, None, :], kk, vv, scale=0.3)[:, 0, :].numpy()
        assert np.max(np.abs(out[b] - ref)) <= 1e-12
    assert np.array_equal(out[1, 0], Vd[table[1, 0], 0, 0])
