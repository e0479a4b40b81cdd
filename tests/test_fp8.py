"""fp8 (E4M3) KV cache on the GPU: reshape_and_cache codes bit-exact against the
oracle, decode attention over code pools within the fp32-output tolerance.

Reading (the pages show kv_cache_dtype="auto" only): the cache holds
e4m3(x / scale), the quotient in fp32, round to nearest even, saturating at
448; an element reads back as code * scale."""
import os

import numpy as np
import pytest
import torch

import pa_workloads as W
from harness import fp8_case, TORCH_DTYPE, prepare, to_dev

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_STORED = 2e-3
NAN_E4M3 = 0x7F


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _codes_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def _scales(k, v):
    return (torch.tensor([k], dtype=torch.float32, device="cuda"),
            torch.tensor([v], dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_fp8_reshape_codes_bit_exact(pa, orc, dtype):
    rng = np.random.default_rng(1)
    nb, bs, hkv, d, T = 12, 16, 8, 128, 40
    g = torch.Generator().manual_seed(9)
    rows_k = W.randn_bits((T, hkv, d), dtype, g)
    rows_v = W.randn_bits((T, hkv, d), dtype, g)
    # some large values saturate at 448 after the division
    big = (torch.from_numpy(rows_k[:3].view(np.int16)).view(TORCH_DTYPE[dtype]) * 300)
    rows_k[:3] = big.view(torch.int16).numpy().view(np.uint16)
    kc = rng.integers(0, 256, (nb, bs, hkv, d), dtype=np.uint8)
    vc = rng.integers(0, 256, (nb, bs, hkv, d), dtype=np.uint8)
    slots = rng.permutation(nb * bs)[:T].astype(np.int32)
    slots[::7] = -1
    ek, ev = kc.copy(), vc.copy()
    orc.reshape_and_cache_fp8(rows_k, rows_v, ek, ev, slots, dtype, 0.5, 2.0)
    dk, dv = _codes_dev(kc), _codes_dev(vc)
    ks, vs = _scales(0.5, 2.0)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.reshape_and_cache(to_dev(rows_k, dtype), to_dev(rows_v, dtype), dk, dv, to_dev(slots),
                         kv_cache_dtype="fp8_e4m3", k_scale=ks, v_scale=vs, error_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), ek)
    assert np.array_equal(dv.cpu().numpy(), ev)
    assert int(flag.item()) == 0
    assert (ek.reshape(-1, hkv, d)[slots[:3][slots[:3] >= 0]] & 0x7F == 0x7E).any()  # saturated


def _fp8_case(seed, **kw):
    return fp8_case(seed, **kw)


@pytest.mark.parametrize("q_dtype,psize", [("bf16", 0), ("f16", 0), ("bf16", 512)])
def test_fp8_decode_matches_oracle(pa, orc, q_dtype, psize):
    ks_v, vs_v = 0.05, 0.04
    spec, prep, kc, vc = _fp8_case(21, q_dtype=q_dtype, ks=ks_v, vs=vs_v)
    ref = orc.decode_fp8(prep.case.q, kc, vc, ks_v, vs_v, prep.tables, prep.seq_lens,
                         W.scale_of(spec), q_dtype, nthreads=8)
    q = to_dev(prep.case.q, q_dtype)
    ks, vs = _scales(ks_v, vs_v)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.decode_attention_fp8(out, q, _codes_dev(kc), _codes_dev(vc), ks, vs, to_dev(prep.tables),
                            to_dev(prep.seq_lens), int(prep.seq_lens.max()), W.scale_of(spec),
                            partition_size=psize, error_flag=flag)
    torch.cuda.synchronize()
    o = out.double().cpu().numpy()
    assert np.all(np.isfinite(o))
    assert float(np.max(np.abs(o - ref))) <= TOL_F32
    assert int(flag.item()) == 0
    out16 = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    pa.decode_attention_fp8(out16, q, _codes_dev(kc), _codes_dev(vc), ks, vs,
                            to_dev(prep.tables), to_dev(prep.seq_lens), int(prep.seq_lens.max()),
                            W.scale_of(spec), partition_size=psize)
    torch.cuda.synchronize()
    assert float(np.max(np.abs(out16.double().cpu().numpy() - ref))) <= TOL_STORED


def test_fp8_write_then_attend(pa, orc):
    """New rows written with the fp8 reshape_and_cache at the next slots are read
    back by the fp8 decode over lengths + 1 (block sizes 4 and 32 included)."""
    for bs in (4, 32):
        spec, prep, kc, vc = _fp8_case(33 + bs, B=5, lo=1, hi=400, bs=bs)
        bm = prep.extra["bm"]
        B = spec.num_seqs
        slots = np.array([bm.append_slot(b)[0] for b in range(B)], np.int32)
        lens = (prep.seq_lens + 1).astype(np.int32)
        width = prep.tables.shape[1] + 1
        tables = np.full((B, width), -1, np.int32)
        for b in range(B):
            t = bm.block_table(b)
            tables[b, :len(t)] = t
        g = torch.Generator().manual_seed(5)
        nk = W.randn_bits((B, spec.num_kv_heads, 128), "bf16", g)
        nv = W.randn_bits((B, spec.num_kv_heads, 128), "bf16", g)
        ek, ev = kc.copy(), vc.copy()
        orc.reshape_and_cache_fp8(nk, nv, ek, ev, slots, "bf16", 0.05, 0.04)
        ref = orc.decode_fp8(prep.case.q, ek, ev, 0.05, 0.04, tables, lens, W.scale_of(spec),
                             "bf16", nthreads=8)
        dk, dv = _codes_dev(kc), _codes_dev(vc)
        ks, vs = _scales(0.05, 0.04)
        pa.reshape_and_cache(to_dev(nk, "bf16"), to_dev(nv, "bf16"), dk, dv, to_dev(slots),
                             kv_cache_dtype="fp8_e4m3", k_scale=ks, v_scale=vs)
        q = to_dev(prep.case.q, "bf16")
        out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        pa.decode_attention_fp8(out, q, dk, dv, ks, vs, to_dev(tables), to_dev(lens),
                                int(lens.max()), W.scale_of(spec))
        torch.cuda.synchronize()
        assert np.array_equal(dk.cpu().numpy(), ek)
        assert float(np.max(np.abs(out.double().cpu().numpy() - ref))) <= TOL_F32


@pytest.mark.slow
def test_full_size_fp8_workload(pa, orc):
    """The benchmark's E4M3 workload (llama8b shape) in its launch
    configuration, every sequence compared; NaN codes outside the tokens."""
    from harness import used_slot_mask
    spec = W.WORKLOADS["llama8b_fp8"]
    prep = prepare(spec, poison=False)
    kc, vc = prep.k_pool.copy(), prep.v_pool.copy()
    used = used_slot_mask(prep.tables, prep.seq_lens, prep.case.num_blocks, spec.block_size)
    kc[~used] = NAN_E4M3
    vc[~used] = NAN_E4M3
    q = to_dev(prep.case.q, spec.dtype)
    ks, vs = _scales(spec.k_scale, spec.v_scale)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    pa.decode_attention_fp8(out, q, _codes_dev(kc), _codes_dev(vc), ks, vs, to_dev(prep.tables),
                            to_dev(prep.seq_lens), int(prep.seq_lens.max()), W.scale_of(spec))
    torch.cuda.synchronize()
    o = out.double().cpu().numpy()
    assert np.all(np.isfinite(o))
    ref = orc.decode_fp8(prep.case.q, kc, vc, spec.k_scale, spec.v_scale, prep.tables,
                         prep.seq_lens, W.scale_of(spec), spec.dtype,
                         nthreads=max(1, len(os.sched_getaffinity(0))))
    assert float(np.max(np.abs(o - ref))) <= TOL_F32
