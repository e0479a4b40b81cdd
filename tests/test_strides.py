"""Pools in other layouts, passed as strided views with no copy ("How PagedAttention
Works in vLLM ...", "Code Example" and "split_kv_cache": K and V are views of one
cache tensor).  Three layouts of the logical [num_blocks, block_size, Hkv, D] pool:

  interleaved  one (nb, 2, bs, Hkv, D) tensor per layer; K = t[:, 0], V = t[:, 1]
  head_major   (nb, Hkv, bs, D) tensors seen through permute(0, 2, 1, 3)
  layered      (nb, 3, bs, Hkv, D) tensors holding three layers; layer 1's view

reshape_and_cache and copy_blocks must be bit-exact on the logical view and leave
every other byte of the tensor alone; decode must match the oracle run on the
logical (contiguous) pools.  Bytes outside the logical view are NaN bit patterns."""
import numpy as np
import pytest
import torch

import oracle
import pa_workloads as W
from harness import TOL_F32, as_f64, fp8_case, prepare, stored_within, to_dev

pytestmark = pytest.mark.gpu

LAYOUTS = ["interleaved", "head_major", "layered"]


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


def _physical(layout, nb, bs, hkv, d, np_dtype, fill):
    """(physical K array, physical V array, view function) for a layout; the
    view function maps a physical array (numpy or torch) to its logical K or V
    pool."""
    if layout == "interleaved":
        t = np.full((nb, 2, bs, hkv, d), fill, dtype=np_dtype)
        return t, None, (lambda a, which: a[:, which])
    if layout == "head_major":
        k = np.full((nb, hkv, bs, d), fill, dtype=np_dtype)
        v = np.full((nb, hkv, bs, d), fill, dtype=np_dtype)
        return k, v, (lambda a, which: a.permute(0, 2, 1, 3) if isinstance(a, torch.Tensor)
                      else a.transpose(0, 2, 1, 3))
    if layout == "layered":
        k = np.full((nb, 3, bs, hkv, d), fill, dtype=np_dtype)
        v = np.full((nb, 3, bs, hkv, d), fill, dtype=np_dtype)
        return k, v, (lambda a, which: a[:, 1])
    raise ValueError(layout)


class Pools:
    """Logical K / V pools living inside physical tensors of a layout, on host
    (numpy, for the oracle) and device (torch views, for the library)."""

    def __init__(self, layout, k_logical, v_logical, fill, torch_dtype):
        nb, bs, hkv, d = k_logical.shape
        self.layout = layout
        pk, pv, self.view = _physical(layout, nb, bs, hkv, d, k_logical.dtype, fill)
        self.shared = pv is None  # K and V share one tensor
        self.host_k = pk
        self.host_v = pk if self.shared else pv
        self._vk(self.host_k, 0)[...] = k_logical
        self._vk(self.host_v, 1)[...] = v_logical
        def dev(a):
            a = a.copy()
            return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()
        self.dev_k = dev(self.host_k)
        self.dev_v = self.dev_k if self.shared else dev(self.host_v)
        if torch_dtype is not None:
            self.dev_k = self.dev_k.view(torch_dtype)
            self.dev_v = self.dev_k if self.shared else self.dev_v.view(torch_dtype)

    def _vk(self, a, which):
        return self.view(a, which)

    def k(self):
        return self.view(self.dev_k, 0)

    def v(self):
        return self.view(self.dev_v, 1)

    def dev_arrays(self):
        """The physical device tensors as raw integer arrays."""
        def raw(t):
            t = t.detach().cpu()
            if t.dtype in (torch.float16, torch.bfloat16):
                t = t.view(torch.int16)
            return t.numpy().view(self.host_k.dtype)
        return raw(self.dev_k), (None if self.shared else raw(self.dev_v))


def _spec_tiny():
    return W.WORKLOADS["tiny"]


@pytest.mark.parametrize("layout", LAYOUTS)
def test_reshape_and_cache_strided_bit_exact(pa, layout):
    prep = prepare(_spec_tiny())
    s = prep.case.spec
    pools = Pools(layout, prep.k_pool, prep.v_pool, W.NAN_BITS[s.dtype], torch.float16)
    # the expected physical tensors: the oracle's write into the logical views
    exp_k = pools.host_k.copy()
    exp_v = exp_k if pools.shared else pools.host_v.copy()
    lk = np.ascontiguousarray(pools.view(exp_k, 0))
    lv = np.ascontiguousarray(pools.view(exp_v, 1))
    oracle.reshape_and_cache(prep.case.new_k, prep.case.new_v, lk, lv, prep.new_slots)
    pools.view(exp_k, 0)[...] = lk
    pools.view(exp_v, 1)[...] = lv
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.reshape_and_cache(to_dev(prep.case.new_k, s.dtype), to_dev(prep.case.new_v, s.dtype),
                         pools.k(), pools.v(), to_dev(prep.new_slots), error_flag=flag)
    torch.cuda.synchronize()
    got_k, got_v = pools.dev_arrays()
    assert np.array_equal(got_k, exp_k)
    if not pools.shared:
        assert np.array_equal(got_v, exp_v)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("layout", LAYOUTS)
def test_copy_blocks_strided_bit_exact(pa, layout):
    prep = prepare(_spec_tiny())
    s = prep.case.spec
    pools = Pools(layout, prep.k_pool, prep.v_pool, W.NAN_BITS[s.dtype], torch.float16)
    nb = prep.k_pool.shape[0]
    rng = np.random.default_rng(7)
    ids = rng.permutation(nb)
    pairs = np.stack([ids[:6], ids[6:12]], axis=1).astype(np.int32)
    exp_k = pools.host_k.copy()
    exp_v = exp_k if pools.shared else pools.host_v.copy()
    for arr, which in ((exp_k, 0), (exp_v, 1)):
        view = pools.view(arr, which)
        for src, dst in pairs:
            view[dst] = view[src]
    pa.copy_blocks([pools.k()], [pools.v()], to_dev(pairs))
    torch.cuda.synchronize()
    got_k, got_v = pools.dev_arrays()
    assert np.array_equal(got_k, exp_k)
    if not pools.shared:
        assert np.array_equal(got_v, exp_v)


def _reduced_llama(**kw):
    return W.WORKLOADS["llama8b"].replace(num_seqs=6, len_lo=300, len_hi=900, **kw)


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("psize", [0, 64])
def test_decode_strided_matches_oracle(pa, orc, layout, psize):
    prep = prepare(_reduced_llama())
    s = prep.case.spec
    pools = Pools(layout, prep.k_pool, prep.v_pool, W.NAN_BITS[s.dtype], torch.bfloat16)
    ref = orc.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                     W.scale_of(s), s.dtype)
    q = to_dev(prep.case.q, s.dtype)
    lens = to_dev(prep.seq_lens)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for out_dtype in (torch.bfloat16, torch.float32):
        out = torch.empty(q.shape, dtype=out_dtype, device="cuda")
        pa.decode_attention(out, q, pools.k(), pools.v(), to_dev(prep.tables), lens,
                            int(prep.seq_lens.max()), W.scale_of(s), partition_size=psize,
                            error_flag=flag)
        torch.cuda.synchronize()
        if out_dtype == torch.float32:
            assert float(np.max(np.abs(as_f64(out) - ref))) <= TOL_F32
        else:
            assert stored_within(out, ref, s.dtype)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("layout", LAYOUTS)
def test_decode_strided_256_token_blocks(pa, orc, layout):
    """256-token blocks in every layout: a tile covers a sixteenth of a block."""
    prep = prepare(W.WORKLOADS["llama8b"].replace(num_seqs=5, len_lo=100, len_hi=1400,
                                                  block_size=256, seed=61))
    s = prep.case.spec
    pools = Pools(layout, prep.k_pool, prep.v_pool, W.NAN_BITS[s.dtype], torch.bfloat16)
    ref = orc.decode(prep.case.q, prep.k_pool, prep.v_pool, prep.tables, prep.seq_lens,
                     W.scale_of(s), s.dtype)
    q = to_dev(prep.case.q, s.dtype)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.decode_attention(out, q, pools.k(), pools.v(), to_dev(prep.tables), to_dev(prep.seq_lens),
                        int(prep.seq_lens.max()), W.scale_of(s), error_flag=flag)
    torch.cuda.synchronize()
    assert float(np.max(np.abs(as_f64(out) - ref))) <= TOL_F32
    assert int(flag.item()) == 0


def test_decode_fp8_head_major(pa, orc):
    """E4M3 code pools in the head-major layout (NaN codes outside the tokens)."""
    spec, prep, kc, vc = fp8_case(31, B=5, lo=200, hi=700)
    pools = Pools("head_major", kc, vc, 0x7F, None)
    ref = orc.decode_fp8(prep.case.q, kc, vc, 0.05, 0.04, prep.tables, prep.seq_lens,
                         W.scale_of(spec), spec.dtype)
    q = to_dev(prep.case.q, spec.dtype)
    ks = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    vs = torch.tensor([0.04], dtype=torch.float32, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    pa.decode_attention_fp8(out, q, pools.k(), pools.v(), ks, vs, to_dev(prep.tables),
                            to_dev(prep.seq_lens), int(prep.seq_lens.max()), W.scale_of(spec))
    torch.cuda.synchronize()
    o = as_f64(out)
    assert np.all(np.isfinite(o))
    assert float(np.max(np.abs(o - ref))) <= TOL_F32


def test_strided_host_validation(pa):
    """Strides the TMA loads cannot take are refused before any launch."""
    lib = pa.lib
    bad = pa.CacheStrides(2 * 16 * 8 * 128, 8 * 128 + 4, 128)  # token stride not 16-byte
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    st = lib.pa_decode_attention_strided(
        dummy.data_ptr(), 1, dummy.data_ptr(), 1, dummy.data_ptr(), dummy.data_ptr(),
        __import__("ctypes").byref(bad), 0, None, None, dummy.data_ptr(), 64, dummy.data_ptr(),
        1, 1024, 32, 8, 128, 64, 16, 0.1, 0, ws.data_ptr(), ws.numel(), None, None)
    assert st == 1
