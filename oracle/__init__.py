"""Oracle for the paged KV-cache hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it,
and it shares no code with the CUDA sources: its C half (``pa_oracle.c``) has
its own 16-bit float decoders, slot arithmetic and fp64 attention.

What each function follows (page title and section):

* ``slot_mapping``   -- "PagedAttention", "How attention reads paged memory"
  and its block-size-4 figure: token p of a sequence sits in logical block
  p // block_size at offset p % block_size of the physical block that the
  block table names.
* ``reshape_and_cache`` -- "How PagedAttention Works in vLLM to Maximize
  Memory Efficiency", "write_to_paged_cache: Direct In-Place Updates" and
  "Code Example: Direct PagedAttention Usage".
* ``copy_blocks``    -- "PagedAttention", "How does copy-on-write work for
  parallel sampling?".
* ``decode``         -- "PagedAttention", "How attention reads paged memory":
  gather through the block table, then softmax(scale q K^T) V in fp64.
* ``reshape_and_cache_fp8`` / ``decode_fp8`` -- the same over a cache of 8-bit
  E4M3 codes ("write_to_paged_cache" takes kv_cache_dtype, k_scale, v_scale;
  the pages show only "auto", so the fp8 rule is a reading: the cache holds
  e4m3(x / scale) and reads back code * scale).

Pins (tests/test_oracle.py): the pages' worked example and code example, a
pure-Python ``math.fsum`` brute force (``oracle.brute``), the float64 library
attention of torch on an identity block table, closed forms and placement
invariance.  No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
LIB_PATH = os.path.join(_HERE, "libpa_oracle.so")

F16 = 0
BF16 = 1
_DTYPES = {"f16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16}

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(LIB_PATH) or (
            os.path.getmtime(LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", _SRC, "-o", tmp, "-lm", "-lpthread"])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB_PATH)
        i32, i64, p = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
        lib.orc_half_to_double.restype = ctypes.c_double
        lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_double.restype = ctypes.c_double
        lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_slot_mapping.restype = None
        lib.orc_slot_mapping.argtypes = [p, i64, p, p, i64, i32, p]
        lib.orc_reshape_and_cache.restype = None
        lib.orc_reshape_and_cache.argtypes = [p, p, i64, i64, p, p, p, i64,
                                              i32, i32, i32]
        lib.orc_copy_blocks.restype = None
        lib.orc_copy_blocks.argtypes = [p, i32, p, i64, i64]
        lib.orc_e4m3_to_double.restype = ctypes.c_double
        lib.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.orc_float_to_e4m3.restype = ctypes.c_uint8
        lib.orc_float_to_e4m3.argtypes = [ctypes.c_float]
        lib.orc_reshape_and_cache_fp8.restype = None
        lib.orc_reshape_and_cache_fp8.argtypes = [p, p, i64, i64, p, p, p, i64, i32, i32, i32,
                                                  i32, ctypes.c_float, ctypes.c_float]
        lib.orc_decode_fp8.restype = ctypes.c_int
        lib.orc_decode_fp8.argtypes = [p, p, p, p, ctypes.c_double, ctypes.c_double, p, i64, p,
                                       i32, i32, i32, i32, i32, ctypes.c_double, i32, i32]
        lib.orc_decode_multi.restype = ctypes.c_int
        lib.orc_decode_multi.argtypes = [p, p, p, p, p, p, i64, p, i32, i32, i32, i32, i32,
                                         ctypes.c_double, i32, i32]
        lib.orc_decode.restype = ctypes.c_int
        lib.orc_decode.argtypes = [p, p, p, p, p, i64, p, i32, i32, i32, i32,
                                   i32, ctypes.c_double, i32, i32]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _dtype_code(dtype) -> int:
    return _DTYPES[str(dtype).replace("torch.", "")]


def half_to_double(bits) -> np.ndarray:
    """Decode IEEE binary16 bit patterns (uint16) to float64, element by element."""
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.orc_half_to_double(int(b)) for b in flat],
                    dtype=np.float64).reshape(np.shape(bits))


def bf16_to_double(bits) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16) to float64, element by element."""
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.orc_bf16_to_double(int(b)) for b in flat],
                    dtype=np.float64).reshape(np.shape(bits))


def slot_mapping(block_tables: np.ndarray, seq_idx, pos, block_size: int) -> np.ndarray:
    """Flat pool slot of position pos[i] of sequence seq_idx[i] (int64)."""
    lib = _load()
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    si = np.ascontiguousarray(seq_idx, dtype=np.int32)
    ps = np.ascontiguousarray(pos, dtype=np.int32)
    out = np.empty(si.shape[0], dtype=np.int64)
    lib.orc_slot_mapping(_ptr(bt), bt.shape[1], _ptr(si), _ptr(ps), si.shape[0],
                         int(block_size), _ptr(out))
    return out


def reshape_and_cache(key: np.ndarray, value: np.ndarray, key_cache: np.ndarray,
                      value_cache: np.ndarray, slot_mapping: np.ndarray) -> None:
    """Scatter key/value [T, Hkv, D] (uint16 bits) into the pools in place.

    Pools are uint16 arrays [num_blocks, block_size, Hkv, D]; a negative slot
    skips its token."""
    lib = _load()
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    k = np.ascontiguousarray(key, dtype=np.uint16)
    v = np.ascontiguousarray(value, dtype=np.uint16)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
    _, bs, hkv, d = key_cache.shape
    lib.orc_reshape_and_cache(_ptr(k), _ptr(v), hkv * d, hkv * d,
                              _ptr(key_cache), _ptr(value_cache), _ptr(sm),
                              sm.shape[0], bs, hkv, d)


def copy_blocks(caches, block_mapping: np.ndarray, block_bytes: int) -> None:
    """caches: list [K0, V0, K1, V1, ...] of C-contiguous arrays, modified in place."""
    lib = _load()
    assert len(caches) % 2 == 0
    for c in caches:
        assert c.flags.c_contiguous
    arr = (ctypes.c_void_p * len(caches))(*[c.ctypes.data for c in caches])
    bm = np.ascontiguousarray(block_mapping, dtype=np.int32).reshape(-1, 2)
    lib.orc_copy_blocks(ctypes.cast(arr, ctypes.c_void_p), len(caches) // 2,
                        _ptr(bm), bm.shape[0], int(block_bytes))


def decode(q: np.ndarray, key_cache: np.ndarray, value_cache: np.ndarray,
           block_tables: np.ndarray, seq_lens: np.ndarray, scale: float,
           dtype, nthreads: int = 1) -> np.ndarray:
    """fp64 paged decode attention.  q [B, Hq, D] and the pools are uint16 bits
    of ``dtype`` ('f16' or 'bf16'); returns float64 [B, Hq, D]."""
    lib = _load()
    qq = np.ascontiguousarray(q, dtype=np.uint16)
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, D = qq.shape
    _, bs, hkv, d2 = key_cache.shape
    assert d2 == D and bt.shape[0] == B and sl.shape[0] == B
    out = np.empty((B, Hq, D), dtype=np.float64)
    rc = lib.orc_decode(_ptr(out), _ptr(qq), _ptr(key_cache), _ptr(value_cache),
                        _ptr(bt), bt.shape[1], _ptr(sl), B, Hq, hkv, D, bs,
                        float(scale), _dtype_code(dtype), int(nthreads))
    if rc != 0:
        raise RuntimeError("orc_decode failed with code %d" % rc)
    return out


def decode_multi(q: np.ndarray, q_start: np.ndarray, key_cache: np.ndarray,
                 value_cache: np.ndarray, block_tables: np.ndarray, seq_lens: np.ndarray,
                 scale: float, dtype, nthreads: int = 1) -> np.ndarray:
    """fp64 multi-query paged attention: sequence b owns query rows
    q_start[b] .. q_start[b+1]-1 of q [T, Hq, D] (its last tokens); query i of
    its n attends the first seq_lens[b] - n + i + 1 tokens.  Returns float64
    [T, Hq, D]."""
    lib = _load()
    qq = np.ascontiguousarray(q, dtype=np.uint16)
    qs = np.ascontiguousarray(q_start, dtype=np.int32)
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    T, Hq, D = qq.shape
    B = sl.shape[0]
    _, bs, hkv, d2 = key_cache.shape
    assert d2 == D and bt.shape[0] == B and qs.shape[0] == B + 1 and int(qs[-1]) == T
    out = np.empty((T, Hq, D), dtype=np.float64)
    rc = lib.orc_decode_multi(_ptr(out), _ptr(qq), _ptr(qs), _ptr(key_cache), _ptr(value_cache),
                              _ptr(bt), bt.shape[1], _ptr(sl), B, Hq, hkv, D, bs, float(scale),
                              _dtype_code(dtype), int(nthreads))
    if rc != 0:
        raise RuntimeError("orc_decode_multi failed with code %d" % rc)
    return out


# --------------------------------------------------------------------------
# fp8 (E4M3) cache: codes = e4m3(x / scale) taken in float; reads code * scale
# --------------------------------------------------------------------------
def e4m3_to_double(codes) -> np.ndarray:
    """Decode E4M3 codes (uint8), element by element."""
    lib = _load()
    flat = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.orc_e4m3_to_double(int(c)) for c in flat],
                    dtype=np.float64).reshape(np.shape(codes))


def float_to_e4m3(x) -> np.ndarray:
    """Nearest E4M3 code of each float32 value (ties to even, saturating at 448)."""
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib.orc_float_to_e4m3(float(v)) for v in flat],
                    dtype=np.uint8).reshape(np.shape(x))


def reshape_and_cache_fp8(key: np.ndarray, value: np.ndarray, key_cache: np.ndarray,
                          value_cache: np.ndarray, slot_mapping: np.ndarray, dtype,
                          k_scale: float, v_scale: float) -> None:
    """Write key/value [T, Hkv, D] (uint16 bits of ``dtype``) into uint8 code
    pools [num_blocks, block_size, Hkv, D] in place."""
    lib = _load()
    assert key_cache.dtype == np.uint8 and key_cache.flags.c_contiguous
    assert value_cache.dtype == np.uint8 and value_cache.flags.c_contiguous
    k = np.ascontiguousarray(key, dtype=np.uint16)
    v = np.ascontiguousarray(value, dtype=np.uint16)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
    _, bs, hkv, d = key_cache.shape
    lib.orc_reshape_and_cache_fp8(_ptr(k), _ptr(v), hkv * d, hkv * d, _ptr(key_cache),
                                  _ptr(value_cache), _ptr(sm), sm.shape[0], bs, hkv, d,
                                  _dtype_code(dtype), float(k_scale), float(v_scale))


def decode_fp8(q: np.ndarray, key_cache: np.ndarray, value_cache: np.ndarray,
               k_scale: float, v_scale: float, block_tables: np.ndarray,
               seq_lens: np.ndarray, scale: float, q_dtype, nthreads: int = 1) -> np.ndarray:
    """fp64 paged decode attention over an E4M3 cache (elements read as
    code * k_scale / code * v_scale); q holds uint16 bits of ``q_dtype``."""
    lib = _load()
    qq = np.ascontiguousarray(q, dtype=np.uint16)
    assert key_cache.dtype == np.uint8 and value_cache.dtype == np.uint8
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, D = qq.shape
    _, bs, hkv, d2 = key_cache.shape
    assert d2 == D and bt.shape[0] == B and sl.shape[0] == B
    out = np.empty((B, Hq, D), dtype=np.float64)
    rc = lib.orc_decode_fp8(_ptr(out), _ptr(qq), _ptr(key_cache), _ptr(value_cache),
                            float(k_scale), float(v_scale), _ptr(bt), bt.shape[1], _ptr(sl), B,
                            Hq, hkv, D, bs, float(scale), _dtype_code(q_dtype), int(nthreads))
    if rc != 0:
        raise RuntimeError("orc_decode_fp8 failed with code %d" % rc)
    return out
