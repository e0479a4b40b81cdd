"""paged_kv_cache_343_b200 -- Python binding of libpagedattn.so.

The library is the product: hand-written sm_100a CUDA kernels behind a C ABI
(``include/pagedattn.h``).  This module only marshals arguments: it turns
torch tensors into pointers, sizes and the current CUDA stream, calls the C
entry point of the same name and raises on a non-OK status.  Every step of
the hot path runs in the library's kernels; there is no fallback.  Importing
this package fails loudly if the library has not been built
(``python paged_kv_cache_343_b200/build.py``).

Entry points (see the header for argument meaning, layout and errors):

* ``reshape_and_cache`` -- scatter new K/V rows into pool slots
  ("How PagedAttention Works in vLLM ...", "write_to_paged_cache").
* ``copy_blocks``       -- copy-on-write block copies ("PagedAttention",
  "How does copy-on-write work for parallel sampling?").
* ``decode_attention``  -- paged decode attention with split-KV partials and a
  combine pass ("PagedAttention", "How attention reads paged memory").
* ``decode_attention_fp8`` -- the same over E4M3 (fp8) code pools written by
  ``reshape_and_cache(..., kv_cache_dtype="fp8_e4m3")``.
* ``decode_attention_shared_prefix`` -- the same result for batches whose
  neighbouring sequences share leading blocks (parallel samples of one
  prompt, "Sharing and copy-on-write"): a shared prefix is read once per pack
  of sequences instead of once per sequence.
* ``decode_attention_multi_query`` -- several new tokens per sequence (a
  recomputed partial block, verified speculated tokens), each attending the
  paged cache causally.
* ``BlockManager``      -- the native host block manager (free list,
  refcounts, copy-on-write planning, shared-prefix counts).
* ``decode_plan`` / ``decode_attention_planned`` -- the split plan made on the
  host from host lengths, and the decode that reads it instead of running its
  plan kernel.
* ``DecodeStep``        -- one decode step from pinned host buffers through the
  C entry points ``pa_decode_step`` / ``_upload`` / ``_run`` / ``_download``:
  the plan on the host, one copy in, the kernels, one copy out (the
  end-to-end call).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "LIB_PATH", "PagedAttnError", "reshape_and_cache", "copy_blocks", "decode_attention",
    "decode_workspace_bytes", "decode_attention_fp8", "decode_attention_noalloc",
    "decode_attention_shared_prefix", "shared_prefix_workspace_bytes",
    "decode_attention_multi_query", "multi_query_workspace_bytes", "BlockManager",
    "DEVERR_BAD_BLOCK", "DEVERR_BAD_SLOT", "DEVERR_BAD_SEQLEN",
    "DEVERR_TIMEOUT", "DEVERR_BAD_SHARE", "DEVERR_BAD_PLAN", "CacheStrides", "version",
    "stream_read", "decode_plan_bytes", "decode_plan", "decode_attention_planned", "split_plan",
    "DecodeStep", "StepShape", "StepLayout", "set_consumer_wait_limit_ns",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")

DEVERR_BAD_BLOCK = 0x1
DEVERR_BAD_SLOT = 0x2
DEVERR_BAD_SEQLEN = 0x4
DEVERR_TIMEOUT = 0x8
DEVERR_BAD_SHARE = 0x10
DEVERR_BAD_PLAN = 0x20

_PA_F16, _PA_BF16, _PA_F32 = 0, 1, 2
_DTYPE_CODE = {torch.float16: _PA_F16, torch.bfloat16: _PA_BF16, torch.float32: _PA_F32}


class PagedAttnError(RuntimeError):
    """A libpagedattn entry point returned a status other than PA_OK."""

    def __init__(self, what: str, status: int, name: str):
        super().__init__("%s failed: %s (%d)" % (what, name, status))
        self.status = status
        self.name = name


class CacheStrides(ctypes.Structure):
    """pa_cache_strides: element strides of a pool whose head_dim is contiguous."""
    _fields_ = [("block_stride", ctypes.c_int64), ("token_stride", ctypes.c_int64),
                ("head_stride", ctypes.c_int64)]


class BmStats(ctypes.Structure):
    """pa_bm_stats_t: memory held by a block manager's sequences."""
    _fields_ = [(name, ctypes.c_int64) for name in (
        "num_blocks", "free_blocks", "held_blocks", "logical_blocks", "num_seqs", "tokens",
        "stored_slots", "waste_slots", "max_waste_per_seq", "cached_blocks")]


class StepShape(ctypes.Structure):
    """pa_step_shape: the batch shape of pa_decode_step."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_seqs", "num_q_heads", "num_kv_heads", "head_dim", "num_blocks", "block_size",
        "table_width", "max_seq_len", "partition_size", "max_cow")] + [
        ("dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("kv_cache_dtype", ctypes.c_int)]


class StepLayout(ctypes.Structure):
    """pa_step_layout: where pa_decode_step's inputs sit in its staging buffer."""
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "query", "new_k", "new_v", "slot_mapping", "block_tables", "seq_lens", "cow_pairs",
        "plan", "host_bytes", "out_bytes", "device_bytes")]


def _pool_strides(cache: torch.Tensor) -> Optional[CacheStrides]:
    """None for a contiguous [nb, bs, Hkv, D] pool, else its strides (head_dim
    must be contiguous)."""
    _need(cache.dim() == 4 and cache.stride(3) == 1, "pools are [nb, bs, Hkv, D] views "
          "with head_dim contiguous")
    if cache.is_contiguous():
        return None
    return CacheStrides(cache.stride(0), cache.stride(1), cache.stride(2))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libpagedattn.so is missing at %s; build it with "
                          "`python paged_kv_cache_343_b200/build.py`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, p, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_status_string.argtypes = [ctypes.c_int]
    lib.pa_version.restype = i32
    lib.pa_version.argtypes = []
    lib.pa_reshape_and_cache.restype = ctypes.c_int
    lib.pa_reshape_and_cache.argtypes = [p, p, i64, i64, p, p, p, i32, i32, i32, i32, i32,
                                         ctypes.c_int, ctypes.c_int, p, p, p, p]
    lib.pa_copy_blocks.restype = ctypes.c_int
    lib.pa_copy_blocks.argtypes = [p, p, i32, p, i32, i32, i64, p, p]
    lib.pa_reshape_and_cache_strided.restype = ctypes.c_int
    lib.pa_reshape_and_cache_strided.argtypes = [p, p, i64, i64, p, p, ctypes.POINTER(CacheStrides),
                                                 p, i32, i32, i32, i32, i32, ctypes.c_int,
                                                 ctypes.c_int, p, p, p, p]
    lib.pa_copy_blocks_strided.restype = ctypes.c_int
    lib.pa_copy_blocks_strided.argtypes = [p, p, i32, ctypes.POINTER(CacheStrides), p, i32, i32,
                                           i32, i32, i32, i32, p, p]
    lib.pa_decode_attention_strided.restype = ctypes.c_int
    lib.pa_decode_attention_strided.argtypes = [p, ctypes.c_int, p, ctypes.c_int, p, p,
                                                ctypes.POINTER(CacheStrides), ctypes.c_int, p, p,
                                                p, i32, p, i32, i32, i32, i32, i32, i32, i32,
                                                ctypes.c_float, i32, p, sz, p, p]
    lib.pa_decode_workspace_bytes.restype = ctypes.c_int
    lib.pa_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32,
                                              ctypes.POINTER(sz)]
    lib.pa_decode_attention.restype = ctypes.c_int
    lib.pa_decode_attention.argtypes = [p, ctypes.c_int, p, p, p, p, i32, p, i32, i32, i32, i32,
                                        i32, i32, i32, ctypes.c_float, ctypes.c_int, i32, p, sz,
                                        p, p]
    lib.pa_decode_attention_fp8.restype = ctypes.c_int
    lib.pa_decode_attention_fp8.argtypes = [p, ctypes.c_int, p, ctypes.c_int, p, p, p, p, p, i32,
                                            p, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                            i32, p, sz, p, p]
    lib.pa_decode_shared_prefix_workspace_bytes.restype = ctypes.c_int
    lib.pa_decode_shared_prefix_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32,
                                                            ctypes.POINTER(sz)]
    lib.pa_decode_attention_shared_prefix.restype = ctypes.c_int
    lib.pa_decode_attention_shared_prefix.argtypes = [p, ctypes.c_int, p, p, p, p, i32, p, p, i32,
                                                      i32, i32, i32, i32, i32, i32,
                                                      ctypes.c_float, ctypes.c_int, i32, p, sz,
                                                      p, p]
    lib.pa_decode_multi_query_workspace_bytes.restype = ctypes.c_int
    lib.pa_decode_multi_query_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32,
                                                          i32, ctypes.POINTER(sz)]
    lib.pa_decode_attention_multi_query.restype = ctypes.c_int
    lib.pa_decode_attention_multi_query.argtypes = [p, ctypes.c_int, p, p, i32, i32, p, p, p, i32,
                                                    p, i32, i32, i32, i32, i32, i32, i32,
                                                    ctypes.c_float, ctypes.c_int, i32, p, sz, p,
                                                    p]
    lib.pa_decode_attention_noalloc.restype = ctypes.c_int
    lib.pa_decode_attention_noalloc.argtypes = [p, ctypes.c_int, p, p, p, p, i32, p, i32, i32, i32,
                                                i32, i32, i32, i32, ctypes.c_float, ctypes.c_int,
                                                i32, p, p]
    lib.pa_decode_plan_bytes.restype = ctypes.c_int
    lib.pa_decode_plan_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32, ctypes.c_int,
                                         ctypes.POINTER(sz)]
    lib.pa_decode_plan.restype = ctypes.c_int
    lib.pa_decode_plan.argtypes = [p, i32, i32, i32, i32, i32, i32, i32, ctypes.c_int, p, sz,
                                   ctypes.POINTER(i32)]
    lib.pa_decode_attention_planned.restype = ctypes.c_int
    lib.pa_decode_attention_planned.argtypes = [p, ctypes.c_int, p, ctypes.c_int, p, p,
                                                ctypes.c_int, p, p, p, i32, p, i32, i32, i32, i32,
                                                i32, i32, i32, ctypes.c_float, i32, p, p, sz, p, p]
    lib.pa_split_plan.restype = ctypes.c_int
    lib.pa_split_plan.argtypes = [p, i32, i32, i32, i32, p, p, p, p, p, ctypes.POINTER(i32),
                                  ctypes.POINTER(i32)]
    lib.pa_decode_step_layout.restype = ctypes.c_int
    lib.pa_decode_step_layout.argtypes = [ctypes.POINTER(StepShape), ctypes.POINTER(StepLayout)]
    lib.pa_decode_step_upload.restype = ctypes.c_int
    lib.pa_decode_step_upload.argtypes = [ctypes.POINTER(StepShape), p, p, sz, p]
    lib.pa_decode_step_run.restype = ctypes.c_int
    lib.pa_decode_step_run.argtypes = [ctypes.POINTER(StepShape), p, i32, p, p, p, p,
                                       ctypes.c_float, p, sz, p, p]
    lib.pa_decode_step_download.restype = ctypes.c_int
    lib.pa_decode_step_download.argtypes = [ctypes.POINTER(StepShape), p, sz, p, p]
    lib.pa_decode_step.restype = ctypes.c_int
    lib.pa_decode_step.argtypes = [ctypes.POINTER(StepShape), p, i32, p, p, p, p, ctypes.c_float,
                                   p, sz, p, p, p]
    lib.pa_set_consumer_wait_limit_ns.restype = None
    lib.pa_set_consumer_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.pa_stream_read.restype = ctypes.c_int
    lib.pa_stream_read.argtypes = [p, i64, p, i32, p]
    lib.pa_bm_create.restype = ctypes.c_int
    lib.pa_bm_create.argtypes = [i32, i32, p, ctypes.POINTER(p)]
    lib.pa_bm_destroy.restype = None
    lib.pa_bm_destroy.argtypes = [p]
    lib.pa_bm_add_sequence.restype = ctypes.c_int
    lib.pa_bm_add_sequence.argtypes = [p, i64, i64]
    lib.pa_bm_add_sequence_with_prefix.restype = ctypes.c_int
    lib.pa_bm_add_sequence_with_prefix.argtypes = [p, i64, ctypes.POINTER(i32), i64,
                                                   ctypes.POINTER(i64)]
    lib.pa_bm_fork.restype = ctypes.c_int
    lib.pa_bm_fork.argtypes = [p, i64, i64]
    lib.pa_bm_append_slot.restype = ctypes.c_int
    lib.pa_bm_append_slot.argtypes = [p, i64, ctypes.POINTER(i64), ctypes.POINTER(i32),
                                      ctypes.POINTER(i32)]
    lib.pa_bm_free_sequence.restype = ctypes.c_int
    lib.pa_bm_free_sequence.argtypes = [p, i64]
    lib.pa_bm_block_table.restype = ctypes.c_int
    lib.pa_bm_block_table.argtypes = [p, i64, p, i32, ctypes.POINTER(i32), ctypes.POINTER(i64)]
    lib.pa_bm_refcount.restype = i32
    lib.pa_bm_refcount.argtypes = [p, i32]
    lib.pa_bm_shared_blocks.restype = ctypes.c_int
    lib.pa_bm_shared_blocks.argtypes = [p, ctypes.POINTER(i64), i32, ctypes.POINTER(i32)]
    lib.pa_bm_num_free.restype = i32
    lib.pa_bm_num_free.argtypes = [p]
    lib.pa_bm_append_slots.restype = ctypes.c_int
    lib.pa_bm_append_slots.argtypes = [p, ctypes.POINTER(i64), i32, ctypes.POINTER(i32),
                                       ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.pa_bm_append_tokens.restype = ctypes.c_int
    lib.pa_bm_append_tokens.argtypes = [p, ctypes.POINTER(i64), i32, ctypes.POINTER(i32),
                                        ctypes.POINTER(i32), ctypes.POINTER(i32),
                                        ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.pa_bm_blocks_needed.restype = ctypes.c_int
    lib.pa_bm_blocks_needed.argtypes = [p, ctypes.POINTER(i64), i32, p, ctypes.POINTER(i64)]
    lib.pa_bm_order_by_prefix.restype = ctypes.c_int
    lib.pa_bm_order_by_prefix.argtypes = [p, ctypes.POINTER(i64), i32, ctypes.POINTER(i32)]
    lib.pa_bm_fill_tables.restype = ctypes.c_int
    lib.pa_bm_fill_tables.argtypes = [p, ctypes.POINTER(i64), i32, p, i32, p]
    lib.pa_bm_stats.restype = ctypes.c_int
    lib.pa_bm_stats.argtypes = [p, ctypes.POINTER(BmStats)]
    return lib


lib = _load()


def version() -> int:
    return int(lib.pa_version())


def _check(status: int, what: str) -> None:
    if status != 0:
        raise PagedAttnError(what, status, lib.pa_status_string(status).decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _dtype_code(dtype: torch.dtype) -> int:
    _need(dtype in _DTYPE_CODE, "unsupported dtype %s: float16 or bfloat16 (float32 for outputs)"
          % dtype)
    return _DTYPE_CODE[dtype]


_KV_CACHE_DTYPE = {"auto": 0, "fp8": 1, "fp8_e4m3": 1}


def reshape_and_cache(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                      value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                      kv_cache_dtype: str = "auto", k_scale: Optional[torch.Tensor] = None,
                      v_scale: Optional[torch.Tensor] = None,
                      error_flag: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> None:
    """key/value [T, Hkv, D] (rows may be strided), caches [nb, bs, Hkv, D], slot_mapping int32 [T].

    kv_cache_dtype "auto": caches hold key's 16-bit type.  "fp8_e4m3": caches
    are uint8 code pools and k_scale / v_scale are one-element float32 device
    tensors (codes = e4m3(x / scale))."""
    _need(kv_cache_dtype in _KV_CACHE_DTYPE, "kv_cache_dtype must be 'auto' or 'fp8_e4m3'")
    fp8 = _KV_CACHE_DTYPE[kv_cache_dtype] == 1
    _need(key.dim() == 3 and value.shape == key.shape, "key/value must be [T, Hkv, D]")
    _need(key_cache.dim() == 4 and tuple(key.shape[1:]) == tuple(key_cache.shape[2:]),
          "key/value rows [Hkv, D] must match the pools' [.., Hkv, D]")
    _need(key.stride(2) == 1 and key.stride(1) == key.shape[2] and
          value.stride(2) == 1 and value.stride(1) == value.shape[2],
          "heads and head_dim must be contiguous inside a row")
    _need(key_cache.shape == value_cache.shape and key_cache.stride() == value_cache.stride(),
          "K and V pools share shape and strides")
    strides = _pool_strides(key_cache)
    _need(slot_mapping.dtype == torch.int32 and slot_mapping.is_contiguous(), "slot_mapping int32")
    if fp8:
        _need(key.dtype == value.dtype and key_cache.dtype == value_cache.dtype == torch.uint8,
              "fp8 caches are uint8 code pools")
        _need(k_scale is not None and v_scale is not None and k_scale.dtype == torch.float32 and
              v_scale.dtype == torch.float32, "fp8 caches need float32 k_scale / v_scale")
    else:
        _need(key.dtype == key_cache.dtype == value.dtype == value_cache.dtype, "dtype mismatch")
    nb, bs, hkv, d = key_cache.shape
    if strides is None:
        _check(lib.pa_reshape_and_cache(
            _ptr(key), _ptr(value), key.stride(0), value.stride(0), _ptr(key_cache),
            _ptr(value_cache), _ptr(slot_mapping), key.shape[0], nb, bs, hkv, d,
            _dtype_code(key.dtype), _KV_CACHE_DTYPE[kv_cache_dtype], _ptr(k_scale),
            _ptr(v_scale), _ptr(error_flag), _stream_handle(stream)), "pa_reshape_and_cache")
    else:
        _check(lib.pa_reshape_and_cache_strided(
            _ptr(key), _ptr(value), key.stride(0), value.stride(0), _ptr(key_cache),
            _ptr(value_cache), ctypes.byref(strides), _ptr(slot_mapping), key.shape[0], nb, bs,
            hkv, d, _dtype_code(key.dtype), _KV_CACHE_DTYPE[kv_cache_dtype], _ptr(k_scale),
            _ptr(v_scale), _ptr(error_flag), _stream_handle(stream)),
            "pa_reshape_and_cache_strided")


def copy_blocks(key_caches: Sequence[torch.Tensor], value_caches: Sequence[torch.Tensor],
                block_mapping: torch.Tensor, error_flag: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> None:
    """block_mapping int32 [N, 2] (src, dst) on the device; one K and one V pool per layer."""
    _need(len(key_caches) == len(value_caches) and len(key_caches) > 0, "one K and V pool per layer")
    _need(block_mapping.dtype == torch.int32 and block_mapping.is_contiguous(), "mapping int32 [N,2]")
    k0 = key_caches[0]
    block_bytes = k0[0].numel() * k0.element_size()
    for c in list(key_caches) + list(value_caches):
        _need(c.shape == k0.shape and c.dtype == k0.dtype and c.stride() == k0.stride(),
              "pool shapes, types and strides differ")
    strides = _pool_strides(k0)
    n = len(key_caches)
    karr = (ctypes.c_void_p * n)(*[c.data_ptr() for c in key_caches])
    varr = (ctypes.c_void_p * n)(*[c.data_ptr() for c in value_caches])
    kp, vp = ctypes.cast(karr, ctypes.c_void_p), ctypes.cast(varr, ctypes.c_void_p)
    if strides is None:
        _check(lib.pa_copy_blocks(kp, vp, n, _ptr(block_mapping), block_mapping.numel() // 2,
                                  k0.shape[0], block_bytes, _ptr(error_flag),
                                  _stream_handle(stream)), "pa_copy_blocks")
    else:
        nb, bs, hkv, d = k0.shape
        _check(lib.pa_copy_blocks_strided(kp, vp, n, ctypes.byref(strides), _ptr(block_mapping),
                                          block_mapping.numel() // 2, nb, bs, hkv, d,
                                          k0.element_size(), _ptr(error_flag),
                                          _stream_handle(stream)), "pa_copy_blocks_strided")


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                           block_size: int, max_seq_len: int, partition_size: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                         block_size, max_seq_len, partition_size,
                                         ctypes.byref(out)), "pa_decode_workspace_bytes")
    return int(out.value)


def shared_prefix_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                  head_dim: int, block_size: int, max_seq_len: int,
                                  partition_size: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.pa_decode_shared_prefix_workspace_bytes(
        num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len, partition_size,
        ctypes.byref(out)), "pa_decode_shared_prefix_workspace_bytes")
    return int(out.value)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A device buffer of nbytes, 256-byte aligned (torch's allocator aligns to 512)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _decode_args(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                 value_cache: torch.Tensor, block_tables: torch.Tensor, seq_lens: torch.Tensor,
                 allow_strided_pools: bool = True) -> Optional[CacheStrides]:
    """Checks of the 16-bit decode entry points, made before any library call:
    contiguous query and out of one shape, 16-bit query and pools of one dtype,
    K and V pools of one shape and strides, int32 tables with contiguous rows,
    int32 contiguous lengths, a supported out dtype.  Returns the pools'
    strides (None when contiguous); allow_strided_pools=False refuses strided
    pools instead."""
    _need(query.dim() == 3 and query.is_contiguous(), "query must be contiguous [B, Hq, D]")
    _need(out.shape == query.shape and out.is_contiguous(), "out must be contiguous [B, Hq, D]")
    _need(key_cache.shape == value_cache.shape and key_cache.stride() == value_cache.stride(),
          "K and V pools share shape and strides")
    strides = _pool_strides(key_cache)
    _need(allow_strided_pools or strides is None, "pools must be contiguous [nb, bs, Hkv, D]")
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.stride(1) == 1, "block_tables int32 [B, W], rows contiguous")
    _need(seq_lens.dtype == torch.int32 and seq_lens.is_contiguous(), "seq_lens int32")
    _need(query.dtype == key_cache.dtype == value_cache.dtype, "query and caches share a dtype")
    _need(key_cache.shape[3] == query.shape[2], "query and pools must share head_dim")
    _need(query.dtype in (torch.float16, torch.bfloat16), "query and pools must be float16 or "
          "bfloat16 (fp8 code pools: decode_attention_fp8)")
    _dtype_code(out.dtype)
    return strides


def decode_attention(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                     value_cache: torch.Tensor, block_tables: torch.Tensor,
                     seq_lens: torch.Tensor, max_seq_len: int, scale: float,
                     partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                     error_flag: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """out/query [B, Hq, D]; caches [nb, bs, Hkv, D] (any strided view with head_dim
    contiguous, e.g. the K and V halves of one interleaved tensor); block_tables
    int32 [B, W]; seq_lens int32 [B]."""
    strides = _decode_args(out, query, key_cache, value_cache, block_tables, seq_lens)
    B, hq, d = query.shape
    nb, bs, hkv, _ = key_cache.shape
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_bytes(B, hq, hkv, d, bs, max_seq_len,
                                                           partition_size), query.device)
    wsb = workspace.numel() * workspace.element_size()
    if strides is None:
        _check(lib.pa_decode_attention(
            _ptr(out), _dtype_code(out.dtype), _ptr(query), _ptr(key_cache), _ptr(value_cache),
            _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens), B, int(max_seq_len), hq,
            hkv, d, nb, bs, float(scale), _dtype_code(query.dtype), int(partition_size),
            _ptr(workspace), wsb, _ptr(error_flag), _stream_handle(stream)),
            "pa_decode_attention")
    else:
        _check(lib.pa_decode_attention_strided(
            _ptr(out), _dtype_code(out.dtype), _ptr(query), _dtype_code(query.dtype),
            _ptr(key_cache), _ptr(value_cache), ctypes.byref(strides), 0, None, None,
            _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens), B, int(max_seq_len), hq,
            hkv, d, nb, bs, float(scale), int(partition_size), _ptr(workspace), wsb,
            _ptr(error_flag), _stream_handle(stream)), "pa_decode_attention_strided")
    return out


def decode_attention_fp8(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                         value_cache: torch.Tensor, k_scale: torch.Tensor, v_scale: torch.Tensor,
                         block_tables: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                         scale: float, partition_size: int = 0,
                         workspace: Optional[torch.Tensor] = None,
                         error_flag: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode attention over uint8 E4M3 code pools [nb, bs, Hkv, D]; elements read
    as code * k_scale / code * v_scale (one-element float32 device tensors)."""
    _need(query.dim() == 3 and query.is_contiguous(), "query must be contiguous [B, Hq, D]")
    _need(out.shape == query.shape and out.is_contiguous(), "out must be contiguous [B, Hq, D]")
    _need(key_cache.dtype == value_cache.dtype == torch.uint8, "fp8 pools are uint8 codes")
    _need(key_cache.shape == value_cache.shape and key_cache.stride() == value_cache.stride(),
          "K and V pools share shape and strides")
    strides = _pool_strides(key_cache)
    _need(k_scale.dtype == torch.float32 and v_scale.dtype == torch.float32, "float32 scales")
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.stride(1) == 1, "block_tables int32 [B, W], rows contiguous")
    _need(seq_lens.dtype == torch.int32 and seq_lens.is_contiguous(), "seq_lens int32")
    B, hq, d = query.shape
    nb, bs, hkv, _ = key_cache.shape
    _need(key_cache.shape[3] == d, "query and pools must share head_dim")
    _dtype_code(out.dtype), _dtype_code(query.dtype)  # refused before any library call
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_bytes(B, hq, hkv, d, bs, max_seq_len,
                                                           partition_size), query.device)
    wsb = workspace.numel() * workspace.element_size()
    if strides is None:
        _check(lib.pa_decode_attention_fp8(
            _ptr(out), _dtype_code(out.dtype), _ptr(query), _dtype_code(query.dtype),
            _ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
            block_tables.stride(0), _ptr(seq_lens), B, int(max_seq_len), hq, hkv, d, nb, bs,
            float(scale), int(partition_size), _ptr(workspace), wsb, _ptr(error_flag),
            _stream_handle(stream)), "pa_decode_attention_fp8")
    else:
        _check(lib.pa_decode_attention_strided(
            _ptr(out), _dtype_code(out.dtype), _ptr(query), _dtype_code(query.dtype),
            _ptr(key_cache), _ptr(value_cache), ctypes.byref(strides), 1, _ptr(k_scale),
            _ptr(v_scale), _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens), B,
            int(max_seq_len), hq, hkv, d, nb, bs, float(scale), int(partition_size),
            _ptr(workspace), wsb, _ptr(error_flag), _stream_handle(stream)),
            "pa_decode_attention_strided")
    return out


def decode_attention_shared_prefix(out: torch.Tensor, query: torch.Tensor,
                                   key_cache: torch.Tensor, value_cache: torch.Tensor,
                                   block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                   shared_blocks: torch.Tensor, max_seq_len: int, scale: float,
                                   partition_size: int = 0,
                                   workspace: Optional[torch.Tensor] = None,
                                   error_flag: Optional[torch.Tensor] = None,
                                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """decode_attention for batches whose consecutive sequences share leading
    blocks (parallel samples of one prompt): shared_blocks int32 [B] on the
    device, shared_blocks[b] = leading table entries b holds in common with
    b + 1 (BlockManager.shared_blocks gives it).  Same result; a shared prefix
    is read once per pack of up to min(8, 32 // (Hq / Hkv)) sequences."""
    _need(query.dim() == 3 and query.is_contiguous(), "query must be contiguous [B, Hq, D]")
    _need(out.shape == query.shape and out.is_contiguous(), "out must be contiguous [B, Hq, D]")
    _need(key_cache.is_contiguous() and value_cache.is_contiguous(), "caches must be contiguous")
    _need(key_cache.shape == value_cache.shape, "K and V pools differ")
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.stride(1) == 1, "block_tables int32 [B, W], rows contiguous")
    _need(seq_lens.dtype == torch.int32 and seq_lens.is_contiguous(), "seq_lens int32")
    _need(shared_blocks.dtype == torch.int32 and shared_blocks.is_contiguous() and
          shared_blocks.numel() == query.shape[0], "shared_blocks int32 [B]")
    _need(query.dtype == key_cache.dtype == value_cache.dtype, "query and caches share a dtype")
    B, hq, d = query.shape
    nb, bs, hkv, _ = key_cache.shape
    _need(key_cache.shape[3] == d, "query and pools must share head_dim")
    _dtype_code(out.dtype), _dtype_code(query.dtype)  # refused before any library call
    if workspace is None:
        workspace = alloc_workspace(shared_prefix_workspace_bytes(
            B, hq, hkv, d, bs, max_seq_len, partition_size), query.device)
    _check(lib.pa_decode_attention_shared_prefix(
        _ptr(out), _dtype_code(out.dtype), _ptr(query), _ptr(key_cache), _ptr(value_cache),
        _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens), _ptr(shared_blocks), B,
        int(max_seq_len), hq, hkv, d, nb, bs, float(scale), _dtype_code(query.dtype),
        int(partition_size), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(error_flag), _stream_handle(stream)), "pa_decode_attention_shared_prefix")
    return out


def multi_query_workspace_bytes(num_seqs: int, num_query_rows: int, max_q_len: int,
                                num_q_heads: int, num_kv_heads: int, head_dim: int,
                                block_size: int, max_seq_len: int,
                                partition_size: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.pa_decode_multi_query_workspace_bytes(
        num_seqs, num_query_rows, max_q_len, num_q_heads, num_kv_heads, head_dim, block_size,
        max_seq_len, partition_size, ctypes.byref(out)), "pa_decode_multi_query_workspace_bytes")
    return int(out.value)


def decode_attention_multi_query(out: torch.Tensor, query: torch.Tensor, q_start: torch.Tensor,
                                 key_cache: torch.Tensor, value_cache: torch.Tensor,
                                 block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                 max_seq_len: int, max_q_len: int, scale: float,
                                 partition_size: int = 0,
                                 workspace: Optional[torch.Tensor] = None,
                                 error_flag: Optional[torch.Tensor] = None,
                                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Several new tokens per sequence: query/out [T, Hq, D]; q_start int32 [B + 1]
    on the device (sequence b owns rows q_start[b] .. q_start[b+1]-1, its last
    tokens, already in the cache); query i of a sequence's n attends positions
    0 .. seq_len - n + i.  max_q_len bounds n (host side)."""
    _need(query.dim() == 3 and query.is_contiguous(), "query must be contiguous [T, Hq, D]")
    _need(out.shape == query.shape and out.is_contiguous(), "out must be contiguous [T, Hq, D]")
    _need(key_cache.is_contiguous() and value_cache.is_contiguous(), "caches must be contiguous")
    _need(key_cache.shape == value_cache.shape, "K and V pools differ")
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.stride(1) == 1, "block_tables int32 [B, W], rows contiguous")
    _need(seq_lens.dtype == torch.int32 and seq_lens.is_contiguous(), "seq_lens int32")
    _need(q_start.dtype == torch.int32 and q_start.is_contiguous() and
          q_start.numel() == seq_lens.numel() + 1, "q_start int32 [B + 1]")
    _need(query.dtype == key_cache.dtype == value_cache.dtype, "query and caches share a dtype")
    T, hq, d = query.shape
    B = seq_lens.numel()
    nb, bs, hkv, _ = key_cache.shape
    _need(key_cache.shape[3] == d, "query and pools must share head_dim")
    _dtype_code(out.dtype), _dtype_code(query.dtype)  # refused before any library call
    if workspace is None:
        workspace = alloc_workspace(multi_query_workspace_bytes(
            B, T, int(max_q_len), hq, hkv, d, bs, int(max_seq_len), partition_size), query.device)
    _check(lib.pa_decode_attention_multi_query(
        _ptr(out), _dtype_code(out.dtype), _ptr(query), _ptr(q_start), T, int(max_q_len),
        _ptr(key_cache), _ptr(value_cache), _ptr(block_tables), block_tables.stride(0),
        _ptr(seq_lens), B, int(max_seq_len), hq, hkv, d, nb, bs, float(scale),
        _dtype_code(query.dtype), int(partition_size), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(error_flag), _stream_handle(stream)),
        "pa_decode_attention_multi_query")
    return out


_KV_CODE = {"auto": 0, "fp8": 1, "fp8_e4m3": 1}


def decode_plan_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                      block_size: int, max_seq_len: int, partition_size: int = 0,
                      kv_cache_dtype: str = "auto") -> int:
    out = ctypes.c_size_t(0)
    _check(lib.pa_decode_plan_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                    max_seq_len, partition_size, _KV_CODE[kv_cache_dtype],
                                    ctypes.byref(out)), "pa_decode_plan_bytes")
    return int(out.value)


def decode_plan(seq_lens: torch.Tensor, num_q_heads: int, num_kv_heads: int, head_dim: int,
                block_size: int, max_seq_len: int, partition_size: int = 0,
                kv_cache_dtype: str = "auto", plan: Optional[torch.Tensor] = None):
    """The split plan for HOST int32 lengths, computed on the host
    (pa_decode_plan).  Returns (plan, needs_combine): plan is a host uint8
    tensor (pinned when allocated here) to copy to 256-byte aligned device
    memory for decode_attention_planned."""
    _need(seq_lens.device.type == "cpu" and seq_lens.dtype == torch.int32 and
          seq_lens.is_contiguous(), "seq_lens: contiguous int32 on the host")
    B = seq_lens.numel()
    n = decode_plan_bytes(B, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                          partition_size, kv_cache_dtype)
    if plan is None:
        plan = torch.empty(n, dtype=torch.uint8).pin_memory()
    _need(plan.device.type == "cpu" and plan.numel() >= n and plan.is_contiguous(),
          "plan: a contiguous host buffer of decode_plan_bytes() bytes")
    comb = ctypes.c_int32(0)
    _check(lib.pa_decode_plan(_ptr(seq_lens), B, num_q_heads, num_kv_heads, head_dim, block_size,
                              max_seq_len, partition_size, _KV_CODE[kv_cache_dtype], _ptr(plan),
                              plan.numel(), ctypes.byref(comb)), "pa_decode_plan")
    return plan, bool(comb.value)


def decode_attention_planned(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                             value_cache: torch.Tensor, block_tables: torch.Tensor,
                             seq_lens: torch.Tensor, max_seq_len: int, scale: float,
                             plan: torch.Tensor, partition_size: int = 0,
                             workspace: Optional[torch.Tensor] = None,
                             k_scale: Optional[torch.Tensor] = None,
                             v_scale: Optional[torch.Tensor] = None,
                             error_flag: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """decode_attention (decode_attention_fp8 for uint8 code pools, with the
    scales) with the split plan read from the device copy `plan` of a
    decode_plan() result: no plan kernel.  Contiguous pools."""
    fp8 = key_cache.dtype == torch.uint8
    if fp8:
        _need(query.dim() == 3 and query.is_contiguous() and out.shape == query.shape and
              out.is_contiguous(), "query / out must be contiguous [B, Hq, D]")
        _need(value_cache.dtype == torch.uint8 and key_cache.shape == value_cache.shape and
              key_cache.is_contiguous() and value_cache.is_contiguous(),
              "fp8 pools: contiguous uint8 codes of one shape")
        _need(k_scale is not None and v_scale is not None and k_scale.dtype == torch.float32 and
              v_scale.dtype == torch.float32, "fp8 pools need float32 k_scale and v_scale")
        _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
              block_tables.stride(1) == 1, "block_tables int32 [B, W], rows contiguous")
        _need(seq_lens.dtype == torch.int32 and seq_lens.is_contiguous(), "seq_lens int32")
        _need(key_cache.shape[3] == query.shape[2], "query and pools must share head_dim")
        _dtype_code(out.dtype), _dtype_code(query.dtype)
    else:
        _decode_args(out, query, key_cache, value_cache, block_tables, seq_lens,
                     allow_strided_pools=False)
    _need(plan.is_cuda and plan.is_contiguous() and plan.data_ptr() % 256 == 0,
          "plan: the decode_plan() bytes in 256-byte aligned device memory")
    B, hq, d = query.shape
    nb, bs, hkv, _ = key_cache.shape
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_bytes(B, hq, hkv, d, bs, max_seq_len,
                                                           partition_size), query.device)
    _check(lib.pa_decode_attention_planned(
        _ptr(out), _dtype_code(out.dtype), _ptr(query), _dtype_code(query.dtype),
        _ptr(key_cache), _ptr(value_cache), 1 if fp8 else 0, _ptr(k_scale), _ptr(v_scale),
        _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens), B, int(max_seq_len), hq, hkv,
        d, nb, bs, float(scale), int(partition_size), _ptr(plan), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(error_flag), _stream_handle(stream)),
        "pa_decode_attention_planned")
    return out


def split_plan(seq_lens, max_seq_len: int, partition_size: int, num_ctas: int) -> dict:
    """pa_split_plan on host lengths (no GPU): the tile and segment prefix
    sums, each CTA's start and the first tile of each CTA's share, as numpy
    arrays."""
    import numpy as np
    lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    B = lens.size
    tiles = np.zeros(B + 1, np.int32)
    segs = np.zeros(B + 1, np.int32)
    start = np.zeros(num_ctas, np.int32)
    firstk = np.zeros(num_ctas, np.int32)
    ctalo = np.zeros(num_ctas + 1, np.int32)
    nseg, comb = ctypes.c_int32(0), ctypes.c_int32(0)
    vp = lambda a: ctypes.c_void_p(a.ctypes.data)
    _check(lib.pa_split_plan(vp(lens), B, int(max_seq_len), int(partition_size), int(num_ctas),
                             vp(tiles), vp(segs), vp(start), vp(firstk), vp(ctalo),
                             ctypes.byref(nseg), ctypes.byref(comb)), "pa_split_plan")
    return {"tiles": tiles, "seg_base": segs, "start_seq": start, "first_k": firstk,
            "cta_first_tile": ctalo, "num_segments": int(nseg.value),
            "needs_combine": bool(comb.value)}


class DecodeStep:
    """One decode step from pinned host memory through the C entry points
    pa_decode_step_upload / _run / _download (argument marshalling only: the
    library computes the split plan on the host, makes the one host-to-device
    copy, launches the kernels and makes the one device-to-host copy).

    ``host(slot)`` gives the pinned staging views to write the step's inputs
    into (``q``, ``new_k``, ``new_v``, ``slots``, ``tables``, ``lens``,
    ``cow``); ``submit(slot, num_cow)`` enqueues the step and returns at once;
    ``wait(slot)`` returns the slot's pinned output once it has arrived.
    Each slot has its own staging buffer, device scratch and output, so a
    serving loop can fill and submit step i + 1 while step i runs.  The
    uploads run on a copy-in stream and the downloads on a copy-out stream,
    so they overlap other steps' kernels; the kernels of every step run on
    one compute stream, in submission order, so a step attends the rows the
    steps before it wrote.  A slot may be refilled once its step has been
    waited for.  ``__call__`` runs one step with pa_decode_step (the three
    parts on one stream) and waits for it.
    """

    def __init__(self, key_cache: torch.Tensor, value_cache: torch.Tensor, num_seqs: int,
                 num_q_heads: int, table_width: int, max_seq_len: int, scale: float,
                 partition_size: int = 0, query_dtype: Optional[torch.dtype] = None,
                 out_dtype: Optional[torch.dtype] = None, k_scale: Optional[torch.Tensor] = None,
                 v_scale: Optional[torch.Tensor] = None, max_cow: int = 0, slots: int = 1):
        _need(slots >= 1, "at least one slot")
        _need(key_cache.shape == value_cache.shape and key_cache.is_contiguous() and
              value_cache.is_contiguous(), "contiguous K and V pools of one shape")
        self.fp8 = key_cache.dtype == torch.uint8
        _need(not self.fp8 or (query_dtype is not None and k_scale is not None and
                               v_scale is not None), "fp8 pools need query_dtype and scales")
        dt = query_dtype if query_dtype is not None else key_cache.dtype
        nb, bs, hkv, d = key_cache.shape
        self.k, self.v, self.k_scale, self.v_scale = key_cache, value_cache, k_scale, v_scale
        self.scale = float(scale)
        self.shape = StepShape(num_seqs, num_q_heads, hkv, d, nb, bs, table_width, max_seq_len,
                               partition_size, max_cow, _dtype_code(dt),
                               _dtype_code(out_dtype or dt), 1 if self.fp8 else 0)
        lay = StepLayout()
        _check(lib.pa_decode_step_layout(ctypes.byref(self.shape), ctypes.byref(lay)),
               "pa_decode_step_layout")
        self.layout = lay
        dev = key_cache.device
        fields = [("q", lay.query, (num_seqs, num_q_heads, d), dt),
                  ("new_k", lay.new_k, (num_seqs, hkv, d), dt),
                  ("new_v", lay.new_v, (num_seqs, hkv, d), dt),
                  ("slots", lay.slot_mapping, (num_seqs,), torch.int32),
                  ("tables", lay.block_tables, (num_seqs, table_width), torch.int32),
                  ("lens", lay.seq_lens, (num_seqs,), torch.int32),
                  ("cow", lay.cow_pairs, (max_cow, 2), torch.int32)]

        def views(buf):
            v = {}
            for name, off, shape, dtype in fields:
                n = int(torch.Size(shape).numel()) * torch.empty((), dtype=dtype).element_size()
                v[name] = buf[off:off + n].view(dtype).view(shape)
            return v

        self._staging = [torch.zeros(lay.host_bytes, dtype=torch.uint8).pin_memory()
                         for _ in range(slots)]
        self._views = [views(b) for b in self._staging]
        self._scratch = [torch.empty(lay.device_bytes, dtype=torch.uint8, device=dev)
                         for _ in range(slots)]
        out_shape = (num_seqs, num_q_heads, d)
        self._outs = [torch.empty(out_shape, dtype=out_dtype or dt).pin_memory()
                      for _ in range(slots)]
        self.stream = torch.cuda.Stream(device=dev)       # kernels, in submission order
        self._copy_in = torch.cuda.Stream(device=dev)
        self._copy_out = torch.cuda.Stream(device=dev)
        self._ev_in = [torch.cuda.Event() for _ in range(slots)]
        self._ev_run = [torch.cuda.Event() for _ in range(slots)]
        self._ev_out = [torch.cuda.Event() for _ in range(slots)]
        self._pending = [False] * slots

    def h2d_bytes(self) -> int:
        return int(self.layout.host_bytes)

    def d2h_bytes(self) -> int:
        return int(self.layout.out_bytes)

    def host(self, slot: int = 0) -> dict:
        return self._views[slot]

    def submit(self, slot: int = 0, num_cow: int = 0,
               error_flag: Optional[torch.Tensor] = None) -> None:
        _need(not self._pending[slot], "wait for the slot's previous step first")
        sh, st, sc = ctypes.byref(self.shape), self._staging[slot], self._scratch[slot]
        nbytes = sc.numel()
        # the slot's scratch is free once its previous kernels have finished
        self._copy_in.wait_event(self._ev_run[slot])
        _check(lib.pa_decode_step_upload(sh, _ptr(st), _ptr(sc), nbytes,
                                         _stream_handle(self._copy_in)), "pa_decode_step_upload")
        self._ev_in[slot].record(self._copy_in)
        self.stream.wait_event(self._ev_in[slot])
        _check(lib.pa_decode_step_run(sh, _ptr(st), int(num_cow), _ptr(self.k), _ptr(self.v),
                                      _ptr(self.k_scale), _ptr(self.v_scale), self.scale,
                                      _ptr(sc), nbytes, _ptr(error_flag),
                                      _stream_handle(self.stream)), "pa_decode_step_run")
        self._ev_run[slot].record(self.stream)
        self._copy_out.wait_event(self._ev_run[slot])
        _check(lib.pa_decode_step_download(sh, _ptr(sc), nbytes, _ptr(self._outs[slot]),
                                           _stream_handle(self._copy_out)),
               "pa_decode_step_download")
        self._ev_out[slot].record(self._copy_out)
        self._pending[slot] = True

    def wait(self, slot: int = 0) -> torch.Tensor:
        self._ev_out[slot].synchronize()
        self._pending[slot] = False
        return self._outs[slot]

    def __call__(self, num_cow: int = 0, error_flag: Optional[torch.Tensor] = None):
        """One step through pa_decode_step on the compute stream, waited for."""
        _need(not self._pending[0], "wait for slot 0's previous step first")
        sc = self._scratch[0]
        _check(lib.pa_decode_step(ctypes.byref(self.shape), _ptr(self._staging[0]),
                                  int(num_cow), _ptr(self.k), _ptr(self.v), _ptr(self.k_scale),
                                  _ptr(self.v_scale), self.scale, _ptr(sc), sc.numel(),
                                  _ptr(self._outs[0]), _ptr(error_flag),
                                  _stream_handle(self.stream)), "pa_decode_step")
        self.stream.synchronize()
        return self._outs[0]


# Bytes of the library's static scratch array used by decode_attention_noalloc.
NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_attention_noalloc(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                             value_cache: torch.Tensor, block_tables: torch.Tensor,
                             seq_lens: torch.Tensor, max_seq_len: int, scale: float,
                             partition_size: int = 0, error_flag: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """decode_attention for callers that must not allocate device memory: the
    scratch is the library's static per-device array (NOALLOC_SCRATCH_BYTES),
    so this wrapper allocates nothing either.  Arguments are checked as in
    decode_attention, except that the pools must be contiguous (there is no
    strided form of this entry point).  Shapes needing more scratch raise
    PagedAttnError PA_ERR_TOO_LARGE.  Calls overlapping on the GPU share the
    array and race; the first call on a device should precede stream capture."""
    _decode_args(out, query, key_cache, value_cache, block_tables, seq_lens,
                 allow_strided_pools=False)
    B, hq, d = query.shape
    nb, bs, hkv, _ = key_cache.shape
    _check(lib.pa_decode_attention_noalloc(
        _ptr(out), _dtype_code(out.dtype), _ptr(query), _ptr(key_cache), _ptr(value_cache),
        _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens), B, int(max_seq_len), hq, hkv,
        d, nb, bs, float(scale), _dtype_code(query.dtype), int(partition_size),
        _ptr(error_flag), _stream_handle(stream)), "pa_decode_attention_noalloc")
    return out


def set_consumer_wait_limit_ns(ns: int) -> None:
    """Diagnostic: the limit of the consuming warps' waits for the decode calls
    that follow (0 restores the 2 s default); see the header."""
    lib.pa_set_consumer_wait_limit_ns(int(ns))


def stream_read(buf: torch.Tensor, sink: torch.Tensor,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Read every byte of the contiguous device tensor `buf` once (a
    measurement of the read-bandwidth ceiling, not a step of the method);
    sink (int32 or uint32, one entry per CTA) gets each CTA's XOR of the
    32-bit words it read."""
    _need(buf.is_cuda and buf.is_contiguous(), "buf must be a contiguous device tensor")
    _need(sink.is_cuda and sink.is_contiguous() and sink.element_size() == 4,
          "sink must be a contiguous 32-bit device tensor")
    _check(lib.pa_stream_read(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink),
                              sink.numel(), _stream_handle(stream)), "pa_stream_read")
    return sink


class BlockManager:
    """Native host block manager (pa_bm_*): free list, refcounts, copy-on-write."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.block_size = int(block_size)
        self.num_blocks = int(num_blocks)
        h = ctypes.c_void_p()
        if free_order is not None:
            order = torch.as_tensor(free_order, dtype=torch.int32).contiguous()
            _check(lib.pa_bm_create(num_blocks, block_size, _ptr(order), ctypes.byref(h)),
                   "pa_bm_create")
        else:
            _check(lib.pa_bm_create(num_blocks, block_size, None, ctypes.byref(h)), "pa_bm_create")
        self._h = h
        # held here: at interpreter exit the module's globals may be gone first
        self._destroy = lib.pa_bm_destroy

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    def add_sequence(self, seq: int, num_tokens: int) -> None:
        _check(lib.pa_bm_add_sequence(self._h, seq, num_tokens), "pa_bm_add_sequence")

    def add_sequence_with_prefix(self, seq: int, token_ids: Sequence[int]) -> int:
        """A new request with its prompt's token ids: shares the leading full
        blocks the prefix cache holds for the same tokens and returns how many
        tokens those hold (their rows are already in the pool)."""
        n = len(token_ids)
        toks = (ctypes.c_int32 * max(n, 1))(*[int(t) for t in token_ids])
        cached = ctypes.c_int64()
        _check(lib.pa_bm_add_sequence_with_prefix(self._h, seq, toks, n, ctypes.byref(cached)),
               "pa_bm_add_sequence_with_prefix")
        return int(cached.value)

    def fork(self, parent: int, child: int) -> None:
        _check(lib.pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def append_slot(self, seq: int):
        slot = ctypes.c_int64()
        src, dst = ctypes.c_int32(), ctypes.c_int32()
        _check(lib.pa_bm_append_slot(self._h, seq, ctypes.byref(slot), ctypes.byref(src),
                                     ctypes.byref(dst)), "pa_bm_append_slot")
        return int(slot.value), (None if src.value < 0 else (int(src.value), int(dst.value)))

    def free_sequence(self, seq: int) -> None:
        _check(lib.pa_bm_free_sequence(self._h, seq), "pa_bm_free_sequence")

    def block_table(self, seq: int):
        n = ctypes.c_int32()
        toks = ctypes.c_int64()
        _check(lib.pa_bm_block_table(self._h, seq, None, 0, ctypes.byref(n), ctypes.byref(toks)),
               "pa_bm_block_table")
        buf = (ctypes.c_int32 * max(1, n.value))()
        _check(lib.pa_bm_block_table(self._h, seq, ctypes.cast(buf, ctypes.c_void_p), n.value,
                                     ctypes.byref(n), ctypes.byref(toks)), "pa_bm_block_table")
        return [int(buf[i]) for i in range(n.value)]

    def seq_len(self, seq: int) -> int:
        n = ctypes.c_int32()
        toks = ctypes.c_int64()
        _check(lib.pa_bm_block_table(self._h, seq, None, 0, ctypes.byref(n), ctypes.byref(toks)),
               "pa_bm_block_table")
        return int(toks.value)

    def refcount(self, block: int) -> int:
        return int(lib.pa_bm_refcount(self._h, block))

    def num_free(self) -> int:
        return int(lib.pa_bm_num_free(self._h))

    def shared_blocks(self, seqs: Sequence[int]) -> torch.Tensor:
        """int32 [len(seqs)] host tensor: leading blocks seqs[i] shares with seqs[i + 1]."""
        n = len(seqs)
        ids = (ctypes.c_int64 * max(n, 1))(*[int(s) for s in seqs])
        out = (ctypes.c_int32 * max(n, 1))()
        _check(lib.pa_bm_shared_blocks(self._h, ids, n, out), "pa_bm_shared_blocks")
        return torch.tensor(list(out)[:n], dtype=torch.int32)

    def order_by_prefix(self, seqs: Sequence[int]) -> list:
        """The batch reordered so that sequences holding the same leading
        blocks are neighbours (for decode_attention_shared_prefix): a list of
        indices into seqs."""
        n = len(seqs)
        ids = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in seqs])
        out = (ctypes.c_int32 * max(n, 1))()
        _check(lib.pa_bm_order_by_prefix(self._h, ids, n, out), "pa_bm_order_by_prefix")
        return [int(out[i]) for i in range(n)]

    def tables(self, seqs: Sequence[int], width: int) -> torch.Tensor:
        """int32 [len(seqs), width] host tensor of block tables, padded with -1."""
        return self.fill_tables(seqs, width)[0]

    def fill_tables(self, seqs: Sequence[int], width: int):
        """(tables int32 [n, width] padded with -1, seq_lens int32 [n]): the
        decode kernels' metadata for the batch, as host tensors."""
        n = len(seqs)
        ids = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in seqs])
        tables = torch.empty((n, width), dtype=torch.int32)
        lens = torch.empty((n,), dtype=torch.int32)
        _check(lib.pa_bm_fill_tables(self._h, ids, n, tables.data_ptr() if tables.numel() else None,
                                     width, lens.data_ptr() if n else None),
               "pa_bm_fill_tables")
        return tables, lens

    def append_slots(self, seqs: Sequence[int]):
        """One new token for each of seqs, in order, all or nothing: (slot_mapping
        int32 [n], copy-on-write pairs int32 [k, 2]) as host tensors."""
        n = len(seqs)
        ids = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in seqs])
        slots = (ctypes.c_int32 * max(n, 1))()
        pairs = (ctypes.c_int32 * max(2 * n, 2))()
        ncow = ctypes.c_int32()
        _check(lib.pa_bm_append_slots(self._h, ids, n, slots, pairs, ctypes.byref(ncow)),
               "pa_bm_append_slots")
        k = ncow.value
        return (torch.tensor(list(slots)[:n], dtype=torch.int32),
                torch.tensor(list(pairs)[:2 * k], dtype=torch.int32).reshape(k, 2))

    def append_tokens(self, seqs: Sequence[int], counts: Sequence[int]):
        """counts[i] new tokens for each seqs[i], in order, all or nothing:
        (slot_mapping int32 [sum(counts)], q_start int32 [n + 1],
        copy-on-write pairs int32 [k, 2]) as host tensors -- the inputs of
        reshape_and_cache and decode_attention_multi_query."""
        n = len(seqs)
        _need(len(counts) == n, "one count per sequence")
        ids = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in seqs])
        cnt = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in counts])
        total = sum(int(x) for x in counts)
        slots = (ctypes.c_int32 * max(total, 1))()
        qs = (ctypes.c_int32 * (n + 1))()
        pairs = (ctypes.c_int32 * max(2 * n, 2))()
        ncow = ctypes.c_int32()
        _check(lib.pa_bm_append_tokens(self._h, ids, n, cnt, slots, qs, pairs, ctypes.byref(ncow)),
               "pa_bm_append_tokens")
        k = ncow.value
        return (torch.tensor(list(slots)[:total], dtype=torch.int32),
                torch.tensor(list(qs)[:n + 1] if n else [0], dtype=torch.int32),
                torch.tensor(list(pairs)[:2 * k], dtype=torch.int32).reshape(k, 2))

    def blocks_needed(self, seqs: Sequence[int], counts: Optional[Sequence[int]] = None) -> int:
        """Free blocks append_tokens(seqs, counts) (or append_slots(seqs) when
        counts is None) would take, with no change to any table."""
        n = len(seqs)
        ids = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in seqs])
        cnt = None
        if counts is not None:
            _need(len(counts) == n, "one count per sequence")
            cnt = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in counts])
        need = ctypes.c_int64()
        _check(lib.pa_bm_blocks_needed(self._h, ids, n, cnt, ctypes.byref(need)),
               "pa_bm_blocks_needed")
        return int(need.value)

    def stats(self) -> dict:
        """Memory the sequences hold (pa_bm_stats), plus occupancy = stored
        slots / held slots and the saving of sharing = 1 - held / logical."""
        st = BmStats()
        _check(lib.pa_bm_stats(self._h, ctypes.byref(st)), "pa_bm_stats")
        d = {name: int(getattr(st, name)) for name, _ in BmStats._fields_}
        held_slots = d["held_blocks"] * self.block_size
        d["occupancy"] = d["stored_slots"] / held_slots if held_slots else 1.0
        d["sharing_saving"] = (1.0 - d["held_blocks"] / d["logical_blocks"]
                               if d["logical_blocks"] else 0.0)
        return d
