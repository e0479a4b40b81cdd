"""Seeded synthetic inputs for the paged decode hot path.

This module only draws random numbers and names workload shapes: sequence
lengths, the order in which physical block ids leave the free list, Q/K/V
values and new K/V rows.  It holds none of the method's arithmetic (no slot,
table, softmax or copy logic), so both the oracle and the CUDA path may use
it.  Values are N(0, 1) drawn in float32 with a CPU ``torch.Generator`` and
rounded to the storage type (round to nearest even); arrays are returned as
uint16 bit patterns (numpy) so either side can consume them byte for byte.

Draw order for every workload: sequence lengths -> free-list permutation ->
Q -> K pool -> V pool -> new K/V rows.

The named workloads follow the pages' serving scenarios ("PagedAttention":
block size 4 worked example, 16-token default blocks, long-tailed lengths,
parallel sampling with a shared prompt):

  tiny          4 seqs, lengths {1,5,16,22}, bs 4, 32-block pool, Hq 4 / Hkv 2,
                D 64, fp16, plus 4 new rows at the next slots
  llama8b       64 seqs, lengths U[512, 4096], bs 16, Hq 32 / Hkv 8, D 128, bf16
  longtail      256 seqs, lengths round(exp(ln 300 + z)) clipped to [1, 8192],
                bs 16, Hq 32 / Hkv 8, D 128, fp16, plus 256 new rows
  longctx       8 seqs of 32768, bs 32, Hq 64 / Hkv 8, D 128, bf16,
                512-token partitions
  shared_prefix 32 prompts of 2047 tokens x 8 samples, each sample then
                appending U[1, 200] tokens, bs 16, Hq 32 / Hkv 8, D 128, bf16
  llama8b_fp8   the llama8b shape over an fp8 (E4M3) cache, scales 1/32
  llama8b_mq4   the llama8b shape with 4 new tokens per sequence attending
                together (causal), as when speculated tokens are verified
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch

_TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


@dataclass(frozen=True)
class Spec:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                       # 'f16' or 'bf16'
    seed: int
    len_dist: str = "uniform"        # 'fixed' | 'uniform' | 'lognormal' | 'shared_prefix'
    fixed_lens: Tuple[int, ...] = ()
    len_lo: int = 1
    len_hi: int = 1
    lognormal_median: float = 300.0
    lognormal_sigma: float = 1.0
    pool_blocks: Optional[int] = None  # fixed pool size; else ceil(pool_factor * need)
    pool_factor: float = 1.2
    new_rows: int = 0                # new K/V rows written by reshape_and_cache
    partition_size: int = 0          # 0: automatic split
    prompts: int = 0                 # shared_prefix only
    samples: int = 0
    prompt_len: int = 0
    extra_lo: int = 1
    extra_hi: int = 1
    kv_dtype: str = "auto"           # 'auto' (16-bit pools) or 'fp8_e4m3' (code pools)
    k_scale: float = 1.0             # fp8 pools: element = code * scale
    v_scale: float = 1.0
    q_len: int = 1                   # new tokens per sequence attending at once

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def fp8(self) -> bool:
        return self.kv_dtype == "fp8_e4m3"

    @property
    def elem_bytes(self) -> int:
        return 1 if self.fp8 else 2

    def replace(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Spec("tiny", 4, 4, 2, 64, 4, "f16", seed=1000, len_dist="fixed",
                 fixed_lens=(1, 5, 16, 22), pool_blocks=32, new_rows=4),
    "llama8b": Spec("llama8b", 64, 32, 8, 128, 16, "bf16", seed=1001,
                    len_dist="uniform", len_lo=512, len_hi=4096),
    "longtail": Spec("longtail", 256, 32, 8, 128, 16, "f16", seed=1002,
                     len_dist="lognormal", len_lo=1, len_hi=8192, new_rows=256),
    "longctx": Spec("longctx", 8, 64, 8, 128, 32, "bf16", seed=1003,
                    len_dist="fixed", fixed_lens=(32768,) * 8, partition_size=512),
    "shared_prefix": Spec("shared_prefix", 256, 32, 8, 128, 16, "bf16", seed=1004,
                          len_dist="shared_prefix", prompts=32, samples=8,
                          prompt_len=2047, extra_lo=1, extra_hi=200),
    # the llama8b shape over an fp8 (E4M3) cache: elements read code * 1/32
    "llama8b_fp8": Spec("llama8b_fp8", 64, 32, 8, 128, 16, "bf16", seed=1005,
                        len_dist="uniform", len_lo=512, len_hi=4096,
                        kv_dtype="fp8_e4m3", k_scale=1.0 / 32, v_scale=1.0 / 32),
    # the llama8b shape, 4 new tokens per sequence
    "llama8b_mq4": Spec("llama8b_mq4", 64, 32, 8, 128, 16, "bf16", seed=1006,
                        len_dist="uniform", len_lo=512, len_hi=4096, q_len=4),
}


@dataclass
class Case:
    spec: Spec
    seq_lens: np.ndarray          # int32 [B]; for shared_prefix: prompt + extra
    extra_tokens: np.ndarray      # int32 [B]; shared_prefix only (else zeros)
    num_blocks: int
    free_order: np.ndarray        # int32 [num_blocks], a permutation
    q: np.ndarray                 # uint16 [B, Hq, D]
    k_pool: np.ndarray            # uint16 [num_blocks, bs, Hkv, D] (uint8 codes if fp8)
    v_pool: np.ndarray
    new_k: np.ndarray             # uint16 [new_rows, Hkv, D]
    new_v: np.ndarray
    meta: dict = field(default_factory=dict)


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _draw_lengths(spec: Spec, g: torch.Generator):
    B = spec.num_seqs
    extra = np.zeros(B, dtype=np.int32)
    if spec.len_dist == "fixed":
        lens = np.asarray(spec.fixed_lens, dtype=np.int32)
        assert lens.shape[0] == B
    elif spec.len_dist == "uniform":
        lens = torch.randint(spec.len_lo, spec.len_hi + 1, (B,), generator=g).numpy().astype(np.int32)
    elif spec.len_dist == "lognormal":
        z = torch.randn(B, generator=g, dtype=torch.float64).numpy()
        raw = np.rint(np.exp(math.log(spec.lognormal_median) + spec.lognormal_sigma * z))
        lens = np.clip(raw, spec.len_lo, spec.len_hi).astype(np.int32)
    elif spec.len_dist == "shared_prefix":
        assert spec.prompts * spec.samples == B
        extra = torch.randint(spec.extra_lo, spec.extra_hi + 1, (B,), generator=g).numpy().astype(np.int32)
        lens = (spec.prompt_len + extra).astype(np.int32)
    else:
        raise ValueError(spec.len_dist)
    return lens, extra


def pool_blocks_needed(spec: Spec, seq_lens: np.ndarray, extra: np.ndarray) -> int:
    """Upper bound on the blocks a workload occupies (pool sizing only)."""
    bs = spec.block_size
    if spec.len_dist == "shared_prefix":
        return (spec.prompts * _ceil_div(spec.prompt_len, bs)
                + int(sum(_ceil_div(int(e), bs) + 1 for e in extra)))
    grow = 1 if spec.new_rows else 0
    return int(sum(_ceil_div(int(L) + grow, bs) for L in seq_lens))


def randn_bits(shape, dtype: str, g: torch.Generator, chunk: int = 1 << 26) -> np.ndarray:
    """N(0,1) float32 draws rounded to `dtype`, as uint16 bits, drawn in chunks."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    td = _TORCH_DTYPE[dtype]
    for lo in range(0, n, chunk):
        m = min(chunk, n - lo)
        x = torch.randn(m, generator=g, dtype=torch.float32).to(td)
        out[lo:lo + m] = x.view(torch.int16).numpy().view(np.uint16)
    return out.reshape(shape)


def randn_e4m3_codes(shape, g: torch.Generator, magnitude: float = 1.0,
                     chunk: int = 1 << 26) -> np.ndarray:
    """N(0, magnitude^2) float32 draws rounded to E4M3 codes (uint8) by torch's
    float8_e4m3fn conversion, drawn in chunks: random contents for fp8 pools."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)
    for lo in range(0, n, chunk):
        m = min(chunk, n - lo)
        x = torch.randn(m, generator=g, dtype=torch.float32) * magnitude
        out[lo:lo + m] = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return out.reshape(shape)


def draw(spec: Spec) -> Case:
    g = torch.Generator().manual_seed(spec.seed)
    lens, extra = _draw_lengths(spec, g)
    if spec.pool_blocks is not None:
        nb = int(spec.pool_blocks)
    else:
        nb = int(math.ceil(spec.pool_factor * pool_blocks_needed(spec, lens, extra)))
    free_order = torch.randperm(nb, generator=g).numpy().astype(np.int32)
    B, Hq, Hkv, D, bs = (spec.num_seqs, spec.num_q_heads, spec.num_kv_heads,
                         spec.head_dim, spec.block_size)
    q = randn_bits((B, Hq, D), spec.dtype, g)
    if spec.fp8:  # code pools whose elements read back about N(0, 1)
        k_pool = randn_e4m3_codes((nb, bs, Hkv, D), g, 1.0 / spec.k_scale)
        v_pool = randn_e4m3_codes((nb, bs, Hkv, D), g, 1.0 / spec.v_scale)
    else:
        k_pool = randn_bits((nb, bs, Hkv, D), spec.dtype, g)
        v_pool = randn_bits((nb, bs, Hkv, D), spec.dtype, g)
    if spec.len_dist == "shared_prefix":
        n_new = int(extra.sum())
    else:
        n_new = spec.new_rows
    new_k = randn_bits((n_new, Hkv, D), spec.dtype, g)
    new_v = randn_bits((n_new, Hkv, D), spec.dtype, g)
    return Case(spec, lens, extra, nb, free_order, q, k_pool, v_pool, new_k, new_v)


def scale_of(spec: Spec) -> float:
    return 1.0 / math.sqrt(spec.head_dim)
