"""Test-side assembly of workloads: oracle-built metadata, NaN-poisoned pools,
device copies.  Block tables and slots here come from the oracle's reference
block manager (oracle/blockmgr.py), never from the product."""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
import pa_workloads as W
from oracle.blockmgr import RefBlockManager

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class Prepared:
    case: W.Case
    tables: np.ndarray                 # int32 [B, width], -1 padded
    seq_lens: np.ndarray               # int32 [B], tokens attended by the decode step
    k_pool: np.ndarray                 # uint16, possibly poisoned
    v_pool: np.ndarray
    new_slots: np.ndarray = None       # int32 [T_new] slots of the new rows (or None)
    cow_pairs: np.ndarray = None       # int32 [N, 2] copy-on-write pairs (or None)
    lens_before: np.ndarray = None     # lengths before the appends
    extra: dict = field(default_factory=dict)


def used_slot_mask(tables: np.ndarray, seq_lens: np.ndarray, num_blocks: int, bs: int) -> np.ndarray:
    """bool [num_blocks, bs]: slot holds a token of some sequence (oracle slot arithmetic)."""
    mask = np.zeros(num_blocks * bs, dtype=bool)
    B = tables.shape[0]
    seq_idx = np.repeat(np.arange(B, dtype=np.int32), seq_lens)
    pos = np.concatenate([np.arange(L, dtype=np.int32) for L in seq_lens]) if B else np.zeros(0, np.int32)
    if seq_idx.size:
        slots = oracle.slot_mapping(tables, seq_idx, pos, bs)
        mask[slots] = True
    return mask.reshape(num_blocks, bs)


def poison_unused(pool: np.ndarray, used: np.ndarray, dtype: str) -> np.ndarray:
    p = pool.copy()
    p[~used] = W.NAN_BITS[dtype]
    return p


def prepare(spec: W.Spec, poison: bool = True, width_extra: int = 1) -> Prepared:
    """Draw the workload and build its metadata with the reference block manager.

    Plain workloads: sequences 0..B-1 take their blocks from the free list in
    order; if the spec has new rows, each sequence then appends one token at
    position seq_len (the next slot) -- the decode step attends to the old
    lengths, a second step to lengths + 1.
    shared_prefix: each prompt is a sequence forked into `samples` samples;
    samples then append their extra tokens in order (copy-on-write on the
    first append into the shared partial block)."""
    case = W.draw(spec)
    bs = spec.block_size
    bm = RefBlockManager(case.num_blocks, bs, case.free_order)
    B = spec.num_seqs
    new_slots = None
    cow = None
    lens_before = None
    if spec.len_dist == "shared_prefix":
        sid = 0
        for pr in range(spec.prompts):
            bm.add_sequence(sid, spec.prompt_len)
            for s in range(1, spec.samples):
                bm.fork(sid, sid + s)
            sid += spec.samples
        slots = []
        for b in range(B):
            for _ in range(int(case.extra_tokens[b])):
                slot, _c = bm.append_slot(b)
                slots.append(slot)
        new_slots = np.array(slots, dtype=np.int32)
        cow = np.array(bm.copies, dtype=np.int32).reshape(-1, 2)
        seq_lens = case.seq_lens.copy()
        lens_before = np.full(B, spec.prompt_len, np.int32)
    else:
        for b in range(B):
            bm.add_sequence(b, int(case.seq_lens[b]))
        seq_lens = case.seq_lens.copy()
        lens_before = seq_lens.copy()
        if spec.new_rows:
            assert spec.new_rows == B
            new_slots = np.array([bm.append_slot(b)[0] for b in range(B)], dtype=np.int32)
    bm.check_invariants()
    width = max(len(bm.block_table(b)) for b in range(B)) + width_extra
    tables = np.full((B, width), -1, dtype=np.int32)
    for b in range(B):
        t = bm.block_table(b)
        tables[b, :len(t)] = t
    k_pool, v_pool = case.k_pool, case.v_pool
    prep = Prepared(case, tables, seq_lens.astype(np.int32), k_pool, v_pool, new_slots, cow,
                    lens_before)
    if poison:
        # Every slot that holds no token of any sequence (after all appends) is NaN.
        final_lens = seq_lens + (1 if (spec.new_rows and spec.len_dist != "shared_prefix") else 0)
        used = used_slot_mask(tables, final_lens.astype(np.int32), case.num_blocks, bs)
        prep.k_pool = poison_unused(k_pool, used, spec.dtype)
        prep.v_pool = poison_unused(v_pool, used, spec.dtype)
        prep.extra["used"] = used
    prep.extra["bm"] = bm
    return prep


def to_dev(a: np.ndarray, dtype: str = None, device="cuda") -> torch.Tensor:
    """uint16 bit arrays become fp16/bf16 tensors; int arrays keep their type."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(torch.int16).view(TORCH_DTYPE[dtype])
    return t.to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


TOL_F32 = 1e-4


def half_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    """Half a unit in the last place of the 16-bit storage type at |ref|: the
    rounding that storing an exact result in that type may add."""
    mant, emin = (7, -126) if dtype == "bf16" else (10, -14)
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** emin)))
    return 0.5 * np.exp2(e - mant)


def stored_within(out, ref, dtype, tol_f32: float = TOL_F32) -> bool:
    """Stored outputs: the fp32-path error plus the storage rounding."""
    o = as_f64(out)
    assert np.all(np.isfinite(o))
    return bool(np.all(np.abs(o - ref) <= tol_f32 + half_ulp(ref, dtype)))


def shared_blocks_of(tables: np.ndarray, seq_lens: np.ndarray, bs: int) -> np.ndarray:
    """int32 [B]: leading block-table entries row b holds in common with row
    b + 1 among the blocks each sequence uses (last entry 0)."""
    B = tables.shape[0]
    out = np.zeros(B, dtype=np.int32)
    for b in range(B - 1):
        n = min(-(-int(seq_lens[b]) // bs), -(-int(seq_lens[b + 1]) // bs))
        eq = tables[b, :n] == tables[b + 1, :n]
        out[b] = n if eq.all() else int(np.argmin(eq))
    return out


def pools_after_appends(prep: "Prepared"):
    """The pools the decode step reads: after the copy-on-write copies and the
    appended rows (oracle routines), else the prepared pools."""
    k, v = prep.k_pool, prep.v_pool
    if prep.cow_pairs is not None:
        k, v = k.copy(), v.copy()
        oracle.copy_blocks([k, v], prep.cow_pairs, int(np.prod(k.shape[1:])) * 2)
        oracle.reshape_and_cache(prep.case.new_k, prep.case.new_v, k, v, prep.new_slots)
    return k, v


def fp8_case(seed, B=6, lo=200, hi=1300, q_dtype="bf16", bs=16, hq=32, hkv=8, ks=0.05, vs=0.04):
    spec = W.Spec("fp8", B, hq, hkv, 128, bs, q_dtype, seed=seed, len_dist="uniform",
                  len_lo=lo, len_hi=hi)
    prep = prepare(spec, poison=False)
    g = torch.Generator().manual_seed(seed + 1)
    nb = prep.case.num_blocks
    # codes of N(0,1) / scale, so elements read back about N(0,1)
    kc = W.randn_e4m3_codes((nb, bs, hkv, 128), g, 1.0 / ks)
    vc = W.randn_e4m3_codes((nb, bs, hkv, 128), g, 1.0 / vs)
    used = used_slot_mask(prep.tables, prep.seq_lens, nb, bs)
    kc[~used] = 0x7F
    vc[~used] = 0x7F
    return spec, prep, kc, vc
