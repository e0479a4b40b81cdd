"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one decode step of the workload over its whole batch:
copy_blocks (only where the workload has copy-on-write pairs) ->
reshape_and_cache of the step's new K/V rows -> decode_attention (plan, main,
combine).  Inputs are resident in HBM when the timed region starts; block
tables and slots come from the native host block manager.

Prints ONE JSON line (rank 0).  `value` is KV-read GB/s: the algorithmic KV
bytes of a step (sum of seq_len * 2 * Hkv * D * 2 bytes, valid tokens only)
times the steps and ranks, divided by the device time (CUDA events, max over
ranks).  `--impl reference` times the fp64 CPU oracle instead, on bounded
samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import pa_workloads as W  # noqa: E402

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); decode tokens/s"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_main_llama8b.md")
KERNEL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_343_b200", "csrc", f)
                  for f in ("pa_decode.cu", "pa_decode_common.cuh", "pa_device.cuh")]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic():
    """DRAM bytes per launch of the main kernel from the committed ncu summary,
    or None if there is none or the kernel changed since it was taken."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    txt = open(PROFILE_SUMMARY).read()
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", txt)
    m_bytes = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        def parse(r):
            parts = [x.strip() for x in r.split(",")]
            try:
                return {"sm": float(parts[1]), "max": float(parts[2]), "active": parts[4],
                        "hw": parts[5], "hwt": parts[6], "swt": parts[7], "pcap": parts[8]}
            except (ValueError, IndexError):
                return None
        inside = [parse(r) for (t, r) in self.rows if t0 <= t <= t1]
        inside = [x for x in inside if x]
        window = "timed region"
        if not inside:  # region shorter than the sampling period: nearest samples
            near = sorted(self.rows, key=lambda tr: min(abs(tr[0] - t0), abs(tr[0] - t1)))[:3]
            inside = [x for x in (parse(r) for _, r in near) if x]
            window = "nearest samples (timed region shorter than the 50 ms period)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        reasons = set()
        for x in inside:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if x[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x["sm"] for x in inside),
                "sm_max_mhz": max(x["max"] for x in inside), "reasons": sorted(reasons),
                "samples": len(inside), "window": window}


# --------------------------------------------------------------------------- workload
def kv_bytes(spec, lens) -> int:
    return int(np.sum(lens.astype(np.int64))) * 2 * spec.num_kv_heads * spec.head_dim * spec.elem_bytes


def build_workload(spec, pa):
    """Seeded inputs and metadata from the native block manager.

    Plain workloads: every sequence holds seq_len - 1 tokens and the step
    appends its current token (position seq_len - 1), which the attention then
    reads.  shared_prefix: prompts forked into samples, each sample appending
    its extra tokens (copy-on-write on the first append)."""
    case = W.draw(spec)
    bs = spec.block_size
    bm = pa.BlockManager(case.num_blocks, bs, case.free_order)
    B = spec.num_seqs
    lens = case.seq_lens.astype(np.int32)
    cow = []
    if spec.len_dist == "shared_prefix":
        sid = 0
        for _ in range(spec.prompts):
            bm.add_sequence(sid, spec.prompt_len)
            for s in range(1, spec.samples):
                bm.fork(sid, sid + s)
            sid += spec.samples
        slots = []
        for b in range(B):
            for _ in range(int(case.extra_tokens[b])):
                slot, c = bm.append_slot(b)
                slots.append(slot)
                if c is not None:
                    cow.append(c)
        new_k, new_v = case.new_k, case.new_v
    else:
        slots, new_k, new_v = _append_new_tokens(spec, bm, lens)
    width = max(len(bm.block_table(b)) for b in range(B))
    tables = bm.tables(list(range(B)), width).numpy()
    wl = dict(case=case, lens=lens, tables=tables, slots=np.array(slots, np.int32),
              cow=np.array(cow, np.int32).reshape(-1, 2), new_k=new_k, new_v=new_v,
              shared_blocks=bm.shared_blocks(list(range(B))).numpy(), bm_stats=bm.stats())
    _add_queries(spec, wl)
    return wl


def _append_new_tokens(spec, bm, lens):
    """Every sequence holds seq_len - q_len tokens and the step appends its
    q_len current tokens (positions seq_len - q_len .. seq_len - 1), which the
    attention then reads.  Returns (slots, new K rows, new V rows)."""
    B, q = spec.num_seqs, spec.q_len
    slots = []
    for b in range(B):
        bm.add_sequence(b, int(lens[b]) - q)
        for _ in range(q):
            slots.append(bm.append_slot(b)[0])
    g = torch.Generator().manual_seed(spec.seed + 7)
    new_k = W.randn_bits((B * q, spec.num_kv_heads, spec.head_dim), spec.dtype, g)
    new_v = W.randn_bits((B * q, spec.num_kv_heads, spec.head_dim), spec.dtype, g)
    return slots, new_k, new_v


def _add_queries(spec, wl):
    """Query rows: the workload's [B, Hq, D] draw, or with q_len > 1 the
    [B * q_len, Hq, D] rows of every sequence's new tokens (sequence b owns rows
    b q_len .. b q_len + q_len - 1)."""
    B, q = spec.num_seqs, spec.q_len
    if q == 1:
        wl["q"] = wl["case"].q
        wl["q_start"] = None
        return
    g = torch.Generator().manual_seed(spec.seed + 11)
    wl["q"] = W.randn_bits((B * q, spec.num_q_heads, spec.head_dim), spec.dtype, g)
    wl["q_start"] = (np.arange(B + 1) * q).astype(np.int32)


def kv_memory(spec, wl) -> dict:
    """KV-cache memory held by the step's sequences ("PagedAttention": waste is
    under one block per sequence; shared prompt blocks are held once)."""
    bs = spec.block_size
    lens = wl["lens"].astype(np.int64)
    per_seq_blocks = -(-lens // bs)
    logical_blocks = int(per_seq_blocks.sum())
    held = set()
    for b in range(spec.num_seqs):
        held.update(int(x) for x in wl["tables"][b, :per_seq_blocks[b]])
    tokens = int(lens.sum())
    waste = per_seq_blocks * bs - lens
    return {"block_size": bs, "tokens": tokens, "blocks_held": len(held),
            "blocks_if_unshared": logical_blocks,
            "occupancy": round(tokens / (logical_blocks * bs), 4),
            "mean_waste_tokens_per_seq": round(float(waste.mean()), 2),
            "max_waste_tokens_per_seq": int(waste.max()),
            "sharing_saving": round(1.0 - len(held) / logical_blocks, 4)}


def unique_kv_bytes(spec, wl) -> int:
    """KV bytes of distinct (block, offset) slots read by the step."""
    bs = spec.block_size
    seen = set()
    for b in range(spec.num_seqs):
        L = int(wl["lens"][b])
        for i in range(-(-L // bs)):
            blk = int(wl["tables"][b, i])
            n = min(bs, L - i * bs)
            seen.add((blk, n))
    slots = {}
    for blk, n in seen:
        slots[blk] = max(slots.get(blk, 0), n)
    return sum(slots.values()) * 2 * spec.num_kv_heads * spec.head_dim * spec.elem_bytes


def packed_kv_bytes(spec, wl) -> int:
    """KV bytes the shared-prefix decode reads: aligned windows of
    P = min(8, 32 // group) neighbouring sequences (else the aligned pairs
    inside a window, or inside the shorter last window) read their common prefix -- whole 16-token tiles of blocks
    full in every member, at least 64 tokens -- once, and every sequence its
    remaining tokens."""
    G = spec.num_q_heads // spec.num_kv_heads
    P = min(8, 32 // G)
    bs = spec.block_size
    lens = wl["lens"].astype(np.int64)
    sb = wl["shared_blocks"].astype(np.int64)

    def common(b0, n):
        c = min(int(lens[b0 + m]) // bs for m in range(n))
        c = min([c] + [max(0, int(sb[b0 + m])) for m in range(n - 1)])
        t = c * bs // 16
        return t if t >= 4 else 0

    tokens = int(lens.sum())
    if P >= 2:
        for w in range(-(-spec.num_seqs // P)):
            n = min(P, spec.num_seqs - w * P)
            whole = common(w * P, P) if n == P else 0
            if whole:
                tokens -= (P - 1) * whole * 16
            elif P > 2:
                for j in range(n // 2):
                    tokens -= common(w * P + 2 * j, 2) * 16
    return tokens * 2 * spec.num_kv_heads * spec.head_dim * spec.elem_bytes


# --------------------------------------------------------------------------- our arm
def read_ceiling(device, stream):
    """The read-bandwidth ceiling measured in the same run: the library's read
    stream over 1 GiB (eight times the L2), the best of 2, 4 and 8 CTAs per SM,
    ten passes each between two events after three untimed ones."""
    import paged_kv_cache_343_b200 as pa
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    buf = torch.ones(1 << 28, dtype=torch.int32, device=device)
    nbytes = buf.numel() * buf.element_size()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best, best_per_sm, sweep = 0.0, 0, {}
    for per_sm in (2, 4, 8):
        sink = torch.empty(sms * per_sm, dtype=torch.int32, device=device)
        for _ in range(3):
            pa.stream_read(buf, sink, stream)
        e0.record(stream)
        for _ in range(10):
            pa.stream_read(buf, sink, stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
        gbs = 10 * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9
        sweep["%d_per_sm" % per_sm] = round(gbs, 1)
        if gbs > best:
            best, best_per_sm = gbs, per_sm
    del buf
    return {"gbs": round(best, 1), "bytes": nbytes, "sweep": sweep,
            "how": "pa_stream_read: 16-byte loads, %d CTAs of 512 threads per SM, 1 GiB read "
                   "10 times" % best_per_sm}


def latency_distribution(attention, read_bytes, device, stream, runs=100):
    """One attention call per run, the L2 flushed before each (a write of twice
    its size), timed alone between two events: median, p10 and p90."""
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(1, 2 * l2 // 4), dtype=torch.int32, device=device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(runs)]
    with torch.cuda.stream(stream):
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            attention()
            b.record(stream)
    torch.cuda.synchronize(device)
    us = np.array(sorted(a.elapsed_time(b) * 1e3 for a, b in ev))
    p10, med, p90 = (float(np.percentile(us, q)) for q in (10, 50, 90))
    return {"runs": runs, "l2": "flushed before each run (%d MB written)" % (2 * l2 // 2**20),
            "median_us": round(med, 2), "p10_us": round(p10, 2), "p90_us": round(p90, 2),
            "gbs_at_median": round(read_bytes / (med / 1e6) / 1e9, 2)}


def run_ours(args, rank, world, local_rank):
    import paged_kv_cache_343_b200 as pa

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    spec = rank_spec(W.WORKLOADS[args.workload], rank, world)
    if args.block_size:
        spec = spec.replace(block_size=args.block_size)
    wl = build_workload(spec, pa)
    case = wl["case"]
    td = {"f16": torch.float16, "bf16": torch.bfloat16}[spec.dtype]

    def dev_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(td).to(device)

    if spec.fp8:  # uint8 code pools and one-element scales
        k_cache = torch.from_numpy(case.k_pool).to(device)
        v_cache = torch.from_numpy(case.v_pool).to(device)
        k_scale = torch.tensor([spec.k_scale], dtype=torch.float32, device=device)
        v_scale = torch.tensor([spec.v_scale], dtype=torch.float32, device=device)
    else:
        k_cache, v_cache = dev_bits(case.k_pool), dev_bits(case.v_pool)
        k_scale = v_scale = None
    q = dev_bits(wl["q"])
    multi = spec.q_len > 1
    q_start = torch.from_numpy(wl["q_start"]).to(device) if multi else None
    new_k, new_v = dev_bits(wl["new_k"]), dev_bits(wl["new_v"])
    slots = torch.from_numpy(wl["slots"]).to(device)
    tables = torch.from_numpy(wl["tables"]).to(device)
    lens = torch.from_numpy(wl["lens"]).to(device)
    cow = torch.from_numpy(wl["cow"]).to(device) if wl["cow"].size else None
    out = torch.empty_like(q)
    B, Hq, D = spec.num_seqs, spec.num_q_heads, spec.head_dim
    max_len = int(wl["lens"].max())
    psize = spec.partition_size
    # parallel samples: read each shared prompt block once per pack of sequences
    shared = spec.len_dist == "shared_prefix" and not args.no_shared_prefix and not spec.fp8
    if shared:
        shared_blocks = torch.from_numpy(wl["shared_blocks"]).to(device)
        ws = pa.alloc_workspace(pa.shared_prefix_workspace_bytes(
            B, Hq, spec.num_kv_heads, D, spec.block_size, max_len, psize), device)
    elif multi:
        ws = pa.alloc_workspace(pa.multi_query_workspace_bytes(
            B, q.shape[0], spec.q_len, Hq, spec.num_kv_heads, D, spec.block_size, max_len,
            psize), device)
    else:
        ws = pa.alloc_workspace(pa.decode_workspace_bytes(
            B, Hq, spec.num_kv_heads, D, spec.block_size, max_len, psize), device)
    flag = torch.zeros(1, dtype=torch.int32, device=device)
    scale = W.scale_of(spec)
    stream = torch.cuda.current_stream(device)
    # one query token per sequence, no packs: the host-planned decode applies
    plannable = not shared and not multi
    launches_per_step = 1 + 3 + (1 if cow is not None else 0)

    def step():
        if cow is not None:
            pa.copy_blocks([k_cache], [v_cache], cow, error_flag=flag)
        if spec.fp8:
            pa.reshape_and_cache(new_k, new_v, k_cache, v_cache, slots, kv_cache_dtype="fp8_e4m3",
                                 k_scale=k_scale, v_scale=v_scale, error_flag=flag)
        else:
            pa.reshape_and_cache(new_k, new_v, k_cache, v_cache, slots, error_flag=flag)
        attention()

    def attention():
        if spec.fp8:
            pa.decode_attention_fp8(out, q, k_cache, v_cache, k_scale, v_scale, tables, lens,
                                    max_len, scale, psize, ws, error_flag=flag)
        elif shared:
            pa.decode_attention_shared_prefix(out, q, k_cache, v_cache, tables, lens,
                                              shared_blocks, max_len, scale, psize, ws,
                                              error_flag=flag)
        elif multi:
            pa.decode_attention_multi_query(out, q, q_start, k_cache, v_cache, tables, lens,
                                            max_len, spec.q_len, scale, psize, ws,
                                            error_flag=flag)
        else:
            pa.decode_attention(out, q, k_cache, v_cache, tables, lens, max_len, scale, psize, ws,
                                error_flag=flag)

    bytes_step = kv_bytes(spec, wl["lens"])
    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    clocks.start()
    time.sleep(1.0)  # let nvidia-smi attach
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(flag.item()) != 0:
        raise RuntimeError("device error flag %#x during warm-up" % int(flag.item()))

    # The timed steps replay one captured step (its kernels chained by
    # programmatic dependent launch, no host launch cost); --no-graph launches
    # them one by one instead.
    run_stream = stream
    graph = None
    if not args.no_graph:
        run_stream = torch.cuda.Stream(device=device)
        run_stream.wait_stream(stream)
        with torch.cuda.stream(run_stream):
            step()
        run_stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=run_stream, capture_error_mode="thread_local"):
            step()
        torch.cuda.synchronize()
        for _ in range(3):  # warm-up replays
            with torch.cuda.stream(run_stream):
                graph.replay()
        torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    with torch.cuda.stream(run_stream):
        t_start.record(run_stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step()
        t_end.record(run_stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    # The attention call alone, for the roofline: its average duration over
    # att_calls calls launched back to back on its stream between two events
    # (an event between the calls of one chain would break the programmatic
    # dependent launch that overlaps them), whatever --steps is.
    att_calls = args.att_calls

    def chained(fn):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a0.record(stream)
        for _ in range(att_calls):
            fn()
        a1.record(stream)
        torch.cuda.synchronize()
        return a0.elapsed_time(a1) / att_calls

    att_avg_ms = chained(attention)
    clock_info = clocks.summary(wall0, wall1)
    clocks.stop()
    # the same decode with its split plan made on the host (pa_decode_plan,
    # copied to the device once): main kernel + combine, no plan kernel
    planned = None
    if plannable:
        hplan, _ = pa.decode_plan(torch.from_numpy(np.ascontiguousarray(wl["lens"])), Hq,
                                  spec.num_kv_heads, D, spec.block_size, max_len, psize,
                                  "fp8_e4m3" if spec.fp8 else "auto")
        dplan = hplan.to(device)

        def planned():
            pa.decode_attention_planned(out, q, k_cache, v_cache, tables, lens, max_len, scale,
                                        dplan, psize, ws, k_scale=k_scale, v_scale=v_scale,
                                        error_flag=flag)
        planned_avg_ms = chained(planned)
    read_bytes = unique_kv_bytes(spec, wl) if spec.len_dist == "shared_prefix" else bytes_step
    latency = latency_distribution(attention, read_bytes, device, stream)
    latency_planned = (latency_distribution(planned, read_bytes, device, stream)
                       if planned is not None else None)
    ceiling = read_ceiling(device, stream)
    if int(flag.item()) != 0:
        raise RuntimeError("device error flag %#x in the timed region" % int(flag.item()))

    # ---------------- end to end: pinned host buffers through the C entry point
    # pa_decode_step (plan on the host, one H2D copy, the kernels, one D2H copy)
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e_ok = plannable and wl["slots"].shape[0] == B
    e2e = None
    if e2e_ok:
        ncow = 0 if cow is None else int(cow.shape[0])
        runner = pa.DecodeStep(k_cache, v_cache, B, Hq, wl["tables"].shape[1], max_len, scale,
                               psize, query_dtype=td, k_scale=k_scale, v_scale=v_scale,
                               max_cow=ncow, slots=2)

        def fill(dst, a, dtype=None):
            t = torch.from_numpy(np.ascontiguousarray(a))
            dst.copy_(t.view(torch.int16).view(dtype) if dtype is not None else t)

        for sl in range(2):
            h = runner.host(sl)
            fill(h["q"], case.q, td)
            fill(h["new_k"], wl["new_k"], td)
            fill(h["new_v"], wl["new_v"], td)
            fill(h["slots"], wl["slots"])
            fill(h["tables"], wl["tables"])
            fill(h["lens"], wl["lens"])
            if ncow:
                fill(h["cow"], wl["cow"])
        for i in range(4):  # warm-up
            runner.submit(i % 2, ncow, error_flag=flag)
            runner.wait(i % 2)
        if world > 1:
            torch.distributed.barrier()
        # serving loop: step i + 1 (its own slot and stream) is submitted
        # before the host waits for step i, so one step's copies overlap
        # another's kernels; every step copies its inputs in and its output out
        t0 = time.perf_counter()
        runner.submit(0, ncow, error_flag=flag)
        for i in range(1, e2e_steps):
            runner.submit(i % 2, ncow, error_flag=flag)
            runner.wait((i - 1) % 2)
        runner.wait((e2e_steps - 1) % 2)
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, device)
        # the same step alone through the single call pa_decode_step (its three
        # parts on one stream), each waited for: no overlap between steps
        t0 = time.perf_counter()
        for i in range(e2e_steps):
            runner(ncow, error_flag=flag)
        serial_s = max_over_ranks(time.perf_counter() - t0, world, device)
        e2e = {"value": round(bytes_step * e2e_steps * world / e2e_s / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": runner.h2d_bytes(), "d2h_bytes_per_step": runner.d2h_bytes(),
               "steps": e2e_steps, "ms_per_step": round(e2e_s * 1e3 / e2e_steps, 4),
               "serial": {"value": round(bytes_step * e2e_steps * world / serial_s / 1e9, 2),
                          "ms_per_step": round(serial_s * 1e3 / e2e_steps, 4),
                          "how": "pa_decode_step (upload, run, download on one stream), each "
                                 "step waited for before the next is issued"},
               "how": "C ABI from pinned host buffers, two slots: per step "
                      "pa_decode_step_upload (split plan computed on the host, one H2D copy of "
                      "the staging buffer) on a copy stream, pa_decode_step_run "
                      "(reshape_and_cache + the decode's main kernel + combine, no plan kernel) "
                      "on the compute stream in submission order, pa_decode_step_download (one "
                      "D2H copy of the output) on a second copy stream; step i + 1 is submitted "
                      "before the host waits for step i (wall clock, max over ranks)"}
        if int(flag.item()) != 0:
            raise RuntimeError("device error flag %#x in the end-to-end steps" % int(flag.item()))

    elapsed_ms = max_over_ranks(elapsed_ms, world, device)
    att_avg_ms = max_over_ranks(att_avg_ms, world, device)
    total_bytes = sum_over_ranks(float(bytes_step), world, device)
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    ms_per_step = elapsed_ms / args.steps
    value = total_bytes * args.steps / (elapsed_ms / 1e3) / 1e9
    # the roofline counts the bytes that must come from HBM: for shared
    # prompts each distinct (block, slot) once, else every token's K and V
    achieved = read_bytes / (att_avg_ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    traffic = profiled_traffic() if args.workload == "llama8b" else None
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": spec.dtype + ("/e4m3 cache" if spec.fp8 else ""),
        "data": "synthetic (seeded N(0,1) values; lengths, placement and sharing per workload)",
        "config": {
            "workload": describe_workload(spec),
            "global_batch": spec.num_seqs * world, "kv_bytes_per_step": bytes_step,
            "sum_seq_len": int(wl["lens"].sum()), "partition_size": psize,
            "num_blocks": case.num_blocks, "parallelism": "dp%d (independent batches)" % world,
            "l2": "no flush: each step reads %.0f MB of KV, more than the 126 MB L2" % (bytes_step / 1e6),
            "timed_as": ("a CUDA graph of one step, replayed %d times" % args.steps
                         if graph is not None else "%d steps launched one by one" % args.steps),
        },
        "decode_tokens_per_s": round(spec.num_seqs * spec.q_len * world / (ms_per_step / 1e3), 1),
        "attention_gbs": round(achieved, 2),
        "pct_of_8tbs": round(100.0 * value / 8000.0, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": ("pa_decode_attention_shared_prefix" if shared else
                                "pa_decode_attention_multi_query" if multi else
                                "pa_decode_attention") + " (plan + main + combine launches)",
                     "bytes_per_launch": read_bytes,
                     "peak_kind": ("measured (MEASURED_PEAKS.json hbm_gbs, copy read+write)"
                                   if peak_kind == "measured" else
                                   "fallback (6.65 TB/s copy, an earlier measurement on this "
                                   "pool; MEASURED_PEAKS.json absent)")},
        "attention_calls_averaged": att_calls,
        "attention_latency": latency,
        "read_ceiling": dict(ceiling, frac=round(achieved / ceiling["gbs"], 4)),
        "kv_memory": dict(kv_memory(spec, wl), block_manager={
            k: wl["bm_stats"][k] for k in ("held_blocks", "free_blocks", "stored_slots",
                                           "waste_slots", "max_waste_per_seq")}),
        "clocks": clock_info,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
    }
    if planned is not None:
        planned_avg_ms = max_over_ranks(planned_avg_ms, world, device)
        line["attention_planned"] = {
            "gbs": round(read_bytes / (planned_avg_ms / 1e3) / 1e9, 2),
            "us": round(planned_avg_ms * 1e3, 2), "calls": att_calls,
            "frac_of_peak": round(read_bytes / (planned_avg_ms / 1e3) / 1e9 / peak, 4),
            "how": "pa_decode_attention_planned (plan from pa_decode_plan on the host, copied "
                   "once): main kernel + combine, back to back between two events"}
        line["attention_latency_planned"] = latency_planned
    if spec.len_dist == "shared_prefix":
        ub = unique_kv_bytes(spec, wl)
        line["config"]["unique_kv_bytes_per_step"] = ub
        line["config"]["entry_point"] = ("decode_attention_shared_prefix (packs of up to %d)" % (
            min(8, 32 // spec.group)) if shared else "decode_attention")
        if shared:
            line["config"]["packed_kv_bytes_per_step"] = packed_kv_bytes(spec, wl)
        line["roofline"]["basis"] = "unique KV bytes (each shared block once)"
        line["unique_gbs"] = round(ub * args.steps / (elapsed_ms / 1e3) / 1e9, 2)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(spec, wl, budget_s=args.cpu_budget)
    return line


def describe_workload(spec):
    return "%s: B %d, Hq %d / Hkv %d, D %d, block %d, %s%s, lengths %s" % (
        spec.name, spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
        spec.block_size, spec.dtype, ", fp8 E4M3 cache" if spec.fp8 else "",
        describe_lengths(spec))


def describe_lengths(spec):
    if spec.q_len > 1:
        return "%s, %d new tokens per sequence attending causally" % (
            describe_lengths(spec.replace(q_len=1)), spec.q_len)
    if spec.len_dist == "uniform":
        return "U[%d, %d]" % (spec.len_lo, spec.len_hi)
    if spec.len_dist == "lognormal":
        return "lognormal(median %g, sigma %g) clipped [%d, %d]" % (
            spec.lognormal_median, spec.lognormal_sigma, spec.len_lo, spec.len_hi)
    if spec.len_dist == "shared_prefix":
        return "%d-token prompt x %d samples + U[%d, %d]" % (spec.prompt_len, spec.samples,
                                                            spec.extra_lo, spec.extra_hi)
    return "fixed %s" % (sorted(set(spec.fixed_lens)),)


def rank_spec(spec, rank: int, world: int):
    """Each rank decodes its own, independently seeded batch of the workload
    (weak scaling: sequences are independent, so no data crosses ranks)."""
    return spec if world == 1 else spec.replace(seed=spec.seed + 100 * rank)


def max_over_ranks(x, world, device):
    """Slowest rank's value (device time is reported as the max over ranks)."""
    if world == 1:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------- oracle
def _oracle_sample(spec, wl, seqs):
    """One oracle step over the sequences `seqs`: the writes of their new rows,
    then fp64 attention.  Returns (seconds, kv bytes)."""
    import oracle
    case = wl["case"]
    k, v = case.k_pool, case.v_pool
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    if spec.fp8:
        oracle.reshape_and_cache_fp8(wl["new_k"][seqs], wl["new_v"][seqs], k, v,
                                     wl["slots"][seqs], spec.dtype, spec.k_scale, spec.v_scale)
        oracle.decode_fp8(case.q[seqs], k, v, spec.k_scale, spec.v_scale, wl["tables"][seqs],
                          wl["lens"][seqs], W.scale_of(spec), spec.dtype, nthreads=threads)
        return time.perf_counter() - t0, kv_bytes(spec, wl["lens"][seqs])
    if spec.q_len > 1:  # each sequence's q_len new rows, then its q_len queries
        q = spec.q_len
        rows = (seqs[:, None] * q + np.arange(q)[None, :]).reshape(-1)
        oracle.reshape_and_cache(wl["new_k"][rows], wl["new_v"][rows], k, v, wl["slots"][rows])
        oracle.decode_multi(wl["q"][rows], (np.arange(len(seqs) + 1) * q).astype(np.int32), k, v,
                            wl["tables"][seqs], wl["lens"][seqs], W.scale_of(spec), spec.dtype,
                            nthreads=threads)
        return time.perf_counter() - t0, kv_bytes(spec, wl["lens"][seqs])
    if spec.len_dist != "shared_prefix":
        oracle.reshape_and_cache(wl["new_k"][seqs], wl["new_v"][seqs], k, v, wl["slots"][seqs])
    oracle.decode(case.q[seqs], k, v, wl["tables"][seqs], wl["lens"][seqs], W.scale_of(spec),
                  spec.dtype, nthreads=threads)
    return time.perf_counter() - t0, kv_bytes(spec, wl["lens"][seqs])


def cpu_baseline(spec, wl, budget_s=20.0):
    """The oracle, as it stands, on all host cores, over a bounded sample:
    whole-batch steps repeated while they fit in the budget (at least one)."""
    B = spec.num_seqs
    threads = len(os.sched_getaffinity(0))
    total_t, total_b, n = 0.0, 0, 0
    seqs = np.arange(B)
    while True:
        t, b = _oracle_sample(spec, wl, seqs)
        total_t += t
        total_b += b
        n += 1
        if total_t + t > budget_s or n >= 40:
            break
    return {"value": round(total_b / total_t / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle", "sample": describe_oracle_sample(spec, wl, n, B, total_t)}


def describe_oracle_sample(spec, wl, steps, per_step, seconds):
    """One wording for both oracle legs (cpu_baseline and --impl reference)."""
    B = spec.num_seqs
    what = ("full step(s) of the %s batch (%d sequences, %d tokens each step)" % (
        spec.name, B, int(wl["lens"].sum())) if per_step == B else
        "step(s) of %d of the %s batch's %d sequences (seeded random sample)" % (
            per_step, spec.name, B))
    return "%d %s: reshape_and_cache + fp64 decode on all host cores, %.1f s timed" % (
        steps, what, seconds)


def run_reference(args, rank, world):
    if rank != 0:
        return None
    spec = W.WORKLOADS[args.workload]

    # the oracle's own block manager builds the metadata for the reference arm
    from oracle.blockmgr import RefBlockManager
    case = W.draw(spec)
    bm = RefBlockManager(case.num_blocks, spec.block_size, case.free_order)
    lens = case.seq_lens.astype(np.int32)
    slots, new_k, new_v = _append_new_tokens(spec, bm, lens)
    width = max(len(bm.block_table(b)) for b in range(spec.num_seqs))
    tables = np.full((spec.num_seqs, width), -1, np.int32)
    for b in range(spec.num_seqs):
        t = bm.block_table(b)
        tables[b, :len(t)] = t
    wl = dict(case=case, lens=lens, tables=tables, slots=np.array(slots, np.int32),
              new_k=new_k, new_v=new_v)
    _add_queries(spec, wl)
    # Each step is the whole batch, as in the cpu_baseline leg, when warm-up +
    # timed steps fit in args.ref_budget seconds; otherwise a seeded sample of
    # the batch's sequences sized to fit.
    B = spec.num_seqs
    t_full, _ = _oracle_sample(spec, wl, np.arange(B))
    n_steps = args.warmup + args.steps
    per_step = B if t_full * n_steps <= args.ref_budget else max(
        1, min(B, int(args.ref_budget / n_steps / max(t_full / B, 1e-4))))
    rng = np.random.default_rng(0)

    def pick():
        return np.arange(B) if per_step == B else np.sort(rng.choice(B, per_step, replace=False))

    for _ in range(args.warmup):
        _oracle_sample(spec, wl, pick())
    tt, tb = 0.0, 0
    for _ in range(args.steps):
        t, b = _oracle_sample(spec, wl, pick())
        tt += t
        tb += b
    value = tb / tt / 1e9
    threads = len(os.sched_getaffinity(0))
    sample = describe_oracle_sample(spec, wl, args.steps, per_step, tt)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) values; lengths and placement per workload)",
        "config": {"workload": describe_workload(spec), "global_batch": spec.num_seqs,
                   "kv_bytes_per_step": kv_bytes(spec, wl["lens"]),
                   "sum_seq_len": int(wl["lens"].sum()), "partition_size": spec.partition_size,
                   "parallelism": "host cores (the fp64 oracle)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama8b", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--att-calls", type=int, default=500,
                    help="back-to-back attention calls averaged for the roofline")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--ref-budget", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying a graph")
    ap.add_argument("--no-shared-prefix", action="store_true",
                    help="shared_prefix workload: use the plain decode entry point")
    ap.add_argument("--block-size", type=int, default=0,
                    help="override the workload's block size (block-size sweep)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
