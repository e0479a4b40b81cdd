"""The split plan computed on the host (pa_split_plan; CPU, no GPU).

The decode lays every sequence's 16-token tiles end to end and cuts the
line into C shares evenly in weighted tiles: a sequence with tiles is
preceded by PA_PLAN_ENTRY_WEIGHT = 3 virtual tiles (the cost of a CTA moving
to it), a cut that falls there starting the share at the sequence's first
tile (unweighted above PA_PLAN_WEIGHTED_MAX_ENTRIES = 4096 sequences).  A
sequence is cut wherever a CTA's share or a partition starts.  This file
restates that definition in Python (the virtual line listed tile by tile,
a set of segment starts per sequence) and checks the library's walk against
it on random batches: the tile and segment prefix sums, each CTA's first
tile, first sequence and segment index, and whether any sequence is split
(which decides if the combine runs)."""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def pa():
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location(
        "_pa_build", os.path.join(root, "paged_kv_cache_343_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()
    import paged_kv_cache_343_b200 as pa
    return pa


def brute_plan(lens, max_len, partition_size, C):
    """Segment starts enumerated tile by tile."""
    tiles_of = [(min(max(int(L), 0), max_len) + 15) // 16 for L in lens]
    t = np.concatenate([[0], np.cumsum(tiles_of)]).astype(np.int64)
    N = int(t[-1])
    tpp = partition_size // 16 if partition_size else None
    # the virtual line: each sequence with tiles is W switch slots (its first
    # tile) followed by its tiles; a cut at virtual x starts at real[x]
    W = 3 if len(lens) <= 4096 else 0
    real = []
    for b, n in enumerate(tiles_of):
        if n > 0:
            real += [int(t[b])] * W + list(range(int(t[b]), int(t[b]) + n))
    V = len(real)
    lo = [real[c * V // C] if c * V // C < V else N for c in range(C + 1)]
    starts = []  # per sequence: sorted segment starts (global tile index)
    for b in range(len(lens)):
        t0, t1 = int(t[b]), int(t[b + 1])
        S = set()
        for x in range(t0, t1):
            if x == t0 or (tpp and (x - t0) % tpp == 0) or x in lo:
                S.add(x)
        starts.append(sorted(S))
    seg_base = np.concatenate([[0], np.cumsum([len(S) for S in starts])]).astype(np.int32)
    start_seq = np.zeros(C, np.int32)
    first_k = np.zeros(C, np.int32)
    for c in range(C):
        if N == 0:
            continue
        x = lo[c]
        b = max(i for i in range(len(lens)) if t[i] <= x and t[i + 1] > x)
        start_seq[c] = b
        first_k[c] = sum(1 for s in starts[b] if s < x)
    return dict(tiles=t.astype(np.int32), seg_base=seg_base, start_seq=start_seq,
                first_k=first_k, cta_first_tile=np.array(lo, np.int32),
                num_segments=int(seg_base[-1]),
                needs_combine=any(len(S) > 1 for S in starts))


CASES = [
    # lengths, max_seq_len, partition_size, CTAs
    ([5, 40, 0, 100], 128, 0, 7),
    ([1, 5, 16, 22], 22, 0, 148),           # more CTAs than tiles: empty shares
    ([32768] * 8, 32768, 512, 148),         # long context, 512-token partitions
    ([0, 0, 0], 8, 0, 4),                   # nothing to attend
    ([16, 16, 16, 16], 16, 16, 2),          # every tile its own partition
]


@pytest.mark.parametrize("lens,max_len,psize,C", CASES)
def test_split_plan_matches_the_definition(pa, lens, max_len, psize, C):
    got = pa.split_plan(lens, max_len, psize, C)
    ref = brute_plan(lens, max_len, psize, C)
    for k in ("tiles", "seg_base", "cta_first_tile"):
        assert np.array_equal(got[k], ref[k]), k
    N = int(ref["tiles"][-1])
    if N:
        # CTAs with an empty share never read their entry; compare the others
        lo = ref["cta_first_tile"]
        busy = lo[:-1] < lo[1:]
        assert np.array_equal(got["start_seq"][busy], ref["start_seq"][busy])
        assert np.array_equal(got["first_k"][busy], ref["first_k"][busy])
    assert got["num_segments"] == ref["num_segments"]
    assert got["needs_combine"] == ref["needs_combine"]


@pytest.mark.parametrize("seed", range(6))
def test_split_plan_random_batches(pa, seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 90))
    max_len = int(rng.integers(1, 3000))
    lens = rng.integers(0, max_len + 1, B)
    psize = int(rng.choice([0, 16, 64, 512]))
    C = int(rng.choice([1, 3, 37, 148, 296]))
    got = pa.split_plan(lens, max_len, psize, C)
    ref = brute_plan(lens, max_len, psize, C)
    assert np.array_equal(got["tiles"], ref["tiles"])
    assert np.array_equal(got["seg_base"], ref["seg_base"])
    assert np.array_equal(got["cta_first_tile"], ref["cta_first_tile"])
    lo = ref["cta_first_tile"]
    busy = lo[:-1] < lo[1:]
    assert np.array_equal(got["start_seq"][busy], ref["start_seq"][busy])
    assert np.array_equal(got["first_k"][busy], ref["first_k"][busy])
    assert got["needs_combine"] == ref["needs_combine"]


@pytest.mark.parametrize("B", [4096, 4097, 5000])
def test_split_plan_weight_limit(pa, B):
    """The switch weight applies while the batch's prefix sums fit the plan
    kernel's shared table (PA_PLAN_WEIGHTED_MAX_ENTRIES = 4096 sequences);
    above it the line is cut evenly in real tiles, so share c starts at
    tile floor(c N / C)."""
    rng = np.random.default_rng(B)
    lens = rng.integers(0, 65, B)
    C = 148
    got = pa.split_plan(lens, 64, 0, C)
    ref = brute_plan(lens, 64, 0, C)
    assert np.array_equal(got["tiles"], ref["tiles"])
    assert np.array_equal(got["seg_base"], ref["seg_base"])
    assert np.array_equal(got["cta_first_tile"], ref["cta_first_tile"])
    N = int(ref["tiles"][-1])
    even = np.array([c * N // C for c in range(C + 1)], np.int32)
    if B > 4096:
        assert np.array_equal(got["cta_first_tile"], even)
    else:
        assert not np.array_equal(got["cta_first_tile"], even)
    lo = ref["cta_first_tile"]
    busy = lo[:-1] < lo[1:]
    assert np.array_equal(got["start_seq"][busy], ref["start_seq"][busy])
    assert np.array_equal(got["first_k"][busy], ref["first_k"][busy])
    assert got["needs_combine"] == ref["needs_combine"]


def test_split_plan_refuses_bad_arguments(pa):
    import paged_kv_cache_343_b200 as m
    with pytest.raises(m.PagedAttnError):      # a length above max_seq_len
        pa.split_plan([5, 300], 200, 0, 4)
    with pytest.raises(m.PagedAttnError):      # partitions not in whole tiles
        pa.split_plan([5, 30], 200, 24, 4)
    with pytest.raises(m.PagedAttnError):      # no CTA
        pa.split_plan([5, 30], 200, 0, 0)


def test_line_cut_matches_the_definition(tmp_path):
    """The cut of the tile line into CTA shares that the plan kernel and the
    decode kernels share (LineCut): a host program built by nvcc with the
    library's flags checks it against its definition written out as loops
    (even shares, the packs' tiles and the sequences' tiles cut separately
    when a shared-prompt call runs two kernels, and the count of shares
    starting below every tile) on the benchmark's shapes, edge cases and 400
    random ones."""
    import os
    import shutil
    import subprocess
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    if not os.path.exists(nvcc) and shutil.which("nvcc") is None:
        pytest.skip("no nvcc")
    if not os.path.exists(nvcc):
        nvcc = shutil.which("nvcc")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = tmp_path / "linecut_check"
    build = subprocess.run(
        [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
         "--expt-relaxed-constexpr", "-I", os.path.join(root, "include"),
         os.path.join(root, "tests", "c", "linecut_check.cu"), "-o", str(exe)],
        capture_output=True, text=True, timeout=300)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "all checks held" in run.stdout
