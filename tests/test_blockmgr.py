"""Host block manager: the reference (oracle) manager against the pages'
rules, CPU only.  ("PagedAttention": a new block only once the last one is
out of slots; refcounts; copy-on-write of a shared partial block; full
blocks are never copied; at most one copy per sequence.)"""
import pytest

from oracle.blockmgr import OutOfBlocks, RefBlockManager


def test_allocate_when_previous_block_full():
    bm = RefBlockManager(8, 4)
    bm.add_sequence(0, 5)            # 2 blocks, the second holds 1 token
    assert len(bm.block_table(0)) == 2
    for _ in range(3):               # positions 5, 6, 7 fill block 2
        bm.append_slot(0)
    assert len(bm.block_table(0)) == 2
    slot, cow = bm.append_slot(0)    # position 8: first touch of block 3
    assert cow is None
    assert len(bm.block_table(0)) == 3
    assert slot == bm.block_table(0)[2] * 4
    bm.check_invariants()


def test_blocks_come_from_the_free_list_in_order():
    order = [5, 1, 7, 0, 3, 2, 6, 4]
    bm = RefBlockManager(8, 4, order)
    bm.add_sequence(0, 9)
    bm.add_sequence(1, 2)
    assert bm.block_table(0) == [5, 1, 7]
    assert bm.block_table(1) == [0]


def test_copy_on_write_parallel_sampling():
    bs, prompt, n = 4, 7, 4          # one full block + a 3-token partial block
    bm = RefBlockManager(32, bs, list(range(32)))
    bm.add_sequence(0, prompt)
    for s in range(1, n):
        bm.fork(0, s)
    full, partial = bm.block_table(0)
    assert bm.refcount[full] == n and bm.refcount[partial] == n
    copies = {}
    for s in range(n):
        slot, cow = bm.append_slot(s)
        if cow is not None:
            copies[s] = cow
        bm.check_invariants()
    # samples that found the partial block shared copied it; the last one wrote in place
    assert sorted(copies) == list(range(n - 1))
    assert all(src == partial for src, _ in copies.values())
    assert bm.block_table(n - 1)[-1] == partial
    # the full prompt block stays shared by everyone and is never copied
    assert bm.refcount[full] == n
    assert all(bm.block_table(s)[0] == full for s in range(n))
    # at most one copy per sequence
    assert len(bm.copies) == n - 1
    # appending past the block boundary allocates, never copies
    for s in range(n):
        _, cow = bm.append_slot(s)
        assert cow is None
        _, cow = bm.append_slot(s)
        assert cow is None
    bm.check_invariants()


def test_free_returns_blocks_and_keeps_shared_ones():
    bm = RefBlockManager(6, 4, list(range(6)))
    bm.add_sequence(0, 8)
    bm.fork(0, 1)
    bm.free_sequence(0)
    assert bm.refcount[0] == 1 and bm.refcount[1] == 1
    assert list(bm.free) == [2, 3, 4, 5]
    bm.free_sequence(1)
    assert list(bm.free) == [2, 3, 4, 5, 0, 1]
    bm.check_invariants()


def test_out_of_blocks():
    bm = RefBlockManager(2, 4)
    bm.add_sequence(0, 8)
    with pytest.raises(OutOfBlocks):
        bm.append_slot(0)


def test_waste_below_one_block_per_sequence():
    bm = RefBlockManager(200, 16)
    lens = [1, 15, 16, 17, 100, 333]
    for i, L in enumerate(lens):
        bm.add_sequence(i, L)
    for i, L in enumerate(lens):
        held = len(bm.block_table(i)) * 16
        assert 0 <= held - L < 16


def test_invariant_checker_catches_planted_errors():
    bm = RefBlockManager(8, 4)
    bm.add_sequence(0, 6)
    bm.refcount[bm.block_table(0)[0]] += 1          # a lost decrement
    with pytest.raises(AssertionError):
        bm.check_invariants()
    bm = RefBlockManager(8, 4)
    bm.add_sequence(0, 6)
    bm.free.append(bm.block_table(0)[1])            # a referenced block freed
    with pytest.raises(AssertionError):
        bm.check_invariants()
