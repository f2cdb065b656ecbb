"""Pins for the oracle's slot-mapped write, block copy and block-manager model."""
import numpy as np
import pytest

from oracle import cache_ops as C
from oracle.allocator import BlockManagerModel, NoBlocks


# ------------------------------------------------------------------- write --

def test_write_places_rows_by_slot_and_skips_minus_one():
    rng = np.random.default_rng(0)
    cache = rng.integers(0, 1 << 16, size=(5, 2, 16, 4), dtype=np.uint16)
    x = rng.integers(0, 1 << 16, size=(4, 2, 4), dtype=np.uint16)
    slots = [17, -1, 0, 79]
    out = C.kv_write(cache, x, slots)
    assert np.array_equal(out[1, :, 1], x[0])      # slot 17 = block 1, offset 1
    assert np.array_equal(out[0, :, 0], x[2])
    assert np.array_equal(out[4, :, 15], x[3])
    touched = np.zeros((5, 16), bool)
    touched[1, 1] = touched[0, 0] = touched[4, 15] = True
    assert np.array_equal(out.transpose(0, 2, 1, 3)[~touched], cache.transpose(0, 2, 1, 3)[~touched])


def test_write_idempotent():
    rng = np.random.default_rng(1)
    cache = rng.standard_normal((3, 1, 16, 8))
    x = rng.standard_normal((2, 1, 8))
    once = C.kv_write(cache, x, [5, 40])
    assert np.array_equal(C.kv_write(once, x, [5, 40]), once)


def test_scale_write():
    sc = np.zeros((2, 3, 16), np.float32)
    out = C.scale_write(sc, np.array([[1, 2, 3], [4, 5, 6]], np.float32), [31, -1])
    assert out[1, :, 15].tolist() == [1, 2, 3] and out.sum() == 6


def test_copy_blocks_reads_pre_call_state():
    a = np.arange(4 * 3).reshape(4, 3)
    (b,) = C.copy_blocks([a], [(0, 1), (1, 0), (2, 3)])
    assert b[1].tolist() == a[0].tolist() and b[0].tolist() == a[1].tolist()
    assert b[3].tolist() == a[2].tolist() and b[2].tolist() == a[2].tolist()


# --------------------------------------------------------- block manager --

def test_lifo_from_highest_id():
    m = BlockManagerModel(8)
    m.add(0)
    slots, pairs = m.append(0, 33)
    assert m.block_table(0) == [7, 6, 5] and pairs == []
    assert slots[0] == 7 * 16 and slots[16] == 6 * 16 and slots[32] == 5 * 16


def test_initial_free_order_is_popped_from_the_end():
    m = BlockManagerModel(4, initial_free_order=[2, 0, 3, 1])
    m.add(1)
    m.append(1, 20)
    assert m.block_table(1) == [1, 3]


def test_oom_leaves_state_unchanged():
    m = BlockManagerModel(3)
    m.add(0)
    m.append(0, 20)
    before = (list(m.free), list(m.rc), m.block_table(0), m.seq_len(0))
    with pytest.raises(NoBlocks):
        m.append(0, 40)
    assert (list(m.free), list(m.rc), m.block_table(0), m.seq_len(0)) == before


def test_internal_waste_at_most_one_block():
    rng = np.random.default_rng(2)
    m = BlockManagerModel(400)
    for s in range(10):
        m.add(s)
        m.append(s, int(rng.integers(1, 300)))
        assert len(m.block_table(s)) * 16 - m.seq_len(s) < 16


def test_fork_shares_ceil_prefix_blocks_and_counts_refs():
    m = BlockManagerModel(20)
    m.add(0)
    m.append(0, 50)                      # 4 blocks
    m.fork(0, 1, prefix_len=33)           # ceil(33/16) = 3 shared
    assert m.block_table(1) == m.block_table(0)[:3]
    assert [m.refcount(b) for b in m.block_table(0)] == [2, 2, 2, 1]
    assert sum(m.rc) == sum(len(t) for t in m.tables.values())


def test_cow_n_sharers_make_n_minus_1_copies():
    m = BlockManagerModel(200)
    m.add(0)
    m.append(0, 40)                       # last block half full, shared below
    for c in range(1, 5):
        m.fork(0, c)
    shared_last = m.block_table(0)[-1]
    copies = []
    for s in range(5):
        _, pairs = m.append(s, 1)
        copies += pairs
    assert len(copies) == 4 and all(src == shared_last for src, _ in copies)
    assert m.block_table(4)[-1] == shared_last       # last holder writes in place
    assert m.refcount(shared_last) == 1
    assert sum(m.rc) == sum(len(t) for t in m.tables.values())


def test_block_aligned_prefix_needs_no_copy():
    m = BlockManagerModel(50)
    m.add(0)
    m.append(0, 32)
    m.fork(0, 1)
    _, p0 = m.append(0, 1)
    _, p1 = m.append(1, 1)
    assert p0 == [] and p1 == []


def test_free_returns_blocks_at_refcount_zero():
    m = BlockManagerModel(10)
    m.add(0)
    m.append(0, 20)
    m.fork(0, 1)
    m.free_seq(0)
    assert len(m.free) == 8
    m.free_seq(1)
    assert len(m.free) == 10 and sum(m.rc) == 0


def test_stats_fragmentation_run():
    m = BlockManagerModel(8, initial_free_order=list(range(8)))
    m.add(0)
    m.append(0, 16 * 3)                   # takes 7, 6, 5
    nfree, nshared, run = m.stats()
    assert (nfree, nshared, run) == (5, 0, 5)
