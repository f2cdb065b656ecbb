"""Pins for the oracle's prefix-cache model ("大模型推理的KV Cache管理…优化实战",
§三 AutomaticPrefixCache / PrefixRadixTree): hits in whole blocks, longest
match against a brute-force search over what was cached, LRU order, leaves
first, held blocks never evicted, the key's byte layout."""
import hashlib

import numpy as np
import pytest

from oracle.allocator import BlockManagerModel, NoBlocks, prefix_key


def _cached(m, seq, tokens):
    m.add(seq)
    m.append(seq, len(tokens))
    m.prefix_insert(seq, tokens)


def test_hit_rounds_down_to_whole_blocks():
    m = BlockManagerModel(64)
    toks = list(range(100, 137))                       # 37 tokens: two full blocks cached
    _cached(m, 0, toks)
    assert m.prefix_match(toks + [5, 6])[0] == 32
    assert m.prefix_match(toks[:35])[0] == 32
    assert m.prefix_match(toks[:31])[0] == 16
    assert m.prefix_match(toks[:15])[0] == 0
    assert m.prefix_match([7] + toks[1:])[0] == 0      # first block differs


def test_key_is_blake2b_of_little_endian_int32():
    m = BlockManagerModel(8)
    toks = [258] * 16
    _cached(m, 0, toks)
    hit, key = m.prefix_match(toks)
    assert hit == 16
    assert key == hashlib.blake2b(bytes([2, 1, 0, 0]) * 16, digest_size=16).digest()
    assert prefix_key([-1]) == hashlib.blake2b(b"\xff\xff\xff\xff", digest_size=16).digest()
    assert m.prefix_match([1] * 16)[1] == bytes(16)


def test_longest_match_against_brute_force():
    rng = np.random.default_rng(0)
    m = BlockManagerModel(400)
    inserted = []
    base = rng.integers(0, 4, 200).tolist()
    for s in range(12):
        cut = int(rng.integers(0, 200))
        toks = base[:cut] + rng.integers(0, 4, int(rng.integers(0, 60))).tolist()
        _cached(m, s, toks)
        inserted.append(toks)
    for _ in range(200):
        cut = int(rng.integers(0, 200))
        q = base[:cut] + rng.integers(0, 4, int(rng.integers(0, 40))).tolist()
        best = 0
        for t in inserted:
            k = 0
            while (k + 1) * 16 <= min(len(q), len(t)) and q[k * 16:(k + 1) * 16] == t[k * 16:(k + 1) * 16]:
                k += 1
            best = max(best, k * 16)
        hit, key = m.prefix_match(q)
        assert hit == best
        assert key == (prefix_key(q[:hit]) if hit else bytes(16))


def test_lru_and_leaves_first():
    m = BlockManagerModel(32)
    a, b = [1] * 48, [2] * 32                            # 3 + 2 cached blocks
    _cached(m, 0, a)
    _cached(m, 1, b)
    m.free_seq(0)
    m.free_seq(1)
    assert m.prefix_stats()[:2] == (5, 2)                # only the two leaves are evictable
    m.prefix_match(a)                                    # a is now the more recent
    assert m.prefix_evict(4) == 1
    assert m.prefix_match(b)[0] == 16 and m.prefix_match(a)[0] == 48
    # b's remaining block became a leaf and was used before a's last match
    assert m.prefix_evict(3) == 1
    assert m.prefix_match(b)[0] == 0 and m.prefix_match(a)[0] == 48
    assert m.prefix_evict(2) == 1                        # a's chain shrinks from its leaf
    assert m.prefix_match(a)[0] == 32
    assert m.prefix_evict(0) == 2
    assert m.prefix_stats()[0] == 0 and len(m.free) == 32


def test_blocks_held_by_sequences_are_never_evicted():
    m = BlockManagerModel(8)
    _cached(m, 0, [3] * 64)                              # 4 blocks, all held by seq 0 and the cache
    assert m.prefix_evict(0) == 0
    hit = m.add_cached(1, [3] * 40)
    assert hit == 32 and m.block_table(1) == m.block_table(0)[:2]
    assert [m.refcount(b) for b in m.block_table(0)] == [3, 3, 2, 2]
    m.free_seq(0)
    assert m.prefix_evict(0) == 2                        # the two blocks seq 1 does not hold
    assert m.prefix_stats()[0] == 2


def test_allocation_evicts_when_the_free_list_is_empty_and_failure_restores():
    m = BlockManagerModel(4)
    _cached(m, 0, [9] * 48)                              # 3 blocks cached
    m.free_seq(0)
    assert len(m.free) == 1
    m.add(1)
    m.append(1, 32)                                      # takes the free block, then evicts one leaf
    assert m.prefix_stats()[0] == 2 and m.evictions == 1
    before = (list(m.free), list(m.rc), m.prefix_stats(), m.prefix_match([9] * 48)[0])
    m.add(2)
    with pytest.raises(NoBlocks):
        m.append(2, 64)                                  # needs 4 blocks, only 2 evictable
    after = (list(m.free), list(m.rc), m.prefix_stats(), m.prefix_match([9] * 48)[0])
    assert before[0] == after[0] and before[1] == after[1] and before[3] == after[3] == 32
