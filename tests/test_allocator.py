"""The C++ block allocator against the oracle's pure-Python model, step by
step, plus its transactional and error behaviour."""
import numpy as np
import pytest

from oracle.allocator import BlockManagerModel, NoBlocks
from paged_kv_cache_438_b200 import pagedkv as P


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_438_b200 import build
    build.build()


def _same(alloc, model, seqs):
    for s in seqs:
        assert alloc.block_table(s) == model.block_table(s)
        assert alloc.seq_len(s) == model.seq_len(s)
    for b in range(model.num_blocks):
        assert alloc.refcount(b) == model.refcount(b)
    assert alloc.stats() == model.stats()


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_model(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(20, 120))
    order = rng.permutation(nb).tolist() if seed % 2 else None
    a = P.BlockAllocator(nb, initial_free_order=order)
    m = BlockManagerModel(nb, initial_free_order=order)
    live, nxt = [], 0
    for _ in range(300):
        op = rng.integers(0, 10)
        if op == 0 or not live:
            a.add(nxt); m.add(nxt); live.append(nxt); nxt += 1
        elif op == 1:
            parent = live[int(rng.integers(len(live)))]
            plen = int(rng.integers(0, m.seq_len(parent) + 1)) if rng.random() < 0.5 else -1
            a.fork(parent, nxt, plen); m.fork(parent, nxt, None if plen < 0 else plen)
            live.append(nxt); nxt += 1
        elif op == 2 and len(live) > 1:
            s = live.pop(int(rng.integers(len(live))))
            a.free(s); m.free_seq(s)
        elif op == 3:
            ids = [live[i] for i in rng.permutation(len(live))[: int(rng.integers(1, len(live) + 1))]]
            try:
                ref = []
                exp_pairs = []
                snap = (list(m.free), list(m.rc), {k: list(v) for k, v in m.tables.items()}, dict(m.lens))
                for s in ids:
                    sl, pr = m.append(s, 1)
                    ref += sl; exp_pairs += pr
                ok = True
            except NoBlocks:
                m.free, m.rc, m.tables, m.lens = snap[0], snap[1], snap[2], snap[3]
                ok = False
            if ok:
                slots, pairs = a.batch_append(ids)
                assert slots.tolist() == ref and [tuple(p) for p in pairs.tolist()] == exp_pairs
            else:
                with pytest.raises(P.NoBlocksError):
                    a.batch_append(ids)
        else:
            s = live[int(rng.integers(len(live)))]
            n = int(rng.integers(1, 40))
            try:
                ref, exp_pairs = m.append(s, n)
            except NoBlocks:
                with pytest.raises(P.NoBlocksError):
                    a.append(s, n)
            else:
                slots, pairs = a.append(s, n)
                assert slots.tolist() == ref and [tuple(p) for p in pairs.tolist()] == exp_pairs
        _same(a, m, live)
    a.close()


def test_oom_is_transactional():
    a = P.BlockAllocator(4)
    a.add(0)
    a.append(0, 20)
    before = (a.block_table(0), a.seq_len(0), a.stats())
    with pytest.raises(P.NoBlocksError):
        a.append(0, 100)
    assert (a.block_table(0), a.seq_len(0), a.stats()) == before


def test_batch_tables_export_and_errors():
    a = P.BlockAllocator(64)
    for s in range(3):
        a.add(s)
        a.append(s, 10 * (s + 1))
    bt, cl = a.batch_tables([0, 1, 2], 4)
    assert cl.tolist() == [10, 20, 30]
    assert bt[0, 0] == a.block_table(0)[0] and bt[0, 1:].tolist() == [0, 0, 0]
    with pytest.raises(P.PagedKVError):
        a.batch_tables([0, 1, 2], 1)          # sequence 1 needs 2 blocks
    with pytest.raises(P.PagedKVError):
        a.add(1)                              # exists
    with pytest.raises(P.PagedKVError):
        a.free(99)                            # unknown
    with pytest.raises(P.PagedKVError):
        P.BlockAllocator(8, initial_free_order=[0, 1, 2, 3, 4, 5, 6, 6])
    with pytest.raises(P.PagedKVError):
        P.BlockAllocator(8, block_size=32)


def test_prefix_share_2040_gives_127_copies():
    # 128 sequences share a 2040-token prefix; the last prefix block holds 8
    # tokens, so every sharer but the last copies it on its first write.
    a = P.BlockAllocator(128 + 200)
    a.add(0)
    a.append(0, 2040)
    for c in range(1, 128):
        a.fork(0, c)
    slots, pairs = a.batch_append(list(range(128)))
    assert pairs.shape[0] == 127
    assert len(set(pairs[:, 0].tolist())) == 1 and len(set(pairs[:, 1].tolist())) == 127
    assert a.refcount(int(pairs[0, 0])) == 1
    nfree, nshared, _ = a.stats()
    assert nshared == 127                     # the 127 full prefix blocks stay shared


def test_block_aligned_prefix_2048_needs_no_copy():
    a = P.BlockAllocator(128 + 200)
    a.add(0)
    a.append(0, 2048)
    for c in range(1, 128):
        a.fork(0, c)
    _, pairs = a.batch_append(list(range(128)))
    assert pairs.shape[0] == 0
