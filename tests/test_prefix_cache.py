"""The C++ allocator's automatic prefix cache against the oracle's model,
step by step on random request streams, plus the BLAKE2b key against
Python's hashlib (CPU only)."""
import hashlib
import struct

import numpy as np
import pytest

from oracle.allocator import BlockManagerModel, NoBlocks, prefix_key
from paged_kv_cache_438_b200 import pagedkv as P


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_438_b200 import build
    build.build()


def test_key_matches_hashlib_blake2b():
    rng = np.random.default_rng(0)
    for n in [0, 1, 15, 16, 31, 32, 33, 64, 100, 513]:
        t = rng.integers(-2 ** 31, 2 ** 31, n).tolist()
        assert P.prefix_key(t) == hashlib.blake2b(struct.pack("<%di" % n, *t), digest_size=16).digest()
        assert P.prefix_key(t) == prefix_key(t)


def _same(a, m, live):
    for s in live:
        assert a.block_table(s) == m.block_table(s)
        assert a.seq_len(s) == m.seq_len(s)
    for b in range(m.num_blocks):
        assert a.refcount(b) == m.refcount(b), b
    assert a.stats() == m.stats()
    assert a.prefix_stats() == m.prefix_stats()


@pytest.mark.parametrize("seed", range(8))
def test_random_request_streams_match_model(seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(24, 90))
    a = P.BlockAllocator(nb, initial_free_order=rng.permutation(nb).tolist())
    m = BlockManagerModel(nb, initial_free_order=a._order.tolist())
    # a few "system prompts" that requests share, over a tiny vocabulary
    prompts = [rng.integers(0, 3, int(rng.integers(16, 80))).tolist() for _ in range(3)]
    toks, live, nxt = {}, [], 0
    for _ in range(400):
        op = int(rng.integers(0, 8))
        if op <= 1 or not live:
            req = prompts[int(rng.integers(3))][: int(rng.integers(0, 80))] + \
                rng.integers(0, 3, int(rng.integers(0, 30))).tolist()
            assert a.add_cached(nxt, req) == m.add_cached(nxt, req)
            toks[nxt] = req[: m.seq_len(nxt)]
            rest = req[m.seq_len(nxt):]
            try:
                ref = m.append(nxt, len(rest))
                ok = True
            except NoBlocks:
                ok = False
            if ok:
                slots, pairs = a.append(nxt, len(rest))
                assert slots.tolist() == ref[0] and [tuple(p) for p in pairs.tolist()] == ref[1]
                toks[nxt] += rest
            else:
                with pytest.raises(P.NoBlocksError):
                    a.append(nxt, len(rest))
            live.append(nxt)
            nxt += 1
        elif op == 2:
            s = live[int(rng.integers(len(live)))]
            extra = rng.integers(0, 3, int(rng.integers(1, 20))).tolist()
            try:
                ref = m.append(s, len(extra))
                ok = True
            except NoBlocks:
                ok = False
            if ok:
                slots, pairs = a.append(s, len(extra))
                assert slots.tolist() == ref[0] and [tuple(p) for p in pairs.tolist()] == ref[1]
                toks[s] += extra
            else:
                with pytest.raises(P.NoBlocksError):
                    a.append(s, len(extra))
        elif op == 3:
            s = live[int(rng.integers(len(live)))]
            assert a.prefix_insert(s, toks[s]) == m.prefix_insert(s, toks[s])
        elif op == 4 and live:
            s = live.pop(int(rng.integers(len(live))))
            a.free(s)
            m.free_seq(s)
        elif op == 5:
            q = prompts[int(rng.integers(3))][: int(rng.integers(0, 80))] + rng.integers(0, 3, 8).tolist()
            assert a.prefix_match(q) == m.prefix_match(q)
        elif op == 6:
            k = int(rng.integers(0, 20))
            assert a.prefix_evict(k) == m.prefix_evict(k)
        else:
            # fork a live sequence (its cached blocks become shared three ways)
            s = live[int(rng.integers(len(live)))]
            a.fork(s, nxt)
            m.fork(s, nxt)
            toks[nxt] = list(toks[s])
            live.append(nxt)
            nxt += 1
        _same(a, m, live)


def test_shared_system_prompt_is_computed_once():
    """Sixty-four requests with one 200-token system prompt: after the first
    is cached, every later one starts with 12 cached blocks (192 tokens) and
    appends only its own part."""
    a = P.BlockAllocator(2000)
    sys_prompt = list(range(1000, 1200))
    a.add_cached(0, sys_prompt + [1, 2, 3])
    a.append(0, 203)
    assert a.prefix_insert(0, sys_prompt + [1, 2, 3]) == 12
    for r in range(1, 64):
        req = sys_prompt + [r] * 10
        assert a.add_cached(r, req) == 192
        a.append(r, len(req) - 192)
    cached, _, lookups, hits, _ = a.prefix_stats()
    assert cached == 12 and lookups == 64 and hits == 63
    first = a.block_table(0)[:12]
    assert all(a.block_table(r)[:12] == first for r in range(64))
    assert all(a.refcount(b) == 65 for b in first)          # 64 sequences + the cache
