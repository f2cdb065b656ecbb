"""Pure-Python model of the paged KV block manager (oracle; test infrastructure only).

Follows "大模型推理的KV Cache管理从内存碎片到前缀缓存的优化实战" (wmrh.cn), §二:

* BlockTable: the free list starts as range(num_blocks); ``allocate`` pops
  from its end (LIFO) and fails (None) when it is empty; ``free`` pushes a
  block back.  A caller-supplied initial order replaces range(num_blocks).
* PagedKVCache.append_slot: token ``pos`` lives in logical block
  ``pos // block_size``; a physical block is allocated when that logical block
  is not mapped yet; allocation failure reports out-of-memory.
* copy_prefix: a child sequence maps its first ceil(prefix_len / block_size)
  logical blocks to the parent's physical blocks and each shared block's
  reference count grows by one.

Copy-on-write (ascendai.csdn.net article, §二 写时复制; "LLM 推理优化深度解析",
§意外的收获：prefix sharing): shared blocks stay shared until a token is
written into one.  Readings taken where the pages are silent: a fresh block
has reference count 1; writing into a block whose count is > 1 takes a fresh
block, emits the pair (old, new) for a block copy and decrements the old
count; the last holder (count 1) writes in place, so n sharers that all
diverge cause n - 1 copies.  An ``append`` that runs out of blocks leaves the
state exactly as before the call.  Slots are physical * block_size + offset.

Automatic prefix caching (same page, §三 Prefix Caching, AutomaticPrefixCache
and PrefixRadixTree): a radix tree over token ids finds the longest cached
prefix of a request, the hit is rounded down to whole blocks, the cache key
is a 16-byte BLAKE2b digest of the token ids as little-endian int32, and the
least recently used entries are evicted when the cache is over budget.
Readings taken:

* the KV of a cached sequence covers every prefix of it, so each full block
  of an inserted sequence is a tree node whose edge is that block's 16 token
  ids (hits come in whole blocks, as the page's rounding makes them); the
  node's key is the digest of all token ids from the root through it;
* the cache holds one reference on every cached block; a block can be
  evicted only when no sequence holds it (count 1) and no cached block
  below it in the tree remains (leaves first);
* "least recently used" follows a logical clock that ticks once per cache
  call (insert, match, add-from-cache); ties go to the node created first;
* when an allocation finds the free list empty it evicts one block that way
  (and fails only if none is evictable); a failed append restores the whole
  prior state, evicted cache entries included.
"""
import copy
import hashlib
import struct


class NoBlocks(Exception):
    pass


def prefix_key(tokens):
    """BLAKE2b, 16-byte digest, of token ids packed as little-endian int32."""
    h = hashlib.blake2b(digest_size=16)
    h.update(struct.pack("<%di" % len(tokens), *tokens))
    return h.digest()


class BlockManagerModel:
    def __init__(self, num_blocks, block_size=16, initial_free_order=None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = list(range(num_blocks)) if initial_free_order is None else list(initial_free_order)
        self.rc = [0] * num_blocks
        self.tables = {}
        self.lens = {}
        # prefix cache: node id -> dict(parent, chunk, block, key, last, order, children)
        self.nodes = {0: dict(parent=None, chunk=None, block=None, key=b"", last=0, order=0, children={})}
        self.clock = 0
        self.next_order = 1
        self.lookups = self.hits = self.evictions = 0

    # -- BlockTable ------------------------------------------------------
    def _allocate(self):
        if not self.free and not self._evict_one():
            return None
        b = self.free.pop()
        self.rc[b] = 1
        return b

    # -- prefix cache ------------------------------------------------------
    def _evictable(self):
        return [(n["last"], n["order"], i) for i, n in self.nodes.items()
                if i != 0 and not n["children"] and self.rc[n["block"]] == 1]

    def _evict_one(self):
        cand = self._evictable()
        if not cand:
            return False
        _, _, i = min(cand)
        n = self.nodes.pop(i)
        del self.nodes[n["parent"]]["children"][n["chunk"]]
        self.rc[n["block"]] = 0
        self.free.append(n["block"])
        self.evictions += 1
        return True

    def _walk(self, tokens):
        """Nodes of the longest cached whole-block prefix of tokens."""
        bs = self.block_size
        path, cur = [], 0
        for i in range(len(tokens) // bs):
            nxt = self.nodes[cur]["children"].get(tuple(tokens[i * bs:(i + 1) * bs]))
            if nxt is None:
                break
            path.append(nxt)
            cur = nxt
        return path

    def prefix_match(self, tokens):
        """(hit tokens, key of the hit prefix or 16 zero bytes)."""
        self.clock += 1
        path = self._walk(tokens)
        for i in path:
            self.nodes[i]["last"] = self.clock
        self.lookups += 1
        if path:
            self.hits += 1
        hit = len(path) * self.block_size
        return hit, (self.nodes[path[-1]]["key"] if path else bytes(16))

    def add_cached(self, seq, tokens):
        """New sequence starting with the blocks of its longest cached prefix."""
        if seq in self.tables:
            raise KeyError(seq)
        hit, _ = self.prefix_match(tokens)
        path = self._walk(tokens)
        blocks = [self.nodes[i]["block"] for i in path]
        for b in blocks:
            self.rc[b] += 1
        self.tables[seq] = blocks
        self.lens[seq] = hit
        return hit

    def prefix_insert(self, seq, tokens):
        """Caches the sequence's first len(tokens) // bs blocks under the token
        prefix; returns how many blocks became newly cached."""
        bs = self.block_size
        n = min(len(tokens), self.lens[seq]) // bs
        self.clock += 1
        cur, new = 0, 0
        for i in range(n):
            chunk = tuple(tokens[i * bs:(i + 1) * bs])
            nxt = self.nodes[cur]["children"].get(chunk)
            if nxt is None:
                b = self.tables[seq][i]
                nxt = max(self.nodes) + 1
                self.nodes[nxt] = dict(parent=cur, chunk=chunk, block=b, key=prefix_key(tokens[:(i + 1) * bs]),
                                       last=self.clock, order=self.next_order, children={})
                self.next_order += 1
                self.nodes[cur]["children"][chunk] = nxt
                self.rc[b] += 1
                new += 1
            else:
                self.nodes[nxt]["last"] = self.clock
            cur = nxt
        return new

    def prefix_evict(self, max_cached_blocks):
        """Evicts LRU evictable blocks until at most max_cached_blocks stay
        cached (or none is evictable); returns how many were evicted."""
        k = 0
        while len(self.nodes) - 1 > max_cached_blocks and self._evict_one():
            k += 1
        return k

    def prefix_stats(self):
        """(cached blocks, evictable now, lookups, hits, evictions)."""
        return len(self.nodes) - 1, len(self._evictable()), self.lookups, self.hits, self.evictions

    # -- sequences -------------------------------------------------------
    def add(self, seq):
        if seq in self.tables:
            raise KeyError(seq)
        self.tables[seq] = []
        self.lens[seq] = 0

    def fork(self, parent, child, prefix_len=None):
        if child in self.tables or parent not in self.tables:
            raise KeyError(child)
        plen = self.lens[parent] if prefix_len is None else prefix_len
        if plen > self.lens[parent]:
            raise ValueError("prefix longer than parent")
        nb = (plen + self.block_size - 1) // self.block_size
        shared = self.tables[parent][:nb]
        for b in shared:
            self.rc[b] += 1
        self.tables[child] = list(shared)
        self.lens[child] = plen

    def append(self, seq, n_tokens):
        """Returns (slots, cow_pairs); raises NoBlocks with the state unchanged."""
        snap = (list(self.free), list(self.rc), list(self.tables[seq]), self.lens[seq], copy.deepcopy(self.nodes),
                self.evictions)
        slots, pairs = [], []
        bs = self.block_size
        try:
            table = self.tables[seq]
            for _ in range(n_tokens):
                pos = self.lens[seq]
                lb = pos // bs
                if pos % bs == 0:
                    b = self._allocate()
                    if b is None:
                        raise NoBlocks()
                    table.append(b)
                else:
                    old = table[lb]
                    if self.rc[old] > 1:
                        b = self._allocate()
                        if b is None:
                            raise NoBlocks()
                        self.rc[old] -= 1
                        table[lb] = b
                        pairs.append((old, b))
                slots.append(table[lb] * bs + pos % bs)
                self.lens[seq] = pos + 1
        except NoBlocks:
            self.free, self.rc, self.tables[seq], self.lens[seq], self.nodes, self.evictions = snap
            raise
        return slots, pairs

    def free_seq(self, seq):
        for b in self.tables.pop(seq):
            self.rc[b] -= 1
            if self.rc[b] == 0:
                self.free.append(b)
        del self.lens[seq]

    # -- queries -----------------------------------------------------------
    def block_table(self, seq):
        return list(self.tables[seq])

    def seq_len(self, seq):
        return self.lens[seq]

    def refcount(self, block):
        return self.rc[block]

    def stats(self):
        """(num_free, num_shared, largest run of consecutive free block ids).

        The page's fragmentation indicator is total free / largest contiguous
        free run ("大模型推理的KV Cache管理…优化实战", §三 metrics table)."""
        free = set(self.free)
        best = run = 0
        for b in range(self.num_blocks):
            run = run + 1 if b in free else 0
            best = max(best, run)
        shared = sum(1 for r in self.rc if r > 1)
        return len(self.free), shared, best
