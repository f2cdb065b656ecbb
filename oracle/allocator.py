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
"""


class NoBlocks(Exception):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks, block_size=16, initial_free_order=None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = list(range(num_blocks)) if initial_free_order is None else list(initial_free_order)
        self.rc = [0] * num_blocks
        self.tables = {}
        self.lens = {}

    # -- BlockTable ------------------------------------------------------
    def _allocate(self):
        if not self.free:
            return None
        b = self.free.pop()
        self.rc[b] = 1
        return b

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
        snap = (list(self.free), list(self.rc), list(self.tables[seq]), self.lens[seq])
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
            self.free, self.rc, self.tables[seq], self.lens[seq] = snap
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
