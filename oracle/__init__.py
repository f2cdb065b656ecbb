"""Plain, slow, fp64 CPU oracle for paged KV-cache decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no common kernels, headers, helpers or tables)
and imports nothing from ``paged_kv_cache_438_b200``.

What it computes, and the passages it follows (pages are named by title):

* ``kv_size``    -- the KV-cache size formula and its worked example
  ("LLM 推理优化深度解析", §KV Cache 的本质; "KV Cache 与 PagedAttention",
  §KV cache 有多大).
* ``attention``  -- single-query decode attention over a block-table-indexed
  cache: gather each sequence's K/V through its block table into a logically
  contiguous array, then softmax(scale * K q) V, all in fp64
  ("LLM 推理优化深度解析", §KV Cache 的本质 and §PagedAttention; the
  ascendai.csdn.net article, §二 核心突破 Fig. 2).
* ``quant``      -- the per-token-per-head absmax INT8 / FP8-e4m3 quantising
  rule with its own e4m3 encoder / decoder (OCP FP8 E4M3 definition), and
  the asymmetric min/max uint8 rule with a zero point and its 128-token
  grouped form ("大模型推理的KV Cache管理…优化实战", §四).
* ``cache_ops``  -- the slot-mapped KV write (logical block = token // 16) and
  the block copy behind copy-on-write.
* ``allocator``  -- a pure-Python free-list / refcount / fork / copy-on-write
  model of the block manager ("大模型推理的KV Cache管理…优化实战", §二
  class BlockTable, append_slot, copy_prefix).

Every function is pinned by tests in ``tests/test_oracle_*.py`` against facts
the pages or the mathematics fix (printed arithmetic, closed forms,
invariants, brute force on tiny inputs, library routines); none is
"parity unpinned".
"""
