"""Slot-mapped KV write and block copy (oracle; test infrastructure only).

Write: the page "大模型推理的KV Cache管理…优化实战" §二 (PagedKVCache.append_slot)
places token ``token_idx`` in logical block ``token_idx // block_size``; the
caller turns (physical block, offset) into one flat slot number
slot = physical * block_size + offset, so token t's K (and V) for KV head h
lands at cache[slot // bs, h, slot % bs, :].  A slot of -1 means "skip".

Copy: copy-on-write lets branches share blocks until a new token is written,
and only then is a block copied (ascendai.csdn.net article, §二 写时复制;
"LLM 推理优化深度解析", §意外的收获：prefix sharing).  ``copy_blocks`` gives
every (src, dst) pair dst := src for K, V and (for quantised caches) the
scales, all pairs reading the state before the call.
"""
import numpy as np


def kv_write(cache, x, slot_mapping):
    """Return a copy of ``cache`` [NB, H, bs, D] with rows of x [T, H, D]
    scattered by slot.  Works on any dtype (raw bit views included)."""
    out = np.array(cache, copy=True)
    bs = out.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        out[slot // bs, :, slot % bs, :] = x[t]
    return out


def scale_write(scale, s, slot_mapping):
    """Scatter per-(token, head) scales s [T, H] into scale [NB, H, bs]."""
    out = np.array(scale, copy=True)
    bs = out.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        out[slot // bs, :, slot % bs] = s[t]
    return out


def copy_blocks(arrays, pairs):
    """Apply dst := src for every (src, dst) in ``pairs`` to each array in
    ``arrays`` (indexed by physical block on axis 0), reading the pre-call
    state.  Returns new arrays."""
    out = []
    for a in arrays:
        before = np.array(a, copy=True)
        after = np.array(a, copy=True)
        for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
            after[dst] = before[src]
        out.append(after)
    return out
