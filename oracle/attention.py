"""Single-query paged decode attention in fp64 (oracle; test infrastructure only).

The method: each decode step feeds one token per sequence; its query attends
to every cached key/value of that sequence ("LLM 推理优化深度解析", §KV Cache
的本质, the decode loop).  The cache is stored in fixed-size physical blocks
and a per-sequence block table maps logical block j to a physical block
(same page, §PagedAttention：vLLM 的显存碎片治理; ascendai.csdn.net article,
§二 核心突破 Fig. 2).  Paged storage changes where the bytes live, not the
result, so the oracle is the plain definition written out:

1. gather: K_s[j] = k_cache[block_table[s][j // bs], :, j % bs, :] for j < ctx_s
   (and V likewise), converted to fp64; quantised caches are dequantised as
   code * scale of that (block, head, slot), or (code - zero_point) * scale
   for the asymmetric uint8 format ("大模型推理的KV Cache管理…优化实战", §四
   dequantize_key);
2. attend: for query head i with KV head h = i // G (consecutive grouping,
   "LLM 推理优化深度解析", §MQA 与 GQA), logits = scale * K_s[:, h] @ q[s, i],
   p = softmax(logits), out[s, i] = p @ V_s[:, h].

A sequence with ctx = 0 yields a zero output row.

Sliding window ("KV Cache 与 PagedAttention", §三个直接推论, the KV-saving
table: keep only the most recent window): with window W > 0 a query at
position P sees keys max(0, P - W + 1) .. P only (W = 0: no window).
"""
import numpy as np


def gather_sequence(cache, block_table, ctx, scale=None, zero=None):
    """Logically contiguous [ctx, H, D] fp64 copy of one sequence's K or V.

    cache: [NB, H, bs, D] array of values (fp64-convertible) or of codes when
    ``scale`` ([NB, H, bs]) is given, with zero points ``zero`` ([NB, H, bs])
    for the asymmetric format; block_table: 1-D int array.
    """
    bs = cache.shape[2]
    j = np.arange(ctx)
    blocks = np.asarray(block_table)[j // bs]
    offs = j % bs
    rows = cache[blocks, :, offs, :].astype(np.float64)          # [ctx, H, D]
    if zero is not None:
        rows = rows - zero[blocks, :, offs].astype(np.float64)[:, :, None]
    if scale is not None:
        rows = rows * scale[blocks, :, offs].astype(np.float64)[:, :, None]
    return rows


def contiguous_attention(q, K, V, scale):
    """Attention of one sequence's queries over contiguous K/V.

    q: [Hq, D]; K, V: [ctx, Hkv, D]; returns [Hq, D] fp64.
    """
    q = np.asarray(q, np.float64)
    Hq, D = q.shape
    ctx, Hkv, _ = K.shape
    out = np.zeros((Hq, D), np.float64)
    if ctx == 0:
        return out
    G = Hq // Hkv
    for i in range(Hq):
        h = i // G
        logits = scale * (K[:, h, :] @ q[i])
        p = np.exp(logits - logits.max())
        p /= p.sum()
        out[i] = p @ V[:, h, :]
    return out


def _window_start(vis, window):
    """First visible key of a query that sees keys < vis, under window W."""
    return max(0, vis - window) if window > 0 else 0


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale,
                           k_scale=None, v_scale=None, seqs=None, k_zero=None, v_zero=None, window=0):
    """Decode attention for every (or the listed) sequence of a batch.

    q: [B, Hq, D]; k_cache, v_cache: [NB, Hkv, bs, D] (values, or codes with
    k_scale / v_scale [NB, Hkv, bs] and, for the asymmetric format, zero
    points k_zero / v_zero [NB, Hkv, bs]); block_tables: [B, MB];
    context_lens: [B].
    Returns [B, Hq, D] fp64 (rows of sequences not in ``seqs`` stay zero).
    """
    q = np.asarray(q, np.float64)
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D), np.float64)
    for s in (range(B) if seqs is None else seqs):
        ctx = int(context_lens[s])
        K = gather_sequence(k_cache, block_tables[s], ctx, k_scale, k_zero)
        V = gather_sequence(v_cache, block_tables[s], ctx, v_scale, v_zero)
        lo = _window_start(ctx, window)
        out[s] = contiguous_attention(q[s], K[lo:], V[lo:], scale)
    return out


def paged_decode_attention_heads(q, k_cache, v_cache, block_tables, context_lens, scale,
                                 pairs, k_scale=None, v_scale=None, k_zero=None, v_zero=None):
    """Oracle output for a sample of (sequence, query head) pairs only.

    Used at full workload sizes where the whole batch would take too long;
    returns an array [len(pairs), D] fp64 in the order of ``pairs``.
    """
    q = np.asarray(q, np.float64)
    _, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.zeros((len(pairs), D), np.float64)
    cache = {}
    for n, (s, i) in enumerate(pairs):
        ctx = int(context_lens[s])
        if ctx == 0:
            continue
        h = i // G
        key = (s, h)
        if key not in cache:
            cache.clear()
            bt = block_tables[s]
            K = gather_sequence(k_cache[:, h:h + 1], bt, ctx,
                                None if k_scale is None else k_scale[:, h:h + 1],
                                None if k_zero is None else k_zero[:, h:h + 1])
            V = gather_sequence(v_cache[:, h:h + 1], bt, ctx,
                                None if v_scale is None else v_scale[:, h:h + 1],
                                None if v_zero is None else v_zero[:, h:h + 1])
            cache[key] = (K[:, 0, :], V[:, 0, :])
        K, V = cache[key]
        logits = scale * (K @ q[s, i])
        p = np.exp(logits - logits.max())
        p /= p.sum()
        out[n] = p @ V
    return out


def paged_multi_query_attention(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
                                k_scale=None, v_scale=None, k_zero=None, v_zero=None, window=0):
    """Attention of several new tokens per sequence over the paged cache.

    Several query tokens of one sequence in one pass serve chunked prefill
    (a long prompt cut into chunks interleaved with decode steps, "LLM 推理
    优化深度解析", §Continuous Batching and §调优心法) and the verify pass of
    speculative decoding (one forward of the large model scores the k drafted
    positions at once, same page, §投机解码).  Reading taken: the n_s new
    tokens of sequence s are the last n_s of its context_lens[s] tokens, their
    K/V already in the cache; new token t (0-based) sits at position
    ctx_s - n_s + t and attends keys 0 .. ctx_s - n_s + t (causal among the
    new tokens, everything before them visible).

    q: [T, Hq, D] packed by sequence, rows query_start_loc[s] ..
    query_start_loc[s + 1] - 1 belonging to sequence s (query_start_loc
    [B + 1], non-decreasing, starting at 0); returns [T, Hq, D] fp64.
    """
    q = np.asarray(q, np.float64)
    T, Hq, D = q.shape
    out = np.zeros((T, Hq, D), np.float64)
    qsl = np.asarray(query_start_loc).tolist()
    for s in range(len(qsl) - 1):
        n = qsl[s + 1] - qsl[s]
        if n == 0:
            continue
        ctx = int(context_lens[s])
        if n > ctx:
            raise ValueError("a sequence has more new tokens than context")
        K = gather_sequence(k_cache, block_tables[s], ctx, k_scale, k_zero)
        V = gather_sequence(v_cache, block_tables[s], ctx, v_scale, v_zero)
        for t in range(n):
            vis = ctx - n + t + 1
            lo = _window_start(vis, window)
            out[qsl[s] + t] = contiguous_attention(q[qsl[s] + t], K[lo:vis], V[lo:vis], scale)
    return out
