"""Pins for the oracle's KV-size arithmetic and decode attention.

Each test ties the oracle to something other than itself: numbers printed on
the pages (tests/golden), closed forms, invariants the method states, a
brute-force loop written independently, or torch's own attention routine.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import kv_size as K

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- KV size --

def test_worked_example_llama2_7b_4k():
    g = _golden("kv_size_worked_example.json")
    got = K.kv_cache_bytes(g["n_layers"], g["n_kv_heads"], g["head_dim"], g["seq_len"],
                           g["batch"], g["bytes_per_elt"])
    assert got == g["kv_bytes"]


def test_worked_example_batch16_is_32gb():
    g = _golden("kv_size_worked_example.json")
    got = K.kv_cache_bytes(g["n_layers"], g["n_kv_heads"], g["head_dim"], g["seq_len"],
                           g["batch16"], g["bytes_per_elt"])
    assert got == g["batch16_kv_gb_printed"] * 2 ** 30


def test_per_token_per_layer_form_reproduces_the_worked_example():
    # "KV Cache 与 PagedAttention" (ai-infra-wiki) §KV cache 有多大: one token adds
    # 2 x n_kv x head_dim x 2 bytes to one layer (16-bit values); times the
    # layers and tokens of the worked example it must give the printed total
    g = _golden("kv_size_worked_example.json")
    per = K.kv_bytes_per_token_per_layer(g["n_kv_heads"], g["head_dim"], g["bytes_per_elt"])
    assert per == 2 * 32 * 128 * 2
    assert per * g["n_layers"] * g["seq_len"] * g["batch"] == g["kv_bytes"]
    # and it agrees with the product form for other shapes and element sizes
    for L, H, D, S, B, e in [(80, 8, 128, 32768, 1, 2), (32, 8, 128, 4096, 64, 1), (1, 1, 64, 1, 1, 4)]:
        assert K.kv_cache_bytes(L, H, D, S, B, e) == L * S * B * K.kv_bytes_per_token_per_layer(H, D, e)


def test_decode_bound_about_140():
    g = _golden("decode_bound.json")
    v = K.decode_tokens_per_s_bound(g["bandwidth_gb_s"], g["weights_gb"])
    assert abs(v - g["printed_tokens_per_s_approx"]) < 5


def test_paged_waste_below_one_block():
    # "at most one block is wasted per sequence" (LLM 推理优化深度解析, §PagedAttention table)
    for n in range(0, 2000):
        w = K.paged_waste_tokens(n)
        assert 0 <= w < 16
        assert K.paged_blocks_needed(n) * 16 >= n


def test_gqa_shrinks_kv_by_group_factor():
    # 32 q heads over 8 KV heads cut the cache 4x (LLM 推理优化深度解析, §MQA 与 GQA)
    mha = K.kv_cache_bytes(32, 32, 128, 4096)
    gqa = K.kv_cache_bytes(32, 8, 128, 4096)
    mqa = K.kv_cache_bytes(32, 1, 128, 4096)
    assert mha == 4 * gqa and mha == 32 * mqa


# ------------------------------------------------------------- attention --

def _scatter(K_log, perm_blocks, bs=16):
    """Place logical [ctx, H, D] rows into a pool so that logical block j lives
    in physical block perm_blocks[j] (test-side helper)."""
    ctx, H, D = K_log.shape
    nb = int(max(perm_blocks)) + 1
    pool = np.full((nb, H, bs, D), np.nan)
    for j in range(ctx):
        pool[perm_blocks[j // bs], :, j % bs, :] = K_log[j]
    return pool


def _brute(q, K_log, V_log, scale):
    """Triple loop with math.exp, no numpy reductions."""
    Hq, D = len(q), len(q[0])
    ctx, Hkv = len(K_log), len(K_log[0])
    G = Hq // Hkv
    out = []
    for i in range(Hq):
        h = i // G
        logits = []
        for j in range(ctx):
            acc = 0.0
            for d in range(D):
                acc += q[i][d] * K_log[j][h][d]
            logits.append(scale * acc)
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        tot = sum(w)
        row = []
        for d in range(D):
            acc = 0.0
            for j in range(ctx):
                acc += w[j] / tot * V_log[j][h][d]
            row.append(acc)
        out.append(row)
    return np.array(out)


@pytest.mark.parametrize("ctx,hq,hkv,d", [(1, 2, 1, 4), (15, 4, 2, 8), (16, 2, 2, 8),
                                          (17, 4, 1, 8), (40, 8, 2, 4)])
def test_paged_equals_contiguous_bitwise(ctx, hq, hkv, d):
    rng = np.random.default_rng(ctx * 100 + hq)
    K_log = rng.standard_normal((ctx, hkv, d))
    V_log = rng.standard_normal((ctx, hkv, d))
    q = rng.standard_normal((1, hq, d))
    nblk = (ctx + 15) // 16
    perm = rng.permutation(nblk + 3)[:nblk]
    kc, vc = _scatter(K_log, perm), _scatter(V_log, perm)
    bt = np.array([perm])
    paged = A.paged_decode_attention(q, kc, vc, bt, [ctx], 0.3)
    contig = A.contiguous_attention(q[0], K_log, V_log, 0.3)
    assert np.array_equal(paged[0], contig)


def test_block_permutation_invariance():
    rng = np.random.default_rng(7)
    nb, hkv, d, hq = 12, 2, 8, 4
    kc = rng.standard_normal((nb, hkv, 16, d))
    vc = rng.standard_normal((nb, hkv, 16, d))
    q = rng.standard_normal((2, hq, d))
    bt = np.array([[3, 7, 1, 0], [5, 2, 9, 11]])
    ctx = [50, 61]
    ref = A.paged_decode_attention(q, kc, vc, bt, ctx, 0.5)
    perm = rng.permutation(nb)            # new physical position of old block b is perm[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    got = A.paged_decode_attention(q, kc2, vc2, perm[bt], ctx, 0.5)
    assert np.array_equal(ref, got)


@pytest.mark.parametrize("ctx,hq,hkv,d", [(1, 2, 2, 3), (7, 4, 2, 8), (16, 2, 1, 4),
                                          (33, 6, 3, 5), (40, 8, 8, 2)])
def test_against_brute_force(ctx, hq, hkv, d):
    rng = np.random.default_rng(1 + ctx + d)
    K_log = rng.standard_normal((ctx, hkv, d))
    V_log = rng.standard_normal((ctx, hkv, d))
    q = rng.standard_normal((hq, d))
    nblk = (ctx + 15) // 16
    perm = rng.permutation(nblk)
    got = A.paged_decode_attention(q[None], _scatter(K_log, perm), _scatter(V_log, perm),
                                   np.array([perm]), [ctx], 0.7)[0]
    ref = _brute(q.tolist(), K_log.tolist(), V_log.tolist(), 0.7)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 2), (4, 1)])
def test_against_torch_sdpa(hq, hkv):
    ctx, d = 100, 16
    g = torch.Generator().manual_seed(11)
    K_log = torch.randn(ctx, hkv, d, generator=g, dtype=torch.float64)
    V_log = torch.randn(ctx, hkv, d, generator=g, dtype=torch.float64)
    q = torch.randn(hq, d, generator=g, dtype=torch.float64)
    scale = 1 / math.sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], K_log.permute(1, 0, 2), V_log.permute(1, 0, 2),
        scale=scale, enable_gqa=True)[:, 0, :]
    perm = np.arange(7)[::-1]
    got = A.paged_decode_attention(q.numpy()[None], _scatter(K_log.numpy(), perm),
                                   _scatter(V_log.numpy(), perm), np.array([perm]), [ctx], scale)[0]
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_ctx1_returns_v0_exactly():
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((4, 2, 16, 8))
    vc = rng.standard_normal((4, 2, 16, 8))
    q = rng.standard_normal((1, 4, 8)) * 100
    out = A.paged_decode_attention(q, kc, vc, np.array([[2]]), [1], 1.0)
    assert np.array_equal(out[0, 0], vc[2, 0, 0]) and np.array_equal(out[0, 3], vc[2, 1, 0])


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(4)
    kc = np.broadcast_to(rng.standard_normal((1, 1, 1, 8)), (3, 1, 16, 8)).copy()
    vc = rng.standard_normal((3, 1, 16, 8))
    q = rng.standard_normal((1, 2, 8))
    ctx = 37
    out = A.paged_decode_attention(q, kc, vc, np.array([[1, 0, 2]]), [ctx], 0.9)
    V = np.concatenate([vc[1, 0], vc[0, 0], vc[2, 0]])[:ctx]
    np.testing.assert_allclose(out[0, 0], V.mean(0), atol=1e-14)


def test_one_hot_query_large_scale_selects_argmax_key():
    rng = np.random.default_rng(5)
    kc = rng.standard_normal((2, 1, 16, 8))
    vc = rng.standard_normal((2, 1, 16, 8))
    q = np.zeros((1, 1, 8))
    q[0, 0, 3] = 1.0
    out = A.paged_decode_attention(q, kc, vc, np.array([[1, 0]]), [32], 1e4)
    K_log = np.concatenate([kc[1, 0], kc[0, 0]])
    V_log = np.concatenate([vc[1, 0], vc[0, 0]])
    np.testing.assert_allclose(out[0, 0], V_log[np.argmax(K_log[:, 3])], atol=1e-9)


def test_ctx0_gives_zero_row():
    kc = np.ones((2, 1, 16, 4))
    out = A.paged_decode_attention(np.ones((2, 1, 4)), kc, kc, np.array([[0], [1]]), [0, 3], 1.0)
    assert np.all(out[0] == 0) and np.allclose(out[1], 1.0)


def test_dequantised_gather_matches_scaled_codes():
    rng = np.random.default_rng(6)
    codes = rng.integers(-127, 128, size=(3, 2, 16, 4)).astype(np.int8)
    sc = rng.random((3, 2, 16)).astype(np.float32)
    K_log = A.gather_sequence(codes, [2, 0], 20, sc)
    for j in range(20):
        b = [2, 0][j // 16]
        for h in range(2):
            assert np.array_equal(K_log[j, h], codes[b, h, j % 16].astype(np.float64) * np.float64(sc[b, h, j % 16]))


def test_head_sample_matches_full_oracle():
    rng = np.random.default_rng(8)
    kc = rng.standard_normal((10, 2, 16, 8))
    vc = rng.standard_normal((10, 2, 16, 8))
    q = rng.standard_normal((3, 4, 8))
    bt = np.array([[0, 1, 2], [3, 4, 5], [9, 8, 7]])
    ctx = [33, 48, 5]
    full = A.paged_decode_attention(q, kc, vc, bt, ctx, 0.4)
    pairs = [(0, 0), (2, 3), (1, 2), (1, 1)]
    part = A.paged_decode_attention_heads(q, kc, vc, bt, ctx, 0.4, pairs)
    for n, (s, i) in enumerate(pairs):
        np.testing.assert_allclose(part[n], full[s, i], rtol=0, atol=1e-14)


def test_asymmetric_gather_subtracts_zero_point_then_scales():
    # an integer-grid cache stored as (code, scale 2^-k, zero point) must give
    # back the grid values, and paged attention over it must equal contiguous
    # attention over those values (a sign or order slip in the zero point fails)
    rng = np.random.default_rng(9)
    ctx, hkv, hq, d = 37, 2, 4, 8
    zp = rng.integers(20, 236, size=(ctx, hkv))
    codes_log = rng.integers(0, 256, size=(ctx, hkv, d))
    sc = np.exp2(-rng.integers(2, 6, size=(ctx, hkv))).astype(np.float32)
    vals = (codes_log - zp[:, :, None]) * sc.astype(np.float64)[:, :, None]
    nblk = (ctx + 15) // 16
    perm = rng.permutation(nblk + 2)[:nblk]
    nb = nblk + 2
    kc = np.zeros((nb, hkv, 16, d), np.uint8)
    kz = np.zeros((nb, hkv, 16), np.uint8)
    ks = np.zeros((nb, hkv, 16), np.float32)
    for j in range(ctx):
        kc[perm[j // 16], :, j % 16] = codes_log[j]
        kz[perm[j // 16], :, j % 16] = zp[j]
        ks[perm[j // 16], :, j % 16] = sc[j]
    got = A.gather_sequence(kc, perm, ctx, ks, kz)
    assert np.array_equal(got, vals)
    q = rng.standard_normal((1, hq, d))
    paged = A.paged_decode_attention(q, kc, kc, np.array([perm]), [ctx], 0.5, ks, ks, k_zero=kz, v_zero=kz)
    np.testing.assert_allclose(paged[0], _brute(q[0], vals, vals, 0.5), rtol=0, atol=1e-12)


# ---------------------------------------------------------- multi-query --

def _mq_case(rng, ctxs, nq, hq, hkv, d, spare=3):
    nblk = [(c + 15) // 16 for c in ctxs]
    nb = sum(nblk) + spare
    perm = rng.permutation(nb)
    bt = np.zeros((len(ctxs), max(nblk)), np.int64)
    cur = 0
    for s, k in enumerate(nblk):
        bt[s, :k] = perm[cur:cur + k]
        cur += k
    kc = rng.standard_normal((nb, hkv, 16, d))
    vc = rng.standard_normal((nb, hkv, 16, d))
    qsl = np.concatenate([[0], np.cumsum(nq)])
    q = rng.standard_normal((int(qsl[-1]), hq, d))
    return q, kc, vc, bt, qsl


def test_multi_query_with_one_token_is_decode_bitwise():
    rng = np.random.default_rng(21)
    ctxs = [1, 17, 40, 33]
    q, kc, vc, bt, qsl = _mq_case(rng, ctxs, [1, 1, 1, 1], 8, 2, 8)
    mq = A.paged_multi_query_attention(q, kc, vc, bt, ctxs, qsl, 0.37)
    dec = A.paged_decode_attention(q, kc, vc, bt, ctxs, 0.37)
    assert np.array_equal(mq, dec)


def test_multi_query_full_prefill_matches_sdpa_causal():
    # all of a sequence's tokens new at once: plain causal self-attention
    rng = np.random.default_rng(22)
    ctx, hq, hkv, d = 45, 8, 2, 16
    q, kc, vc, bt, qsl = _mq_case(rng, [ctx], [ctx], hq, hkv, d)
    got = A.paged_multi_query_attention(q, kc, vc, bt, [ctx], qsl, 0.25)
    K = torch.from_numpy(np.stack([kc[bt[0, j // 16], :, j % 16] for j in range(ctx)]))   # [ctx, hkv, d]
    V = torch.from_numpy(np.stack([vc[bt[0, j // 16], :, j % 16] for j in range(ctx)]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(0, 1), K.transpose(0, 1), V.transpose(0, 1), is_causal=True, scale=0.25,
        enable_gqa=True).transpose(0, 1).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_multi_query_is_independent_of_chunking():
    # the output for a token does not depend on how the new tokens are split
    # into passes: one pass of 12 tokens == three passes of 5, 4 and 3 tokens
    # (each pass seeing the context up to its own last token), == 12 decodes
    rng = np.random.default_rng(23)
    ctx, n, hq, hkv, d = 70, 12, 4, 4, 8
    q, kc, vc, bt, _ = _mq_case(rng, [ctx], [n], hq, hkv, d)
    one = A.paged_multi_query_attention(q, kc, vc, bt, [ctx], [0, n], 0.5)
    parts, start = [], 0
    for m in (5, 4, 3):
        c = ctx - n + start + m
        parts.append(A.paged_multi_query_attention(q[start:start + m], kc, vc, bt, [c], [0, m], 0.5))
        start += m
    assert np.array_equal(np.concatenate(parts), one)
    for t in range(n):
        dec = A.paged_decode_attention(q[t:t + 1], kc, vc, bt, [ctx - n + t + 1], 0.5)[0]
        assert np.array_equal(dec, one[t])


def test_multi_query_brute_force_and_empty_sequences():
    rng = np.random.default_rng(24)
    ctxs = [20, 0, 9, 33]
    nq = [3, 0, 9, 2]
    hq, hkv, d = 4, 2, 4
    q, kc, vc, bt, qsl = _mq_case(rng, [max(c, 1) for c in ctxs], nq, hq, hkv, d)
    got = A.paged_multi_query_attention(q, kc, vc, bt, ctxs, qsl, 0.6)
    for s, (c, n) in enumerate(zip(ctxs, nq)):
        K_log = [[kc[bt[s, j // 16], h, j % 16] for h in range(hkv)] for j in range(c)]
        V_log = [[vc[bt[s, j // 16], h, j % 16] for h in range(hkv)] for j in range(c)]
        for t in range(n):
            vis = c - n + t + 1
            ref = _brute(q[qsl[s] + t], K_log[:vis], V_log[:vis], 0.6)
            np.testing.assert_allclose(got[qsl[s] + t], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------- sliding window --

def test_window_covering_the_context_changes_nothing():
    rng = np.random.default_rng(31)
    ctxs = [5, 40, 17]
    q, kc, vc, bt, qsl = _mq_case(rng, ctxs, [2, 7, 1], 4, 2, 8)
    full = A.paged_multi_query_attention(q, kc, vc, bt, ctxs, qsl, 0.4)
    assert np.array_equal(A.paged_multi_query_attention(q, kc, vc, bt, ctxs, qsl, 0.4, window=40), full)
    dq = rng.standard_normal((3, 4, 8))
    assert np.array_equal(A.paged_decode_attention(dq, kc, vc, bt, ctxs, 0.4, window=10 ** 6),
                          A.paged_decode_attention(dq, kc, vc, bt, ctxs, 0.4))


def test_window_of_one_returns_the_own_value_row():
    rng = np.random.default_rng(32)
    ctxs = [33, 18]
    q, kc, vc, bt, qsl = _mq_case(rng, ctxs, [3, 18], 4, 2, 8)
    got = A.paged_multi_query_attention(q, kc, vc, bt, ctxs, qsl, 0.4, window=1)
    for s, (c, n) in enumerate(zip(ctxs, [3, 18])):
        for t in range(n):
            pos = c - n + t
            v = vc[bt[s, pos // 16], :, pos % 16]                 # [hkv, d]
            assert np.array_equal(got[qsl[s] + t], np.repeat(v, 2, axis=0))


def test_window_brute_force():
    rng = np.random.default_rng(33)
    ctxs = [50, 9]
    nq = [6, 9]
    q, kc, vc, bt, qsl = _mq_case(rng, ctxs, nq, 4, 2, 4)
    W = 13
    got = A.paged_multi_query_attention(q, kc, vc, bt, ctxs, qsl, 0.7, window=W)
    for s, (c, n) in enumerate(zip(ctxs, nq)):
        K_log = [[kc[bt[s, j // 16], h, j % 16] for h in range(2)] for j in range(c)]
        V_log = [[vc[bt[s, j // 16], h, j % 16] for h in range(2)] for j in range(c)]
        for t in range(n):
            pos = c - n + t
            keep = [j for j in range(c) if pos - W < j <= pos]
            ref = _brute(q[qsl[s] + t], [K_log[j] for j in keep], [V_log[j] for j in keep], 0.7)
            np.testing.assert_allclose(got[qsl[s] + t], ref, rtol=0, atol=1e-12)
