"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Bars: writes, block copies and quantisation are bit-exact; attention is within
max-abs 2e-2 and mean-rel 1e-2 (sum |gpu - ref| / sum |ref|) for fp16 / bf16
caches, and within 6e-2 max-abs of the oracle on the unquantised values for
INT8 / FP8 / asymmetric uint8 caches (2.5e-1 for the 4-bit formats, whose own
rounding error against unquantised attention reaches about 0.1 on these
mixes); every quantised format is also held to the 16-bit bars against the
oracle on its stored codes.  Inputs come from the seeded generators in
paged_kv_cache_438_b200.inputs; nothing the oracle sees is produced by the
library's kernels.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache_ops as OC
from oracle import quant as OQ
from oracle.allocator import BlockManagerModel
from paged_kv_cache_438_b200 import inputs as I
from paged_kv_cache_438_b200 import pagedkv as P

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
ATOL, MEANREL, QATOL, Q4ATOL = 2e-2, 1e-2, 6e-2, 2.5e-1
FOUR_BIT = ("int4", "fp4")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_kv_cache_438_b200 import build
    build.build()
    P.lib()
    P.device_status(clear=True)
    yield
    assert P.device_status(clear=True) == 0, "a kernel raised a device status bit"


# ----------------------------------------------------------------- helpers --

def np64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def bits(t):
    """Raw bits of a tensor as a numpy integer array."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    return t.numpy()


def cache_values(t, kind):
    """Cache contents as the oracle reads them: fp64 values, or fp64 codes
    (decoded by the oracle's own e4m3 decoder for FP8)."""
    if kind == "fp8":
        return OQ.e4m3_decode(t.detach().cpu().contiguous().view(torch.uint8).numpy())
    if kind in ("int8", "u8asym"):
        return t.detach().cpu().numpy().astype(np.float64)
    if kind == "int4":
        return OQ.int4_values(t.detach().cpu().numpy())
    if kind == "fp4":
        return OQ.fp4_values(t.detach().cpu().numpy())
    return np64(t)


def cpu_or_none(case, key):
    t = case.get(key)
    return None if t is None else t.detach().cpu().numpy()


def check_attn(got, ref, atol=ATOL, meanrel=MEANREL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    mr = float(err.sum() / max(np.abs(ref).sum(), 1e-30))
    assert mx <= atol, f"max-abs {mx:.3e} > {atol}"
    if meanrel is not None:
        assert mr <= meanrel, f"mean-rel {mr:.3e} > {meanrel}"
    return mx, mr


def gpu_case(case):
    out = {}
    for k, v in case.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.to(DEV)
        else:
            out[k] = v
    return out


def run_decode(g, partition_tokens=0, max_context_len=None, window=0):
    P.device_status(clear=True)
    out = P.paged_attention_decode(g["q"], g["k_cache"], g["v_cache"], g["block_tables"], g["context_lens"],
                                   g["scale"], k_scale=g.get("k_scale"), v_scale=g.get("v_scale"),
                                   max_context_len=max_context_len, partition_tokens=partition_tokens,
                                   k_zero=g.get("k_zero"), v_zero=g.get("v_zero"), sliding_window=window,
                                   kv_format=g.get("cache_kind") if g.get("cache_kind") in FOUR_BIT else None)
    torch.cuda.synchronize()
    assert P.device_status(clear=True) == 0
    return out


def oracle_full(case, window=0):
    kind = case["cache_kind"]
    return OA.paged_decode_attention(np64(case["q"]), cache_values(case["k_cache"], kind),
                                     cache_values(case["v_cache"], kind), case["block_tables"].numpy(),
                                     case["context_lens"].numpy(), case["scale"],
                                     cpu_or_none(case, "k_scale"), cpu_or_none(case, "v_scale"),
                                     k_zero=cpu_or_none(case, "k_zero"), v_zero=cpu_or_none(case, "v_zero"),
                                     window=window)


def oracle_sampled(g, pairs, seed=0):
    """Oracle outputs for sampled (sequence, query head) pairs of a device
    case: the blocks of each sampled (sequence, KV head) are fetched to the
    host into a small pool in a shuffled order with a matching table."""
    kind = g["cache_kind"]
    G = g["hq"] // g["hkv"]
    bt = g["block_tables_cpu"]
    ctxs = g["context_lens_cpu"]
    rng = np.random.default_rng(seed)
    res = {}
    by_group = {}
    for s, i in pairs:
        by_group.setdefault((s, i // G), []).append(i)
    for (s, h), heads in by_group.items():
        ctx = int(ctxs[s])
        nblk = (ctx + 15) // 16
        if nblk == 0:
            for i in heads:
                res[(s, i)] = np.zeros(g["d"])
            continue
        blocks = bt[s, :nblk].to(DEV).long()
        perm = rng.permutation(nblk)
        pool_idx = torch.as_tensor(np.argsort(perm), device=DEV)  # logical j stored at pool row perm[j]
        kc = g["k_cache"][blocks][:, h:h + 1][pool_idx]
        vc = g["v_cache"][blocks][:, h:h + 1][pool_idx]
        side = {}
        for key in ("k_scale", "v_scale", "k_zero", "v_zero"):
            if key in g:
                side[key] = g[key][blocks][:, h:h + 1][pool_idx].cpu().numpy()
        q = np64(g["q"][s, heads])[None]
        ref = OA.paged_decode_attention(q, cache_values(kc, kind), cache_values(vc, kind), perm[None],
                                        [ctx], g["scale"], side.get("k_scale"), side.get("v_scale"),
                                        k_zero=side.get("k_zero"), v_zero=side.get("v_zero"))[0]
        for n, i in enumerate(heads):
            res[(s, i)] = ref[n]
    return np.stack([res[p] for p in pairs])


# ------------------------------------------------------------------ writes --

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d,T,nb", [(64, 37, 20), (128, 64, 40), (128, 4096, 300)])
def test_write_16bit_bit_exact(dtype, d, T, nb):
    hkv = 8
    gen = I.generator(11 + T)
    kc = I.randn((nb, hkv, 16, d), gen, dtype)
    vc = I.randn((nb, hkv, 16, d), gen, dtype)
    k, v = I.new_tokens(T, hkv, d, dtype, seed=T + d)
    slots = I.distinct_slots(T, nb, seed=T, skip_every=7)
    gk, gv = kc.to(DEV), vc.to(DEV)
    P.kv_cache_write(k.to(DEV), v.to(DEV), gk, gv, slots.to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(bits(gk), OC.kv_write(bits(kc), bits(k), slots.numpy()))
    assert np.array_equal(bits(gv), OC.kv_write(bits(vc), bits(v), slots.numpy()))


def _special_rows(k):
    """Rows that exercise the quantisers' edge cases: all zero, exact ties at
    scale 1 (INT8), signed zeros; for the asymmetric rule also a constant
    row, rows that do not contain 0 (zero point clamped to 0 or 255) and a
    scale-1 grid with ties in both the zero point and the codes."""
    d = k.shape[-1]
    k[0, 0].zero_()
    row = torch.zeros(d)
    row[:9] = torch.tensor([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 126.5])
    k[1, 0] = row.to(k.dtype)
    k[2, 0, 1::2] = -0.0
    k[3, 0] = torch.full((d,), 3.25).to(k.dtype)
    k[4, 0] = (1.0 + torch.arange(d) % 7).to(k.dtype)
    k[5, 0] = (-2.0 - torch.arange(d) % 5).to(k.dtype)
    row = torch.zeros(d)
    row[:5] = torch.tensor([-0.5, 0.0, 1.0, 2.0, 254.5])
    k[6, 0] = row.to(k.dtype)
    return k


QUANT = {"int8": (torch.int8, np.int8, lambda x: OQ.quantize_int8(x) + (None,)),
         "fp8": (torch.uint8, np.uint8, lambda x: OQ.quantize_fp8_e4m3(x) + (None,)),
         "u8asym": (torch.uint8, np.uint8, OQ.quantize_u8_asym),
         "int4": (torch.uint8, np.uint8, lambda x: OQ.quantize_int4(x) + (None,)),
         "fp4": (torch.uint8, np.uint8, lambda x: OQ.quantize_fp4_e2m1(x) + (None,))}


def fmt(kind):
    """kv_format argument of the binding for a cache kind."""
    return kind if kind in FOUR_BIT else None


@pytest.mark.parametrize("kind", ["int8", "fp8", "u8asym", "int4", "fp4"])
@pytest.mark.parametrize("in_dtype", ["bf16", "f16"])
@pytest.mark.parametrize("d,T", [(64, 50), (128, 600)])
def test_write_quantised_bit_exact(kind, in_dtype, d, T):
    hkv, nb = 4, 64
    k, v = I.new_tokens(T, hkv, d, in_dtype, seed=3 * T + d)
    k = _special_rows(k)
    slots = I.distinct_slots(T, nb, seed=T + 1)
    slots[9::9] = -1                                    # skip some tokens, keep the special rows
    cdt, ndt, quant = QUANT[kind]
    dc = d // 2 if kind in FOUR_BIT else d
    gk = torch.zeros((nb, hkv, 16, dc), dtype=cdt, device=DEV)
    gv = torch.zeros_like(gk)
    gks = torch.zeros((nb, hkv, 16), dtype=torch.float32, device=DEV)
    gvs = torch.zeros_like(gks)
    gkz = gvz = None
    if kind == "u8asym":
        gkz = torch.full((nb, hkv, 16), 7, dtype=torch.uint8, device=DEV)
        gvz = torch.full_like(gkz, 7)
    P.kv_cache_write(k.to(DEV), v.to(DEV), gk, gv, slots.to(DEV), gks, gvs, k_zero=gkz, v_zero=gvz,
                     kv_format=fmt(kind))
    torch.cuda.synchronize()
    zero_codes = np.zeros((nb, hkv, 16, dc), ndt)
    zero_sc = np.zeros((nb, hkv, 16), np.float32)
    for x, gc, gs, gz in ((k, gk, gks, gkz), (v, gv, gvs, gvz)):
        codes, sc, zp = quant(x.float().numpy())
        assert np.array_equal(bits(gc), OC.kv_write(zero_codes, codes, slots.numpy()))
        assert np.array_equal(bits(gs), OC.scale_write(zero_sc, sc, slots.numpy()).view(np.int32))
        if gz is not None:
            assert np.array_equal(bits(gz), OC.scale_write(np.full((nb, hkv, 16), 7, np.uint8), zp,
                                                           slots.numpy()))


# ------------------------------------------------------------ block copy --

@pytest.mark.parametrize("kind", ["float", "int8", "fp8", "u8asym", "int4"])
def test_copy_blocks_bit_exact(kind):
    case = I.decode_case("llama3_8b", batch=4, cache_kind=None if kind == "float" else kind, num_blocks=200,
                         ctx_override=[300, 500, 17, 1])
    g = gpu_case(case)
    rng = np.random.default_rng(5)
    perm = rng.permutation(200)
    pairs = np.stack([perm[:40], perm[40:80]], 1).astype(np.int32)   # sources and destinations disjoint
    P.copy_blocks(g["k_cache"], g["v_cache"], torch.as_tensor(pairs, device=DEV), g.get("k_scale"),
                  g.get("v_scale"), k_zero=g.get("k_zero"), v_zero=g.get("v_zero"), kv_format=fmt(kind))
    torch.cuda.synchronize()
    arrays = [bits(case["k_cache"]), bits(case["v_cache"])]
    got = [bits(g["k_cache"]), bits(g["v_cache"])]
    for key in ("k_scale", "v_scale", "k_zero", "v_zero"):
        if key in case:
            arrays.append(bits(case[key]))
            got.append(bits(g[key]))
    for ref, out in zip(OC.copy_blocks(arrays, pairs), got):
        assert np.array_equal(ref, out)


# ------------------------------------------------------- attention: sweeps --

CTX_MIX = [0, 1, 15, 16, 17, 255, 256, 257, 1000]


def test_decode_tiny_workload_all_outputs():
    case = I.decode_case("tiny")
    g = gpu_case(case)
    ref = oracle_full(case)
    check_attn(np64(run_decode(g)), ref)
    check_attn(np64(run_decode(g, partition_tokens=32)), ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group", [1, 4, 8, 16])
@pytest.mark.parametrize("ptok", [0, 64, 16])
def test_decode_sweep_16bit(dtype, d, group, ptok):
    hkv = 2
    case = I.decode_case("llama3_8b", seed=d * 100 + group, ctx_override=CTX_MIX, hq=hkv * group, hkv=hkv, d=d,
                         dtype=dtype)
    g = gpu_case(case)
    out = run_decode(g, partition_tokens=ptok)
    ref = oracle_full(case)
    got = np64(out)
    assert np.all(got[0] == 0)                       # context 0 gives a zero row
    check_attn(got, ref)
    # a single-token context returns that token's value row (up to output rounding)
    v0 = np64(case["v_cache"][case["block_tables"][1, 0], :, 0])
    np.testing.assert_allclose(got[1], np.repeat(v0, group, axis=0), atol=1e-2)


@pytest.mark.parametrize("kind", ["int8", "fp8", "u8asym", "int4", "fp4"])
@pytest.mark.parametrize("qdtype", ["bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group", [1, 8, 16])
@pytest.mark.parametrize("ptok", [0, 32])
def test_decode_sweep_quantised(kind, qdtype, d, group, ptok):
    hkv = 2
    case = I.decode_case("quant_mha", seed=d + group, ctx_override=CTX_MIX, hq=hkv * group, hkv=hkv, d=d,
                         dtype=qdtype, cache_kind=kind)
    g = gpu_case(case)
    got = np64(run_decode(g, partition_tokens=ptok))
    check_attn(got, oracle_full(case))


@pytest.mark.parametrize("kind", ["int8", "fp8", "u8asym", "int4", "fp4"])
def test_decode_quantised_large_value_scales(kind):
    """Value scales in the hundreds to thousands (values up to ~4e4): the
    probabilities enter the MMA multiplied by the value scale in fp16, so
    the kernel must keep them small enough not to overflow; compared with the
    oracle relative to the output's magnitude."""
    hkv, group = 2, 4
    case = I.decode_case("quant_mha", seed=77, ctx_override=CTX_MIX, hq=hkv * group, hkv=hkv, d=128,
                         dtype="bf16", cache_kind=kind)
    case["v_scale"] = case["v_scale"] * 1.0e4
    g = gpu_case(case)
    got = np64(run_decode(g))
    ref = oracle_full(case)
    scale = float(np.abs(ref).max())
    assert scale > 1e3
    check_attn(got / scale, ref / scale)


@pytest.mark.parametrize("window", [1, 16, 40, 300])
@pytest.mark.parametrize("group,d", [(4, 128), (16, 128), (8, 64)])
@pytest.mark.parametrize("ptok", [0, 16])
def test_decode_sliding_window(window, group, d, ptok):
    hkv = 2
    case = I.decode_case("llama3_8b", seed=window + group, ctx_override=CTX_MIX, hq=hkv * group, hkv=hkv, d=d)
    g = gpu_case(case)
    # blocks wholly before the window are never read: poison their table entries
    bt = g["block_tables"].clone()
    for s, c in enumerate(CTX_MIX):
        first = max(0, c - window) // 16
        bt[s, :first] = case["num_blocks"] + 7
    g["block_tables"] = bt
    got = np64(run_decode(g, partition_tokens=ptok, window=window))
    check_attn(got, oracle_full(case, window=window))


def test_decode_sliding_window_quantised():
    case = I.decode_case("quant_mha", seed=41, ctx_override=CTX_MIX, hq=8, hkv=2, d=128, cache_kind="u8asym")
    check_attn(np64(run_decode(gpu_case(case), window=100)), oracle_full(case, window=100))


def test_max_context_len_above_actual_is_fine():
    case = I.decode_case("tiny", seed=3)
    g = gpu_case(case)
    mb = case["block_tables"].shape[1]
    bt = torch.zeros((case["batch"], mb + 8), dtype=torch.int32)
    bt[:, :mb] = case["block_tables"]
    g["block_tables"] = bt.to(DEV)
    check_attn(np64(run_decode(g, max_context_len=(mb + 8) * 16)), oracle_full(case))


# --------------------------------------------------- attention: full sizes --

def _sample_pairs(B, hq, n, seed):
    rng = np.random.default_rng(seed)
    pairs = {(int(rng.integers(B)), int(rng.integers(hq))) for _ in range(n)}
    pairs |= {(0, i) for i in range(hq)}
    return sorted(pairs)


@pytest.mark.parametrize("name,kind,n", [("llama3_8b", None, 48), ("llama3_70b_32k", None, 16),
                                         ("prefix_shared", None, 40), ("quant_mha", "int8", 40),
                                         ("quant_mha", "fp8", 40), ("quant_mha", "u8asym", 40),
                                         ("quant_mha", "int4", 24), ("quant_mha", "fp4", 24)])
def test_decode_full_workload_sampled(name, kind, n):
    g = I.device_decode_case(name, DEV, cache_kind=kind)
    maxc = int(g["context_lens_cpu"].max())
    out = run_decode(g, max_context_len=maxc)          # the automatic plan, as the bench runs it
    pairs = _sample_pairs(g["batch"], g["hq"], n, seed=len(name))
    got = np.stack([np64(out[s, i]) for s, i in pairs])
    check_attn(got, oracle_sampled(g, pairs))
    # every output is a convex combination of value rows
    o = out.float()
    assert torch.isfinite(o).all()
    if kind is None:
        assert float(o.abs().max()) <= float(g["v_cache"].float().abs().max()) + 1e-2


def test_decode_batch_beyond_the_eight_warp_scan_limit():
    """30,000 sequences of 0-16 tokens (at most one block each, some empty):
    the context-length scan of the batch no longer fits beside 8 warps'
    rings at head_dim 128, so the plan runs 4 warps per CTA.  Sampled
    outputs against the oracle; empty sequences give zero rows."""
    B = 30000
    ctx = np.random.default_rng(31).integers(0, 17, B).astype(np.int32)
    g = I.device_decode_case("llama3_8b", DEV, batch=B, ctx_override=ctx)
    nw, _, _ = P.decode_plan(B, g["hq"], g["hkv"], g["d"], 16, P.PKV_BF16)
    assert nw == 4 * 148
    out = run_decode(g, max_context_len=16)
    pairs = _sample_pairs(B, g["hq"], 64, seed=5)
    pairs += [(int(s), 3) for s in np.flatnonzero(ctx == 0)[:4]]
    got = np.stack([np64(out[s, i]) for s, i in pairs])
    check_attn(got, oracle_sampled(g, pairs))
    assert torch.isfinite(out.float()).all()


# --------------------------------------------------------- end to end ------

def test_prefix_sharing_copy_on_write_end_to_end():
    """128 sequences fork one 2040-token prefix (its last block half full),
    then each appends its own suffix: the first write copies the shared block
    (127 copies), the rest write in place.  The C++ allocator, copy_blocks and
    the write kernel build the cache; the oracle's model and scatter build
    their own; caches, tables and attention must agree."""
    B, hkv, hq, d, prefix = 128, 8, 32, 128, 2040
    gen = I.generator(77)
    suffix = torch.randint(64, 1025, (B,), generator=gen).tolist()
    need = (prefix + 15) // 16 + sum((prefix + s + 15) // 16 - prefix // 16 for s in suffix) + 8
    nb = int(math.ceil(need * 1.1))
    order = torch.randperm(nb, generator=gen).tolist()
    alloc = P.BlockAllocator(nb, initial_free_order=order)
    model = BlockManagerModel(nb, initial_free_order=order)
    kc = torch.zeros((nb, hkv, 16, d), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    ref_k = np.zeros((nb, hkv, 16, d), np.int16)
    ref_v = np.zeros_like(ref_k)

    def write(slots, ref_slots, seed):
        nonlocal ref_k, ref_v
        assert slots.tolist() == list(ref_slots)
        k, v = I.new_tokens(len(ref_slots), hkv, d, "bf16", seed)
        P.kv_cache_write(k.to(DEV), v.to(DEV), kc, vc, slots.to(DEV))
        ref_k = OC.kv_write(ref_k, bits(k), ref_slots)
        ref_v = OC.kv_write(ref_v, bits(v), ref_slots)

    alloc.add(0)
    model.add(0)
    write(alloc.append(0, prefix)[0], model.append(0, prefix)[0], 1)
    for c in range(1, B):
        alloc.fork(0, c)
        model.fork(0, c)
    slots, pairs = alloc.batch_append(list(range(B)))
    ref_slots, ref_pairs = [], []
    for s in range(B):
        sl, pr = model.append(s, 1)
        ref_slots += sl
        ref_pairs += pr
    assert [tuple(p) for p in pairs.tolist()] == ref_pairs and len(ref_pairs) == 127
    P.copy_blocks(kc, vc, pairs.to(DEV))
    ref_k, ref_v = OC.copy_blocks([ref_k, ref_v], np.array(ref_pairs, np.int32))
    write(slots, ref_slots, 2)
    for s in range(B):
        sl, pr = alloc.append(s, suffix[s] - 1)
        rsl, rpr = model.append(s, suffix[s] - 1)
        assert pr.shape[0] == 0 and rpr == []
        write(sl, rsl, 100 + s)
    torch.cuda.synchronize()
    assert np.array_equal(bits(kc), ref_k) and np.array_equal(bits(vc), ref_v)
    mb = max(len(model.block_table(s)) for s in range(B))
    bt, cl = alloc.batch_tables(list(range(B)), mb)
    for s in range(B):
        assert bt[s, :len(model.block_table(s))].tolist() == model.block_table(s)
    q = I.randn((B, hq, d), I.generator(5), "bf16")
    out = P.paged_attention_decode(q.to(DEV), kc, vc, bt.to(DEV), cl.to(DEV), 1 / math.sqrt(d),
                                   max_context_len=int(cl.max()))
    sample = list(range(0, B, 9))
    kv = torch.from_numpy(ref_k).view(torch.bfloat16)
    vv = torch.from_numpy(ref_v).view(torch.bfloat16)
    ref = OA.paged_decode_attention(np64(q), np64(kv), np64(vv), bt.numpy(), cl.numpy(), 1 / math.sqrt(d),
                                    seqs=sample)
    check_attn(np64(out)[sample], ref[sample])


@pytest.mark.parametrize("kind", ["int8", "fp8", "u8asym", "int4", "fp4"])
def test_quantised_write_then_decode_end_to_end(kind):
    """bf16 token rows are quantised by the write kernel and attended by the
    decode kernel; against the oracle on the unquantised rows (6e-2) and on
    the oracle's own quantisation of the same rows (2e-2 / 1e-2)."""
    B, hkv, hq, d = 24, 32, 32, 128
    gen = I.generator(91)
    ctx = torch.exp(torch.empty(B).uniform_(math.log(128), math.log(2048), generator=gen)).round().int()
    need = sum((int(c) + 15) // 16 for c in ctx)
    nb = int(need * 1.1) + 1
    bt = I.random_block_tables(ctx, nb, gen)
    slots = torch.cat([bt[s, torch.arange(int(c)) // 16].long() * 16 + torch.arange(int(c)) % 16
                       for s, c in enumerate(ctx.tolist())])
    T = slots.numel()
    k, v = I.new_tokens(T, hkv, d, "bf16", seed=92)
    cdt, _, quant = QUANT[kind]
    gk = torch.zeros((nb, hkv, 16, d // 2 if kind in FOUR_BIT else d), dtype=cdt, device=DEV)
    gv = torch.zeros_like(gk)
    gks = torch.zeros((nb, hkv, 16), dtype=torch.float32, device=DEV)
    gvs = torch.zeros_like(gks)
    gkz = gvz = None
    if kind == "u8asym":
        gkz = torch.zeros((nb, hkv, 16), dtype=torch.uint8, device=DEV)
        gvz = torch.zeros_like(gkz)
    P.kv_cache_write(k.to(DEV), v.to(DEV), gk, gv, slots.to(DEV), gks, gvs, k_zero=gkz, v_zero=gvz,
                     kv_format=fmt(kind))
    q = I.randn((B, hq, d), gen, "bf16")
    out = np64(P.paged_attention_decode(q.to(DEV), gk, gv, bt.to(DEV), ctx.to(DEV), 1 / math.sqrt(d), gks, gvs,
                                        max_context_len=int(ctx.max()), k_zero=gkz, v_zero=gvz,
                                        kv_format=fmt(kind)))
    # (i) against attention over the unquantised bf16 rows
    raw_k = OC.kv_write(np.zeros((nb, hkv, 16, d)), k.double().numpy(), slots.numpy())
    raw_v = OC.kv_write(np.zeros((nb, hkv, 16, d)), v.double().numpy(), slots.numpy())
    ref_raw = OA.paged_decode_attention(np64(q), raw_k, raw_v, bt.numpy(), ctx.numpy(), 1 / math.sqrt(d))
    check_attn(out, ref_raw, atol=Q4ATOL if kind in FOUR_BIT else QATOL, meanrel=None)
    # (ii) against the oracle's own quantisation of the same rows
    dec = {"fp8": OQ.e4m3_decode, "int4": OQ.int4_values, "fp4": OQ.fp4_values}.get(
        kind, lambda c: c.astype(np.float64))
    ck, sk, zk = quant(k.float().numpy())
    cv, sv, zv = quant(v.float().numpy())
    zc = np.zeros((nb, hkv, 16, d))
    zs = np.zeros((nb, hkv, 16), np.float32)
    zz = np.zeros((nb, hkv, 16), np.uint8)
    # (the 4-bit codes are unpacked by ``dec`` before the scatter)
    sl = slots.numpy()
    ref_q = OA.paged_decode_attention(np64(q), OC.kv_write(zc, dec(ck), sl), OC.kv_write(zc, dec(cv), sl),
                                      bt.numpy(), ctx.numpy(), 1 / math.sqrt(d), OC.scale_write(zs, sk, sl),
                                      OC.scale_write(zs, sv, sl),
                                      k_zero=None if zk is None else OC.scale_write(zz, zk, sl),
                                      v_zero=None if zv is None else OC.scale_write(zz, zv, sl))
    check_attn(out, ref_q)


# ------------------------------------------------------- host validation --

def test_validation_mode_rejects_bad_indices_before_launch():
    case = I.decode_case("tiny", seed=9)
    g = gpu_case(case)
    P.set_validation(True)
    try:
        bad = g["block_tables"].clone()
        bad[0, 0] = case["num_blocks"] + 5
        with pytest.raises(P.PagedKVError, match="out of range"):
            P.paged_attention_decode(g["q"], g["k_cache"], g["v_cache"], bad, g["context_lens"], 0.1,
                                     max_context_len=256)
        k = torch.zeros((2, 2, 64), dtype=torch.float16, device=DEV)
        with pytest.raises(P.PagedKVError, match="twice"):
            P.kv_cache_write(k, k, g["k_cache"], g["v_cache"], torch.tensor([5, 5], device=DEV))
        with pytest.raises(P.PagedKVError, match="both"):
            P.copy_blocks(g["k_cache"], g["v_cache"], torch.tensor([[1, 2], [2, 3]], dtype=torch.int32,
                                                                    device=DEV))
    finally:
        P.set_validation(False)
    torch.cuda.synchronize()


# ------------------------------------------------- workspace reuse, determinism --

def test_workspace_reused_across_shapes_matches_fresh_workspaces():
    """One workspace serving calls of different shapes (the arrival counters
    and the partial slots of one call overlap different fields of the next)
    must give exactly what a fresh zero-filled workspace gives, and repeated
    calls must give identical bits."""
    cases = [I.device_decode_case("llama3_8b", DEV, batch=32, seed=5),
             I.device_decode_case("prefix_shared", DEV, batch=48, seed=6),
             I.device_decode_case("quant_mha", DEV, batch=64, cache_kind="int8", seed=7)]
    shared = P.new_workspace(DEV, 256 << 20)
    for c in cases + cases[:1]:
        maxc = int(c["context_lens_cpu"].max())
        nw, _, wsb = P.decode_plan(c["batch"], c["hq"], c["hkv"], c["d"], maxc, c["k_cache"].dtype)
        assert nw > 1 and wsb <= shared.numel()
        run = lambda ws: P.paged_attention_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                                                  c["context_lens"], c["scale"], c.get("k_scale"), c.get("v_scale"),
                                                  max_context_len=maxc, workspace=ws)
        got = run(shared)
        ref = run(P.new_workspace(DEV, wsb))
        again = run(shared)
        torch.cuda.synchronize()
        assert torch.equal(got, ref) and torch.equal(got, again)
    assert P.device_status(clear=True) == 0


def test_workspace_needs_no_zero_fill_and_survives_a_growing_counter_area():
    """A workspace holding arbitrary bytes, and one whose next call has more
    (sequence, KV head) pairs than the last (its counter area then covers
    bytes that held the last call's partial floats), give the same bits as a
    fresh workspace: the library clears whatever part of a call's counter
    area it has not seen hold counters."""
    small = I.device_decode_case("llama3_8b", DEV, batch=4, seed=21)
    large = I.device_decode_case("quant_mha", DEV, batch=96, cache_kind="fp8", seed=22)
    runs = []
    for c in (small, large, small, large):
        maxc = int(c["context_lens_cpu"].max())
        nw, _, wsb = P.decode_plan(c["batch"], c["hq"], c["hkv"], c["d"], maxc, c["k_cache"].dtype, 256)
        assert nw > 1
        runs.append((c, maxc, wsb))
    wsb_max = max(w for _, _, w in runs)
    garbage = torch.randint(0, 256, (wsb_max,), dtype=torch.uint8, device=DEV)
    for c, maxc, wsb in runs:
        run = lambda ws: P.paged_attention_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                                                  c["context_lens"], c["scale"], c.get("k_scale"), c.get("v_scale"),
                                                  max_context_len=maxc, workspace=ws, partition_tokens=256)
        got = run(garbage)
        ref = run(P.new_workspace(DEV, wsb))
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    assert P.device_status(clear=True) == 0


@pytest.mark.parametrize("kind", ["float", "fp8", "u8asym", "fp4"])
def test_never_written_tail_positions_do_not_leak(kind):
    """Positions of a sequence's last block at or beyond its context were
    never written and may hold NaN bit patterns (codes and scales alike):
    the output must be the oracle's, which never reads them."""
    case = I.decode_case("llama3_8b", seed=13, ctx_override=CTX_MIX, hq=8, hkv=2, d=128,
                         cache_kind=None if kind == "float" else kind)
    g = gpu_case(case)
    for s, c in enumerate(CTX_MIX):
        if c == 0 or c % 16 == 0:
            continue
        b = int(case["block_tables"][s, (c - 1) // 16])
        for key in ("k_cache", "v_cache"):
            t = g[key]
            if kind == "float":
                t[b, :, c % 16:] = float("nan")
            else:
                t[b, :, c % 16:] = 0x7F if kind == "fp8" else 0xFF     # e4m3 NaN / arbitrary codes
        for key in ("k_scale", "v_scale"):
            if key in g:
                g[key][b, :, c % 16:] = float("nan")
    got = np64(run_decode(g))
    assert np.all(np.isfinite(got))
    check_attn(got, oracle_full(case))
