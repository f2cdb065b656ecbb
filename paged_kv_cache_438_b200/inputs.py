"""Seeded synthetic inputs for the five decode workloads.

This module only draws random numbers and lays out random block tables; it
holds none of the method's arithmetic (no attention, no quantisation rule, no
slot formula, no allocator).  Both the oracle-side tests and the CUDA-side
tests/bench take their inputs from here, so they see identical data.

Workloads (shapes of the Llama families the pages discuss; values N(0, 1)):

* ``tiny``        1 layer, batch 4, 8 q / 2 KV heads, head_dim 64, fp16,
                  context U[1, 256], a 128-block pool randomly permuted.
* ``llama3_8b``   32 q / 8 KV heads, head_dim 128, bf16, batch 64,
                  context U[512, 4096], shuffled pool of 1.1 x total need.
* ``llama3_70b_32k`` 64 q / 8 KV heads, head_dim 128, bf16, batch 32,
                  context 32768 each (split-KV territory).
* ``prefix_shared`` Llama-3-8B heads, 128 sequences sharing the physical
                  blocks of one 2048-token prefix plus own suffixes U[64, 1024].
* ``quant_mha``   Llama-2-7B heads (32 q / 32 KV), batch 256, context
                  log-uniform[128, 8192], INT8 or FP8-e4m3 codes with fp32
                  per-(token, head) scales, or uint8 codes with a scale and
                  a uint8 zero point per (token, head).

Multi-query workloads (several new tokens per sequence; context includes
them):

* ``spec_verify``      Llama-3-8B heads, batch 64, context U[512, 4096],
                       4 new tokens per sequence (verifying 4 drafted tokens).
* ``chunked_prefill``  Llama-3-8B heads, batch 8, context U[1024, 4096], the
                       last 512 tokens new (one prefill chunk per sequence).
"""
import math

import torch

BLOCK_SIZE = 16

WORKLOADS = {
    "tiny": dict(batch=4, hq=8, hkv=2, d=64, dtype="f16", ctx=("uniform", 1, 256),
                 pool=("fixed", 128), seed=1000),
    "llama3_8b": dict(batch=64, hq=32, hkv=8, d=128, dtype="bf16", ctx=("uniform", 512, 4096),
                      pool=("need", 1.1), seed=1001),
    "llama3_70b_32k": dict(batch=32, hq=64, hkv=8, d=128, dtype="bf16", ctx=("fixed", 32768),
                           pool=("need", 1.1), seed=1002),
    "prefix_shared": dict(batch=128, hq=32, hkv=8, d=128, dtype="bf16", ctx=("uniform", 64, 1024),
                          prefix=2048, pool=("need", 1.1), seed=1003),
    "quant_mha": dict(batch=256, hq=32, hkv=32, d=128, dtype="bf16", ctx=("loguniform", 128, 8192),
                      pool=("need", 1.1), cache=("int8", "fp8", "u8asym", "int4", "fp4"), seed=1004),
    "spec_verify": dict(batch=64, hq=32, hkv=8, d=128, dtype="bf16", ctx=("uniform", 512, 4096),
                        q_len=4, pool=("need", 1.1), seed=1005),
    "chunked_prefill": dict(batch=8, hq=32, hkv=8, d=128, dtype="bf16", ctx=("uniform", 1024, 4096),
                            q_len=512, pool=("need", 1.1), seed=1006),
}

TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


def generator(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def context_lens(spec, gen, batch=None):
    """int32 [batch] context lengths drawn from the workload's length mix
    (for ``prefix_shared`` these are the suffix lengths)."""
    b = spec["batch"] if batch is None else batch
    kind = spec["ctx"][0]
    if kind == "fixed":
        return torch.full((b,), spec["ctx"][1], dtype=torch.int32)
    lo, hi = spec["ctx"][1], spec["ctx"][2]
    if kind == "uniform":
        return torch.randint(lo, hi + 1, (b,), generator=gen, dtype=torch.int64).to(torch.int32)
    if kind == "loguniform":
        u = torch.rand((b,), generator=gen, dtype=torch.float64)
        v = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
        return v.round().clamp(lo, hi).to(torch.int32)
    raise ValueError(kind)


def blocks_for(n_tokens):
    return (n_tokens + BLOCK_SIZE - 1) // BLOCK_SIZE


def pool_size(spec, need_blocks):
    kind, val = spec["pool"]
    if kind == "fixed":
        return int(val)
    return int(math.ceil(need_blocks * val))


def random_block_tables(ctx, num_blocks, gen, shared_prefix_tokens=0, max_blocks=None):
    """Block tables [B, max_blocks] int32 drawn from a seeded permutation of
    the physical pool: the first blocks of the permutation hold the shared
    prefix (if any), the rest are handed to sequences in index order.  Unused
    entries are 0.  ``ctx`` are the full context lengths."""
    B = ctx.numel()
    perm = torch.randperm(num_blocks, generator=gen).to(torch.int32)
    n_pref = blocks_for(shared_prefix_tokens) if shared_prefix_tokens else 0
    assert shared_prefix_tokens % BLOCK_SIZE == 0, "shared prefix must fill whole blocks"
    need = [blocks_for(int(c)) for c in ctx.tolist()]
    MB = max(need) if max_blocks is None else max_blocks
    bt = torch.zeros((B, max(MB, 1)), dtype=torch.int32)
    cur = n_pref
    for s in range(B):
        own = need[s] - n_pref
        if n_pref:
            bt[s, :n_pref] = perm[:n_pref]
        bt[s, n_pref:n_pref + own] = perm[cur:cur + own]
        cur += own
    if cur > num_blocks:
        raise ValueError("pool too small for the drawn contexts")
    return bt


def randn(shape, gen, dtype):
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(TORCH_DTYPES[dtype])


def random_codes(shape, gen, kind):
    """Random cache codes with a bell-shaped value mix: N(0, 1) values spread
    over the code range and converted by torch's own casts (int8: rounded and
    clamped to +-127; fp8: torch.float8_e4m3fn, raw bytes returned as uint8;
    u8asym: centred on 127.5, rounded and clamped to [0, 255]).  The 4-bit
    kinds (int4, fp4) are uniformly random bytes, two codes each, over the
    last axis halved."""
    if kind in ("int4", "fp4"):
        return torch.randint(0, 256, shape[:-1] + (shape[-1] // 2,), generator=gen, dtype=torch.int64).to(torch.uint8)
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if kind == "u8asym":
        return (x * (255.0 / 6.0) + 127.5).round().clamp(0, 255).to(torch.uint8)
    if kind == "int8":
        return (x * (127.0 / 3.0)).round().clamp(-127, 127).to(torch.int8)
    if kind == "fp8":
        y = (x * (448.0 / 3.0)).clamp(-448.0, 448.0)
        return y.to(torch.float8_e4m3fn).view(torch.uint8)
    raise ValueError(kind)


def random_scales(shape, gen, kind):
    """Positive fp32 scales of the size an absmax rule (or, for u8asym, a
    min/max rule over 128 values) gives N(0, 1) data."""
    qmax = {"int8": 127.0, "fp8": 448.0, "u8asym": 255.0, "int4": 7.0, "fp4": 6.0}[kind]
    u = torch.rand(shape, generator=gen, dtype=torch.float32)
    if kind == "u8asym":
        return (4.0 + 2.0 * u) / qmax
    return (2.0 + 2.0 * u) / qmax


def random_zero_points(shape, gen):
    """uint8 zero points around the middle of the code range."""
    return torch.randint(96, 161, shape, generator=gen, dtype=torch.int64).to(torch.uint8)


def decode_case(name, seed=None, batch=None, ctx_override=None, cache_kind=None, num_blocks=None,
                **shape):
    """A complete random decode problem for workload ``name`` on the CPU.

    Returns a dict with q [B, Hq, D], k_cache / v_cache [NB, Hkv, 16, D]
    (values, or codes for int8 / fp8 with k_scale / v_scale [NB, Hkv, 16]),
    block_tables [B, MB] int32, context_lens [B] int32, scale and the shape
    fields.  ``ctx_override`` replaces the drawn context lengths; ``shape``
    may override hq, hkv, d and dtype.
    """
    spec = dict(WORKLOADS[name])
    spec.update(shape)
    if batch is not None:
        spec["batch"] = batch
    gen = generator(spec["seed"] if seed is None else seed)
    B, hq, hkv, d = spec["batch"], spec["hq"], spec["hkv"], spec["d"]
    if ctx_override is not None:
        ctx = torch.as_tensor(ctx_override, dtype=torch.int32).reshape(-1)
        B = ctx.numel()
        prefix = 0
    else:
        ctx = context_lens(spec, gen, B)
        prefix = spec.get("prefix", 0)
        ctx = ctx + prefix
    need = sum(blocks_for(int(c)) for c in ctx.tolist())
    if prefix:
        need -= (B - 1) * blocks_for(prefix)
    nb = pool_size(spec, max(need, 1)) if num_blocks is None else num_blocks
    nb = max(nb, need, 1)
    bt = random_block_tables(ctx, nb, gen, shared_prefix_tokens=prefix)
    kind = cache_kind or "float"
    out = dict(name=name, batch=B, hq=hq, hkv=hkv, d=d, block_size=BLOCK_SIZE,
               num_blocks=nb, dtype=spec["dtype"], cache_kind=kind,
               scale=1.0 / math.sqrt(d), block_tables=bt, context_lens=ctx)
    out["q"] = randn((B, hq, d), gen, spec["dtype"])
    if kind == "float":
        out["k_cache"] = randn((nb, hkv, BLOCK_SIZE, d), gen, spec["dtype"])
        out["v_cache"] = randn((nb, hkv, BLOCK_SIZE, d), gen, spec["dtype"])
    else:
        out["k_cache"] = random_codes((nb, hkv, BLOCK_SIZE, d), gen, kind)
        out["v_cache"] = random_codes((nb, hkv, BLOCK_SIZE, d), gen, kind)
        out["k_scale"] = random_scales((nb, hkv, BLOCK_SIZE), gen, kind)
        out["v_scale"] = random_scales((nb, hkv, BLOCK_SIZE), gen, kind)
        if kind == "u8asym":
            out["k_zero"] = random_zero_points((nb, hkv, BLOCK_SIZE), gen)
            out["v_zero"] = random_zero_points((nb, hkv, BLOCK_SIZE), gen)
    return out


def new_tokens(n_tokens, hkv, d, dtype, seed):
    """K and V rows [n_tokens, hkv, d] for a write, N(0, 1) in ``dtype``."""
    gen = generator(seed)
    return randn((n_tokens, hkv, d), gen, dtype), randn((n_tokens, hkv, d), gen, dtype)


def distinct_slots(n_tokens, num_blocks, seed, skip_every=0):
    """``n_tokens`` distinct random slots in [0, num_blocks * 16) as int64;
    every ``skip_every``-th entry (if > 0) is -1."""
    gen = generator(seed)
    perm = torch.randperm(num_blocks * BLOCK_SIZE, generator=gen)[:n_tokens].to(torch.int64)
    if skip_every:
        perm[::skip_every] = -1
    return perm


def device_decode_case(name, device, seed=None, batch=None, cache_kind=None, ctx_override=None):
    """Like ``decode_case`` but the large arrays (q and the caches) are drawn
    directly on ``device`` from a seeded CUDA generator, so full-size
    workloads need no host copy.  Context lengths and block tables are drawn
    on the CPU exactly as in ``decode_case`` and then moved to the device."""
    spec = dict(WORKLOADS[name])
    if batch is not None:
        spec["batch"] = batch
    base_seed = spec["seed"] if seed is None else seed
    gen = generator(base_seed)
    B, hq, hkv, d = spec["batch"], spec["hq"], spec["hkv"], spec["d"]
    if ctx_override is not None:
        ctx = torch.as_tensor(ctx_override, dtype=torch.int32).reshape(-1)
        B = ctx.numel()
        prefix = 0
    else:
        ctx = context_lens(spec, gen, B)
        prefix = spec.get("prefix", 0)
        ctx = ctx + prefix
    need = sum(blocks_for(int(c)) for c in ctx.tolist())
    if prefix:
        need -= (B - 1) * blocks_for(prefix)
    nb = max(pool_size(spec, max(need, 1)), need, 1)
    bt = random_block_tables(ctx, nb, gen, shared_prefix_tokens=prefix)
    dg = torch.Generator(device=device)
    dg.manual_seed(base_seed + 7919)
    kind = cache_kind or "float"
    dt = TORCH_DTYPES[spec["dtype"]]
    out = dict(name=name, batch=B, hq=hq, hkv=hkv, d=d, block_size=BLOCK_SIZE, num_blocks=nb,
               dtype=spec["dtype"], cache_kind=kind, scale=1.0 / math.sqrt(d),
               block_tables=bt.to(device), context_lens=ctx.to(device),
               block_tables_cpu=bt, context_lens_cpu=ctx)
    out["q"] = torch.randn((B, hq, d), generator=dg, device=device, dtype=dt)
    shape = (nb, hkv, BLOCK_SIZE, d)
    if kind == "float":
        out["k_cache"] = torch.randn(shape, generator=dg, device=device, dtype=dt)
        out["v_cache"] = torch.randn(shape, generator=dg, device=device, dtype=dt)
    else:
        for key in ("k_cache", "v_cache"):
            x = torch.randn(shape, generator=dg, device=device, dtype=torch.float16)
            if kind in ("int4", "fp4"):
                out[key] = torch.randint(0, 256, shape[:-1] + (shape[-1] // 2,), generator=dg, device=device,
                                         dtype=torch.int64).to(torch.uint8)
            elif kind == "int8":
                out[key] = (x * (127.0 / 3.0)).round().clamp(-127, 127).to(torch.int8)
            elif kind == "u8asym":
                out[key] = (x.float() * (255.0 / 6.0) + 127.5).round().clamp(0, 255).to(torch.uint8)
            else:
                out[key] = (x.float() * (448.0 / 3.0)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
            del x
        qmax = {"int8": 127.0, "fp8": 448.0, "u8asym": 255.0, "int4": 7.0, "fp4": 6.0}[kind]
        span = 4.0 if kind == "u8asym" else 2.0
        for key in ("k_scale", "v_scale"):
            u = torch.rand((nb, hkv, BLOCK_SIZE), generator=dg, device=device, dtype=torch.float32)
            out[key] = (span + 2.0 * u) / qmax
        if kind == "u8asym":
            for key in ("k_zero", "v_zero"):
                out[key] = torch.randint(96, 161, (nb, hkv, BLOCK_SIZE), generator=dg, device=device,
                                         dtype=torch.int64).to(torch.uint8)
    return out


def multi_query_case(name, seed=None, batch=None, ctx_override=None, q_lens=None, cache_kind=None,
                     num_blocks=None, **shape):
    """A random multi-query problem on the CPU: ``decode_case`` plus
    query_start_loc [B + 1] int32 and q [T, Hq, D] packed by sequence.  The
    new-token counts are the workload's q_len (clamped to each context) unless
    ``q_lens`` gives them."""
    case = decode_case(name, seed=seed, batch=batch, ctx_override=ctx_override, cache_kind=cache_kind,
                       num_blocks=num_blocks, **shape)
    spec = WORKLOADS[name]
    ctx = case["context_lens"]
    if q_lens is None:
        n = torch.clamp(torch.full_like(ctx, spec.get("q_len", 1)), max=ctx)
    else:
        n = torch.as_tensor(q_lens, dtype=torch.int32).reshape(-1)
    qsl = torch.zeros(ctx.numel() + 1, dtype=torch.int32)
    qsl[1:] = torch.cumsum(n, 0)
    gen = generator((spec["seed"] if seed is None else seed) + 31)
    case["query_start_loc"] = qsl
    case["max_query_len"] = int(n.max()) if n.numel() else 0
    case["q"] = randn((int(qsl[-1]), case["hq"], case["d"]), gen, shape.get("dtype", spec["dtype"]))
    return case


def device_multi_query_case(name, device, seed=None, batch=None, cache_kind=None):
    """``device_decode_case`` plus query_start_loc (on the device, and a CPU
    copy) and q [T, Hq, D] drawn on the device; each sequence gets the
    workload's q_len new tokens (clamped to its context)."""
    case = device_decode_case(name, device, seed=seed, batch=batch, cache_kind=cache_kind)
    spec = WORKLOADS[name]
    ctx = case["context_lens_cpu"]
    n = torch.clamp(torch.full_like(ctx, spec.get("q_len", 1)), max=ctx)
    qsl = torch.zeros(ctx.numel() + 1, dtype=torch.int32)
    qsl[1:] = torch.cumsum(n, 0)
    dg = torch.Generator(device=device)
    dg.manual_seed((spec["seed"] if seed is None else seed) + 104729)
    case["query_start_loc_cpu"] = qsl
    case["query_start_loc"] = qsl.to(device)
    case["max_query_len"] = int(n.max()) if n.numel() else 0
    case["q"] = torch.randn((int(qsl[-1]), case["hq"], case["d"]), generator=dg, device=device,
                            dtype=TORCH_DTYPES[spec["dtype"]])
    return case
