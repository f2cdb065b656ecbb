"""GPU parity of multi-query paged attention (several new tokens per
sequence: chunked prefill, speculative verification) against the fp64
oracle, through the C ABI.

Bars as for decode: max-abs 2e-2 and mean-rel 1e-2 for fp16 / bf16 caches,
the same against the oracle on the stored codes for 8-bit caches.  With one
new token per sequence the result must equal the decode entry point's bit
for bit (same arithmetic in the same order).
"""
import numpy as np
import pytest
import torch

from oracle import attention as OA
from paged_kv_cache_438_b200 import inputs as I
from paged_kv_cache_438_b200 import pagedkv as P
from test_gpu_parity import DEV, check_attn, cache_values, cpu_or_none, gpu_case, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_kv_cache_438_b200 import build
    build.build()
    P.lib()
    P.device_status(clear=True)
    yield
    assert P.device_status(clear=True) == 0, "a kernel raised a device status bit"


def run_mq(g, partition_tokens=0, max_query_len=None, window=0):
    out = P.paged_attention_multi_query(
        g["q"], g["k_cache"], g["v_cache"], g["block_tables"], g["context_lens"], g["query_start_loc"], g["scale"],
        max_query_len=g["max_query_len"] if max_query_len is None else max_query_len,
        max_context_len=int(g["context_lens"].max()), k_scale=g.get("k_scale"), v_scale=g.get("v_scale"),
        k_zero=g.get("k_zero"), v_zero=g.get("v_zero"), partition_tokens=partition_tokens, sliding_window=window,
        kv_format=g.get("cache_kind") if g.get("cache_kind") in ("int4", "fp4") else None)
    torch.cuda.synchronize()
    assert P.device_status(clear=True) == 0
    return out


def oracle_mq(case, seqs=None, window=0):
    """Oracle rows for all sequences, or only for ``seqs`` (others zero)."""
    kind = case["cache_kind"]
    qsl = case["query_start_loc"].numpy()
    ctx = case["context_lens"].numpy()
    bt = case["block_tables"].numpy()
    if seqs is not None:
        keep = np.zeros(len(ctx), bool)
        keep[list(seqs)] = True
        ctx = np.where(keep, ctx, 0)
        n = np.where(keep, np.diff(qsl), 0)
        q = np64(case["q"])
        sub_qsl = np.concatenate([[0], np.cumsum(n)])
        rows = np.concatenate([np.arange(qsl[s], qsl[s + 1]) for s in range(len(n)) if keep[s]] or [[]]).astype(int)
        sub = OA.paged_multi_query_attention(q[rows], cache_values(case["k_cache"], kind),
                                             cache_values(case["v_cache"], kind), bt, ctx, sub_qsl, case["scale"],
                                             cpu_or_none(case, "k_scale"), cpu_or_none(case, "v_scale"),
                                             cpu_or_none(case, "k_zero"), cpu_or_none(case, "v_zero"), window)
        return rows, sub
    return OA.paged_multi_query_attention(np64(case["q"]), cache_values(case["k_cache"], kind),
                                          cache_values(case["v_cache"], kind), bt, ctx, qsl, case["scale"],
                                          cpu_or_none(case, "k_scale"), cpu_or_none(case, "v_scale"),
                                          cpu_or_none(case, "k_zero"), cpu_or_none(case, "v_zero"), window)


CTX = [1, 15, 16, 17, 40, 257, 1000, 33, 0, 300]
NQ = [1, 15, 3, 17, 40, 5, 24, 1, 0, 9]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group", [1, 4, 8, 16])
@pytest.mark.parametrize("ptok", [0, 16])
def test_multi_query_sweep_16bit(dtype, d, group, ptok):
    hkv = 2
    case = I.multi_query_case("spec_verify", seed=d * 10 + group, ctx_override=CTX, q_lens=NQ, hq=hkv * group,
                              hkv=hkv, d=d, dtype=dtype)
    got = np64(run_mq(gpu_case(case), partition_tokens=ptok))
    check_attn(got, oracle_mq(case))


@pytest.mark.parametrize("kind", ["int8", "fp8", "u8asym", "int4", "fp4"])
@pytest.mark.parametrize("group", [1, 4])
def test_multi_query_quantised(kind, group):
    hkv = 4
    case = I.multi_query_case("spec_verify", seed=group + 70, ctx_override=CTX, q_lens=NQ, hq=hkv * group, hkv=hkv,
                              d=128, cache_kind=kind)
    check_attn(np64(run_mq(gpu_case(case))), oracle_mq(case))


@pytest.mark.parametrize("window", [1, 7, 33, 200])
@pytest.mark.parametrize("group", [1, 4])
@pytest.mark.parametrize("ptok", [0, 16])
def test_multi_query_sliding_window(window, group, ptok):
    hkv = 2
    case = I.multi_query_case("spec_verify", seed=window * 3 + group, ctx_override=CTX, q_lens=NQ, hq=hkv * group,
                              hkv=hkv, d=128)
    g = gpu_case(case)
    bt = g["block_tables"].clone()
    for s, (c, n) in enumerate(zip(CTX, NQ)):
        if n:
            bt[s, :max(0, c - n + 1 - window) // 16] = case["num_blocks"] + 3   # never read
    g["block_tables"] = bt
    check_attn(np64(run_mq(g, partition_tokens=ptok, window=window)), oracle_mq(case, window=window))


@pytest.mark.parametrize("group", [4, 16])
def test_one_new_token_equals_decode_bitwise(group):
    hkv = 2
    ctx = [1, 17, 300, 1000, 0, 64]
    case = I.multi_query_case("spec_verify", seed=5, ctx_override=ctx, q_lens=[min(c, 1) for c in ctx],
                              hq=hkv * group, hkv=hkv, d=128)
    g = gpu_case(case)
    mq = run_mq(g)
    # decode reads one query row per sequence: scatter the packed rows
    qd = torch.zeros((len(ctx), hkv * group, 128), dtype=g["q"].dtype, device=DEV)
    has = torch.tensor([c > 0 for c in ctx], device=DEV)
    qd[has] = g["q"]
    dec = P.paged_attention_decode(qd, g["k_cache"], g["v_cache"], g["block_tables"], g["context_lens"],
                                   g["scale"], max_context_len=max(ctx))
    torch.cuda.synchronize()
    assert torch.equal(mq, dec[has])


def test_chunking_does_not_change_results():
    """Twelve new tokens in one pass against three passes of 5, 4 and 3
    tokens over the context up to each pass's last token."""
    hkv, group = 2, 4
    ctx, n = 500, 12
    case = I.multi_query_case("spec_verify", seed=8, ctx_override=[ctx], q_lens=[n], hq=hkv * group, hkv=hkv, d=128)
    g = gpu_case(case)
    one = np64(run_mq(g))
    parts, start = [], 0
    for m in (5, 4, 3):
        c = ctx - n + start + m
        sub = dict(g)
        sub["q"] = g["q"][start:start + m]
        sub["context_lens"] = torch.tensor([c], dtype=torch.int32, device=DEV)
        sub["query_start_loc"] = torch.tensor([0, m], dtype=torch.int32, device=DEV)
        sub["max_query_len"] = m
        parts.append(np64(run_mq(sub)))
        start += m
    check_attn(np.concatenate(parts), one, atol=4e-3, meanrel=1e-3)


@pytest.mark.parametrize("name,nseq", [("spec_verify", 6), ("chunked_prefill", 2)])
def test_multi_query_full_workload_sampled(name, nseq):
    g = I.device_multi_query_case(name, DEV)
    out = P.paged_attention_multi_query(g["q"], g["k_cache"], g["v_cache"], g["block_tables"], g["context_lens"],
                                        g["query_start_loc"], g["scale"], max_query_len=g["max_query_len"],
                                        max_context_len=int(g["context_lens_cpu"].max()))
    torch.cuda.synchronize()
    assert P.device_status(clear=True) == 0
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(len(name))
    seqs = sorted(rng.choice(g["batch"], size=nseq, replace=False).tolist())
    # oracle on the sampled sequences only: move just their blocks to the host
    qsl = g["query_start_loc_cpu"]
    for s in seqs:
        ctx = int(g["context_lens_cpu"][s])
        nblk = (ctx + 15) // 16
        blocks = g["block_tables_cpu"][s, :nblk].long()
        kc = g["k_cache"][blocks.to(DEV)].cpu()
        vc = g["v_cache"][blocks.to(DEV)].cpu()
        rows = np.arange(int(qsl[s]), int(qsl[s + 1]))
        ref = OA.paged_multi_query_attention(np64(g["q"][rows[0]:rows[-1] + 1]), np64(kc), np64(vc),
                                             np.arange(nblk)[None], [ctx], [0, len(rows)], g["scale"])
        check_attn(np64(out[rows[0]:rows[-1] + 1]), ref)


def test_validation_rejects_inconsistent_query_runs():
    case = I.multi_query_case("spec_verify", seed=3, ctx_override=[20, 40], q_lens=[4, 4], hq=8, hkv=2, d=64)
    g = gpu_case(case)
    P.set_validation(True)
    try:
        bad = dict(g)
        bad["query_start_loc"] = torch.tensor([0, 25, 8], dtype=torch.int32, device=DEV)
        with pytest.raises(P.PagedKVError, match="new tokens"):
            run_mq(bad, max_query_len=30)
        bad["query_start_loc"] = torch.tensor([0, 4, 7], dtype=torch.int32, device=DEV)
        with pytest.raises(P.PagedKVError, match="num_q_tokens"):
            run_mq(bad)
    finally:
        P.set_validation(False)


def test_multi_query_never_written_tail_positions_do_not_leak():
    case = I.multi_query_case("spec_verify", seed=17, ctx_override=CTX, q_lens=NQ, hq=8, hkv=2, d=128)
    g = gpu_case(case)
    for s, c in enumerate(CTX):
        if c == 0 or c % 16 == 0:
            continue
        b = int(case["block_tables"][s, (c - 1) // 16])
        g["k_cache"][b, :, c % 16:] = float("nan")
        g["v_cache"][b, :, c % 16:] = float("nan")
    got = np64(run_mq(g))
    assert np.all(np.isfinite(got))
    check_attn(got, oracle_mq(case))


@pytest.mark.parametrize("dtype,d,group", [("bf16", 128, 8), ("f16", 128, 4), ("bf16", 64, 16), ("f16", 64, 2)])
def test_query_major_kernel_against_oracle_and_decode_mode(dtype, d, group):
    """Runs long enough for the query-major tcgen05 kernel (>= 128 rows of
    (token, head)): against the oracle, and against the decode kernel's
    multi-query mode (forced with an explicit partition)."""
    hkv = 2
    ctx = [700, 130, 257, 64, 1, 300]
    nq = [300, 130, 17, 64, 1, 0]
    case = I.multi_query_case("chunked_prefill", seed=d + group, ctx_override=ctx, q_lens=nq, hq=hkv * group,
                              hkv=hkv, d=d, dtype=dtype)
    g = gpu_case(case)
    nw, _, _ = P.multi_query_plan(len(ctx), hkv * group, hkv, d, max(ctx), max(nq), g["k_cache"].dtype)
    assert nw == len(ctx) * hkv * (((max(nq) * group + 127) // 128 + 1) // 2)     # the query-major plan
    fast = np64(run_mq(g))
    ref = oracle_mq(case)
    check_attn(fast, ref)
    slow = np64(run_mq(g, partition_tokens=64))
    check_attn(fast, slow, atol=2e-2, meanrel=5e-3)        # two bf16-rounded outputs: within 2 ulps


@pytest.mark.parametrize("ctx,nq", [
    ([300] * 5, [300, 129, 64, 200, 32]),                       # every context length equal
    ([500, 200, 500, 200, 64, 500], [200, 150, 40, 200, 64, 1]),  # repeated lengths
    ([int(32 + (97 * i) % 170) for i in range(70)],               # more sequences than are ranked
     [min(40, int(32 + (97 * i) % 170)) for i in range(70)]),
])
def test_query_major_launch_order_covers_every_sequence(ctx, nq):
    """The query-major kernel starts sequences in decreasing context length
    (ties by index; beyond 64 sequences in launch order): every run of every
    sequence must still be computed exactly once."""
    hkv, group = 2, 4
    case = I.multi_query_case("chunked_prefill", seed=len(ctx) + sum(nq), ctx_override=ctx, q_lens=nq,
                              hq=hkv * group, hkv=hkv, d=128, dtype="bf16")
    g = gpu_case(case)
    nw, _, _ = P.multi_query_plan(len(ctx), hkv * group, hkv, 128, max(ctx), max(nq), g["k_cache"].dtype)
    assert nw == len(ctx) * hkv * (((max(nq) * group + 127) // 128 + 1) // 2)     # the query-major plan
    got = np64(run_mq(g))
    assert np.all(np.isfinite(got))
    check_attn(got, oracle_mq(case))


@pytest.mark.parametrize("dtype,group", [("bf16", 4), ("f16", 4), ("bf16", 16)])
def test_query_major_kernel_scores_rising_along_the_keys(dtype, group):
    """Scores that climb by about 65 log2 units over each context (about 12
    per 128-key tile; q and the K rows share one direction, the K rows scaled
    by their position): every row keeps moving its exponent base.  A tile
    whose probabilities against the base in use would pass 2^20 (or overflow
    fp16) must take its maximum and be written again, the others keep the
    lagging base; both must match the oracle."""
    hkv, d = 2, 128
    ctx, nq = [700, 1100, 300], [300, 200, 140]
    case = I.multi_query_case("chunked_prefill", seed=77 + group, ctx_override=ctx, q_lens=nq, hq=hkv * group,
                              hkv=hkv, d=d, dtype=dtype)
    gen = torch.Generator().manual_seed(5 + group)
    u = torch.where(torch.rand(d, generator=gen) < 0.5, -1.0, 1.0)
    case["q"] = (2.0 * u + 0.3 * torch.randn(case["q"].shape, generator=gen)).to(case["q"].dtype)
    k = case["k_cache"].float()
    bt = case["block_tables"]
    for s, c in enumerate(ctx):
        for lb in range((c + 15) // 16):
            b = int(bt[s, lb])
            pos = torch.arange(lb * 16, lb * 16 + 16, dtype=torch.float32)
            k[b] = (2.0 * pos / c)[None, :, None] * u + 0.3 * torch.randn(k[b].shape, generator=gen)
    case["k_cache"] = k.to(case["k_cache"].dtype)
    g = gpu_case(case)
    nw, _, _ = P.multi_query_plan(len(ctx), hkv * group, hkv, d, max(ctx), max(nq), g["k_cache"].dtype)
    assert nw == len(ctx) * hkv * (((max(nq) * group + 127) // 128 + 1) // 2)     # the query-major plan
    got = np64(run_mq(g))
    assert np.all(np.isfinite(got))
    check_attn(got, oracle_mq(case))
