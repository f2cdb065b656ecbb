"""The allocation-free decode entry point against the regular one.

pkv_paged_attention_decode_noalloc serves callers that cannot allocate device
memory (a plugin whose host framework owns all device allocations, or a
latency-critical loop where cudaMalloc could synchronise the device); its
split-KV partials live in the library's own fixed device array.  With the
same partition_tokens both entry points run the same kernel on the same plan,
so their outputs must agree bit for bit.  This file is collected last so that
a failure here leaves every other test already run; it passes alone in a
fresh process and after the rest of the suite.
"""
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_438_b200 import inputs as I
from paged_kv_cache_438_b200 import pagedkv as P

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
ATOL, MEANREL = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_kv_cache_438_b200 import build
    build.build()
    P.lib()


def _case(seed, batch, cache_kind=None, name="llama3_8b"):
    c = I.device_decode_case(name, DEV, seed=seed, batch=batch, cache_kind=cache_kind)
    c["maxc"] = int(c["context_lens_cpu"].max())
    return c


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    err = np.abs(a - b)
    assert err.max() <= ATOL
    assert err.sum() / max(np.abs(b).sum(), 1e-30) <= MEANREL


def _noalloc(c, pt):
    out = torch.empty_like(c["q"])
    P.paged_attention_decode_noalloc(c["q"], c["k_cache"], c["v_cache"], c["block_tables"], c["context_lens"],
                                     c["scale"], c["maxc"], out, k_scale=c.get("k_scale"), v_scale=c.get("v_scale"),
                                     k_zero=c.get("k_zero"), v_zero=c.get("v_zero"), partition_tokens=pt)
    return out


def _with_workspace(c, pt):
    _, _, wsb = P.decode_plan(c["batch"], c["hq"], c["hkv"], c["d"], c["maxc"], c["k_cache"].dtype, pt)
    return P.paged_attention_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"], c["context_lens"],
                                    c["scale"], c.get("k_scale"), c.get("v_scale"), max_context_len=c["maxc"],
                                    partition_tokens=pt, workspace=P.new_workspace(DEV, wsb),
                                    k_zero=c.get("k_zero"), v_zero=c.get("v_zero"))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [_case(2024, 16), _case(2025, 24)]
    outs = []
    for c in cases:
        # at most 1024 tokens per warp stream: many pairs split, so the scratch array is used
        np_, _, ws = P.decode_plan(c["batch"], c["hq"], c["hkv"], c["d"], c["maxc"], c["k_cache"].dtype, 1024)
        assert np_ > 1 and 0 < ws <= P.NOALLOC_SCRATCH_BYTES
        outs.append(_noalloc(c, 1024))
    torch.cuda.synchronize()
    for c, out in zip(cases, outs):
        ref = _with_workspace(c, 1024)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert P.device_status(clear=True) == 0


def test_noalloc_calls_that_grow_and_shrink_through_the_shared_array():
    """Calls whose (sequence, KV head) pair counts and GQA groups go up and
    down, on 16-bit, INT8 and FP8 caches: every call's counter area lands on
    bytes an earlier call used for partials, and the result must still be the
    workspace entry point's, bit for bit."""
    seq = [_case(40, 8), _case(41, 48, "int8", "quant_mha"), _case(42, 4), _case(43, 24, "fp8", "quant_mha"),
           _case(44, 32), _case(45, 6, "int8", "quant_mha"), _case(40, 8)]
    got, pts = [], []
    for c in seq:
        # the shortest explicit partition whose partials fit the array (many splits)
        for pt in (512, 1024, 2048, 4096):
            n, _, ws = P.decode_plan(c["batch"], c["hq"], c["hkv"], c["d"], c["maxc"], c["k_cache"].dtype, pt)
            if ws <= P.NOALLOC_SCRATCH_BYTES:
                break
        assert n > 1 and ws <= P.NOALLOC_SCRATCH_BYTES
        pts.append(pt)
        got.append(_noalloc(c, pt))
    torch.cuda.synchronize()
    assert P.device_status(clear=True) == 0
    for c, out, pt in zip(seq, got, pts):
        ref = _with_workspace(c, pt)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert torch.equal(got[0], got[-1])
    assert P.device_status(clear=True) == 0


def test_noalloc_rejects_work_beyond_its_scratch():
    # 4096 sequences x 8 KV heads x 256 blocks split into 16-block streams need far more partials
    big_b, hq, hkv, d, maxc = 4096, 64, 8, 128, 16 * 256
    _, _, ws = P.decode_plan(big_b, hq, hkv, d, maxc, torch.bfloat16, 256)
    assert ws > P.NOALLOC_SCRATCH_BYTES
    q = torch.empty((big_b, hq, d), dtype=torch.bfloat16, device=DEV)
    bt = torch.zeros((big_b, 256), dtype=torch.int32, device=DEV)
    cl = torch.zeros(big_b, dtype=torch.int32, device=DEV)
    kc = torch.empty((8, hkv, 16, d), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(P.PagedKVError, match="scratch"):
        P.paged_attention_decode_noalloc(q, kc, kc, bt, cl, 1 / math.sqrt(d), maxc, torch.empty_like(q),
                                         partition_tokens=256)


def test_noalloc_lengthens_streams_when_the_automatic_plan_needs_more_scratch():
    # a GQA group of 16 (128 q / 8 KV heads): with the automatic plan the
    # partials of a full wave of warp streams need ~19.7 MB, more than the
    # built-in array; the call runs the same work in fewer, longer streams,
    # a plan of its own, so it is checked against the fp64 oracle directly
    from oracle import attention as OA
    case = I.decode_case("llama3_8b", seed=31, batch=16, hq=128, hkv=8)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    maxc = int(case["context_lens"].max())
    _, _, ws = P.decode_plan(16, 128, 8, 128, maxc, g["k_cache"].dtype)
    assert ws > P.NOALLOC_SCRATCH_BYTES
    out = torch.empty_like(g["q"])
    P.paged_attention_decode_noalloc(g["q"], g["k_cache"], g["v_cache"], g["block_tables"], g["context_lens"],
                                     g["scale"], maxc, out)
    ref = P.paged_attention_decode(g["q"], g["k_cache"], g["v_cache"], g["block_tables"], g["context_lens"],
                                   g["scale"], max_context_len=maxc)
    torch.cuda.synchronize()
    assert P.device_status(clear=True) == 0
    want = OA.paged_decode_attention(case["q"].double().numpy(), case["k_cache"].double().numpy(),
                                     case["v_cache"].double().numpy(), case["block_tables"].numpy(),
                                     case["context_lens"].numpy(), case["scale"])
    got = out.double().cpu().numpy()
    err = np.abs(got - want)
    assert err.max() <= ATOL
    assert err.sum() / np.abs(want).sum() <= MEANREL
    _close(out, ref)
