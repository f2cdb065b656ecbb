"""The allocation-free decode entry point against the regular one.

pkv_paged_attention_decode_noalloc serves callers that cannot allocate device
memory (a plugin whose host framework owns all device allocations, or a
latency-critical loop where cudaMalloc could synchronise the device); its
split-KV partials live in the library's own fixed device array.  This file is
collected last so that a failure here leaves every other test already run;
it passes alone in a fresh process and after the rest of the suite.
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


def _case(seed, batch):
    c = I.device_decode_case("llama3_8b", DEV, seed=seed, batch=batch)
    c["maxc"] = int(c["context_lens_cpu"].max())
    return c


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    err = np.abs(a - b)
    assert err.max() <= ATOL
    assert err.sum() / max(np.abs(b).sum(), 1e-30) <= MEANREL


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [_case(2024, 16), _case(2025, 24)]
    outs = []
    for c in cases:
        # at most 1024 tokens per warp stream: many pairs split, so the scratch array is used
        np_, _, ws = P.decode_plan(c["batch"], c["hq"], c["hkv"], c["d"], c["maxc"], c["k_cache"].dtype, 1024)
        assert np_ > 1 and ws > 0   # several warp streams: partials go through the library's array
        out = torch.empty_like(c["q"])
        P.paged_attention_decode_noalloc(c["q"], c["k_cache"], c["v_cache"], c["block_tables"], c["context_lens"],
                                         c["scale"], c["maxc"], out, partition_tokens=1024)
        outs.append(out)
    torch.cuda.synchronize()
    for c, out in zip(cases, outs):
        ref = P.paged_attention_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"], c["context_lens"],
                                       c["scale"], max_context_len=c["maxc"], partition_tokens=1024)
        torch.cuda.synchronize()
        _close(out, ref)
    assert P.device_status(clear=True) == 0


def test_noalloc_rejects_work_beyond_its_scratch():
    c = _case(7, 4)
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
    del c


def test_noalloc_lengthens_streams_when_the_automatic_plan_needs_more_scratch():
    # a GQA group of 16 (128 q / 8 KV heads): with the automatic plan the
    # partials of a full wave of warp streams need ~19.7 MB, more than the
    # built-in array; the call runs the same work in fewer, longer streams
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
    _close(out, ref)
    assert P.device_status(clear=True) == 0
