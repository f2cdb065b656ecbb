"""The C-ABI library loads without a GPU, exports every entry point that
include/pagedkv.h declares, and rejects bad arguments on the host before any
launch (these calls need no device)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_438_b200 import pagedkv as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "pagedkv.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_438_b200 import build
    build.build()
    return P.lib()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 20
    raw = ctypes.CDLL(P.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert sorted(P.EXPORTS) == declared


def test_version(lib):
    assert lib.pkv_version() >= 10000


def _err(rc, code):
    assert rc == code, (rc, P.lib().pkv_last_error())


def test_write_rejects_bad_block_size_and_dtypes(lib):
    n = ctypes.c_void_p(16)
    _err(lib.pkv_kv_cache_write(n, n, n, n, None, None, None, None, n, 4, 2, 64, 8, 10, P.PKV_F16, P.PKV_F16, None),
         P.PKV_ERR_UNSUPPORTED)
    _err(lib.pkv_kv_cache_write(n, n, n, n, None, None, None, None, n, 4, 2, 96, 16, 10, P.PKV_F16, P.PKV_F16, None),
         P.PKV_ERR_UNSUPPORTED)
    _err(lib.pkv_kv_cache_write(n, n, n, n, None, None, None, None, n, 4, 2, 64, 16, 10, P.PKV_BF16, P.PKV_F16, None),
         P.PKV_ERR_UNSUPPORTED)
    # quantised cache without scale arrays
    _err(lib.pkv_kv_cache_write(n, n, n, n, None, None, None, None, n, 4, 2, 64, 16, 10, P.PKV_BF16, P.PKV_I8, None),
         P.PKV_ERR_INVALID_ARG)
    # asymmetric uint8 cache with scales but no zero points
    _err(lib.pkv_kv_cache_write(n, n, n, n, n, n, None, None, n, 4, 2, 64, 16, 10, P.PKV_BF16, P.PKV_U8ASYM, None),
         P.PKV_ERR_INVALID_ARG)
    assert b"k_zero" in lib.pkv_last_error()
    # misaligned cache pointer
    m = ctypes.c_void_p(18)
    _err(lib.pkv_kv_cache_write(n, n, m, n, None, None, None, None, n, 4, 2, 64, 16, 10, P.PKV_F16, P.PKV_F16, None),
         P.PKV_ERR_INVALID_ARG)
    assert b"aligned" in lib.pkv_last_error()


def test_write_zero_tokens_is_a_noop(lib):
    _err(lib.pkv_kv_cache_write(None, None, None, None, None, None, None, None, None, 0, 2, 64, 16, 10, P.PKV_F16, P.PKV_F16,
                                None), P.PKV_OK)


def _decode(lib, **kw):
    n = ctypes.c_void_p(256)
    a = dict(out=n, q=n, kc=n, vc=n, ks=None, vs=None, kz=None, vz=None, bt=n, cl=n, B=2, hq=8, hkv=2, d=128, bs=16, nb=100, mb=4,
             maxc=64, scale=0.1, win=0, qd=P.PKV_BF16, cd=P.PKV_BF16, pt=0, ws=None, wsb=0)
    a.update(kw)
    return lib.pkv_paged_attention_decode(a["out"], a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["kz"], a["vz"],
                                          a["bt"], a["cl"],
                                          a["B"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["mb"], a["maxc"],
                                          a["scale"], a["win"], a["qd"], a["cd"], a["pt"], a["ws"], a["wsb"], None)


def test_decode_host_rejections(lib):
    n = ctypes.c_void_p(256)
    _err(_decode(lib, hq=7), P.PKV_ERR_INVALID_ARG)              # Hq % Hkv != 0
    _err(_decode(lib, hq=64, hkv=2), P.PKV_ERR_UNSUPPORTED)       # G = 32 > 16
    _err(_decode(lib, d=80), P.PKV_ERR_UNSUPPORTED)
    _err(_decode(lib, bs=32), P.PKV_ERR_UNSUPPORTED)
    _err(_decode(lib, qd=P.PKV_F16), P.PKV_ERR_UNSUPPORTED)       # q dtype must match a 16-bit cache
    _err(_decode(lib, maxc=65), P.PKV_ERR_INVALID_ARG)            # > max_blocks * 16
    _err(_decode(lib, scale=float("nan")), P.PKV_ERR_INVALID_ARG)
    _err(_decode(lib, win=-1), P.PKV_ERR_INVALID_ARG)
    _err(_decode(lib, cd=P.PKV_I8), P.PKV_ERR_INVALID_ARG)        # quantised without scales
    _err(_decode(lib, cd=P.PKV_U8ASYM, ks=n, vs=n), P.PKV_ERR_INVALID_ARG)   # without zero points
    _err(_decode(lib, cd=P.PKV_U8ASYM, ks=n, vs=n, kz=n, vz=ctypes.c_void_p(264)),
         P.PKV_ERR_INVALID_ARG)                                    # misaligned zero points
    _err(_decode(lib, cd=9, ks=n, vs=n), P.PKV_ERR_UNSUPPORTED)   # unknown format
    _err(_decode(lib, pt=24), P.PKV_ERR_INVALID_ARG)              # partition not a multiple of 16
    # split plan needs a workspace
    _err(_decode(lib, maxc=64, pt=16), P.PKV_ERR_INVALID_ARG)
    assert b"workspace" in lib.pkv_last_error()
    _err(_decode(lib, B=0), P.PKV_OK)


def test_plan_is_consistent(lib):
    for (B, hq, hkv, d, ctx) in [(4, 8, 2, 64, 256), (64, 32, 8, 128, 4096), (32, 64, 8, 128, 32768),
                                 (256, 32, 32, 128, 8192), (1, 8, 8, 128, 1)]:
        nw, per, ws = P.decode_plan(B, hq, hkv, d, ctx, P.PKV_BF16)
        items = B * hkv * ((ctx + 15) // 16)
        assert 1 <= nw <= items and per % 16 == 0 and nw * per >= items * 16
        G = hq // hkv
        if nw > 1:
            assert ws >= B * hkv * 8 + 2 * nw * (2 * G + G * d) * 4
    nw, per, ws = P.decode_plan(2, 8, 2, 128, 1000, P.PKV_BF16, partition_tokens=64)
    assert nw == (2 * 2 * 63 + 3) // 4 and per == 64


def test_copy_rejections(lib):
    n = ctypes.c_void_p(256)
    _err(lib.pkv_copy_blocks(n, n, None, None, None, None, n, 3, 2, 128, 16, 10, P.PKV_FP8E4M3, None), P.PKV_ERR_INVALID_ARG)
    _err(lib.pkv_copy_blocks(n, n, None, None, None, None, n, 3, 2, 128, 12, 10, P.PKV_BF16, None), P.PKV_ERR_UNSUPPORTED)
    _err(lib.pkv_copy_blocks(n, n, None, None, None, None, n, 0, 2, 128, 16, 10, P.PKV_BF16, None), P.PKV_OK)
    _err(lib.pkv_copy_blocks(n, n, n, n, None, None, n, 3, 2, 128, 16, 10, P.PKV_U8ASYM, None),
         P.PKV_ERR_INVALID_ARG)


def _mq(lib, **kw):
    n = ctypes.c_void_p(256)
    a = dict(out=n, q=n, kc=n, vc=n, ks=None, vs=None, kz=None, vz=None, bt=n, cl=n, qsl=n, B=2, T=8, mq=4, hq=8,
             hkv=2, d=128, bs=16, nb=100, mb=4, maxc=64, scale=0.1, win=0, qd=P.PKV_BF16, cd=P.PKV_BF16, pt=0,
             ws=None, wsb=0)
    a.update(kw)
    return lib.pkv_paged_attention_multi_query(a["out"], a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["kz"],
                                               a["vz"], a["bt"], a["cl"], a["qsl"], a["B"], a["T"], a["mq"],
                                               a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["mb"], a["maxc"],
                                               a["scale"], a["win"], a["qd"], a["cd"], a["pt"], a["ws"], a["wsb"],
                                               None)


def test_multi_query_host_rejections(lib):
    _err(_mq(lib, qsl=None), P.PKV_ERR_INVALID_ARG)               # no query_start_loc
    _err(_mq(lib, T=-1), P.PKV_ERR_INVALID_ARG)
    _err(_mq(lib, hq=7), P.PKV_ERR_INVALID_ARG)
    _err(_mq(lib, d=96), P.PKV_ERR_UNSUPPORTED)
    _err(_mq(lib, pt=16), P.PKV_ERR_INVALID_ARG)                  # split plan needs a workspace
    assert b"workspace" in lib.pkv_last_error()
    _err(_mq(lib, T=0), P.PKV_OK)                                # nothing to do
    _err(_mq(lib, mq=0), P.PKV_OK)


def test_multi_query_plan_tiles(lib):
    # 4 new tokens x G 4 = 16 columns: one tile per KV head, the decode-style plan
    nw, per, ws = P.multi_query_plan(64, 32, 8, 128, 4096, 4, P.PKV_BF16)
    nwd, _, _ = P.decode_plan(64, 32, 8, 128, 4096, P.PKV_BF16)
    assert nw == nwd
    # 512 new tokens x G 4 = 2048 rows on a 16-bit cache: the query-major
    # kernel, one CTA per (sequence, head, 128-row tile) over all its keys
    nw, per, ws = P.multi_query_plan(8, 32, 8, 128, 4096, 512, P.PKV_BF16)
    assert nw == 8 * 8 * 16 // 2 and per == 4096          # one CTA per pair of 128-row tiles
    # an explicit partition keeps the decode kernel's multi-query mode: one
    # stream per (sequence, head, 16-column tile)... capped by the partition
    nw2, per2, ws2 = P.multi_query_plan(8, 32, 8, 128, 4096, 512, P.PKV_BF16, partition_tokens=4096)
    assert per2 == 4096 and nw2 == 8 * 8 * 128 and ws2 == ws
    # 8-bit caches never take the query-major kernel
    nw3, _, _ = P.multi_query_plan(8, 32, 8, 128, 4096, 512, P.PKV_I8)
    assert nw3 == 8 * 8 * 128


def test_small_batches_get_shorter_streams(lib):
    # without a GPU the plan assumes the B200's 148 SMs (as on one): 8 warps each
    wave = 8 * 148
    # 4 sequences x 2 heads x 16 blocks = 128 blocks, far below a wave of
    # 16-block streams: streams of 4 blocks (64 tokens) spread it over 32 warps
    nw, per, _ = P.decode_plan(4, 8, 2, 64, 256, P.PKV_BF16)
    assert (nw, per) == (32, 64)
    # 16 x 8 x 128 blocks: a full wave of shorter streams rather than 128 of 16 blocks
    nw, per, _ = P.decode_plan(16, 32, 8, 128, 2048, P.PKV_BF16)
    assert nw == wave and per < 16 * 16
    # enough work for a wave of 16-block streams: unchanged
    nw, per, _ = P.decode_plan(64, 32, 8, 128, 4096, P.PKV_BF16)
    assert nw == wave and per >= 16 * 16


def test_quantised_caches_run_twelve_warps_per_sm_unless_pairs_are_wide(lib):
    # quantised caches: 12 warps per SM (168 registers each) for pairs of up
    # to 8 columns; 16-column pairs (a GQA group of 16) keep 8
    for code in (P.PKV_I8, P.PKV_FP8E4M3, P.PKV_U8ASYM, P.PKV_I4, P.PKV_FP4E2M1):
        nw, _, _ = P.decode_plan(256, 32, 32, 128, 8192, code)
        assert nw == 12 * 148
        nw, _, _ = P.decode_plan(64, 256, 16, 128, 8192, code)
        assert nw == 8 * 148
    # a 16-bit cache of the same shape: 8 warps per SM, long streams included
    nw, _, _ = P.decode_plan(256, 32, 32, 128, 8192, P.PKV_BF16)
    assert nw == 8 * 148
    nw, _, _ = P.decode_plan(32, 64, 8, 128, 32768, P.PKV_BF16)
    assert nw == 8 * 148


def test_very_large_batches_step_down_to_fewer_warps(lib):
    # a decode CTA holds the context-length scan ((B + 1) x 4 bytes) beside
    # its warps' rings: 16-bit caches at head_dim 128 keep 8 warps up to
    # ~25,000 sequences and run 4 beyond
    nw, _, _ = P.decode_plan(20000, 8, 8, 128, 1024, P.PKV_BF16)
    assert nw == 8 * 148
    nw, _, _ = P.decode_plan(30000, 8, 8, 128, 1024, P.PKV_BF16)
    assert nw == 4 * 148
    # head_dim 64 rings are half the size: 8 warps still fit
    nw, _, _ = P.decode_plan(30000, 8, 8, 64, 1024, P.PKV_BF16)
    assert nw == 8 * 148
    # quantised caches step from 12 warps to 8
    nw, _, _ = P.decode_plan(30000, 32, 32, 128, 1024, P.PKV_I8)
    assert nw == 8 * 148


def test_query_major_routing_threshold_and_group(lib):
    def mq(hq, d, n, cd=P.PKV_BF16):
        return P.multi_query_plan(2, hq, 8, d, 1024, n, cd)[0]
    # the query-major plan: 2 sequences x 8 KV heads x pairs of 128-row tiles
    assert mq(32, 128, 32) == 2 * 8 * 1             # 32 new tokens x G 4 = 128 rows: one tile
    assert mq(32, 64, 512) == 2 * 8 * 8             # head_dim 64 qualifies (16 tiles, 8 pairs)
    assert mq(32, 128, 512, P.PKV_F16) == 2 * 8 * 8  # so does an fp16 cache
    # below 128 rows, or a group that does not divide 128: the decode kernel's
    # multi-query mode, one stream per (sequence, head, 16-column tile)
    assert mq(32, 128, 31) == 2 * 8 * ((31 * 4 + 15) // 16)
    assert mq(24, 128, 512) == 2 * 8 * ((512 * 3 + 15) // 16)
