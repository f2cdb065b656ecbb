"""Pins for the oracle's quantising rule and its own E4M3 encoder/decoder.

The encoder is checked exhaustively against torch's float8_e4m3fn cast (a
library routine implementing the same OCP definition); the INT8 / FP8 rules
are pinned by invariants of round-to-nearest-even absmax quantisation and by
hand-built tie cases.
"""
import numpy as np
import torch

from oracle import quant as Q


def _torch_codes(y):
    return torch.from_numpy(np.asarray(y, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = Q.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0 and nan.sum() == 2


def test_e4m3_encode_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = Q.e4m3_decode(codes)
    assert np.array_equal(Q.e4m3_encode(vals), codes)


def test_e4m3_encode_ties_and_neighbours_match_torch():
    pos = np.sort(Q.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2
    y = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                        np.nextafter(mids.astype(np.float32), np.float32(-np.inf))]).astype(np.float32)
    y = np.concatenate([y, -y])
    assert np.array_equal(Q.e4m3_encode(y), _torch_codes(y))


def test_e4m3_encode_random_fp32_match_torch():
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.uniform(-448, 448, 200000),
                        rng.standard_normal(200000) * 0.01,
                        rng.standard_normal(100000) * 1e-3]).astype(np.float32)
    assert np.array_equal(Q.e4m3_encode(y), _torch_codes(y))


def test_e4m3_negative_zero_keeps_sign():
    assert Q.e4m3_encode(np.array([-0.0]))[0] == 0x80
    assert Q.e4m3_encode(np.array([0.0]))[0] == 0x00


def test_int8_invariants():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((500, 4, 128)).astype(np.float32)
    q, s = Q.quantize_int8(x)
    assert q.dtype == np.int8 and np.all(np.abs(q.astype(np.int32)) <= 127)
    a = np.abs(x).max(-1)
    assert np.array_equal(s, (a / np.float32(127)).astype(np.float32))
    # the element at the absmax maps to +-127
    idx = np.abs(x).argmax(-1)
    top = np.take_along_axis(q, idx[..., None], -1)[..., 0]
    assert np.all(np.abs(top.astype(np.int32)) == 127)
    # round-to-nearest: |x - q s| <= s / 2 up to the fp32 division rounding
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s[..., None].astype(np.float64))
    assert np.all(err <= s[..., None] * (0.5 + 1e-5))


def test_int8_ties_round_half_to_even():
    x = np.array([[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 126.5]], np.float32)
    q, s = Q.quantize_int8(x)
    assert s[0] == 1.0
    assert q[0].tolist() == [127, 2, 4, -2, -4, 0, 0, 2, 126]


def test_int8_dequantize_is_code_times_scale_within_half_a_step():
    # hand case: codes times the row's scale, exactly
    y = Q.dequantize_int8(np.array([[127, -3, 0]], np.int8), np.array([0.5], np.float32))
    assert y.tolist() == [[63.5, -1.5, 0.0]]
    # round trip through the quantiser: within half a quantisation step
    rng = np.random.default_rng(11)
    x = rng.standard_normal((200, 4, 64)).astype(np.float32)
    q, s = Q.quantize_int8(x)
    err = np.abs(x.astype(np.float64) - Q.dequantize_int8(q, s))
    assert np.all(err <= s[..., None].astype(np.float64) * (0.5 + 1e-5))


def test_int8_zero_row():
    q, s = Q.quantize_int8(np.zeros((2, 8), np.float32))
    assert np.all(q == 0) and np.all(s == 0)


def test_fp8_invariants():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((500, 4, 128)).astype(np.float32)
    c, s = Q.quantize_fp8_e4m3(x)
    v = Q.e4m3_decode(c)
    assert np.all(np.abs(v) <= 448)
    idx = np.abs(x).argmax(-1)
    top = np.take_along_axis(v, idx[..., None], -1)[..., 0]
    assert np.all(np.abs(top) == 448.0)
    # relative error of a normal e4m3 value is at most half a unit of the 3-bit mantissa
    y = x.astype(np.float64) / s[..., None]
    normal = np.abs(y) >= 2 ** -6
    assert np.all(np.abs(v - y)[normal] <= np.abs(y)[normal] * 2 ** -4 * (1 + 1e-6))
    assert np.all(np.abs(v - y)[~normal] <= 2 ** -10 * (1 + 1e-6))


def test_fp8_zero_row_and_dequant():
    c, s = Q.quantize_fp8_e4m3(np.zeros((1, 16), np.float32))
    assert np.all(c == 0) and s[0] == 0
    x = np.array([[448.0, -224.0, 1.0, 0.0]], np.float32)
    c, s = Q.quantize_fp8_e4m3(x)
    assert s[0] == 1.0
    assert np.array_equal(Q.dequantize_fp8_e4m3(c, s)[0], x[0].astype(np.float64))


# ---- asymmetric uint8 with zero point ("大模型推理的KV Cache管理…优化实战", §四) ----

def test_u8_asym_exact_grid_row():
    # min -51, max 204: scale (204 + 51) / 255 = 1, zero point 51, codes x + 51,
    # and every value on the integer grid dequantises exactly
    x = np.array([[-51.0, 0.0, 100.0, 204.0, -3.0]], np.float32)
    c, s, z = Q.quantize_u8_asym(x)
    assert s[0] == 1.0 and z[0] == 51
    assert c[0].tolist() == [0, 51, 151, 255, 48]
    assert np.array_equal(Q.dequantize_u8_asym(c, s, z)[0], x[0].astype(np.float64))


def test_u8_asym_ties_round_half_to_even():
    # scale 1, -min / scale = 0.5 -> zero point 0 (even); (x - min) = 0, 0.5,
    # 1.5, 2.5, 255 -> codes 0, 0, 2, 2, 255
    x = np.array([[-0.5, 0.0, 1.0, 2.0, 254.5]], np.float32)
    c, s, z = Q.quantize_u8_asym(x)
    assert s[0] == 1.0 and z[0] == 0
    assert c[0].tolist() == [0, 0, 2, 2, 255]
    # the two roundings can stack: x = 1 comes back as 2, one full step off
    assert Q.dequantize_u8_asym(c, s, z)[0].tolist() == [0.0, 0.0, 2.0, 2.0, 255.0]


def test_u8_asym_codes_are_nearest_of_all_256():
    # brute force: every code is the nearest of all 256 levels to (x - min) / s
    # (ties to the even level), with the division done in fp32 as stated
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 24)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    c, s, z = Q.quantize_u8_asym(x)
    lo = x.min(-1)
    levels = np.arange(256, dtype=np.float64)
    for i in range(x.shape[0]):
        y = ((x[i] - lo[i]) / s[i]).astype(np.float32).astype(np.float64)
        for e in range(x.shape[1]):
            d = np.abs(y[e] - levels)
            ties = levels[d == d.min()]
            pick = ties[0] if len(ties) == 1 else ties[np.mod(ties, 2) == 0][0]
            assert c[i, e] == pick
        zy = np.float32(-lo[i] / s[i])
        assert z[i] == min(255, max(0, int(np.rint(zy))))


def test_u8_asym_invariants_random():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((400, 4, 128)).astype(np.float32)
    c, s, z = Q.quantize_u8_asym(x)
    assert c.dtype == np.uint8 and z.dtype == np.uint8 and s.dtype == np.float32
    lo, hi = x.min(-1), x.max(-1)
    assert np.array_equal(s, ((hi - lo) / np.float32(255)).astype(np.float32))
    # the minimum maps to code 0 and the maximum to 255; codes are monotone in x
    assert np.all(np.take_along_axis(c, x.argmin(-1)[..., None], -1) == 0)
    assert np.all(np.take_along_axis(c, x.argmax(-1)[..., None], -1) == 255)
    order = np.argsort(x, axis=-1)
    assert np.all(np.diff(np.take_along_axis(c.astype(np.int32), order, -1), axis=-1) >= 0)
    # each code is within half a step of (x - min) / s; with the rounded zero
    # point the reconstruction is within one step (rows here contain 0)
    s64 = s.astype(np.float64)[..., None]
    off = c.astype(np.float64) * s64 + lo.astype(np.float64)[..., None]
    assert np.all(np.abs(off - x) <= s64 * (0.5 + 1e-5))
    xh = Q.dequantize_u8_asym(c, s, z)
    assert np.all(np.abs(xh - x) <= s64 * (1.0 + 1e-5))


def test_u8_asym_rows_not_containing_zero_follow_the_page():
    # all positive: -min / scale < 0 clamps the zero point to 0 and the row
    # comes back shifted by -min; all negative: it clamps to 255, shift -max
    x = np.array([[1.0, 256.0, 11.0], [-256.0, -1.0, -246.0]], np.float32)
    c, s, z = Q.quantize_u8_asym(x)
    assert s.tolist() == [1.0, 1.0] and z.tolist() == [0, 255]
    assert c.tolist() == [[0, 255, 10], [0, 255, 10]]
    xh = Q.dequantize_u8_asym(c, s, z)
    assert xh.tolist() == [[0.0, 255.0, 10.0], [-255.0, 0.0, -245.0]]


def test_u8_asym_constant_row():
    c, s, z = Q.quantize_u8_asym(np.full((2, 16), 3.25, np.float32))
    assert np.all(c == 0) and np.all(s == 0) and np.all(z == 0)


def test_grouped_equals_per_row_for_any_group_size():
    # the page's grouped form reduces over head_dim inside each token group,
    # so grouping never changes a (token, head) row's scale, zero point or codes
    rng = np.random.default_rng(5)
    kv = rng.standard_normal((3, 300, 64)).astype(np.float32)
    ref = Q.quantize_u8_asym(kv)
    for gs in (128, 7, 1, 300, 512):
        got = Q.quantize_grouped(kv, gs)
        for a, b in zip(got, ref):
            assert a.shape == b.shape and np.array_equal(a, b)
    # a reduction over the wrong axis would break the per-row extremes
    c, s, z = Q.quantize_grouped(kv, 128)
    assert np.all(c.max(-1) == 255) and np.all(c.min(-1) == 0)


# ---- 4-bit: INT4 and FP4 E2M1 ----

def test_e2m1_decode_table():
    vals = Q.e2m1_decode(np.arange(16))
    assert vals[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert vals[8:].tolist() == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_encode_is_nearest_with_ties_to_even_by_brute_force():
    grid = Q.e2m1_decode(np.arange(8))          # non-negative magnitudes, codes 0..7
    rng = np.random.default_rng(7)
    mids = (grid[:-1] + grid[1:]) / 2
    y = np.concatenate([rng.uniform(-6, 6, 20000), grid, -grid, mids, -mids,
                        np.nextafter(mids, 7), np.nextafter(mids, -1)])
    codes = Q.e2m1_encode(y)
    for v, c in zip(y.tolist(), codes.tolist()):
        d = np.abs(abs(v) - grid)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else best[best % 2 == 0][0]   # even mantissa bit
        assert (c & 0x7) == want, (v, c)
        if abs(v) > 0 or np.signbit(v):
            assert (c >> 3) == int(np.signbit(v))


def test_nibble_packing_layout():
    c = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    p = Q.pack_nibbles(c)
    assert p.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(Q.unpack_nibbles(p), c)


def test_int4_invariants_and_ties():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((300, 4, 128)).astype(np.float32)
    p, s = Q.quantize_int4(x)
    v = Q.int4_values(p)
    assert p.shape == (300, 4, 64) and np.all(np.abs(v) <= 7)
    top = np.take_along_axis(v, np.abs(x).argmax(-1)[..., None], -1)[..., 0]
    assert np.all(np.abs(top) == 7)
    err = np.abs(x - v * s[..., None])
    assert np.all(err <= s[..., None] * (0.5 + 1e-5))
    # scale 1: ties to even, negative codes as two's complement nibbles
    p, s = Q.quantize_int4(np.array([[7.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, -7.0]], np.float32))
    assert s[0] == 1.0
    assert Q.int4_values(p)[0].tolist() == [7, 2, 4, -2, -4, 0, 0, -7]
    assert Q.unpack_nibbles(p)[0].tolist() == [7, 2, 4, 14, 12, 0, 0, 9]


def test_fp4_invariants_and_zero_rows():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((300, 4, 64)).astype(np.float32)
    p, s = Q.quantize_fp4_e2m1(x)
    v = Q.fp4_values(p)
    top = np.take_along_axis(v, np.abs(x).argmax(-1)[..., None], -1)[..., 0]
    assert np.all(np.abs(top) == 6.0)
    y = x.astype(np.float64) / s[..., None]
    # within half a grid step of the nearest representable value
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    step = np.where(np.abs(y) < 2, 0.5, np.where(np.abs(y) < 4, 1.0, 2.0))
    assert np.all(np.abs(np.abs(v) - np.abs(y)) <= step / 2 + 1e-6)
    p0, s0 = Q.quantize_fp4_e2m1(np.zeros((1, 8), np.float32))
    assert np.all(p0 == 0) and s0[0] == 0
    p, s = Q.quantize_fp4_e2m1(np.array([[6.0, 5.0, -5.0, 2.5, 0.25, 0.75, 1.25, 0.0]], np.float32))
    assert s[0] == 1.0
    assert Q.fp4_values(p)[0][:7].tolist() == [6.0, 4.0, -4.0, 2.0, 0.0, 1.0, 1.0]
