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
