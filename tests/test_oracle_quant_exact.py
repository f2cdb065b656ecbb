"""Exact-rational pins of the oracle's symmetric absmax quantisers.

The rule (ascendai.csdn.net article, §三 KV Cache量化; per (token, head),
reduced over head_dim as "大模型推理的KV Cache管理…优化实战" §四 reduces its
statistics): a = max |x|, s = a / qmax rounded once to fp32, y = x / s
rounded once to fp32 (an IEEE division, not a multiply by 1 / s), then y
rounded to the code grid, nearest with ties to even.  Here every step is
computed on exact rationals (``fractions.Fraction``) with rounding written
out from its definition, and the oracle must agree code for code and scale
for scale: on random rows at scales far from 1, and on hand rows found by
search where the division and a reciprocal multiply round to different codes
(so an oracle that multiplied by 1 / s would fail here).
"""
from fractions import Fraction as F

import numpy as np
import pytest

from oracle import quant as Q


# ------------------------------------------------------- exact reference --

def f32_round(q):
    """The fp32 value nearest to the rational q, ties to the even
    significand (normal and subnormal range; no overflow in these tests)."""
    if q == 0:
        return F(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+1), up to one step
    while F(2) ** e > a:
        e -= 1
    while F(2) ** (e + 1) <= a:
        e += 1
    quantum = F(2) ** (max(e, -126) - 23)                       # 24-bit significand
    return sign * round(a / quantum) * quantum                  # Fraction rounds half to even


def e4m3_grid():
    """(value, code) of every finite non-negative E4M3 code (OCP FP8: bias
    7, 3 mantissa bits, subnormals m * 2^-9, largest 448)."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        out.append((F(m, 512) if e == 0 else F(8 + m, 8) * F(2) ** (e - 7), c))
    return out


E2M1_GRID = [(F(0), 0), (F(1, 2), 1), (F(1), 2), (F(3, 2), 3), (F(2), 4), (F(3), 5), (F(4), 6), (F(6), 7)]


def nearest_on_grid(y, grid):
    """Magnitude code of the grid value nearest to |y|, ties to the even
    code (its lowest mantissa bit clear)."""
    a = abs(y)
    return min(grid, key=lambda vc: (abs(vc[0] - a), vc[1] & 1))[1]


def exact_int(x_row, qmax):
    """Integer codes and the scale of one row (INT8: qmax 127, INT4: 7)."""
    xs = [F(float(v)) for v in x_row]
    a = max(abs(v) for v in xs)
    s = f32_round(a / qmax)
    if s == 0:
        return [0] * len(xs), s
    return [max(-qmax, min(qmax, round(f32_round(v / s)))) for v in xs], s


def exact_float(x_row, qmax, grid, sign_bit):
    """Minifloat codes (FP8 E4M3: qmax 448, FP4 E2M1: 6) and the scale."""
    xs = [F(float(v)) for v in x_row]
    a = max(abs(v) for v in xs)
    s = f32_round(a / qmax)
    if s == 0:
        return [0] * len(xs), s
    codes = []
    for v, neg in zip(xs, np.signbit(np.asarray(x_row, np.float32))):
        # y = x / s has the sign of x (s > 0), zero included: the sign bit is x's
        y = max(-F(qmax), min(F(qmax), f32_round(v / s)))
        codes.append(nearest_on_grid(y, grid) | (sign_bit if neg else 0))
    return codes, s


def recip_codes_int(x_row, qmax):
    """The same rule with y = x * fp32(1 / s) (the reading the pins forbid)."""
    x = np.asarray(x_row, np.float32)
    s = np.float32(np.max(np.abs(x)) / np.float32(qmax))
    r = np.float32(np.float32(1.0) / s)
    return np.clip(np.rint((x * r).astype(np.float32)), -qmax, qmax).astype(np.int64)


def recip_codes_float(x_row, qmax, grid, sign_bit):
    x = np.asarray(x_row, np.float32)
    s = np.float32(np.max(np.abs(x)) / np.float32(qmax))
    r = np.float32(np.float32(1.0) / s)
    y = np.clip((x * r).astype(np.float32), -qmax, qmax)
    return [nearest_on_grid(F(float(v)), grid) | (sign_bit if neg else 0) for v, neg in zip(y, np.signbit(x))]


# ---------------------------------------------------------- the formats --

def _oracle_int8(x):
    q, s = Q.quantize_int8(x[None])
    return q[0].astype(np.int64).tolist(), s[0]


def _oracle_int4(x):
    packed, s = Q.quantize_int4(x[None])
    return Q.int4_values(packed)[0].astype(np.int64).tolist(), s[0]


def _oracle_fp8(x):
    c, s = Q.quantize_fp8_e4m3(x[None])
    return c[0].astype(np.int64).tolist(), s[0]


def _oracle_fp4(x):
    packed, s = Q.quantize_fp4_e2m1(x[None])
    return Q.unpack_nibbles(packed)[0].astype(np.int64).tolist(), s[0]


E4M3 = e4m3_grid()
FORMATS = {
    # name: (oracle, exact reference, reciprocal-multiply variant, rounding boundaries of |y|)
    "int8": (_oracle_int8, lambda x: exact_int(x, 127), lambda x: recip_codes_int(x, 127).tolist(),
             [F(2 * k + 1, 2) for k in range(127)]),
    "int4": (_oracle_int4, lambda x: exact_int(x, 7), lambda x: recip_codes_int(x, 7).tolist(),
             [F(2 * k + 1, 2) for k in range(7)]),
    "fp8": (_oracle_fp8, lambda x: exact_float(x, 448, E4M3, 0x80),
            lambda x: recip_codes_float(x, 448, E4M3, 0x80),
            [(E4M3[i][0] + E4M3[i + 1][0]) / 2 for i in range(len(E4M3) - 1)]),
    "fp4": (_oracle_fp4, lambda x: exact_float(x, 6, E2M1_GRID, 0x8),
            lambda x: recip_codes_float(x, 6, E2M1_GRID, 0x8),
            [(E2M1_GRID[i][0] + E2M1_GRID[i + 1][0]) / 2 for i in range(len(E2M1_GRID) - 1)]),
}


def test_f32_round_matches_the_ieee_cast_of_doubles():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-30, 30, 3000),
                        rng.standard_normal(200) * 1e-40])
    for v in x:
        assert f32_round(F(float(v))) == F(float(np.float32(v)))
    # a tie between two fp32 neighbours goes to the even significand
    one = F(1)
    assert f32_round(one + F(1, 2 ** 24)) == one
    assert f32_round(one + F(3, 2 ** 24)) == one + F(2, 2 ** 23)


def test_exact_reference_agrees_with_hand_values():
    # a = 127 gives s = 1 exactly: codes are the inputs rounded half to even
    codes, s = exact_int(np.array([127.0, 2.5, -3.5, 0.5, -0.5, 1.5], np.float32), 127)
    assert s == 1 and codes == [127, 2, -4, 0, 0, 2]
    codes, s = exact_float(np.array([448.0, 272.0, 304.0, -0.0], np.float32), 448, E4M3, 0x80)
    # 272 lies halfway between 256 (code 0x78) and 288 (0x79): even code 0x78; 304 -> 0x7A (320)
    assert s == 1 and codes == [0x7E, 0x78, 0x7A, 0x80]


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_random_rows_at_non_unit_scales_match_exactly(fmt):
    oracle, exact, _, _ = FORMATS[fmt]
    rng = np.random.default_rng(12)
    for i in range(40):
        scale = 10.0 ** rng.uniform(-4, 4)
        x = (rng.standard_normal(64) * scale).astype(np.float32)
        codes, s = exact(x)
        got, gs = oracle(x)
        assert F(float(gs)) == s, (fmt, i)
        assert got == codes, (fmt, i)


def _division_vs_reciprocal_rows(fmt, want=6):
    """Rows [a, x, -x, 0] whose x and -x round to different codes under the
    division and under a reciprocal multiply: candidates are the fp32
    neighbours of s times each rounding boundary of the code grid."""
    _, exact, recip, bounds = FORMATS[fmt]
    rng = np.random.default_rng(13)
    found = []
    for _ in range(200):
        a = np.float32(rng.uniform(0.5, 2.0) * 10.0 ** rng.uniform(-3, 3))
        qmax = {"int8": 127, "int4": 7, "fp8": 448, "fp4": 6}[fmt]
        s = f32_round(F(float(a)) / qmax)
        for b in bounds:
            t = np.float32(float(b * s))
            cand = [t]
            lo = hi = t
            for _ in range(12):
                lo = np.nextafter(lo, np.float32(-np.inf))
                hi = np.nextafter(hi, np.float32(np.inf))
                cand += [lo, hi]
            for x in cand:
                if not (0 < x < a):
                    continue
                row = np.array([a, x, -x, 0.0], np.float32)   # even length: two 4-bit codes per byte
                if exact(row)[0] != recip(row):
                    found.append(row)
                    break
            if len(found) >= want:
                return found
    return found


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_rows_where_division_and_reciprocal_multiply_disagree(fmt):
    oracle, exact, recip, _ = FORMATS[fmt]
    rows = _division_vs_reciprocal_rows(fmt)
    assert rows, f"no discriminating row found for {fmt}"
    for row in rows:
        codes, s = exact(row)
        assert recip(row) != codes            # the row tells the two readings apart
        got, gs = oracle(row)
        assert F(float(gs)) == s
        assert got == codes                   # and the oracle takes the division
