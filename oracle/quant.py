"""KV quantisation rules (oracle; test infrastructure only).

Two families: per-token-per-head symmetric absmax INT8 / FP8-e4m3 (this
docstring), and the page's own asymmetric uint8 rule with a zero point
(``quantize_u8_asym`` and ``quantize_grouped`` further down, with their
readings).

The pages store the KV cache at reduced precision to halve its size: INT8
"几乎无精度损失" and FP8 as a 2x saving (ascendai.csdn.net article, §三 进阶优化
1. KV Cache量化; "KV Cache 与 PagedAttention", §三个直接推论 table: KV 量化
（FP8/INT8）).  The grain used here is one scale per (token, KV head), reduced
over head_dim, as the page "大模型推理的KV Cache管理…优化实战" §四 reduces its
per-channel statistics over the last (head_dim) axis.  The rule is symmetric
absmax (the pages leave the exact scheme open; this is the stated reading):

* a = max_d |x_d| in fp32 (x taken as fp32 from the 16-bit input);
* INT8: s = a / 127 (IEEE fp32 division); q_d = clamp(rint(x_d / s), -127, 127),
  the division IEEE fp32 and rint half-to-even;
* FP8-e4m3: s = a / 448; y_d = clamp(x_d / s, -448, 448) (IEEE fp32);
  q_d = e4m3(y_d) rounded to nearest, ties to even;
* a = 0 gives s = 0 and q = 0 (no division is performed).

The e4m3 encoder / decoder below is written from the OCP 8-bit floating point
definition of E4M3: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
subnormals (exponent field 0) of value m * 2^-9, largest finite 448, no
infinities, and code S.1111.111 reserved for NaN.
"""
import numpy as np

INT8_QMAX = 127
FP8_E4M3_MAX = 448.0


def e4m3_decode(codes):
    """uint8 E4M3 codes -> fp64 values (NaN for the two NaN codes)."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e.astype(np.float64) - 10))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(y):
    """fp32/fp64 values with |y| <= 448 -> uint8 E4M3 codes, round to nearest
    even.  The sign of zero is kept (-0.0 -> 0x80)."""
    y = np.asarray(y, np.float64)
    if np.any(np.abs(y) > FP8_E4M3_MAX) or np.any(np.isnan(y)):
        raise ValueError("e4m3_encode expects finite |y| <= 448")
    sign = np.signbit(y)
    a = np.abs(y)
    _, ex = np.frexp(a)                     # a in [2^(ex-1), 2^ex)
    E = np.maximum(ex - 1, -6)              # binade exponent; below 2^-6 the spacing is 2^-9
    quantum = np.ldexp(1.0, E - 3)          # 3 mantissa bits
    v = np.rint(a / quantum) * quantum      # exact: power-of-two scaling, half-to-even
    # encode the rounded magnitude v
    sub = v < 2.0 ** -6
    m_sub = np.rint(v / 2.0 ** -9)
    _, ex2 = np.frexp(np.where(sub, 1.0, v))
    e_norm = ex2 - 1 + 7
    m_norm = np.rint((np.where(sub, 1.0, v) / np.ldexp(1.0, ex2 - 1) - 1.0) * 8)
    e_field = np.where(sub, 0, e_norm).astype(np.int64)
    m_field = np.where(sub, m_sub, m_norm).astype(np.int64)
    code = (e_field << 3) | m_field
    code = np.where(sign, code | 0x80, code)
    return code.astype(np.uint8)


def absmax_rows(x):
    """fp32 absmax over the last axis."""
    return np.max(np.abs(np.asarray(x, np.float32)), axis=-1)


def quantize_int8(x):
    """x [..., D] (16-bit values as any float array) -> (codes int8 [..., D],
    scales fp32 [...])."""
    x = np.asarray(x, np.float32)
    a = absmax_rows(x)
    s = (a / np.float32(INT8_QMAX)).astype(np.float32)
    q = np.zeros(x.shape, np.int8)
    nz = a > 0
    y = (x[nz] / s[nz][..., None]).astype(np.float32)
    q[nz] = np.clip(np.rint(y), -INT8_QMAX, INT8_QMAX).astype(np.int8)
    return q, s


def quantize_fp8_e4m3(x):
    """x [..., D] -> (codes uint8 [..., D], scales fp32 [...])."""
    x = np.asarray(x, np.float32)
    a = absmax_rows(x)
    s = (a / np.float32(FP8_E4M3_MAX)).astype(np.float32)
    codes = np.zeros(x.shape, np.uint8)
    nz = a > 0
    y = (x[nz] / s[nz][..., None]).astype(np.float32)
    y = np.clip(y, np.float32(-FP8_E4M3_MAX), np.float32(FP8_E4M3_MAX))
    codes[nz] = e4m3_encode(y)
    return codes, s


def dequantize_int8(codes, scales):
    return np.asarray(codes, np.float64) * np.asarray(scales, np.float64)[..., None]


def dequantize_fp8_e4m3(codes, scales):
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[..., None]


# --------------------------------------------------------------------------
# Asymmetric uint8 quantisation with a zero point ("大模型推理的KV Cache管理…
# 优化实战", §四, class KVQuantizationCache: quantize_key, dequantize_key,
# quantize_grouped).  With the page's default per-channel setting the
# statistics are the minimum and maximum over the last (head_dim) axis, so
# every (token, head) row gets its own scale and zero point:
#
#   scale      = (max - min) / 255
#   zero_point = round(-min / scale), clamped to [0, 255], stored as uint8
#   code       = round((x - min) / scale), clamped to [0, 255], uint8
#   x_hat      = (code - zero_point) * scale
#
# Readings where the page leaves a step open:
# * arithmetic is IEEE fp32 from the fp32 value of each 16-bit input (the
#   sketch applies torch ops in the tensor's own dtype; fp32 is the precision
#   the absmax rule above uses too), every round half-to-even;
# * a row with scale 0 (max == min, or a range too small for fp32 / 255) is
#   stored as scale 0, zero point 0 and zero codes (the page's formula would
#   divide by zero there);
# * the page computes the code from (x - min) but dequantises through the
#   rounded, clamped zero point, as written: a row that does not contain 0
#   in [min, max] gets zero point 0 (all positive) or 255 (all negative) and
#   dequantises to x - min or x - max.  This is kept as the page states it.
# --------------------------------------------------------------------------

U8_LEVELS = 255


def quantize_u8_asym(x):
    """x [..., D] -> (codes uint8 [..., D], scales fp32 [...], zero points
    uint8 [...]), statistics over the last axis."""
    x = np.asarray(x, np.float32)
    lo = np.min(x, axis=-1)
    hi = np.max(x, axis=-1)
    s = ((hi - lo) / np.float32(U8_LEVELS)).astype(np.float32)
    codes = np.zeros(x.shape, np.uint8)
    zp = np.zeros(s.shape, np.uint8)
    nz = s > 0
    z = (-lo[nz] / s[nz]).astype(np.float32)
    zp[nz] = np.clip(np.rint(z), 0, U8_LEVELS).astype(np.uint8)
    y = ((x[nz] - lo[nz][..., None]) / s[nz][..., None]).astype(np.float32)
    codes[nz] = np.clip(np.rint(y), 0, U8_LEVELS).astype(np.uint8)
    return codes, s, zp


def dequantize_u8_asym(codes, scales, zero_points):
    """(code - zero_point) * scale in fp64."""
    c = np.asarray(codes, np.float64)
    z = np.asarray(zero_points, np.float64)[..., None]
    return (c - z) * np.asarray(scales, np.float64)[..., None]


def quantize_grouped(kv, group_size=128):
    """kv [num_heads, seq_len, head_dim]: consecutive groups of ``group_size``
    tokens (the last one may be shorter) are quantised independently with
    ``quantize_u8_asym`` and the results concatenated along the token axis.
    Returns (codes, scales, zero points); the page's sketch returns codes and
    scales only, which leaves nothing to dequantise with, so the zero points
    are kept as well."""
    kv = np.asarray(kv, np.float32)
    if kv.ndim != 3:
        raise ValueError("kv must be [num_heads, seq_len, head_dim]")
    n = kv.shape[1]
    num_groups = (n + group_size - 1) // group_size
    parts = [quantize_u8_asym(kv[:, g * group_size:min((g + 1) * group_size, n), :]) for g in range(num_groups)]
    if not parts:
        return (np.zeros(kv.shape, np.uint8), np.zeros(kv.shape[:2], np.float32),
                np.zeros(kv.shape[:2], np.uint8))
    return tuple(np.concatenate([p[i] for p in parts], axis=1) for i in range(3))


# --------------------------------------------------------------------------
# 4-bit KV: INT4 and FP4 (E2M1).  The pages list FP4 KV at a quarter of the
# fp16 size ("ascendai.csdn.net" article, §三 1. KV Cache量化, the precision
# table) and INT4 as the more aggressive step after INT8 ("大模型推理的KV
# Cache管理…优化实战", §四).  They fix no scheme; the reading taken is the
# same per-(token, head) symmetric absmax rule as INT8 / FP8:
#
# * INT4: s = a / 7, code = clamp(rint(x / s), -7, 7) (two's complement
#   nibble; -8 unused);
# * FP4 E2M1: s = a / 6, y = clamp(x / s, -6, 6), code = e2m1(y) rounded to
#   nearest, ties to even.  E2M1 (OCP microscaling formats): 1 sign bit, 2
#   exponent bits with bias 1, 1 mantissa bit; exponent field 0 is
#   subnormal (0 or 0.5); magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
# * a = 0 gives s = 0 and zero codes; arithmetic in IEEE fp32.
# * Two codes per byte along head_dim: element 2k in the low nibble of byte
#   k, element 2k + 1 in the high nibble.
# --------------------------------------------------------------------------

INT4_QMAX = 7
FP4_E2M1_MAX = 6.0


def e2m1_decode(codes):
    """4-bit E2M1 codes (0..15) -> fp64 values."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e.astype(np.float64) - 1))
    return sign * mag


def e2m1_encode(y):
    """Values with |y| <= 6 -> 4-bit E2M1 codes, round to nearest, ties to
    even (the code with mantissa bit 0).  The sign of zero is kept."""
    y = np.asarray(y, np.float64)
    if np.any(np.abs(y) > FP4_E2M1_MAX) or np.any(np.isnan(y)):
        raise ValueError("e2m1_encode expects finite |y| <= 6")
    a = np.abs(y)
    _, ex = np.frexp(a)                       # a in [2^(ex-1), 2^ex)
    E = np.maximum(ex - 1, 0)                 # binade; below 1 the spacing is 0.5
    quantum = np.ldexp(0.5, E)                # 1 mantissa bit
    v = np.rint(a / quantum) * quantum        # exact scaling, half-to-even on the quantum grid
    # encode v: 0 -> 0, 0.5 -> 1, 1 -> 2, 1.5 -> 3, 2 -> 4, 3 -> 5, 4 -> 6, 6 -> 7
    lut = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    mag = np.vectorize(lambda t: lut[float(t)], otypes=[np.int64])(v) if v.size else v.astype(np.int64)
    code = np.where(np.signbit(y), mag | 0x8, mag)
    return code.astype(np.uint8)


def pack_nibbles(codes):
    """[..., D] codes (0..15) -> [..., D / 2] uint8, element 2k in the low nibble."""
    c = np.asarray(codes).astype(np.uint8) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    """[..., D / 2] uint8 -> [..., D] codes 0..15."""
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def quantize_int4(x):
    """x [..., D] -> (packed codes uint8 [..., D / 2], scales fp32 [...])."""
    x = np.asarray(x, np.float32)
    a = absmax_rows(x)
    s = (a / np.float32(INT4_QMAX)).astype(np.float32)
    q = np.zeros(x.shape, np.int64)
    nz = a > 0
    y = (x[nz] / s[nz][..., None]).astype(np.float32)
    q[nz] = np.clip(np.rint(y), -INT4_QMAX, INT4_QMAX).astype(np.int64)
    return pack_nibbles(q & 0xF), s


def quantize_fp4_e2m1(x):
    """x [..., D] -> (packed codes uint8 [..., D / 2], scales fp32 [...])."""
    x = np.asarray(x, np.float32)
    a = absmax_rows(x)
    s = (a / np.float32(FP4_E2M1_MAX)).astype(np.float32)
    codes = np.zeros(x.shape, np.uint8)
    nz = a > 0
    y = (x[nz] / s[nz][..., None]).astype(np.float32)
    y = np.clip(y, np.float32(-FP4_E2M1_MAX), np.float32(FP4_E2M1_MAX))
    codes[nz] = e2m1_encode(y)
    return pack_nibbles(codes), s


def int4_values(packed):
    """Packed INT4 codes -> fp64 code values (-7..7) [..., D]."""
    c = unpack_nibbles(packed).astype(np.int64)
    return np.where(c >= 8, c - 16, c).astype(np.float64)


def fp4_values(packed):
    """Packed E2M1 codes -> fp64 values [..., D]."""
    return e2m1_decode(unpack_nibbles(packed))
