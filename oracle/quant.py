"""Per-token-per-head absmax KV quantisation (oracle; test infrastructure only).

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
