"""Bit-level codecs for the KV-cache element formats (oracle; test infrastructure only).

The pages name fp16 model weights and an FP8 KV cache (page 2, section
"4.2 混合精度策略", table row "KV缓存 FP8"; section "5.1 长文本处理基准", row
"vLLM FP8"). They do not fix the FP8 variant; this oracle reads it as OCP E4M3
("e4m3fn": 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities, S.1111.111 is NaN, largest finite value 448) with one scale per
tensor.

Every decoder below is written from the format's own definition -- sign,
biased exponent, fraction, subnormals -- and returns exact float64 values (all
three formats embed exactly in binary64). None of them reinterprets memory as a
library float type; the tests pin them against numpy / torch on every code.
"""

from __future__ import annotations

import numpy as np


def _decode_binary(codes: np.ndarray, exp_bits: int, man_bits: int, bias: int,
                   ieee_specials: bool, nan_all_ones_only: bool = False) -> np.ndarray:
    """Decode unsigned integer codes of a sign/exponent/fraction format to float64.

    value = (-1)^s * 2^(e - bias) * (1 + f / 2^man_bits)   for 0 < e < e_max (normal)
          = (-1)^s * 2^(1 - bias) * (f / 2^man_bits)       for e == 0 (subnormal)
    With ``ieee_specials`` the all-ones exponent holds inf (f == 0) and NaN.
    With ``nan_all_ones_only`` (E4M3) only exponent and fraction all ones is NaN;
    every other all-ones-exponent code is an ordinary normal number.
    """
    c = np.asarray(codes).astype(np.int64)
    sign = (c >> (exp_bits + man_bits)) & 1
    e = (c >> man_bits) & ((1 << exp_bits) - 1)
    f = c & ((1 << man_bits) - 1)
    e_max = (1 << exp_bits) - 1
    frac = f.astype(np.float64) / float(1 << man_bits)
    mag = np.where(e == 0,
                   np.ldexp(frac, 1 - bias),
                   np.ldexp(1.0 + frac, (e - bias).astype(np.int64)))
    if ieee_specials:
        mag = np.where(e == e_max, np.where(f == 0, np.inf, np.nan), mag)
    if nan_all_ones_only:
        mag = np.where((e == e_max) & (f == (1 << man_bits) - 1), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


def decode_f16(codes: np.ndarray) -> np.ndarray:
    """IEEE 754 binary16: 5 exponent bits (bias 15), 10 fraction bits."""
    return _decode_binary(codes, 5, 10, 15, ieee_specials=True)


def decode_bf16(codes: np.ndarray) -> np.ndarray:
    """bfloat16: 8 exponent bits (bias 127), 7 fraction bits, IEEE specials."""
    return _decode_binary(codes, 8, 7, 127, ieee_specials=True)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """OCP E4M3: 4 exponent bits (bias 7), 3 fraction bits, NaN = S.1111.111, no inf."""
    return _decode_binary(codes, 4, 3, 7, ieee_specials=False, nan_all_ones_only=True)


E4M3_MAX = 448.0   # 2^(15-7) * (1 + 6/8): exponent 15 with fraction 111 is NaN
E4M3_NAN = 0x7F


def encode_e4m3(x) -> np.ndarray:
    """Round float values to OCP E4M3 codes: round-to-nearest-even, saturating.

    Reading of the pages (which only say "FP8 KV cache"): finite values whose
    rounded magnitude would exceed 448 -- and infinities -- saturate to +-448;
    NaN maps to the code 0x7F. The sign of zero is kept (-0.0 -> 0x80).

    Each E4M3 binade [2^E, 2^(E+1)) holds 8 values spaced 2^(E-3); below 2^-6
    the subnormals are spaced 2^-9. Because codes grow linearly with the value
    inside a binade and carry over into the next exponent, the code of a
    rounded magnitude q * step is ((E + 7) << 3) + (q - 8) for normals and q for
    subnormals. The division by ``step`` is a power-of-two scaling, so it is
    exact in float64 and ``np.rint`` (ties to even) performs the rounding.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    finite = np.isfinite(a)
    a_f = np.where(finite, a, 0.0)
    # binade exponent E with 2^E <= a < 2^(E+1); frexp gives a = m * 2^k, m in [0.5, 1)
    _, k = np.frexp(a_f)
    E = k.astype(np.int64) - 1
    is_sub = a_f < 2.0 ** -6
    step_exp = np.where(is_sub, -9, E - 3)
    q = np.rint(np.ldexp(a_f, (-step_exp).astype(np.int64)))
    code = np.where(is_sub, q, ((E + 7) << 3) + (q.astype(np.int64) - 8)).astype(np.int64)
    # saturation: anything that rounded past 448 (code 0x7E), or was infinite
    code = np.where(code > 0x7E, 0x7E, code)
    code = np.where(np.isinf(a), 0x7E, code)
    code = np.where(np.signbit(x), code | 0x80, code)
    code = np.where(np.isnan(x), E4M3_NAN, code)
    return code.astype(np.uint8)


def f32_div(x_f32: np.ndarray, s_f32: float) -> np.ndarray:
    """IEEE binary32 quotient x / s, rounded to nearest even (numpy float32 division)."""
    return (np.asarray(x_f32, dtype=np.float32) / np.float32(s_f32)).astype(np.float32)


DECODERS = {"f16": decode_f16, "bf16": decode_bf16, "e4m3": decode_e4m3}
BYTES = {"f16": 2, "bf16": 2, "e4m3": 1}
CODE_DTYPE = {"f16": np.uint16, "bf16": np.uint16, "e4m3": np.uint8}


def decode(codes: np.ndarray, dtype: str) -> np.ndarray:
    """Decode an array of raw codes of the named element format to float64."""
    return DECODERS[dtype](codes)
