"""Bit-exact codecs for the three storage element types (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

The pages fix the types but not their encodings: "BF16 for RoPE dimensions,
FP8 for the rest" ("DeepSeek V4 Architecture Explained", Key numbers, row
"KV storage precision") and an "FP4 quantized indexer" ("Inside
DeepSeek-V4", section 1).  The encodings are the public definitions:

* FP8 E4M3 (OCP 8-bit floating point spec, "E4M3"): sign, 4 exponent bits
  with bias 7, 3 mantissa bits; exponent field 0 is subnormal (m * 2^-9);
  no infinities; S.1111.111 is NaN, so the largest finite value is 448.
* FP4 E2M1 (OCP Microscaling spec, "FP4 E2M1"): sign, 2 exponent bits with
  bias 1, 1 mantissa bit; finite values 0, 0.5, 1, 1.5, 2, 3, 4, 6.
* bfloat16: the upper 16 bits of an IEEE binary32.

Every encoder rounds to nearest, ties to even, and saturates to the largest
finite magnitude ("satfinite").  Inputs must be finite.  Encoders take the
value as float32 (the precision in which the stored code is decided) and do
all further work exactly in float64.
"""
import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def e4m3_decode(codes):
    """Value of each E4M3 byte, as float64 (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    mant = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, mant * 2.0 ** -9, (1.0 + mant / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def e2m1_decode(nibbles):
    """Value of each E2M1 code (low 4 bits of each byte), as float64."""
    c = np.asarray(nibbles, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    mant = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, mant * 0.5, (1.0 + mant / 2.0) * np.exp2(e - 1.0))
    return sign * mag


def _round_magnitude(a, mant_bits, min_normal_exp, max_finite):
    """Round float32 magnitudes ``a`` to the grid of a binary format with
    ``mant_bits`` stored mantissa bits whose smallest normal exponent is
    ``min_normal_exp``; ties to even; clamp to ``max_finite``.

    Every operation below is exact in float32 for the formats used here:
    the quantum is a power of two, so a / quantum only shifts the exponent.
    """
    _, e = np.frexp(a)  # a = f * 2^e with f in [0.5, 1), so floor(log2 a) = e - 1
    binade = np.maximum(e - 1, min_normal_exp)
    quantum = np.ldexp(np.float32(1.0), binade - mant_bits).astype(np.float32)
    # np.rint is round-half-even, and an even multiple of the quantum is an
    # even mantissa (the leading 1 of a normal value is 2^mant_bits quanta).
    r = (np.rint(a / quantum) * quantum).astype(np.float32)
    return np.minimum(r, np.float32(max_finite))


def _code_of_magnitude(r, mant_bits, min_normal_exp, exp_bias):
    """Unsigned code of representable magnitudes r: subnormals are r / 2^(emin
    - mant_bits); normals are (biased exponent << mant_bits) | mantissa."""
    sub_quantum = np.float32(2.0 ** (min_normal_exp - mant_bits))
    f, e = np.frexp(r)
    exp_field = (e - 1) + exp_bias
    mant = (f * np.float32(2 ** (mant_bits + 1))).astype(np.int64) - (1 << mant_bits)
    normal = (exp_field.astype(np.int64) << mant_bits) | mant
    sub = (r / sub_quantum).astype(np.int64)
    return np.where(r < np.float32(2.0 ** min_normal_exp), sub, normal).astype(np.uint8)


def e4m3_encode(x):
    """E4M3 code of each float32 value: RNE, satfinite, sign kept (-0 -> 0x80)."""
    x32 = np.asarray(x, dtype=np.float32)
    r = _round_magnitude(np.abs(x32), 3, -6, E4M3_MAX)
    code = _code_of_magnitude(r, 3, -6, 7)
    return np.where(np.signbit(x32), code | np.uint8(0x80), code).astype(np.uint8)


def e2m1_encode(x):
    """E2M1 code (0..15) of each float32 value: RNE, satfinite, sign kept."""
    x32 = np.asarray(x, dtype=np.float32)
    r = _round_magnitude(np.abs(x32), 1, 0, E2M1_MAX)
    code = _code_of_magnitude(r, 1, 0, 1)
    return np.where(np.signbit(x32), code | np.uint8(0x8), code).astype(np.uint8)


def bf16_encode(x):
    """bfloat16 bit pattern (uint16) of each float32 value, RNE."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    hi = u >> np.uint64(16)
    lo = u & np.uint64(0xFFFF)
    round_up = (lo > 0x8000) | ((lo == 0x8000) & ((hi & np.uint64(1)) == 1))
    return (hi + round_up.astype(np.uint64)).astype(np.uint16)


def bf16_decode(bits):
    """float64 value of each bfloat16 bit pattern."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def to_bf16(x):
    """Round float values (via float32) to bfloat16 and return them as float64."""
    return bf16_decode(bf16_encode(np.asarray(x, dtype=np.float32)))
