"""Cache row formats and their quantisation rules (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: "DeepSeek V4 Architecture Explained", Key numbers table, row "KV
storage precision" (FP8 for the non-RoPE dims, BF16 for the RoPE dims);
"Inside DeepSeek-V4", section 1 ("FP4 Lightning Indexer").  The pages give
no scale rule; the reading used here (one per-row float32 scale for FP8,
one E4M3 scale per 16-element block for FP4) is:

* KV row (``kv``): s = amax(|c[:D-R]|) / 448 in float32 (s = 1 when the
  amax is 0); the first D-R values are stored as E4M3(c / s); the last R
  ("RoPE") values as BF16(c).  Payload = (D-R) + 2R bytes, scale apart.
* FP8 indexer key (``fp8``): the same rule over all d values (R = 0).
* FP4 indexer key (``fp4``): per block of 16, b = amax / 6 in float32; the
  scale byte is E4M3(b); if it decodes to 0 the block is all-zero codes,
  else each value is E2M1(c / decode(scale byte)).  Payload = d/2 bytes,
  element 2i in the low nibble of byte i; scales = d/16 bytes apart.
* ``f32``: the float32 values themselves.

Every rule takes its decisions in float32: the pooled / raw value is first
rounded to float32, and the scale and the divisions are float32 operations
(numpy float32 arithmetic is IEEE round-to-nearest).
"""
import numpy as np

from .formats import (E2M1_MAX, E4M3_MAX, bf16_decode, bf16_encode, e2m1_decode,
                      e2m1_encode, e4m3_decode, e4m3_encode)

FP4_BLOCK = 16


def row_scale_fp8(c32):
    """Per-row float32 scale amax/448 over the last axis (1 where amax is 0)."""
    amax = np.max(np.abs(c32), axis=-1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def encode_fp8_rows(c):
    """Rows [..., d] -> (E4M3 codes uint8 [..., d], scale float32 [...])."""
    c32 = np.asarray(c, dtype=np.float32)
    s = row_scale_fp8(c32)
    y = (c32 / s[..., None]).astype(np.float32)
    return e4m3_encode(y), s


def decode_fp8_rows(codes, scale):
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]


def encode_kv_rows(c, rope_dim):
    """Rows [..., D] -> (payload uint8 [..., (D-R) + 2R], scale float32 [...])."""
    c32 = np.asarray(c, dtype=np.float32)
    d_nope = c32.shape[-1] - rope_dim
    codes, s = encode_fp8_rows(c32[..., :d_nope])
    rope = bf16_encode(c32[..., d_nope:])  # little-endian bf16 bytes follow the codes
    payload = np.concatenate([codes, rope.view(np.uint8).reshape(*rope.shape[:-1], 2 * rope_dim)],
                             axis=-1)
    return payload, s


def decode_kv_rows(payload, scale, rope_dim):
    payload = np.ascontiguousarray(np.asarray(payload, dtype=np.uint8))
    d_nope = payload.shape[-1] - 2 * rope_dim
    nope = decode_fp8_rows(payload[..., :d_nope], scale)
    rope_bits = np.ascontiguousarray(payload[..., d_nope:]).view(np.uint16)
    return np.concatenate([nope, bf16_decode(rope_bits)], axis=-1)


def encode_fp4_rows(c):
    """Rows [..., d] -> (packed E2M1 uint8 [..., d/2], E4M3 block scales uint8 [..., d/16])."""
    c32 = np.asarray(c, dtype=np.float32)
    d = c32.shape[-1]
    blocks = c32.reshape(*c32.shape[:-1], d // FP4_BLOCK, FP4_BLOCK)
    amax = np.max(np.abs(blocks), axis=-1)
    b = (amax / np.float32(E2M1_MAX)).astype(np.float32)
    sc = e4m3_encode(b)
    dsc = e4m3_decode(sc).astype(np.float32)
    safe = np.where(dsc > 0, dsc, np.float32(1.0)).astype(np.float32)
    y = (blocks / safe[..., None]).astype(np.float32)
    codes = np.where(dsc[..., None] > 0, e2m1_encode(y), np.uint8(0)).astype(np.uint8)
    codes = codes.reshape(*c32.shape[:-1], d)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, sc


def decode_fp4_rows(packed, scales):
    packed = np.asarray(packed, dtype=np.uint8)
    lo = e2m1_decode(packed & 0xF)
    hi = e2m1_decode(packed >> 4)
    vals = np.stack([lo, hi], axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    blocks = vals.reshape(*vals.shape[:-1], vals.shape[-1] // FP4_BLOCK, FP4_BLOCK)
    dsc = e4m3_decode(scales)
    return (blocks * dsc[..., None]).reshape(vals.shape)


# ---------------------------------------------------------------------------
# One interface over the four formats: encode(rows) -> Stored, decode(Stored).
# ---------------------------------------------------------------------------

class Stored:
    """Stored rows: ``payload`` (float32 rows or uint8 bytes) and ``scale``
    (float32 per row, uint8 per FP4 block, or None for f32)."""

    def __init__(self, fmt, payload, scale, dim, rope_dim=0):
        self.fmt, self.payload, self.scale = fmt, payload, scale
        self.dim, self.rope_dim = dim, rope_dim

    def rows(self, index):
        sc = None if self.scale is None else self.scale[index]
        return Stored(self.fmt, self.payload[index], sc, self.dim, self.rope_dim)


_ENCODERS = {
    "kv": lambda c, r: encode_kv_rows(c, r),
    "fp8": lambda c, r: encode_fp8_rows(c),
    "fp4": lambda c, r: encode_fp4_rows(c),
}


def encode(fmt, c, rope_dim=0):
    """Stored rows of ``c`` [..., dim].  Large inputs are encoded a few
    thousand rows at a time (same result; only the memory footprint of the
    temporaries changes)."""
    c = np.asarray(c)
    dim = c.shape[-1]
    if fmt == "f32":
        return Stored(fmt, np.asarray(c, dtype=np.float32), None, dim)
    if fmt not in _ENCODERS:
        raise ValueError(fmt)
    enc = _ENCODERS[fmt]
    flat = c.reshape(-1, dim)
    step = max(1, (1 << 16) // dim)
    parts = [enc(flat[i:i + step], rope_dim) for i in range(0, flat.shape[0], step)]
    if parts:
        p = np.concatenate([x[0] for x in parts])
        s = np.concatenate([x[1] for x in parts])
    else:
        p, s = enc(flat, rope_dim)
    lead = c.shape[:-1]
    return Stored(fmt, p.reshape(*lead, p.shape[-1]), s.reshape(*lead, *s.shape[1:]), dim,
                  rope_dim if fmt == "kv" else 0)


def decode(st):
    """float64 values of stored rows."""
    if st.fmt == "f32":
        return np.asarray(st.payload, dtype=np.float64)
    if st.fmt == "kv":
        return decode_kv_rows(st.payload, st.scale, st.rope_dim)
    if st.fmt == "fp8":
        return decode_fp8_rows(st.payload, st.scale)
    if st.fmt == "fp4":
        return decode_fp4_rows(st.payload, st.scale)
    raise ValueError(st.fmt)


def quantize(fmt, c, rope_dim=0):
    """Round trip: the float64 values a row takes once stored in ``fmt``."""
    return decode(encode(fmt, c, rope_dim))
