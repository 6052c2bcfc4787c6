"""Pins of the oracle's codecs and storage rules against library casts,
published value tables and brute force (CPU only)."""
import os

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import storage as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _finite_e4m3_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = F.e4m3_decode(codes)
    ok = ~np.isnan(vals)
    return codes[ok], vals[ok]


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_decode(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(ours))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], ours[ok])
    assert np.nanmax(ours) == 448.0 and np.isnan(ours).sum() == 2


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200_000) * 50,
        rng.standard_normal(50_000) * 1e-2,       # subnormal range
        rng.uniform(-463.9, 463.9, 50_000),
    ]).astype(np.float32)
    # exact midpoints between neighbouring finite values: RNE ties
    _, vals = _finite_e4m3_values()
    pos = np.unique(vals[vals >= 0])
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(x), ref)


def test_e4m3_saturates():
    x = np.array([448.0, 460.0, 464.0, 1000.0, 1e30, -500.0, -1e30], dtype=np.float32)
    assert list(F.e4m3_encode(x)) == [0x7E] * 5 + [0xFE] * 2


def _brute_nearest(x, values, codes):
    """Nearest finite value; ties to the even code (even mantissa)."""
    d = np.abs(x[:, None].astype(np.float64) - values[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates prefer the even code
    even = (codes[None, :] & 1) == 0
    pick = np.where((cand & even).any(axis=1, keepdims=True), cand & even, cand)
    return values[np.argmax(pick, axis=1)]


def test_e4m3_encode_is_nearest_value_brute_force():
    codes, vals = _finite_e4m3_values()
    keep = codes < 0x80  # magnitudes
    rng = np.random.default_rng(2)
    x = np.abs(np.concatenate([rng.standard_normal(20_000) * 30, rng.standard_normal(5_000) * 1e-2,
                               (vals[keep][1:] + vals[keep][:-1]) / 2])).astype(np.float32)
    x = x[x <= 448]
    want = _brute_nearest(x, vals[keep], codes[keep])
    got = F.e4m3_decode(F.e4m3_encode(x))
    assert np.array_equal(got, want)


def test_e2m1_table_matches_ocp_spec():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "ocp_e2m1_values.txt"))
            if ln.strip() and not ln.startswith("#")]
    codes = np.array([int(r[0]) for r in rows], dtype=np.uint8)
    want = np.array([float(r[1]) for r in rows])
    got = F.e2m1_decode(codes)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_e2m1_encode_is_nearest_value_brute_force_and_saturates():
    codes = np.arange(8, dtype=np.uint8)
    vals = F.e2m1_decode(codes)
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(0, 6, 20_000), (vals[1:] + vals[:-1]) / 2, vals]).astype(np.float32)
    want = _brute_nearest(x, vals, codes)
    assert np.array_equal(F.e2m1_decode(F.e2m1_encode(x)), want)
    assert np.array_equal(F.e2m1_decode(F.e2m1_encode(-x)), -want)
    assert list(F.e2m1_encode(np.array([6.5, 100.0, -7.0], np.float32))) == [7, 7, 15]


def test_e2m1_values_are_e4m3_values():
    vals = F.e2m1_decode(np.arange(16, dtype=np.uint8))
    assert np.array_equal(F.e4m3_decode(F.e4m3_encode(vals.astype(np.float32))), vals)


def test_bf16_matches_torch_cast():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(300_000) * np.exp(rng.uniform(-30, 30, 300_000))).astype(np.float32)
    # exact ties: low 16 bits == 0x8000
    u = rng.integers(0, 2 ** 31, 10_000, dtype=np.uint64).astype(np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    ties = ties[np.isfinite(ties)]
    x = np.concatenate([x, ties]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(F.bf16_encode(x), ref)
    assert np.array_equal(F.bf16_decode(ref), torch.from_numpy(x).to(torch.bfloat16).double().numpy())


# ---------------------------------------------------------------- storage rules

def test_kv_row_scale_and_bounds():
    rng = np.random.default_rng(5)
    c = (rng.standard_normal((300, 512)) / np.sqrt(512)).astype(np.float32)
    st = S.encode("kv", c, rope_dim=64)
    assert st.payload.shape == (300, 448 + 128) and st.scale.dtype == np.float32
    amax = np.abs(c[:, :448]).max(axis=1)
    assert np.array_equal(st.scale, (amax / np.float32(448)).astype(np.float32))
    codes = st.payload[:, :448]
    # the largest magnitude lands on +-448 (code 0x7E / 0xFE)
    arg = np.abs(c[:, :448]).argmax(axis=1)
    assert np.all((codes[np.arange(300), arg] & 0x7F) == 0x7E)
    back = S.decode(st)
    # rope dims: bf16 RNE of the float32 value, checked with torch's cast
    rope_ref = torch.from_numpy(np.ascontiguousarray(c[:, 448:])).to(torch.bfloat16).double().numpy()
    assert np.array_equal(back[:, 448:], rope_ref)
    # fp8 dims: error at most half a quantum of the value's E4M3 binade (relative 2^-4),
    # or half the subnormal quantum 2^-10 * s
    err = np.abs(back[:, :448] - c[:, :448])
    bound = np.maximum(np.abs(c[:, :448]) * 2.0 ** -4, st.scale[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_fp8_key_rows_match_torch_cast_of_scaled_values():
    rng = np.random.default_rng(6)
    c = (rng.standard_normal((200, 128)) / np.sqrt(128)).astype(np.float32)
    st = S.encode("fp8", c)
    y = (c / st.scale[:, None]).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(st.payload, ref)


def test_zero_rows():
    st = S.encode("kv", np.zeros((2, 512), np.float32), rope_dim=64)
    assert np.all(st.scale == 1.0) and np.all(st.payload == 0)
    st4 = S.encode("fp4", np.zeros((2, 128), np.float32))
    assert np.all(st4.scale == 0) and np.all(st4.payload == 0)
    assert np.all(S.decode(st4) == 0)


def test_fp4_block_scale_rule_and_nibble_order():
    rng = np.random.default_rng(7)
    c = (rng.standard_normal((100, 128)) / np.sqrt(128)).astype(np.float32)
    st = S.encode("fp4", c)
    assert st.payload.shape == (100, 64) and st.scale.shape == (100, 8)
    amax = np.abs(c.reshape(100, 8, 16)).max(axis=2)
    ref_sc = torch.from_numpy((amax / np.float32(6)).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(st.scale, ref_sc)
    # element 0 in the low nibble: a row whose first two values are 0.5*s and 6*s
    s = np.float32(0.25)  # exact E4M3 value; amax/6 = s
    row = np.zeros((1, 16), np.float32)
    row[0, 0], row[0, 1] = 0.5 * s, 6 * s
    st1 = S.encode("fp4", row)
    assert st1.payload[0, 0] == 0x71 and F.e4m3_decode(st1.scale)[0, 0] == 0.25


def test_fp4_exact_values_round_trip():
    rng = np.random.default_rng(8)
    vals = F.e2m1_decode(np.arange(16, dtype=np.uint8))
    codes = rng.integers(0, 16, (50, 128))
    codes[:, ::16] = 7  # each block holds a 6 so that amax / 6 is the block scale
    scale_codes = rng.integers(0x20, 0x50, (50, 8)).astype(np.uint8)
    sc = F.e4m3_decode(scale_codes)
    c = (vals[codes].reshape(50, 8, 16) * sc[..., None]).reshape(50, 128).astype(np.float32)
    st = S.encode("fp4", c)
    assert np.array_equal(S.decode(st), c.astype(np.float64))


@pytest.mark.parametrize("fmt,dim", [("kv", 512), ("fp8", 128), ("fp4", 128), ("f32", 32)])
def test_chunked_encode_equals_rowwise(fmt, dim):
    rng = np.random.default_rng(9)
    c = (rng.standard_normal((1000, dim)) / np.sqrt(dim)).astype(np.float32)
    st = S.encode(fmt, c, rope_dim=64 if fmt == "kv" else 0)
    for i in (0, 511, 999):
        one = S.encode(fmt, c[i:i + 1], rope_dim=64 if fmt == "kv" else 0)
        assert np.array_equal(one.payload[0], st.payload[i])
        if st.scale is not None:
            assert np.array_equal(one.scale[0], st.scale[i])
