"""The C-ABI library loads, exports every function include/lcsc.h declares,
and rejects bad arguments on the host before any launch (CPU only: no
call below reaches the GPU)."""
import ctypes
import os
import re

import pytest

from long_context_sparse_compress_b200 import lib as L
from long_context_sparse_compress_b200 import workloads as W

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lcsc.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lcsc_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_compress_b200 import build
    if not os.path.exists(L.LIB_PATH):
        build.build()
    return L.load()


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(L.EXPORTS) == set(names)


def test_abi_version_and_strings(lib):
    assert lib.lcsc_abi_version() == L.ABI_VERSION
    for code in range(5):
        assert lib.lcsc_status_string(code)
    assert L.Params.sink_mode.offset == 68 and L.Params.gate_src.offset == 72
    assert lib.lcsc_row_bytes(L.FMT["kv"], 512, 64) == 576
    assert lib.lcsc_row_bytes(L.FMT["fp8"], 128, 0) == 128
    assert lib.lcsc_row_bytes(L.FMT["fp4"], 128, 0) == 64
    assert lib.lcsc_row_bytes(L.FMT["f32"], 128, 0) == 512


def test_wait_test_switch_is_host_only(lib):
    assert lib.lcsc_set_wait_test(-1, 0) == 1  # LCSC_ERR_INVALID_ARG
    assert lib.lcsc_set_wait_test(5_000_000, 1) == 0
    assert lib.lcsc_set_wait_test(0, 0) == 0


def test_workspace_sizes_are_host_only(lib):
    p = L.params(W.PAIR_DECODE_1M_B16.layer("csa"))
    out = ctypes.c_size_t(0)
    assert lib.lcsc_index_topk_workspace_size(ctypes.byref(p), 16, 1, 262144, ctypes.byref(out)) == 0
    # scores (4 B per entry) and the capped candidate (index, key) lists
    assert out.value >= 16 * 262144 * 4 + 16 * 65536 * 8
    assert lib.lcsc_step_workspace_size(ctypes.byref(p), 1, 16, 1, 262144, ctypes.byref(out)) == 0
    assert lib.lcsc_attn_workspace_size(ctypes.byref(p), 16, 1, 8192, 1, ctypes.byref(out)) == 0


def test_bad_arguments_are_rejected_before_launch(lib):
    p = L.params(W.CSA_DECODE_128K)
    null = None
    # null params
    assert lib.lcsc_csa_decode(null, null, null, 0, null, null) == 1
    # null step
    assert lib.lcsc_csa_decode(ctypes.byref(p), null, null, 0, null, null) == 1
    # k beyond 2048
    bad = L.params(W.CSA_DECODE_128K.with_(k=4096))
    out = ctypes.c_size_t(0)
    assert lib.lcsc_index_topk_workspace_size(ctypes.byref(bad), 1, 1, 10, ctypes.byref(out)) == 1
    # group length beyond 2m
    bad = L.params(W.CSA_DECODE_128K.with_(G=12))
    assert lib.lcsc_index_topk_workspace_size(ctypes.byref(bad), 1, 1, 10, ctypes.byref(out)) == 1
    # the output's inverse RoPE: a base that is negative, not a number or
    # infinite, and rotated dims that are not a multiple of 4 or exceed Dv
    rope_on = L.params(W.CSA_DECODE_128K.with_(out_rope_base=10000.0))
    assert lib.lcsc_attn_workspace_size(ctypes.byref(rope_on), 1, 1, 10, 0, ctypes.byref(out)) == 0
    for field, value in (("out_rope_base", -1.0), ("out_rope_base", float("nan")),
                         ("out_rope_base", float("inf")), ("out_rope_dim", 6), ("out_rope_dim", 0),
                         ("out_rope_dim", 516)):
        bad = L.params(W.CSA_DECODE_128K.with_(out_rope_base=10000.0))
        setattr(bad, field, value)
        assert lib.lcsc_attn_workspace_size(ctypes.byref(bad), 1, 1, 10, 0, ctypes.byref(out)) == 1, field
    # the sink and gate readings take only their two values; the softmax
    # scale must be a positive number
    for field, value in (("sink_mode", 2), ("sink_mode", -1), ("gate_src", 2), ("sm_scale", 0.0),
                         ("sm_scale", -0.1), ("sm_scale", float("nan")), ("sm_scale", float("inf"))):
        bad = L.params(W.CSA_DECODE_128K)
        setattr(bad, field, value)
        assert lib.lcsc_attn_workspace_size(ctypes.byref(bad), 1, 1, 10, 0, ctypes.byref(out)) == 1, field
    # with a sink token the sink logit pointer must be NULL and the position-0
    # rows given (checked before any pointer is dereferenced on the device)
    tok = L.params(W.HCA_DECODE_64K.with_(sink_mode="token"))
    c = L.Cache(data=16, scale=16, capacity=1000)  # room for the window: only the sink arguments are wrong
    q_ptr = ctypes.c_void_p(16)
    assert lib.lcsc_hca_dense_attn(ctypes.byref(tok), q_ptr, ctypes.byref(c), null, ctypes.byref(c), null,
                                   ctypes.c_void_p(16), ctypes.byref(c), null, ctypes.c_void_p(16), 1, 1, 4,
                                   q_ptr, null, ctypes.c_void_p(256), 1 << 20, null, null) == 1
    assert lib.lcsc_hca_dense_attn(ctypes.byref(tok), q_ptr, ctypes.byref(c), null, ctypes.byref(c), null,
                                   null, null, null, ctypes.c_void_p(16), 1, 1, 4, q_ptr, null,
                                   ctypes.c_void_p(256), 1 << 20, null, null) == 1
    # a dimension the kernels are not built for
    odd = L.params(W.CSA_DECODE_128K.with_(d_I=96))
    s = L.Step(B=1, T=1, n_max=10, ctx_len=16)
    ws = ctypes.create_string_buffer(64)
    assert lib.lcsc_csa_decode(ctypes.byref(odd), ctypes.byref(s), ws, 64, null, null) == 2
    # misaligned pointer in encode_rows
    assert lib.lcsc_encode_rows(ctypes.byref(p), 0, 3, 1, 1, 0, null, null) == 1


def _attn_splits(lib, wl, B, T, n_max, dense):
    """The attention's split count, read back from its workspace size: one
    [B*T][splits][H][Dv] fp32 partial O, one [B*T][splits][H][2] fp32
    (max, sum) array and the tensor-core path's [B*T] query images of
    64 KB + 256 B, each rounded up to 256 bytes."""
    p = L.params(wl)
    out = ctypes.c_size_t(0)
    assert lib.lcsc_attn_workspace_size(ctypes.byref(p), B, T, n_max, int(dense), ctypes.byref(out)) == 0
    up = lambda x: (x + 255) // 256 * 256
    img = up(B * T * (65536 + 256))
    for s in range(1, 4096):
        if up(B * T * s * wl.H * wl.Dv * 4) + up(B * T * s * wl.H * 2 * 4) + img == out.value:
            return s
    raise AssertionError(f"no split count gives {out.value} bytes")


def test_attention_split_counts(lib):
    """The split cost model on this host (no GPU: 148 SMs assumed): one wave
    of several splits for the decode pair, fewer for five queries per
    sequence, one for chunked prefill (the kernel then writes the output
    itself)."""
    pair = W.PAIR_DECODE_1M_B16
    csa, hca = pair.layer("csa"), pair.layer("hca")
    assert _attn_splits(lib, hca, 16, 1, 8192, True) == 9       # 8,320 rows: 144 CTAs
    assert _attn_splits(lib, csa, 16, 1, 262144, False) == 9    # 1,152 rows: 144 CTAs
    assert _attn_splits(lib, hca, 16, 5, 8192, True) == 5       # 80 queries: 400 CTAs
    assert _attn_splits(lib, csa, 16, 5, 262144, False) == 1    # 80 queries, 18 tiles each
    assert _attn_splits(lib, W.CSA_PREFILL_256K, 1, 4096, 66560, False) == 1
    assert _attn_splits(lib, W.CSA_DECODE_128K, 8, 1, 32768, False) == 18  # a 64-row tile per split
