"""Per-stage parity of the CUDA library against the oracle (small shapes that
still span several tiles and ragged tails).  Every input is seeded; every
expected value comes from ``oracle/``."""
import zlib

import numpy as np
import pytest
import torch

from long_context_sparse_compress_b200 import lib as L
from long_context_sparse_compress_b200 import workloads as W
from oracle import storage
from oracle.compress import compress_entries
from oracle.indexer import quantize_query, scores as oracle_scores, topk as oracle_topk
from oracle.attention import joint_attention, window_positions
from tests.gpu_harness import TORCH_DT, dev, download, upload
from tests.harness import max_abs, rel_l2, topk_set_ok

pytestmark = pytest.mark.gpu

ATTN_RTOL, ATTN_ATOL = 1e-2, 2e-2
FP32_RTOL, Q_RTOL = 1e-5, 1e-2


def _rows(rng, n, d, scale=None):
    scale = d ** -0.5 if scale is None else scale
    return (rng.standard_normal((n, d)) * scale).astype(np.float32)


def _wl_for(fmt_kv="kv", fmt_idx="fp8"):
    if fmt_kv == "f32":
        return W.CSA_DECODE_4K_F32
    return W.CSA_DECODE_128K.with_(idx_fmt=fmt_idx)


# ------------------------------------------------------------------ encode

@pytest.mark.parametrize("fmt,dim,rope", [("kv", 512, 64), ("fp8", 128, 0), ("fp4", 128, 0),
                                          ("f32", 128, 0), ("f32", 32, 0)])
def test_encode_rows_bit_exact(cuda_lib, fmt, dim, rope):
    rng = np.random.default_rng(11)
    B, n = 2, 300
    rows = _rows(rng, B * n, dim).reshape(B, n, dim)
    rows[0, 0] = 0.0                                  # zero row
    rows[0, 1] *= 1e4                                 # large values
    rows[0, 2] *= 1e-6                                # tiny values (subnormal codes)
    rows[1, 3, ::3] = 0.0
    if fmt == "f32":
        wl = W.CSA_DECODE_4K_F32.with_(d_I=dim) if dim == 32 else W.CSA_DECODE_4K_F32
        tensor = "idx" if dim == 32 else "kv"
    else:
        wl = W.CSA_DECODE_128K.with_(idx_fmt=fmt if fmt != "kv" else "fp8")
        tensor = "kv" if fmt == "kv" else "idx"
    p = L.params(wl)
    out = L.DeviceCache(B, n + 5, fmt, dim, rope)
    L.encode_rows(p, tensor, dev(rows), 5, out)
    torch.cuda.synchronize()
    for b in range(B):
        st = storage.encode(fmt, rows[b], rope)
        d, s = download(out, b)
        assert np.array_equal(d[5:], st.payload), f"payload mismatch b={b}"
        if s is not None:
            assert np.array_equal(s[5:], st.scale), f"scale mismatch b={b}"


# ---------------------------------------------------------------- compress

COMPRESS_CASES = {
    "f32_k_m4": ("f32", "kv", 4, 4, 128, "f32"),
    "f32_idx_m4": ("f32", "idx", 4, 4, 32, "f32"),
    "kv512_m4": ("kv", "kv", 4, 4, 512, "bf16"),
    "fp8idx_m4": ("fp8", "idx", 4, 4, 128, "bf16"),
    "fp4idx_m4": ("fp4", "idx", 4, 4, 128, "bf16"),
    "kv512_m128": ("kv", "kv", 128, 128, 512, "bf16"),
    "kv512_m4_overlap8": ("kv", "kv", 4, 8, 512, "bf16"),
    "f32_k_m4_overlap8": ("f32", "kv", 4, 8, 128, "f32"),
}


@pytest.mark.parametrize("case", sorted(COMPRESS_CASES))
@pytest.mark.parametrize("with_window", [False, True])
def test_compress_matches_oracle(cuda_lib, case, with_window):
    fmt, tensor, m, G, dim, xdt = COMPRESS_CASES[case]
    rng = np.random.default_rng(zlib.crc32(case.encode()))
    B = 3
    tok_begin = 0 if m == 128 else 8 * m
    n_entries = 5 if m == 128 else 70            # > 2 CTAs of 32 entries, ragged
    tok_end = tok_begin + n_entries * m + (m // 2)  # a trailing partial group (not pooled)
    n_x = tok_end - tok_begin + G - m
    x = _rows(rng, B * n_x, dim).reshape(B, n_x, dim)
    if xdt == "bf16":
        x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    Wg = (rng.standard_normal((dim, dim)) * 0.02).astype(np.float32)
    if xdt == "bf16":
        Wg = torch.from_numpy(Wg).to(torch.bfloat16).float().numpy()
    Bp = rng.standard_normal((G, dim)).astype(np.float32)
    if fmt == "f32":
        wl = W.CSA_DECODE_4K_F32.with_(m=m, G=G)
    else:
        wl = W.CSA_DECODE_128K.with_(m=m, G=G, idx_fmt=fmt if tensor == "idx" else "fp8")
    p = L.params(wl)
    rope = wl.rope_dim if fmt == "kv" else 0
    n_cap = tok_end // m + 3
    ent = L.DeviceCache(B, n_cap, fmt, dim, rope)
    win = L.DeviceCache(B, 64, fmt, dim, rope) if (with_window and tensor != "idx") else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.compress(p, tensor, dev(x, TORCH_DT[xdt]), B, tok_begin, tok_end, dev(Wg, TORCH_DT[xdt]), dev(Bp),
               ent, win, status, hca=(m == 128))
    torch.cuda.synchronize()
    assert status.item() == 0
    g_lo, g_hi = tok_begin // m, tok_end // m
    x_pos0 = tok_begin - (G - m)
    for b in range(B):
        want = compress_entries(x[b], x_pos0, Wg, Bp, m, G, range(g_lo, g_hi))
        d, s = download(ent, b)
        got = storage.Stored(fmt, d[g_lo:g_hi], None if s is None else s[g_lo:g_hi], dim, rope)
        got_v = storage.decode(got)
        if fmt == "f32":
            assert rel_l2(got_v, want) <= FP32_RTOL
        else:
            # stored values: the oracle stores its own pooled rows by the same rule
            st = storage.encode(fmt, want, rope)
            assert rel_l2(got_v, storage.decode(st)) <= Q_RTOL
            # codes are decided in float32 on both sides: nearly all agree (a
            # pooled value within a float32 rounding of a code boundary may flip)
            same = np.mean(st.payload == got.payload)
            assert same > 0.99, f"only {same:.4f} of stored bytes identical"
        # untouched rows stay zero
        assert not np.any(d[:g_lo]) and not np.any(d[g_hi:])
        if win is not None:
            wd, ws_ = download(win, b)
            lo = max(tok_begin, tok_end - 64)
            for pos in range(lo, tok_end):
                st = storage.encode(fmt, x[b][pos - x_pos0][None], rope)
                assert np.array_equal(wd[pos % 64], st.payload[0])


# ----------------------------------------------------------- index + top-k

@pytest.mark.parametrize("fmt", ["f32", "fp8", "fp4"])
def test_index_topk_matches_oracle(cuda_lib, fmt):
    # three lists per sequence (an odd query index among them); tensor-core
    # scoring runs several CTAs per list here
    lengths = [4 * 5000 + 3, 4 * 37, 4 * 2100 + 1]  # one list shorter than k
    check_index_topk(fmt, lengths, T=3, seed=21)


# 150 lists: one tensor-core scoring CTA per query, whose own histogram gives
# the threshold bins; 78 and 80 lists: two CTAs per query (some wait for an
# SM and join late).  T = 5: five draft-token queries per sequence.
@pytest.mark.parametrize("fmt,B,T", [("fp8", 50, 3), ("fp4", 30, 5), ("fp8", 26, 3), ("fp4", 16, 5)])
def test_index_topk_many_lists(cuda_lib, fmt, B, T):
    rng = np.random.default_rng(5)
    lengths = [int(v) for v in rng.integers(4 * 300, 4 * 2500, size=B)]
    check_index_topk(fmt, lengths, T=T, seed=22)


def test_index_topk_whole_lists(cuda_lib):
    """Four FP8 queries per scoring CTA and one CTA per query group (600
    lists: chunked prefill's configuration, where each CTA's own histograms
    give its lists' threshold bins): lists shorter than k, one of exactly k
    entries, long lists, and a run of equal keys."""
    rng = np.random.default_rng(23)
    lengths = [4 * 200 + 1, 4 * 300 + 3, 4 * 20000, 4 * 9000 + 2]
    lengths += [int(v) for v in rng.integers(4 * 300, 4 * 2500, size=146)]
    check_index_topk("fp8", lengths, T=4, seed=24)


def test_topk_resolves_the_last_digit(cuda_lib):
    """Forty keys whose scores are s0 (1 + 4e-6 j), about seven to a bin of
    the first 24 key bits: the 17th largest falls inside such a bin, so the
    last 8 bits decide which of its scores are kept.  fp32 keys (no
    quantisation) keep the spacing; the band of uncertainty is 1e-6, well
    under it."""
    rng = np.random.default_rng(9)
    wl = W.CSA_DECODE_4K_F32.with_(k=17)
    H_I, d_I, m = wl.H_I, wl.d_I, wl.m
    L_ctx = 4096
    n = L_ctx // m
    qi = (rng.standard_normal((1, 1, H_I, d_I)) * d_I ** -0.5).astype(np.float32)
    wi = np.full((1, 1, H_I), 0.5, dtype=np.float32)
    k0 = qi[0, 0].sum(axis=0)  # positive against every head's query (checked below)
    assert np.all(qi[0, 0] @ k0 > 0)
    keys_v = _rows(rng, n, d_I, scale=1e-3 * d_I ** -0.5)
    pos = rng.choice(n, size=40, replace=False)
    for j, g in enumerate(pos):
        keys_v[g] = (k0 * (1.0 + 4e-6 * j)).astype(np.float32)
    p = L.params(wl)
    keys = L.DeviceCache(1, n, "f32", d_I)
    st = storage.encode("f32", keys_v)
    upload(keys, 0, st)
    ctx = torch.tensor([L_ctx], dtype=torch.int32, device="cuda")
    out_idx = torch.full((1, 1, wl.k), -5, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.index_topk(p, dev(qi), dev(wi), keys, ctx, n, out_idx, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    sc = oracle_scores(quantize_query(qi[0, 0], "f32"), wi[0, 0], storage.decode(st))
    ok, msg = topk_set_ok(out_idx.cpu().numpy()[0, 0], sc, wl.k, band=1e-6)
    assert ok, msg
    assert set(out_idx.cpu().numpy()[0, 0].tolist()) == set(pos[23:].tolist())


def check_index_topk(fmt, lengths, T, seed, stalled=False):
    """Scores and top-k of a seeded case against the oracle.  ``stalled``:
    the bounded waits were set to run out (lcsc_set_wait_test); the call must
    then report LCSC_DEV_TIMEOUT and end without a CUDA error."""
    rng = np.random.default_rng(seed)
    if fmt == "f32":
        wl = W.CSA_DECODE_4K_F32.with_(k=64)
    else:
        wl = W.CSA_DECODE_128K.with_(idx_fmt=fmt, k=300)
    H_I, d_I, m = wl.H_I, wl.d_I, wl.m
    B = len(lengths)
    n_cap = L.round_capacity(max(lengths) // m + 1, fmt)
    keys_v = _rows(rng, B * n_cap, d_I).reshape(B, n_cap, d_I)
    keys_v[0, 100:110] = keys_v[0, 99]                 # a run of equal keys
    qi = (rng.standard_normal((B, T, H_I, d_I)) * d_I ** -0.5).astype(np.float32)
    if wl.q_dtype == "bf16":
        qi = torch.from_numpy(qi).to(torch.bfloat16).float().numpy()
    wi = (np.abs(rng.standard_normal((B, T, H_I))) * H_I ** -0.5).astype(np.float32)
    wi[2] *= np.where(rng.random(H_I) < 0.3, -1, 1).astype(np.float32)  # signed weights
    p = L.params(wl)
    keys = L.DeviceCache(B, n_cap, fmt, d_I)
    sts = []
    for b in range(B):
        st = storage.encode(fmt, keys_v[b])
        sts.append(st)
        upload(keys, b, st)
    ctx = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out_idx = torch.full((B, T, wl.k), -5, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros((B, T, wl.k), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.index_topk(p, dev(qi, TORCH_DT[wl.q_dtype]), dev(wi), keys, ctx, n_cap, out_idx, out_sc, status=status)
    torch.cuda.synchronize()
    if stalled:
        assert status.item() & L.DEV_TIMEOUT
        return
    assert status.item() == 0
    oi, osc = out_idx.cpu().numpy(), out_sc.cpu().numpy()
    for b in range(B):
        k_all = storage.decode(sts[b])
        for t in range(T):
            p_pos = lengths[b] - T + t
            n = (p_pos + 1) // m
            s = oracle_scores(quantize_query(qi[b, t], fmt), wi[b, t], k_all[:n])
            ok, msg = topk_set_ok(oi[b, t], s, wl.k)
            assert ok, f"b={b} t={t}: {msg}"
            k_eff = min(wl.k, n)
            assert np.all(oi[b, t, k_eff:] == -1)
            sel = oi[b, t, :k_eff]
            assert np.allclose(osc[b, t, :k_eff], s[sel], rtol=1e-5, atol=1e-6 * np.abs(s).max())


# -------------------------------------------------------------- attention

def _attn_case(kind, fmt_kv, rng):
    if fmt_kv == "f32":
        wl = W.CSA_DECODE_4K_F32.with_(k=64, w=40)
    else:
        wl = W.CSA_DECODE_128K.with_(k=200, w=100)
    if kind == "hca":
        wl = wl.with_(kind="hca", m=16, G=16)
    return wl


@pytest.mark.parametrize("kind", ["csa", "hca"])
@pytest.mark.parametrize("fmt_kv,q_dtype", [("f32", None), ("kv", None), ("kv", "f32")])
def test_attention_matches_oracle(cuda_lib, kind, fmt_kv, q_dtype):
    """fp32 rows (CUDA-core path) and FP8 + BF16 rows (tensor-core path),
    the latter with bf16 queries and outputs and with fp32 ones."""
    check_attention(kind, fmt_kv, q_dtype)


def check_attention(kind, fmt_kv, q_dtype, stalled=False):
    """One seeded sparse (CSA) or dense (HCA) attention call against the
    oracle.  ``stalled``: as in check_index_topk."""
    rng = np.random.default_rng(31)
    wl = _attn_case(kind, fmt_kv, rng)
    if q_dtype:
        wl = wl.with_(q_dtype=q_dtype)
    T = 2
    lengths = [3000, 30, 1500]                 # one context shorter than the window
    B = len(lengths)
    wl = wl.with_(T=T)
    m, D, Dv, H = wl.m, wl.D, wl.Dv, wl.H
    rope = wl.rope_dim if fmt_kv == "kv" else 0
    n_cap = max(lengths) // m + 1
    cap = wl.win_cap
    sep = wl.separate_v
    kv = L.DeviceCache(B, n_cap, fmt_kv, D, rope)
    v = L.DeviceCache(B, n_cap, fmt_kv, Dv, rope) if sep else None
    wk = L.DeviceCache(B, cap, fmt_kv, D, rope)
    wv = L.DeviceCache(B, cap, fmt_kv, Dv, rope) if sep else None
    st = {}
    for b in range(B):
        st[b] = {"kv": storage.encode(fmt_kv, _rows(rng, n_cap, D), rope),
                 "wk": storage.encode(fmt_kv, _rows(rng, cap, D), rope)}
        upload(kv, b, st[b]["kv"])
        upload(wk, b, st[b]["wk"])
        if sep:
            st[b]["v"] = storage.encode(fmt_kv, _rows(rng, n_cap, Dv), rope)
            st[b]["wv"] = storage.encode(fmt_kv, _rows(rng, cap, Dv), rope)
            upload(v, b, st[b]["v"])
            upload(wv, b, st[b]["wv"])
    q = (rng.standard_normal((B, T, H, D)) * D ** -0.5 * 8).astype(np.float32)
    if wl.q_dtype == "bf16":
        q = torch.from_numpy(q).to(torch.bfloat16).float().numpy()
    sink = rng.standard_normal(H).astype(np.float32)
    ctx = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, T, H, Dv), dtype=TORCH_DT[wl.q_dtype], device="cuda")
    lse = torch.zeros((B, T, H), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = L.params(wl)
    idx = None
    if kind == "csa":
        idx = np.full((B, T, wl.k), -1, dtype=np.int32)
        for b in range(B):
            for t in range(T):
                n = (lengths[b] - T + t + 1) // m
                k_eff = min(wl.k, n)
                idx[b, t, :k_eff] = rng.permutation(n)[:k_eff]
        L.sparse_attn(p, dev(q, TORCH_DT[wl.q_dtype]), kv, v, wk, wv, dev(idx, torch.int32), dev(sink), ctx,
                      out, lse, status=status)
    else:
        L.dense_attn(p, dev(q, TORCH_DT[wl.q_dtype]), kv, v, wk, wv, dev(sink), ctx, n_cap, out, lse,
                     status=status)
    torch.cuda.synchronize()
    if stalled:
        assert status.item() & L.DEV_TIMEOUT
        return
    assert status.item() == 0
    o_gpu, lse_gpu = out.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        K_all = storage.decode(st[b]["kv"])
        V_all = storage.decode(st[b]["v"]) if sep else K_all
        WK = storage.decode(st[b]["wk"])
        WV = storage.decode(st[b]["wv"]) if sep else WK
        for t in range(T):
            pp = lengths[b] - T + t
            n = (pp + 1) // m
            ent = idx[b, t][idx[b, t] >= 0] if kind == "csa" else np.arange(n)
            wpos = window_positions(pp, wl.w) % cap
            Kr = np.concatenate([K_all[ent], WK[wpos]])
            Vr = np.concatenate([V_all[ent], WV[wpos]])
            o, ls = joint_attention(q[b, t], Kr, Vr, sink, wl.sm_scale)
            assert rel_l2(o_gpu[b, t], o) <= ATTN_RTOL, (b, t, rel_l2(o_gpu[b, t], o))
            assert max_abs(o_gpu[b, t], o) <= ATTN_ATOL
            assert np.allclose(lse_gpu[b, t], ls, rtol=1e-4, atol=1e-4)


# two splits per query (combined) / one split with 148 SMs (written directly)
@pytest.mark.parametrize("T", [64, 148])
def test_attention_rescales_when_the_max_grows(cuda_lib, T):
    """Scores that jump by more than e^8 part-way through a split: the running
    reference max moves and the partial O accumulated so far is rescaled.
    Keys of a few entries point along the queries' shared direction with
    growing lengths, so every head's max jumps three times."""
    rng = np.random.default_rng(43)
    wl = W.CSA_DECODE_128K.with_(k=200, w=100, kind="hca", m=16, G=16, T=T)
    m, D, H = wl.m, wl.D, wl.H
    n_ent = 2048
    L0 = n_ent * m  # context of the last query
    n_cap = n_ent + 1
    K = _rows(rng, n_cap, D)
    u = rng.standard_normal(D)
    u /= np.linalg.norm(u)
    q = (u[None, None, :] * 2.0 + rng.standard_normal((1, T, H, D)) * D ** -0.5 * 0.3).astype(np.float32)
    q = torch.from_numpy(q).to(torch.bfloat16).float().numpy()
    base = float(np.mean(q[0] @ u))  # typical q . u
    for first, s_target in ((180, 9.5), (700, 19.0), (1500, 28.5)):
        for r in range(first, first + 3):
            K[r] = (u * s_target / (wl.sm_scale * base)).astype(np.float32)
    kv_st = storage.encode("kv", K, wl.rope_dim)
    wk_st = storage.encode("kv", _rows(rng, wl.win_cap, D), wl.rope_dim)
    kv = L.DeviceCache(1, n_cap, "kv", D, wl.rope_dim)
    wk = L.DeviceCache(1, wl.win_cap, "kv", D, wl.rope_dim)
    upload(kv, 0, kv_st)
    upload(wk, 0, wk_st)
    sink = rng.standard_normal(H).astype(np.float32)
    ctx = torch.tensor([L0], dtype=torch.int32, device="cuda")
    out = torch.zeros((1, T, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, T, H), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.dense_attn(L.params(wl), dev(q, torch.bfloat16), kv, None, wk, None, dev(sink), ctx, n_cap, out, lse,
                 status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_gpu, lse_gpu = out.float().cpu().numpy(), lse.cpu().numpy()
    K_all, WK = storage.decode(kv_st), storage.decode(wk_st)
    for t in list(range(0, T, 16)) + [T - 1]:
        pp = L0 - T + t
        n = (pp + 1) // m
        wpos = window_positions(pp, wl.w) % wl.win_cap
        Kr = np.concatenate([K_all[:n], WK[wpos]])
        o, ls = joint_attention(q[0, t], Kr, Kr, sink, wl.sm_scale)
        assert rel_l2(o_gpu[0, t], o) <= ATTN_RTOL, (t, rel_l2(o_gpu[0, t], o))
        # the boosted rows are also the values (shared KV), so the output is
        # far from unit scale: the absolute bound scales with it (bf16 output)
        assert max_abs(o_gpu[0, t], o) <= ATTN_ATOL * max(1.0, float(np.abs(o).max()))
        assert np.allclose(lse_gpu[0, t], ls, rtol=1e-4, atol=1e-4)


def test_attention_flags_out_of_range_index(cuda_lib):
    rng = np.random.default_rng(41)
    wl = W.CSA_DECODE_4K_F32.with_(k=8, w=4)
    B, T, H, D = 1, 1, wl.H, wl.D
    n_cap = 64
    kv = L.DeviceCache(B, n_cap, "f32", D)
    v = L.DeviceCache(B, n_cap, "f32", D)
    wk = L.DeviceCache(B, wl.win_cap, "f32", D)
    wv = L.DeviceCache(B, wl.win_cap, "f32", D)
    for c in (kv, v, wk, wv):
        c.data.copy_(torch.from_numpy(_rows(rng, c.capacity, D)).cuda()[None])
    ctx = torch.tensor([40], dtype=torch.int32, device="cuda")  # N = 10 visible entries
    idx = torch.tensor([[[0, 3, 9, 10, 500, -1, -3, 2]]], dtype=torch.int32, device="cuda")
    q = dev(_rows(rng, H, D)[None, None])
    out = torch.zeros((B, T, H, D), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.sparse_attn(L.params(wl), q, kv, v, wk, wv, idx, None, ctx, out, None, status=status)
    torch.cuda.synchronize()
    assert status.item() & L.DEV_BAD_INDEX
    # the result equals attention over the valid indices alone
    Kn, Vn = kv.data[0].cpu().double().numpy(), v.data[0].cpu().double().numpy()
    Wk, Wv = wk.data[0].cpu().double().numpy(), wv.data[0].cpu().double().numpy()
    wpos = window_positions(39, 4) % wl.win_cap
    ent = [0, 3, 9, 2]
    o, _ = joint_attention(q[0, 0].cpu().double().numpy(), np.concatenate([Kn[ent], Wk[wpos]]),
                           np.concatenate([Vn[ent], Wv[wpos]]), np.full(H, -np.inf), wl.sm_scale)
    assert rel_l2(out[0, 0].cpu().numpy(), o) < 1e-5


def _dense_kv_case(rng, wl, n_cap, rope_scale=1.0):
    """One sequence of stored KV entries and window rows for the 512-dim
    FP8 + BF16 path; the BF16 RoPE dims multiplied by ``rope_scale``."""
    D, R = wl.D, wl.rope_dim
    K = _rows(rng, n_cap, D)
    K[:, D - R:] *= rope_scale
    Wr = _rows(rng, wl.win_cap, D)
    Wr[:, D - R:] *= rope_scale
    kv_st, wk_st = storage.encode("kv", K, R), storage.encode("kv", Wr, R)
    kv = L.DeviceCache(1, n_cap, "kv", D, R)
    wk = L.DeviceCache(1, wl.win_cap, "kv", D, R)
    upload(kv, 0, kv_st)
    upload(wk, 0, wk_st)
    return kv, wk, storage.decode(kv_st), storage.decode(wk_st)


@pytest.mark.parametrize("q_scale", [2.0 ** 20, 2.0 ** -20, 2.0 ** 60, 2.0 ** -60])
def test_attention_query_magnitude_outside_f16(cuda_lib, q_scale):
    """Queries far outside the f16 range (bf16 holds them) with the softmax
    scale divided by the same factor, so the logits stay as they were: the
    tensor-core path scales each head into range and gives the oracle's
    answer (before that scaling, 2^20 overflowed f16 and 2^-20 lost the
    queries to f16 subnormals)."""
    rng = np.random.default_rng(51)
    wl = W.CSA_DECODE_128K.with_(k=200, w=100, kind="hca", m=16, G=16, T=2)
    n_cap = 600
    L0 = (n_cap - 1) * wl.m
    kv, wk, K_all, WK = _dense_kv_case(rng, wl, n_cap)
    q = (rng.standard_normal((1, 2, wl.H, wl.D)) * wl.D ** -0.5 * 8 * q_scale)
    q = torch.from_numpy(q.astype(np.float32)).to(torch.bfloat16)
    p = L.params(wl)
    p.sm_scale = wl.sm_scale / q_scale
    sink = rng.standard_normal(wl.H).astype(np.float32)
    ctx = torch.tensor([L0], dtype=torch.int32, device="cuda")
    out = torch.zeros((1, 2, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, wl.H), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.dense_attn(p, q.cuda(), kv, None, wk, None, dev(sink), ctx, n_cap, out, lse, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    qf = q.float().numpy().astype(np.float64)
    for t in range(2):
        pp = L0 - 2 + t
        wpos = window_positions(pp, wl.w) % wl.win_cap
        Kr = np.concatenate([K_all[:(pp + 1) // wl.m], WK[wpos]])
        o, ls = joint_attention(qf[0, t], Kr, Kr, sink, float(np.float32(p.sm_scale)))
        got = out[0, t].float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_l2(got, o) <= ATTN_RTOL, (q_scale, t, rel_l2(got, o))
        assert max_abs(got, o) <= ATTN_ATOL
        assert np.allclose(lse[0, t].cpu().numpy(), ls, rtol=1e-4, atol=1e-4)


def test_attention_kv_range(cuda_lib):
    """Stored KV rows far from unit scale give the oracle's answer: tiny BF16
    RoPE dims, RoPE dims far beyond the f16 range, and an FP8 row scale whose
    codes times the scale pass 65504 (the E4M3 codes and the BF16 dims enter
    the tensor cores as stored; the row scale is applied in float32)."""
    rng = np.random.default_rng(52)
    wl = W.CSA_DECODE_128K.with_(k=200, w=100, kind="hca", m=16, G=16, T=1)
    n_cap = 300
    L0 = (n_cap - 1) * wl.m
    q = torch.from_numpy((rng.standard_normal((1, 1, wl.H, wl.D)) * wl.D ** -0.5 * 8).astype(np.float32))
    q = q.to(torch.bfloat16)
    qf = q.float().numpy()[0, 0].astype(np.float64)
    sink = dev(rng.standard_normal(wl.H).astype(np.float32))
    ctx = torch.tensor([L0], dtype=torch.int32, device="cuda")
    wpos = window_positions(L0 - 1, wl.w) % wl.win_cap

    def check(kv, wk, K_all, WK):
        out = torch.zeros((1, 1, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.dense_attn(L.params(wl), q.cuda(), kv, None, wk, None, sink, ctx, n_cap, out, None, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        Kr = np.concatenate([K_all[:L0 // wl.m], WK[wpos]])
        o, _ = joint_attention(qf, Kr, Kr, sink.cpu().numpy(), wl.sm_scale)
        got = out[0, 0].float().cpu().numpy()
        assert np.all(np.isfinite(got))
        # outputs far from unit scale: the absolute bound scales with them (bf16 output)
        assert rel_l2(got, o) <= ATTN_RTOL, rel_l2(got, o)
        assert max_abs(got, o) <= ATTN_ATOL * max(1.0, float(np.abs(o).max()))

    check(*_dense_kv_case(rng, wl, n_cap, rope_scale=1e-6))
    check(*_dense_kv_case(rng, wl, n_cap, rope_scale=300.0))  # RoPE dims ~ 1e3 .. 1e4
    kv, wk, K_all, WK = _dense_kv_case(rng, wl, n_cap)
    kv.scale[0, 7] *= 200.0  # one entry's E4M3 codes times its scale pass 65504
    K_all = K_all.copy()
    K_all[7, :wl.D - wl.rope_dim] *= 200.0
    check(kv, wk, K_all, WK)
