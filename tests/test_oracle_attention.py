"""Pins of the oracle's joint attention and of whole oracle steps (CPU only):
reductions to textbook dense attention, masked brute force, closed forms of
the sink and the window, and CSA/HCA consistency."""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import storage
from oracle.attention import attention_weights, inverse_rope, joint_attention, window_positions
from oracle.step import layer_step


def _sdpa(q, K, V, mask=None):
    """Library attention (torch, float64, CPU): q [H, D], K [S, D], V [S, Dv]."""
    qt = torch.from_numpy(q)[None]               # [1, H, D] as (batch, L=H, D)
    out = Fn.scaled_dot_product_attention(qt, torch.from_numpy(K)[None], torch.from_numpy(V)[None],
                                          attn_mask=mask, scale=1.0 / np.sqrt(q.shape[1]))
    return out[0].numpy()


def test_no_sink_is_library_softmax_attention():
    rng = np.random.default_rng(1)
    q, K, V = rng.standard_normal((4, 32)), rng.standard_normal((50, 32)), rng.standard_normal((50, 24))
    o, lse = joint_attention(q, K, V, np.full(4, -np.inf), 1 / np.sqrt(32))
    assert np.allclose(o, _sdpa(q, K, V), rtol=1e-12, atol=1e-13)
    ref_lse = torch.logsumexp(torch.from_numpy(q @ K.T / np.sqrt(32)), dim=1).numpy()
    assert np.allclose(lse, ref_lse, rtol=1e-13)


def test_selected_set_is_masked_brute_force():
    rng = np.random.default_rng(2)
    q, K = rng.standard_normal((3, 16)), rng.standard_normal((40, 16))
    sel = np.array([3, 7, 8, 20, 39])
    mask = torch.zeros(3, 40, dtype=torch.bool)
    mask[:, torch.from_numpy(sel)] = True
    o, _ = joint_attention(q, K[sel], K[sel], np.full(3, -np.inf), 0.25)
    assert np.allclose(o, _sdpa(q, K, K, mask), rtol=1e-12, atol=1e-13)


def test_sink_closed_form_single_key():
    q = np.array([[0.5, -1.0, 2.0]])
    k = np.array([[1.0, 0.25, 0.5]])
    v = np.array([[3.0, -2.0]])
    sigma = 0.7
    o, lse = joint_attention(q, k, v, np.array([sigma]), 1.0)
    l = float(q[0] @ k[0])
    assert np.allclose(o[0], v[0] * np.exp(l) / (np.exp(sigma) + np.exp(l)), rtol=1e-14)
    assert np.isclose(lse[0], np.log(np.exp(sigma) + np.exp(l)), rtol=1e-14)


def test_sink_makes_weights_sum_below_one():
    rng = np.random.default_rng(3)
    q, K = rng.standard_normal((5, 8)), rng.standard_normal((30, 8))
    sink = rng.standard_normal(5)
    wts = attention_weights(q, K, sink, 0.3)
    _, lse = joint_attention(q, K, K, sink, 0.3)
    tot = wts.sum(axis=1)
    assert np.all(tot < 1)
    assert np.allclose(tot, 1 - np.exp(sink - lse), rtol=1e-13)


def test_empty_set():
    o, lse = joint_attention(np.ones((2, 4)), np.zeros((0, 4)), np.zeros((0, 3)), np.array([0.5, -np.inf]), 1.0)
    assert np.all(o == 0) and lse[0] == 0.5 and lse[1] == -np.inf


def test_window_positions():
    assert list(window_positions(5, 3)) == [3, 4, 5]
    assert list(window_positions(1, 128)) == [0, 1]
    assert list(window_positions(7, 1)) == [7]


# ------------------------------------------------------------- whole steps

def _f32_state(n_cap, d, rows=None):
    payload = np.zeros((n_cap, d), np.float32) if rows is None else rows.astype(np.float32)
    return storage.Stored("f32", payload, None, d)


def _f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _run(kind, x, q, *, m, G, w, k, L, T, sink, qi=None, wi=None, xi=None, cap=None, rope_dim=0,
         out_rope_base=0.0):
    """A step over raw f32 tokens x [L, D] (float32-exact values, as the f32
    format stores them) whose cache already holds every entry before the
    step's tokens (pooled with zero gates)."""
    D = x.shape[1]
    n_cap = L // m + 1
    W0, B0 = np.zeros((D, D)), np.zeros((G, D))
    from oracle.compress import compress_entries
    n_old = (L - T) // m
    kv = _f32_state(n_cap, D)
    kv.payload[:n_old] = compress_entries(x, 0, W0, B0, m, G, range(n_old))
    idx = None
    if kind == "csa":
        di = xi.shape[1]
        idx = _f32_state(n_cap, di)
        idx.payload[:n_old] = compress_entries(xi, 0, np.zeros((di, di)), np.zeros((G, di)), m, G,
                                               range(n_old))
    cap = cap or max(T + w - 1, 1)
    ring = _f32_state(cap, D)
    for pos in range(max(0, L - T - w + 1), L - T):
        ring.payload[pos % cap] = x[pos]
    R = T + G - 1
    lo = L - R
    xt = np.concatenate([np.zeros((max(0, -lo), D)), x[max(lo, 0):L]])
    xit = None
    if kind == "csa":
        xit = np.concatenate([np.zeros((max(0, -lo), xi.shape[1])), xi[max(lo, 0):L]])
    return layer_step(kind, m=m, G=G, w=w, k=k, sm_scale=1 / np.sqrt(D), kv_fmt="f32", rope_dim=rope_dim,
                      idx_fmt="f32", L=L, T=T, kv=kv, v=None, idx=idx, ring_kv=ring, ring_v=None,
                      x_kv=xt, x_v=None, x_idx=xit, W_kv=W0, B_kv=B0, W_v=None, B_v=None,
                      W_idx=None if kind != "csa" else np.zeros((xi.shape[1],) * 2),
                      B_idx=None if kind != "csa" else np.zeros((G, xi.shape[1])),
                      q=q, q_idx=qi, w_idx=wi, sink=sink, out_rope_base=out_rope_base)


def _causal_sdpa(x, q, L, T):
    """Textbook causal attention of the T last queries over raw tokens."""
    outs = []
    for i in range(T):
        p = L - T + i
        outs.append(_sdpa(q[i], x[:p + 1], x[:p + 1]))
    return np.stack(outs)


@pytest.mark.parametrize("T", [1, 5])
def test_m1_all_entries_no_window_no_sink_is_dense_causal_attention(T):
    rng = np.random.default_rng(4)
    L, D, H = 37, 16, 3
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((T, H, D))
    xi = rng.standard_normal((L, 8))
    qi = rng.standard_normal((T, 2, 8))
    wi = np.abs(rng.standard_normal((T, 2)))
    no_sink = np.full(H, -np.inf)
    out = _run("csa", x, q, m=1, G=1, w=0, k=L, L=L, T=T, sink=no_sink, qi=qi, wi=wi, xi=xi)
    assert np.allclose(out["o"], _causal_sdpa(x, q, L, T), rtol=1e-11, atol=1e-12)
    out_h = _run("hca", x, q, m=1, G=1, w=0, k=0, L=L, T=T, sink=no_sink)
    assert np.allclose(out_h["o"], out["o"], rtol=1e-12, atol=1e-13)


def test_window_covering_everything_is_dense_causal_attention():
    rng = np.random.default_rng(5)
    L, D, H, T = 29, 8, 2, 3
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((T, H, D))
    xi, qi = rng.standard_normal((L, 4)), rng.standard_normal((T, 1, 4))
    out = _run("csa", x, q, m=4, G=4, w=L, k=0, L=L, T=T, sink=np.full(H, -np.inf), qi=qi,
               wi=np.ones((T, 1)), xi=xi)
    assert np.allclose(out["o"], _causal_sdpa(x, q, L, T), rtol=1e-11, atol=1e-12)


def test_window_of_one_is_the_own_token_with_sink():
    rng = np.random.default_rng(6)
    L, D, H = 20, 8, 2
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((1, H, D))
    sink = np.array([0.3, -0.4])
    out = _run("hca", x, q, m=128, G=128, w=1, k=0, L=L, T=1, sink=sink)  # no entry yet
    l = (q[0] @ x[L - 1]) / np.sqrt(D)
    want = x[L - 1][None] * (np.exp(l) / (np.exp(sink) + np.exp(l)))[:, None]
    assert np.allclose(out["o"][0], want, rtol=1e-13)


def test_csa_with_k_at_least_n_equals_hca_same_m():
    rng = np.random.default_rng(7)
    L, D, H, T = 64, 8, 2, 2
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((T, H, D))
    xi, qi = rng.standard_normal((L, 4)), rng.standard_normal((T, 2, 4))
    sink = rng.standard_normal(H)
    c = _run("csa", x, q, m=4, G=4, w=5, k=1000, L=L, T=T, sink=sink, qi=qi,
             wi=np.abs(rng.standard_normal((T, 2))), xi=xi)
    h = _run("hca", x, q, m=4, G=4, w=5, k=0, L=L, T=T, sink=sink)
    assert np.allclose(c["o"], h["o"], rtol=1e-12, atol=1e-13)
    assert np.allclose(c["lse"], h["lse"], rtol=1e-13)


def test_step_compresses_only_closing_groups():
    rng = np.random.default_rng(8)
    D, H = 4, 1
    for L, T, want in [(16, 1, (3, 4)), (17, 1, (4, 4)), (16, 8, (2, 4)), (18, 5, (3, 4))]:
        x = _f32(rng.standard_normal((L, D)))
        q = rng.standard_normal((T, H, D))
        out = _run("hca", x, q, m=4, G=4, w=2, k=0, L=L, T=T, sink=np.zeros(H))
        assert out["new_entries"] == want


# ------------------------------------------------------- output inverse RoPE

def _rotate_complex(v, p, base, sign):
    """Pairs (2j, 2j + 1) as complex numbers x + iy times exp(sign i p theta_j),
    theta_j = base^(-2j / d): an independent statement of the rotation."""
    d = v.shape[-1]
    z = v[..., 0::2] + 1j * v[..., 1::2]
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    z = z * np.exp(sign * 1j * p * theta)
    out = np.empty_like(v, dtype=np.float64)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def test_inverse_rope_closed_forms():
    # one pair, theta_0 = 1: (1, 0) turned by -1 radian
    o = np.array([[7.0, 1.0, 0.0]])
    got = inverse_rope(o, 1, 2, 10000.0)
    assert got[0, 0] == 7.0
    assert np.allclose(got[0, 1:], [np.cos(1.0), -np.sin(1.0)], rtol=0, atol=1e-15)
    # second pair of four dims with base 100: theta_1 = 0.1, p = 5 -> -0.5 rad
    o = np.array([0.0, 0.0, 0.0, 2.0])
    got = inverse_rope(o, 5, 4, 100.0)
    assert np.allclose(got[2:], [-2.0 * np.sin(-0.5), 2.0 * np.cos(-0.5)], rtol=0, atol=1e-15)
    # position 0 and a zero base leave the output unchanged
    rng = np.random.default_rng(1)
    o = rng.standard_normal((3, 16))
    assert np.array_equal(inverse_rope(o, 0, 8, 10000.0), o)
    assert np.array_equal(inverse_rope(o, 123, 8, 0.0), o)


def test_inverse_rope_matches_complex_rotation_and_undoes_rope():
    rng = np.random.default_rng(2)
    H, D, R = 4, 24, 8
    o = rng.standard_normal((H, D))
    p = 1_000_003
    got = inverse_rope(o, p, R, 10000.0)
    assert np.array_equal(got[:, :D - R], o[:, :D - R])            # the other dims untouched
    assert np.allclose(got[:, D - R:], _rotate_complex(o[:, D - R:], p, 10000.0, -1), rtol=1e-9, atol=1e-12)
    pair_norm = lambda v: np.hypot(v[..., 0::2], v[..., 1::2])
    assert np.allclose(pair_norm(got[:, D - R:]), pair_norm(o[:, D - R:]), rtol=1e-12)
    forward = o.copy()
    forward[:, D - R:] = _rotate_complex(o[:, D - R:], p, 10000.0, +1)
    assert np.allclose(inverse_rope(forward, p, R, 10000.0), o, rtol=1e-9, atol=1e-12)


def test_inverse_rope_leaves_relative_positions():
    """Values whose rope dims are a vector turned by their key positions: after
    the inverse rotation by the query position the output depends only on
    the key positions relative to the query (a common shift changes nothing).
    The query's rope dims are zero, so the weights do not move either."""
    rng = np.random.default_rng(3)
    S, D, R, H = 6, 16, 8, 2
    base_rows = rng.standard_normal((S, D))
    q = rng.standard_normal((H, D))
    q[:, D - R:] = 0.0
    key_pos = rng.integers(0, 500, size=S)
    p_q = 700

    def out(shift):
        K = base_rows.copy()
        for j in range(S):
            K[j, D - R:] = _rotate_complex(base_rows[j, D - R:], key_pos[j] + shift, 10000.0, +1)
        o, _ = joint_attention(q, K, K, np.full(H, -np.inf), 0.3)
        return inverse_rope(o, p_q + shift, R, 10000.0)

    assert np.allclose(out(0), out(12345), rtol=1e-9, atol=1e-12)
    # turning the other way (a sign slip) would not be shift-invariant
    o0 = joint_attention(q, base_rows, base_rows, np.full(H, -np.inf), 0.3)[0]
    assert not np.allclose(inverse_rope(o0, 1, R, 10000.0), inverse_rope(o0, -1, R, 10000.0))


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_t_token_step_equals_t_decode_steps(kind):
    """Five new tokens in one step (draft-token decode) answer each query as
    five successive one-token steps would: same visible entries (groups
    closing inside the chunk included), same window, same selection, same
    output after the inverse rotation by each query's own position."""
    rng = np.random.default_rng(11)
    L, D, H, T, R = 61, 8, 2, 5, 4
    m, G, w, k = 4, 8, 5, 6
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((T, H, D))
    sink = rng.standard_normal(H)
    kw = dict(m=m, G=G, w=w, k=k if kind == "csa" else 0, sink=sink, rope_dim=R, out_rope_base=100.0)
    if kind == "csa":
        xi = _f32(rng.standard_normal((L, 4)))
        qi, wi = rng.standard_normal((T, 2, 4)), np.abs(rng.standard_normal((T, 2)))
    whole = _run(kind, x, q, L=L, T=T, **kw, **({"qi": qi, "wi": wi, "xi": xi} if kind == "csa" else {}))
    for t in range(T):
        Lt = L - T + t + 1
        one = _run(kind, x[:Lt], q[t:t + 1], L=Lt, T=1, cap=T + w - 1, **kw,
                   **({"qi": qi[t:t + 1], "wi": wi[t:t + 1], "xi": xi[:Lt]} if kind == "csa" else {}))
        assert np.allclose(whole["o"][t], one["o"][0], rtol=1e-12, atol=1e-13)
        assert np.allclose(whole["lse"][t], one["lse"][0], rtol=1e-12)
        if kind == "csa":
            assert np.array_equal(np.sort(whole["sel"][t]), np.sort(one["sel"][0]))
