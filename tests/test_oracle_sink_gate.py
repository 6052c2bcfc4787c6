"""Pins of the two readings added as parameters (CPU only):

* the sink token ("DeepSeek V4 Architecture Explained", "How
  compress-then-sparsify attention works": the sink lets a head keep part of
  its weight off every row; read here as the raw row of position 0 joining
  every row set, counted once), pinned against library attention over an
  explicit mask, closed forms and a step-by-step restatement;
* caller-given gate logits (the same section: trainable compression weights,
  a softmax over the group, learnable positional biases; the logit row of a
  token given by the caller in place of x W), pinned against the projection
  form, the mean closed form and a dominance case that shows the positional
  bias is added per place in each overlapping group.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import storage
from oracle.compress import compress_entries, pool_group
from oracle.step import layer_step


def _sdpa_masked(q, K, keep):
    """torch SDPA (float64, CPU) of q [H, D] over the rows K[keep]."""
    mask = torch.zeros(q.shape[0], K.shape[0], dtype=torch.bool)
    mask[:, torch.from_numpy(np.asarray(keep))] = True
    out = Fn.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(K)[None],
                                          torch.from_numpy(K)[None], attn_mask=mask,
                                          scale=1.0 / np.sqrt(q.shape[1]))
    return out[0].numpy()


def _f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _stored(n, d, rows=None):
    pay = np.zeros((n, d), np.float32) if rows is None else np.asarray(rows, np.float32)
    return storage.Stored("f32", pay, None, d)


def _token_step(x, q, *, m, w, L, T, tok=None, sink=None, kind="hca", xi=None, qi=None, wi=None, k=0,
                sink_mode="token"):
    """One f32 step over raw tokens x [>= L, D] with the caches holding what
    precedes the step (zero-gate entries, window ring rows, the position-0
    row when the step does not receive it).  Returns (out, tok_kv)."""
    D = x.shape[1]
    G = m
    n_cap = L // m + 1
    zW, zB = np.zeros((D, D)), np.zeros((G, D))
    n_old = (L - T) // m
    kv = _stored(n_cap, D)
    kv.payload[:n_old] = compress_entries(x, 0, zW, zB, m, G, range(n_old))
    idx = None
    if kind == "csa":
        di = xi.shape[1]
        idx = _stored(n_cap, di)
        idx.payload[:n_old] = compress_entries(xi, 0, np.zeros((di, di)), np.zeros((G, di)), m, G,
                                               range(n_old))
    cap = max(T + w - 1, 1)
    ring = _stored(cap, D)
    for pos in range(max(0, L - T - w + 1), L - T):
        ring.payload[pos % cap] = x[pos]
    tok_kv = tok if tok is not None else _stored(1, D, x[:1] if L - T > 0 else None)
    R = T + G - 1
    lo = L - R
    pad = lambda a: np.concatenate([np.zeros((max(0, -lo), a.shape[1])), a[max(lo, 0):L]])
    out = layer_step(kind, m=m, G=G, w=w, k=k, sm_scale=1 / np.sqrt(D), kv_fmt="f32", rope_dim=0,
                     idx_fmt="f32", L=L, T=T, kv=kv, v=None, idx=idx, ring_kv=ring, ring_v=None,
                     x_kv=pad(x), x_v=None, x_idx=None if xi is None else pad(xi), W_kv=zW, B_kv=zB,
                     W_v=None, B_v=None, W_idx=None if xi is None else np.zeros((xi.shape[1],) * 2),
                     B_idx=None if xi is None else np.zeros((G, xi.shape[1])), q=q, q_idx=qi, w_idx=wi,
                     sink=sink if sink is not None else np.zeros(q.shape[1]), sink_mode=sink_mode,
                     tok_kv=tok_kv)
    return out, tok_kv


# ------------------------------------------------------------------ sink token

def test_token_with_window_covering_everything_is_causal_attention():
    """w >= L: position 0 is already in the window and enters once, so the
    step is textbook causal attention over the raw tokens."""
    rng = np.random.default_rng(11)
    L, D, H, T = 23, 8, 3, 4
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((T, H, D))
    out, _ = _token_step(x, q, m=128, w=L, L=L, T=T)  # m > L: no entries
    for i in range(T):
        p = L - T + i
        assert np.allclose(out["o"][i], _sdpa_masked(q[i], x, np.arange(p + 1)), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("w", [0, 1, 3])
def test_token_joins_the_window_as_one_more_key(w):
    """w small: the row set is {0} plus the window, a masked library attention."""
    rng = np.random.default_rng(12 + w)
    L, D, H = 30, 8, 2
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((1, H, D))
    out, _ = _token_step(x, q, m=128, w=w, L=L, T=1)
    keep = [0] + list(range(max(0, L - w), L))
    assert np.allclose(out["o"][0], _sdpa_masked(q[0], x, keep), rtol=1e-12, atol=1e-13)
    # no learned logit: the weights of the row set sum to one (lse = log of the full sum)
    l = (q[0] @ x[keep].T) / np.sqrt(D)
    assert np.allclose(out["lse"][0], np.log(np.exp(l).sum(axis=1)), rtol=1e-13)


def test_token_two_key_closed_form():
    """w = 1 and no entries: o = (e^l0 x_0 + e^lp x_p) / (e^l0 + e^lp)."""
    rng = np.random.default_rng(15)
    L, D, H = 9, 4, 2
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((1, H, D))
    out, _ = _token_step(x, q, m=128, w=1, L=L, T=1)
    l0, lp = (q[0] @ x[0]) / 2.0, (q[0] @ x[L - 1]) / 2.0
    want = (np.exp(l0)[:, None] * x[0] + np.exp(lp)[:, None] * x[L - 1]) / (np.exp(l0) + np.exp(lp))[:, None]
    assert np.allclose(out["o"][0], want, rtol=1e-13)


def test_first_token_attends_to_itself_once():
    rng = np.random.default_rng(16)
    D, H = 4, 3
    x = _f32(rng.standard_normal((1, D)))
    q = rng.standard_normal((1, H, D))
    out, tok = _token_step(x, q, m=4, w=128, L=1, T=1)
    assert np.allclose(out["o"][0], np.tile(x[0], (H, 1)), rtol=1e-15)
    assert np.allclose(out["lse"][0], (q[0] @ x[0]) / 2.0, rtol=1e-14)  # one key: lse = its logit
    assert np.array_equal(tok.payload[0], x[0].astype(np.float32))


def test_step_receiving_position_0_keeps_its_row_for_later_steps():
    rng = np.random.default_rng(17)
    D, H, w = 8, 2, 3
    x = _f32(rng.standard_normal((40, D)))
    tok = _stored(1, D)  # empty: the first chunk must fill it
    _token_step(x, rng.standard_normal((6, H, D)), m=128, w=w, L=6, T=6, tok=tok)
    assert np.array_equal(tok.payload[0], x[0].astype(np.float32))
    q = rng.standard_normal((1, H, D))
    out, _ = _token_step(x, q, m=128, w=w, L=40, T=1, tok=tok)
    assert np.allclose(out["o"][0], _sdpa_masked(q[0], x, [0, 37, 38, 39]), rtol=1e-12, atol=1e-13)


def test_token_sink_with_entries_matches_brute_force_row_set():
    """CSA with entries: S = top-k entries + window + {0}, against SDPA over
    the explicit rows (entries are zero-gate means of their groups)."""
    rng = np.random.default_rng(18)
    L, D, H, m, w, k = 64, 8, 2, 4, 5, 6
    x = _f32(rng.standard_normal((L, D)))
    xi = rng.standard_normal((L, 4))
    q, qi, wi = rng.standard_normal((1, H, D)), rng.standard_normal((1, 2, 4)), np.ones((1, 2))
    out, _ = _token_step(x, q, m=m, w=w, L=L, T=1, kind="csa", xi=xi, qi=qi, wi=wi, k=k)
    ent = _f32(x[: (L // m) * m].reshape(-1, m, D).mean(axis=1))  # stored as float32
    sel = np.asarray(out["sel"][0])
    K = np.concatenate([ent[sel], x[L - w:], x[:1]])
    assert np.allclose(out["o"][0], _sdpa_masked(q[0], K, np.arange(K.shape[0])), rtol=1e-12, atol=1e-13)


def test_token_t_step_equals_t_one_token_steps():
    rng = np.random.default_rng(19)
    L, D, H, T = 26, 8, 2, 5
    x = _f32(rng.standard_normal((L, D)))
    q = rng.standard_normal((T, H, D))
    many, _ = _token_step(x, q, m=4, w=3, L=L, T=T)
    for i in range(T):
        one, _ = _token_step(x, q[i:i + 1], m=4, w=3, L=L - T + i + 1, T=1)
        assert np.allclose(many["o"][i], one["o"][0], rtol=1e-13, atol=1e-14)


# ------------------------------------------------------- caller-given gate logits

@pytest.mark.parametrize("m,G", [(4, 4), (4, 8), (128, 128)])
def test_logits_equal_to_the_projection_reproduce_it(m, G):
    rng = np.random.default_rng(20 + G)
    n, D = 3 * m + (G - m), 16
    x = rng.standard_normal((n, D))
    W, Bp = rng.standard_normal((D, D)) * 0.3, rng.standard_normal((G, D))
    x_pos0 = -(G - m)
    ents = range(0, n // m)
    ents = [g for g in ents if (g + 1) * m - x_pos0 <= n]
    a = compress_entries(x, x_pos0, W, Bp, m, G, ents)
    b = compress_entries(x, x_pos0, np.full((D, D), np.nan), Bp, m, G, ents, U=x @ W)
    assert np.allclose(a, b, rtol=1e-14, atol=1e-15)


def test_constant_logits_without_bias_give_the_mean():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((12, 6))
    U = np.tile(rng.standard_normal((1, 6)), (12, 1))
    e = compress_entries(x, 0, None, np.zeros((4, 6)), 4, 4, range(3), U=U)
    assert np.allclose(e, x.reshape(3, 4, 6).mean(axis=1), atol=1e-15)


def test_logits_keep_the_positional_bias_of_each_place():
    """Token 4 has a huge logit in channel 2.  With overlapping groups (m = 4,
    G = 8) it is place 4 of entry 1 and place 0 of entry 2; a bias that sinks
    place 0 flips the winner of entry 2 only."""
    rng = np.random.default_rng(22)
    x = rng.standard_normal((16, 5))
    U = np.zeros((16, 5))
    U[4, 2] = 1e4
    Bp = np.zeros((8, 5))
    e = compress_entries(x, 0, None, Bp, 4, 8, [1, 2], U=U)
    assert np.isclose(e[0, 2], x[4, 2]) and np.isclose(e[1, 2], x[4, 2])
    Bp[0, 2] = -3e4
    e = compress_entries(x, 0, None, Bp, 4, 8, [1, 2], U=U)
    assert np.isclose(e[0, 2], x[4, 2])                       # place 4 of entry 1: no bias
    assert np.isclose(e[1, 2], x[5:12, 2].mean(), atol=1e-12)  # place 0 sunk: the other 7 tie
    _, alpha = pool_group(x[4:12], None, Bp, U[4:12])
    assert alpha[0, 2] == 0.0
