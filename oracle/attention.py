"""Joint attention over compressed entries, the sliding window and a sink.

Test infrastructure only (see ``oracle/__init__.py``).

Sources: "DeepSeek V4 Architecture Explained", "How compress-then-sparsify
attention works" (exact attention over the selected compressed entries, a
small sliding-window branch of uncompressed recent tokens, and a sink term
that leaves part of each head's probability mass unassigned to any row; HCA
is the same with larger groups and no selection, with the shared-KV
multi-query layout); "Inside DeepSeek-V4", sections 1-2 (window w = 128);
"How DeepSeek V4 Handles 1M Token Context", Component 3 (scaled dot-product
attention over the gathered entries, plus the 128-token window).

Readings: the entries and the window rows form ONE softmax (one normaliser
across both branches, no de-duplication of tokens that appear in both); the
sink is a learned logit sigma[h] per head with a zero value vector, so it
only adds exp(sigma[h]) to the denominator; every head attends to the same
(shared) key rows; the window of a query at position p is the raw rows at
positions max(0, p - w + 1) .. p.

For head h with logits l_j = sm_scale * q[h] . K_j over the row set S:

    o[h] = sum_j exp(l_j - M) V_j / (exp(sigma[h] - M) + sum_j exp(l_j - M))
    lse[h] = M + log(exp(sigma[h] - M) + sum_j exp(l_j - M))

with M = max(sigma[h], max_j l_j).  An empty S with sigma = -inf gives
o = 0 and lse = -inf.
"""
import numpy as np


def joint_attention(q, K, V, sink, sm_scale):
    """q [H, D], K [S, D], V [S, Dv], sink [H] -> (o [H, Dv], lse [H])."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    sink = np.asarray(sink, dtype=np.float64)
    H = q.shape[0]
    Dv = V.shape[1]
    if K.shape[0] == 0:
        M = sink.copy()
        with np.errstate(invalid="ignore"):
            lse = np.where(np.isfinite(sink), sink, -np.inf)
        return np.zeros((H, Dv)), lse
    logits = sm_scale * (q @ K.T)                     # [H, S]
    M = np.maximum(sink, logits.max(axis=1))
    e = np.exp(logits - M[:, None])
    Z = np.exp(sink - M) + e.sum(axis=1)
    o = (e @ V) / Z[:, None]
    return o, M + np.log(Z)


def attention_weights(q, K, sink, sm_scale):
    """The softmax weights of each row (sink excluded), [H, S]; they sum to
    1 - exp(sigma - lse) < 1 per head when sigma is finite."""
    q = np.asarray(q, dtype=np.float64)
    logits = sm_scale * (q @ np.asarray(K, dtype=np.float64).T)
    M = np.maximum(sink, logits.max(axis=1))
    e = np.exp(logits - M[:, None])
    Z = np.exp(np.asarray(sink, dtype=np.float64) - M) + e.sum(axis=1)
    return e / Z[:, None]


def inverse_rope(o, p, rope_dim, base):
    """The output rotated back by its query's position ("How DeepSeek V4
    Handles 1M Token Context", Component 1: keys and values are one shared
    vector, and inverse RoPE restores the positional information).

    Reading (the page gives no formula): the last ``rope_dim`` dims of o,
    which carry the keys' rotary components through V = K, are turned back
    by the query position p, so that the output holds the keys' positions
    relative to the query.  Pairs (2j, 2j + 1) of those dims, the common
    interleaved convention, turn by the angle -p * base^(-2j / rope_dim):
        (x, y) -> (x cos a - y sin a, x sin a + y cos a),  a = -p theta_j.
    ``base`` <= 0 leaves o as it is."""
    o = np.array(o, dtype=np.float64, copy=True)
    if base <= 0 or rope_dim <= 0:
        return o
    j = np.arange(rope_dim // 2, dtype=np.float64)
    a = -float(p) * np.power(float(base), -2.0 * j / rope_dim)
    c, s = np.cos(a), np.sin(a)
    lo = o.shape[-1] - rope_dim
    x = o[..., lo::2].copy()
    y = o[..., lo + 1::2].copy()
    o[..., lo::2] = x * c - y * s
    o[..., lo + 1::2] = x * s + y * c
    return o


def window_positions(p, w):
    """Raw positions in the sliding window of a query at position p."""
    return np.arange(max(0, p - w + 1), p + 1)
