"""Softmax-gated pooling of token groups into compressed entries (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Source: "DeepSeek V4 Architecture Explained", "How compress-then-sparsify
attention works": each group of m consecutive tokens' keys and values is
folded into one entry with trainable compression weights, a softmax over the
group and learnable positional biases; "Inside DeepSeek-V4", section 1
(softmax-gated pooling with learned positional biases, m = 4) and section 2
(m = 128 for HCA); "How DeepSeek V4 Handles 1M Token Context", Component 2
(8-token groups at stride 4 as an overlapping variant).

Reading (the pages give the ingredients, not the formula): entry g pools the
tokens j in [g*m + m - G, g*m + m) (G = m, or 2m for the overlapping
variant; positions < 0 do not exist and are left out).  For every channel c
separately the gate logit of token j is

    z_j[c] = sum_d x_j[d] * W[d, c]  +  Bpos[j - (g*m + m - G), c]

the weights are alpha_j[c] = softmax over the group's tokens of z_j[c], and
the entry is  e_g[c] = sum_j alpha_j[c] * x_j[c].  Each compressed tensor
(the shared KV latent, a separate V, the indexer keys) has its own W, Bpos.

Caller-given gate logits (a second reading, since the pages do not say
what the trainable compression weights act on): a per-token logit row u_j
takes the place of x_j W, and the positional bias of the token's place in
the group is still added, z_j[c] = u_j[c] + Bpos[j - (g*m + m - G), c].  A
token shared by two overlapping groups keeps its u_j and gets the bias of
its place in each group.
"""
import numpy as np


def group_span(g, m, G):
    """First (possibly negative) and one-past-last token position of entry g."""
    return g * m + m - G, g * m + m


def pool_group(x_tok, W, bpos_rows, u_tok=None):
    """One entry from its tokens.

    x_tok: [J, D] token rows (float64) of the group, oldest first.
    W: [D, D] gate projection (input channel d, output channel c).
    bpos_rows: [J, D] the positional-bias rows of those tokens.
    u_tok: optional [J, D] caller-given gate logits of those tokens, used in
    place of x_tok @ W (W is then not read).
    Returns the pooled row [D] and the gate weights alpha [J, D].
    """
    x_tok = np.asarray(x_tok, dtype=np.float64)
    gate = (x_tok @ np.asarray(W, dtype=np.float64)) if u_tok is None else np.asarray(u_tok, dtype=np.float64)
    z = gate + np.asarray(bpos_rows, dtype=np.float64)
    z = z - z.max(axis=0, keepdims=True)
    a = np.exp(z)
    alpha = a / a.sum(axis=0, keepdims=True)
    return (alpha * x_tok).sum(axis=0), alpha


def compress_entries(x, x_pos0, W, Bpos, m, G, entries, U=None):
    """Pool entries ``entries`` (iterable of g) from raw rows.

    x: [n, D] raw token rows for positions x_pos0 .. x_pos0 + n - 1; every
    non-negative position an entry needs must be present.
    U: optional [n, D] caller-given gate logits of the same positions (in
    place of x W).
    Returns float64 [len(entries), D].
    """
    x = np.asarray(x, dtype=np.float64)
    out = []
    for g in entries:
        start, stop = group_span(g, m, G)
        first = max(start, 0)
        if first - x_pos0 < 0 or stop - x_pos0 > x.shape[0]:
            raise ValueError(f"entry {g} needs positions [{first}, {stop}) not all in x")
        rows = x[first - x_pos0: stop - x_pos0]
        brows = np.asarray(Bpos)[first - start: stop - start]
        urows = None if U is None else np.asarray(U)[first - x_pos0: stop - x_pos0]
        e, _ = pool_group(rows, W, brows, urows)
        out.append(e)
    return np.stack(out) if out else np.zeros((0, x.shape[1]))


def compress_entries_batched(x, W, Bpos, m, G):
    """All ``n // m`` entries of x (positions 0..n-1), vectorised over entries.

    Same arithmetic as ``compress_entries`` (it is checked against it), in a
    form fast enough for a few thousand entries.
    """
    x = np.asarray(x, dtype=np.float64)
    n, D = x.shape
    n_e = n // m
    pad = G - m
    xp = np.concatenate([np.zeros((pad, D)), x[: n_e * m]], axis=0)
    idx = np.arange(n_e)[:, None] * m + np.arange(G)[None, :]  # rows in xp
    xg = xp[idx]                                              # [n_e, G, D]
    valid = (idx - pad) >= 0                                   # real positions
    z = xg @ np.asarray(W, dtype=np.float64) + np.asarray(Bpos, dtype=np.float64)[None]
    z = np.where(valid[..., None], z, -np.inf)
    z = z - z.max(axis=1, keepdims=True)
    a = np.exp(z)
    alpha = a / a.sum(axis=1, keepdims=True)
    return (alpha * xg).sum(axis=1)


def n_visible(p, m):
    """Entries visible to a query at position p: entry g exists once its last
    token g*m + m - 1 has arrived, so N(p) = floor((p + 1) / m)."""
    return (p + 1) // m
