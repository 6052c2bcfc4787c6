"""One decode / chunked-prefill step of a CSA or HCA layer (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

The order of the steps follows "How DeepSeek V4 Handles 1M Token Context",
Component 3 (score every compressed entry -> select the top-k -> gather ->
attend) with the window of the same page and the sink of "DeepSeek V4
Architecture Explained"; HCA skips scoring and selection ("the same idea
with a much larger group per entry and no sparse selection stage").

A step appends T tokens to a sequence whose length becomes L; its queries
sit at positions p = L - T + i.  Before attending, the step

1. pools every group that closes inside the new tokens, i.e. the entries
   g in [floor((L - T) / m), floor(L / m)), and stores them in the caches;
2. stores the T new raw rows in the window ring (row = position mod cap).

Raw rows reach the step as ``x_*`` arrays covering positions
L - (T + G - 1) .. L - 1 (rows at negative positions are never read).

Sink token (``sink_mode="token"``), the other reading of the pages' sink
("DeepSeek V4 Architecture Explained", "How compress-then-sparsify attention
works"): instead of a learned logit, the raw row of position 0 is a member
of every query's row set.  It enters once: when the window already holds
position 0 nothing is added.  The step that receives position 0 stores its
raw row (in the KV format) in a one-row array, which later steps read.
"""
import numpy as np

from . import storage
from .attention import inverse_rope, joint_attention, window_positions
from .compress import compress_entries, n_visible
from .indexer import quantize_query, scores, topk


def _store_rows(cache, rows_idx, values, fmt, rope_dim):
    st = storage.encode(fmt, values, rope_dim)
    cache.payload[rows_idx] = st.payload
    if cache.scale is not None:
        cache.scale[rows_idx] = st.scale


def layer_step(kind, *, m, G, w, k, sm_scale, kv_fmt, rope_dim, idx_fmt, L, T,
               kv, v, idx, ring_kv, ring_v, x_kv, x_v, x_idx,
               W_kv, B_kv, W_v, B_v, W_idx, B_idx,
               q, q_idx, w_idx, sink, queries=None, out_rope_base=0.0,
               U_kv=None, U_v=None, U_idx=None, sink_mode="logit", tok_kv=None, tok_v=None):
    """Run one step for ONE sequence.

    kind: "csa" or "hca".  kv / v / idx / ring_kv / ring_v are
    ``storage.Stored`` arrays (entries, and the window ring), updated in
    place with the new entries and rows; v / ring_v / x_v / W_v / B_v are
    None when V is the shared latent (V = K).  q [T, H, D]; q_idx
    [T, H_I, d_I] and w_idx [T, H_I] (CSA only); sink [H].
    ``queries``: optional subset of query indices i to evaluate.
    ``out_rope_base`` > 0: each output is rotated back by its query's
    position (``inverse_rope`` over the last ``rope_dim`` dims).
    ``U_*``: caller-given gate logits aligned with ``x_*`` (None: x W).
    ``sink_mode``: "logit" (``sink`` holds sigma per head) or "token" (the
    raw row of position 0 joins every row set; ``sink`` is not used);
    ``tok_kv`` / ``tok_v`` are that row's one-row ``Stored`` arrays (updated
    in place by the step that receives position 0).

    Returns dict with o [nq, H, Dv], lse [nq, H], and for CSA sel (list of
    index arrays) and sel_scores (list of score arrays), plus new_entries
    (g range) for reference.
    """
    x_pos0 = L - (T + G - 1)
    g_lo, g_hi = (L - T) // m, L // m
    new_g = range(g_lo, g_hi)
    if len(new_g):
        e_kv = compress_entries(x_kv, x_pos0, W_kv, B_kv, m, G, new_g, U_kv)
        _store_rows(kv, np.arange(g_lo, g_hi), e_kv, kv_fmt, rope_dim)
        if v is not None:
            e_v = compress_entries(x_v, x_pos0, W_v, B_v, m, G, new_g, U_v)
            _store_rows(v, np.arange(g_lo, g_hi), e_v, kv_fmt, rope_dim)
        if kind == "csa":
            e_i = compress_entries(x_idx, x_pos0, W_idx, B_idx, m, G, new_g, U_idx)
            _store_rows(idx, np.arange(g_lo, g_hi), e_i, idx_fmt, 0)
    token = sink_mode == "token"
    if sink_mode not in ("logit", "token"):
        raise ValueError(sink_mode)
    if token:
        sink = np.full(q.shape[1], -np.inf)  # no learned logit in this reading
        if L - T <= 0:  # position 0 is one of the new tokens: keep its raw row
            _store_rows(tok_kv, [0], np.asarray(x_kv)[-x_pos0][None], kv_fmt, rope_dim)
            if tok_v is not None:
                _store_rows(tok_v, [0], np.asarray(x_v)[-x_pos0][None], kv_fmt, rope_dim)

    win_cap = ring_kv.payload.shape[0]
    new_pos = np.arange(L - T, L)
    ring_rows = new_pos % win_cap
    _store_rows(ring_kv, ring_rows, np.asarray(x_kv)[-T:], kv_fmt, rope_dim)
    if ring_v is not None:
        _store_rows(ring_v, ring_rows, np.asarray(x_v)[-T:], kv_fmt, rope_dim)

    if queries is None:
        queries = range(T)
    n_max = n_visible(L - 1, m)
    k_all = storage.decode(idx.rows(slice(0, n_max))) if kind == "csa" else None

    o_all, lse_all, sel_all, sc_all = [], [], [], []
    for i in queries:
        p = L - T + i
        n = n_visible(p, m)
        if kind == "csa":
            qt = quantize_query(q_idx[i], idx_fmt)
            s = scores(qt, w_idx[i], k_all[:n])
            sel = topk(s, k)
            sel_all.append(sel)
            sc_all.append(s[sel])
            ent = sel
        else:
            ent = np.arange(n)
        wpos = window_positions(p, w)
        parts_k = [storage.decode(kv.rows(ent)), storage.decode(ring_kv.rows(wpos % win_cap))]
        parts_v = None if v is None else [storage.decode(v.rows(ent)),
                                          storage.decode(ring_v.rows(wpos % win_cap))]
        if token and not (len(wpos) and wpos[0] == 0):  # position 0 not in the window yet
            parts_k.append(storage.decode(tok_kv.rows([0])))
            if parts_v is not None:
                parts_v.append(storage.decode(tok_v.rows([0])))
        K_rows = np.concatenate(parts_k, axis=0)
        V_rows = K_rows if v is None else np.concatenate(parts_v, axis=0)
        o, lse = joint_attention(q[i], K_rows, V_rows, sink, sm_scale)
        o = inverse_rope(o, p, rope_dim, out_rope_base)
        o_all.append(o)
        lse_all.append(lse)
    out = dict(o=np.stack(o_all), lse=np.stack(lse_all), new_entries=(g_lo, g_hi))
    if kind == "csa":
        out["sel"], out["sel_scores"] = sel_all, sc_all
    return out
