"""Seeded synthetic inputs for one layer step (no arithmetic of the method).

Every array is drawn from its own numpy PCG64 stream keyed by
(seed, layer, tensor, sequence), so any one sequence can be regenerated
alone.  Values follow the benchmark recipe:

* raw token rows, queries, indexer queries, and pre-storage compressed entries
  ~ N(0, 1/d) (standard deviation 1/sqrt(d), d the row length);
* gate projections W ~ N(0, 0.02^2); positional biases ~ N(0, 1);
* sink logits ~ N(0, 1); indexer head weights |N(0, 1)| / sqrt(H_I);
* ``n_planted`` entries per sequence, at uniform distinct indices whose
  tokens lie before the window, are replaced by unit vectors along the
  queries' common direction (plus N(0, 0.01/d) noise): the KV latent along
  the mean query head, the indexer key along sum_h w[h] q_idx[h] (averaged
  over the step's queries).  This makes the top-k non-degenerate.

Layers with caller-given gate logits get per-token logit rows U ~ N(0, 1)
aligned with the raw rows.  Layers whose sink is the position-0 token get
that token's raw row as a sink would look: gamma times the unit mean query
head (plus N(0, 0.01/d) noise), gamma = sqrt(D H) / 8: its logit sits
about 0.125 above the others' and, with values of about sqrt(H) / 8 each,
it is the row that dominates short contexts while the outputs stay within
a few units (a query at position 0 returns the row itself); when the tail
reaches position 0, that tail row is the same row.

Rows that the layer stores as bf16 (raw rows, gate weights, queries) are
rounded to bf16 here with torch's own cast; everything else is float32.
The existing cache is described by its *pre-storage* float32 entry values;
storing them (FP8/FP4/BF16) is the job of whoever consumes them.
"""
import numpy as np
import torch

SEED = 20261202

_LAYER = {"csa": 0, "hca": 1}
_TENSOR = {name: i + 1 for i, name in enumerate(
    ["x_kv", "x_v", "x_idx", "W_kv", "B_kv", "W_v", "B_v", "W_idx", "B_idx", "q", "q_idx",
     "w_idx", "sink", "e_kv", "e_v", "e_idx", "planted", "x0_kv", "x0_v", "U_kv", "U_v", "U_idx"])}


def stream(seed, layer, tensor, b=0):
    key = [int(seed), _LAYER[layer], _TENSOR[tensor], int(b)]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def normal(rng, shape, std):
    out = np.empty(shape, dtype=np.float32)
    rng.standard_normal(dtype=np.float32, out=out)
    out *= np.float32(std)
    return out


def as_dtype(dtype, a):
    """Round float32 values to the storage dtype of an input ("bf16" or "f32")."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float32).numpy()
    return np.asarray(a, dtype=np.float32)


def tail_rows(wl):
    """Raw rows a step needs: the window rows before it plus the new tokens and
    the history of the groups they close: positions L - R .. L - 1."""
    return wl.T + max(wl.w, wl.G) - 1


def layer_params(wl, seed=SEED):
    """Per-layer inputs shared by every sequence: gates, biases, sink."""
    lay = wl.kind
    P = {
        "W_kv": as_dtype(wl.x_dtype, normal(stream(seed, lay, "W_kv"), (wl.D, wl.D), 0.02)),
        "B_kv": normal(stream(seed, lay, "B_kv"), (wl.G, wl.D), 1.0),
        "sink": normal(stream(seed, lay, "sink"), (wl.H,), 1.0),
    }
    if wl.separate_v:
        P["W_v"] = as_dtype(wl.x_dtype, normal(stream(seed, lay, "W_v"), (wl.Dv, wl.Dv), 0.02))
        P["B_v"] = normal(stream(seed, lay, "B_v"), (wl.G, wl.Dv), 1.0)
    if wl.kind == "csa":
        P["W_idx"] = as_dtype(wl.x_dtype, normal(stream(seed, lay, "W_idx"), (wl.d_I, wl.d_I), 0.02))
        P["B_idx"] = normal(stream(seed, lay, "B_idx"), (wl.G, wl.d_I), 1.0)
    return P


def _unit(v):
    n = float(np.linalg.norm(v))
    return (v / n) if n > 0 else v


def sequence_inputs(wl, b, seed=SEED, entries=True):
    """Inputs of sequence b for one step of a single layer ``wl``.

    Returns float32 arrays:
      x_kv [R, D], x_v [R, Dv], x_idx [R, d_I]: raw rows of positions L-R..L-1;
      q [T, H, D]; q_idx [T, H_I, d_I]; w_idx [T, H_I];
      e_kv [n_old, D], e_v [n_old, Dv], e_idx [n_old, d_I]: the pre-storage
      values of the n_old = (L - T) // m entries that exist before the step
      (only when ``entries``); planted: their planted indices.
    """
    lay = wl.kind
    R = tail_rows(wl)
    out = {
        "x_kv": as_dtype(wl.x_dtype, normal(stream(seed, lay, "x_kv", b), (R, wl.D), wl.D ** -0.5)),
        "q": as_dtype(wl.q_dtype, normal(stream(seed, lay, "q", b), (wl.T, wl.H, wl.D), wl.D ** -0.5)),
    }
    if wl.separate_v:
        out["x_v"] = as_dtype(wl.x_dtype, normal(stream(seed, lay, "x_v", b), (R, wl.Dv), wl.Dv ** -0.5))
    if wl.kind == "csa":
        out["x_idx"] = as_dtype(wl.x_dtype,
                                normal(stream(seed, lay, "x_idx", b), (R, wl.d_I), wl.d_I ** -0.5))
        out["q_idx"] = as_dtype(wl.q_dtype, normal(stream(seed, lay, "q_idx", b),
                                                   (wl.T, wl.H_I, wl.d_I), wl.d_I ** -0.5))
        w = np.abs(normal(stream(seed, lay, "w_idx", b), (wl.T, wl.H_I), 1.0)) * np.float32(wl.H_I ** -0.5)
        out["w_idx"] = w.astype(np.float32)
    if wl.gate_src == "logits":
        out["U_kv"] = normal(stream(seed, lay, "U_kv", b), (R, wl.D), 1.0)
        if wl.separate_v:
            out["U_v"] = normal(stream(seed, lay, "U_v", b), (R, wl.Dv), 1.0)
        if wl.kind == "csa":
            out["U_idx"] = normal(stream(seed, lay, "U_idx", b), (R, wl.d_I), 1.0)
    if wl.sink_mode == "token":
        u_q = _unit(out["q"].astype(np.float64).mean(axis=(0, 1)))
        gamma = 0.125 * np.sqrt(wl.D * wl.H)
        x0 = gamma * u_q + normal(stream(seed, lay, "x0_kv", b), (wl.D,), 0.1 * wl.D ** -0.5)
        out["x0_kv"] = as_dtype(wl.x_dtype, x0.astype(np.float32))
        if wl.separate_v:
            out["x0_v"] = as_dtype(wl.x_dtype, normal(stream(seed, lay, "x0_v", b), (wl.Dv,), wl.Dv ** -0.5))
        if wl.L - R <= 0:  # the tail reaches position 0: it holds the same row
            out["x_kv"][R - wl.L] = out["x0_kv"]
            if wl.separate_v:
                out["x_v"][R - wl.L] = out["x0_v"]
    if not entries:
        return out
    n_old = (wl.L - wl.T) // wl.m
    out["e_kv"] = normal(stream(seed, lay, "e_kv", b), (n_old, wl.D), wl.D ** -0.5)
    if wl.separate_v:
        out["e_v"] = normal(stream(seed, lay, "e_v", b), (n_old, wl.Dv), wl.Dv ** -0.5)
    if wl.kind == "csa":
        out["e_idx"] = normal(stream(seed, lay, "e_idx", b), (n_old, wl.d_I), wl.d_I ** -0.5)
    n_pl = min(wl.n_planted, n_old)
    planted = np.zeros(0, dtype=np.int64)
    if n_pl > 0:
        rng = stream(seed, lay, "planted", b)
        n_lim = max(n_pl, (wl.L - wl.T - wl.w) // wl.m)
        planted = np.sort(rng.choice(min(n_lim, n_old), size=n_pl, replace=False))
        u_kv = _unit(out["q"].astype(np.float64).mean(axis=(0, 1)))
        out["e_kv"][planted] = (u_kv[None, :] + normal(rng, (n_pl, wl.D), 0.1 * wl.D ** -0.5)).astype(np.float32)
        if wl.kind == "csa":
            v = (out["w_idx"].astype(np.float64)[..., None] * out["q_idx"].astype(np.float64)).sum(axis=1)
            u_idx = _unit(v.mean(axis=0))
            out["e_idx"][planted] = (u_idx[None, :] +
                                     normal(rng, (n_pl, wl.d_I), 0.1 * wl.d_I ** -0.5)).astype(np.float32)
    out["planted"] = planted
    return out
