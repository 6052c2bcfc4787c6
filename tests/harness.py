"""Test-side glue: builds oracle states from the seeded synthetic inputs and
compares GPU results with oracle results.  Test infrastructure only."""
import numpy as np

from long_context_sparse_compress_b200 import synth
from oracle import storage
from oracle.step import layer_step


def stored_entries(wl, inp, which):
    """The existing entries of one sequence, stored by the oracle's rules,
    in an array with room for the entries the step adds."""
    n_cap = wl.L // wl.m + 1
    if which == "idx":
        fmt, d, rope = wl.idx_fmt, wl.d_I, 0
    else:
        fmt, d, rope = wl.kv_fmt, (wl.D if which == "kv" else wl.Dv), wl.rope_dim
    vals = inp["e_" + which]
    st = storage.encode(fmt, vals, rope)
    pay = np.zeros((n_cap,) + st.payload.shape[1:], dtype=st.payload.dtype)
    pay[: vals.shape[0]] = st.payload
    sc = None
    if st.scale is not None:
        sc = np.zeros((n_cap,) + st.scale.shape[1:], dtype=st.scale.dtype)
        sc[: vals.shape[0]] = st.scale
    return storage.Stored(fmt, pay, sc, d, rope if fmt == "kv" else 0)


def stored_ring(wl, x_tail, dim):
    """The window ring before the step: raw rows of positions L-T-w+1..L-T-1."""
    cap = wl.win_cap
    R = x_tail.shape[0]
    pos0 = wl.L - R
    rope = wl.rope_dim if wl.kv_fmt == "kv" else 0
    st = storage.encode(wl.kv_fmt, np.zeros((cap, dim), np.float32), rope)
    for pos in range(max(0, wl.L - wl.T - wl.w + 1), wl.L - wl.T):
        one = storage.encode(wl.kv_fmt, x_tail[pos - pos0][None], rope)
        st.payload[pos % cap] = one.payload[0]
        if st.scale is not None:
            st.scale[pos % cap] = one.scale[0]
    return st


def step_tail(wl, x_tail):
    """The raw rows the step itself reads: positions L-(T+G-1)..L-1."""
    return x_tail[x_tail.shape[0] - (wl.T + wl.G - 1):]


class OracleSequence:
    """Oracle state and inputs of one sequence of a single-layer workload."""

    def __init__(self, wl, b, P=None, seed=synth.SEED):
        self.wl, self.b = wl, b
        self.P = P if P is not None else synth.layer_params(wl, seed)
        self.inp = synth.sequence_inputs(wl, b, seed)
        self.kv = stored_entries(wl, self.inp, "kv")
        self.v = stored_entries(wl, self.inp, "v") if wl.separate_v else None
        self.idx = stored_entries(wl, self.inp, "idx") if wl.kind == "csa" else None
        self.ring_kv = stored_ring(wl, self.inp["x_kv"], wl.D)
        self.ring_v = stored_ring(wl, self.inp["x_v"], wl.Dv) if wl.separate_v else None
        # sink token: the stored row of position 0, present once a step before this one received it
        self.tok_kv = self._tok_row("kv", wl.D) if wl.sink_mode == "token" else None
        self.tok_v = self._tok_row("v", wl.Dv) if wl.sink_mode == "token" and wl.separate_v else None

    def _tok_row(self, key, dim):
        rope = self.wl.rope_dim if self.wl.kv_fmt == "kv" else 0
        row = self.inp["x0_" + key] if self.wl.L - self.wl.T > 0 else np.zeros(dim, np.float32)
        return storage.encode(self.wl.kv_fmt, np.asarray(row, np.float32)[None], rope)

    def snapshot(self):
        """Copies of the stored arrays (the GPU side gets these bytes)."""
        def cp(st):
            if st is None:
                return None
            return storage.Stored(st.fmt, st.payload.copy(), None if st.scale is None else st.scale.copy(),
                                  st.dim, st.rope_dim)
        return {k: cp(getattr(self, k)) for k in ("kv", "v", "idx", "ring_kv", "ring_v", "tok_kv", "tok_v")}

    def step(self, queries=None):
        wl, P, inp = self.wl, self.P, self.inp
        t = lambda key: None if key not in inp else step_tail(wl, inp[key])
        return layer_step(
            wl.kind, m=wl.m, G=wl.G, w=wl.w, k=wl.k, sm_scale=wl.sm_scale, kv_fmt=wl.kv_fmt,
            rope_dim=wl.rope_dim, idx_fmt=wl.idx_fmt, L=wl.L, T=wl.T, kv=self.kv, v=self.v,
            idx=self.idx, ring_kv=self.ring_kv, ring_v=self.ring_v, x_kv=t("x_kv"), x_v=t("x_v"),
            x_idx=t("x_idx"), W_kv=P["W_kv"], B_kv=P["B_kv"], W_v=P.get("W_v"), B_v=P.get("B_v"),
            W_idx=P.get("W_idx"), B_idx=P.get("B_idx"), q=inp["q"], q_idx=inp.get("q_idx"),
            w_idx=inp.get("w_idx"), sink=P["sink"] if wl.sink else np.full(wl.H, -np.inf), queries=queries,
            out_rope_base=wl.out_rope_base,
            U_kv=t("U_kv"), U_v=t("U_v"), U_idx=t("U_idx"), sink_mode=wl.sink_mode, tok_kv=self.tok_kv,
            tok_v=self.tok_v)


# ---------------------------------------------------------------- comparisons

def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def max_abs(got, want):
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64)))) if np.size(want) else 0.0


def topk_set_ok(gpu_idx, scores_all, k, band=1e-3):
    """Top-k parity: the GPU's set equals the oracle's exact top-k set, except
    entries whose oracle score is within ``band`` (relative) of the k-th
    oracle score.  ``scores_all`` are the oracle scores of every visible
    entry.  Returns (ok, message)."""
    gpu = np.asarray(gpu_idx)
    gpu = gpu[gpu >= 0]
    n = scores_all.shape[0]
    k_eff = min(k, n)
    if gpu.shape[0] != k_eff:
        return False, f"{gpu.shape[0]} indices, want {k_eff}"
    if len(set(gpu.tolist())) != gpu.shape[0]:
        return False, "duplicate indices"
    if np.any(gpu >= n):
        return False, "index beyond the visible entries"
    if k_eff == 0:
        return True, ""
    kth = np.sort(scores_all)[::-1][k_eff - 1]
    tol = band * abs(kth)
    sure_in = np.nonzero(scores_all > kth + tol)[0]
    sure_out = scores_all < kth - tol
    gset = set(gpu.tolist())
    missing = [i for i in sure_in if i not in gset]
    extra = [i for i in gpu if sure_out[i]]
    if missing or extra:
        return False, f"missing {missing[:5]} extra {extra[:5]}"
    return True, ""
