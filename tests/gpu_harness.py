"""GPU-side test glue: uploads oracle-built states to device caches and runs
the library's calls.  Test infrastructure only."""
import numpy as np
import torch

from long_context_sparse_compress_b200 import lib as L
from tests.harness import OracleSequence, step_tail

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).cuda()


def upload(cache, b, st):
    """Copy oracle ``Stored`` rows into sequence b of a DeviceCache."""
    cache.set_rows(b, np.ascontiguousarray(st.payload),
                   None if st.scale is None else np.ascontiguousarray(st.scale))


def download(cache, b):
    return cache.get_rows(b)


class GpuBatch:
    """Device buffers of one step of a single-layer workload over B
    sequences (per-sequence workloads may differ in L only)."""

    def __init__(self, seqs):
        self.seqs = seqs
        wl = seqs[0].wl
        self.wl = wl
        B = len(seqs)
        self.B = B
        self.n_cap = max(s.wl.L for s in seqs) // wl.m + 1
        n_cap_idx = L.round_capacity(self.n_cap, wl.idx_fmt)
        self.n_max = max(s.wl.L for s in seqs) // wl.m
        rope = wl.rope_dim if wl.kv_fmt == "kv" else 0
        self.kv = L.DeviceCache(B, self.n_cap, wl.kv_fmt, wl.D, rope)
        self.v = L.DeviceCache(B, self.n_cap, wl.kv_fmt, wl.Dv, rope) if wl.separate_v else None
        self.idx = L.DeviceCache(B, n_cap_idx, wl.idx_fmt, wl.d_I) if wl.kind == "csa" else None
        self.win_kv = L.DeviceCache(B, wl.win_cap, wl.kv_fmt, wl.D, rope)
        self.win_v = L.DeviceCache(B, wl.win_cap, wl.kv_fmt, wl.Dv, rope) if wl.separate_v else None
        tok = wl.sink_mode == "token"
        self.tok_kv = L.DeviceCache(B, 1, wl.kv_fmt, wl.D, rope) if tok else None
        self.tok_v = L.DeviceCache(B, 1, wl.kv_fmt, wl.Dv, rope) if tok and wl.separate_v else None
        xdt, qdt = TORCH_DT[wl.x_dtype], TORCH_DT[wl.q_dtype]
        for b, s in enumerate(seqs):
            snap = s.snapshot()
            upload(self.kv, b, snap["kv"])
            if self.v is not None:
                upload(self.v, b, snap["v"])
            if self.idx is not None:
                upload(self.idx, b, snap["idx"])
            upload(self.win_kv, b, snap["ring_kv"])
            if self.win_v is not None:
                upload(self.win_v, b, snap["ring_v"])
            if self.tok_kv is not None:
                upload(self.tok_kv, b, snap["tok_kv"])
            if self.tok_v is not None:
                upload(self.tok_v, b, snap["tok_v"])
        stack = lambda key, dt: dev(np.stack([s.inp[key] for s in seqs]), dt)
        stack_tail = lambda key: dev(np.stack([step_tail(s.wl, s.inp[key]) for s in seqs]), xdt)
        self.x_kv = stack_tail("x_kv")
        self.x_v = stack_tail("x_v") if wl.separate_v else None
        self.x_idx = stack_tail("x_idx") if wl.kind == "csa" else None
        P = seqs[0].P
        # gates: W, or with caller-given logits the float32 logit rows of the step's positions
        logits = wl.gate_src == "logits"
        gate = lambda key, Wkey: (dev(np.stack([step_tail(s.wl, s.inp[key]) for s in seqs]))
                                  if logits else dev(P[Wkey], xdt))
        self.w_kv, self.b_kv = gate("U_kv", "W_kv"), dev(P["B_kv"])
        self.w_v = gate("U_v", "W_v") if wl.separate_v else None
        self.b_v = dev(P["B_v"]) if wl.separate_v else None
        self.w_idx = gate("U_idx", "W_idx") if wl.kind == "csa" else None
        self.b_idx = dev(P["B_idx"]) if wl.kind == "csa" else None
        self.sink = dev(P["sink"]) if wl.sink and not tok else None
        self.q = stack("q", qdt)
        self.q_idx = stack("q_idx", qdt) if wl.kind == "csa" else None
        self.w_heads = stack("w_idx", torch.float32) if wl.kind == "csa" else None
        self.ctx_len = torch.tensor([s.wl.L for s in seqs], dtype=torch.int32, device="cuda")
        self.out = torch.zeros((B, wl.T, wl.H, wl.Dv), dtype=qdt, device="cuda")
        self.lse = torch.zeros((B, wl.T, wl.H), dtype=torch.float32, device="cuda")
        self.out_idx = (torch.full((B, wl.T, wl.k), -7, dtype=torch.int32, device="cuda")
                        if wl.kind == "csa" else None)
        self.out_score = (torch.zeros((B, wl.T, wl.k), dtype=torch.float32, device="cuda")
                          if wl.kind == "csa" else None)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.p = L.params(wl)

    def step_struct(self):
        return L.make_step(self.B, self.wl.T, self.n_max, self.ctx_len, self.x_kv, self.x_v, self.x_idx,
                           self.w_kv, self.b_kv, self.w_v, self.b_v, self.w_idx, self.b_idx, self.kv,
                           self.v, self.idx, self.win_kv, self.win_v, self.q, self.q_idx, self.w_heads,
                           self.sink, self.out, self.lse, self.out_idx, self.out_score, self.tok_kv,
                           self.tok_v)

    def run_step(self):
        csa = self.wl.kind == "csa"
        ws = L.workspace(L.step_workspace(self.p, csa, self.B, self.wl.T, self.n_max))
        L.decode_step(self.p, self.step_struct(), csa, ws, self.status)
        torch.cuda.synchronize()
        return ws


def make_seqs(wl, lengths=None, seed=None):
    """OracleSequence per batch element; ``lengths`` gives per-sequence L."""
    from long_context_sparse_compress_b200 import synth
    seed = synth.SEED if seed is None else seed
    lengths = lengths or [wl.L] * wl.B
    P = synth.layer_params(wl, seed)
    return [OracleSequence(wl.with_(L=Lb), b, P=P, seed=seed) for b, Lb in enumerate(lengths)]
