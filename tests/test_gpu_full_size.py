"""Parity at the benchmark workloads' full sizes, in the launch configuration
the benchmark times (the fused step over the whole batch), on sampled
outputs.

Every sequence of the batch gets its seeded raw rows and queries; the
sampled sequences also get their full seeded caches, stored by the
oracle's rules (built on the CPU, then uploaded), and their outputs are
compared with the oracle's step.  The other sequences' caches are filled on
the device with seeded random entries stored by the library: they only
make the launch the full-size one, and their outputs are not compared.
Long prefill steps compare a sample of their query rows.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_compress_b200 import lib as L
from long_context_sparse_compress_b200 import synth
from long_context_sparse_compress_b200 import workloads as W
from oracle import storage
from oracle.indexer import quantize_query, scores as oracle_scores
from tests.gpu_harness import TORCH_DT, dev, download, upload
from tests.harness import OracleSequence, max_abs, rel_l2, step_tail, topk_set_ok

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


class SampledBatch:
    """The device buffers of one full-size step; sequences in ``sampled``
    carry oracle-built caches."""

    def __init__(self, wl, sampled, seed=synth.SEED):
        self.wl, self.B = wl, wl.B
        P = synth.layer_params(wl, seed)
        self.seqs = {b: OracleSequence(wl, b, P=P, seed=seed) for b in sampled}
        for s in self.seqs.values():  # the pre-storage values are no longer needed
            for key in ("e_kv", "e_v", "e_idx"):
                s.inp.pop(key, None)
        inputs = [self.seqs[b].inp if b in self.seqs else synth.sequence_inputs(wl, b, seed, entries=False)
                  for b in range(wl.B)]
        self.n_max = wl.L // wl.m
        n_cap = self.n_max + 1
        rope = wl.rope_dim if wl.kv_fmt == "kv" else 0
        csa = wl.kind == "csa"
        self.p = L.params(wl)
        self.kv = L.DeviceCache(wl.B, n_cap, wl.kv_fmt, wl.D, rope)
        self.idx = L.DeviceCache(wl.B, L.round_capacity(n_cap, wl.idx_fmt), wl.idx_fmt, wl.d_I) if csa else None
        self.win = L.DeviceCache(wl.B, wl.win_cap, wl.kv_fmt, wl.D, rope)
        sep = wl.separate_v
        self.v = L.DeviceCache(wl.B, n_cap, wl.kv_fmt, wl.Dv, rope) if sep else None
        self.win_v = L.DeviceCache(wl.B, wl.win_cap, wl.kv_fmt, wl.Dv, rope) if sep else None
        n_old = (wl.L - wl.T) // wl.m
        g = torch.Generator(device="cuda")
        for b in range(wl.B):
            if b in self.seqs:
                snap = self.seqs[b].snapshot()
                upload(self.kv, b, snap["kv"])
                if csa:
                    upload(self.idx, b, snap["idx"])
                upload(self.win, b, snap["ring_kv"])
                if sep:
                    upload(self.v, b, snap["v"])
                    upload(self.win_v, b, snap["ring_v"])
                continue
            g.manual_seed(seed + 7919 * (b + 1))
            for c0 in range(0, n_old, 65536):  # device-random entries, in chunks
                c1 = min(n_old, c0 + 65536)
                vals = torch.randn((1, c1 - c0, wl.D), generator=g, device="cuda") * wl.D ** -0.5
                L.encode_rows(self.p, "kv", vals, c0, self.kv.seq(b))
                if sep:
                    vals = torch.randn((1, c1 - c0, wl.Dv), generator=g, device="cuda") * wl.Dv ** -0.5
                    L.encode_rows(self.p, "v", vals, c0, self.v.seq(b))
                if csa:
                    vals = torch.randn((1, c1 - c0, wl.d_I), generator=g, device="cuda") * wl.d_I ** -0.5
                    L.encode_rows(self.p, "idx", vals, c0, self.idx.seq(b))
            vals = torch.randn((1, wl.win_cap, wl.D), generator=g, device="cuda") * wl.D ** -0.5
            L.encode_rows(self.p, "kv", vals, 0, self.win.seq(b))
            if sep:
                vals = torch.randn((1, wl.win_cap, wl.Dv), generator=g, device="cuda") * wl.Dv ** -0.5
                L.encode_rows(self.p, "v", vals, 0, self.win_v.seq(b))
        xdt, qdt = TORCH_DT[wl.x_dtype], TORCH_DT[wl.q_dtype]
        stack = lambda key, dt: dev(np.stack([inputs[b][key] for b in range(wl.B)]), dt)
        self.x_kv = dev(np.stack([step_tail(wl, inputs[b]["x_kv"]) for b in range(wl.B)]), xdt)
        self.x_idx = dev(np.stack([step_tail(wl, inputs[b]["x_idx"]) for b in range(wl.B)]), xdt) if csa else None
        self.x_v = dev(np.stack([step_tail(wl, inputs[b]["x_v"]) for b in range(wl.B)]), xdt) if sep else None
        self.w_kv, self.b_kv = dev(P["W_kv"], xdt), dev(P["B_kv"])
        self.w_v = dev(P["W_v"], xdt) if sep else None
        self.b_v = dev(P["B_v"]) if sep else None
        self.w_idx = dev(P["W_idx"], xdt) if csa else None
        self.b_idx = dev(P["B_idx"]) if csa else None
        self.sink = dev(P["sink"]) if wl.sink else None
        self.q = stack("q", qdt)
        self.q_idx = stack("q_idx", qdt) if csa else None
        self.w_heads = stack("w_idx", torch.float32) if csa else None
        self.ctx_len = torch.full((wl.B,), wl.L, dtype=torch.int32, device="cuda")
        self.out = torch.zeros((wl.B, wl.T, wl.H, wl.Dv), dtype=qdt, device="cuda")
        self.lse = torch.zeros((wl.B, wl.T, wl.H), dtype=torch.float32, device="cuda")
        self.out_idx = torch.full((wl.B, wl.T, wl.k), -7, dtype=torch.int32, device="cuda") if csa else None
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self):
        csa = self.wl.kind == "csa"
        st = L.make_step(self.B, self.wl.T, self.n_max, self.ctx_len, self.x_kv, self.x_v, self.x_idx, self.w_kv,
                         self.b_kv, self.w_v, self.b_v, self.w_idx, self.b_idx, self.kv, self.v, self.idx, self.win,
                         self.win_v, self.q, self.q_idx, self.w_heads, self.sink, self.out, self.lse, self.out_idx,
                         None)
        ws = L.workspace(L.step_workspace(self.p, csa, self.B, self.wl.T, self.n_max))
        L.decode_step(self.p, st, csa, ws, self.status)
        torch.cuda.synchronize()


def check(wl, sampled, query_sample=None):
    sb = SampledBatch(wl, sampled)
    sb.run()
    assert sb.status.item() == 0
    o_gpu = sb.out.float().cpu().numpy()
    lse_gpu = sb.lse.cpu().numpy()
    sel_gpu = sb.out_idx.cpu().numpy() if sb.out_idx is not None else None
    qs = query_sample if query_sample is not None else list(range(wl.T))
    for b, s in sb.seqs.items():
        ref = s.step(queries=qs)
        g_lo, g_hi = ref["new_entries"]
        if g_hi > g_lo:  # the new entries, stored like the oracle stores them
            d, sc = download(sb.kv, b)
            got = storage.decode(storage.Stored(s.kv.fmt, d[g_lo:g_hi], None if sc is None else sc[g_lo:g_hi],
                                                s.kv.dim, s.kv.rope_dim))
            want = storage.decode(s.kv.rows(slice(g_lo, g_hi)))
            assert rel_l2(got, want) <= (1e-5 if s.kv.fmt == "f32" else 1e-2), (wl.name, b)
        wd, _ = download(sb.win, b)
        for pos in range(wl.L - wl.T, wl.L):
            assert np.array_equal(wd[pos % wl.win_cap], s.ring_kv.payload[pos % wl.win_cap]), (wl.name, b, pos)
        for j, i in enumerate(qs):
            o = ref["o"][j]
            assert rel_l2(o_gpu[b, i], o) <= 1e-2, (wl.name, b, i, rel_l2(o_gpu[b, i], o))
            assert max_abs(o_gpu[b, i], o) <= 2e-2, (wl.name, b, i)
            assert np.allclose(lse_gpu[b, i], ref["lse"][j], rtol=1e-3, atol=1e-3)
            if sel_gpu is not None:
                n = (wl.L - wl.T + i + 1) // wl.m
                k_all = storage.decode(s.idx.rows(slice(0, n)))
                sc_all = oracle_scores(quantize_query(s.inp["q_idx"][i], wl.idx_fmt), s.inp["w_idx"][i], k_all)
                ok, msg = topk_set_ok(sel_gpu[b, i], sc_all, wl.k)
                assert ok, (wl.name, b, i, msg)
                # planted entries point along the queries' mean direction, which
                # singles them out for a lone decode query but not for one of
                # several with directions of their own
                if len(s.inp["planted"]) and wl.T == 1:
                    assert set(s.inp["planted"].tolist()) <= set(sel_gpu[b, i].tolist())


# (workload at its full size, sampled sequences, sampled query rows)
CASES = {
    "csa_decode_4k_fp32": (W.CSA_DECODE_4K_F32, [0], None),
    "hca_decode_64k": (W.HCA_DECODE_64K, [0, 3], None),
    "csa_decode_128k": (W.CSA_DECODE_128K, [0, 7], None),
    "csa_prefill_256k": (W.CSA_PREFILL_256K, [0], [0, 1, 2047, 4094, 4095]),
    "pair_1m_b16.csa": (W.PAIR_DECODE_1M_B16.layer("csa"), [15], None),
    "pair_1m_b16.hca": (W.PAIR_DECODE_1M_B16.layer("hca"), [0, 15], None),
    "pair_1m_b1.csa": (W.PAIR_DECODE_1M_B1.layer("csa"), [0], None),
    "pair_1m_b1.hca": (W.PAIR_DECODE_1M_B1.layer("hca"), [0], None),
    # five draft tokens per sequence, outputs rotated back by their positions
    # (angles up to 1e6 radians)
    "pair_1m_b16_t5.csa": (W.PAIR_DECODE_1M_B16_T5.layer("csa"), [15], None),
    "pair_1m_b16_t5.hca": (W.PAIR_DECODE_1M_B16_T5.layer("hca"), [0], None),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_full_size_step_matches_oracle(cuda_lib, name):
    wl, sampled, qs = CASES[name]
    check(wl, sampled, qs)
