"""The entry-sharded decode step (long_context_sparse_compress_b200.sharded)
across two and three gloo ranks on the CPU: its phases, who pools which
entry, who holds the window, and its two all-gathers, with each phase's
compute done by the oracle on the rank's own entry range.  Every rank must
end with the single-device oracle step's selection and output.  (The
kernels behind the phases are checked against the oracle on the GPU by
tests/test_gpu_sharded.py.)"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import storage
from oracle.attention import inverse_rope, joint_attention, window_positions
from oracle.compress import compress_entries
from oracle.indexer import quantize_query, scores as oracle_scores, topk as oracle_topk


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class HostCache:
    """Stored rows of B sequences on the host (an entry shard when rows > 0)."""

    def __init__(self, stored_per_seq, row0=0, rows=0):
        self.st, self.row0, self.rows = stored_per_seq, row0, rows
        self.capacity = stored_per_seq[0].payload.shape[0]

    def put(self, b, r, one):
        self.st[b].payload[r] = one.payload[0]
        if one.scale is not None:
            self.st[b].scale[r] = one.scale[0]


class OracleOps:
    """Each phase's compute by the oracle, over HostCache shards."""

    @staticmethod
    def compress(p, tensor, x, B, tok_begin, tok_end, w, bpos, entries, window=None, status=None):
        m, G = p.m, p.group_len
        x = x.numpy().astype(np.float64)
        x0 = tok_begin - (G - m)
        for b in range(B):
            st = entries.st[b]
            for g in range(tok_begin // m, tok_end // m):
                r = g - entries.row0 if entries.rows else g
                if entries.rows and not 0 <= r < entries.rows:
                    continue
                e = compress_entries(x[b], x0, w.numpy(), bpos.numpy(), m, G, [g])
                entries.put(b, r, storage.encode(st.fmt, e, st.rope_dim))
            if window is not None:
                for pos in range(max(tok_begin, tok_end - window.capacity), tok_end):
                    window.put(b, pos % window.capacity, storage.encode(st.fmt, x[b][pos - x0][None], st.rope_dim))

    @staticmethod
    def index_topk(p, q_idx, w_idx, keys, ctx_len, n_max, out_idx, out_score=None, status=None):
        B, T, k = q_idx.shape[0], q_idx.shape[1], p.top_k
        out_idx.fill_(-1)
        out_score.fill_(-np.inf)
        for b in range(B):
            for t in range(T):
                pos = int(ctx_len[b]) - T + t
                n = (pos + 1) // p.m
                nl = max(0, min(n - keys.row0, keys.rows, n_max))
                kr = storage.decode(keys.st[b].rows(slice(0, nl)))
                s = oracle_scores(quantize_query(q_idx[b, t].numpy(), keys.st[b].fmt), w_idx[b, t].numpy(), kr)
                sel = np.sort(oracle_topk(s, k))
                out_idx[b, t, :len(sel)] = torch.from_numpy(sel + keys.row0)
                out_score[b, t, :len(sel)] = torch.from_numpy(s[sel])

    @staticmethod
    def topk_merge(p, parts_idx, parts_score, out_idx, out_score=None):
        n, B, T, k = parts_idx.shape
        out_idx.fill_(-1)
        for b in range(B):
            for t in range(T):
                cand = [(float(parts_score[r, b, t, j]), int(parts_idx[r, b, t, j]), r * k + j)
                        for r in range(n) for j in range(k) if parts_idx[r, b, t, j] >= 0]
                best = sorted(cand, key=lambda c: (-c[0], c[1]))[:k]
                keep = sorted(best, key=lambda c: c[2])  # the parts' order
                out_idx[b, t, :len(keep)] = torch.tensor([c[1] for c in keep], dtype=torch.int32)

    @staticmethod
    def sparse_attn(p, q, kv, v, win_kv, win_v, idx, sink, ctx_len, out, lse=None, status=None, sink_kv=None):
        B, T = q.shape[0], q.shape[1]
        for b in range(B):
            for t in range(T):
                pos = int(ctx_len[b]) - T + t
                n_vis = (pos + 1) // p.m
                ent = [int(g) - kv.row0 for g in idx[b, t] if 0 <= int(g) < n_vis and 0 <= int(g) - kv.row0 < kv.rows]
                rows = [storage.decode(kv.st[b].rows(np.array(ent, dtype=np.int64)))]
                wpos = window_positions(pos, p.window) if p.window > 0 else np.zeros(0, dtype=np.int64)
                rows.append(storage.decode(win_kv.st[b].rows(wpos % win_kv.capacity)))
                if p.sink_mode == 1 and not (len(wpos) and wpos[0] == 0):
                    rows.append(storage.decode(sink_kv.st[b].rows([0])))
                K = np.concatenate(rows)
                sg = np.full(q.shape[2], -np.inf) if sink is None else sink.numpy().astype(np.float64)
                o, l = joint_attention(q[b, t].numpy(), K, K, sg, p.sm_scale)
                out[b, t] = torch.from_numpy(o).to(out.dtype)
                lse[b, t] = torch.from_numpy(l).float()

    @staticmethod
    def attn_merge(p, parts_out, parts_lse, sink, ctx_len, out, lse=None):
        n, B, T, H = parts_lse.shape
        for b in range(B):
            for t in range(T):
                ls = parts_lse[:, b, t].numpy().astype(np.float64)           # [n, H]
                sg = np.full(H, -np.inf) if sink is None else sink.numpy().astype(np.float64)
                M = np.maximum(sg, ls.max(axis=0))
                w = np.exp(ls - M)                                           # [n, H]
                den = np.exp(sg - M) + w.sum(axis=0)
                o = (w[..., None] * parts_out[:, b, t].numpy().astype(np.float64)).sum(axis=0) / den[:, None]
                pos = int(ctx_len[b]) - T + t
                out[b, t] = torch.from_numpy(inverse_rope(o, pos, p.out_rope_dim, p.out_rope_base)).to(out.dtype)
                if lse is not None:
                    lse[b, t] = torch.from_numpy(M + np.log(den)).float()


def _rank_main(rank, ws, port, sink_mode, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    from long_context_sparse_compress_b200 import lib as L
    from long_context_sparse_compress_b200 import sharded
    from long_context_sparse_compress_b200 import workloads as W
    from tests.gpu_harness import make_seqs
    from tests.harness import step_tail

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        Lctx = 1024
        wl = W.CSA_DECODE_4K_F32.with_(B=2, L=Lctx, separate_v=False, Dv=128, sink_mode=sink_mode,
                                       out_rope_base=300.0)
        seqs = make_seqs(wl, [Lctx, Lctx])
        snaps = [s.snapshot() for s in seqs]
        refs = [s.step() for s in seqs]
        p = L.params(wl)
        n_cap = Lctx // wl.m + 1
        lo, n = sharded.shard_ranges(n_cap, ws, granule=32)[rank]

        def shard(key):
            sts = []
            for sn in snaps:
                st = sn[key]
                pay = np.zeros_like(st.payload)
                pay[:n] = st.payload[lo:lo + n]
                sts.append(storage.Stored(st.fmt, pay, None, st.dim, st.rope_dim))
            return HostCache(sts, lo, max(n, 1))

        win = HostCache([sn["ring_kv"] for sn in snaps])
        tok = HostCache([sn["tok_kv"] for sn in snaps]) if sink_mode == "token" else None
        dec = sharded.ShardedCsaDecode(p, rank, ws, shard("kv"), shard("idx"), win, max(n, 1), ops=OracleOps,
                                       sink_kv=tok)
        f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
        stack = lambda key: f32(np.stack([s.inp[key] for s in seqs]))
        tail = lambda key: f32(np.stack([step_tail(s.wl, s.inp[key]) for s in seqs]))
        P = seqs[0].P
        pool_args = (tail("x_kv"), tail("x_idx"), f32(P["W_kv"]), f32(P["B_kv"]), f32(P["W_idx"]), f32(P["B_idx"]),
                     Lctx - wl.m, Lctx)
        ctx = torch.tensor([Lctx] * wl.B, dtype=torch.int32)
        out = torch.zeros((wl.B, 1, wl.H, wl.Dv))
        lse = torch.zeros((wl.B, 1, wl.H))
        sink = f32(P["sink"]) if sink_mode == "logit" else None
        sel = dec.step(stack("q"), stack("q_idx"), stack("w_idx"), ctx, sink, out, lse, pool_args=pool_args)
        res = []
        for b, ref in enumerate(refs):
            res.append((sorted(sel[b, 0][sel[b, 0] >= 0].tolist()) == sorted(ref["sel"][0].tolist()),
                        float(np.abs(out[b, 0].numpy() - ref["o"][0]).max()),
                        float(np.abs(lse[b, 0].numpy() - ref["lse"][0]).max())))
        out_q.put((rank, lo, n, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,sink_mode", [(2, "logit"), (3, "token")])
def test_sharded_step_on_gloo_ranks_equals_one_device(ws, sink_mode):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, sink_mode, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == list(range(ws))
    assert sum(r[2] for r in res) == 1024 // 4 + 1 and all(r[2] > 0 for r in res)  # the ranges tile the entries
    for rank, lo, n, per_seq in res:
        for same_sel, o_err, l_err in per_seq:
            assert same_sel, rank
            assert o_err < 1e-6 and l_err < 1e-6, (rank, o_err, l_err)
