"""Entry shards on one GPU: a long sequence's CSA entries split by range into
G caches (lcsc_cache row0 / rows), each phase of the sharded decode step run
for every shard in turn (long_context_sparse_compress_b200.sharded), the
gathers done by stacking, and the merged answer compared with the oracle's
single-device step.  This is the arithmetic of the multi-GPU path with the
same kernels; its collectives are covered by the gloo test on the CPU."""
import numpy as np
import pytest
import torch

from long_context_sparse_compress_b200 import lib as L
from long_context_sparse_compress_b200 import sharded
from long_context_sparse_compress_b200 import workloads as W
from oracle import storage
from oracle.indexer import quantize_query, scores as oracle_scores
from tests.gpu_harness import TORCH_DT, dev, download, make_seqs
from tests.harness import max_abs, rel_l2, step_tail, topk_set_ok

pytestmark = pytest.mark.gpu


def _slice_upload(cache, b, st, lo, n):
    if n == 0:
        return
    cache.set_rows(b, np.ascontiguousarray(st.payload[lo:lo + n]),
                   None if st.scale is None else np.ascontiguousarray(st.scale[lo:lo + n]))


@pytest.mark.parametrize("G,fmt,sink_mode", [(2, "fp4", "logit"), (3, "fp8", "logit"), (4, "fp4", "token")])
def test_entry_shards_merge_to_the_single_device_answer(cuda_lib, G, fmt, sink_mode):
    Lctx = 4 * 6000  # one group closes at this step
    wl = W.PAIR_DECODE_1M_B1.layer("csa").with_(B=2, L=Lctx, idx_fmt=fmt, n_planted=16, sink_mode=sink_mode,
                                                out_rope_base=10000.0)
    seqs = make_seqs(wl, [Lctx, Lctx])
    snaps = [s.snapshot() for s in seqs]
    refs = [s.step() for s in seqs]          # the oracle on one device (mutates its own caches)
    B, D, R = wl.B, wl.D, wl.rope_dim
    n_cap = Lctx // wl.m + 1
    p = L.params(wl)
    xdt, qdt = TORCH_DT[wl.x_dtype], TORCH_DT[wl.q_dtype]
    # the window ring and the sink token row, on the window rank only
    win = L.DeviceCache(B, wl.win_cap, "kv", D, R)
    tok = L.DeviceCache(B, 1, "kv", D, R) if sink_mode == "token" else None
    for b in range(B):
        _slice_upload(win, b, snaps[b]["ring_kv"], 0, wl.win_cap)
        if tok is not None:
            _slice_upload(tok, b, snaps[b]["tok_kv"], 0, 1)
    ranges = sharded.shard_ranges(n_cap, G)
    shards = []
    for r, (lo, n) in enumerate(ranges):
        cap = max(128, (n + 127) // 128 * 128)
        kv = L.DeviceCache(B, cap, "kv", D, R, row0=lo, rows=max(n, 1))
        ik = L.DeviceCache(B, cap, fmt, wl.d_I, row0=lo, rows=max(n, 1))
        for b in range(B):
            _slice_upload(kv, b, snaps[b]["kv"], lo, n)
            _slice_upload(ik, b, snaps[b]["idx"], lo, n)
        shards.append(sharded.ShardedCsaDecode(p, r, G, kv, ik, win, max(n, 1), sink_kv=tok))
    stack = lambda key, dt: dev(np.stack([s.inp[key] for s in seqs]), dt)
    tail = lambda key: dev(np.stack([step_tail(s.wl, s.inp[key]) for s in seqs]), xdt)
    P = seqs[0].P
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # phase 1: every shard pools the closing group; only its holder stores it
    for sh in shards:
        sh.pool(tail("x_kv"), tail("x_idx"), dev(P["W_kv"], xdt), dev(P["B_kv"]), dev(P["W_idx"], xdt),
                dev(P["B_idx"]), Lctx - wl.m, Lctx, status=status)
    q, q_idx, w_idx = stack("q", qdt), stack("q_idx", qdt), stack("w_idx", torch.float32)
    ctx = torch.tensor([Lctx] * B, dtype=torch.int32, device="cuda")
    # phases 2-3: local candidates, their merge, local attention
    cands = [sh.local_candidates(q_idx, w_idx, ctx, status) for sh in shards]
    sel = shards[0].merge_candidates(torch.stack([c[0] for c in cands]), torch.stack([c[1] for c in cands]))
    parts = [sh.local_attention(q, sel, ctx, status) for sh in shards]
    out = torch.zeros((B, 1, wl.H, wl.Dv), dtype=qdt, device="cuda")
    lse = torch.zeros((B, 1, wl.H), dtype=torch.float32, device="cuda")
    sink = dev(P["sink"]) if sink_mode == "logit" else None
    shards[0].merge_outputs(torch.stack([o for o, _ in parts]), torch.stack([l for _, l in parts]), sink, ctx,
                            out, lse)
    torch.cuda.synchronize()
    assert status.item() == 0
    g_new = Lctx // wl.m - 1
    for b, (s, ref) in enumerate(zip(seqs, refs)):
        # the closing group's entry went to the shard that holds it, in both tensors
        owner = next(i for i, (lo, n) in enumerate(ranges) if lo <= g_new < lo + n)
        lo = ranges[owner][0]
        d, sc = download(shards[owner].kv, b)
        got = storage.decode(storage.Stored("kv", d[g_new - lo:g_new - lo + 1],
                                            sc[g_new - lo:g_new - lo + 1], D, R))
        assert rel_l2(got, storage.decode(s.kv.rows(slice(g_new, g_new + 1)))) <= 1e-2
        # the merged selection is the top-k over all entries
        n = Lctx // wl.m
        k_all = storage.decode(s.idx.rows(slice(0, n)))
        sc_all = oracle_scores(quantize_query(s.inp["q_idx"][0], fmt), s.inp["w_idx"][0], k_all)
        ok, msg = topk_set_ok(sel[b, 0].cpu().numpy(), sc_all, wl.k)
        assert ok, msg
        assert set(s.inp["planted"].tolist()) <= set(sel[b, 0].cpu().numpy().tolist())
        o = out[b, 0].float().cpu().numpy()
        assert rel_l2(o, ref["o"][0]) <= 1e-2, rel_l2(o, ref["o"][0])
        assert max_abs(o, ref["o"][0]) <= 2e-2
        assert np.allclose(lse[b, 0].cpu().numpy(), ref["lse"][0], rtol=1e-3, atol=1e-3)


def test_topk_merge_ties_and_short_lists(cuda_lib):
    """Equal scores across parts go to the lower entry; fewer candidates than
    k leave -1 pads; the output follows the parts' order."""
    wl = W.CSA_DECODE_128K.with_(k=4)
    p = L.params(wl)
    idx = torch.tensor([[[[1, 5, 9, -1]]], [[[12, 20, -1, -1]]]], dtype=torch.int32, device="cuda")
    sc = torch.tensor([[[[2.0, 1.0, 3.0, -np.inf]]], [[[1.0, 1.0, -np.inf, -np.inf]]]], device="cuda")
    out = torch.empty((1, 1, 4), dtype=torch.int32, device="cuda")
    out_s = torch.empty((1, 1, 4), dtype=torch.float32, device="cuda")
    L.topk_merge(p, idx, sc, out, out_s)
    torch.cuda.synchronize()
    # 3.0 (entry 9), 2.0 (1), then two of the 1.0 ties at 5, 12, 20: the lower ones
    assert out[0, 0].tolist() == [1, 5, 9, 12]
    assert out_s[0, 0].tolist() == [2.0, 1.0, 3.0, 1.0]
    wl8 = wl.with_(k=8)
    out8 = torch.empty((1, 1, 8), dtype=torch.int32, device="cuda")
    idx8 = torch.nn.functional.pad(idx, (0, 4), value=-1)
    sc8 = torch.nn.functional.pad(sc, (0, 4), value=-np.inf)
    L.topk_merge(L.params(wl8), idx8, sc8, out8)
    torch.cuda.synchronize()
    assert out8[0, 0].tolist() == [1, 5, 9, 12, 20, -1, -1, -1]
