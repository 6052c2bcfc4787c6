"""Oracle steps on scaled-down versions of the benchmark workloads (CPU
only): structure checks of the synthetic inputs and of the stored formats."""
import numpy as np
import pytest

from long_context_sparse_compress_b200 import workloads as W
from oracle import storage
from oracle.compress import compress_entries
from oracle.indexer import quantize_query, scores
from tests.harness import OracleSequence, step_tail, topk_set_ok

SMALL = {
    "csa_f32": W.CSA_DECODE_4K_F32.with_(L=1024),
    "csa_fp8": W.CSA_DECODE_128K.with_(L=8192, B=1),
    "csa_fp4": W.PAIR_DECODE_1M_B1.layer("csa").with_(L=16384, n_planted=16),
    "hca": W.HCA_DECODE_64K.with_(L=4096, B=1),
    "csa_prefill": W.CSA_PREFILL_256K.with_(L=4096 + 64, T=64, n_planted=16),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_step_runs_and_planted_entries_are_selected(name):
    wl = SMALL[name]
    seq = OracleSequence(wl, 0)
    q_sel = [0, wl.T - 1] if wl.T > 1 else None
    out = seq.step(queries=q_sel)
    assert np.all(np.isfinite(out["o"]))
    nq = len(q_sel) if q_sel else wl.T
    assert out["o"].shape == (nq, wl.H, wl.Dv)
    if wl.kind == "csa":
        for sel in out["sel"]:
            assert len(sel) == min(wl.k, wl.L // wl.m) and len(set(sel.tolist())) == len(sel)
            assert set(seq.inp["planted"].tolist()) <= set(sel.tolist())


def test_step_stores_new_entry_and_window_row():
    wl = SMALL["csa_fp8"]
    seq = OracleSequence(wl, 1)
    seq.step()
    g = wl.L // wl.m - 1
    x = step_tail(wl, seq.inp["x_kv"])
    want = compress_entries(x, wl.L - (wl.T + wl.G - 1), seq.P["W_kv"], seq.P["B_kv"], wl.m, wl.G, [g])
    st = storage.encode("kv", want, wl.rope_dim)
    assert np.array_equal(seq.kv.payload[g], st.payload[0])
    row = (wl.L - 1) % wl.win_cap
    st_r = storage.encode("kv", x[-1:], wl.rope_dim)
    assert np.array_equal(seq.ring_kv.payload[row], st_r.payload[0])


def test_topk_band_comparator():
    s = np.array([5.0, 4.0, 3.0, 3.0005, 1.0])
    ok, _ = topk_set_ok([0, 1, 3], s, 3)
    assert ok
    ok, _ = topk_set_ok([0, 1, 2], s, 3)   # 3.0 vs 3.0005: inside the 1e-3 band
    assert ok
    ok, _ = topk_set_ok([0, 1, 4], s, 3)
    assert not ok
    ok, _ = topk_set_ok([0, 0, 1], s, 3)
    assert not ok


def test_indexer_scores_use_quantized_query_and_keys():
    wl = SMALL["csa_fp4"]
    seq = OracleSequence(wl, 0)
    n = (wl.L - wl.T) // wl.m
    k_tilde = storage.decode(seq.idx.rows(slice(0, n)))
    q_tilde = quantize_query(seq.inp["q_idx"][0], "fp4")
    s = scores(q_tilde, seq.inp["w_idx"][0], k_tilde)
    # the planted keys score far above the background
    bg = np.delete(s, seq.inp["planted"])
    assert s[seq.inp["planted"]].min() > bg.mean() + 4 * bg.std()
