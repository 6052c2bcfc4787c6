"""Parity of the fused decode / chunked-prefill steps (lcsc_csa_decode,
lcsc_hca_decode) with the oracle's step, on scaled-down workloads with
ragged batches (different context lengths per sequence)."""
import numpy as np
import pytest
import torch

from long_context_sparse_compress_b200 import workloads as W
from oracle import storage
from tests.gpu_harness import GpuBatch, download, make_seqs
from tests.harness import max_abs, rel_l2, topk_set_ok
from oracle.indexer import quantize_query, scores as oracle_scores

pytestmark = pytest.mark.gpu

CASES = {
    # name: (workload, per-sequence context lengths)
    "csa_f32_decode": (W.CSA_DECODE_4K_F32.with_(B=3), [4096, 1000, 101]),
    "csa_fp8_decode": (W.CSA_DECODE_128K.with_(B=3), [8192, 4100, 300]),
    "csa_fp4_decode": (W.PAIR_DECODE_1M_B1.layer("csa").with_(B=2, n_planted=16), [16384, 6000]),
    # five draft tokens per sequence
    "csa_fp4_multitoken": (W.PAIR_DECODE_1M_B16_T5.layer("csa").with_(B=2, n_planted=16), [16384, 6003]),
    "hca_multitoken": (W.PAIR_DECODE_1M_B16_T5.layer("hca").with_(B=2), [16384 + 2, 5000]),
    # the output's inverse RoPE where the attention writes the output itself
    # (one split: prefill) and through the CUDA-core fp32 path
    "csa_prefill_inverse_rope": (W.CSA_PREFILL_256K.with_(B=2, T=40, n_planted=8, out_rope_base=10000.0),
                                 [4096 + 40, 2002]),
    "csa_f32_inverse_rope": (W.CSA_DECODE_4K_F32.with_(B=3, out_rope_base=500.0), [4096, 1000, 101]),
    "hca_decode": (W.HCA_DECODE_64K.with_(B=3), [4096, 1024 + 128, 100]),
    "csa_fp8_prefill": (W.CSA_PREFILL_256K.with_(B=2, T=40, n_planted=8), [4096 + 40, 2002]),
    "hca_prefill": (W.HCA_DECODE_64K.with_(B=1, T=130), [4096 + 130]),
    "csa_overlap_decode": (W.CSA_DECODE_128K.with_(B=2, G=8), [8192, 1001]),
    # the 2,048-token window reading of the pages, without a sink
    "csa_window2048_nosink": (W.CSA_DECODE_128K.with_(B=2, w=2048, sink=False), [12000, 1500]),
    "hca_window2048_nosink": (W.HCA_DECODE_64K.with_(B=2, w=2048, sink=False), [16384, 2000]),
    # the sink-token reading: the raw row of position 0 in every row set
    # (L = 100 keeps position 0 inside the window: it enters once)
    "csa_fp8_sink_token": (W.CSA_DECODE_128K.with_(B=3, sink_mode="token"), [8192, 4100, 100]),
    "hca_sink_token": (W.HCA_DECODE_64K.with_(B=3, sink_mode="token"), [4096, 1152, 100]),
    "csa_f32_sink_token": (W.CSA_DECODE_4K_F32.with_(B=3, sink_mode="token"), [4096, 1000, 101]),
    # a chunk that starts at position 0 stores the position-0 row itself, and
    # its later queries (past the 4-token window) attend to it
    "hca_sink_token_from_zero": (W.HCA_DECODE_64K.with_(B=2, T=16, w=4, sink_mode="token"), [16, 4096 + 16]),
    "csa_fp8_sink_token_from_zero": (W.CSA_PREFILL_256K.with_(B=2, T=40, w=8, n_planted=0, sink_mode="token"),
                                     [40, 2002]),
    # caller-given gate logits, with and without overlapping groups
    "csa_fp4_gate_logits": (W.PAIR_DECODE_1M_B1.layer("csa").with_(B=2, n_planted=16, gate_src="logits"),
                            [16384, 6000]),
    "csa_overlap_gate_logits": (W.CSA_DECODE_128K.with_(B=2, G=8, gate_src="logits"), [8192, 1001]),
    "hca_gate_logits": (W.HCA_DECODE_64K.with_(B=3, gate_src="logits"), [4096, 1024 + 128, 100]),
    "csa_f32_gate_logits_sink_token": (W.CSA_DECODE_4K_F32.with_(B=2, gate_src="logits", sink_mode="token"),
                                       [4096, 1000]),
}


def check_step(name, wl, lengths, query_sample=None):
    seqs = make_seqs(wl, lengths)
    gb = GpuBatch(seqs)
    gb.run_step()
    assert gb.status.item() == 0
    o_gpu = gb.out.float().cpu().numpy()
    lse_gpu = gb.lse.cpu().numpy()
    sel_gpu = gb.out_idx.cpu().numpy() if gb.out_idx is not None else None
    for b, s in enumerate(seqs):
        qs = query_sample if query_sample is not None else list(range(wl.T))
        ref = s.step(queries=qs)
        # new entries and window rows were stored like the oracle stores them
        g_lo, g_hi = ref["new_entries"]
        d, sc = download(gb.kv, b)
        if g_hi > g_lo:
            got = storage.decode(storage.Stored(s.kv.fmt, d[g_lo:g_hi], None if sc is None else sc[g_lo:g_hi],
                                                s.kv.dim, s.kv.rope_dim))
            want = storage.decode(s.kv.rows(slice(g_lo, g_hi)))
            assert rel_l2(got, want) <= (1e-5 if s.kv.fmt == "f32" else 1e-2)
        if gb.tok_kv is not None:  # the position-0 row, stored by the oracle's rule
            td, tsc = download(gb.tok_kv, b)
            assert np.array_equal(td[0], s.tok_kv.payload[0]), "position-0 row"
            if tsc is not None:
                assert tsc[0] == s.tok_kv.scale[0]
        wd, _ = download(gb.win_kv, b)
        for pos in range(s.wl.L - wl.T, s.wl.L):
            r = pos % wl.win_cap
            if s.kv.fmt == "f32":
                assert np.array_equal(wd[r], s.ring_kv.payload[r])
            else:
                assert np.array_equal(wd[r], s.ring_kv.payload[r]), f"ring row {pos}"
        for j, i in enumerate(qs):
            o = ref["o"][j]
            assert rel_l2(o_gpu[b, i], o) <= 1e-2, (name, b, i, rel_l2(o_gpu[b, i], o))
            assert max_abs(o_gpu[b, i], o) <= 2e-2
            assert np.allclose(lse_gpu[b, i], ref["lse"][j], rtol=1e-3, atol=1e-3)
            if sel_gpu is not None:
                p = s.wl.L - wl.T + i
                n = (p + 1) // wl.m
                k_all = storage.decode(s.idx.rows(slice(0, n)))
                sc_all = oracle_scores(quantize_query(s.inp["q_idx"][i], wl.idx_fmt), s.inp["w_idx"][i], k_all)
                ok, msg = topk_set_ok(sel_gpu[b, i], sc_all, wl.k)
                assert ok, (name, b, i, msg)
                if len(s.inp["planted"]) and n > len(s.inp["planted"]):
                    assert set(s.inp["planted"].tolist()) <= set(sel_gpu[b, i].tolist())


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_step_matches_oracle(cuda_lib, name):
    wl, lengths = CASES[name]
    sample = None if wl.T <= 8 else [0, 1, wl.T // 2, wl.T - 2, wl.T - 1]
    check_step(name, wl, lengths, sample)


def test_step_twice_is_deterministic(cuda_lib):
    wl = W.CSA_DECODE_128K.with_(B=2)
    gb = GpuBatch(make_seqs(wl, [8192, 5000]))
    gb.run_step()
    o1, i1 = gb.out.clone(), gb.out_idx.clone()
    gb.run_step()
    # the selection is sorted by index and ties go to the lower index, so a
    # repeated step reproduces every bit
    assert torch.equal(gb.out_idx, i1)
    assert torch.equal(gb.out, o1)
    sel = i1.cpu().numpy()
    for b in range(2):
        v = sel[b, 0][sel[b, 0] >= 0]
        assert np.all(np.diff(v) > 0)


@pytest.mark.parametrize("name,expected", [
    # every sequence completes a group this step (16384 and 6000 are multiples
    # of 4): pooling of the indexer keys and of the KV latent, one cluster per
    # sequence, each storing its rows (2); query quantisation + tensor-core
    # scoring (2); top-k collect + final (2); the attention's query images,
    # the attention with several splits per query and the combine pass (3)
    ("csa_fp4_decode", 9),
    # 4096 and 1152 complete a 128-token group: one pooling launch that stores
    # the entries and window rows itself (three clusters fit); the query
    # images, and attention over at most 32 entries + 128 window rows in one
    # split per query, which writes the output itself
    ("hca_decode", 3),
])
def test_library_counts_its_launches(cuda_lib, name, expected):
    from long_context_sparse_compress_b200 import lib as L
    wl, lengths = CASES[name]
    gb = GpuBatch(make_seqs(wl, lengths))
    n0 = L.kernel_launches()
    gb.run_step()
    assert L.kernel_launches() - n0 == expected
    assert gb.status.item() == 0
