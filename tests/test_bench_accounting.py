"""The benchmark's algorithmic work per step (CPU only): the byte and flop
counts behind its step rooflines, against the per-configuration figures
worked out by hand from the shapes (HBM bytes each decode step must move at
least once; indexer and attention flops of the chunked-prefill step)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_sparse_compress_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("wl,mb", [
    (W.PAIR_DECODE_1M_B16, 398.0),   # 16 x (19.7 MB CSA + 5.09 MB HCA) + 1.35 MB of gates
    (W.PAIR_DECODE_1M_B1, 26.1),
    (W.CSA_DECODE_128K, 41.8),       # 8 x (4.33 MB keys + 0.59 MB gathered + window, q, o)
    (W.HCA_DECODE_64K, 3.3),
    (W.CSA_DECODE_4K_F32, 0.48),
    (W.CSA_PREFILL_256K, 0.67e3),    # queries and outputs (0.54 GB) dominate
])
def test_step_bytes(wl, mb):
    nbytes, _ = bench.step_work(wl)
    assert abs(nbytes / 1e6 - mb) <= 0.02 * mb, nbytes


def test_prefill_flops_by_type():
    _, fl = bench.step_work(W.CSA_PREFILL_256K)
    # 270,531,584 causal (query, entry) pairs x 2 x 64 x 128
    assert fl["fp8"] == 270531584 * 16384
    assert abs(fl["bf16"] / 1e12 - 0.62) < 0.01


def test_step_roofline_fractions():
    peaks = {"hbm_gbs": 6446.0, "bf16_tflops": 1686.5, "source": "measured"}
    r = bench.step_roofline(W.PAIR_DECODE_1M_B16, 0.274, peaks)
    assert r["bound"] == "hbm" and abs(r["frac"] - 0.225) < 0.002
    r = bench.step_roofline(W.CSA_PREFILL_256K, 4.93, peaks)
    # (4.43 T / 3373 T + 0.62 T / 1686.5 T) / 4.93 ms
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.341) < 0.003
