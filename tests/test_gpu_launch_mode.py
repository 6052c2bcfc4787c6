"""Programmatic dependent launch changes no bit of a step's results.

Every kernel of the library is launched with programmatic stream
serialisation and starts by waiting for the stream's previous grid
(griddepcontrol.wait).  A kernel that touched memory before that wait could
read a predecessor's output before it is complete, and would show as results
that differ between launch modes.  Each value the steps produce has a fixed
arithmetic order (scores per key, the radix top-k with ties to the lower
index, the split-then-combine attention), so the same seeded step run with
the attribute (this process) and without it (a child process with
LCSC_PDL=0, read once per process) must agree bit for bit: outputs, lse,
the selection and every cache row the step wrote.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from long_context_sparse_compress_b200 import workloads as W

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = {
    # FP4 scoring (tiles claimed at run time), tensor-core attention, two streams
    "csa_fp4_decode": (W.PAIR_DECODE_1M_B1.layer("csa").with_(B=2, n_planted=16), [16384, 6000]),
    # FP4 scoring two queries per CTA, several queries per sequence
    "csa_fp4_multitoken": (W.PAIR_DECODE_1M_B16_T5.layer("csa").with_(B=2, n_planted=16), [16384, 6003]),
    # dense attention with split partials and their combine
    "hca_decode": (W.HCA_DECODE_64K.with_(B=3), [4096, 1024 + 128, 100]),
    # chunked prefill: FP8 scoring four queries per CTA, many lists
    "csa_fp8_prefill": (W.CSA_PREFILL_256K.with_(B=2, T=40, n_planted=8), [4096 + 40, 2002]),
}


def results(name):
    """Every array the step of case `name` writes, as host arrays."""
    from tests.gpu_harness import GpuBatch, make_seqs

    wl, lengths = CASES[name]
    gb = GpuBatch(make_seqs(wl, lengths))
    gb.run_step()
    assert gb.status.item() == 0
    out = {"out": gb.out, "lse": gb.lse, "kv": gb.kv.data, "kv_scale": gb.kv.scale, "win": gb.win_kv.data,
           "win_scale": gb.win_kv.scale}
    if gb.out_idx is not None:
        out.update(out_idx=gb.out_idx, out_score=gb.out_score, idx=gb.idx.data, idx_scale=gb.idx.scale)
    return {k: v.contiguous().view(-1).view(torch.uint8).cpu().numpy() for k, v in out.items() if v is not None}


def dump(directory):
    """Child process entry: write every case's results to `directory`."""
    for name in CASES:
        np.savez(os.path.join(directory, name + ".npz"), **results(name))


def test_programmatic_launch_changes_no_bit(cuda_lib, tmp_path):
    env = dict(os.environ, LCSC_PDL="0")
    code = "import sys; from tests import test_gpu_launch_mode as t; t.dump(sys.argv[1])"
    subprocess.run([sys.executable, "-c", code, str(tmp_path)], cwd=ROOT, env=env, check=True, timeout=600)
    for name in CASES:
        plain = np.load(os.path.join(tmp_path, name + ".npz"))
        got = results(name)
        assert sorted(got) == sorted(plain.files), name
        for key, arr in got.items():
            assert np.array_equal(arr, plain[key]), (name, key)
