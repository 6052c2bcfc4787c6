"""lcsc_csa_index_topk_noalloc, the indexer + top-k call that allocates
nothing: for callers that cannot allocate device memory (hosts that give all
device memory to their own pool up front, or callers reaching the library
through a foreign-function interface without a device allocator).  Its
results must equal those of lcsc_csa_index_topk, which takes a caller
workspace, call after call.  Collected last (file name) so that a run that
stops at its first failure has run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_compress_b200 import lib as L
from long_context_sparse_compress_b200 import workloads as W
from oracle import storage


def _inputs(fmt, lengths, T, seed):
    wl = W.PAIR_DECODE_1M_B1.layer("csa").with_(idx_fmt=fmt, k=512)
    rng = np.random.default_rng(seed)
    B = len(lengths)
    n_cap = L.round_capacity(max(lengths) // wl.m + 1, fmt)
    keys = L.DeviceCache(B, n_cap, fmt, wl.d_I)
    for b in range(B):
        vals = (rng.standard_normal((n_cap, wl.d_I)) * wl.d_I ** -0.5).astype(np.float32)
        st = storage.encode(fmt, vals)
        keys.set_rows(b, st.payload, st.scale)
    qi = torch.from_numpy((rng.standard_normal((B, T, wl.H_I, wl.d_I)) * wl.d_I ** -0.5).astype(np.float32))
    wi = torch.from_numpy((np.abs(rng.standard_normal((B, T, wl.H_I))) * wl.H_I ** -0.5).astype(np.float32))
    ctx = torch.tensor(lengths, dtype=torch.int32)
    return wl, keys, qi.to(torch.bfloat16).cuda(), wi.cuda(), ctx.cuda(), n_cap - 1


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["fp4", "fp8"])
def test_noalloc_equals_workspace_call_twice(cuda_lib, fmt):
    wl, keys, qi, wi, ctx, n_max = _inputs(fmt, [4 * 60000, 4 * 300 + 2, 4 * 9000], T=2, seed=5)
    B, T, k = qi.shape[0], qi.shape[1], wl.k
    p = L.params(wl)
    ref_idx = torch.full((B, T, k), -9, dtype=torch.int32, device="cuda")
    ref_sc = torch.zeros((B, T, k), dtype=torch.float32, device="cuda")
    L.index_topk(p, qi, wi, keys, ctx, n_max, ref_idx, ref_sc)
    torch.cuda.synchronize()
    # a larger request first (more lists, longer lists, the other key format),
    # so that the calls compared below start on scratch it left behind
    other = "fp8" if fmt == "fp4" else "fp4"
    wl2, keys2, qi2, wi2, ctx2, n_max2 = _inputs(other, [4 * 200000] * 4, T=3, seed=6)
    p2 = L.params(wl2)
    big_idx = torch.empty((4, 3, wl2.k), dtype=torch.int32, device="cuda")
    L.index_topk_noalloc(p2, qi2, wi2, keys2, ctx2, n_max2, big_idx, None)
    torch.cuda.synchronize()
    for call in range(2):
        out_idx = torch.full((B, T, k), -9, dtype=torch.int32, device="cuda")
        out_sc = torch.zeros((B, T, k), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.index_topk_noalloc(p, qi, wi, keys, ctx, n_max, out_idx, out_sc, status)
        torch.cuda.synchronize()
        assert status.item() == 0, call
        assert torch.equal(out_idx, ref_idx), f"call {call}: selections differ"
        ri, rs = ref_idx.cpu().numpy(), ref_sc.cpu().numpy()
        gs = out_sc.cpu().numpy()
        valid = ri >= 0
        assert np.allclose(gs[valid], rs[valid], rtol=1e-5, atol=0), f"call {call}: scores differ"
        assert np.all(np.isneginf(gs[~valid]))


def test_noalloc_rejects_requests_beyond_its_scratch():
    lib = L.load()
    wl = W.PAIR_DECODE_1M_B16.layer("csa")
    p = L.params(wl)
    # 64 lists of 2^20 entries need far more than the fixed scratch: refused
    # on the host before any launch (no pointer below is dereferenced)
    rc = lib.lcsc_csa_index_topk_noalloc(ctypes.byref(p), None, None, None, None, 64, 1, 1 << 20, None, None,
                                         None, None)
    assert rc == 4
    # sizes whose products would overflow are refused before any size is formed
    for B, T, n in ((1 << 40, 1 << 40, 10), (70000, 1, 10), (1, 1, 1 << 62)):
        rc = lib.lcsc_csa_index_topk_noalloc(ctypes.byref(p), None, None, None, None, B, T, n, None, None,
                                             None, None)
        assert rc == 1, (B, T, n)
    need = L.index_topk_workspace(p, 16, 1, 262144)
    assert need <= L.NOALLOC_SCRATCH_BYTES
