"""The failure path of the bounded waits of the tensor-core kernels.

lcsc_set_wait_test shortens the waits of the tensor-core attention and
scoring kernels and makes one thread of each CTA wait on a barrier that
cannot complete (the attention's Q K^T issuer on the barrier it commits to at
its end, the scoring's first lane on the drain of an accumulator it has not
filled).  Every CTA then gives up: the device status reports
LCSC_DEV_TIMEOUT, the call ends without a CUDA error (each role waited for
its copies and MMAs in flight, and the CTA freed its tensor memory), and the
calls that follow, with the waits restored, match the oracle again on the
same context.  No GPU fault is involved: only waits with a limit run out.
"""
import pytest

from long_context_sparse_compress_b200 import lib as L
from tests import test_gpu_stages as stages

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms: the calls below take microseconds when nothing stalls


def _stalled(run):
    L.set_wait_test(LIMIT_NS, True)
    try:
        run()
    finally:
        L.set_wait_test(0, False)


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_attention_wait_runs_out_then_recovers(cuda_lib, kind):
    _stalled(lambda: stages.check_attention(kind, "kv", None, stalled=True))
    stages.check_attention(kind, "kv", None)


# FP4 with one query per CTA (four lanes, tiles claimed at run time), FP4 with
# two (two lanes, static shares) and FP8 with one (two lanes)
@pytest.mark.parametrize("fmt,T", [("fp4", 1), ("fp4", 3), ("fp8", 3)])
def test_scoring_wait_runs_out_then_recovers(cuda_lib, fmt, T):
    lengths = [4 * 5000 + 3, 4 * 37, 4 * 2100 + 1]  # one list shorter than k
    _stalled(lambda: stages.check_index_topk(fmt, lengths, T, seed=7, stalled=True))
    stages.check_index_topk(fmt, lengths, T, seed=7)
