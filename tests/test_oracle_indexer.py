"""Pins of the oracle's indexer scores and top-k (CPU only)."""
import numpy as np
import torch

from oracle import storage
from oracle.indexer import quantize_query, scores, topk


def test_scores_equal_library_matmul_relu_weighted_sum():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((6, 32))
    w = rng.standard_normal(6)  # signed weights included
    k = rng.standard_normal((200, 32))
    ref = torch.relu(torch.from_numpy(k) @ torch.from_numpy(q).T) @ torch.from_numpy(w)
    assert np.allclose(scores(q, w, k), ref.numpy(), rtol=1e-13, atol=1e-13)


def test_single_head_unit_weight_is_relu_of_dot():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 16))
    k = rng.standard_normal((50, 16))
    assert np.allclose(scores(q, [1.0], k), np.maximum(k @ q[0], 0), rtol=1e-14)


def test_negative_dots_are_dropped():
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    k = np.array([[-1.0, 2.0], [3.0, -4.0]])
    # head 0 sees -1 and 3, head 1 sees 2 and -4; weights 10 and 1
    assert np.array_equal(scores(q, [10.0, 1.0], k), [2.0, 30.0])


def test_quantized_query_equals_stored_key_round_trip():
    rng = np.random.default_rng(3)
    q = (rng.standard_normal((4, 128)) / 11).astype(np.float32)
    for fmt in ("fp8", "fp4"):
        assert np.array_equal(quantize_query(q, fmt), storage.quantize(fmt, q))
    assert np.array_equal(quantize_query(q, "f32"), q.astype(np.float64))


def test_topk_equals_library_topk_on_distinct_scores():
    rng = np.random.default_rng(4)
    s = rng.standard_normal(5000)
    for k in (1, 17, 1024):
        ref = torch.topk(torch.from_numpy(s), k).indices.numpy()
        assert set(topk(s, k)) == set(ref)


def test_topk_brute_force_and_short_lists():
    rng = np.random.default_rng(5)
    s = rng.standard_normal(40)
    got = topk(s, 7)
    kth = np.sort(s)[-7]
    assert len(got) == 7 and np.all(s[got] >= kth)
    assert sorted(topk(s, 100)) == list(range(40))  # k >= N keeps every entry
    assert len(topk(s[:0], 5)) == 0


def test_topk_ties_take_lower_index():
    assert list(topk(np.zeros(10), 3)) == [0, 1, 2]
