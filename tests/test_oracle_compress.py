"""Pins of the oracle's softmax-gated pooling (CPU only): invariants, closed
forms, special cases and the counts the pages print."""
import os

import numpy as np
import pytest

from oracle.compress import compress_entries, compress_entries_batched, n_visible, pool_group

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_gate_weights_sum_to_one_per_channel():
    x, W, Bp = _rand((4, 16), 1), _rand((16, 16), 2, 0.3), _rand((4, 16), 3)
    _, alpha = pool_group(x, W, Bp)
    assert np.allclose(alpha.sum(axis=0), 1.0, atol=1e-14)
    assert np.all(alpha > 0)


def test_group_of_one_is_the_token():
    x = _rand((10, 8), 4)
    e = compress_entries(x, 0, _rand((8, 8), 5), _rand((1, 8), 6), m=1, G=1, entries=range(10))
    assert np.array_equal(e, x)


def test_zero_gate_is_the_mean():
    x = _rand((12, 8), 7)
    e = compress_entries(x, 0, np.zeros((8, 8)), np.zeros((4, 8)), m=4, G=4, entries=range(3))
    assert np.allclose(e, x.reshape(3, 4, 8).mean(axis=1), atol=1e-15)


def test_constant_group_and_convexity():
    W, Bp = _rand((8, 8), 8, 0.5), _rand((4, 8), 9)
    const = np.tile(_rand((1, 8), 10), (4, 1))
    e, _ = pool_group(const, W, Bp)
    assert np.allclose(e, const[0], atol=1e-14)
    x = _rand((4, 8), 11)
    e, _ = pool_group(x, W, Bp)
    assert np.all(e <= x.max(axis=0) + 1e-15) and np.all(e >= x.min(axis=0) - 1e-15)


def test_dominant_positional_bias_selects_that_token():
    x = _rand((8, 6), 12)
    Bp = np.zeros((4, 6))
    Bp[2] = 1e4
    e = compress_entries(x, 0, np.zeros((6, 6)), Bp, m=4, G=4, entries=range(2))
    assert np.array_equal(e, x[[2, 6]])


def test_gate_projection_orientation():
    # W[a, b] large: channel b's gate follows input channel a (z = x @ W);
    # channel a keeps a zero gate and is the plain mean.
    a, b = 1, 4
    x = _rand((4, 6), 13)
    x[:, a] = [0.0, 3.0, -1.0, 0.5]  # token 1 has the largest x[:, a]
    W = np.zeros((6, 6))
    W[a, b] = 1e3
    e, _ = pool_group(x, W, np.zeros((4, 6)))
    assert np.isclose(e[b], x[1, b], atol=1e-12)
    assert np.isclose(e[a], x[:, a].mean(), atol=1e-15)


def test_overlapping_groups_cover_2m_tokens():
    m, G = 4, 8
    x = _rand((16, 5), 14)
    Bp = np.zeros((G, 5))
    Bp[0] = 1e4  # the oldest token of each group dominates
    e = compress_entries(x, 0, np.zeros((5, 5)), Bp, m=m, G=G, entries=range(4))
    # entry g covers [4g - 4, 4g + 4): its oldest token is 4g - 4 (absent for g = 0)
    assert np.array_equal(e[1:], x[[0, 4, 8]])
    assert np.allclose(e[0], x[0:4].mean(axis=0), atol=1e-15)


@pytest.mark.parametrize("m,G", [(4, 4), (4, 8), (128, 128), (1, 1)])
def test_batched_form_equals_per_entry_form(m, G):
    n = 4 * max(m, 8)
    x, W, Bp = _rand((n, 8), 15), _rand((8, 8), 16, 0.3), _rand((G, 8), 17)
    a = compress_entries(x, 0, W, Bp, m, G, range(n // m))
    b = compress_entries_batched(x, W, Bp, m, G)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-15)


def test_compress_needs_its_tokens():
    with pytest.raises(ValueError):
        compress_entries(_rand((4, 3), 18), 4, np.zeros((3, 3)), np.zeros((4, 3)), 4, 4, [0])


def test_entry_counts_printed_on_the_pages():
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "entry_counts.txt"))
            if ln.strip() and not ln.startswith("#")]
    counts = {}
    for ctx, stride, glen, printed in rows:
        n = n_visible(ctx - 1, stride)
        counts[stride] = n
        assert abs(n - printed) / printed < 0.01, (ctx, stride, n, printed)
    assert counts[4] == 250000
    assert counts[4] / counts[128] == pytest.approx(32, rel=0.001)


def test_visibility_is_causal():
    # entry g becomes visible when its last token g*m + m - 1 arrives
    assert [n_visible(p, 4) for p in range(9)] == [0, 0, 0, 1, 1, 1, 1, 2, 2]
