"""Lightning-indexer scores and exact top-k selection (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: "DeepSeek V4 Architecture Explained", "How compress-then-sparsify
attention works" (low-rank indexer queries and compressed indexer keys are
scored and each query keeps its top-k compressed entries); "Inside
DeepSeek-V4", section 1 (FP4 indexer, top-1,024); "How DeepSeek V4 Handles
1M Token Context", Component 3 (score every compressed entry, select the
top-k, attend to those).

Reading of the score (the pages name its parts, not its formula): with the
indexer query of head h quantised to the key's format, q~[h], and the stored
key k~[g] (both dequantised),

    s[g] = sum_h  w[h] * ReLU( q~[h] . k~[g] )      for g < N(p)

with no softmax scale and no bias; w[h] is a per-query, per-head weight.
Top-k keeps the min(k, N(p)) entries with the largest s; the order of the
returned set carries no meaning (ties here go to the lower index).
"""
import numpy as np

from . import storage


def quantize_query(q_idx, fmt):
    """Indexer query rows [..., d] rounded through the key format (f32 keeps
    the float32 values; fp8: per-row scale; fp4: per-16-block scale)."""
    return storage.quantize(fmt, np.asarray(q_idx, dtype=np.float32))


def scores(q_tilde, w, k_tilde):
    """s[g] for every key row.  q_tilde [H_I, d], w [H_I], k_tilde [N, d]."""
    dots = np.asarray(k_tilde, dtype=np.float64) @ np.asarray(q_tilde, dtype=np.float64).T
    return np.maximum(dots, 0.0) @ np.asarray(w, dtype=np.float64)


def topk(s, k):
    """Indices of the min(k, len(s)) largest scores (stable: lower index wins ties)."""
    s = np.asarray(s, dtype=np.float64)
    k_eff = min(int(k), s.shape[0])
    order = np.argsort(-s, kind="stable")
    return order[:k_eff]
