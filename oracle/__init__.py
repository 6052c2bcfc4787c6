"""Plain fp64 CPU oracle of one DeepSeek-V4 compressed-attention layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import anything in this package.  The CUDA library never
calls it, and it shares no code, table or helper with the CUDA sources.

What it computes (each module cites the passage it restates):

* ``formats``   -- OCP E4M3 / E2M1 and bfloat16 round-to-nearest-even codecs.
* ``storage``   -- the cache row formats: FP8 with BF16 RoPE dims
                   ("DeepSeek V4 Architecture Explained", Key numbers table,
                   row "KV storage precision"), FP8 / FP4 indexer keys
                   ("Inside DeepSeek-V4", section 1, "FP4 Lightning Indexer").
* ``compress``  -- softmax-gated pooling of m-token groups with learned
                   positional biases ("DeepSeek V4 Architecture Explained",
                   "How compress-then-sparsify attention works").
* ``indexer``   -- lightning-indexer scores and exact top-k selection
                   (same section; "How DeepSeek V4 Handles 1M Token Context",
                   Component 3).
* ``attention`` -- one joint softmax over the selected (CSA) or all (HCA)
                   compressed entries, the uncompressed sliding window and a
                   per-head attention sink (a learned logit, or the raw row
                   of position 0 in the sink-token reading, see ``step``).
* ``step``      -- one decode / chunked-prefill step of a CSA or HCA layer.

All arithmetic is float64 except the decisions that produce stored codes
(FP8/FP4/BF16 encodes), which are taken in float32 exactly as the stored
format is defined, so that both sides of a parity test take them in the
same precision.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against library routines, closed forms, invariants or brute force.  What is
*not* pinned is whether the readings of the pages (gate form, scale rules,
score form, sink form) match DeepSeek's released model: the pages do not
define them, so they are fixed here as parameters.
"""
