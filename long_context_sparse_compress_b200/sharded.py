"""One long sequence decoded on several GPUs, its compressed entries split by
range ("Inside DeepSeek-V4", section 1: top-1,024 selection over the ~262K
entries of a 1M-token context).

Rank r of a process group holds the entries [row0_r, row0_r + rows_r) of
the CSA layer's caches (KV latent and indexer keys, ``lcsc_cache`` entry
shards); the window ring lives on one rank.  A decode step is four phases
with two gathers between them:

1. ``pool``: every rank pools the group that closes at this step; only the
   rank that holds its entry stores it (the window rank also stores the new
   raw rows);
2. ``local_candidates``: the rank's own top-k (scores and global entry
   numbers) from ``lcsc_csa_index_topk`` on its keys;
   gather of the G candidate lists;
3. ``merge_candidates``: ``lcsc_topk_merge``: the global top-k, the same on
   every rank;
   ``local_attention``: ``lcsc_csa_sparse_attn`` over the listed entries the
   rank holds (plus the window on the window rank), no sink, no output
   rotation: a normalised output and its log-sum-exp;
   gather of the G (output, lse) pairs;
4. ``merge_outputs``: ``lcsc_attn_merge``: one softmax over every part, the
   sink and the inverse RoPE added once.

The two gathers carry G x k x 8 bytes and G x H x (Dv x 2 + 4) bytes per
query.  Remote data lands in this rank's own buffers before any kernel reads
it.  ``ShardedCsaDecode.step`` runs the phases with ``torch.distributed``
all-gathers; the phases are also callable one by one (a test emulates the
ranks in one process with them).  The compute of every phase goes through
``ops`` (this package's C-ABI binding by default).
"""
import ctypes
import math

import torch

from . import lib as L


def shard_ranges(n_entries, world, granule=128):
    """Contiguous entry ranges (row0, rows) of ``world`` ranks over
    ``n_entries`` entries, each a multiple of ``granule`` rows (whole key
    tiles) except the last; a rank past the end gets (row0, 0)."""
    per = max(granule, math.ceil(n_entries / world / granule) * granule)
    out = []
    for r in range(world):
        lo = min(r * per, n_entries)
        out.append((lo, max(0, min(per, n_entries - lo))))
    return out


class DeviceOps:
    """The compute of each phase on this rank's GPU, through the C ABI."""

    compress = staticmethod(L.compress)
    index_topk = staticmethod(L.index_topk)
    topk_merge = staticmethod(L.topk_merge)
    sparse_attn = staticmethod(L.sparse_attn)
    attn_merge = staticmethod(L.attn_merge)


def local_params(p, window_rank):
    """The layer's parameters for one rank's share of the attention: the
    window rank keeps the window (and a sink token, which it attends once);
    the others have no window and no sink; the output rotation is left to
    the merge."""
    q = L.Params()
    ctypes.memmove(ctypes.addressof(q), ctypes.addressof(p), ctypes.sizeof(L.Params))
    if not window_rank:
        q.window = 0
        q.sink_mode = L.SINK["logit"]
    q.out_rope_base = 0.0
    q.out_rope_dim = 0
    return q


class ShardedCsaDecode:
    """The CSA decode step of B sequences (T = 1) on this rank's entry shard.

    p: the layer's ``lcsc_params`` (G = m groups); kv, idx_keys: this rank's
    shard caches (``rows`` > 0; the last rank may hold fewer); win_kv: the
    window ring (read on the window rank only; any valid cache elsewhere);
    sink_kv: with a sink token, its one-row cache (window rank); n_local:
    the shard's rows; group: the process group (None: the default one)."""

    def __init__(self, p, rank, world, kv, idx_keys, win_kv, n_local, window_rank=None, group=None, ops=None,
                 sink_kv=None):
        if p.group_len != p.m:
            raise ValueError("entry shards pool non-overlapping groups (G = m)")
        self.p, self.rank, self.world, self.group = p, rank, world, group
        self.kv, self.idx_keys, self.win_kv, self.n_local = kv, idx_keys, win_kv, n_local
        self.window_rank = world - 1 if window_rank is None else window_rank
        self.p_attn = local_params(p, rank == self.window_rank)
        self.sink_kv = sink_kv if rank == self.window_rank else None
        self.ops = ops or DeviceOps

    # ------------------------------------------------------------ phases
    def pool(self, x_kv, x_idx, w_kv, b_kv, w_idx, b_idx, tok_begin, tok_end, status=None):
        """Phase 1: pool the groups closing in [tok_begin, tok_end) (tok_begin
        a multiple of m; x rows cover tok_begin .. tok_end - 1); only this
        rank's entries are stored, the window rank also stores the raw rows."""
        win = self.win_kv if self.rank == self.window_rank else None
        B = x_kv.shape[0]
        self.ops.compress(self.p, "kv", x_kv, B, tok_begin, tok_end, w_kv, b_kv, self.kv, win, status)
        self.ops.compress(self.p, "idx", x_idx, B, tok_begin, tok_end, w_idx, b_idx, self.idx_keys, None, status)

    def local_candidates(self, q_idx, w_idx, ctx_len, status=None):
        """Phase 2: this shard's top-k: (idx [B][1][k] global, scores)."""
        B, T = q_idx.shape[0], q_idx.shape[1]
        idx = torch.empty((B, T, self.p.top_k), dtype=torch.int32, device=q_idx.device)
        sc = torch.empty((B, T, self.p.top_k), dtype=torch.float32, device=q_idx.device)
        self.ops.index_topk(self.p, q_idx, w_idx, self.idx_keys, ctx_len, self.n_local, idx, sc, status=status)
        return idx, sc

    def merge_candidates(self, parts_idx, parts_score):
        """Phase 3a: the top-k over every shard's candidates."""
        sel = torch.empty(parts_idx.shape[1:], dtype=torch.int32, device=parts_idx.device)
        self.ops.topk_merge(self.p, parts_idx, parts_score, sel)
        return sel

    def local_attention(self, q, sel, ctx_len, status=None):
        """Phase 3b: attention over the selected entries this shard holds
        (and the window on the window rank): (out, lse)."""
        B, T, H = q.shape[0], q.shape[1], q.shape[2]
        out = torch.empty((B, T, H, self.p.v_dim), dtype=q.dtype, device=q.device)
        lse = torch.empty((B, T, H), dtype=torch.float32, device=q.device)
        self.ops.sparse_attn(self.p_attn, q, self.kv, None, self.win_kv, None, sel, None, ctx_len, out, lse,
                             status=status, sink_kv=self.sink_kv)
        return out, lse

    def merge_outputs(self, parts_out, parts_lse, sink, ctx_len, out, lse=None):
        """Phase 4: one softmax over every shard's share, with the sink."""
        self.ops.attn_merge(self.p, parts_out, parts_lse, sink, ctx_len, out, lse)

    # ------------------------------------------------------------ a whole step
    def _gather(self, t):
        import torch.distributed as dist
        parts = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(parts, t.contiguous(), group=self.group)
        return parts.view((self.world,) + tuple(t.shape))

    def step(self, q, q_idx, w_idx, ctx_len, sink, out, lse=None, status=None, pool_args=None):
        """One decode step on every rank (each calls it with the same
        queries); ``pool_args``: the arguments of ``pool`` when a group
        closes at this step, else None.  Every rank ends with the output."""
        if pool_args is not None:
            self.pool(*pool_args, status=status)
        idx, sc = self.local_candidates(q_idx, w_idx, ctx_len, status)
        sel = self.merge_candidates(self._gather(idx), self._gather(sc))
        o, l = self.local_attention(q, sel, ctx_len, status)
        self.merge_outputs(self._gather(o), self._gather(l), sink, ctx_len, out, lse)
        return sel
