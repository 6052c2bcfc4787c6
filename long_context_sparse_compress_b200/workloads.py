"""The synthetic workloads: shapes and layer parameters, nothing else.

Each workload is one attention layer step of DeepSeek-V4's hybrid compressed
attention.  Parameter values come from "Inside DeepSeek-V4" (sections 1-2:
m = 4 and top-1,024 for CSA, m = 128 for HCA, window 128) and "DeepSeek V4
Architecture Explained" (FP8 KV with BF16 RoPE dims; shared-KV multi-query
layout); sizes are the benchmark shapes of this library.

This module holds no arithmetic of the method.  It is shared by the tests,
the benchmark and the input generator (``synth``).
"""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa", "hca" or "pair" (a CSA layer and an HCA layer)
    B: int               # sequences
    L: int               # context length after the step (new tokens included)
    T: int               # new tokens = queries per sequence (1 = decode)
    H: int = 64          # query heads
    D: int = 512         # shared KV latent dim (keys)
    rope_dim: int = 64   # trailing dims stored BF16 (kv format)
    Dv: int = 512        # value dim (= D when V is the shared latent)
    separate_v: bool = False
    m: int = 4           # compression ratio (CSA layer, or the only layer)
    G: int = 4           # group length (m, or 2m for overlapping groups)
    m_hca: int = 128     # compression ratio of the HCA layer of a pair
    w: int = 128         # sliding window
    k: int = 1024        # top-k
    H_I: int = 64        # indexer heads
    d_I: int = 128       # indexer dim
    kv_fmt: str = "kv"   # "kv" (FP8 + BF16 RoPE) or "f32"
    idx_fmt: str = "fp8"  # "fp8", "fp4" or "f32"
    x_dtype: str = "bf16"  # raw rows and gate weights
    q_dtype: str = "bf16"  # queries and the output
    n_planted: int = 0   # planted relevant entries per sequence
    sink: bool = True    # a sink is present (sink_mode "logit": a learned logit per head)
    out_rope_base: float = 0.0  # > 0: the output's rope dims rotated back by the query position
    sink_mode: str = "logit"    # "logit" or "token" (the raw row of position 0 joins every row set)
    gate_src: str = "proj"      # "proj" (z = x W) or "logits" (per-token gate logits given)

    @property
    def sm_scale(self):
        return 1.0 / (self.D ** 0.5)

    @property
    def win_cap(self):
        """Window ring rows: a step of T tokens needs T + w - 1 rows resident."""
        return max(self.w, self.T + self.w - 1)

    def n_entries(self, m=None):
        """Compressed entries visible to the last query: floor(L / m)."""
        return self.L // (m or self.m)

    def with_(self, **kw):
        return replace(self, **kw)

    def layer(self, which):
        """The single-layer view of a pair ('csa' or 'hca')."""
        if self.kind != "pair":
            return self
        if which == "csa":
            return replace(self, kind="csa", name=self.name + ".csa")
        return replace(self, kind="hca", m=self.m_hca, G=self.m_hca, name=self.name + ".hca",
                       n_planted=0)


# The five benchmark workloads (sizes as stated beside each).
CSA_DECODE_4K_F32 = Workload(
    name="csa_decode_4k_fp32", kind="csa", B=1, L=4096, T=1, H=8, D=128, rope_dim=32, Dv=128,
    separate_v=True, m=4, G=4, w=128, k=64, H_I=4, d_I=32, kv_fmt="f32", idx_fmt="f32",
    x_dtype="f32", q_dtype="f32", n_planted=8)

HCA_DECODE_64K = Workload(
    name="hca_decode_64k", kind="hca", B=4, L=65536, T=1, m=128, G=128, w=128)

CSA_DECODE_128K = Workload(
    name="csa_decode_128k", kind="csa", B=8, L=131072, T=1, m=4, G=4, k=1024, idx_fmt="fp8",
    n_planted=64)

CSA_PREFILL_256K = Workload(
    name="csa_prefill_256k", kind="csa", B=1, L=262144 + 4096, T=4096, m=4, G=4, k=1024,
    idx_fmt="fp8", n_planted=256)

PAIR_DECODE_1M_B16 = Workload(
    name="csa_hca_pair_decode_1m_b16", kind="pair", B=16, L=1048576, T=1, m=4, G=4,
    m_hca=128, k=1024, idx_fmt="fp4", n_planted=256)

PAIR_DECODE_1M_B1 = PAIR_DECODE_1M_B16.with_(name="csa_hca_pair_decode_1m_b1", B=1)

# Multi-token decode: five new tokens per sequence (a draft to verify) on the
# 1M pair, each its own query, outputs rotated back by their positions.
PAIR_DECODE_1M_B16_T5 = PAIR_DECODE_1M_B16.with_(name="csa_hca_pair_decode_1m_b16_t5", T=5,
                                                 out_rope_base=10000.0)

# Single-layer halves of the 1M pair at B = 8, for kernel profiles (inputs
# still larger than L2, a smaller device footprint).
CSA_DECODE_1M_B8 = PAIR_DECODE_1M_B16.layer("csa").with_(name="csa_decode_1m_b8_fp4", B=8)
HCA_DECODE_1M_B8 = PAIR_DECODE_1M_B16.layer("hca").with_(name="hca_decode_1m_b8", B=8)

ALL = {w.name: w for w in (CSA_DECODE_4K_F32, HCA_DECODE_64K, CSA_DECODE_128K,
                           CSA_PREFILL_256K, PAIR_DECODE_1M_B16, PAIR_DECODE_1M_B1, PAIR_DECODE_1M_B16_T5,
                           CSA_DECODE_1M_B8, HCA_DECODE_1M_B8)}
