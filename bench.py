#!/usr/bin/env python3
"""Decode throughput of one DeepSeek-V4 CSA + HCA attention layer pair at a
1,048,576-token context (default workload: 16 sequences), on B200.

A step is one decode token per sequence through both layers, every stage
included: pooling of the group that closes at this token (CSA m = 4 and HCA
m = 128), the window-ring write, FP4 indexer scoring, exact top-1024,
sparse attention over 1024 entries + 128 window rows + sink (CSA), and
dense attention over 8192 entries + window + sink (HCA).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl lcsc|reference]

Prints ONE JSON line on rank 0.  Multi-GPU (torchrun): every rank runs its
own sequences (weak scaling, no data-path collective); the timed region is
bracketed by a barrier and synchronisation, and the time is the max over
ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_sparse_compress_b200 import lib as L  # noqa: E402
from long_context_sparse_compress_b200 import synth, workloads  # noqa: E402

METRIC = "CSA/HCA decode queries/s at 128K-1M ctx; % HBM roofline; prefill % tensor peak"
DEFAULT_WORKLOAD = workloads.PAIR_DECODE_1M_B16.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
# dense tensor-core rate of an operand type relative to bf16 (nominal B200 ratios)
TENSOR_RATIO = {"fp8": 2.0, "fp4": 4.0}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        d["source"] = "measured"
        return d
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


# --------------------------------------------------------------- inputs

class Layer:
    """Device state of one layer for B sequences: caches filled with seeded
    synthetic entries (the recipe of ``synth``, drawn on the device), the
    window ring, raw tail rows, queries and gates."""

    def __init__(self, wl, seed, device):
        self.wl, self.dev = wl, device
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        B, T, D, m = wl.B, wl.T, wl.D, wl.m
        self.p = L.params(wl)
        rope = wl.rope_dim if wl.kv_fmt == "kv" else 0
        xdt = torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32
        qdt = torch.bfloat16 if wl.q_dtype == "bf16" else torch.float32
        rn = lambda shape, std: torch.randn(shape, generator=g, device=device) * std
        self.n_max = wl.L // m
        n_cap = self.n_max + 1
        n_old = (wl.L - T) // m
        csa = wl.kind == "csa"
        self.q = rn((B, T, wl.H, D), D ** -0.5).to(qdt)
        self.q_idx = rn((B, T, wl.H_I, wl.d_I), wl.d_I ** -0.5).to(qdt) if csa else None
        self.w_idx = (rn((B, T, wl.H_I), 1.0).abs() * wl.H_I ** -0.5) if csa else None
        self.sink = rn((wl.H,), 1.0)
        self.w_kv = rn((D, D), 0.02).to(xdt)
        self.b_kv = rn((wl.G, D), 1.0)
        self.w_ik = rn((wl.d_I, wl.d_I), 0.02).to(xdt) if csa else None
        self.b_ik = rn((wl.G, wl.d_I), 1.0) if csa else None
        self.kv = L.DeviceCache(B, n_cap, wl.kv_fmt, D, rope, device)
        self.idx = L.DeviceCache(B, L.round_capacity(n_cap, wl.idx_fmt), wl.idx_fmt, wl.d_I, 0, device) if csa else None
        self.win = L.DeviceCache(B, wl.win_cap, wl.kv_fmt, D, rope, device)
        R = synth.tail_rows(wl)
        tail_kv = rn((B, R, D), D ** -0.5).to(xdt)
        tail_ik = rn((B, R, wl.d_I), wl.d_I ** -0.5).to(xdt) if csa else None
        self.x_kv = tail_kv[:, R - (T + wl.G - 1):].contiguous()
        self.x_ik = tail_ik[:, R - (T + wl.G - 1):].contiguous() if csa else None
        self.planted = []
        for b in range(B):
            u_kv = self.q[b].float().mean(dim=(0, 1))
            u_kv = u_kv / u_kv.norm()
            vals = rn((n_old, D), D ** -0.5)
            n_pl = min(wl.n_planted, n_old)
            pl = None
            if n_pl:
                n_lim = max(n_pl, min(n_old, (wl.L - T - wl.w) // m))
                pl = torch.randperm(n_lim, generator=g, device=device)[:n_pl]
                vals[pl] = u_kv[None] + rn((n_pl, D), 0.1 * D ** -0.5)
            L.encode_rows(self.p, "kv", vals[None].contiguous(), 0, self.kv.seq(b))
            del vals
            if csa:
                v = (self.w_idx[b][..., None] * self.q_idx[b].float()).sum(dim=1).mean(dim=0)
                v = v / v.norm()
                ik = rn((n_old, wl.d_I), wl.d_I ** -0.5)
                if pl is not None:
                    ik[pl] = v[None] + rn((n_pl, wl.d_I), 0.1 * wl.d_I ** -0.5)
                L.encode_rows(self.p, "idx", ik[None].contiguous(), 0, self.idx.seq(b))
                del ik
            self.planted.append(pl)
            # the window ring: raw rows of positions L - T - w + 1 .. L - T - 1
            ring = torch.zeros((wl.win_cap, D), device=device)
            for pos in range(max(0, wl.L - T - wl.w + 1), wl.L - T):
                ring[pos % wl.win_cap] = tail_kv[b, pos - (wl.L - R)].float()
            L.encode_rows(self.p, "kv", ring[None].contiguous(), 0, self.win.seq(b))
        self.ctx_len = torch.full((B,), wl.L, dtype=torch.int32, device=device)
        self.out = torch.empty((B, T, wl.H, wl.Dv), dtype=qdt, device=device)
        self.lse = torch.empty((B, T, wl.H), dtype=torch.float32, device=device)
        self.sel = torch.empty((B, T, wl.k), dtype=torch.int32, device=device) if csa else None
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws = L.workspace(L.step_workspace(self.p, csa, B, T, self.n_max), device)
        self.step = L.make_step(B, T, self.n_max, self.ctx_len, self.x_kv, None, self.x_ik, self.w_kv,
                                self.b_kv, None, None, self.w_ik, self.b_ik, self.kv, None, self.idx,
                                self.win, None, self.q, self.q_idx, self.w_idx, self.sink, self.out,
                                self.lse, self.sel, None)
        self._ev_arr = None

    def set_events(self, events):
        self._ev_arr = L.set_step_events(self.step, events)

    def clear_events(self):
        self.step.events = None
        self.step.n_events = 0
        self._ev_arr = None

    def run(self, stream=None):
        L.decode_step(self.p, self.step, self.wl.kind == "csa", self.ws, self.status, stream)

    # host-side copies for the end-to-end measurement
    def io_slot(self):
        """A second set of the step's per-step device inputs and outputs (the
        caches, weights and workspace are shared) with a step struct over
        them, for the double-buffered end-to-end loop: (step, [(device input,
        pinned host input)], (device output, pinned host output)).  The inputs
        a decode step receives: the T new tokens' raw rows (the G - 1 older
        rows of the closing group arrived with earlier steps and stay on the
        device, the way a caller keeps a group's rows in a ring written twice
        so that they are always contiguous), the queries, the indexer queries
        and weights, and the context lengths.  The dense ones (queries, their
        indexer queries and weights, lengths) share one device buffer and one
        pinned host buffer at 16-byte aligned offsets, so that they travel in
        one copy; the raw rows are a strided slice of each sequence's rows
        and travel in a copy of their own."""
        clone = lambda t: None if t is None else t.clone()
        csa = self.wl.kind == "csa"
        dense = [self.q, self.ctx_len] + ([self.q_idx, self.w_idx] if csa else [])
        sizes = [t.numel() * t.element_size() for t in dense]
        offs = [sum((n + 15) // 16 * 16 for n in sizes[:i]) for i in range(len(sizes))]
        total = offs[-1] + (sizes[-1] + 15) // 16 * 16
        dbuf = torch.empty(total, dtype=torch.uint8, device=self.dev)
        hbuf = torch.zeros(total, dtype=torch.uint8).pin_memory()
        views = []
        for t, o, n in zip(dense, offs, sizes):
            dv = dbuf[o:o + n].view(t.dtype).view(t.shape)
            dv.copy_(t)
            hbuf[o:o + n].view(t.dtype).view(t.shape).copy_(t.cpu())
            views.append(dv)
        q, ctx = views[0], views[1]
        q_idx, w_idx = (views[2], views[3]) if csa else (None, None)
        x_kv, x_ik = clone(self.x_kv), clone(self.x_ik)
        out, lse, sel = torch.empty_like(self.out), torch.empty_like(self.lse), clone(self.sel)
        step = L.make_step(self.wl.B, self.wl.T, self.n_max, ctx, x_kv, None, x_ik, self.w_kv, self.b_kv, None,
                           None, self.w_ik, self.b_ik, self.kv, None, self.idx, self.win, None, q, q_idx, w_idx,
                           self.sink, out, lse, sel, None)
        T = self.wl.T
        rows = [(x_kv[:, -T:], self.x_kv[:, -T:].contiguous().cpu().pin_memory())]
        if csa:
            rows.append((x_ik[:, -T:], self.x_ik[:, -T:].contiguous().cpu().pin_memory()))
        return step, [(dbuf, hbuf)] + rows, (out, torch.empty(out.shape, dtype=out.dtype).pin_memory())


class StepRunner:
    """Issues one step of a workload's layers.  The two layers of a pair take
    independent inputs (queries and caches of their own), so the HCA layer
    runs on a second stream beside the CSA layer: every step forks it from the
    caller's stream and joins it back, so a step still ends when both layers
    have.  ``hca_first``: which layer is enqueued first."""

    def __init__(self, layers, stream, hca_first=True):
        self.layers, self.stream, self.hca_first = layers, stream, hca_first
        self.streams = [stream] + [torch.cuda.Stream(device=stream.device) for _ in layers[1:]]
        self.fork = torch.cuda.Event()
        self.joins = [torch.cuda.Event() for _ in layers]

    def run(self, before=None):
        """One step; ``before(i, s)`` runs on layer i's stream before it (the
        end-to-end loop waits there for the layer's uploads)."""
        if len(self.layers) > 1:
            self.fork.record(self.stream)
            for s in self.streams[1:]:
                s.wait_event(self.fork)
        order = list(range(len(self.layers)))
        if self.hca_first:
            order.reverse()
        for i in order:
            if before is not None:
                before(i, self.streams[i])
            self.layers[i].run(self.streams[i])
        for i in range(1, len(self.layers)):
            self.joins[i].record(self.streams[i])
            self.stream.wait_event(self.joins[i])


# ------------------------------------------------------------ measurement

class ClockSampler:
    """nvidia-smi clock / throttle samples of one GPU while it runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.samples, self.proc = [], None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.target = str(device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.target, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        self.proc.wait()
        self.thread.join(timeout=2)
        rows = [s for t, s in self.samples if t0 <= t <= t1] or [s for _, s in self.samples]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def strip_c_comments(src):
    """C/C++/CUDA source with its comments removed and blank lines dropped:
    what the compiler sees of the code, so that an edit to a comment does not
    count as a change of the kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = ("".join(out)).split("\n")
    return "\n".join(l.rstrip() for l in lines if l.strip())


def source_sha(*names):
    """Hash of the named kernel sources, comments excluded."""
    h = hashlib.sha256()
    for n in names:
        src = open(os.path.join(ROOT, "long_context_sparse_compress_b200", "csrc", n)).read()
        h.update(strip_c_comments(src).encode())
    return h.hexdigest()[:16]


def index_dtype(layer_wls):
    """The indexer's arithmetic type, as the dtype string's first part."""
    fmts = {lw.idx_fmt for lw in layer_wls if lw.kind == "csa"}
    names = {"fp4": "e2m1 x e2m1 block-scaled MMA (indexer), ", "fp8": "e4m3 x e4m3 MMA (indexer), ",
             "f32": "f32 (indexer), ", "bf16": "f32 from bf16 (indexer), "}
    return "".join(names.get(f, f + " (indexer), ") for f in sorted(fmts))


# ------------------------------------------------- algorithmic work of a step
# What one step of a layer must move and compute at least once, from the
# shapes alone (the per-unit figures of the kernels' rooflines): every stored
# row it reads once, every row it writes once, the queries and outputs once.

def _kv_row_bytes(lw):
    """Stored KV row with its scale."""
    rope = lw.rope_dim if lw.kv_fmt == "kv" else 0
    return L.row_bytes(lw.kv_fmt, lw.D, rope) + (4 if lw.kv_fmt != "f32" else 0)


def _idx_row_bytes(lw):
    """Stored indexer key with its scales (FP4: one byte per 16 values)."""
    extra = {"fp4": lw.d_I // 16, "fp8": 4, "f32": 0}[lw.idx_fmt]
    return L.row_bytes(lw.idx_fmt, lw.d_I) + extra


def layer_step_bytes(lw):
    """Algorithmic bytes of one step of a single layer over its B sequences."""
    x_b = 2 if lw.x_dtype == "bf16" else 4
    q_b = 2 if lw.q_dtype == "bf16" else 4
    nv = 2 if lw.separate_v else 1            # K and V tensors
    kv_row = _kv_row_bytes(lw)
    T, m, G = lw.T, lw.m, lw.G
    n_new = lw.L // m - (lw.L - T) // m       # entries the step pools
    seq = T * lw.H * (lw.D + lw.Dv) * q_b     # queries in, outputs out
    seq += (T + G - 1) * lw.D * x_b * nv      # raw rows of the closing groups and new tokens
    seq += (n_new + T) * kv_row * nv          # new entries and window rows written
    seq += min(T + lw.w - 1, lw.L) * kv_row * nv  # window rows read (distinct positions)
    if lw.kind == "csa":
        ik = _idx_row_bytes(lw)
        seq += (lw.L // m) * ik                           # every visible indexer key, once
        seq += (T + G - 1) * lw.d_I * x_b + n_new * ik    # its raw rows and new keys
        seq += T * lw.H_I * (lw.d_I * q_b + 4)            # indexer queries and head weights
        n_ent = lw.L // m
        seq += min(T * min(lw.k, n_ent), n_ent) * kv_row * nv  # gathered entries (each stored row once)
        seq += T * min(lw.k, n_ent) * 4                      # selection written
    else:
        seq += (lw.L // m) * kv_row * nv                  # every visible entry, once
    layer = nv * (lw.D * lw.D * x_b + G * lw.D * 4) + lw.H * 4  # gates, biases, sink
    if lw.kind == "csa":
        layer += lw.d_I * lw.d_I * x_b + G * lw.d_I * 4
    return lw.B * seq + layer


def layer_step_flops(lw):
    """Algorithmic flops of one step of a layer, by the operand type of the
    contraction that carries them: {"fp4" / "fp8" / "f32": indexer scoring,
    "bf16": attention and the gate GEMM}.  The attention's code dims run as
    pairs of E4M3 MMAs (two-term query and weights), which together take the
    time of one bf16 MMA, and its RoPE dims as bf16 MMAs: its flops count at
    the bf16 rate."""
    out = {}
    T, m = lw.T, lw.m
    pos = [lw.L - T + t for t in range(T)]
    vis = [(p + 1) // m for p in pos]
    if lw.kind == "csa":
        out[lw.idx_fmt] = lw.B * sum(vis) * 2 * lw.H_I * lw.d_I
        rows = [min(lw.k, n) + min(lw.w, p + 1) for n, p in zip(vis, pos)]
    else:
        rows = [n + min(lw.w, p + 1) for n, p in zip(vis, pos)]
    attn = lw.B * sum(rows) * 2 * lw.H * (lw.D + lw.Dv)
    n_new = lw.L // m - (lw.L - T) // m
    gate = lw.B * n_new * lw.G * 2 * (lw.D * lw.D * (2 if lw.separate_v else 1) +
                                      (lw.d_I * lw.d_I if lw.kind == "csa" else 0))
    out["bf16"] = out.get("bf16", 0) + attn + gate
    return out


def step_work(wl):
    """(bytes, flops by type) of one step of a workload (both layers of a pair)."""
    layers_wl = [wl.layer("csa"), wl.layer("hca")] if wl.kind == "pair" else [wl]
    fl = {}
    for lw in layers_wl:
        for k, v in layer_step_flops(lw).items():
            fl[k] = fl.get(k, 0) + v
    return sum(layer_step_bytes(lw) for lw in layers_wl), fl


def step_roofline(wl, ms_step, peaks):
    """The whole step against its bound: decode steps against HBM (bytes /
    time / measured copy bandwidth), chunked prefill against the tensor pipe
    (sum of flops_i / peak_i over the contractions, divided by the time, with
    the burst bf16 peak times the nominal ratio of each operand type: the
    step lasts milliseconds, not seconds)."""
    nbytes, fl = step_work(wl)
    if wl.T >= 64:
        bf = float(peaks["bf16_tflops"])
        ideal_s = sum(v / (bf * TENSOR_RATIO.get(k, 1.0) * 1e12) for k, v in fl.items())
        return {"bound": "tensor", "frac": round(ideal_s / (ms_step / 1e3), 4),
                "ideal_ms": round(ideal_s * 1e3, 4), "ms_per_step": round(ms_step, 5),
                "flops_by_type": fl, "peak": f"{peaks['source']} bf16_tflops {bf} x nominal ratio per type",
                "algorithmic_bytes": nbytes}
    gbs = nbytes / (ms_step / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
            "frac": round(gbs / float(peaks["hbm_gbs"]), 4), "algorithmic_bytes": nbytes,
            "ms_per_step": round(ms_step, 5), "peak_source": peaks["source"] + " hbm_gbs"}


def recorded_traffic(kernel, workload, sha):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel][workload]
    except (OSError, ValueError, KeyError):
        return None
    if rec.get("source_sha") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


def dist_setup():
    """One process per GPU under torchrun: NCCL on GPUs (gloo on a host
    without one, which the CPU tests use).  Returns (world size, rank, local
    rank)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return 1, 0, 0
    import datetime
    import torch.distributed as dist
    rank, local = int(os.environ["RANK"]), int(os.environ.get("LOCAL_RANK", "0"))
    timeout = datetime.timedelta(seconds=120)
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=timeout)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, x):
    """The largest x over the ranks (every rank gets it)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(rank, layer):
    """Seed of a rank's sequences for one layer: every rank owns its own
    sequences and caches (the decode batch shards by sequence)."""
    return synth.SEED + 1000 * rank + layer


def job_throughput(B, T, ws, steps, ms_total):
    """Queries per second of the whole job: the queries every rank answered
    over the slowest rank's time."""
    return B * T * ws * steps / (ms_total / 1e3)


L2_BYTES = 126 * 2 ** 20
SUB_WORKLOADS = (workloads.PAIR_DECODE_1M_B1.name, workloads.CSA_DECODE_128K.name,
                 workloads.CSA_PREFILL_256K.name, workloads.PAIR_DECODE_1M_B16_T5.name)


def measure_sub(name, dev, peaks, warmup, target_s=0.4, max_steps=5000):
    """One more workload timed in the same run: its own layers, warm-up,
    clocks and timed steps (as many as fill about ``target_s``).  A step
    whose working set fits in L2 is timed alone, with L2 flushed before it
    (a 256 MiB buffer written, then a second one read, outside the step's
    events); larger ones run back to back."""
    wl = workloads.ALL[name]
    layers_wl = [wl.layer("csa"), wl.layer("hca")] if wl.kind == "pair" else [wl]
    layers = [Layer(lw, shard_seed(0, i), dev) for i, lw in enumerate(layers_wl)]
    stream = torch.cuda.current_stream()
    step = StepRunner(layers, stream).run

    nbytes, _ = step_work(wl)
    flush = nbytes < 2 * L2_BYTES
    if flush:
        fw = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        fr = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        fw.fill_(1)
        fr.sum()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    for ly in layers:
        if int(ly.status.item()) != 0:
            raise RuntimeError(f"device status {int(ly.status.item())} in {ly.wl.name}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    step()
    e1.record(stream)
    torch.cuda.synchronize()
    est_ms = max(e0.elapsed_time(e1), 1e-3)
    steps = int(min(max_steps, max(20, target_s * 1e3 / est_ms)))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    # stage boundaries of every layer's step (the library records them), in
    # a pass of their own after the timed steps: the events add to a step
    n_ev = {"csa": 6, "hca": 3}
    n_stage = min(steps, 50)
    stage_ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(n_ev[ly.wl.kind])] for ly in layers]
                for _ in range(n_stage)]
    for evs in stage_ev:
        for le in evs:
            for e in le:
                e.record(stream)  # creates the events
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0 = time.time()
    n0 = L.kernel_launches()
    def with_events(i):
        for ly, le in zip(layers, stage_ev[i]):
            ly.set_events(le)

    if flush:
        for i in range(steps):
            flush_l2()
            starts[i].record(stream)
            step()
            stops[i].record(stream)
    else:
        starts[0].record(stream)
        for i in range(steps):
            step()
        stops[0].record(stream)
    launches = L.kernel_launches() - n0
    torch.cuda.synchronize()
    t1 = time.time()
    time.sleep(0.25)
    clocks = sampler.stop(t0, t1)
    if flush:
        ms = float(np.mean([a.elapsed_time(b) for a, b in zip(starts, stops)]))
    else:
        ms = starts[0].elapsed_time(stops[0]) / steps
    for i in range(n_stage):  # the stage pass
        if flush:
            flush_l2()
        with_events(i)
        step()
    torch.cuda.synchronize()
    for ly in layers:
        ly.clear_events()
        if int(ly.status.item()) != 0:
            raise RuntimeError(f"device status {int(ly.status.item())} in {ly.wl.name}")
    names = {"csa": ("idx_compress", "quantize_join", "index_score", "topk", "kv_join_sparse_attn"),
             "hca": ("compress", "dense_attn")}
    stage_ms = {}
    for j, ly in enumerate(layers):
        for k, nm in enumerate(names[ly.wl.kind]):
            stage_ms[ly.wl.kind + "." + nm] = round(float(np.mean(
                [stage_ev[i][j][k].elapsed_time(stage_ev[i][j][k + 1]) for i in range(n_stage)])), 4)
    unit = "tokens/s" if wl.T >= 64 else "queries/s"
    rec = {"workload": wl.name, "layers": [lw.name for lw in layers_wl], "batch": wl.B, "context": wl.L,
           "new_tokens": wl.T, "steps": steps, "warmup": warmup, "ms_per_step": round(ms, 5),
           "value": round(wl.B * wl.T / (ms / 1e3), 2), "unit": unit,
           "step_roofline": step_roofline(wl, ms, peaks), "gpu_launches_per_step": launches / steps,
           "stage_ms": stage_ms,
           "clocks": clocks,
           "l2": ("flushed before every step (256 MiB written, 256 MiB read; outside the step's events); "
                  "the step's own events, mean over steps") if flush else
                 "inputs larger than L2; steps back to back"}
    del layers
    if flush:
        del fw, fr
    torch.cuda.empty_cache()
    return rec


def workload_config(wl):
    """The ``config`` object of a bench line (both arms)."""
    layers_wl = [wl.layer("csa"), wl.layer("hca")] if wl.kind == "pair" else [wl]
    nbytes, _ = step_work(wl)
    return {"workload": wl.name, "layers": [lw.name for lw in layers_wl], "batch_per_gpu": wl.B,
            "context": wl.L, "new_tokens": wl.T, "heads": wl.H, "kv_dim": wl.D, "top_k": wl.k, "window": wl.w,
            "csa_entries": wl.L // wl.m, "hca_entries": wl.L // wl.m_hca if wl.kind == "pair" else None,
            "l2": ("inputs larger than L2 (working set per step > 126 MB)" if nbytes > 2 * L2_BYTES
                   else "working set fits in L2")}


def run_lcsc(args):
    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    L.load()
    wl = workloads.ALL[args.workload]
    layers_wl = [wl.layer("csa"), wl.layer("hca")] if wl.kind == "pair" else [wl]
    layers = [Layer(lw, shard_seed(rank, i), dev) for i, lw in enumerate(layers_wl)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    runner = StepRunner(layers, stream)
    step = runner.run

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for ly in layers:
        if int(ly.status.item()) != 0:
            raise RuntimeError(f"device status {int(ly.status.item())} in {ly.wl.name}")

    # ---- timed region: K steps, inputs resident in HBM (working set > L2).
    # The only events recorded inside it are the two around each step's
    # scoring launch (the dominant kernel's duration, on the stream it runs
    # on); the other stage boundaries are timed in a separate pass below,
    # since their events add to the step time.
    csa = layers[0] if layers[0].wl.kind == "csa" else None
    hca = next((ly for ly in layers if ly.wl.kind == "hca"), None)

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)  # creates the event
        return evs

    score_ev = [new_events(2) for _ in range(args.steps)]
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    t0 = time.time()
    launches0 = L.kernel_launches()
    start.record(stream)
    for i in range(args.steps):
        if csa is not None:
            csa.set_events([None, None] + score_ev[i])
        step()
    stop.record(stream)
    launches = L.kernel_launches() - launches0
    torch.cuda.synchronize()
    barrier(ws)
    t1 = time.time()
    time.sleep(0.25)
    clocks = sampler.stop(t0, t1)
    ms_total = max_over_ranks(ws, start.elapsed_time(stop))
    ms_step = ms_total / args.steps
    value = job_throughput(wl.B, wl.T, ws, args.steps, ms_total)
    score_ms = float(np.mean([a.elapsed_time(b) for a, b in score_ev])) if csa is not None else None

    # ---- stage pass (untimed for the line's value): every stage boundary
    n_stage = min(args.steps, 20)
    events = [new_events(6) for _ in range(n_stage)]
    hevents = [new_events(3) for _ in range(n_stage)]
    torch.cuda.synchronize()
    for i in range(n_stage):
        if csa is not None:
            csa.set_events(events[i])
        if hca is not None:
            hca.set_events(hevents[i])
        step()
    torch.cuda.synchronize()
    for ly in (csa, hca):
        if ly is not None:
            ly.clear_events()
    hca_ms = None
    if hca is not None:
        hca_ms = {name: round(float(np.mean([evs[a].elapsed_time(evs[b]) for evs in hevents])), 4)
                  for name, a, b in (("compress", 0, 1), ("dense_attn", 1, 2))}

    # ---- dominant kernel: the CSA indexer scoring (events 2 -> 3 of each step)
    roof = None
    if csa is not None:
        stage_ms = {name: float(np.mean([evs[a].elapsed_time(evs[b]) for evs in events]))
                    for name, a, b in (("idx_compress", 0, 1), ("quantize_join", 1, 2), ("index_score", 2, 3),
                                       ("topk", 3, 4), ("kv_join_sparse_attn", 4, 5))}
        cw = csa.wl
        peaks = measured_peaks()
        sha = source_sha("indexer_mma.cu", "topk.cuh", "sm100.cuh", "common.cuh", "kernels.cuh")
        traffic = recorded_traffic("index_mma_kernel", wl.name, sha)
        common = {"kernel": "index_mma_kernel (tensor-core indexer scoring)", "traffic": traffic,
                  "ms_per_launch": round(score_ms, 4),
                  "ms_per_launch_source": "events around the scoring launch of every timed step, on its stream",
                  "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()}, "hca_stage_ms": hca_ms,
                  "stage_ms_source": f"a separate pass of {n_stage} steps with every stage event recorded"}
        if cw.T > 1:
            # chunked prefill: the scoring is a contraction of T queries x 64 heads
            # against every visible key; it is bound by the tensor pipe, whose
            # rate for the key format is the measured burst bf16 rate x the
            # nominal ratio (the launch lasts milliseconds, not seconds)
            n_vis = sum((cw.L - cw.T + t + 1) // cw.m for t in range(cw.T))
            flops = cw.B * n_vis * 2 * cw.H_I * cw.d_I
            ratio = TENSOR_RATIO.get(cw.idx_fmt, 1.0)
            peak = float(peaks["bf16_tflops"]) * ratio
            achieved = flops / (score_ms / 1e3) / 1e12
            roof = dict(bound="tensor", achieved=round(achieved, 1), peak=round(peak, 1), unit="TFLOP/s",
                        frac=round(achieved / peak, 4), algorithmic_flops=flops,
                        peak_source=f"{peaks['source']} bf16_tflops (burst) x {ratio:g} ({cw.idx_fmt} / bf16 nominal)",
                        **common)
        else:
            key_b = L.row_bytes(cw.idx_fmt, cw.d_I) + (cw.d_I // 16 if cw.idx_fmt == "fp4" else 4)
            n_keys = cw.B * cw.n_entries()
            q_b = cw.B * cw.T * cw.H_I * (key_b + 4)  # quantised query rows + head weights
            alg_bytes = n_keys * (key_b + 4) + q_b  # keys read + scores written + queries
            peak = float(peaks["hbm_gbs"])
            achieved = alg_bytes / (score_ms / 1e3) / 1e9
            roof = dict(bound="hbm", achieved=round(achieved, 1), peak=peak, unit="GB/s",
                        frac=round(achieved / peak, 4), algorithmic_bytes=alg_bytes,
                        peak_source=peaks["source"] + " hbm_gbs", **common)

    # ---- end to end: pinned host inputs -> device, step, output -> host.
    # Every step copies the inputs of its new tokens in and its outputs out,
    # through two sets of per-step device buffers used in turn: step s+1's
    # inputs upload (one copy stream) while step s computes, and step s's
    # outputs download (a second copy stream) while step s+1 computes.  A
    # slot's inputs are overwritten only after the step two back that read
    # them is done, its outputs only after they were downloaded.
    e2e = None
    if args.e2e_steps > 0:
        slots = [[ly.io_slot() for ly in layers] for _ in range(2)]  # [slot][layer]
        h2d = sum(h.numel() * h.element_size() for _, ins, _ in slots[0] for _, h in ins)
        d2h = sum(h.numel() * h.element_size() for _, _, (_, h) in slots[0])
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        nl = len(layers)
        up_ev = [[torch.cuda.Event() for _ in layers] for _ in range(2)]     # inputs in
        done_ev = [[torch.cuda.Event() for _ in layers] for _ in range(2)]   # step computed
        down_ev = [[torch.cuda.Event() for _ in layers] for _ in range(2)]   # outputs out
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        order = list(range(nl))[::-1] if runner.hca_first else list(range(nl))
        saved = [ly.step for ly in layers]
        used = [False, False]

        def e2e_step(s):
            k = s % 2
            with torch.cuda.stream(up):
                for i in order:
                    if used[k]:
                        up.wait_event(done_ev[k][i])  # the step two back has read this slot's inputs
                    for d, h in slots[k][i][1]:
                        d.copy_(h, non_blocking=True)
                    up_ev[k][i].record(up)
            for i in range(nl):
                layers[i].step = slots[k][i][0]

            def before(i, st):
                st.wait_event(up_ev[k][i])
                if used[k]:
                    st.wait_event(down_ev[k][i])  # this slot's last outputs are out

            runner.run(before=before)
            for i in order:
                done_ev[k][i].record(runner.streams[i])
                down.wait_event(done_ev[k][i])
                with torch.cuda.stream(down):
                    out_d, out_h = slots[k][i][2]
                    out_h.copy_(out_d, non_blocking=True)
                    down_ev[k][i].record(down)
            used[k] = True

        up.wait_stream(stream)
        down.wait_stream(stream)
        for s in range(max(args.warmup, 2)):  # untimed: first copies through the pinned buffers
            e2e_step(s)
        stream.wait_stream(up)
        stream.wait_stream(down)
        barrier(ws)
        torch.cuda.synchronize()
        e0.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        for s in range(args.e2e_steps):
            e2e_step(s)
        stream.wait_stream(up)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        for ly, st in zip(layers, saved):
            ly.step = st
        e2e_ms = max_over_ranks(ws, e0.elapsed_time(e1))
        e2e = {"value": round(job_throughput(wl.B, wl.T, ws, args.e2e_steps, e2e_ms), 2), "unit": "queries/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "pinned host buffers, two sets of per-step device buffers used in turn: step s+1's "
                         "inputs upload on one copy stream while step s computes, step s's outputs download on a "
                         "second while step s+1 computes; per layer and step one copy of the dense inputs "
                         "(queries, indexer queries and weights, lengths in one buffer), one of each layer's raw "
                         "rows and one of the output; every step's uploads and downloads are inside the timed "
                         "region, which ends when the last step's outputs are on the host",
               "inputs": "per sequence and layer: the new token's raw rows, the queries, the indexer queries "
                         "and weights (CSA), the context length; the closing group's G - 1 older raw rows "
                         "stay on the device from earlier steps"}

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "queries/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": index_dtype(layers_wl) + "e4m3 x e4m3 and bf16 x bf16 MMA (attention), f32 accumulate and softmax",
        "data": "synthetic (seeded Gaussian entries with planted relevant blocks, drawn on device)",
        "config": workload_config(wl),
        "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
    }
    line["step_roofline"] = step_roofline(wl, ms_step, measured_peaks())
    if args.sub_records and ws == 1 and wl.name == DEFAULT_WORKLOAD:
        line["sub_records"] = [measure_sub(n, dev, measured_peaks(), args.warmup) for n in SUB_WORKLOADS]
    if args.cpu_baseline and ws == 1:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_queries)
    return line


# ------------------------------------------------------- CPU oracle legs

def oracle_sequence(wl_layer, b, seed):
    """Oracle state of one sequence (test-infrastructure oracle, CPU)."""
    from oracle import storage
    P = synth.layer_params(wl_layer, seed)
    inp = synth.sequence_inputs(wl_layer, b, seed)
    n_cap = wl_layer.L // wl_layer.m + 1
    rope = wl_layer.rope_dim if wl_layer.kv_fmt == "kv" else 0

    def stored(vals, fmt, r):
        st = storage.encode(fmt, vals, r)
        pay = np.zeros((n_cap,) + st.payload.shape[1:], st.payload.dtype)
        pay[:vals.shape[0]] = st.payload
        sc = None
        if st.scale is not None:
            sc = np.zeros((n_cap,) + st.scale.shape[1:], st.scale.dtype)
            sc[:vals.shape[0]] = st.scale
        return storage.Stored(fmt, pay, sc, vals.shape[1], r)

    kv = stored(inp.pop("e_kv"), wl_layer.kv_fmt, rope)
    idx = stored(inp.pop("e_idx"), wl_layer.idx_fmt, 0) if wl_layer.kind == "csa" else None
    cap = wl_layer.win_cap
    R = synth.tail_rows(wl_layer)
    ring = storage.encode(wl_layer.kv_fmt, np.zeros((cap, wl_layer.D), np.float32), rope)
    for pos in range(max(0, wl_layer.L - wl_layer.T - wl_layer.w + 1), wl_layer.L - wl_layer.T):
        one = storage.encode(wl_layer.kv_fmt, inp["x_kv"][pos - (wl_layer.L - R)][None], rope)
        ring.payload[pos % cap] = one.payload[0]
        if ring.scale is not None:
            ring.scale[pos % cap] = one.scale[0]
    return P, inp, kv, idx, ring


def oracle_step(wl_layer, P, inp, kv, idx, ring):
    from oracle.step import layer_step
    w = wl_layer
    tail = lambda a: None if a is None else a[a.shape[0] - (w.T + w.G - 1):]
    return layer_step(w.kind, m=w.m, G=w.G, w=w.w, k=w.k, sm_scale=w.sm_scale, kv_fmt=w.kv_fmt,
                      rope_dim=w.rope_dim, idx_fmt=w.idx_fmt, L=w.L, T=w.T, kv=kv, v=None, idx=idx,
                      ring_kv=ring, ring_v=None, x_kv=tail(inp["x_kv"]), x_v=None,
                      x_idx=tail(inp.get("x_idx")), W_kv=P["W_kv"], B_kv=P["B_kv"], W_v=None, B_v=None,
                      W_idx=P.get("W_idx"), B_idx=P.get("B_idx"), q=inp["q"], q_idx=inp.get("q_idx"),
                      w_idx=inp.get("w_idx"), sink=P["sink"], out_rope_base=w.out_rope_base)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, n_queries):
    """The oracle, as it stands, on a bounded sample: ``n_queries`` decode
    queries of sequence 0 through every layer of the workload."""
    layers_wl = [wl.layer("csa"), wl.layer("hca")] if wl.kind == "pair" else [wl]
    states = [oracle_sequence(lw.with_(B=1), 0, synth.SEED) for lw in layers_wl]
    t0 = time.perf_counter()
    for _ in range(n_queries):
        for lw, st in zip(layers_wl, states):
            oracle_step(lw.with_(B=1), *st)
    dt = time.perf_counter() - t0
    return {"value": round(n_queries * wl.T / dt, 5), "unit": "queries/s", "cores": blas_threads(),
            "kind": "oracle", "cpu": _cpu_model(),
            "sample": f"{n_queries} decode step(s) of 1 sequence (T={wl.T}) through "
                      f"{'+'.join(x.name for x in layers_wl)}, full context, fp64 numpy oracle"}


def _cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


REFERENCE_BUDGET_S = 120.0


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    wl = workloads.ALL[args.workload]
    layers_wl = [wl.layer("csa"), wl.layer("hca")] if wl.kind == "pair" else [wl]
    states = [oracle_sequence(lw.with_(B=1), 0, synth.SEED) for lw in layers_wl]
    t_warm = []
    for _ in range(args.warmup):
        tw = time.perf_counter()
        for lw, st in zip(layers_wl, states):
            oracle_step(lw.with_(B=1), *st)
        t_warm.append(time.perf_counter() - tw)
    # A step of the oracle takes seconds: the timed steps are capped so the
    # run stays within a few minutes (the line reports how many ran).
    steps = max(1, min(args.steps, int(REFERENCE_BUDGET_S / max(min(t_warm), 1e-6))))
    t0 = time.perf_counter()
    for _ in range(steps):
        for lw, st in zip(layers_wl, states):
            oracle_step(lw.with_(B=1), *st)
    dt = time.perf_counter() - t0
    value = steps * wl.T / dt
    sample = (f"each step: 1 decode query of 1 sequence (of {wl.B}) through "
              f"{'+'.join(x.name for x in layers_wl)} at full context; {steps} of the {args.steps} "
              f"requested steps timed (capped at ~{REFERENCE_BUDGET_S:.0f} s)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "queries/s", "n_gpus": ws,
        "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, numpy generator)",
        "config": workload_config(wl),
        "cpu_baseline": {"value": round(value, 5), "unit": "queries/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.ALL))
    ap.add_argument("--impl", default="lcsc", choices=["lcsc", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-sub-records", dest="sub_records", action="store_false",
                    help="skip the 1M pair at B = 1, the 128K decode and the prefill step timed after the main line")
    ap.add_argument("--cpu-queries", type=int, default=2)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    line = run_reference(args) if args.impl == "reference" else run_lcsc(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and args.impl != "reference":
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
