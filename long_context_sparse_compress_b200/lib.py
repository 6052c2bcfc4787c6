"""ctypes binding of liblcsc.so (include/lcsc.h): argument marshalling only.

Every computation happens in the CUDA library.  ``load()`` raises when the
library is missing or was built for another ABI: there is no fallback.
Tensors are torch device tensors; pointers are passed as integers.
"""
import ctypes
import os

import torch

from . import workloads

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblcsc.so")
ABI_VERSION = 3

FMT = {"f32": 0, "kv": 1, "fp8": 2, "fp4": 3}
DT = {"f32": 0, "bf16": 1}
TENSOR = {"kv": 0, "v": 1, "idx": 2}
SINK = {"logit": 0, "token": 1}
GATE = {"proj": 0, "logits": 1}
DEV_BAD_INDEX = 1
DEV_BAD_LENGTH = 2
DEV_TIMEOUT = 4
DEV_RANGE = 8

c_i32, c_i64, c_f32, c_vp, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class Params(ctypes.Structure):
    _fields_ = [("m", c_i32), ("group_len", c_i32), ("window", c_i32), ("top_k", c_i32),
                ("sm_scale", c_f32), ("n_heads", c_i32), ("head_dim", c_i32), ("rope_dim", c_i32),
                ("v_dim", c_i32), ("idx_heads", c_i32), ("idx_dim", c_i32), ("kv_format", c_i32),
                ("idx_format", c_i32), ("x_dtype", c_i32), ("q_dtype", c_i32),
                ("out_rope_dim", c_i32), ("out_rope_base", c_f32), ("sink_mode", c_i32),
                ("gate_src", c_i32)]


class Cache(ctypes.Structure):
    _fields_ = [("data", c_vp), ("scale", c_vp), ("capacity", c_i64), ("row0", c_i64), ("rows", c_i64)]


class Step(ctypes.Structure):
    _fields_ = [("B", c_i64), ("T", c_i64), ("n_max", c_i64), ("ctx_len", c_vp),
                ("x_kv", c_vp), ("x_v", c_vp), ("x_idx", c_vp),
                ("w_kv", c_vp), ("b_kv", c_vp), ("w_v", c_vp), ("b_v", c_vp),
                ("w_idx", c_vp), ("b_idx", c_vp),
                ("kv", Cache), ("v", Cache), ("idx_keys", Cache), ("win_kv", Cache), ("win_v", Cache),
                ("q", c_vp), ("q_idx", c_vp), ("w_heads", c_vp), ("sink", c_vp),
                ("out", c_vp), ("lse", c_vp), ("out_idx", c_vp), ("out_score", c_vp),
                ("events", ctypes.POINTER(c_vp)), ("n_events", c_i32), ("sink_kv", Cache),
                ("sink_v", Cache)]


_SIGS = {
    "lcsc_abi_version": (c_i32, []),
    "lcsc_last_cuda_error": (c_i32, []),
    "lcsc_status_string": (ctypes.c_char_p, [c_i32]),
    "lcsc_kernel_launches": (ctypes.c_uint64, []),
    "lcsc_set_wait_test": (c_i32, [c_i64, c_i32]),
    "lcsc_row_bytes": (c_i64, [c_i32, c_i32, c_i32]),
    "lcsc_compress_workspace_size": (c_i32, [c_vp, c_i64, c_i64, c_vp]),
    "lcsc_csa_compress": (c_i32, [c_vp, c_i32, c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp,
                                  c_vp, c_sz, c_vp, c_vp]),
    "lcsc_hca_compress": (c_i32, [c_vp, c_i32, c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp,
                                  c_vp, c_sz, c_vp, c_vp]),
    "lcsc_encode_rows": (c_i32, [c_vp, c_i32, c_vp, c_i64, c_i64, c_i64, c_vp, c_vp]),
    "lcsc_index_topk_workspace_size": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp]),
    "lcsc_csa_index_topk": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_vp, c_vp,
                                    c_vp, c_sz, c_vp, c_vp]),
    "lcsc_csa_index_topk_noalloc": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_vp,
                                            c_vp, c_vp, c_vp]),
    "lcsc_attn_workspace_size": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_i32, c_vp]),
    "lcsc_csa_sparse_attn": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_i64, c_i64, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "lcsc_hca_dense_attn": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64,
                                    c_i64, c_i64, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "lcsc_step_workspace_size": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, c_vp]),
    "lcsc_csa_decode": (c_i32, [c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "lcsc_hca_decode": (c_i32, [c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "lcsc_topk_merge": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp]),
    "lcsc_attn_merge": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp]),
}

EXPORTS = tuple(_SIGS)
_lib = None


class LcscError(RuntimeError):
    pass


def load(path=LIB_PATH):
    """Load the library (once).  Raises if it is missing: nothing runs without it."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise LcscError(f"{path} is missing: build it with `python -m long_context_sparse_compress_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if lib.lcsc_abi_version() != ABI_VERSION:
        raise LcscError("liblcsc.so ABI version mismatch: rebuild it")
    _lib = lib
    return lib


def kernel_launches():
    """Kernels the library has enqueued since it was loaded (host-side count)."""
    return int(load().lcsc_kernel_launches())


def set_wait_test(limit_ns=0, stall=False):
    """Bounded-wait limit of the tensor-core kernels and the stall of one
    thread per CTA, for tests of the failure path; (0, False) restores the
    normal behaviour."""
    check(load().lcsc_set_wait_test(int(limit_ns), 1 if stall else 0))


def check(status):
    if status != 0:
        lib = load()
        msg = lib.lcsc_status_string(status).decode()
        if status == 3:
            msg += f" (cudaError {lib.lcsc_last_cuda_error()})"
        raise LcscError(f"lcsc call failed: {msg}")


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def ref(s):
    return None if s is None else ctypes.byref(s)


def stream_handle(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def params(wl):
    """lcsc_params of a single-layer workload."""
    return Params(m=wl.m, group_len=wl.G, window=wl.w, top_k=wl.k if wl.kind == "csa" else 0,
                  sm_scale=wl.sm_scale, n_heads=wl.H, head_dim=wl.D,
                  rope_dim=wl.rope_dim if wl.kv_fmt == "kv" else 0, v_dim=wl.Dv, idx_heads=wl.H_I,
                  idx_dim=wl.d_I, kv_format=FMT[wl.kv_fmt], idx_format=FMT[wl.idx_fmt],
                  x_dtype=DT[wl.x_dtype], q_dtype=DT[wl.q_dtype],
                  out_rope_dim=wl.rope_dim if wl.out_rope_base > 0 else 0, out_rope_base=wl.out_rope_base,
                  sink_mode=SINK[wl.sink_mode], gate_src=GATE[wl.gate_src])


def row_bytes(fmt, dim, rope=0):
    return {"f32": 4 * dim, "kv": dim + rope, "fp8": dim, "fp4": dim // 2}[fmt]


def round_capacity(n, fmt):
    """Rows to allocate for n rows: indexer keys in FP8 / FP4 need a multiple of 128."""
    return (n + 127) // 128 * 128 if fmt in ("fp8", "fp4") else n


def fp4_scale_index(capacity, dim):
    """Position, in the tiled FP4 scale array of one sequence, of the block
    scale (row r, block k): the layout include/lcsc.h documents.  Returns an
    int array [capacity, dim // 16]."""
    r = torch.arange(capacity).view(-1, 1)
    k = torch.arange(dim // 16).view(1, -1)
    m = r % 128
    return ((r // 128) * (dim // 64) * 512 + (k // 4) * 512 + (m % 32) * 16 + (m // 32) * 4 + (k % 4))


class DeviceCache:
    """Stored rows of one tensor for B sequences, in device memory.  An entry
    shard (``rows`` > 0) holds the entries row0 .. row0 + rows - 1 in its
    rows 0 .. rows - 1."""

    def __init__(self, B, capacity, fmt, dim, rope=0, device="cuda", row0=0, rows=0):
        self.B, self.capacity, self.fmt, self.dim, self.rope = B, capacity, fmt, dim, rope
        self.row0, self.rows = row0, rows
        if fmt == "f32":
            self.data = torch.zeros((B, capacity, dim), dtype=torch.float32, device=device)
            self.scale = None
        else:
            self.data = torch.zeros((B, capacity, row_bytes(fmt, dim, rope)), dtype=torch.uint8, device=device)
            if fmt == "fp4":
                tiles = (capacity + 127) // 128
                self.scale = torch.zeros((B, tiles * (dim // 64) * 512), dtype=torch.uint8, device=device)
            else:
                self.scale = torch.ones((B, capacity), dtype=torch.float32, device=device)

    def set_rows(self, b, payload, scale=None, row0=0):
        """Copy stored rows (host arrays: payload [n, row], scale [n] or, for
        FP4, [n, dim / 16] row-major block scales) into sequence b."""
        n = payload.shape[0]
        self.data[b, row0:row0 + n] = torch.as_tensor(payload).to(self.data.device)
        if self.scale is None:
            return
        sc = torch.as_tensor(scale).to(self.scale.device)
        if self.fmt == "fp4":
            idx = fp4_scale_index(self.capacity, self.dim)[row0:row0 + n].to(self.scale.device)
            self.scale[b].view(-1)[idx.reshape(-1)] = sc.reshape(-1)
        else:
            self.scale[b, row0:row0 + n] = sc

    def get_rows(self, b):
        """(payload, scale) of sequence b on the host, FP4 scales as [capacity, dim / 16]."""
        d = self.data[b].cpu().numpy()
        if self.scale is None:
            return d, None
        if self.fmt == "fp4":
            idx = fp4_scale_index(self.capacity, self.dim).to(self.scale.device)
            return d, self.scale[b][idx].cpu().numpy()
        return d, self.scale[b].cpu().numpy()

    def c(self):
        return Cache(data=self.data.data_ptr(), scale=None if self.scale is None else self.scale.data_ptr(),
                     capacity=self.capacity, row0=self.row0, rows=self.rows)

    def seq(self, b):
        """A one-sequence view (sequence b) usable wherever a cache is."""
        return _SeqView(self, b)


class _SeqView:
    def __init__(self, cache, b):
        self.cache, self.b, self.capacity = cache, b, cache.capacity

    def c(self):
        c = self.cache
        return Cache(data=c.data[self.b].data_ptr(),
                     scale=None if c.scale is None else c.scale[self.b].data_ptr(), capacity=c.capacity,
                     row0=c.row0, rows=c.rows)


def null_cache():
    return Cache(data=None, scale=None, capacity=0)


# ------------------------------------------------------------------ calls

def _ws_size(fn, *args):
    out = c_sz(0)
    check(fn(*args, ctypes.byref(out)))
    return out.value


def workspace(nbytes, device="cuda"):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def compress(p, tensor, x, B, tok_begin, tok_end, w, bpos, entries, window=None, status=None,
             hca=False, stream=None):
    lib = load()
    n_tok = tok_end - tok_begin
    ws = workspace(_ws_size(lib.lcsc_compress_workspace_size, ctypes.byref(p), B, n_tok), x.device)
    fn = lib.lcsc_hca_compress if hca else lib.lcsc_csa_compress
    win = window.c() if window is not None else None
    check(fn(ctypes.byref(p), TENSOR[tensor], ptr(x), B, tok_begin, tok_end, ptr(w), ptr(bpos),
             ctypes.byref(entries.c()), ref(win), ptr(ws), ws.numel(), ptr(status), stream_handle(stream)))
    return ws


def encode_rows(p, tensor, rows, row0, out, stream=None):
    lib = load()
    B, n = rows.shape[0], rows.shape[1]
    check(lib.lcsc_encode_rows(ctypes.byref(p), TENSOR[tensor], ptr(rows), B, n, row0,
                               ctypes.byref(out.c()), stream_handle(stream)))


def index_topk_workspace(p, B, T, n_max):
    return _ws_size(load().lcsc_index_topk_workspace_size, ctypes.byref(p), B, T, n_max)


def index_topk(p, q_idx, w_idx, keys, ctx_len, n_max, out_idx, out_score=None, ws=None, status=None,
               stream=None):
    lib = load()
    B, T = q_idx.shape[0], q_idx.shape[1]
    if ws is None:
        ws = workspace(index_topk_workspace(p, B, T, n_max), q_idx.device)
    check(lib.lcsc_csa_index_topk(ctypes.byref(p), ptr(q_idx), ptr(w_idx), ctypes.byref(keys.c()),
                                  ptr(ctx_len), B, T, n_max, ptr(out_idx), ptr(out_score), ptr(ws),
                                  ws.numel(), ptr(status), stream_handle(stream)))
    return ws


NOALLOC_SCRATCH_BYTES = 40 << 20


def index_topk_noalloc(p, q_idx, w_idx, keys, ctx_len, n_max, out_idx, out_score=None, status=None,
                       stream=None):
    """lcsc_csa_index_topk_noalloc: same results, no workspace argument; the
    library's fixed scratch is used (one call at a time per device)."""
    lib = load()
    B, T = q_idx.shape[0], q_idx.shape[1]
    check(lib.lcsc_csa_index_topk_noalloc(ctypes.byref(p), ptr(q_idx), ptr(w_idx), ctypes.byref(keys.c()),
                                          ptr(ctx_len), B, T, n_max, ptr(out_idx), ptr(out_score),
                                          ptr(status), stream_handle(stream)))


def attn_workspace(p, B, T, n_max, dense):
    return _ws_size(load().lcsc_attn_workspace_size, ctypes.byref(p), B, T, n_max, int(dense))


def _cref(c):
    return ref(c.c() if c is not None else None)


def sparse_attn(p, q, kv, v, win_kv, win_v, idx, sink, ctx_len, out, lse=None, ws=None, status=None,
                stream=None, sink_kv=None, sink_v=None):
    lib = load()
    B, T = q.shape[0], q.shape[1]
    if ws is None:
        ws = workspace(attn_workspace(p, B, T, kv.capacity, False), q.device)
    check(lib.lcsc_csa_sparse_attn(
        ctypes.byref(p), ptr(q), ctypes.byref(kv.c()), _cref(v), ctypes.byref(win_kv.c()), _cref(win_v),
        ptr(idx), ptr(sink), _cref(sink_kv), _cref(sink_v), ptr(ctx_len), B, T, ptr(out), ptr(lse), ptr(ws),
        ws.numel(), ptr(status), stream_handle(stream)))
    return ws


def dense_attn(p, q, kv, v, win_kv, win_v, sink, ctx_len, n_max, out, lse=None, ws=None, status=None,
               stream=None, sink_kv=None, sink_v=None):
    lib = load()
    B, T = q.shape[0], q.shape[1]
    if ws is None:
        ws = workspace(attn_workspace(p, B, T, n_max, True), q.device)
    check(lib.lcsc_hca_dense_attn(
        ctypes.byref(p), ptr(q), ctypes.byref(kv.c()), _cref(v), ctypes.byref(win_kv.c()), _cref(win_v),
        ptr(sink), _cref(sink_kv), _cref(sink_v), ptr(ctx_len), B, T, n_max, ptr(out), ptr(lse), ptr(ws),
        ws.numel(), ptr(status), stream_handle(stream)))
    return ws


def step_workspace(p, csa, B, T, n_max):
    return _ws_size(load().lcsc_step_workspace_size, ctypes.byref(p), int(csa), B, T, n_max)


def make_step(B, T, n_max, ctx_len, x_kv, x_v, x_idx, w_kv, b_kv, w_v, b_v, w_idx, b_idx, kv, v, idx_keys,
              win_kv, win_v, q, q_idx, w_heads, sink, out, lse=None, out_idx=None, out_score=None,
              sink_kv=None, sink_v=None):
    """An lcsc_step struct over device tensors / caches (None -> NULL).
    With gate logits (gate_src "logits") w_kv / w_v / w_idx are the float32
    logit rows; with a sink token, sink_kv / sink_v are the one-row caches of
    position 0."""
    cc = lambda c: c.c() if c is not None else null_cache()
    s = Step(B=B, T=T, n_max=n_max)
    for name, t in dict(ctx_len=ctx_len, x_kv=x_kv, x_v=x_v, x_idx=x_idx, w_kv=w_kv, b_kv=b_kv, w_v=w_v,
                        b_v=b_v, w_idx=w_idx, b_idx=b_idx, q=q, q_idx=q_idx, w_heads=w_heads, sink=sink,
                        out=out, lse=lse, out_idx=out_idx, out_score=out_score).items():
        setattr(s, name, None if t is None else t.data_ptr())
    s.kv, s.v, s.idx_keys, s.win_kv, s.win_v = cc(kv), cc(v), cc(idx_keys), cc(win_kv), cc(win_v)
    s.sink_kv, s.sink_v = cc(sink_kv), cc(sink_v)
    return s


def set_step_events(step, events):
    """Attach stage-boundary events (torch.cuda.Event, already created; None
    for a boundary not to record) to a step struct; the returned array must
    outlive the call."""
    arr = (c_vp * len(events))(*[None if e is None else e.cuda_event for e in events])
    step.events = ctypes.cast(arr, ctypes.POINTER(c_vp))
    step.n_events = len(events)
    return arr


def decode_step(p, step, csa, ws, status=None, stream=None):
    lib = load()
    fn = lib.lcsc_csa_decode if csa else lib.lcsc_hca_decode
    check(fn(ctypes.byref(p), ctypes.byref(step), ptr(ws), ws.numel(), ptr(status), stream_handle(stream)))


def topk_merge(p, part_idx, part_score, out_idx, out_score=None, stream=None):
    """lcsc_topk_merge: parts [n][B][T][k] -> the top-k over all of them."""
    n, B, T = part_idx.shape[0], part_idx.shape[1], part_idx.shape[2]
    check(load().lcsc_topk_merge(ctypes.byref(p), n, ptr(part_idx), ptr(part_score), B, T, ptr(out_idx),
                                 ptr(out_score), stream_handle(stream)))


def attn_merge(p, part_out, part_lse, sink, ctx_len, out, lse=None, stream=None):
    """lcsc_attn_merge: parts [n][B][T][H][Dv] (+ lse [n][B][T][H]) -> one output."""
    n, B, T = part_out.shape[0], part_out.shape[1], part_out.shape[2]
    check(load().lcsc_attn_merge(ctypes.byref(p), n, ptr(part_out), ptr(part_lse), ptr(sink), ptr(ctx_len), B, T,
                                 ptr(out), ptr(lse), stream_handle(stream)))


__all__ = ["load", "params", "DeviceCache", "compress", "encode_rows", "index_topk", "sparse_attn",
           "dense_attn", "make_step", "decode_step", "workloads"]
