// The C ABI (include/lcsc.h): argument validation, workspace planning and
// the launch sequence of every call.  No device memory is allocated here.
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "kernels.cuh"
#include "launches.h"

namespace lcsc {

std::atomic<uint64_t> g_kernel_launches{0};

void note_launch() { g_kernel_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {
std::atomic<int64_t> g_wait_limit_ns{0};
std::atomic<int32_t> g_wait_stall{0};
}  // namespace

void set_wait_test(int64_t limit_ns, int32_t stall) {
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  g_wait_stall.store(stall, std::memory_order_relaxed);
}

WaitTest wait_test() {
  const int64_t l = g_wait_limit_ns.load(std::memory_order_relaxed);
  return WaitTest{l > 0 ? (uint64_t)l : kDefaultWaitNs, g_wait_stall.load(std::memory_order_relaxed) != 0};
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("LCSC_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

namespace {

thread_local int32_t g_last_cuda_error = 0;

int32_t cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int32_t)e;
  return LCSC_ERR_CUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Bump allocator over the caller's workspace.
struct Carve {
  uint8_t* base;
  size_t used = 0;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += align_up(sizeof(T) * count);
    return p;
  }
};

bool valid_format(int fmt) { return fmt >= LCSC_FMT_F32 && fmt <= LCSC_FMT_FP4; }

int32_t check_params(const lcsc_params* p) {
  if (!p) return LCSC_ERR_INVALID_ARG;
  if (p->m < 1 || p->group_len < p->m || p->group_len > 2 * p->m) return LCSC_ERR_INVALID_ARG;
  if (p->window < 0 || p->top_k < 0 || p->top_k > 2048) return LCSC_ERR_INVALID_ARG;
  if (p->n_heads < 1 || p->head_dim < 1 || p->v_dim < 1) return LCSC_ERR_INVALID_ARG;
  if (p->rope_dim < 0 || p->rope_dim > p->head_dim) return LCSC_ERR_INVALID_ARG;
  if (!valid_format(p->kv_format) || !valid_format(p->idx_format)) return LCSC_ERR_INVALID_ARG;
  if (p->kv_format != LCSC_FMT_F32 && p->kv_format != LCSC_FMT_KV) return LCSC_ERR_INVALID_ARG;
  if (p->idx_format == LCSC_FMT_KV) return LCSC_ERR_INVALID_ARG;
  if (p->x_dtype != LCSC_DT_F32 && p->x_dtype != LCSC_DT_BF16) return LCSC_ERR_INVALID_ARG;
  if (p->q_dtype != LCSC_DT_F32 && p->q_dtype != LCSC_DT_BF16) return LCSC_ERR_INVALID_ARG;
  if (!(p->sm_scale > 0.f) || p->sm_scale == INFINITY) return LCSC_ERR_INVALID_ARG;
  if (p->sink_mode != LCSC_SINK_LOGIT && p->sink_mode != LCSC_SINK_TOKEN) return LCSC_ERR_INVALID_ARG;
  if (p->gate_src != LCSC_GATE_PROJ && p->gate_src != LCSC_GATE_LOGITS) return LCSC_ERR_INVALID_ARG;
  if (!(p->out_rope_base >= 0.f) || p->out_rope_base == INFINITY) return LCSC_ERR_INVALID_ARG;
  if (p->out_rope_base > 0.f &&
      (p->out_rope_dim < 4 || p->out_rope_dim % 4 != 0 || p->out_rope_dim > p->v_dim))
    return LCSC_ERR_INVALID_ARG;
  return LCSC_OK;
}

// The (format, dim) pairs the kernels are built for.
bool kv_supported(const lcsc_params* p) {
  if (p->kv_format == LCSC_FMT_F32) return p->head_dim == 128 && p->v_dim == 128 && p->n_heads % 8 == 0;
  return p->head_dim == 512 && p->v_dim == 512 && p->rope_dim % 16 == 0 && p->n_heads % 16 == 0;
}

bool idx_supported(const lcsc_params* p) {
  if (p->idx_format == LCSC_FMT_F32) return p->idx_dim == 32 && p->idx_heads == 4;
  return (p->idx_format == LCSC_FMT_FP8 || p->idx_format == LCSC_FMT_FP4) && p->idx_dim == 128 &&
         p->idx_heads == 64;
}

int32_t tensor_fmt(const lcsc_params* p, int32_t tensor, RowFmt* f) {
  switch (tensor) {
    case LCSC_TENSOR_KV: *f = {p->kv_format, p->head_dim, p->rope_dim, 0}; break;
    case LCSC_TENSOR_V: *f = {p->kv_format, p->v_dim, p->rope_dim, 0}; break;
    case LCSC_TENSOR_IDX: *f = {p->idx_format, p->idx_dim, 0, 0}; break;
    default: return LCSC_ERR_INVALID_ARG;
  }
  if (f->fmt != LCSC_FMT_KV) f->rope = 0;
  f->row_bytes = row_bytes_of(f->fmt, f->dim, f->rope);
  if (f->dim != 32 && f->dim != 128 && f->dim != 512) return LCSC_ERR_UNSUPPORTED;
  if (f->fmt == LCSC_FMT_KV && ((f->dim - f->rope) % (f->dim / 32) != 0)) return LCSC_ERR_UNSUPPORTED;
  if (f->fmt == LCSC_FMT_FP4 && f->dim % 16 != 0) return LCSC_ERR_UNSUPPORTED;
  return LCSC_OK;
}

// `shard_ok`: the cache may be an entry shard (rows > 0); every other cache
// must have row0 = rows = 0.
int32_t make_view(const lcsc_cache* c, const RowFmt& f, bool need_scale, CacheView* v, bool shard_ok = false) {
  if (!c || !c->data || c->capacity < 1 || !aligned16(c->data)) return LCSC_ERR_INVALID_ARG;
  if (need_scale && (!c->scale || ((uintptr_t)c->scale & 3u))) return LCSC_ERR_INVALID_ARG;
  if (c->rows < 0 || c->row0 < 0 || (c->rows == 0 && c->row0 != 0)) return LCSC_ERR_INVALID_ARG;
  if (c->rows > 0 && (!shard_ok || c->rows > c->capacity || c->row0 > ((int64_t)1 << 40)))
    return LCSC_ERR_INVALID_ARG;
  v->data = reinterpret_cast<uint8_t*>(c->data);
  v->scale = c->scale;
  v->capacity = c->capacity;
  v->f = f;
  v->row0 = c->row0;
  v->rows = c->rows;
  return LCSC_OK;
}

bool same_shard(const lcsc_cache* a, const lcsc_cache* b) { return a->row0 == b->row0 && a->rows == b->rows; }

bool needs_scale(int fmt) { return fmt != LCSC_FMT_F32; }

// ---------------------------------------------------------- workspace plans

void plan_index(const lcsc_params* p, int64_t B, int64_t T, int64_t n_max, Carve& cv,
                IndexLaunch* L) {
  const int64_t lists = B * T;
  const int64_t qrows = lists * p->idx_heads;
  const int rb = row_bytes_of(p->idx_format, p->idx_dim, 0);
  uint8_t* qdata = cv.take<uint8_t>((size_t)qrows * rb);
  void* qscale = nullptr;
  if (p->idx_format == LCSC_FMT_FP8) qscale = cv.take<float>((size_t)qrows);
  else if (p->idx_format == LCSC_FMT_FP4)  // block scales tiled by 128 rows per sequence
    qscale = cv.take<uint8_t>((size_t)B * ((T * p->idx_heads + 127) / 128) * (p->idx_dim / 64) * 512);
  const int64_t stride = (n_max + 3) / 4 * 4;
  float* scores = cv.take<float>((size_t)lists * stride);
  uint32_t* hist = cv.take<uint32_t>((size_t)lists * 2 * 4096);
  uint32_t* ctr = cv.take<uint32_t>((size_t)lists * 8);
  const int64_t cand_cap = stride < 65536 ? stride : 65536;
  uint32_t* cand = cv.take<uint32_t>((size_t)lists * 2 * cand_cap);  // (index, key) pairs
  const int64_t bit_stride = ((stride + 31) / 32 + 3) / 4 * 4;
  uint32_t* bits = cv.take<uint32_t>((size_t)lists * bit_stride);
  if (L) {
    L->q_store.data = qdata;
    L->q_store.scale = qscale;
    L->q_store.capacity = T * p->idx_heads;
    L->q_store.f = {p->idx_format, p->idx_dim, 0, rb};
    L->stride = stride;
    L->scores = scores;
    L->hist = hist;
    L->counters = ctr;
    L->cand = cand;
    L->cand_cap = cand_cap;
    L->sel_bits = bits;
    L->bit_stride = bit_stride;
  }
}

void plan_attn(const lcsc_params* p, int64_t B, int64_t T, int64_t n_max, bool dense, Carve& cv,
               AttnLaunch* L) {
  const int64_t max_rows = (dense ? n_max : p->top_k) + p->window + (p->sink_mode == LCSC_SINK_TOKEN ? 1 : 0);
  int splits, rps;
  uint8_t* q_img = nullptr;
  const bool tc = p->kv_format == LCSC_FMT_KV && p->head_dim == 512 && p->v_dim == 512 && p->n_heads == 64 &&
                  p->rope_dim == 64;
  if (tc) {
    // tensor-core path (attn_mma_supported): one CTA per (query, split) for
    // all heads, one wave; one query image per (sequence, token)
    attention_splits(max_rows, B * T, 64, sm_count(), &splits, &rps);
    q_img = cv.take<uint8_t>((size_t)B * T * kAttnQImageBytes);
  } else {
    const int hpc = p->kv_format == LCSC_FMT_F32 ? 8 : 16;
    attention_splits(max_rows, B * T * (p->n_heads / hpc), 32, 2 * sm_count(), &splits, &rps);
  }
  float* po = cv.take<float>((size_t)B * T * splits * p->n_heads * p->v_dim);
  float* pml = cv.take<float>((size_t)B * T * splits * p->n_heads * 2);
  if (L) {
    L->splits = splits;
    L->rows_per_split = rps;
    L->part_o = po;
    L->part_ml = pml;
    L->q_img = q_img;
  }
}


// Max entries one call pools per sequence.
int64_t new_entries_max(int64_t T, int m) { return T / m + 1; }

void plan_compress(const lcsc_params* p, int64_t B, int64_t n_new, int dim, Carve& cv, float** pooled) {
  float* pl = cv.take<float>((size_t)B * (n_new > 0 ? n_new : 1) * dim);
  if (pooled) *pooled = pl;
}

}  // namespace
}  // namespace lcsc

using namespace lcsc;

extern "C" {

int32_t lcsc_abi_version(void) { return LCSC_ABI_VERSION; }

int32_t lcsc_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t lcsc_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

int32_t lcsc_set_wait_test(int64_t limit_ns, int32_t stall) {
  if (limit_ns < 0) return LCSC_ERR_INVALID_ARG;
  lcsc::set_wait_test(limit_ns, stall);
  return LCSC_OK;
}

const char* lcsc_status_string(int32_t s) {
  switch (s) {
    case LCSC_OK: return "ok";
    case LCSC_ERR_INVALID_ARG: return "invalid argument";
    case LCSC_ERR_UNSUPPORTED: return "unsupported format or dimension";
    case LCSC_ERR_CUDA: return "CUDA launch error";
    case LCSC_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

int64_t lcsc_row_bytes(int32_t format, int32_t dim, int32_t rope_dim) {
  if (!valid_format(format) || dim < 1) return 0;
  return row_bytes_of(format, dim, format == LCSC_FMT_KV ? rope_dim : 0);
}

// ------------------------------------------------------------- compression

int32_t lcsc_compress_workspace_size(const lcsc_params* p, int64_t B, int64_t n_tokens,
                                     size_t* bytes) {
  int32_t st = check_params(p);
  if (st) return st;
  if (!bytes || B < 1 || n_tokens < 0) return LCSC_ERR_INVALID_ARG;
  Carve cv{nullptr};
  const int dim = p->head_dim > p->v_dim ? p->head_dim : p->v_dim;
  plan_compress(p, B, new_entries_max(n_tokens, p->m), dim > p->idx_dim ? dim : p->idx_dim, cv,
                nullptr);
  *bytes = cv.used;
  return LCSC_OK;
}

static int32_t compress_impl(const lcsc_params* p, int32_t tensor, const void* x, int64_t B,
                             int64_t tok_begin, int64_t tok_end, const void* w_gate,
                             const float* b_pos, const lcsc_cache* entries,
                             const lcsc_cache* window, void* ws, size_t ws_bytes, int32_t* status,
                             void* stream, bool hca) {
  int32_t st = check_params(p);
  if (st) return st;
  if (hca && tensor == LCSC_TENSOR_IDX) return LCSC_ERR_INVALID_ARG;
  RowFmt f;
  if ((st = tensor_fmt(p, tensor, &f))) return st;
  if (p->group_len > 128 || (p->group_len - p->m) + p->m > 128) return LCSC_ERR_UNSUPPORTED;
  if (p->x_dtype == LCSC_DT_BF16 && f.dim == 32) return LCSC_ERR_UNSUPPORTED;
  if (p->x_dtype == LCSC_DT_F32 && f.dim == 512) return LCSC_ERR_UNSUPPORTED;
  if (!x || !w_gate || !b_pos || B < 1 || B > 65535) return LCSC_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(b_pos)) return LCSC_ERR_INVALID_ARG;
  if (tok_begin < 0 || tok_end < tok_begin || tok_begin % p->m) return LCSC_ERR_INVALID_ARG;
  CompressLaunch L;
  memset(&L, 0, sizeof(L));
  if ((st = make_view(entries, f, needs_scale(f.fmt), &L.entries, true))) return st;
  if (window) {
    if (tensor == LCSC_TENSOR_IDX) return LCSC_ERR_INVALID_ARG;
    if ((st = make_view(window, f, needs_scale(f.fmt), &L.window))) return st;
  }
  const int64_t g_lo = tok_begin / p->m, g_hi = tok_end / p->m;
  if (entries->rows == 0 && g_hi > entries->capacity) return LCSC_ERR_INVALID_ARG;
  const int64_t n_new = g_hi - g_lo;
  Carve cv{reinterpret_cast<uint8_t*>(ws)};
  plan_compress(p, B, n_new, f.dim, cv, &L.pooled);
  if (n_new > 0 && (!ws || ws_bytes < cv.used)) return LCSC_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return LCSC_ERR_INVALID_ARG;
  L.x = x;
  L.x_dtype = p->x_dtype;
  L.n_x = tok_end - tok_begin + p->group_len - p->m;
  L.w = w_gate;
  L.gate_logits = p->gate_src == LCSC_GATE_LOGITS;
  L.bpos = b_pos;
  L.dim = f.dim;
  L.B = (int)B;
  L.span = {nullptr, 0, tok_begin, tok_end, p->m, p->group_len};
  L.n_new_max = (int)n_new;
  int64_t n_win = 0;
  if (window) {
    const int64_t lo = tok_end - window->capacity > tok_begin ? tok_end - window->capacity : tok_begin;
    n_win = tok_end - lo;
  }
  L.n_win_max = (int)n_win;
  L.status = status;
  cudaError_t e = launch_compress(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

int32_t lcsc_csa_compress(const lcsc_params* p, int32_t tensor, const void* x, int64_t B,
                          int64_t tok_begin, int64_t tok_end, const void* w_gate,
                          const float* b_pos, const lcsc_cache* entries, const lcsc_cache* window,
                          void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  return compress_impl(p, tensor, x, B, tok_begin, tok_end, w_gate, b_pos, entries, window, ws,
                       ws_bytes, status, stream, false);
}

int32_t lcsc_hca_compress(const lcsc_params* p, int32_t tensor, const void* x, int64_t B,
                          int64_t tok_begin, int64_t tok_end, const void* w_gate,
                          const float* b_pos, const lcsc_cache* entries, const lcsc_cache* window,
                          void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  return compress_impl(p, tensor, x, B, tok_begin, tok_end, w_gate, b_pos, entries, window, ws,
                       ws_bytes, status, stream, true);
}

int32_t lcsc_encode_rows(const lcsc_params* p, int32_t tensor, const float* rows, int64_t B,
                         int64_t n, int64_t row0, const lcsc_cache* out, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  RowFmt f;
  if ((st = tensor_fmt(p, tensor, &f))) return st;
  if (!rows || !aligned16(rows) || B < 1 || B > 65535 || n < 0 || row0 < 0) return LCSC_ERR_INVALID_ARG;
  CacheView v;
  if ((st = make_view(out, f, needs_scale(f.fmt), &v, true))) return st;  // a shard: its local rows
  if (row0 + n > out->capacity) return LCSC_ERR_INVALID_ARG;
  cudaError_t e = launch_encode_rows(rows, (int)B, n, row0, v, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

// ---------------------------------------------------------- indexer + top-k

int32_t lcsc_index_topk_workspace_size(const lcsc_params* p, int64_t B, int64_t T, int64_t n_max,
                                       size_t* bytes) {
  int32_t st = check_params(p);
  if (st) return st;
  if (!bytes || B < 1 || T < 1 || T > 65535 || B > 65535 / T || n_max < 0 || n_max > ((int64_t)1 << 40))
    return LCSC_ERR_INVALID_ARG;
  Carve cv{nullptr};
  plan_index(p, B, T, n_max, cv, nullptr);
  *bytes = cv.used;
  return LCSC_OK;
}

static int32_t index_setup(const lcsc_params* p, const void* q_idx, const float* w_idx,
                           const lcsc_cache* idx_keys, const int32_t* ctx_len, int64_t B, int64_t T,
                           int64_t n_max, int32_t* out_idx, float* out_score, Carve& cv,
                           size_t ws_bytes, int32_t* status, IndexLaunch* L) {
  if (!idx_supported(p)) return LCSC_ERR_UNSUPPORTED;
  if (p->top_k < 1) return LCSC_ERR_INVALID_ARG;
  if (!q_idx || !w_idx || !ctx_len || !out_idx) return LCSC_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(w_idx) || !aligned16(out_idx)) return LCSC_ERR_INVALID_ARG;
  if (out_score && !aligned16(out_score)) return LCSC_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || T > 65535 || B > 65535 / T || n_max < 0) return LCSC_ERR_INVALID_ARG;
  RowFmt f;
  int32_t st;
  if ((st = tensor_fmt(p, LCSC_TENSOR_IDX, &f))) return st;
  memset(L, 0, sizeof(*L));
  if ((st = make_view(idx_keys, f, needs_scale(f.fmt), &L->keys, true))) return st;
  if (n_max > idx_keys->capacity) return LCSC_ERR_INVALID_ARG;
  if (f.fmt != LCSC_FMT_F32 && idx_keys->capacity % 128 != 0) return LCSC_ERR_INVALID_ARG;
  plan_index(p, B, T, n_max, cv, L);
  if (!cv.base || !aligned16(cv.base) || ws_bytes < cv.used) return LCSC_ERR_WORKSPACE;
  L->q_idx = q_idx;
  L->q_dtype = p->q_dtype;
  L->w_idx = w_idx;
  L->ctx_len = ctx_len;
  L->B = (int)B;
  L->T = (int)T;
  L->H_I = p->idx_heads;
  L->d_I = p->idx_dim;
  L->m = p->m;
  L->k = p->top_k;
  L->n_max = n_max;
  L->out_idx = out_idx;
  L->out_score = out_score;
  L->status = status;
  return LCSC_OK;
}

int32_t lcsc_csa_index_topk(const lcsc_params* p, const void* q_idx, const float* w_idx,
                            const lcsc_cache* idx_keys, const int32_t* ctx_len, int64_t B,
                            int64_t T, int64_t n_max, int32_t* out_idx, float* out_score, void* ws,
                            size_t ws_bytes, int32_t* status, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  Carve cv{reinterpret_cast<uint8_t*>(ws)};
  IndexLaunch L;
  if ((st = index_setup(p, q_idx, w_idx, idx_keys, ctx_len, B, T, n_max, out_idx, out_score, cv,
                        ws_bytes, status, &L)))
    return st;
  cudaError_t e = launch_index_topk(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

// -------------------------------------------------------------- attention

int32_t lcsc_attn_workspace_size(const lcsc_params* p, int64_t B, int64_t T, int64_t n_max,
                                 int32_t dense, size_t* bytes) {
  int32_t st = check_params(p);
  if (st) return st;
  if (!bytes || B < 1 || T < 1 || T > 65535 || B > 65535 / T || n_max < 0 || n_max > ((int64_t)1 << 40))
    return LCSC_ERR_INVALID_ARG;
  Carve cv{nullptr};
  plan_attn(p, B, T, n_max, dense != 0, cv, nullptr);
  *bytes = cv.used;
  return LCSC_OK;
}

static int32_t attn_setup(const lcsc_params* p, const void* q, const lcsc_cache* kv,
                          const lcsc_cache* v, const lcsc_cache* win_kv, const lcsc_cache* win_v,
                          const int32_t* idx, const float* sink, const lcsc_cache* sink_kv,
                          const lcsc_cache* sink_v, const int32_t* ctx_len, int64_t B,
                          int64_t T, int64_t n_max, void* out, float* lse, Carve& cv,
                          size_t ws_bytes, int32_t* status, AttnLaunch* L) {
  if (!kv_supported(p)) return LCSC_ERR_UNSUPPORTED;
  if (!q || !ctx_len || !out || !aligned16(q) || !aligned16(out)) return LCSC_ERR_INVALID_ARG;
  if (lse && !aligned16(lse)) return LCSC_ERR_INVALID_ARG;
  if (sink && ((uintptr_t)sink & 3u)) return LCSC_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || T > 65535 || B > 65535 / T || n_max < 0) return LCSC_ERR_INVALID_ARG;
  const bool sep = v && v->data;
  if (sep != (win_v && win_v->data)) return LCSC_ERR_INVALID_ARG;
  if (sep && p->kv_format != LCSC_FMT_F32) return LCSC_ERR_UNSUPPORTED;
  if (!sep && p->v_dim != p->head_dim) return LCSC_ERR_INVALID_ARG;
  RowFmt fk, fv;
  int32_t st;
  if ((st = tensor_fmt(p, LCSC_TENSOR_KV, &fk))) return st;
  if ((st = tensor_fmt(p, LCSC_TENSOR_V, &fv))) return st;
  memset(L, 0, sizeof(*L));
  const bool ns = needs_scale(fk.fmt);
  if ((st = make_view(kv, fk, ns, &L->kv, true))) return st;
  if ((st = make_view(win_kv, fk, ns, &L->win_kv))) return st;
  if (sep) {
    if ((st = make_view(v, fv, ns, &L->v, true))) return st;
    if (!same_shard(kv, v)) return LCSC_ERR_INVALID_ARG;
    if ((st = make_view(win_v, fv, ns, &L->win_v))) return st;
    if (win_v->capacity != win_kv->capacity) return LCSC_ERR_INVALID_ARG;
  }
  if (n_max > kv->capacity) return LCSC_ERR_INVALID_ARG;
  if (p->window > 0 && win_kv->capacity < T + p->window - 1) return LCSC_ERR_INVALID_ARG;
  if (p->sink_mode == LCSC_SINK_TOKEN) {  // the stored position-0 row replaces the sink logit
    if (sink) return LCSC_ERR_INVALID_ARG;
    if ((st = make_view(sink_kv, fk, ns, &L->tok_kv))) return st;
    if (sep && (st = make_view(sink_v, fv, ns, &L->tok_v))) return st;
    L->sink_token = 1;
  }
  plan_attn(p, B, T, n_max, idx == nullptr, cv, L);
  if (!cv.base || !aligned16(cv.base) || ws_bytes < cv.used) return LCSC_ERR_WORKSPACE;
  L->q = q;
  L->q_dtype = p->q_dtype;
  L->idx = idx;
  L->sink = sink;
  L->ctx_len = ctx_len;
  L->B = (int)B;
  L->T = (int)T;
  L->H = p->n_heads;
  L->D = p->head_dim;
  L->Dv = p->v_dim;
  L->m = p->m;
  L->w = p->window;
  L->k = p->top_k;
  L->n_max = n_max;
  L->sm_scale = p->sm_scale;
  L->out_rope_dim = p->out_rope_base > 0.f ? p->out_rope_dim : 0;
  L->out_rope_base = p->out_rope_base;
  L->out = out;
  L->lse = lse;
  L->status = status;
  return LCSC_OK;
}

int32_t lcsc_csa_sparse_attn(const lcsc_params* p, const void* q, const lcsc_cache* kv,
                             const lcsc_cache* v, const lcsc_cache* win_kv,
                             const lcsc_cache* win_v, const int32_t* idx, const float* sink,
                             const lcsc_cache* sink_kv, const lcsc_cache* sink_v,
                             const int32_t* ctx_len, int64_t B, int64_t T, void* out, float* lse,
                             void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  if (!idx || !aligned16(idx) || p->top_k < 1) return LCSC_ERR_INVALID_ARG;
  Carve cv{reinterpret_cast<uint8_t*>(ws)};
  AttnLaunch L;
  if ((st = attn_setup(p, q, kv, v, win_kv, win_v, idx, sink, sink_kv, sink_v, ctx_len, B, T,
                       kv ? kv->capacity : 0, out, lse, cv, ws_bytes, status, &L)))
    return st;
  cudaError_t e = launch_attn_prepare(L, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_attention(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

int32_t lcsc_hca_dense_attn(const lcsc_params* p, const void* q, const lcsc_cache* kv,
                            const lcsc_cache* v, const lcsc_cache* win_kv, const lcsc_cache* win_v,
                            const float* sink, const lcsc_cache* sink_kv, const lcsc_cache* sink_v,
                            const int32_t* ctx_len, int64_t B, int64_t T, int64_t n_max, void* out,
                            float* lse, void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  Carve cv{reinterpret_cast<uint8_t*>(ws)};
  AttnLaunch L;
  if ((st = attn_setup(p, q, kv, v, win_kv, win_v, nullptr, sink, sink_kv, sink_v, ctx_len, B, T, n_max,
                       out, lse, cv, ws_bytes, status, &L)))
    return st;
  cudaError_t e = launch_attn_prepare(L, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_attention(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

// ------------------------------------------------------------ fused steps

int32_t lcsc_step_workspace_size(const lcsc_params* p, int32_t csa, int64_t B, int64_t T,
                                 int64_t n_max, size_t* bytes) {
  int32_t st = check_params(p);
  if (st) return st;
  if (!bytes || B < 1 || T < 1 || T > 65535 || B > 65535 / T || n_max < 0 || n_max > ((int64_t)1 << 40))
    return LCSC_ERR_INVALID_ARG;
  Carve cv{nullptr};
  const int64_t n_new = new_entries_max(T, p->m);
  plan_compress(p, B, n_new, p->head_dim, cv, nullptr);
  plan_compress(p, B, n_new, p->v_dim, cv, nullptr);
  if (csa) {
    plan_compress(p, B, n_new, p->idx_dim, cv, nullptr);
    cv.take<int32_t>((size_t)B * T * (p->top_k > 0 ? p->top_k : 1));
    plan_index(p, B, T, n_max, cv, nullptr);
  }
  plan_attn(p, B, T, n_max, !csa, cv, nullptr);
  *bytes = cv.used;
  return LCSC_OK;
}

static int32_t step_compress(const lcsc_params* p, const lcsc_step* s, int32_t tensor,
                             const void* x, const void* w, const float* bpos,
                             const lcsc_cache* ent, const lcsc_cache* win, const lcsc_cache* tok,
                             Carve& cv, int32_t* status, CompressLaunch* L) {
  RowFmt f;
  int32_t st;
  if ((st = tensor_fmt(p, tensor, &f))) return st;
  if (!x || !w || !bpos || !aligned16(x) || !aligned16(w) || !aligned16(bpos)) return LCSC_ERR_INVALID_ARG;
  if (p->x_dtype == LCSC_DT_BF16 && f.dim == 32) return LCSC_ERR_UNSUPPORTED;
  if (p->x_dtype == LCSC_DT_F32 && f.dim == 512) return LCSC_ERR_UNSUPPORTED;
  memset(L, 0, sizeof(*L));
  if ((st = make_view(ent, f, needs_scale(f.fmt), &L->entries))) return st;
  if (win && (st = make_view(win, f, needs_scale(f.fmt), &L->window))) return st;
  if (tok && (st = make_view(tok, f, needs_scale(f.fmt), &L->sink_tok))) return st;
  if (s->n_max > ent->capacity) return LCSC_ERR_INVALID_ARG;
  const int64_t n_new = new_entries_max(s->T, p->m);
  plan_compress(p, s->B, n_new, f.dim, cv, &L->pooled);
  L->x = x;
  L->x_dtype = p->x_dtype;
  L->n_x = s->T + p->group_len - 1;
  L->w = w;
  L->gate_logits = p->gate_src == LCSC_GATE_LOGITS;
  L->bpos = bpos;
  L->dim = f.dim;
  L->B = (int)s->B;
  L->span = {s->ctx_len, (int)s->T, 0, 0, p->m, p->group_len};
  L->n_new_max = (int)n_new;
  L->n_win_max = win ? (int)s->T : 0;
  L->status = status;
  return LCSC_OK;
}

// Two more streams per device for the parts of a CSA step that do not depend
// on each other (the KV latent's compression runs beside the indexer keys'
// compression, scoring and top-k; the query quantisation beside the indexer
// keys' compression), with fork / join events.
// Enqueueing on it is serialised by a mutex; the work itself is ordered
// only by the events.
struct SideStream {
  cudaStream_t s = nullptr, s2 = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr, join2 = nullptr;
};
constexpr int kMaxSideDevices = 64;
std::mutex g_side_mu;
SideStream g_side[kMaxSideDevices];

cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  SideStream& ss = g_side[dev];
  if (!ss.s) {
    if ((e = cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&ss.s2, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&ss.join2, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  *out = &ss;
  return cudaSuccess;
}

static int32_t step_impl(const lcsc_params* p, const lcsc_step* s, void* ws, size_t ws_bytes,
                         int32_t* status, void* stream, bool csa) {
  int32_t st = check_params(p);
  if (st) return st;
  if (!s || s->B < 1 || s->T < 1 || s->T > 65535 || s->B > 65535 / s->T || s->n_max < 0 || !s->ctx_len)
    return LCSC_ERR_INVALID_ARG;
  if (p->group_len > 128) return LCSC_ERR_UNSUPPORTED;
  if (csa && (!idx_supported(p) || p->top_k < 1)) return csa && p->top_k < 1 ? LCSC_ERR_INVALID_ARG : LCSC_ERR_UNSUPPORTED;
  if (!kv_supported(p)) return LCSC_ERR_UNSUPPORTED;
  if (!ws || !aligned16(ws)) return LCSC_ERR_WORKSPACE;
  const bool sep = s->v.data != nullptr;
  if (sep != (s->win_v.data != nullptr) || sep != (s->x_v != nullptr)) return LCSC_ERR_INVALID_ARG;
  if (p->window > 0 && s->win_kv.capacity < s->T + p->window - 1) return LCSC_ERR_INVALID_ARG;
  // the fused steps select over every entry: entry shards go through the
  // separate calls and the merges
  if (s->kv.rows || s->v.rows || s->idx_keys.rows) return LCSC_ERR_INVALID_ARG;

  Carve cv{reinterpret_cast<uint8_t*>(ws)};
  CompressLaunch ck, cvv, ci;
  const bool tok = p->sink_mode == LCSC_SINK_TOKEN;
  if ((st = step_compress(p, s, LCSC_TENSOR_KV, s->x_kv, s->w_kv, s->b_kv, &s->kv, &s->win_kv,
                          tok ? &s->sink_kv : nullptr, cv, status, &ck)))
    return st;
  if (sep) {
    if ((st = step_compress(p, s, LCSC_TENSOR_V, s->x_v, s->w_v, s->b_v, &s->v, &s->win_v,
                            tok ? &s->sink_v : nullptr, cv, status, &cvv)))
      return st;
  } else {
    plan_compress(p, s->B, new_entries_max(s->T, p->m), p->v_dim, cv, nullptr);
  }
  IndexLaunch il;
  int32_t* sel = nullptr;
  if (csa) {
    if ((st = step_compress(p, s, LCSC_TENSOR_IDX, s->x_idx, s->w_idx, s->b_idx, &s->idx_keys,
                            nullptr, nullptr, cv, status, &ci)))
      return st;
    // the selection buffer: the caller's out_idx, else workspace (planned either way)
    int32_t* sel_ws = cv.take<int32_t>((size_t)s->B * s->T * p->top_k);
    sel = s->out_idx ? s->out_idx : sel_ws;
    // workspace bounds are checked once the whole plan is known
    if ((st = index_setup(p, s->q_idx, s->w_heads, &s->idx_keys, s->ctx_len, s->B, s->T, s->n_max,
                          sel, s->out_score, cv, (size_t)-1, status, &il)))
      return st;
  }
  AttnLaunch al;
  if ((st = attn_setup(p, s->q, &s->kv, sep ? &s->v : nullptr, &s->win_kv, sep ? &s->win_v : nullptr,
                       sel, s->sink, &s->sink_kv, sep ? &s->sink_v : nullptr, s->ctx_len, s->B, s->T,
                       s->n_max, s->out, s->lse, cv, (size_t)-1, status, &al)))
    return st;
  if (ws_bytes < cv.used) return LCSC_ERR_WORKSPACE;

  if (s->n_events < 0 || (s->n_events > 0 && !s->events)) return LCSC_ERR_INVALID_ARG;

  cudaStream_t strm = (cudaStream_t)stream;
  cudaError_t e;
  int stage = 0;
  auto mark = [&]() -> cudaError_t {
    const int i = stage++;
    if (i < s->n_events && s->events[i]) return cudaEventRecord((cudaEvent_t)s->events[i], strm);
    return cudaSuccess;
  };
  if ((e = mark()) != cudaSuccess) return cuda_fail(e);
  if (csa) {
    // Fork: the KV latent's pooling (and window rows) on one side stream,
    // joined only before the attention, which alone reads them; the query
    // quantisation on the other, joined before the scoring.  The indexer
    // keys' pooling stays on the caller's stream: the scoring reads it.
    // The lock covers every record of the shared events up to its wait.
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream* ss = nullptr;
    if ((e = side_stream(&ss)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaEventRecord(ss->fork, strm)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(ss->s2, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_compress(ck, ss->s)) != cudaSuccess) return cuda_fail(e);
    if (sep && (e = launch_compress(cvv, ss->s)) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_attn_prepare(al, ss->s)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaEventRecord(ss->join, ss->s)) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_index_quantize(il, ss->s2)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaEventRecord(ss->join2, ss->s2)) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_compress(ci, strm)) != cudaSuccess) return cuda_fail(e);
    if ((e = mark()) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(strm, ss->join2, 0)) != cudaSuccess) return cuda_fail(e);
    if ((e = mark()) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_index_score_only(il, strm)) != cudaSuccess) return cuda_fail(e);
    if ((e = mark()) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_topk(il, strm)) != cudaSuccess) return cuda_fail(e);
    if ((e = mark()) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(strm, ss->join, 0)) != cudaSuccess) return cuda_fail(e);
  } else {
    // the attention's query images on a side stream, beside the compression
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream* ss = nullptr;
    if ((e = side_stream(&ss)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaEventRecord(ss->fork, strm)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_attn_prepare(al, ss->s)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaEventRecord(ss->join, ss->s)) != cudaSuccess) return cuda_fail(e);
    if ((e = launch_compress(ck, strm)) != cudaSuccess) return cuda_fail(e);
    if (sep && (e = launch_compress(cvv, strm)) != cudaSuccess) return cuda_fail(e);
    if ((e = mark()) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(strm, ss->join, 0)) != cudaSuccess) return cuda_fail(e);
  }
  if ((e = launch_attention(al, strm)) != cudaSuccess) return cuda_fail(e);
  if ((e = mark()) != cudaSuccess) return cuda_fail(e);
  return LCSC_OK;
}

// ------------------------------------------------------------ shard merges

int32_t lcsc_topk_merge(const lcsc_params* p, int32_t n_parts, const int32_t* part_idx,
                        const float* part_score, int64_t B, int64_t T, int32_t* out_idx,
                        float* out_score, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  if (p->top_k < 1 || n_parts < 1 || (int64_t)n_parts * p->top_k > LCSC_MERGE_MAX_CANDIDATES)
    return LCSC_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || T > 65535 || B > 65535 / T) return LCSC_ERR_INVALID_ARG;
  if (!part_idx || !part_score || !out_idx) return LCSC_ERR_INVALID_ARG;
  if (!aligned16(part_idx) || !aligned16(part_score) || !aligned16(out_idx)) return LCSC_ERR_INVALID_ARG;
  if (out_score && !aligned16(out_score)) return LCSC_ERR_INVALID_ARG;
  TopkMergeLaunch L;
  L.n_parts = n_parts;
  L.lists = B * T;
  L.k = p->top_k;
  L.part_idx = part_idx;
  L.part_score = part_score;
  L.out_idx = out_idx;
  L.out_score = out_score;
  cudaError_t e = launch_topk_merge(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

int32_t lcsc_attn_merge(const lcsc_params* p, int32_t n_parts, const void* part_out, const float* part_lse,
                        const float* sink, const int32_t* ctx_len, int64_t B, int64_t T, void* out,
                        float* lse, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  if (n_parts < 1 || n_parts > 4096) return LCSC_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || T > 65535 || B > 65535 / T) return LCSC_ERR_INVALID_ARG;
  if (p->v_dim != 512 && p->v_dim != 128) return LCSC_ERR_UNSUPPORTED;
  if (p->n_heads % 4 != 0) return LCSC_ERR_UNSUPPORTED;
  if (p->sink_mode == LCSC_SINK_TOKEN && sink) return LCSC_ERR_INVALID_ARG;
  if (!part_out || !part_lse || !ctx_len || !out) return LCSC_ERR_INVALID_ARG;
  if (!aligned16(part_out) || !aligned16(part_lse) || !aligned16(out)) return LCSC_ERR_INVALID_ARG;
  if ((lse && !aligned16(lse)) || (sink && ((uintptr_t)sink & 3u))) return LCSC_ERR_INVALID_ARG;
  AttnMergeLaunch L;
  L.n_parts = n_parts;
  L.lists = B * T;
  L.T = (int)T;
  L.H = p->n_heads;
  L.Dv = p->v_dim;
  L.dtype = p->q_dtype;
  L.part_out = part_out;
  L.part_lse = part_lse;
  L.sink = sink;
  L.ctx_len = ctx_len;
  L.out_rope_dim = p->out_rope_base > 0.f ? p->out_rope_dim : 0;
  L.out_rope_base = p->out_rope_base;
  L.out = out;
  L.lse = lse;
  cudaError_t e = launch_attn_merge(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}

int32_t lcsc_csa_decode(const lcsc_params* p, const lcsc_step* s, void* ws, size_t ws_bytes,
                        int32_t* status, void* stream) {
  return step_impl(p, s, ws, ws_bytes, status, stream, true);
}

int32_t lcsc_hca_decode(const lcsc_params* p, const lcsc_step* s, void* ws, size_t ws_bytes,
                        int32_t* status, void* stream) {
  return step_impl(p, s, ws, ws_bytes, status, stream, false);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// lcsc_csa_index_topk_noalloc: the indexer + top-k call for callers that
// cannot allocate device memory.  Its scratch is one fixed array in this
// file's module; the caller still passes every input and output.
// ---------------------------------------------------------------------------
#include <mutex>

namespace lcsc {
namespace {

// Scratch of the no-allocation entry point.  Every device that loads this
// library holds it until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[LCSC_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The name of the
// array in host code is a host-side stand-in, so the address is fetched
// once per device with cudaGetSymbolAddress (with that device current).
int32_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return LCSC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return LCSC_OK;
}

}  // namespace
}  // namespace lcsc

extern "C" int32_t lcsc_csa_index_topk_noalloc(const lcsc_params* p, const void* q_idx,
                                               const float* w_idx, const lcsc_cache* idx_keys,
                                               const int32_t* ctx_len, int64_t B, int64_t T,
                                               int64_t n_max, int32_t* out_idx, float* out_score,
                                               int32_t* status, void* stream) {
  int32_t st = check_params(p);
  if (st) return st;
  // the limits index_setup applies, checked before the plan's size products
  // (division: B * T itself cannot overflow), so that the total compared
  // with the fixed scratch size is exact
  if (B < 1 || T < 1 || n_max < 0 || T > 65535 || B > 65535 / T || n_max > ((int64_t)1 << 40))
    return LCSC_ERR_INVALID_ARG;
  Carve need{nullptr};
  plan_index(p, B, T, n_max, need, nullptr);
  if (need.used > (size_t)LCSC_NOALLOC_SCRATCH_BYTES) return LCSC_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  Carve cv{reinterpret_cast<uint8_t*>(scratch)};
  IndexLaunch L;
  if ((st = index_setup(p, q_idx, w_idx, idx_keys, ctx_len, B, T, n_max, out_idx, out_score, cv,
                        (size_t)LCSC_NOALLOC_SCRATCH_BYTES, status, &L)))
    return st;
  cudaError_t e = launch_index_topk(L, (cudaStream_t)stream);
  return e == cudaSuccess ? LCSC_OK : cuda_fail(e);
}
