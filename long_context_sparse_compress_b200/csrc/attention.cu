// Joint attention of all query heads over one shared set of stored rows:
// compressed entries (the top-k selection for CSA, all visible entries for
// HCA) plus the raw sliding-window rows, with a per-head sink logit.
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works": exact attention over the
// selected compressed entries, a sliding-window branch of uncompressed recent
// tokens and a sink term that keeps part of each head's probability mass off
// every row; HCA is the same without selection, with the shared-KV
// multi-query layout.  One softmax spans both branches:
//   o[h] = sum_j e^{l_j - M} V_j / (e^{sigma_h - M} + sum_j e^{l_j - M}).
//
// Work split (flash-decoding): the row list of a query is cut into `splits`
// ranges; a CTA owns (query, range, 16-head group) and keeps an online
// softmax over 32-row tiles; a combine kernel merges the ranges' (max, sum,
// unnormalised output) and adds the sink to the denominator.
#include "kernels.cuh"
#include "launches.h"
#include "rope.cuh"

namespace lcsc {
namespace {

constexpr int kTile = 32;
constexpr int kThreads = 256;

struct QueryRows {
  int64_t p, n_vis;      // position, visible entries
  int64_t n_ent_slots;   // entry slots (k for CSA, n_vis for HCA)
  int64_t w_lo, n_win;   // window positions w_lo .. w_lo + n_win - 1
  int64_t n_tok;         // 1: the stored position-0 row follows the window
  bool ok;
};

__device__ __forceinline__ QueryRows query_rows(const AttnLaunch& a, int b, int t) {
  QueryRows r;
  const int64_t L = a.ctx_len[b];
  // a context whose entries would pass the caches' n_max rows is invalid
  // (an entry shard holds a range of them: no limit)
  r.ok = L >= a.T && (a.kv.rows > 0 || L / a.m <= a.n_max);
  r.p = L - a.T + t;
  r.n_vis = r.ok ? (r.p + 1) / a.m : 0;
  r.n_ent_slots = a.idx ? a.k : a.kv.local_count(r.n_vis);
  r.w_lo = r.p - a.w + 1 > 0 ? r.p - a.w + 1 : 0;
  r.n_win = r.ok ? r.p - r.w_lo + 1 : 0;
  if (a.w == 0) r.n_win = 0;
  // sink token: position 0 joins once, unless the window already holds it
  r.n_tok = (r.ok && a.sink_token && !(r.n_win > 0 && r.w_lo == 0)) ? 1 : 0;
  return r;
}

// Dequantise one stored row into shared memory (row stride RS floats).
// `nthr` threads cooperate, thread `lt` of them.
template <int KVFMT, int DIM>
__device__ __forceinline__ void load_row(const CacheView& cv, int b, int64_t r, float* dst, int lt,
                                         int nthr) {
  const uint8_t* row = cv.row(b, r);
  if (KVFMT == LCSC_FMT_F32) {
    for (int c = lt; c < DIM / 4; c += nthr) {
      const float4 f = reinterpret_cast<const float4*>(row)[c];
      dst[4 * c] = f.x; dst[4 * c + 1] = f.y; dst[4 * c + 2] = f.z; dst[4 * c + 3] = f.w;
    }
  } else {
    const int n_fp8 = cv.f.dim - cv.f.rope;
    const float s = *cv.fscale(b, r);
    const int chunks = cv.f.row_bytes / 16;
    for (int c = lt; c < chunks; c += nthr) {
      const uint4 u = reinterpret_cast<const uint4*>(row)[c];
      const int byte0 = c * 16;
      if (byte0 < n_fp8) {
        const uint16_t* c2 = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 f = e4m3x2_val(c2[j]);
          dst[byte0 + 2 * j] = f.x * s;
          dst[byte0 + 2 * j + 1] = f.y * s;
        }
      } else {
        const uint16_t* h = reinterpret_cast<const uint16_t*>(&u);
        const int e0 = n_fp8 + (byte0 - n_fp8) / 2;
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[e0 + j] = bf16_val(h[j]);
      }
    }
  }
}

// grid: (splits, H / HPC, B*T); block 256.
template <int KVFMT, int D, int DV, int HPC, bool kSepV>
__global__ void __launch_bounds__(kThreads) attn_partial_kernel(AttnLaunch a) {
  grid_dep_wait();
  constexpr int KS = D + 1, VS = DV + 1;
  constexpr int TPH = kThreads / HPC;      // threads per head
  constexpr int OPT = DV / TPH;            // outputs per thread
  constexpr int DOTS = HPC * kTile / kThreads;  // logits per thread
  extern __shared__ float sm[];
  float* qs = sm;                          // [HPC][KS]
  float* ks = qs + HPC * KS;               // [kTile][KS]
  float* vs = kSepV ? ks + kTile * KS : ks;  // [kTile][VS]
  float* ps = (kSepV ? vs + kTile * VS : ks + kTile * KS);  // [HPC][kTile]
  float* ms = ps + HPC * kTile;            // running max [HPC]
  float* ls = ms + HPC;                    // running sum [HPC]
  float* al = ls + HPC;                    // rescale factor [HPC]
  __shared__ int64_t rows_s[kTile];
  __shared__ int8_t src_s[kTile];          // 0 invalid, 1 entry, 2 window, 3 position-0 row

  const int list = blockIdx.z;
  const int b = list / a.T, t = list % a.T;
  const int h0 = blockIdx.y * HPC;
  const int tid = threadIdx.x;
  const QueryRows qr = query_rows(a, b, t);
  if (!qr.ok && tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && a.status)
    atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
  const int64_t total = qr.ok ? qr.n_ent_slots + qr.n_win + qr.n_tok : 0;
  const int64_t s_lo = (int64_t)blockIdx.x * a.rows_per_split;
  int64_t s_hi = s_lo + a.rows_per_split;
  if (s_hi > total) s_hi = total;

  // query rows of this head group
  for (int i = tid; i < HPC * D; i += kThreads) {
    const int h = i / D, d = i % D;
    qs[h * KS + d] = load_elem(a.q, ((int64_t)list * a.H + h0 + h) * D + d, a.q_dtype);
  }
  if (tid < HPC) {
    ms[tid] = -INFINITY;
    ls[tid] = 0.f;
  }
  const int hh = tid / TPH, hl = tid % TPH;  // this thread's head and lane within it
  float o[OPT];
#pragma unroll
  for (int i = 0; i < OPT; ++i) o[i] = 0.f;
  __syncthreads();

  for (int64_t base = s_lo; base < s_hi; base += kTile) {
    // ---- resolve the tile's rows
    if (tid < kTile) {
      const int64_t slot = base + tid;
      int8_t src = 0;
      int64_t row = 0;
      if (slot < s_hi) {
        if (slot < qr.n_ent_slots) {
          const int64_t g = a.idx ? (int64_t)a.idx[(int64_t)list * a.k + slot] : slot + a.kv.row0;
          if (g >= 0 && g < qr.n_vis) {
            row = a.kv.local(g);  // -1: another shard holds it
            src = row >= 0 ? 1 : 0;
            if (row < 0) row = 0;
          } else if (g != -1 || !a.idx) {
            if (a.status) atomicOr(a.status, LCSC_DEV_BAD_INDEX);
          }
        } else if (slot < qr.n_ent_slots + qr.n_win) {
          src = 2;
          row = (qr.w_lo + (slot - qr.n_ent_slots)) % a.win_kv.capacity;
        } else {
          src = 3;
          row = 0;
        }
      }
      rows_s[tid] = row;
      src_s[tid] = src;
    }
    __syncthreads();
    // ---- load K (and V) rows: 8 threads per row
    {
      const int j = tid / 8, lt = tid % 8;
      const int8_t src = src_s[j];
      if (src == 1) {
        load_row<KVFMT, D>(a.kv, b, rows_s[j], ks + j * KS, lt, 8);
        if (kSepV) load_row<KVFMT, DV>(a.v, b, rows_s[j], vs + j * VS, lt, 8);
      } else if (src == 2) {
        load_row<KVFMT, D>(a.win_kv, b, rows_s[j], ks + j * KS, lt, 8);
        if (kSepV) load_row<KVFMT, DV>(a.win_v, b, rows_s[j], vs + j * VS, lt, 8);
      } else if (src == 3) {
        load_row<KVFMT, D>(a.tok_kv, b, 0, ks + j * KS, lt, 8);
        if (kSepV) load_row<KVFMT, DV>(a.tok_v, b, 0, vs + j * VS, lt, 8);
      }
    }
    __syncthreads();
    // ---- logits
#pragma unroll
    for (int q = 0; q < DOTS; ++q) {
      const int idx = tid + q * kThreads;
      const int h = idx / kTile, j = idx % kTile;
      float acc = 0.f;
      if (src_s[j]) {
        const float* qrow = qs + h * KS;
        const float* krow = ks + j * KS;
#pragma unroll 8
        for (int d = 0; d < D; ++d) acc = fmaf(qrow[d], krow[d], acc);
        acc *= a.sm_scale;
      } else {
        acc = -INFINITY;
      }
      ps[h * kTile + j] = acc;
    }
    __syncthreads();
    // ---- online softmax per head (TPH threads per head)
    {
      float mx = -INFINITY;
      for (int j = hl; j < kTile; j += TPH) mx = fmaxf(mx, ps[hh * kTile + j]);
      mx = group_max(mx, TPH);
      const float m_old = ms[hh];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int j = hl; j < kTile; j += TPH) {
        const float l = ps[hh * kTile + j];
        const float p = (m_new == -INFINITY) ? 0.f : __expf(l - m_new);
        ps[hh * kTile + j] = p;
        sum += p;
      }
      for (int off = TPH >> 1; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      __syncwarp();
      if (hl == 0) {
        const float alpha = (m_old == -INFINITY) ? 0.f : __expf(m_old - m_new);
        al[hh] = alpha;
        ls[hh] = ls[hh] * alpha + sum;
        ms[hh] = m_new;
      }
    }
    __syncthreads();
    // ---- o = o * alpha + P V
    {
      const float alpha = al[hh];
      const float* prow = ps + hh * kTile;
#pragma unroll
      for (int i = 0; i < OPT; ++i) o[i] *= alpha;
      for (int j = 0; j < kTile; ++j) {
        const float p = prow[j];
        if (p == 0.f) continue;
        const float* vrow = vs + j * (kSepV ? VS : KS);
#pragma unroll
        for (int i = 0; i < OPT; ++i) o[i] = fmaf(p, vrow[hl + i * TPH], o[i]);
      }
    }
    __syncthreads();
  }
  // ---- partial results
  const int64_t pidx = ((int64_t)list * a.splits + blockIdx.x) * a.H + h0 + hh;
  float* po = a.part_o + pidx * DV;
#pragma unroll
  for (int i = 0; i < OPT; ++i) po[hl + i * TPH] = o[i];
  if (hl == 0) {
    a.part_ml[pidx * 2] = ms[hh];
    a.part_ml[pidx * 2 + 1] = ls[hh];
  }
}

// Merge of the split partials (reference max m_s, sum l_s, unnormalised
// O_s) and the sink: one pass with a running max, every load of a batch of
// splits in flight.  grid (B*T, H): one head per CTA, so that a single query
// still spreads its splits' partials over H CTAs; block DV/4 threads, four
// dims (one float4) per thread.
template <int DV>
__global__ void __launch_bounds__(DV / 4) attn_combine_kernel(AttnLaunch a) {
  grid_dep_wait();
  constexpr int U = 16;         // splits per batch
  const int list = blockIdx.x;
  const int h = blockIdx.y;
  const int d4 = threadIdx.x;
  const float sigma = a.sink ? a.sink[h] : -INFINITY;
  const float* ml = a.part_ml + ((int64_t)list * a.splits * a.H + h) * 2;  // split s at ml[s * H * 2]
  const float4* po = reinterpret_cast<const float4*>(a.part_o + ((int64_t)list * a.splits * a.H + h) * DV) + d4;
  const int64_t ml_step = (int64_t)a.H * 2, o_step = (int64_t)a.H * DV / 4;
  float M = sigma, den = sigma > -INFINITY ? 1.f : 0.f;  // the sink adds e^(sigma - M) to the denominator
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < a.splits; s0 += U) {
    float m[U], l[U];
    float4 o[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool in = s0 + u < a.splits;
      m[u] = in ? ml[(s0 + u) * ml_step] : -INFINITY;
      l[u] = in ? ml[(s0 + u) * ml_step + 1] : 0.f;
      o[u] = in ? po[(s0 + u) * o_step] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mb = -INFINITY;
#pragma unroll
    for (int u = 0; u < U; ++u) mb = fmaxf(mb, m[u]);
    if (mb > M) {  // rescale what has been summed to the new maximum
      const float r = M > -INFINITY ? expf(M - mb) : 0.f;
      den *= r;
      acc.x *= r;
      acc.y *= r;
      acc.z *= r;
      acc.w *= r;
      M = mb;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (m[u] == -INFINITY) continue;  // an empty split (its O and sum are zero)
      const float f = expf(m[u] - M);
      den = fmaf(l[u], f, den);
      acc.x = fmaf(o[u].x, f, acc.x);
      acc.y = fmaf(o[u].y, f, acc.y);
      acc.z = fmaf(o[u].z, f, acc.z);
      acc.w = fmaf(o[u].w, f, acc.w);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float4 o4 = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  RopePair2 rot;
  const int64_t pos = (int64_t)a.ctx_len[list / a.T] - a.T + list % a.T;
  if (inverse_rope_angles(4 * d4, DV, a.out_rope_dim, a.out_rope_base, pos, &rot)) o4 = rotate2(o4, rot);
  const float r[4] = {o4.x, o4.y, o4.z, o4.w};
  const int64_t oi = ((int64_t)list * a.H + h) * DV + 4 * d4;
  if (a.q_dtype == LCSC_DT_BF16) {
    uint16_t* out = reinterpret_cast<uint16_t*>(a.out) + oi;
    out[0] = bf16_code(r[0]);
    out[1] = bf16_code(r[1]);
    out[2] = bf16_code(r[2]);
    out[3] = bf16_code(r[3]);
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + oi) = make_float4(r[0], r[1], r[2], r[3]);
  }
  if (a.lse && d4 == 0) a.lse[(int64_t)list * a.H + h] = (den > 0.f) ? M + logf(den) : -INFINITY;
}

template <int KVFMT, int D, int DV, int HPC, bool kSepV>
cudaError_t launch_attn(const AttnLaunch& a, cudaStream_t stream) {
  constexpr int KS = D + 1, VS = DV + 1;
  const size_t smem = sizeof(float) * (HPC * KS + kTile * KS + (kSepV ? kTile * VS : 0) +
                                       HPC * kTile + 3 * HPC);
  auto kern = attn_partial_kernel<KVFMT, D, DV, HPC, kSepV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.splits, a.H / HPC, a.B * a.T);
  if ((e = launch_pdl(kern, grid, dim3(kThreads), smem, stream, a)) != cudaSuccess) return e;
  return launch_pdl(attn_combine_kernel<DV>, dim3(a.B * a.T, a.H), dim3(DV / 4), 0, stream, a);
}

}  // namespace

void attention_splits(int64_t max_rows, int64_t n_ctas_per_split, int granule, int target_ctas, int* splits,
                      int* rows_per_split) {
  if (max_rows < 1) max_rows = 1;
  if (n_ctas_per_split < 1) n_ctas_per_split = 1;
  if (target_ctas < 1) target_ctas = 1;
  const int64_t tiles = (max_rows + granule - 1) / granule;
  // Time of s splits, in tiles of one CTA: the waves of n * s CTAs that
  // target_ctas resident ones take, times a split's tiles plus about three
  // tiles of fixed work (queries in, the first gathers, partials out), plus
  // about two for the combine pass when s > 1.  The fewest splits within 5%
  // of the best (fewer partials to write and combine).
  auto cost = [&](int64_t s) {
    return ((n_ctas_per_split * s + target_ctas - 1) / target_ctas) * ((tiles + s - 1) / s + 3) + (s > 1 ? 2 : 0);
  };
  int64_t best = cost(1);
  for (int64_t c = 2; c <= tiles; ++c) best = cost(c) < best ? cost(c) : best;
  int64_t s = 1;
  while (s < tiles && cost(s) * 20 > best * 21) ++s;
  int64_t rps = ((max_rows + s - 1) / s + granule - 1) / granule * granule;
  *rows_per_split = (int)rps;
  *splits = (int)((max_rows + rps - 1) / rps);
}

cudaError_t launch_attn_prepare(const AttnLaunch& a, cudaStream_t stream) {
  return attn_mma_supported(a) ? launch_attn_qimage(a, stream) : cudaSuccess;
}

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream) {
  const bool sep = a.v.data != nullptr;
  if (attn_mma_supported(a)) {
    cudaError_t e = launch_attn_mma(a, stream);
    if (e != cudaSuccess) return e;
    if (a.splits == 1) return cudaSuccess;  // one split per query: the kernel wrote the output
    return launch_pdl(attn_combine_kernel<512>, dim3(a.B * a.T, a.H), dim3(128), 0, stream, a);
  }
  if (a.kv.f.fmt == LCSC_FMT_F32 && a.D == 128 && a.Dv == 128 && a.H % 8 == 0) {
    if (sep) return launch_attn<LCSC_FMT_F32, 128, 128, 8, true>(a, stream);
    return launch_attn<LCSC_FMT_F32, 128, 128, 8, false>(a, stream);
  }
  if (a.kv.f.fmt == LCSC_FMT_KV && a.D == 512 && a.Dv == 512 && a.H % 16 == 0 && !sep)
    return launch_attn<LCSC_FMT_KV, 512, 512, 16, false>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace lcsc
