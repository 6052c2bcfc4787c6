// Softmax-gated pooling of token groups into compressed entries, and the
// storing of pooled / raw rows in the cache formats.
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works" -- every group of m consecutive
// tokens' keys/values becomes one entry via trainable compression weights, a
// softmax over the group and learnable positional biases; per channel c:
//   z_j[c] = sum_d x_j[d] W[d][c] + Bpos[j_rel][c],  e[c] = sum_j softmax_j(z[c]) x_j[c].
//
// Kernel design: a CTA owns up to 128 consecutive token rows (E whole groups
// plus the G - m rows of history an overlapping group needs) and 64 output
// channels.  The gate logits z = x W are a [128 x dim] x [dim x 64] GEMM
// (tcgen05 with the accumulator in TMEM for bf16 rows, FP32 FMA for fp32
// rows); the group softmax and the weighted sum run on the tile in shared
// memory.  The channel blocks of the same entries form a thread-block cluster
// that exchanges the FP8 amax through distributed shared memory and stores
// the entries and the raw window rows itself; when the grid's clusters cannot
// all be resident at once, the pooled fp32 rows go to scratch and a second
// kernel stores them (whole rows, for the amax) and the window rows.
#include <cooperative_groups.h>
#include <type_traits>

#include "kernels.cuh"
#include "launches.h"
#include "sm100.cuh"

namespace lcsc {
namespace {

constexpr int kRows = 128;   // token rows per CTA
constexpr int kThreads = 256;
constexpr int kMaxEnt = 32;  // entries per CTA (their pooled rows wait in shared memory)

// Dynamic shared memory of pool_kernel (from a 1024-byte-aligned base): x
// tile, then the W chunk (reused for z and the biases), then the pooled rows
// [kMaxEnt][NC].  bf16: x and W in the tensor cores' 128-byte-swizzled
// layouts (x as DIM / 64 blocks of [128 rows][128 B], W as [DIM][NC = 64
// channels = 128 B]); fp32: padded rows for the CUDA-core GEMM.
template <bool kBf16, int DIM, int NC>
__host__ __device__ constexpr size_t pool_smem_offset() {
  constexpr size_t elem = kBf16 ? 2 : 4;
  constexpr size_t xs = elem * kRows * (kBf16 ? DIM : DIM + 1);
  constexpr size_t wz = elem * DIM * (kBf16 ? NC : NC + 1);
  constexpr size_t zb = sizeof(float) * (kRows * (NC + 1) + kRows * NC);  // z, then biases of <= 128 tokens
  return xs + (wz > zb ? wz : zb);
}
template <bool kBf16, int DIM, int NC>
__host__ __device__ constexpr size_t pool_smem_bytes() {
  return pool_smem_offset<kBf16, DIM, NC>() + sizeof(float) * kMaxEnt * NC + 1024;  // + base alignment
}

// Byte offset of (row, byte) in a [rows][128 B] array with the 128-byte
// swizzle (16-byte chunk index XOR row % 8) that the tensor cores read.
__device__ __forceinline__ uint32_t swz128(int row, int byte) {
  return (uint32_t)(row * 128 + ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
}

struct SeqSpan {
  int64_t g_lo, g_hi;   // entries written
  int64_t x_pos0;       // position of raw row 0
  int64_t w_lo, w_hi;   // window positions written
  bool ok;
};

// `cap` is the entries' capacity: a context length whose entries would not
// fit makes the sequence invalid (nothing is written; the status flags it).
// An entry shard holds a range of the entries (cap < 0: no limit).
__device__ __forceinline__ SeqSpan seq_span(const Span& s, int b, int64_t win_cap, int64_t cap) {
  SeqSpan r;
  if (s.ctx_len) {
    const int64_t L = s.ctx_len[b];
    r.ok = L >= s.T && (cap < 0 || L / s.m <= cap);
    r.g_lo = r.ok ? (L - s.T) / s.m : 0;
    r.g_hi = r.ok ? L / s.m : 0;
    r.x_pos0 = L - (s.T + s.G - 1);
    r.w_lo = r.ok ? L - s.T : 0;
    r.w_hi = r.ok ? L : 0;
  } else {
    r.ok = true;
    r.g_lo = s.tok_begin / s.m;
    r.g_hi = s.tok_end / s.m;
    r.x_pos0 = s.tok_begin - (s.G - s.m);
    r.w_lo = s.tok_end - win_cap > s.tok_begin ? s.tok_end - win_cap : s.tok_begin;
    r.w_hi = s.tok_end;
  }
  return r;
}

// Capacity bound of seq_span: none for an entry shard.
__device__ __forceinline__ int64_t ent_cap(const CompressLaunch& a) {
  return a.entries.rows > 0 ? -1 : a.entries.capacity;
}

// ------------------------------------------------------------ mma helpers

// 16-byte global -> shared copy that completes asynchronously; `live` false
// fills the 16 bytes with zeros (nothing is read from `src`).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool live) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(live ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// ------------------------------------------------------------ fused entry store
// Stores this CTA's NC channels of each pooled entry row in the entries'
// cache format.  FP8 rows (and the FP8 part of KV rows) share one scale over
// the whole row: each CTA publishes its channels' amax and reads the others'
// from the cluster (the DIM / NC channel blocks of the same entries) through
// distributed shared memory.  FP4 block scales (16 values) and fp32 rows need
// nothing from other CTAs.  A warp per entry, a lane per channel pair; the
// arithmetic is the row store's (amax / 448 with a rounded division, codes
// of value / scale).
template <int DIM, int NC>
__device__ __forceinline__ void store_entries(const CompressLaunch& a, const float* pooled_s, float* pamax_s,
                                              const int64_t* ent_out, const int* ent_b, const int64_t* ent_g,
                                              int E_cta, int c0) {
  namespace cg = cooperative_groups;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  constexpr int kWarps = kThreads / kWarp;
  const CacheView& cv = a.entries;
  const int fmt = cv.f.fmt;
  const int ch = 2 * lane;                 // this lane's channel pair (ch, ch + 1) of the block
  const bool has = ch < NC;
  if (fmt == LCSC_FMT_KV || fmt == LCSC_FMT_FP8) {
    const int n_fp8 = cv.f.dim - (fmt == LCSC_FMT_KV ? cv.f.rope : 0);
    const bool fp8 = has && c0 + ch < n_fp8;  // n_fp8 is even: a pair is all FP8 or all BF16
    for (int e = warp; e < E_cta; e += kWarps) {
      float am = 0.f;
      if (fp8) am = fmaxf(fabsf(pooled_s[e * NC + ch]), fabsf(pooled_s[e * NC + ch + 1]));
      am = warp_max(am);
      if (lane == 0) pamax_s[e] = am;
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const unsigned nblk = cluster.num_blocks();
    for (int e = warp; e < E_cta; e += kWarps) {
      if (ent_out[e] < 0) continue;  // uniform over the warp
      float am = 0.f;
      for (unsigned r = 0; r < nblk; ++r) am = fmaxf(am, cluster.map_shared_rank(pamax_s, r)[e]);
      const float sc = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
      uint8_t* row = cv.row(ent_b[e], ent_g[e]);
      if (fp8) {
        const uint16_t c2 = e4m3x2_code(__fdiv_rn(pooled_s[e * NC + ch], sc), __fdiv_rn(pooled_s[e * NC + ch + 1], sc));
        *reinterpret_cast<uint16_t*>(row + c0 + ch) = c2;
      } else if (has) {
        uint16_t* d = reinterpret_cast<uint16_t*>(row + n_fp8) + (c0 + ch - n_fp8);
        d[0] = bf16_code(pooled_s[e * NC + ch]);
        d[1] = bf16_code(pooled_s[e * NC + ch + 1]);
      }
      if (blockIdx.y == 0 && lane == 0) *cv.fscale(ent_b[e], ent_g[e]) = sc;
    }
    cluster.sync();  // no CTA leaves while another may read its amax
  } else if (fmt == LCSC_FMT_FP4) {
    // blocks of 16 channels = 8 lanes
    for (int e = warp; e < E_cta; e += kWarps) {
      if (ent_out[e] < 0) continue;
      const float v0 = has ? pooled_s[e * NC + ch] : 0.f, v1 = has ? pooled_s[e * NC + ch + 1] : 0.f;
      const float amax = group_max(fmaxf(fabsf(v0), fabsf(v1)), 8);
      const uint8_t scode = (uint8_t)(e4m3x2_code(__fdiv_rn(amax, 6.f), 0.f) & 0xff);
      const float dsc = e4m3_val(scode);
      if (has) {
        uint8_t* row = cv.row(ent_b[e], ent_g[e]);
        const float y0 = dsc > 0.f ? __fdiv_rn(v0, dsc) : 0.f, y1 = dsc > 0.f ? __fdiv_rn(v1, dsc) : 0.f;
        row[(c0 + ch) / 2] = dsc > 0.f ? e2m1x2_code(y0, y1) : (uint8_t)0;
        if (ch % 16 == 0) *cv.bscale_at(ent_b[e], ent_g[e], (c0 + ch) / 16) = scode;
      }
    }
  } else {  // fp32 rows
    for (int e = warp; e < E_cta; e += kWarps) {
      if (ent_out[e] < 0 || !has) continue;
      float* row = reinterpret_cast<float*>(cv.row(ent_b[e], ent_g[e]));
      row[c0 + ch] = pooled_s[e * NC + ch];
      row[c0 + ch + 1] = pooled_s[e * NC + ch + 1];
    }
  }
}

// ------------------------------------------------------------ pool kernel
// A CTA owns up to 128 token rows and NC output channels.  Two tilings:
//  * by entries (bulk calls, prefill): grid (ceil(n_new_max / E), dim / NC, B),
//    E consecutive entries of one sequence, entry e on rows e*m .. e*m+G-1
//    (overlapping groups share rows);
//  * packed (a step that closes at most one group per sequence): grid
//    (ceil(B / SP), dim / NC, 1), the groups of SP = 128 / G sequences stacked,
//    entry e = sequence b0 + e on rows e*G .. e*G+G-1.
// Rows whose position is below 0 (or whose sequence closes no group) are
// masked out of the softmax.
template <bool kBf16, int DIM, int NC, bool kFused>
__global__ void __launch_bounds__(kThreads) pool_kernel(CompressLaunch a, int E, bool packed) {
  grid_dep_wait();
  using Elem = typename std::conditional<kBf16, uint16_t, float>::type;
  constexpr int XS = kBf16 ? DIM : DIM + 1;       // x tile row stride (elements; fp32 path)
  constexpr int WS = kBf16 ? NC : NC + 1;         // W chunk row stride (fp32 path)
  constexpr int ZS = NC + 1;                      // z tile row stride (floats)
  static_assert(!kBf16 || NC == 64, "bf16 W chunk rows are one 128-byte swizzle row");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Elem* xs = reinterpret_cast<Elem*>(smem);
  Elem* ws = reinterpret_cast<Elem*>(smem + sizeof(Elem) * kRows * XS);
  float* zs = reinterpret_cast<float*>(ws);  // reuses the W chunk after the GEMM
  __shared__ int64_t row_src[kRows];  // element offset of the row in x, or -1 (masked)
  __shared__ int64_t ent_out[kRows];  // pooled output row, or -1
  __shared__ int ent_row0[kRows];     // first tile row of the entry
  __shared__ int ent_b[kRows];        // its sequence
  __shared__ int64_t ent_g[kRows];    // and entry index in the cache
  __shared__ float pamax_s[kRows];    // this CTA's share of the entry's FP8 amax
  __shared__ int n_ent, rows_used;

  const int c0 = blockIdx.y * NC;
  const int m = a.span.m, G = a.span.G;
  const int tid = threadIdx.x;
  constexpr int VPL = DIM / 32;
  float* pooled_s = reinterpret_cast<float*>(smem + pool_smem_offset<kBf16, DIM, NC>());  // [entries][NC]

  // ---- window rows (the raw rows of the new tokens), a warp per row, spread
  // over the grid; independent of the pooling below
  if (kFused && a.window.data) {
    const int warp = tid / kWarp, lane = tid % kWarp;
    const int64_t cta = ((int64_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    const int64_t n_warps = (int64_t)gridDim.x * gridDim.y * gridDim.z * (kThreads / kWarp);
    const int64_t total = (int64_t)a.B * a.n_win_max;
    for (int64_t t = cta * (kThreads / kWarp) + warp; t < total; t += n_warps) {
      const int b = (int)(t / a.n_win_max);
      const int64_t i = t % a.n_win_max;
      const SeqSpan sp = seq_span(a.span, b, a.window.capacity, ent_cap(a));
      if (!sp.ok || i >= sp.w_hi - sp.w_lo) continue;
      const int64_t pos = sp.w_lo + i;
      const int64_t base = ((int64_t)b * a.n_x + (pos - sp.x_pos0)) * DIM + lane * VPL;
      float v[VPL];
#pragma unroll
      for (int j = 0; j < VPL; ++j) v[j] = load_elem(a.x, base + j, a.x_dtype);
      store_row_warp<VPL>(a.window, b, pos % a.window.capacity, v, lane);
      if (pos == 0 && a.sink_tok.data) store_row_warp<VPL>(a.sink_tok, b, 0, v, lane);
    }
  }
  if (tid == 0) { n_ent = 0; rows_used = 0; }
  __syncthreads();
  if (packed) {
    const int SP = kRows / G < kMaxEnt ? kRows / G : kMaxEnt;
    // one thread per tile row (row r: group j = r % G of sequence r / G)
    for (int r = tid; r < kRows; r += kThreads) {
      const int e = r / G, j = r % G;
      const int b = blockIdx.x * SP + e;
      int64_t src = -1;
      if (e < SP && b < a.B) {
        const SeqSpan sp = seq_span(a.span, b, a.window.capacity, ent_cap(a));
        const int64_t row = a.entries.local(sp.g_lo);  // -1: another shard's entry
        const bool valid = sp.ok && sp.g_hi - sp.g_lo == 1 && row >= 0;
        const int64_t pos = sp.g_lo * m + m - G + j;
        if (valid && pos >= 0) src = ((int64_t)b * a.n_x + (pos - sp.x_pos0)) * DIM;
        if (j == 0) {
          if (!sp.ok && blockIdx.y == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
          ent_out[e] = valid ? (int64_t)b * a.n_new_max : -1;
          ent_row0[e] = e * G;
          ent_b[e] = b;
          ent_g[e] = row;
          atomicMax(&n_ent, e + 1);
          atomicMax(&rows_used, (e + 1) * G);
        }
      } else if (e < SP && j == 0) {
        ent_out[e] = -1;
        ent_row0[e] = e * G;
      }
      row_src[r] = src;
    }
  } else {
    const int b = blockIdx.z;
    const SeqSpan sp = seq_span(a.span, b, a.window.capacity, ent_cap(a));
    const int64_t n_e = sp.ok ? sp.g_hi - sp.g_lo : 0;
    const int64_t e0 = (int64_t)blockIdx.x * E;
    const int E_cta = e0 < n_e ? (int)(n_e - e0 < E ? n_e - e0 : E) : 0;
    const int R = E_cta > 0 ? E_cta * m + G - m : 0;
    const int64_t first_pos = (sp.g_lo + e0) * m + m - G;
    for (int r = tid; r < kRows; r += kThreads) {
      const int64_t pos = first_pos + r;
      row_src[r] = (r < R && pos >= 0) ? ((int64_t)b * a.n_x + (pos - sp.x_pos0)) * DIM : -1;
    }
    for (int e = tid; e < E_cta; e += kThreads) {
      const int64_t row = a.entries.local(sp.g_lo + e0 + e);  // -1: another shard's entry
      ent_out[e] = row >= 0 ? (int64_t)b * a.n_new_max + e0 + e : -1;
      ent_row0[e] = e * m;
      ent_b[e] = b;
      ent_g[e] = row;
    }
    if (tid == 0) {
      n_ent = E_cta;
      rows_used = R;
      if (!sp.ok && blockIdx.x == 0 && blockIdx.y == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
    }
  }
  __syncthreads();
  const int E_cta = n_ent;
  if (E_cta == 0) return;  // uniform

  // ---- x tile (zero for masked rows) and the W chunk (columns c0 .. c0 + NC
  // of W [DIM][DIM]).  bf16: asynchronous 16-byte copies, all in flight at
  // once; fp32: converted to the padded layout through registers.
  const Elem* xg = reinterpret_cast<const Elem*>(a.x);
  const Elem* wg = reinterpret_cast<const Elem*>(a.w);
  constexpr int VEC = 16 / sizeof(Elem);
  const int x_rows = kBf16 ? rows_used : kRows;
  uint8_t* xb = reinterpret_cast<uint8_t*>(xs);
  uint8_t* wb = reinterpret_cast<uint8_t*>(ws);
  if constexpr (kBf16) {  // straight into the swizzled layouts (rows past x_rows are never read back)
    for (int i = tid; i < x_rows * (DIM / VEC); i += kThreads) {
      const int r = i / (DIM / VEC), cv = (i % (DIM / VEC)) * VEC;
      const bool live = row_src[r] >= 0;
      cp_async16(xb + (cv / 64) * (kRows * 128) + swz128(r, (cv % 64) * 2), live ? xg + row_src[r] + cv : xg, live);
    }
    if (!a.gate_logits)
      for (int i = tid; i < DIM * (NC / VEC); i += kThreads) {
        const int k = i / (NC / VEC), cv = (i % (NC / VEC)) * VEC;
        cp_async16(wb + swz128(k, cv * 2), wg + (int64_t)k * DIM + c0 + cv, true);
      }
    cp_async_wait_all();
  } else {
    for (int i = tid; i < x_rows * (DIM / VEC); i += kThreads) {
      const int r = i / (DIM / VEC), cv = (i % (DIM / VEC)) * VEC;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (row_src[r] >= 0) val = *reinterpret_cast<const uint4*>(xg + row_src[r] + cv);
      const float* f = reinterpret_cast<const float*>(&val);
#pragma unroll
      for (int j = 0; j < 4; ++j) xs[r * XS + cv + j] = f[j];
    }
    if (!a.gate_logits)
      for (int i = tid; i < DIM * (NC / VEC); i += kThreads) {
        const int k = i / (NC / VEC), cv = (i % (NC / VEC)) * VEC;
        const uint4 val = *reinterpret_cast<const uint4*>(wg + (int64_t)k * DIM + c0 + cv);
        const float* f = reinterpret_cast<const float*>(&val);
#pragma unroll
        for (int j = 0; j < 4; ++j) ws[k * WS + cv + j] = f[j];
      }
  }
  // rows past the used ones are zero (fp32 path: read by the GEMM's last row block)
  if constexpr (!kBf16)
    for (int i = tid; i < (((x_rows + 15) & ~15) - x_rows) * XS; i += kThreads) xs[x_rows * XS + i] = Elem(0);
  __syncthreads();

  // ---- z = x W for the 128 x NC tile, or the caller's logit rows
  if (a.gate_logits) {
    // u has the rows of x (same element offsets), in float32; masked rows are
    // never read by the softmax below
    const float* ug = reinterpret_cast<const float*>(a.w);
    for (int i = tid; i < x_rows * (NC / 4); i += kThreads) {
      const int r = i / (NC / 4), cv = (i % (NC / 4)) * 4;
      float4 u4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row_src[r] >= 0) u4 = *reinterpret_cast<const float4*>(ug + row_src[r] + c0 + cv);
      zs[r * ZS + cv] = u4.x;
      zs[r * ZS + cv + 1] = u4.y;
      zs[r * ZS + cv + 2] = u4.z;
      zs[r * ZS + cv + 3] = u4.w;
    }
  } else if constexpr (kBf16) {
    // tcgen05: M = 128 token rows, N = 64 channels, K = DIM; x is the K-major
    // A operand, the W chunk the MN-major B operand; z lands in 64 TMEM columns
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tm_slot;
    const int warp = tid / kWarp, lane = tid % kWarp;
    if (tid == 0) {
      sm100::mbar_init(&mma_bar, 1);
      sm100::fence_barrier_init();
    }
    if (warp == 0) sm100::tmem_alloc(&tm_slot, 64);
    sm100::fence_async_smem();  // the cp.async bytes, for the tensor cores
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = tm_slot;
    if (tid == 0) {
      const uint32_t xa = sm100::smem_u32(xb), wa = sm100::smem_u32(wb);
      const uint32_t idesc = sm100::idesc_dense(1, 1, 128, NC, false, true);
#pragma unroll 4
      for (int kk = 0; kk < DIM / 16; ++kk)
        sm100::mma_ss<0>(tmem,
                         sm100::smem_desc(xa + (kk / 4) * (kRows * 128) + (kk % 4) * 32, 16, 1024, sm100::kSw128),
                         sm100::smem_desc(wa + kk * 2048, 8192, 1024, sm100::kSw128), idesc, kk > 0);
      sm100::tc_commit(&mma_bar);
    }
    sm100::mbar_wait(&mma_bar, 0, a.status);
    sm100::tc_fence_after();
    __syncthreads();  // the MMAs are done with the W chunk: z reuses it
    {  // warp w: rows 32 (w % 4) .., columns 32 (w / 4) ..
      uint32_t r[32];
      sm100::tmem_ld_32(tmem + ((uint32_t)(32 * (warp % 4)) << 16) + 32 * (warp / 4), r);
      sm100::tmem_ld_wait(r);
      const int row = 32 * (warp % 4) + lane;
#pragma unroll
      for (int q = 0; q < 32; ++q) zs[row * ZS + 32 * (warp / 4) + q] = __uint_as_float(r[q]);
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      sm100::tc_fence_after();
      sm100::tmem_dealloc(tmem, 64);
    }
  } else {
    constexpr int RG = kThreads / NC;          // row groups
    constexpr int RPT = kRows / RG;            // rows per thread
    const int c = tid % NC, rg = tid / NC;
    float acc[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) acc[i] = 0.f;
    for (int k = 0; k < DIM; ++k) {
      const float wv = ws[k * WS + c];
#pragma unroll
      for (int i = 0; i < RPT; ++i) acc[i] = fmaf(xs[(rg + i * RG) * XS + k], wv, acc[i]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RPT; ++i) zs[(rg + i * RG) * ZS + c] = acc[i];
  }
  // positional biases of the NC channels, [G][NC], behind z in the dead W area
  float* bs = zs + kRows * ZS;
  for (int i = tid; i < G * (NC / 4); i += kThreads) {
    const int j = i / (NC / 4), cv = (i % (NC / 4)) * 4;
    cp_async16(bs + j * NC + cv, a.bpos + (int64_t)j * DIM + c0 + cv, true);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- group softmax over tokens and weighted sum, per (entry, channel)
  // TP threads share one (entry, channel) pair, each taking every TP-th token.
  int TP = kThreads / (E_cta * NC);
  TP = TP < 1 ? 1 : (TP > 32 ? 32 : TP);
  while (TP > 1 && (G % TP != 0)) TP >>= 1;
  {
    int p2 = 1;
    while (p2 * 2 <= TP) p2 *= 2;
    TP = p2;
  }
  const int n_pairs = E_cta * NC;
  const int pairs_per_pass = kThreads / TP;
  for (int pb = 0; pb < n_pairs; pb += pairs_per_pass) {
    const int pair = pb + tid / TP;
    const int sub = tid % TP;
    const bool active = pair < n_pairs && ent_out[pair / NC] >= 0;
    const int e = pair < n_pairs ? pair / NC : 0, c = pair % NC;
    const int r0 = ent_row0[e];
    // tokens j = sub, sub + TP, ...: four at a time.  When the group splits
    // evenly no token index needs a guard, so the loads of the four overlap.
    auto logit = [&](int j, int r) { return zs[r * ZS + c] + bs[j * NC + c]; };
    auto xval = [&](int r) -> float {
      if constexpr (kBf16) {
        const int d = c0 + c;
        return bf16_val(*reinterpret_cast<const uint16_t*>(xb + (d / 64) * (kRows * 128) + swz128(r, (d % 64) * 2)));
      }
      else return xs[r * XS + c0 + c];
    };
    auto ex = [](float v) -> float {
      if constexpr (kBf16) return __expf(v);  // storage is bf16/FP8: the fast exponential is ample
      else return expf(v);
    };
    const bool even = G % (4 * TP) == 0;
    float mx = -INFINITY;
    if (active) {
      for (int j0 = sub; j0 < G; j0 += 4 * TP) {
        float z[4];
        bool live[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u * TP;
          const bool in = even || j < G;
          const int r = r0 + (in ? j : 0);
          z[u] = logit(in ? j : 0, r);
          live[u] = in && row_src[r] >= 0;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (live[u]) mx = fmaxf(mx, z[u]);
      }
    }
    mx = group_max(mx, TP);
    float den = 0.f, num = 0.f;
    if (active) {
      for (int j0 = sub; j0 < G; j0 += 4 * TP) {
        float z[4], xv[4];
        bool live[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u * TP;
          const bool in = even || j < G;
          const int r = r0 + (in ? j : 0);
          z[u] = logit(in ? j : 0, r);
          xv[u] = xval(r);
          live[u] = in && row_src[r] >= 0;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p = live[u] ? ex(z[u] - mx) : 0.f;
          den += p;
          num = fmaf(p, xv[u], num);
        }
      }
    }
    for (int o = TP >> 1; o > 0; o >>= 1) {
      den += __shfl_xor_sync(0xffffffffu, den, o);
      num += __shfl_xor_sync(0xffffffffu, num, o);
    }
    if (active && sub == 0) {
      if constexpr (kFused) pooled_s[e * NC + c] = num / den;
      else a.pooled[ent_out[e] * DIM + c0 + c] = num / den;
    }
  }
  if constexpr (kFused) {
    __syncthreads();
    store_entries<DIM, NC>(a, pooled_s, pamax_s, ent_out, ent_b, ent_g, E_cta, c0);
  }
}

// ------------------------------------------------------------ store kernel
// grid: (ceil((n_new_max + n_win_max) / 8), B); one warp per row.
template <int VPL>
__global__ void __launch_bounds__(256) store_kernel(CompressLaunch a) {
  grid_dep_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int64_t i = (int64_t)blockIdx.x * 8 + warp;
  const SeqSpan sp = seq_span(a.span, b, a.window.capacity, ent_cap(a));
  if (!sp.ok) {
    if (i == 0 && lane == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
    return;
  }
  const int64_t n_e = sp.g_hi - sp.g_lo;
  const int64_t n_w = a.window.data ? sp.w_hi - sp.w_lo : 0;
  constexpr int DIM = VPL * 32;
  float v[VPL];
  if (i < n_e) {
    const int64_t row = a.entries.local(sp.g_lo + i);
    if (row < 0) return;  // another shard's entry
    const float* src = a.pooled + ((int64_t)b * a.n_new_max + i) * DIM + lane * VPL;
#pragma unroll
    for (int j = 0; j < VPL; ++j) v[j] = src[j];
    store_row_warp<VPL>(a.entries, b, row, v, lane);
  } else if (i < n_e + n_w) {
    const int64_t pos = sp.w_lo + (i - n_e);
    const int64_t xr = pos - sp.x_pos0;
    const int64_t base = ((int64_t)b * a.n_x + xr) * DIM + lane * VPL;
#pragma unroll
    for (int j = 0; j < VPL; ++j) v[j] = load_elem(a.x, base + j, a.x_dtype);
    store_row_warp<VPL>(a.window, b, pos % a.window.capacity, v, lane);
    if (pos == 0 && a.sink_tok.data) store_row_warp<VPL>(a.sink_tok, b, 0, v, lane);
  }
}

template <int VPL>
__global__ void __launch_bounds__(256) encode_rows_kernel(const float* rows, int64_t n, int64_t row0,
                                                          CacheView out) {
  grid_dep_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int64_t i = (int64_t)blockIdx.x * 8 + warp;
  if (i >= n) return;
  constexpr int DIM = VPL * 32;
  const float* src = rows + ((int64_t)b * n + i) * DIM + lane * VPL;
  float v[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) v[j] = src[j];
  store_row_warp<VPL>(out, b, row0 + i, v, lane);
}

// The pooled rows are stored by the pool kernel itself when every cluster
// of its grid (the DIM / NC channel blocks of the same entries) can be
// resident at once; otherwise they go through scratch to the store kernel.
template <bool kBf16, int DIM, int NC>
cudaError_t launch_pool(const CompressLaunch& a, int E, cudaStream_t stream, bool* fused) {
  const bool packed = a.span.ctx_len != nullptr && a.n_new_max == 1 && a.span.G <= kRows;
  constexpr size_t smem = pool_smem_bytes<kBf16, DIM, NC>();
  const int SP = kRows / a.span.G < kMaxEnt ? kRows / a.span.G : kMaxEnt;
  const dim3 grid = packed ? dim3((unsigned)((a.B + SP - 1) / SP), DIM / NC, 1)
                           : dim3((unsigned)((a.n_new_max + E - 1) / E), DIM / NC, a.B);
  auto kf = pool_kernel<kBf16, DIM, NC, true>;
  cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = DIM / NC;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kf, &cfg) != cudaSuccess) {
    cudaGetLastError();  // clear: fall back to the unfused path
    max_clusters = 0;
  }
  *fused = (int64_t)grid.x * grid.z <= max_clusters;
  if (*fused) {
    set_pdl(attr[1]);
    cfg.numAttrs = 2;
    return counted(cudaLaunchKernelEx(&cfg, kf, a, E, packed));
  }
  auto ku = pool_kernel<kBf16, DIM, NC, false>;
  e = cudaFuncSetAttribute(ku, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(ku, grid, dim3(kThreads), smem, stream, a, E, packed);
}

}  // namespace

cudaError_t launch_compress(const CompressLaunch& a, cudaStream_t stream) {
  const int m = a.span.m, G = a.span.G;
  int E = (kRows - (G - m)) / m;
  if (E > kMaxEnt) E = kMaxEnt;
  bool fused = false;
  if (a.n_new_max > 0) {
    const bool bf = a.x_dtype == LCSC_DT_BF16;
    cudaError_t e;
    if (bf && a.dim == 512) e = launch_pool<true, 512, 64>(a, E, stream, &fused);
    else if (bf && a.dim == 128) e = launch_pool<true, 128, 64>(a, E, stream, &fused);
    else if (!bf && a.dim == 128) e = launch_pool<false, 128, 64>(a, E, stream, &fused);
    else if (!bf && a.dim == 32) e = launch_pool<false, 32, 32>(a, E, stream, &fused);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
  }
  if (fused) return cudaSuccess;  // entries and window rows were stored
  const int rows = a.n_new_max + (a.window.data ? a.n_win_max : 0);
  if (rows == 0) return cudaSuccess;
  dim3 grid((unsigned)((rows + 7) / 8), a.B);
  switch (a.dim) {
    case 512: return launch_pdl(store_kernel<16>, grid, dim3(256), 0, stream, a);
    case 128: return launch_pdl(store_kernel<4>, grid, dim3(256), 0, stream, a);
    case 32: return launch_pdl(store_kernel<1>, grid, dim3(256), 0, stream, a);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_encode_rows(const float* rows, int B, int64_t n, int64_t row0,
                               const CacheView& out, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  dim3 grid((unsigned)((n + 7) / 8), B);
  switch (out.f.dim) {
    case 512: return launch_pdl(encode_rows_kernel<16>, grid, dim3(256), 0, stream, rows, n, row0, out);
    case 128: return launch_pdl(encode_rows_kernel<4>, grid, dim3(256), 0, stream, rows, n, row0, out);
    case 32: return launch_pdl(encode_rows_kernel<1>, grid, dim3(256), 0, stream, rows, n, row0, out);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lcsc
