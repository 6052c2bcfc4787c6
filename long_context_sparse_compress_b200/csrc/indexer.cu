// Lightning-indexer scoring and exact top-k selection.
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works" (low-rank indexer queries against
// compressed indexer keys; each query keeps its top-k entries); "Inside
// DeepSeek-V4" (llmbytes.dev), section 1 (FP4 indexer, top-1,024).
//   s[g] = sum_h w[h] * ReLU(q~[h] . k~[g]),  g < N(p) = floor((p + 1) / m)
// with q~ the indexer query stored in the key format.
//
// FP8 and FP4 keys are scored on the tensor cores (indexer_mma.cu), fp32 keys
// here.  Scoring keeps the stored codes unscaled in the dot products and
// applies the scales afterwards: FP8 rows have one scale per row, so
// q~[h].k~[g] = sq[h] * sk[g] * (codes . codes); FP4 rows have one scale per
// 16-block, applied per block.  ReLU commutes with the positive scales.
//
// Top-k is an exact radix select on the order-preserving integer image of
// the float scores, three digits of 12 / 12 / 8 bits:
//   digit 1: histogrammed while the scores are written (tensor-core scoring)
//          or by a pass over them; the threshold bin is found by the CTA
//          that scored the list alone, else by the collect pass (several
//          tensor-core scoring CTAs per list), else by the pass's last CTA;
//   collect (all slices of a list): scores above the threshold bin are
//          marked in the list's selection bitmap, those in it become
//          candidates;
//   final (one CTA per list): digits 2 and 3 over the candidates (held in
//          shared memory), ties to the lowest index, the chosen ones marked,
//          and the bitmap compacted into the output in index order.
#include "kernels.cuh"
#include "launches.h"
#include "sm100.cuh"
#include "topk.cuh"

namespace lcsc {
namespace {

constexpr int kBins = kTopkBins;

// Key rows query t of sequence b scores: its N(p) visible entries, or for an
// entry shard those of them the shard holds (at most n_max).  An unsharded
// context length that would reach past the n_max entries the call was sized
// for is invalid: nothing is scored or selected for it, and the status flags
// it.
__device__ __forceinline__ int64_t visible(const IndexLaunch& a, int b, int t, bool* ok) {
  const int64_t L = a.ctx_len[b];
  const int64_t p = L - a.T + t;
  const bool shard = a.keys.rows > 0;
  *ok = L >= a.T && (shard || L / a.m <= a.n_max);
  if (!*ok) return 0;
  const int64_t n = a.keys.local_count((p + 1) / a.m);
  return shard && n > a.n_max ? a.n_max : n;
}

// ------------------------------------------------ indexer query quantisation
// One warp per (b, t, h) row: the query row is stored in the key format.
template <int VPL>
__global__ void __launch_bounds__(256) quantize_queries_kernel(IndexLaunch a, bool zero_hist) {
  grid_dep_wait();
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  {  // the top-k's counters, and the digit-1 histograms when they are summed in memory, start at zero
    const int64_t lists = (int64_t)a.B * a.T;
    const int64_t nh = zero_hist ? lists * kTopkBins : 0;
    const int64_t n_zero = nh + lists * 8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_zero; i += (int64_t)gridDim.x * blockDim.x) {
      if (i < nh) a.hist[(i / kTopkBins) * 2 * kTopkBins + i % kTopkBins] = 0u;
      else a.counters[i - nh] = 0u;
    }
  }
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;  // over B*T*H_I
  const int64_t per_b = (int64_t)a.T * a.H_I;
  if (row >= (int64_t)a.B * per_b) return;
  const int b = (int)(row / per_b);
  const int64_t r = row % per_b;
  float v[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) v[j] = load_elem(a.q_idx, row * (VPL * 32) + lane * VPL + j, a.q_dtype);
  store_row_warp<VPL>(a.q_store, b, r, v, lane);
}

// --------------------------------------------------------------- scoring
// CUDA-core scoring of fp32 keys (FP8 and FP4 keys are scored on the tensor
// cores).  grid (ceil(n_max / 64), B*T); block 256 = 64 keys x 4 head groups.
template <int DI, int HI>
__global__ void __launch_bounds__(256) score_kernel(IndexLaunch a) {
  grid_dep_wait();
  constexpr int KEYS = 64;
  constexpr int HG = HI < 4 ? HI : 4;
  constexpr int HPT = HI / HG;
  constexpr int QS = DI + 1;
  __shared__ float qs[HI * QS];
  __shared__ float wq[HI];

  const int list = blockIdx.y;
  const int b = list / a.T, t = list % a.T;
  bool ok;
  const int64_t n = visible(a, b, t, &ok);
  const int64_t g0 = (int64_t)blockIdx.x * KEYS;
  if (g0 >= n) return;
  const int tid = threadIdx.x;

  for (int i = tid; i < HI * DI; i += 256) {
    const int h = i / DI, c = i % DI;
    qs[h * QS + c] = reinterpret_cast<const float*>(a.q_store.row(b, (int64_t)t * HI + h))[c];
  }
  for (int i = tid; i < HI; i += 256) wq[i] = a.w_idx[(int64_t)list * HI + i];
  __syncthreads();

  const int kk = tid / HG, hg = tid % HG;
  const int64_t g = g0 + kk;
  const bool live = g < n;
  float acc[HPT];
#pragma unroll
  for (int i = 0; i < HPT; ++i) acc[i] = 0.f;
  if (live) {
    const float4* krow = reinterpret_cast<const float4*>(a.keys.row(b, g));
#pragma unroll 1
    for (int blk = 0; blk < DI / 16; ++blk) {
      float kv[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 f = krow[blk * 4 + j];
        kv[4 * j] = f.x; kv[4 * j + 1] = f.y; kv[4 * j + 2] = f.z; kv[4 * j + 3] = f.w;
      }
#pragma unroll
      for (int i = 0; i < HPT; ++i) {
        const float* qrow = qs + (i * HG + hg) * QS + blk * 16;
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) part = fmaf(qrow[j], kv[j], part);
        acc[i] += part;
      }
    }
  }
  float sc = 0.f;
#pragma unroll
  for (int i = 0; i < HPT; ++i) sc = fmaf(wq[i * HG + hg], fmaxf(acc[i], 0.f), sc);
  for (int o = HG >> 1; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
  if (live && hg == 0) a.scores[(int64_t)list * a.stride + g] = sc;
}

// --------------------------------------------------------------- top-k

struct ListInfo {
  int64_t n;
  int64_t k_eff;
  int64_t lo, hi;  // slice
};

__device__ __forceinline__ ListInfo list_info(const IndexLaunch& a, int list, int slices) {
  ListInfo li;
  bool ok;
  li.n = visible(a, list / a.T, list % a.T, &ok);
  li.k_eff = li.n < a.k ? li.n : a.k;
  const int64_t per = ((li.n + slices - 1) / slices + 31) / 32 * 32;  // whole bitmap words
  li.lo = (int64_t)blockIdx.x * per;
  li.hi = li.lo + per < li.n ? li.lo + per : li.n;
  return li;
}

// f(g, score) for every g in [lo, hi) of one score row: four 16-byte loads
// in flight per thread (lo is a multiple of 4 and rows start 16-byte aligned).
template <class F>
__device__ __forceinline__ void scan_scores(const float* s, int64_t lo, int64_t hi, F&& f) {
  const int64_t n4 = hi > lo ? (hi - lo) >> 2 : 0;
  const float4* s4 = reinterpret_cast<const float4*>(s + lo);
  for (int64_t base = 0; base < n4; base += 4 * 512) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = base + u * 512 + threadIdx.x;
      v[u] = i < n4 ? s4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = base + u * 512 + threadIdx.x;
      if (i < n4) {
        const int64_t g = lo + 4 * i;
        f(g, v[u].x);
        f(g + 1, v[u].y);
        f(g + 2, v[u].z);
        f(g + 3, v[u].w);
      }
    }
  }
  for (int64_t g = lo + 4 * n4 + threadIdx.x; g < hi; g += 512) f(g, s[g]);
}

// Digit-1 histogram of one slice of a list (scores written by a kernel that
// did not histogram them); the list's last CTA finds the threshold bin.
__global__ void __launch_bounds__(512) topk_hist_kernel(IndexLaunch a, int slices) {
  grid_dep_wait();
  __shared__ uint32_t h[kBins];
  const int list = blockIdx.y;
  const ListInfo li = list_info(a, list, slices);
  for (int i = threadIdx.x; i < kBins; i += 512) h[i] = 0;
  __syncthreads();
  const float* s = a.scores + (int64_t)list * a.stride;
  if (li.n > a.k) scan_scores(s, li.lo, li.hi, [&](int64_t, float v) { atomicAdd(&h[float_key(v) >> 20], 1u); });
  const int64_t n = li.n;
  hist_finish(h, li.n > a.k, 1, a.hist, a.counters, list, list, gridDim.x, &n, a.k);
}

// All slices of a list: scores above the digit-1 threshold bin go to the
// output, those in it to the candidate list.
__global__ void __launch_bounds__(512) topk_collect_kernel(IndexLaunch a, int slices, bool set_bins) {
  grid_dep_wait();
  extern __shared__ float4 slice_s[];  // the slice's scores, one bulk copy
  __shared__ uint64_t bar;
  constexpr int kLocal = 2048;          // candidates gathered in shared memory first
  __shared__ __align__(16) uint2 cand_s[kLocal];  // (16-byte aligned: also the histogram, read as uint4)
  __shared__ uint32_t n_local, base_g;
  const int list = blockIdx.y;
  const ListInfo li = list_info(a, list, slices);
  const float* s = a.scores + (int64_t)list * a.stride;
  int32_t* out_i = a.out_idx + (int64_t)list * a.k;
  float* out_s = a.out_score ? a.out_score + (int64_t)list * a.k : nullptr;
  if (li.n <= a.k) {  // every visible entry is kept, in index order
    for (int64_t g = li.lo + threadIdx.x; g < li.hi; g += 512) {
      out_i[g] = (int32_t)(g + a.keys.row0);  // global entry number
      if (out_s) out_s[g] = s[g];
    }
    return;
  }
  const int64_t n4 = li.hi > li.lo ? (li.hi - li.lo) >> 2 : 0;  // whole 16-byte groups
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
    n_local = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0 && n4 > 0) {
    sm100::mbar_arrive_expect_tx(&bar, (uint32_t)(n4 * 16));
    sm100::bulk_load(slice_s, s + li.lo, (uint32_t)(n4 * 16), &bar);
  }
  uint32_t* ctr = a.counters + (int64_t)list * 8;
  uint32_t t1;
  if (set_bins) {  // the list's threshold bin from its complete histogram, while the slice loads
    __shared__ uint32_t warp_tot[32];
    __shared__ Thresh res;
    uint32_t* h = reinterpret_cast<uint32_t*>(cand_s);  // free until the scan
    const uint4* hg = reinterpret_cast<const uint4*>(a.hist + (int64_t)list * 2 * kTopkBins);
    static_assert(kTopkBins == 2 * 4 * 512, "two 16-byte loads per thread");
    const uint4 v0 = __ldcg(&hg[threadIdx.x]), v1 = __ldcg(&hg[threadIdx.x + 512]);
    reinterpret_cast<uint4*>(h)[threadIdx.x] = v0;
    reinterpret_cast<uint4*>(h)[threadIdx.x + 512] = v1;
    __syncthreads();
    const Thresh th = block_threshold(h, kTopkBins, (uint32_t)a.k, 256, warp_tot, &res);
    t1 = th.bin;
    if (threadIdx.x == 0 && blockIdx.x == 0) {
      ctr[2] = th.above;
      ctr[3] = th.bin;
    }
  } else {
    t1 = ctr[3];
  }
  uint32_t* bits = a.sel_bits + (int64_t)list * a.bit_stride;
  for (int64_t w = li.lo / 32 + threadIdx.x; w < (li.hi + 31) / 32; w += 512) bits[w] = 0u;
  __syncthreads();
  uint32_t* cand = a.cand + (int64_t)list * 2 * a.cand_cap;  // (index, key) pairs
  // above the bin: a mark (no reply awaited); in it: a shared-memory slot,
  // or past kLocal a workspace slot of its own
  auto visit = [&](int64_t g, float v) {
    const uint32_t key = float_key(v);
    const uint32_t d1 = key >> 20;
    if (d1 > t1) atomicOr(&bits[g >> 5], 1u << (g & 31));
    if (d1 == t1) {
      const uint32_t c = atomicAdd(&n_local, 1u);
      if (c < (uint32_t)kLocal) {
        cand_s[c] = make_uint2((uint32_t)g, key);
      } else {
        const uint32_t cg = atomicAdd(&ctr[1], 1u);
        if (cg < a.cand_cap) reinterpret_cast<uint2*>(cand)[cg] = make_uint2((uint32_t)g, key);
      }
    }
  };
  if (n4 > 0 && sm100::mbar_wait(&bar, 0, a.status)) {
    // whole warps step together; one vote per four scores, and only a warp
    // holding a score at or above the bin takes the per-score path
    for (int64_t i0 = 0; i0 < n4; i0 += 512) {
      const int64_t i = i0 + threadIdx.x;
      const bool in = i < n4;
      const float4 v = in ? slice_s[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      const bool hit = in && ((float_key(v.x) >> 20) >= t1 || (float_key(v.y) >> 20) >= t1 ||
                              (float_key(v.z) >> 20) >= t1 || (float_key(v.w) >> 20) >= t1);
      if (__any_sync(0xffffffffu, hit) && in) {
        const int64_t g = li.lo + 4 * i;
        visit(g, v.x);
        visit(g + 1, v.y);
        visit(g + 2, v.z);
        visit(g + 3, v.w);
      }
    }
  }
  for (int64_t g = li.lo + 4 * n4 + threadIdx.x; g < li.hi; g += 512) visit(g, s[g]);
  // the shared-memory candidates: one reservation for the CTA, then a copy
  __syncthreads();
  const uint32_t nl = n_local < (uint32_t)kLocal ? n_local : (uint32_t)kLocal;
  if (threadIdx.x == 0) base_g = nl ? atomicAdd(&ctr[1], nl) : 0u;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < nl; i += 512)
    if (base_g + i < a.cand_cap) reinterpret_cast<uint2*>(cand)[base_g + i] = cand_s[i];
}

// Smallest index bound tau such that at least `need` of the tied candidates
// (key == tkey) have index < tau: ties then go to the lowest indices, as in
// a stable sort.  512 threads; returns n when every tied candidate is needed.
// `each(f)` calls f(index, key) for this thread's share of the candidates.
template <class Each>
__device__ uint32_t tie_bound(Each each, uint32_t tkey, uint32_t need, uint32_t n, uint32_t* cnt) {
  uint32_t lo = 0, hi = n;  // count(idx < hi) >= need holds for hi = n
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo) / 2;
    if (threadIdx.x == 0) *cnt = 0;
    __syncthreads();
    uint32_t local = 0;
    each([&](uint32_t g, uint32_t key) { local += (g < mid && key == tkey) ? 1u : 0u; });
    if (local) atomicAdd(cnt, local);
    __syncthreads();
    const uint32_t total = *cnt;
    __syncthreads();
    if (total >= need) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

constexpr int kCandCap = 12288;  // candidates held in shared memory (keys + indices: 96 KB)
constexpr size_t kFinalSmem = (size_t)kCandCap * 8;

// One CTA per list: digits 2 and 3 over the candidates (the scores in the
// digit-1 threshold bin), ties to the lowest index; the chosen candidates
// join the collect pass's marks in the bitmap, which is then compacted into
// the output (index order).
__global__ void __launch_bounds__(512) topk_final_kernel(IndexLaunch a) {
  grid_dep_wait();
  __shared__ uint32_t h[kBins];
  __shared__ Thresh th;
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t cnt;
  __shared__ uint32_t warp_sum[16];
  extern __shared__ uint32_t dyn[];
  uint32_t* ck = dyn;              // candidate keys
  uint32_t* cg = dyn + kCandCap;   // candidate indices
  const int list = blockIdx.x;
  const int tid = threadIdx.x;
  bool ok;
  const int64_t n = visible(a, list / a.T, list % a.T, &ok);
  if (!ok && tid == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
  const int64_t k_eff = n < a.k ? n : a.k;
  int32_t* out_i = a.out_idx + (int64_t)list * a.k;
  float* out_s = a.out_score ? a.out_score + (int64_t)list * a.k : nullptr;
  for (int64_t j = k_eff + tid; j < a.k; j += 512) {
    out_i[j] = -1;
    if (out_s) out_s[j] = -INFINITY;
  }
  if (n <= a.k) return;  // every visible entry was written in order by the collect pass
  const uint32_t* ctr = a.counters + (int64_t)list * 8;
  const uint32_t need2 = (uint32_t)k_eff - ctr[2];  // >= 1 by construction
  const uint32_t t1 = ctr[3];
  const uint32_t n_cand = ctr[1];
  const uint2* cand = reinterpret_cast<const uint2*>(a.cand + (int64_t)list * 2 * a.cand_cap);
  const float* s = a.scores + (int64_t)list * a.stride;
  uint32_t* bits = a.sel_bits + (int64_t)list * a.bit_stride;
  const bool cached = n_cand <= (uint32_t)kCandCap;
  if (cached) {  // eight pairs in flight per thread
    for (uint32_t c0 = 0; c0 < n_cand; c0 += 8 * 512) {
      uint2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t c = c0 + u * 512 + tid;
        v[u] = c < n_cand ? cand[c] : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t c = c0 + u * 512 + tid;
        if (c < n_cand) {
          cg[c] = v[u].x;
          ck[c] = v[u].y;
        }
      }
    }
  }
  // Candidates: in shared memory, else the workspace list, else (a list
  // that overflowed the workspace) every score of the row in the bin again.
  const int mode = cached ? 0 : (n_cand <= (uint32_t)a.cand_cap ? 1 : 2);
  auto each = [&](auto&& f) {
    if (mode == 0) {
      for (uint32_t c = tid; c < n_cand; c += 512) f(cg[c], ck[c]);
    } else if (mode == 1) {
      for (uint32_t c = tid; c < n_cand; c += 512) {
        const uint2 v = cand[c];
        f(v.x, v.y);
      }
    } else {
      for (int64_t g = tid; g < n; g += 512) {
        const uint32_t key = float_key(s[g]);
        if ((key >> 20) == t1) f((uint32_t)g, key);
      }
    }
  };
  auto threshold = [&](int nbins, uint32_t need) { return block_threshold(h, nbins, need, 512, warp_tot, &th); };
  // digit 2 (key bits 8 .. 19)
  for (int i = tid; i < kBins; i += 512) h[i] = 0;
  __syncthreads();
  each([&](uint32_t, uint32_t key) { atomicAdd(&h[(key >> 8) & 0xFFF], 1u); });
  __syncthreads();
  const Thresh t2 = threshold(kBins, need2);
  const uint32_t need3 = need2 - t2.above;
  // digit 3 (key bits 0 .. 7) inside the digit-2 threshold bin
  for (int i = tid; i < kBins; i += 512) h[i] = 0;
  __syncthreads();
  each([&](uint32_t, uint32_t key) {
    if (((key >> 8) & 0xFFF) == t2.bin) atomicAdd(&h[key & 0xFF], 1u);
  });
  __syncthreads();
  const Thresh t3 = threshold(256, need3);
  const uint32_t ties = need3 - t3.above;
  const uint32_t n_tied = h[t3.bin];
  __syncthreads();
  const uint32_t tkey = (t1 << 20) | (t2.bin << 8) | t3.bin;
  uint32_t tau = (uint32_t)n;  // ties go to the lowest indices
  if (n_tied > ties) tau = tie_bound(each, tkey, ties, (uint32_t)n, &cnt);
  each([&](uint32_t g, uint32_t key) {
    if (key > tkey || (key == tkey && g < tau)) atomicOr(&bits[g >> 5], 1u << (g & 31));
  });
  __syncthreads();
  // compaction: thread t owns bitmap words [16 t, 16 t + 16) of each 8192-word block
  const int64_t words = (n + 31) / 32;
  uint32_t base = 0;
  for (int64_t w0 = 0; w0 < words; w0 += 16 * 512) {
    const int64_t wt = w0 + 16 * tid;
    uint32_t wv[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = wt + 4 * q < words ? __ldcg(reinterpret_cast<const uint4*>(bits + wt) + q) : make_uint4(0, 0, 0, 0);
      wv[4 * q] = v.x;
      wv[4 * q + 1] = v.y;
      wv[4 * q + 2] = v.z;
      wv[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (wt + q >= words) wv[q] = 0u;  // past the list's last word (never cleared)
    uint32_t local = 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) local += __popc(wv[q]);
    // exclusive scan of `local` over the 512 threads
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if ((tid & 31) >= o) incl += v;
    }
    if ((tid & 31) == 31) warp_sum[tid >> 5] = incl;
    __syncthreads();
    uint32_t before = 0, block_total = 0;
    for (int w = 0; w < 16; ++w) {
      const uint32_t ws = warp_sum[w];
      if (w < (tid >> 5)) before += ws;
      block_total += ws;
    }
    uint32_t off = base + before + incl - local;
#pragma unroll
    for (int q = 0; q < 16; ++q) {  // unrolled: wv stays in registers
      uint32_t bw = wv[q];
      while (bw) {
        const int bit = __ffs(bw) - 1;
        bw &= bw - 1;
        const int64_t g = (wt + q) * 32 + bit;
        if (off < (uint32_t)k_eff) out_i[off] = (int32_t)(g + a.keys.row0);
        ++off;
      }
    }
    base += block_total;
    __syncthreads();
  }
  if (out_s) {  // the scores, gathered once every index is out (independent loads)
    __syncthreads();
    for (int64_t jj = tid; jj < k_eff; jj += 512) {
      const int64_t g = (int64_t)out_i[jj] - a.keys.row0;
      out_s[jj] = (out_i[jj] >= 0 && g >= 0 && g < n) ? s[g] : -INFINITY;
    }
  }
}

}  // namespace

cudaError_t launch_index_quantize(const IndexLaunch& a, cudaStream_t stream) {
  const int lists = a.B * a.T;
  const int64_t q_rows = (int64_t)lists * a.H_I;
  const unsigned qgrid = (unsigned)((q_rows + 7) / 8);
  // tensor-core scoring with one CTA per list group keeps its histograms in
  // shared memory: the global ones are then never read
  const bool zero_hist = !index_mma_supported(a) || index_bins_in_collect(a) || !index_whole_lists(a);
  switch (a.d_I) {
    case 128: return launch_pdl(quantize_queries_kernel<4>, dim3(qgrid), dim3(256), 0, stream, a, zero_hist);
    case 32: return launch_pdl(quantize_queries_kernel<1>, dim3(qgrid), dim3(256), 0, stream, a, zero_hist);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_index_scores(const IndexLaunch& a, cudaStream_t stream) {
  cudaError_t e = launch_index_quantize(a, stream);
  if (e != cudaSuccess) return e;
  return launch_index_score_only(a, stream);
}

cudaError_t launch_index_score_only(const IndexLaunch& a, cudaStream_t stream) {
  const int lists = a.B * a.T;
  if (index_mma_supported(a)) return launch_index_mma(a, stream);
  dim3 sgrid((unsigned)((a.n_max + 63) / 64), lists);
  if (a.keys.f.fmt == LCSC_FMT_F32 && a.d_I == 32 && a.H_I == 4)
    return launch_pdl(score_kernel<32, 4>, sgrid, dim3(256), 0, stream, a);
  return cudaErrorInvalidValue;
}

cudaError_t launch_topk(const IndexLaunch& a, cudaStream_t stream) {
  // the histograms and counters were zeroed by the query quantisation of
  // the scoring launch; tensor-core scoring also built the digit-1 histogram
  const int lists = a.B * a.T;
  cudaError_t e;
  int slices = (int)((a.n_max + 16383) / 16384);
  if (slices < 1) slices = 1;
  dim3 tgrid(slices, lists);
  if (!index_mma_supported(a)) {
    if ((e = launch_pdl(topk_hist_kernel, tgrid, dim3(512), 0, stream, a, slices)) != cudaSuccess) return e;
  }
  // the collect pass copies each slice into shared memory in one bulk copy
  const int64_t per_max = ((a.n_max + slices - 1) / slices + 31) / 32 * 32;
  const size_t slice_bytes = (size_t)per_max * 4;
  e = cudaFuncSetAttribute(topk_collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)slice_bytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(topk_collect_kernel, tgrid, dim3(512), slice_bytes, stream, a, slices, index_bins_in_collect(a));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(topk_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFinalSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_final_kernel, dim3(lists), dim3(512), kFinalSmem, stream, a);
}

cudaError_t launch_index_topk(const IndexLaunch& a, cudaStream_t stream) {
  cudaError_t e = launch_index_scores(a, stream);
  if (e != cudaSuccess) return e;
  return launch_topk(a, stream);
}

}  // namespace lcsc
