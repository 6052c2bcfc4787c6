// Lightning-indexer scoring and exact top-k selection.
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works" (low-rank indexer queries against
// compressed indexer keys; each query keeps its top-k entries); "Inside
// DeepSeek-V4" (llmbytes.dev), section 1 (FP4 indexer, top-1,024).
//   s[g] = sum_h w[h] * ReLU(q~[h] . k~[g]),  g < N(p) = floor((p + 1) / m)
// with q~ the indexer query stored in the key format.
//
// Scoring keeps the stored codes unscaled in the dot products and applies
// the scales afterwards: FP8 rows have one scale per row, so
// q~[h].k~[g] = sq[h] * sk[g] * (codes . codes); FP4 rows have one scale per
// 16-block, applied per block.  ReLU commutes with the positive scales.
//
// Top-k is an exact radix select on the order-preserving integer image of
// the float scores, three digits of 12 / 12 / 8 bits:
//   pass 1 (all slices of a list): histogram of digit 1;
//   pass 2 (all slices): every score above the threshold bin goes straight to
//          the output, scores in the threshold bin become candidates and are
//          histogrammed on digit 2;
//   pass 3 (one CTA per list): digits 2 and 3 over the candidates; ties at
//          the final threshold are taken in arbitrary order.
#include "kernels.cuh"

namespace lcsc {
namespace {

constexpr int kBins = 4096;

// Entries visible to query t of sequence b.  A context length that would
// reach past the n_max entries the call was sized for is invalid: nothing is
// scored or selected for it, and the status flags it.
__device__ __forceinline__ int64_t visible(const IndexLaunch& a, int b, int t, bool* ok) {
  const int64_t L = a.ctx_len[b];
  const int64_t p = L - a.T + t;
  *ok = L >= a.T && L / a.m <= a.n_max;
  return *ok ? (p + 1) / a.m : 0;
}

// ------------------------------------------------ indexer query quantisation
// One warp per (b, t, h) row: the query row is stored in the key format.
template <int VPL>
__global__ void __launch_bounds__(256) quantize_queries_kernel(IndexLaunch a) {
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
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
// grid (ceil(n_max / 64), B*T); block 256 = 64 keys x 4 head groups.
template <int FMT, int DI, int HI>
__global__ void __launch_bounds__(256) score_kernel(IndexLaunch a) {
  constexpr int KEYS = 64;
  constexpr int HG = HI < 4 ? HI : 4;
  constexpr int HPT = HI / HG;
  constexpr int QS = DI + 1;
  constexpr int NB = DI / 16;
  __shared__ float qs[HI * QS];
  __shared__ float sq[HI * NB];
  __shared__ float wq[HI];

  const int list = blockIdx.y;
  const int b = list / a.T, t = list % a.T;
  bool ok;
  const int64_t n = visible(a, b, t, &ok);
  const int64_t g0 = (int64_t)blockIdx.x * KEYS;
  if (g0 >= n) return;
  const int tid = threadIdx.x;

  // stored query rows (codes, unscaled) and their scales
  for (int i = tid; i < HI * DI; i += 256) {
    const int h = i / DI, c = i % DI;
    const int64_t qr = (int64_t)t * HI + h;
    const uint8_t* row = a.q_store.row(b, qr);
    float v;
    if (FMT == LCSC_FMT_F32) v = reinterpret_cast<const float*>(row)[c];
    else if (FMT == LCSC_FMT_FP8) v = e4m3_val(row[c]);
    else {
      const float2 p = e2m1x2_val(row[c >> 1]);
      v = (c & 1) ? p.y : p.x;
    }
    qs[h * QS + c] = v;
  }
  for (int i = tid; i < HI * NB; i += 256) {
    const int h = i / NB, blk = i % NB;
    const int64_t qr = (int64_t)t * HI + h;
    float s = 1.f;
    if (FMT == LCSC_FMT_FP8) s = *a.q_store.fscale(b, qr);
    else if (FMT == LCSC_FMT_FP4) s = e4m3_val(*a.q_store.bscale_at(b, qr, blk));
    sq[i] = s;
  }
  for (int i = tid; i < HI; i += 256) wq[i] = a.w_idx[(int64_t)list * HI + i];
  __syncthreads();

  const int kk = tid / HG, hg = tid % HG;
  const int64_t g = g0 + kk;
  const bool live = g < n;
  float acc[HPT];
#pragma unroll
  for (int i = 0; i < HPT; ++i) acc[i] = 0.f;
  float sk_row = 1.f;
  if (live) {
    const uint8_t* krow = a.keys.row(b, g);
    if (FMT == LCSC_FMT_FP8) sk_row = *a.keys.fscale(b, g);
#pragma unroll 1
    for (int blk = 0; blk < NB; ++blk) {
      float kv[16];
      if (FMT == LCSC_FMT_F32) {
        const float4* p = reinterpret_cast<const float4*>(krow) + blk * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 f = p[j];
          kv[4 * j] = f.x; kv[4 * j + 1] = f.y; kv[4 * j + 2] = f.z; kv[4 * j + 3] = f.w;
        }
      } else if (FMT == LCSC_FMT_FP8) {
        const uint4 u = reinterpret_cast<const uint4*>(krow)[blk];
        const uint16_t* c2 = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 f = e4m3x2_val(c2[j]);
          kv[2 * j] = f.x; kv[2 * j + 1] = f.y;
        }
      } else {
        const uint2 u = reinterpret_cast<const uint2*>(krow)[blk];
        const uint8_t* c2 = reinterpret_cast<const uint8_t*>(&u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 f = e2m1x2_val(c2[j]);
          kv[2 * j] = f.x; kv[2 * j + 1] = f.y;
        }
      }
      const float skb = FMT == LCSC_FMT_FP4 ? e4m3_val(*a.keys.bscale_at(b, g, blk)) : 1.f;
#pragma unroll
      for (int i = 0; i < HPT; ++i) {
        const int h = i * HG + hg;
        const float* qrow = qs + h * QS + blk * 16;
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) part = fmaf(qrow[j], kv[j], part);
        if (FMT == LCSC_FMT_FP4) acc[i] = fmaf(sq[h * NB + blk] * skb, part, acc[i]);
        else acc[i] += part;
      }
    }
  }
  float sc = 0.f;
#pragma unroll
  for (int i = 0; i < HPT; ++i) {
    const int h = i * HG + hg;
    const float wh = FMT == LCSC_FMT_FP8 ? wq[h] * sq[h * NB] : wq[h];
    sc = fmaf(wh, fmaxf(acc[i], 0.f), sc);
  }
  for (int o = HG >> 1; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
  if (live && hg == 0) a.scores[(int64_t)list * a.n_max + g] = sc * sk_row;
}

// --------------------------------------------------------------- top-k

struct Thresh {
  uint32_t bin;    // threshold bin
  uint32_t above;  // elements in bins above it
};

// Threshold bin of a 4096-bin histogram for `need` (>= 1) elements: the
// largest bin t with sum_{d >= t} hist[d] >= need.  512 threads.
__device__ Thresh find_threshold(const uint32_t* hist_s, uint32_t need, uint32_t* scratch) {
  const int tid = threadIdx.x;  // 512 threads x 8 bins, bins in descending order
  uint32_t local = 0;
  for (int j = 0; j < 8; ++j) local += hist_s[kBins - 1 - (tid * 8 + j)];
  scratch[tid] = local;
  __syncthreads();
  // inclusive scan (Hillis-Steele) over 512 values
  for (int off = 1; off < 512; off <<= 1) {
    uint32_t v = tid >= off ? scratch[tid - off] : 0;
    __syncthreads();
    scratch[tid] += v;
    __syncthreads();
  }
  __shared__ Thresh res;
  const uint32_t incl = scratch[tid];
  const uint32_t excl = incl - local;
  if (excl < need && incl >= need) {
    uint32_t run = excl;
    for (int j = 0; j < 8; ++j) {
      const uint32_t bin = kBins - 1 - (tid * 8 + j);
      const uint32_t c = hist_s[bin];
      if (run + c >= need) {
        res.bin = bin;
        res.above = run;
        break;
      }
      run += c;
    }
  }
  __syncthreads();
  Thresh r = res;
  __syncthreads();
  return r;
}

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
  const int64_t per = (li.n + slices - 1) / slices;
  li.lo = (int64_t)blockIdx.x * per;
  li.hi = li.lo + per < li.n ? li.lo + per : li.n;
  return li;
}

__global__ void __launch_bounds__(512) topk_hist_kernel(IndexLaunch a, int slices) {
  __shared__ uint32_t h[kBins];
  const int list = blockIdx.y;
  const ListInfo li = list_info(a, list, slices);
  if (li.n <= a.k) return;
  for (int i = threadIdx.x; i < kBins; i += 512) h[i] = 0;
  __syncthreads();
  const float* s = a.scores + (int64_t)list * a.n_max;
  for (int64_t g = li.lo + threadIdx.x; g < li.hi; g += 512) atomicAdd(&h[float_key(s[g]) >> 20], 1u);
  __syncthreads();
  uint32_t* gh = a.hist + (int64_t)list * 2 * kBins;
  for (int i = threadIdx.x; i < kBins; i += 512)
    if (h[i]) atomicAdd(&gh[i], h[i]);
}

__global__ void __launch_bounds__(512) topk_collect_kernel(IndexLaunch a, int slices) {
  __shared__ uint32_t h[kBins];
  __shared__ uint32_t scratch[512];
  const int list = blockIdx.y;
  const ListInfo li = list_info(a, list, slices);
  const float* s = a.scores + (int64_t)list * a.n_max;
  int32_t* out_i = a.out_idx + (int64_t)list * a.k;
  float* out_s = a.out_score ? a.out_score + (int64_t)list * a.k : nullptr;
  if (li.n <= a.k) {  // every visible entry is kept
    for (int64_t g = li.lo + threadIdx.x; g < li.hi; g += 512) {
      out_i[g] = (int32_t)g;
      if (out_s) out_s[g] = s[g];
    }
    return;
  }
  uint32_t* gh = a.hist + (int64_t)list * 2 * kBins;
  for (int i = threadIdx.x; i < kBins; i += 512) h[i] = gh[i];
  __syncthreads();
  const Thresh th = find_threshold(h, (uint32_t)li.k_eff, scratch);
  for (int i = threadIdx.x; i < kBins; i += 512) h[i] = 0;
  __syncthreads();
  uint32_t* ctr = a.counters + (int64_t)list * 4;
  uint32_t* cand = a.cand + (int64_t)list * a.n_max;
  for (int64_t g = li.lo + threadIdx.x; g < li.hi; g += 512) {
    const float v = s[g];
    const uint32_t key = float_key(v);
    const uint32_t d1 = key >> 20;
    if (d1 > th.bin) {
      const uint32_t slot = atomicAdd(&ctr[0], 1u);
      out_i[slot] = (int32_t)g;
      if (out_s) out_s[slot] = v;
    } else if (d1 == th.bin) {
      const uint32_t c = atomicAdd(&ctr[1], 1u);
      cand[c] = (uint32_t)g;
      atomicAdd(&h[(key >> 8) & 0xFFF], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh2 = gh + kBins;
  for (int i = threadIdx.x; i < kBins; i += 512)
    if (h[i]) atomicAdd(&gh2[i], h[i]);
  if (blockIdx.x == 0 && threadIdx.x == 0) ctr[2] = th.above;
}

// Smallest index bound tau such that at least `need` of the tied candidates
// (key == tkey) have index < tau: ties then go to the lowest indices, as in
// a stable sort.  512 threads; returns n when every tied candidate is needed.
__device__ uint32_t tie_bound(const uint32_t* cand, uint32_t n_cand, const float* s, uint32_t tkey,
                              uint32_t need, uint32_t n, uint32_t* cnt) {
  uint32_t lo = 0, hi = n;  // count(idx < hi) >= need holds for hi = n
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo) / 2;
    if (threadIdx.x == 0) *cnt = 0;
    __syncthreads();
    uint32_t local = 0;
    for (uint32_t c = threadIdx.x; c < n_cand; c += 512) {
      const uint32_t g = cand[c];
      local += (g < mid && float_key(s[g]) == tkey) ? 1u : 0u;
    }
    if (local) atomicAdd(cnt, local);
    __syncthreads();
    const uint32_t total = *cnt;
    __syncthreads();
    if (total >= need) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

// Sort the k_eff selected (index, score) pairs by index, in shared memory
// (bitonic network over the next power of two, <= 2048).
__device__ void sort_selection(int32_t* out_i, float* out_s, int k_eff, int32_t* si, float* sv) {
  int P = 1;
  while (P < k_eff) P <<= 1;
  for (int j = threadIdx.x; j < P; j += 512) {
    si[j] = j < k_eff ? out_i[j] : INT32_MAX;
    sv[j] = (j < k_eff && out_s) ? out_s[j] : 0.f;
  }
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int j = threadIdx.x; j < P; j += 512) {
        const int partner = j ^ stride;
        if (partner > j) {
          const bool up = (j & size) == 0;
          const int32_t a = si[j], b = si[partner];
          if ((a > b) == up) {
            si[j] = b;
            si[partner] = a;
            const float t = sv[j];
            sv[j] = sv[partner];
            sv[partner] = t;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int j = threadIdx.x; j < k_eff; j += 512) {
    out_i[j] = si[j];
    if (out_s) out_s[j] = sv[j];
  }
}

__global__ void __launch_bounds__(512) topk_final_kernel(IndexLaunch a) {
  __shared__ uint32_t h[kBins];
  __shared__ uint32_t scratch[512];
  __shared__ uint32_t cnt;
  __shared__ int32_t si[2048];
  __shared__ float sv[2048];
  const int list = blockIdx.x;
  bool ok;
  const int64_t n = visible(a, list / a.T, list % a.T, &ok);
  if (!ok && threadIdx.x == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
  const int64_t k_eff = n < a.k ? n : a.k;
  int32_t* out_i = a.out_idx + (int64_t)list * a.k;
  float* out_s = a.out_score ? a.out_score + (int64_t)list * a.k : nullptr;
  for (int64_t j = k_eff + threadIdx.x; j < a.k; j += 512) {
    out_i[j] = -1;
    if (out_s) out_s[j] = -INFINITY;
  }
  if (n <= a.k) return;  // every visible entry was written in order by the collect pass
  uint32_t* ctr = a.counters + (int64_t)list * 4;
  const uint32_t above1 = ctr[2];
  const uint32_t n_cand = ctr[1];
  const uint32_t need = (uint32_t)k_eff - above1;  // >= 1 by construction
  const uint32_t* cand = a.cand + (int64_t)list * a.n_max;
  const float* s = a.scores + (int64_t)list * a.n_max;
  uint32_t* gh2 = a.hist + (int64_t)list * 2 * kBins + kBins;
  for (int i = threadIdx.x; i < kBins; i += 512) h[i] = gh2[i];
  __syncthreads();
  const Thresh t2 = find_threshold(h, need, scratch);
  for (int i = threadIdx.x; i < kBins; i += 512) h[i] = 0;
  __syncthreads();
  // digit 2 above the threshold: keep; at it: histogram digit 3
  for (uint32_t c = threadIdx.x; c < n_cand; c += 512) {
    const uint32_t g = cand[c];
    const float v = s[g];
    const uint32_t key = float_key(v);
    const uint32_t d2 = (key >> 8) & 0xFFF;
    if (d2 > t2.bin) {
      const uint32_t slot = atomicAdd(&ctr[0], 1u);
      out_i[slot] = (int32_t)g;
      if (out_s) out_s[slot] = v;
    } else if (d2 == t2.bin) {
      atomicAdd(&h[key & 0xFF], 1u);
    }
  }
  __syncthreads();
  const uint32_t need3 = need - t2.above;
  const Thresh t3 = find_threshold(h, need3, scratch);
  const uint32_t ties = need3 - t3.above;
  const uint32_t n_tied = h[t3.bin];
  __syncthreads();
  // the threshold key itself: candidate digit 1 is shared; rebuild it from any tied element
  uint32_t tau = (uint32_t)n;
  if (n_tied > ties) {
    // every tied element has the same full key: digit 1 | digit 2 | digit 3
    __shared__ uint32_t tkey;
    if (threadIdx.x == 0) tkey = 0xFFFFFFFFu;
    __syncthreads();
    for (uint32_t c = threadIdx.x; c < n_cand; c += 512) {
      const uint32_t key = float_key(s[cand[c]]);
      if (((key >> 8) & 0xFFF) == t2.bin && (key & 0xFF) == t3.bin) atomicMin(&tkey, key);
    }
    __syncthreads();
    tau = tie_bound(cand, n_cand, s, tkey, ties, (uint32_t)n, &cnt);
  }
  for (uint32_t c = threadIdx.x; c < n_cand; c += 512) {
    const uint32_t g = cand[c];
    const float v = s[g];
    const uint32_t key = float_key(v);
    if (((key >> 8) & 0xFFF) != t2.bin) continue;
    const uint32_t d3 = key & 0xFF;
    if (d3 > t3.bin || (d3 == t3.bin && g < tau)) {
      const uint32_t slot = atomicAdd(&ctr[0], 1u);
      out_i[slot] = (int32_t)g;
      if (out_s) out_s[slot] = v;
    }
  }
  __threadfence_block();
  __syncthreads();
  sort_selection(out_i, out_s, (int)k_eff, si, sv);
}

}  // namespace

cudaError_t launch_index_scores(const IndexLaunch& a, cudaStream_t stream) {
  const int lists = a.B * a.T;
  cudaError_t e;
  const int64_t q_rows = (int64_t)lists * a.H_I;
  const unsigned qgrid = (unsigned)((q_rows + 7) / 8);
  switch (a.d_I) {
    case 128: quantize_queries_kernel<4><<<qgrid, 256, 0, stream>>>(a); break;
    case 32: quantize_queries_kernel<1><<<qgrid, 256, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  if (index_mma_supported(a)) return launch_index_mma(a, stream);
  dim3 sgrid((unsigned)((a.n_max + 63) / 64), lists);
  const int fmt = a.keys.f.fmt;
  if (fmt == LCSC_FMT_F32 && a.d_I == 32 && a.H_I == 4)
    score_kernel<LCSC_FMT_F32, 32, 4><<<sgrid, 256, 0, stream>>>(a);
  else if (fmt == LCSC_FMT_FP8 && a.d_I == 128 && a.H_I == 64)
    score_kernel<LCSC_FMT_FP8, 128, 64><<<sgrid, 256, 0, stream>>>(a);
  else if (fmt == LCSC_FMT_FP4 && a.d_I == 128 && a.H_I == 64)
    score_kernel<LCSC_FMT_FP4, 128, 64><<<sgrid, 256, 0, stream>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_topk(const IndexLaunch& a, cudaStream_t stream) {
  const int lists = a.B * a.T;
  cudaError_t e;
  // histograms and counters start at zero
  e = cudaMemsetAsync(a.hist, 0, sizeof(uint32_t) * (size_t)lists * 2 * kBins, stream);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(a.counters, 0, sizeof(uint32_t) * (size_t)lists * 4, stream);
  if (e != cudaSuccess) return e;
  int slices = (int)((a.n_max + 16383) / 16384);
  if (slices < 1) slices = 1;
  dim3 tgrid(slices, lists);
  topk_hist_kernel<<<tgrid, 512, 0, stream>>>(a, slices);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  topk_collect_kernel<<<tgrid, 512, 0, stream>>>(a, slices);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  topk_final_kernel<<<lists, 512, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_index_topk(const IndexLaunch& a, cudaStream_t stream) {
  cudaError_t e = launch_index_scores(a, stream);
  if (e != cudaSuccess) return e;
  return launch_topk(a, stream);
}

}  // namespace lcsc
