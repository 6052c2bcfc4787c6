// Pieces of the exact top-k shared by the scoring kernels (which build the
// first-digit histogram as they write the scores) and the selection kernels.
//
// First digit: the top 12 bits of the order-preserving integer image of the
// score (float_key).  Per list, hist[list][0 .. 4095] counts the visible
// scores per digit and counters[list][8] holds
//   [0] output slots taken, [1] candidates, [2] scores above the threshold
//   bin, [3] the threshold bin, [6] CTAs done with the histogram.
#pragma once

#include "common.cuh"

namespace lcsc {

constexpr int kTopkBins = 4096;

struct Thresh {
  uint32_t bin;    // threshold bin
  uint32_t above;  // elements in bins above it
};

// Threshold bin of an `nbins`-bin histogram in shared memory for `need`
// (>= 1) elements: the largest bin t with sum_{d >= t} hist[d] >= need.
// Every thread of the CTA calls it; threads tid < T (T, or nbins when that
// is smaller: a multiple of 32 that divides nbins, <= blockDim) each sum
// nbins / T consecutive bins (in descending order), a warp scan and a scan
// of the warp totals give each its prefix, and the one whose range holds the
// need walks its bins.  `warp_tot` is 32 words and `res` one Thresh of
// shared memory.
__device__ __forceinline__ Thresh block_threshold(const uint32_t* h, int nbins, uint32_t need, int T,
                                                  uint32_t* warp_tot, Thresh* res) {
  if (T > nbins) T = nbins;  // at least one bin per summing thread
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per = nbins / T;
  const int top = nbins - 1 - tid * per;  // this thread's highest bin
  uint32_t local = 0;
  if (tid < T)
    for (int j = 0; j < per; ++j) local += h[top - j];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (tid == 0) *res = Thresh{0u, 0u};
  if (tid < T && lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (tid < T) {
    uint32_t before = 0;
    for (int i = 0; i < w; ++i) before += warp_tot[i];
    uint32_t run = before + incl - local;
    if (run < need && run + local >= need) {
      for (int j = 0; j < per; ++j) {
        const uint32_t c = h[top - j];
        if (run + c >= need) {
          *res = Thresh{(uint32_t)(top - j), run};
          break;
        }
        run += c;
      }
    }
  }
  __syncthreads();
  const Thresh r = *res;
  __syncthreads();  // `res` and `warp_tot` may be reused right after
  return r;
}

// Slot for this lane in an output list whose length is *counter, taken
// with one atomic per warp.  Lanes with pred false get no slot (the return
// value is meaningless for them).
__device__ __forceinline__ uint32_t warp_append(uint32_t* counter, bool pred) {
  const uint32_t mask = __activemask();
  const uint32_t bal = __ballot_sync(mask, pred);
  if (!bal) return 0u;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(bal) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(counter, (uint32_t)__popc(bal));
  base = __shfl_sync(mask, base, leader);
  return base + (uint32_t)__popc(bal & ((1u << lane) - 1u));
}

// End of a histogram-building CTA: adds its shared histograms of `nlists`
// consecutive lists (from list0) to the global ones, and the last of the
// `total_ctas` CTAs that count on counters[done_list][6] turns the complete
// histograms into each list's threshold bin (counters [2], [3]) for the
// first k of its n[l] visible scores (lists with n <= k need none).  A CTA
// that built its lists' histograms alone (total_ctas 1) sets the bins from
// shared memory directly; with set_bins false the CTAs only add their
// histograms and a later kernel (the collect pass) sets the bins.
// `hist_s` is nlists x 4096 words of shared memory; every thread of the CTA
// calls this.
__device__ __forceinline__ void hist_finish(uint32_t* hist_s, bool flush, int nlists, uint32_t* hist_g,
                                            uint32_t* ctr_g, int64_t list0, int64_t done_list,
                                            unsigned total_ctas, const int64_t* n, int64_t k,
                                            bool set_bins = true) {
  __shared__ unsigned last_cta;
  __shared__ uint32_t warp_tot[32];
  __shared__ Thresh res;
  __syncthreads();
  if (total_ctas == 1) {  // this CTA's histograms are the whole ones: no round trip through memory
    for (int l = 0; l < nlists; ++l) {
      if (n[l] <= k) continue;  // uniform over the CTA
      const Thresh t = block_threshold(hist_s + l * kTopkBins, kTopkBins, (uint32_t)k, 256, warp_tot, &res);
      if (threadIdx.x == 0) {
        ctr_g[(list0 + l) * 8 + 2] = t.above;
        ctr_g[(list0 + l) * 8 + 3] = t.bin;
      }
    }
    return;
  }
  if (flush) {
    for (int i = threadIdx.x; i < nlists * kTopkBins; i += blockDim.x) {
      const uint32_t c = hist_s[i];
      if (c) atomicAdd(&hist_g[(list0 + i / kTopkBins) * 2 * kTopkBins + i % kTopkBins], c);
    }
  }
  if (!set_bins) return;  // the next kernel takes the bins from the flushed histograms
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_cta = atomicAdd(&ctr_g[done_list * 8 + 6], 1u) == total_ctas - 1 ? 1u : 0u;
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  for (int i = threadIdx.x; i < nlists * kTopkBins; i += blockDim.x)
    hist_s[i] = __ldcg(&hist_g[(list0 + i / kTopkBins) * 2 * kTopkBins + i % kTopkBins]);
  __syncthreads();
  for (int l = 0; l < nlists; ++l) {
    if (n[l] <= k) continue;  // uniform over the CTA
    const Thresh t = block_threshold(hist_s + l * kTopkBins, kTopkBins, (uint32_t)k, 256, warp_tot, &res);
    if (threadIdx.x == 0) {
      ctr_g[(list0 + l) * 8 + 2] = t.above;
      ctr_g[(list0 + l) * 8 + 3] = t.bin;
    }
  }
}

}  // namespace lcsc
