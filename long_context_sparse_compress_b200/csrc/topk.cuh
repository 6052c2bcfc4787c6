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

// Threshold bin of a 4096-bin histogram in shared memory for `need` (>= 1)
// elements: the largest bin t with sum_{d >= t} hist[d] >= need.  Called by
// one whole warp; every lane gets the result.
__device__ __forceinline__ Thresh warp_threshold(const uint32_t* h, uint32_t need) {
  const int lane = threadIdx.x & 31;
  const int top = kTopkBins - 128 * lane;  // lane l owns bins [top - 128, top): descending by lane
  uint32_t local = 0;
  for (int j = 0; j < 128; ++j) local += h[top - 1 - ((j + lane) & 127)];  // skewed: no bank conflicts
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t excl = incl - local;
  const bool mine = excl < need && incl >= need;
  Thresh r{0u, 0u};
  if (mine) {
    uint32_t run = excl;
    for (int d = top - 1; d >= top - 128; --d) {
      const uint32_t c = h[d];
      if (run + c >= need) {
        r.bin = (uint32_t)d;
        r.above = run;
        break;
      }
      run += c;
    }
  }
  const uint32_t owners = __ballot_sync(0xffffffffu, mine);
  if (owners) {
    const int src = __ffs(owners) - 1;
    r.bin = __shfl_sync(0xffffffffu, r.bin, src);
    r.above = __shfl_sync(0xffffffffu, r.above, src);
  }
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
// first k of its n[l] visible scores (lists with n <= k need none).
// `hist_s` is nlists x 4096 words of shared memory; every thread of the CTA
// calls this.
__device__ __forceinline__ void hist_finish(uint32_t* hist_s, bool flush, int nlists, uint32_t* hist_g,
                                            uint32_t* ctr_g, int64_t list0, int64_t done_list,
                                            unsigned total_ctas, const int64_t* n, int64_t k) {
  __shared__ unsigned last_cta;
  __syncthreads();
  if (flush) {
    for (int i = threadIdx.x; i < nlists * kTopkBins; i += blockDim.x) {
      const uint32_t c = hist_s[i];
      if (c) atomicAdd(&hist_g[(list0 + i / kTopkBins) * 2 * kTopkBins + i % kTopkBins], c);
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_cta = atomicAdd(&ctr_g[done_list * 8 + 6], 1u) == total_ctas - 1 ? 1u : 0u;
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  for (int i = threadIdx.x; i < nlists * kTopkBins; i += blockDim.x)
    hist_s[i] = __ldcg(&hist_g[(list0 + i / kTopkBins) * 2 * kTopkBins + i % kTopkBins]);
  __syncthreads();
  if (threadIdx.x < 32) {
    for (int l = 0; l < nlists; ++l) {
      if (n[l] <= k) continue;
      const Thresh t = warp_threshold(hist_s + l * kTopkBins, (uint32_t)k);
      if (threadIdx.x == 0) {
        ctr_g[(list0 + l) * 8 + 2] = t.above;
        ctr_g[(list0 + l) * 8 + 3] = t.bin;
      }
    }
  }
}

}  // namespace lcsc
