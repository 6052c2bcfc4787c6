// Merges of the results of entry shards: one long sequence whose compressed
// entries are split by range over several GPUs ("Inside DeepSeek-V4",
// section 1: top-1,024 selection over the entries of a 1M-token context).
// Each shard scores and selects among its own entries and attends to its
// share of the row set; these kernels give back the answer of one GPU
// holding every entry:
//  * topk_merge_kernel: the k best of the shards' candidate lists (each the
//    exact top-k of its range, so the global top-k is among them);
//  * attn_merge_kernel: the shards' softmax-normalised outputs and
//    log-sum-exps folded into one softmax, with the sink logit added to the
//    denominator once and the output's inverse RoPE applied once.
#include "kernels.cuh"
#include "launches.h"
#include "rope.cuh"
#include "topk.cuh"

namespace lcsc {
namespace {

constexpr int kMergeThreads = 512;

// One CTA per list: the candidates of every part go to shared memory as
// 64-bit keys (score key << 32 | ~index, so that a larger score wins and, for
// equal scores, the lower index); a radix select over the eight bytes finds
// the k_eff-th largest key, and the candidates at or above it are written in
// the parts' order (index order when the parts are shards in range order and
// each part's list is index-ordered).
__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(TopkMergeLaunch a) {
  grid_dep_wait();
  extern __shared__ uint64_t ck[];  // [n_parts * k] candidate keys (0: none)
  __shared__ uint32_t h[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ Thresh th;
  __shared__ uint32_t n_valid, scan_s[kMergeThreads / 32];
  const int list = blockIdx.x, tid = threadIdx.x;
  const int64_t total = (int64_t)a.n_parts * a.k;
  if (tid == 0) n_valid = 0;
  __syncthreads();
  uint32_t my_valid = 0;
  for (int64_t c = tid; c < total; c += kMergeThreads) {
    const int64_t part = c / a.k, j = c % a.k;
    const int64_t src = (part * a.lists + list) * a.k + j;
    const int32_t g = a.part_idx[src];
    uint64_t key = 0;
    if (g >= 0) {
      key = ((uint64_t)float_key(a.part_score[src]) << 32) | (uint64_t)(~(uint32_t)g);
      ++my_valid;
    }
    ck[c] = key;
  }
  atomicAdd(&n_valid, my_valid);
  __syncthreads();
  const int64_t k_eff = (int64_t)n_valid < a.k ? (int64_t)n_valid : a.k;
  // radix select of the k_eff-th largest key, most significant byte first
  uint64_t prefix = 0, pmask = 0;
  uint32_t need = (uint32_t)k_eff;
  for (int byte = 7; byte >= 0 && need > 0; --byte) {
    for (int i = tid; i < 256; i += kMergeThreads) h[i] = 0;
    __syncthreads();
    for (int64_t c = tid; c < total; c += kMergeThreads) {
      const uint64_t key = ck[c];
      if (key != 0 && (key & pmask) == prefix) atomicAdd(&h[(key >> (8 * byte)) & 0xFF], 1u);
    }
    __syncthreads();
    const Thresh t = block_threshold(h, 256, need, kMergeThreads, warp_tot, &th);
    prefix |= (uint64_t)t.bin << (8 * byte);
    pmask |= (uint64_t)0xFF << (8 * byte);
    need -= t.above;
  }
  // keys are distinct (distinct indices), so exactly k_eff are >= prefix;
  // compaction in candidate order by a block scan of the selection flags
  int32_t* out_i = a.out_idx + (int64_t)list * a.k;
  float* out_s = a.out_score ? a.out_score + (int64_t)list * a.k : nullptr;
  uint32_t base = 0;
  for (int64_t c0 = 0; c0 < total; c0 += kMergeThreads) {
    const int64_t c = c0 + tid;
    const uint64_t key = c < total ? ck[c] : 0;
    const bool sel = k_eff > 0 && key != 0 && key >= prefix;
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    const int lane = tid & 31, w = tid >> 5;
    if (lane == 0) scan_s[w] = __popc(bal);
    __syncthreads();
    uint32_t before = base;
    for (int i = 0; i < w; ++i) before += scan_s[i];
    uint32_t block_total = 0;
    for (int i = 0; i < kMergeThreads / 32; ++i) block_total += scan_s[i];
    if (sel) {
      const uint32_t off = before + __popc(bal & ((1u << lane) - 1u));
      const int64_t part = c / a.k, j = c % a.k;
      const int64_t src = (part * a.lists + list) * a.k + j;
      if (off < (uint32_t)a.k) {
        out_i[off] = a.part_idx[src];
        if (out_s) out_s[off] = a.part_score[src];
      }
    }
    base += block_total;
    __syncthreads();
  }
  for (int64_t j = k_eff + tid; j < a.k; j += kMergeThreads) {
    out_i[j] = -1;
    if (out_s) out_s[j] = -INFINITY;
  }
}

// grid (lists, H / 4); block 4 heads x Dv / 4 threads, four dims each.  Part r
// holds o_r (normalised over its rows) and lse_r (-inf: no rows); the merged
// row is sum_r e^{lse_r - M} o_r / (e^{sigma - M} + sum_r e^{lse_r - M}).
template <int DV>
__global__ void __launch_bounds__(DV) attn_merge_kernel(AttnMergeLaunch a) {
  grid_dep_wait();
  constexpr int TPH = DV / 4;
  const int list = blockIdx.x;
  const int h = blockIdx.y * 4 + threadIdx.x / TPH;
  const int d4 = threadIdx.x % TPH;
  const float sigma = a.sink ? a.sink[h] : -INFINITY;
  float M = sigma;
  for (int r = 0; r < a.n_parts; ++r) M = fmaxf(M, a.part_lse[((int64_t)r * a.lists + list) * a.H + h]);
  float den = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M > -INFINITY) {
    den = sigma > -INFINITY ? expf(sigma - M) : 0.f;
    for (int r = 0; r < a.n_parts; ++r) {
      const int64_t row = ((int64_t)r * a.lists + list) * a.H + h;
      const float l = a.part_lse[row];
      if (l == -INFINITY) continue;
      const float f = expf(l - M);
      den += f;
      float v[4];
      if (a.dtype == LCSC_DT_BF16) {
        const uint2 raw = reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a.part_out) + row * DV)[d4];
        v[0] = bf16_val((uint16_t)(raw.x & 0xFFFF));
        v[1] = bf16_val((uint16_t)(raw.x >> 16));
        v[2] = bf16_val((uint16_t)(raw.y & 0xFFFF));
        v[3] = bf16_val((uint16_t)(raw.y >> 16));
      } else {
        const float4 f4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.part_out) + row * DV)[d4];
        v[0] = f4.x, v[1] = f4.y, v[2] = f4.z, v[3] = f4.w;
      }
      acc.x = fmaf(f, v[0], acc.x);
      acc.y = fmaf(f, v[1], acc.y);
      acc.z = fmaf(f, v[2], acc.z);
      acc.w = fmaf(f, v[3], acc.w);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float4 o4 = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  RopePair2 rot;
  const int64_t pos = (int64_t)a.ctx_len[list / a.T] - a.T + list % a.T;
  if (inverse_rope_angles(4 * d4, DV, a.out_rope_dim, a.out_rope_base, pos, &rot)) o4 = rotate2(o4, rot);
  const int64_t oi = ((int64_t)list * a.H + h) * DV + 4 * d4;
  if (a.dtype == LCSC_DT_BF16) {
    uint16_t* out = reinterpret_cast<uint16_t*>(a.out) + oi;
    out[0] = bf16_code(o4.x);
    out[1] = bf16_code(o4.y);
    out[2] = bf16_code(o4.z);
    out[3] = bf16_code(o4.w);
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + oi) = o4;
  }
  if (a.lse && d4 == 0) a.lse[(int64_t)list * a.H + h] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace

cudaError_t launch_topk_merge(const TopkMergeLaunch& a, cudaStream_t stream) {
  const size_t smem = sizeof(uint64_t) * (size_t)a.n_parts * (size_t)a.k;
  cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_merge_kernel, dim3((unsigned)a.lists), dim3(kMergeThreads), smem, stream, a);
}

cudaError_t launch_attn_merge(const AttnMergeLaunch& a, cudaStream_t stream) {
  const dim3 grid((unsigned)a.lists, (unsigned)(a.H / 4));
  switch (a.Dv) {
    case 512: return launch_pdl(attn_merge_kernel<512>, grid, dim3(512), 0, stream, a);
    case 128: return launch_pdl(attn_merge_kernel<128>, grid, dim3(128), 0, stream, a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lcsc
