// Joint attention on the 5th-generation tensor cores: all 64 query heads of
// one query against one shared 512-d KV row set (FP8 + BF16 RoPE storage).
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works" (exact attention over the selected
// compressed entries plus the uncompressed window, shared-KV multi-query
// layout; the sink enters in the combine step).
//
// One CTA owns (query, range of rows) and walks it in tiles of 128 rows:
//   1. the tile's stored rows are read (gathered by index for CSA) and
//      dequantised once into shared memory as f16, in a 128-byte-swizzled
//      layout that is a K-major operand for Q K^T and an MN-major operand
//      for P V (the same bytes serve as K and as V);
//   2. S = Q K^T on tcgen05 (M = 64 heads, N = 128 rows, K = 512), into TMEM;
//   3. one thread per head reads its S row from TMEM, applies the scale and
//      the row mask, updates its running max (rescaling O only when the max
//      grows by more than e^8) and writes P = exp(S - max) as f16;
//   4. O += P V on tcgen05 (M = 64 heads, N = 2 x 256 dims, K = 128 rows).
// Heads live on M = 64, so S and O use the half-lane TMEM layout: O at
// lanes 0-15 of each 32-lane sub-partition (all 512 columns), S at lanes
// 16-31 (columns 0-127).  The partial (max, sum, O) goes to the same
// workspace the combine kernel merges.
#include "kernels.cuh"
#include "sm100.cuh"

namespace lcsc {
namespace {

using namespace sm100;

constexpr int kH = 64;      // heads (MMA M)
constexpr int kD = 512;     // row length (K of Q K^T, N of P V)
constexpr int kTR = 128;    // rows per tile
constexpr int kThr = 256;
constexpr int kChunks = 36;  // 16-byte chunks of a 576-byte stored row
constexpr int kLoads = kTR * kChunks / kThr;  // 18 chunks per thread per tile
constexpr float kRescale = 8.f;  // rescale O only when the max grows by more

// shared memory (offsets from a 1024-aligned base)
constexpr int OFF_Q = 0;                    // 8 K-blocks [64 heads][128 B]  = 64 KB
constexpr int OFF_K = OFF_Q + 8 * 64 * 128;  // 8 K-blocks [128 rows][128 B] = 128 KB
constexpr int OFF_P = OFF_K + 8 * 128 * 128;  // 2 K-blocks [64 heads][128 B] = 16 KB
constexpr int OFF_BAR = OFF_P + 2 * 64 * 128;  // s_full, pv_done
constexpr int OFF_ROW = OFF_BAR + 64;         // int64 [2][128]
constexpr int OFF_SRC = OFF_ROW + 2 * kTR * 8;  // int32 [2][128]
constexpr int OFF_SCL = OFF_SRC + 2 * kTR * 4;  // float [2][128]
constexpr int OFF_TM = OFF_SCL + 2 * kTR * 4;
constexpr int SMEM = OFF_TM + 16 + 1024;

// Byte offset of (row, byte) in a [rows][128 B] block with the 128-byte swizzle
// (16-byte chunk index XOR row % 8) that TMA and the tensor cores use.
__device__ __forceinline__ uint32_t swz(int row, int byte) {
  return (uint32_t)(row * 128 + ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

struct Rows {
  int64_t n_vis, n_ent_slots, w_lo, n_win;
  bool ok;
};

__device__ __forceinline__ Rows rows_of(const AttnLaunch& a, int b, int t) {
  Rows r;
  const int64_t L = a.ctx_len[b];
  r.ok = L >= a.T && L / a.m <= a.n_max;
  const int64_t p = L - a.T + t;
  r.n_vis = r.ok ? (p + 1) / a.m : 0;
  r.n_ent_slots = a.idx ? a.k : r.n_vis;
  r.w_lo = p - a.w + 1 > 0 ? p - a.w + 1 : 0;
  r.n_win = (r.ok && a.w > 0) ? p - r.w_lo + 1 : 0;
  return r;
}

__global__ void __launch_bounds__(kThr, 1) attn_mma_kernel(const AttnLaunch a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* s_full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* pv_done = s_full + 1;
  int64_t* row_s = reinterpret_cast<int64_t*>(sm + OFF_ROW);
  int32_t* src_s = reinterpret_cast<int32_t*>(sm + OFF_SRC);
  float* scl_s = reinterpret_cast<float*>(sm + OFF_SCL);
  uint32_t* tm_slot = reinterpret_cast<uint32_t*>(sm + OFF_TM);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int list = blockIdx.y;
  const int b = list / a.T, t = list % a.T;
  const Rows qr = rows_of(a, b, t);
  if (!qr.ok && tid == 0 && blockIdx.x == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
  const int64_t total = qr.ok ? qr.n_ent_slots + qr.n_win : 0;
  const int64_t s_lo = (int64_t)blockIdx.x * a.rows_per_split;
  const int64_t s_hi = s_lo + a.rows_per_split < total ? s_lo + a.rows_per_split : total;
  const int ntiles = s_hi > s_lo ? (int)((s_hi - s_lo + kTR - 1) / kTR) : 0;
  const int n_fp8 = a.kv.f.dim - a.kv.f.rope;

  if (tid == 0) {
    mbar_init(s_full, 1);
    mbar_init(pv_done, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tm_slot, 512);

  // ---- Q (64 x 512) -> f16, K-major swizzled blocks of 64 dims
  for (int i = tid; i < kH * (kD / 8); i += kThr) {
    const int h = i / (kD / 8), d0 = (i % (kD / 8)) * 8;
    const int64_t base = ((int64_t)list * a.H + h) * kD + d0;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = load_elem(a.q, base + j, a.q_dtype);
    uint4 u = make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]), pack_h2(v[6], v[7]));
    *reinterpret_cast<uint4*>(sm + OFF_Q + (d0 / 64) * (kH * 128) + swz(h, (d0 % 64) * 2)) = u;
  }

  // ---- tile row resolution (threads 0..127) into buffer `buf`
  auto resolve = [&](int tile, int buf) {
    if (tid < kTR) {
      const int64_t slot = s_lo + (int64_t)tile * kTR + tid;
      int src = 0;
      int64_t row = 0;
      float sc = 1.f;
      if (slot < s_hi) {
        if (slot < qr.n_ent_slots) {
          const int64_t g = a.idx ? (int64_t)a.idx[(int64_t)list * a.k + slot] : slot;
          if (g >= 0 && g < qr.n_vis) {
            src = 1;
            row = g;
            sc = *a.kv.fscale(b, g);
          } else if (g != -1 || !a.idx) {
            if (a.status) atomicOr(a.status, LCSC_DEV_BAD_INDEX);
          }
        } else {
          src = 2;
          row = (qr.w_lo + (slot - qr.n_ent_slots)) % a.win_kv.capacity;
          sc = *a.win_kv.fscale(b, row);
        }
      }
      row_s[buf * kTR + tid] = row;
      src_s[buf * kTR + tid] = src;
      scl_s[buf * kTR + tid] = sc;
    }
  };
  // ---- raw 16-byte chunks of a tile into registers
  uint4 raw[kLoads];
  auto fetch = [&](int buf) {
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      const int idx = tid + i * kThr;
      const int r = idx / kChunks, c = idx % kChunks;
      const int src = src_s[buf * kTR + r];
      raw[i] = make_uint4(0, 0, 0, 0);
      if (src) {
        const CacheView& cv = src == 1 ? a.kv : a.win_kv;
        raw[i] = reinterpret_cast<const uint4*>(cv.row(b, row_s[buf * kTR + r]))[c];
      }
    }
  };
  // ---- dequantise the registers into the f16 K tile
  auto convert = [&](int buf) {
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      const int idx = tid + i * kThr;
      const int r = idx / kChunks, c = idx % kChunks;
      const int byte0 = c * 16;
      if (byte0 < n_fp8) {
        const float s = scl_s[buf * kTR + r];
        const uint16_t* c2 = reinterpret_cast<const uint16_t*>(&raw[i]);
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 f = e4m3x2_val(c2[j]);
          h[j] = pack_h2(f.x * s, f.y * s);
        }
        const int d0 = byte0;  // one byte per value
        uint8_t* blk = sm + OFF_K + (d0 / 64) * (kTR * 128);
        *reinterpret_cast<uint4*>(blk + swz(r, (d0 % 64) * 2)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(blk + swz(r, (d0 % 64) * 2 + 16)) = make_uint4(h[4], h[5], h[6], h[7]);
      } else {
        const uint16_t* bf = reinterpret_cast<const uint16_t*>(&raw[i]);
        uint32_t h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = pack_h2(bf16_val(bf[2 * j]), bf16_val(bf[2 * j + 1]));
        const int d0 = n_fp8 + (byte0 - n_fp8) / 2;
        uint8_t* blk = sm + OFF_K + (d0 / 64) * (kTR * 128);
        *reinterpret_cast<uint4*>(blk + swz(r, (d0 % 64) * 2)) = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
  };

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tm_slot;
  const uint32_t tm_s = tmem + (16u << 16);  // S: lanes 16-31 of each sub-partition
  const bool softmax_thread = warp < 4 && lane >= 16;
  const int head = warp * 16 + (lane & 15);  // warps 0-3: O (lane < 16) / S (lane >= 16) row
  float m_ref = -INFINITY, l_sum = 0.f;
  bool live = true;

  if (ntiles > 0) {
    resolve(0, 0);
    __syncthreads();
    fetch(0);
  }
  const uint32_t idesc_qk = idesc_dense(0, 0, 64, kTR);
  const uint32_t idesc_pv = idesc_dense(0, 0, 64, 256, false, true);
  // `live` stays uniform over the CTA: every bounded wait is folded in at a
  // barrier, so a time-out makes all threads leave the loop together.
  for (int j = 0; j < ntiles; ++j) {
    const int buf = j & 1;
    bool ok = true;
    if (j > 0) ok = mbar_wait(pv_done, (uint32_t)(j - 1) & 1u, a.status);  // K and P smem free
    convert(buf);
    fence_async_smem();
    live = __syncthreads_and(ok) != 0;
    if (!live) break;
    if (tid == 128) {  // ---- S = Q K^T
      tc_fence_after();
      const uint32_t qa = smem_u32(sm + OFF_Q), ka = smem_u32(sm + OFF_K);
#pragma unroll 4
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t kb = kk / 4, ko = (kk % 4) * 32;
        mma_ss<0>(tm_s, smem_desc(qa + kb * (kH * 128) + ko, 16, 1024, kSw128),
                  smem_desc(ka + kb * (kTR * 128) + ko, 16, 1024, kSw128), idesc_qk, kk > 0);
      }
      tc_commit(s_full);
    }
    if (j + 1 < ntiles) resolve(j + 1, buf ^ 1);
    __syncthreads();
    if (j + 1 < ntiles) fetch(buf ^ 1);  // in flight while this tile finishes

    // ---- softmax: one thread per head, S row from TMEM
    bool need_rescale = false;
    float alpha = 1.f;
    bool ok2 = true;
    if (warp < 4) {
      ok2 = mbar_wait(s_full, (uint32_t)j & 1u, a.status);
      tc_fence_after();
      const int rows_here = (int)((s_hi - s_lo) - (int64_t)j * kTR < kTR ? (s_hi - s_lo) - (int64_t)j * kTR : kTR);
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < kTR; c += 32) {
        uint32_t r[32];
        tmem_ld_32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int col = c + q;
          const bool valid = col < rows_here && src_s[buf * kTR + col] != 0;
          if (valid) mx = fmaxf(mx, __uint_as_float(r[q]) * a.sm_scale);
        }
      }
      if (softmax_thread) {
        if (mx > m_ref + kRescale || (m_ref == -INFINITY && mx > -INFINITY)) {
          const float m_new = mx;
          if (m_ref > -INFINITY) {
            alpha = __expf(m_ref - m_new);
            need_rescale = true;
            l_sum *= alpha;
          }
          m_ref = m_new;
        }
      }
      float sum = 0.f;
#pragma unroll 1
      for (int c = 0; c < kTR; c += 32) {
        uint32_t r[32];
        tmem_ld_32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
        tmem_ld_wait();
        if (softmax_thread) {
          float p[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int col = c + q;
            const bool valid = col < rows_here && src_s[buf * kTR + col] != 0;
            p[q] = (valid && m_ref > -INFINITY) ? __expf(__uint_as_float(r[q]) * a.sm_scale - m_ref) : 0.f;
            sum += p[q];
          }
          // P row `head`, columns c..c+31: K-major [64 heads][128 rows] in two 64-row blocks
          uint8_t* blk = sm + OFF_P + (c / 64) * (kH * 128);
#pragma unroll
          for (int q = 0; q < 32; q += 8)
            *reinterpret_cast<uint4*>(blk + swz(head, ((c % 64) + q) * 2)) =
                make_uint4(pack_h2(p[q], p[q + 1]), pack_h2(p[q + 2], p[q + 3]), pack_h2(p[q + 4], p[q + 5]),
                           pack_h2(p[q + 6], p[q + 7]));
        }
      }
      if (softmax_thread) l_sum += sum;
      // ---- rare: rescale O rows whose max moved (O owners are lanes 0-15)
      const float a_own = __shfl_sync(0xffffffffu, alpha, (lane & 15) + 16);
      const bool warp_rescale = __any_sync(0xffffffffu, need_rescale);
      if (warp_rescale && j > 0) {
        for (int c = 0; c < kD; c += 32) {
          uint32_t r[32];
          tmem_ld_32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
          tmem_ld_wait();
          if (lane < 16) {
#pragma unroll
            for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * a_own);
          }
          tmem_st_32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
        }
        tmem_st_wait();
      }
      fence_async_smem();
      tc_fence_before();
    }
    live = __syncthreads_and(ok2) != 0;
    if (!live) break;
    if (tid == 128) {  // ---- O += P V
      tc_fence_after();
      const uint32_t pa = smem_u32(sm + OFF_P), ka = smem_u32(sm + OFF_K);
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
        for (int kk = 0; kk < kTR / 16; ++kk) {
          const uint64_t adesc = smem_desc(pa + (kk / 4) * (kH * 128) + (kk % 4) * 32, 16, 1024, kSw128);
          const uint64_t bdesc = smem_desc(ka + nh * 4 * (kTR * 128) + kk * 2048, kTR * 128, 1024, kSw128);
          mma_ss<0>(tmem + nh * 256, adesc, bdesc, idesc_pv, j > 0 || kk > 0);
        }
      }
      tc_commit(pv_done);
    }
  }
  // ---- partial results
  if (ntiles > 0 && live) live = __syncthreads_and(mbar_wait(pv_done, (uint32_t)(ntiles - 1) & 1u, a.status)) != 0;
  tc_fence_after();
  const int64_t pidx = ((int64_t)list * a.splits + blockIdx.x) * a.H + head;
  if (warp < 4) {
    for (int c = 0; c < kD; c += 32) {
      uint32_t r[32];
      tmem_ld_32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
      tmem_ld_wait();
      if (lane < 16) {
        float* po = a.part_o + pidx * kD + c;
#pragma unroll
        for (int q = 0; q < 32; q += 4)
          *reinterpret_cast<float4*>(po + q) =
              (ntiles > 0 && live) ? make_float4(__uint_as_float(r[q]), __uint_as_float(r[q + 1]),
                                                 __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (softmax_thread) {
      a.part_ml[pidx * 2] = live ? m_ref : -INFINITY;
      a.part_ml[pidx * 2 + 1] = live ? l_sum : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attn_mma_supported(const AttnLaunch& a) {
  return a.kv.f.fmt == LCSC_FMT_KV && a.D == 512 && a.Dv == 512 && a.H == 64 && a.v.data == nullptr &&
         a.kv.f.row_bytes == 576 && (a.kv.f.dim - a.kv.f.rope) % 16 == 0 && a.rows_per_split % kTR == 0;
}

cudaError_t launch_attn_mma(const AttnLaunch& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  attn_mma_kernel<<<dim3(a.splits, a.B * a.T), kThr, SMEM, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace lcsc
