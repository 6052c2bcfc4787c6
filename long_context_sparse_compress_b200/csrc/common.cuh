// Shared device helpers of the CUDA path: stored-row codecs, reductions,
// small PTX wrappers.  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lcsc.h"

namespace lcsc {

constexpr int kWarp = 32;

// Programmatic dependent launch: the first statement of every kernel of this
// library.  Returns once the stream's previous grid has completed and its
// memory operations are visible (at once when the launch had no programmatic
// dependency), so each grid still completes after all earlier work of its
// stream and touches no global memory or TMEM before that.  No kernel
// signals its dependents early (griddepcontrol.launch_dependents): the next
// grid's launch then starts as this one's last CTA exits, which removes the
// launch gap without CTAs that wait on an SM for a whole kernel while the
// other layer's stream could use it (measured slower with two streams).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ----------------------------------------------------------------- row layout

struct RowFmt {
  int fmt;        // LCSC_FMT_*
  int dim;        // values per row
  int rope;       // trailing BF16 values (LCSC_FMT_KV)
  int row_bytes;  // payload bytes per row
};

__host__ __device__ inline int row_bytes_of(int fmt, int dim, int rope) {
  switch (fmt) {
    case LCSC_FMT_F32: return 4 * dim;
    case LCSC_FMT_KV: return dim + rope;
    case LCSC_FMT_FP8: return dim;
    case LCSC_FMT_FP4: return dim / 2;
  }
  return 0;
}

// Device view of one stored tensor for B sequences.
struct CacheView {
  uint8_t* data;
  void* scale;
  int64_t capacity;
  RowFmt f;
  int64_t row0;  // an entry shard holds the entries [row0, row0 + rows) in rows 0 ..
  int64_t rows;  // 0: unsharded (entry g in row g)
  // Local row of global entry g in this view, or -1 when another shard holds it.
  __host__ __device__ __forceinline__ int64_t local(int64_t g) const {
    if (rows <= 0) return g;
    const int64_t r = g - row0;
    return (r >= 0 && r < rows) ? r : -1;
  }
  // Visible entries of this view among the first n global ones: the count of
  // local rows 0 .. that hold entries below n.
  __host__ __device__ __forceinline__ int64_t local_count(int64_t n) const {
    if (rows <= 0) return n;
    const int64_t c = n - row0;
    return c <= 0 ? 0 : (c < rows ? c : rows);
  }
  __device__ __forceinline__ uint8_t* row(int b, int64_t r) const {
    return data + ((int64_t)b * capacity + r) * f.row_bytes;
  }
  __device__ __forceinline__ float* fscale(int b, int64_t r) const {
    return reinterpret_cast<float*>(scale) + (int64_t)b * capacity + r;
  }
  // FP4 block scales are tiled by 128 rows so that one tile's scales are one
  // contiguous 512-byte chunk per 64 values of the row (the order the tensor
  // cores read them in): byte of row r, block k =
  //   [b][r / 128][k / 4][r % 32][(r % 128) / 32][k % 4].
  __device__ __forceinline__ uint8_t* bscale_at(int b, int64_t r, int k) const {
    const int64_t tiles = (capacity + 127) / 128;
    const int64_t tile_bytes = (int64_t)(f.dim / 64) * 512;
    const int m = (int)(r & 127);
    return reinterpret_cast<uint8_t*>(scale) + ((int64_t)b * tiles + (r >> 7)) * tile_bytes + (k >> 2) * 512 +
           (m & 31) * 16 + (m >> 5) * 4 + (k & 3);
  }
};

// ------------------------------------------------------------ scalar codecs

__device__ __forceinline__ float e4m3_val(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ float2 e4m3x2_val(uint16_t c2) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c2, __NV_E4M3);
  return __half22float2(__half2(h));
}

__device__ __forceinline__ float2 e2m1x2_val(uint8_t c2) {
  __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(c2, __NV_E2M1);
  return __half22float2(__half2(h));
}

__device__ __forceinline__ uint16_t e4m3x2_code(float a, float b) {
  return __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint8_t e2m1x2_code(float a, float b) {
  return __nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest);
}

__device__ __forceinline__ float bf16_val(uint16_t bits) {
  return __uint_as_float(((uint32_t)bits) << 16);
}

__device__ __forceinline__ uint16_t bf16_code(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Load one element of an x_dtype array as float.
__device__ __forceinline__ float load_elem(const void* p, int64_t i, int dtype) {
  if (dtype == LCSC_DT_BF16) return bf16_val(reinterpret_cast<const uint16_t*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

// ------------------------------------------------------------- reductions

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Max over aligned groups of `width` lanes (width a power of two <= 32).
__device__ __forceinline__ float group_max(float v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------- row storing
// One warp stores one row.  Lane l holds VPL = dim / 32 consecutive values
// v[0..VPL) of elements l*VPL ...  (dim in {32, 128, 512}).
template <int VPL>
__device__ __forceinline__ void store_row_warp(const CacheView& cv, int b, int64_t r,
                                               const float (&v)[VPL], int lane) {
  const RowFmt f = cv.f;
  uint8_t* dst = cv.row(b, r);
  const int e0 = lane * VPL;
  if (f.fmt == LCSC_FMT_F32) {
    float* d = reinterpret_cast<float*>(dst) + e0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) d[i] = v[i];
    return;
  }
  if (f.fmt == LCSC_FMT_KV || f.fmt == LCSC_FMT_FP8) {
    const int n_fp8 = f.dim - (f.fmt == LCSC_FMT_KV ? f.rope : 0);
    const bool is_fp8 = e0 < n_fp8;
    float a = 0.f;
    if (is_fp8) {
#pragma unroll
      for (int i = 0; i < VPL; ++i) a = fmaxf(a, fabsf(v[i]));
    }
    const float amax = warp_max(a);
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    if (is_fp8) {
      uint8_t codes[VPL];
#pragma unroll
      for (int i = 0; i < VPL; i += 2) {
        float y0 = __fdiv_rn(v[i], s);
        float y1 = (VPL > 1) ? __fdiv_rn(v[i + 1 < VPL ? i + 1 : i], s) : 0.f;
        uint16_t c2 = e4m3x2_code(y0, y1);
        codes[i] = (uint8_t)(c2 & 0xff);
        if (i + 1 < VPL) codes[i + 1] = (uint8_t)(c2 >> 8);
      }
      if constexpr (VPL == 16) {
        *reinterpret_cast<uint4*>(dst + e0) = *reinterpret_cast<const uint4*>(codes);
      } else if constexpr (VPL == 4) {
        *reinterpret_cast<uint32_t*>(dst + e0) = *reinterpret_cast<const uint32_t*>(codes);
      } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i) dst[e0 + i] = codes[i];
      }
    } else {
      uint16_t* d = reinterpret_cast<uint16_t*>(dst + n_fp8) + (e0 - n_fp8);
#pragma unroll
      for (int i = 0; i < VPL; ++i) d[i] = bf16_code(v[i]);
    }
    if (lane == 0) *cv.fscale(b, r) = s;
    return;
  }
  // LCSC_FMT_FP4: blocks of 16 values, one E4M3 scale byte each.
  constexpr int LPB = VPL >= 16 ? 1 : 16 / VPL;  // lanes per block
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) a = fmaxf(a, fabsf(v[i]));
  // VPL == 16: a lane is one block; VPL < 16: LPB lanes form a block.
  const float amax = group_max(a, LPB);
  const float bsc = __fdiv_rn(amax, 6.f);
  const uint8_t sc = (uint8_t)(e4m3x2_code(bsc, 0.f) & 0xff);
  const float dsc = e4m3_val(sc);
  uint8_t packed[VPL / 2 > 0 ? VPL / 2 : 1];
#pragma unroll
  for (int i = 0; i + 1 < VPL; i += 2) {
    float y0 = dsc > 0.f ? __fdiv_rn(v[i], dsc) : 0.f;
    float y1 = dsc > 0.f ? __fdiv_rn(v[i + 1], dsc) : 0.f;
    packed[i / 2] = dsc > 0.f ? e2m1x2_code(y0, y1) : (uint8_t)0;
  }
  if constexpr (VPL == 1) {
    // Two lanes share a byte: the even lane writes it.
    float y = dsc > 0.f ? __fdiv_rn(v[0], dsc) : 0.f;
    float yn = __shfl_down_sync(0xffffffffu, y, 1);
    if ((lane & 1) == 0) dst[lane >> 1] = dsc > 0.f ? e2m1x2_code(y, yn) : (uint8_t)0;
  } else if constexpr (VPL == 16) {
    *reinterpret_cast<uint2*>(dst + e0 / 2) = *reinterpret_cast<const uint2*>(packed);
  } else if constexpr (VPL == 4) {
    *reinterpret_cast<uint16_t*>(dst + e0 / 2) = *reinterpret_cast<const uint16_t*>(packed);
  } else {
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) dst[e0 / 2 + i] = packed[i];
  }
  if (lane % LPB == 0) *cv.bscale_at(b, r, e0 / 16) = sc;
}

// Dequantised value of element e of a stored row (slow path, any format).
__device__ __forceinline__ float stored_elem(const CacheView& cv, int b, int64_t r, int e) {
  const uint8_t* row = cv.row(b, r);
  switch (cv.f.fmt) {
    case LCSC_FMT_F32: return reinterpret_cast<const float*>(row)[e];
    case LCSC_FMT_KV: {
      const int n_fp8 = cv.f.dim - cv.f.rope;
      if (e < n_fp8) return e4m3_val(row[e]) * *cv.fscale(b, r);
      return bf16_val(reinterpret_cast<const uint16_t*>(row + n_fp8)[e - n_fp8]);
    }
    case LCSC_FMT_FP8: return e4m3_val(row[e]) * *cv.fscale(b, r);
    case LCSC_FMT_FP4: {
      float2 v = e2m1x2_val(row[e >> 1]);
      return ((e & 1) ? v.y : v.x) * e4m3_val(*cv.bscale_at(b, r, e >> 4));
    }
  }
  return 0.f;
}

// Order-preserving map of float bits to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

}  // namespace lcsc
