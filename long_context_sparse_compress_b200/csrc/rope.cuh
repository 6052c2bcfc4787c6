// Inverse rotary embedding of attention outputs ("How DeepSeek V4 Handles 1M
// Token Context", Component 1: K and V are one shared vector, and inverse
// RoPE restores the positional information).  The last rope_dim dims of an
// output row, in pairs (2j, 2j + 1), turn by -p * base^(-2j / rope_dim), p
// the query's position: the output then carries the keys' positions
// relative to the query.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lcsc {

// cos / sin of the angles of the two pairs in dims d0 .. d0 + 3 of a row of
// `dim` values (d0 a multiple of 4, rope_dim a multiple of 4).  Returns false
// when those dims are not rotated.
struct RopePair2 {
  float c0, s0, c1, s1;
};

// cos and sin of -p * base^(-2j / rope_dim).  The angle reaches 1e6 radians
// at long contexts, so it is formed in double and brought into [-pi, pi] by
// subtracting the nearest multiple k of 2 pi (k * 2pi in double is off by
// about k * 1e-15 radians); the reduced angle then goes through the fast
// single-precision sine and cosine, whose error there is a few 1e-7.
__device__ __forceinline__ void rope_cos_sin(int64_t p, float base, int j, int rope_dim, float* c, float* s) {
  const double a = -(double)p * pow((double)base, -2.0 * j / rope_dim);
  const double two_pi = 6.283185307179586;
  const double k = rint(a * (1.0 / two_pi));
  __sincosf((float)fma(-k, two_pi, a), s, c);
}

__device__ __forceinline__ bool inverse_rope_angles(int d0, int dim, int rope_dim, float base, int64_t p,
                                                    RopePair2* r) {
  const int lo = dim - rope_dim;
  if (rope_dim <= 0 || !(base > 0.f) || d0 < lo) return false;
  const int j0 = (d0 - lo) >> 1;
  rope_cos_sin(p, base, j0, rope_dim, &r->c0, &r->s0);
  rope_cos_sin(p, base, j0 + 1, rope_dim, &r->c1, &r->s1);
  return true;
}

__device__ __forceinline__ float4 rotate2(float4 v, const RopePair2& r) {
  return make_float4(v.x * r.c0 - v.y * r.s0, v.x * r.s0 + v.y * r.c0, v.z * r.c1 - v.w * r.s1,
                     v.z * r.s1 + v.w * r.c1);
}

}  // namespace lcsc
