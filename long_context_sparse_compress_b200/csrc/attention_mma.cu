// Joint attention on the 5th-generation tensor cores: all 64 query heads of
// one query against one shared 512-d KV row set (FP8 + BF16 RoPE storage).
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works" (exact attention over the selected
// compressed entries plus the uncompressed window, shared-KV multi-query
// layout; the sink enters in the combine step); storage: the same page's Key
// numbers, row "KV storage precision" (FP8 with BF16 RoPE dims).
//
// The stored rows enter the tensor cores as they are stored: the 448 E4M3
// codes of a row are the operand of S = Q K^T and of O += P V through
// kind::f8f6f4, the 64 BF16 RoPE dims through kind::f16; nothing is
// dequantised.  Per row r with scale c_r and per head h:
//   s_hr = c_r (Q_nope . codes_r) + Q_rope . rope_r     (two TMEM accumulators)
//   O_nope += sum_r (p_hr c_r) codes_r,  O_rope += sum_r p_hr rope_r.
// The E4M3 operands that are not stored values -- the query's 448 dims and
// the weights p_hr c_r -- are each written as the sum of two E4M3 numbers
// (a leading part and the rounding error of it), so each product is a pair
// of MMAs into one accumulator and keeps about 8 significant bits, the
// precision of the BF16 query.  The query is first multiplied, per head, by
// a power of two that brings its largest |value| into [128, 256); the
// weights p c_r by a per-head power of two g_h that the softmax keeps near
// [8, 16) for the largest weight of a tile (O_nope is divided by g_h at the
// end, and rescaled in TMEM when g_h changes).
//
// One CTA owns (query, range of rows) and walks it in tiles of 64 rows with a
// warp-specialised pipeline:
//  * 11 loader warps resolve the tile's rows (gathered by index for CSA) and
//    copy them with cp.async, two tiles ahead, into one of three tile
//    buffers: the codes in 64-byte-swizzled 64-dim atoms, the RoPE dims in a
//    128-byte-swizzled block; the same bytes are the K-major operand of
//    Q K^T and the MN-major operand of P V;
//  * 1 MMA warp issues Q K^T (M = 64 heads, N = 64 rows) of a loaded tile or
//    P V (N = 256 + 192 code dims and 64 RoPE dims) of a tile whose weights
//    are out, whichever is ready;
//  * 4 softmax warps read S in the mma-fragment layout (each thread two heads
//    x 16 rows), keep a lazy reference max per head (O rescaled only when the
//    max grows by more than e^8), and write P as BF16 and p c_r g_h as two
//    E4M3 terms.
// Heads live on M = 64, so the accumulators use the half-lane TMEM layout: O
// at lanes 0-15 of each 32-lane sub-partition (all 512 columns), S (codes
// and RoPE parts, two buffers each) at lanes 16-31.  With several splits per
// query the partial (ref max, sum, O) goes to the workspace the combine
// kernel merges; with one, the kernel merges the sink itself and writes the
// output.
#include "kernels.cuh"
#include "launches.h"
#include "rope.cuh"
#include "sm100.cuh"

namespace lcsc {
namespace {

static_assert(kDefaultWaitNs == sm100::kWaitLimitNs, "one default limit for the bounded waits");

using namespace sm100;

constexpr int kH = 64;       // heads (MMA M)
constexpr int kD = 512;      // row length
constexpr int kNope = 448;   // E4M3 dims of a stored row
constexpr int kTR = 64;      // rows per tile
constexpr int kNB = 3;       // tile buffers
constexpr int kLW = 10;      // loader warps (16 warps in all: 4 per SM sub-partition)
constexpr int kSW = 4;       // softmax warps
constexpr int kThr = (kSW + kLW + 2) * 32;
constexpr int kPvWarp = kSW + kLW;   // issues P V
constexpr int kMmaWarp = kPvWarp + 1;  // issues Q K^T; owns TMEM
constexpr int kLT = kLW * 32;                                    // loader threads
constexpr int kCodeChunks = kNope / 16, kRopeChunks = 8;         // 16-byte chunks of a stored row
constexpr int kUnits = kTR * (kCodeChunks + kRopeChunks);        // 16-byte copies of a tile
constexpr int kLoads = (kUnits + kLT - 1) / kLT;                 // per loader thread
static_assert((kUnits % kLT) % 32 == 0, "the partial last round is taken by whole warps");
constexpr float kRescale = 8.f;  // rescale O only when the max grows by more (natural log units)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kWeightHi = 256.f;  // largest p c_r g_h before g_h is lowered (E4M3 holds 448)

// shared memory (offsets from a 1024-aligned base)
constexpr int kAtom = 64 * 64;                   // one 64-dim E4M3 atom: [64 rows][64 B], 64-byte swizzle
constexpr int kCodeBytes = 7 * kAtom;            // 448 dims
constexpr int OFF_QHI = 0;                       // query codes, leading terms (28 KB)
constexpr int OFF_QLO = OFF_QHI + kCodeBytes;    // their rounding errors (28 KB)
constexpr int OFF_QR = OFF_QLO + kCodeBytes;     // query RoPE dims, bf16 [64][128 B] (8 KB)
constexpr int OFF_K = OFF_QR + kH * 128;         // tile buffers
constexpr int KB_ROPE = kCodeBytes;              // RoPE block inside a tile buffer ([64 rows][128 B])
constexpr int KBUF = kCodeBytes + kTR * 128;     // 36 KB per buffer
constexpr int OFF_P = OFF_K + kNB * KBUF;        // 2 buffers x (E4M3 weights 8 KB + bf16 P 8 KB)
constexpr int PBUF = 2 * kH * 128;
constexpr int OFF_BAR = OFF_P + 2 * PBUF;  // k_full[3] k_free[3] s_full[2] p_full[2] pv_done[2] drain q_full
constexpr int kBars = 14;
constexpr int OFF_QSC = OFF_BAR + kBars * 8;     // float [64]: per-head power-of-two scale of q
constexpr int OFF_ROW = OFF_QSC + kH * 4;        // int64 [4][64]: row pointers of tiles j % 4
constexpr int OFF_SCL = OFF_ROW + 4 * kTR * 8;   // float [4][64]: row scales (0: no row)
constexpr int OFF_MASK = OFF_SCL + 4 * kTR * 4;  // uint32 [4][2]: valid-row bits
constexpr int OFF_TM = OFF_MASK + 32;
constexpr int OFF_ABORT = OFF_TM + 4;
constexpr int OFF_LSTOP = OFF_ABORT + 4;
constexpr int SMEM = OFF_LSTOP + 4 + 1024;
// The query image a CTA copies in: the query part of this layout (E4M3
// terms and RoPE dims, 64 KB) followed by the per-head scales.
constexpr int kQImg = OFF_K;
static_assert(kQImg + kH * 4 == (int)kAttnQImageBytes, "query image layout");
static_assert(OFF_QSC % 16 == 0, "bulk copy destination");
constexpr int kOS = kD + 4;                      // row stride (floats) of the partial O staged in shared memory
static_assert(OFF_QR % 1024 == 0 && OFF_K % 1024 == 0 && KBUF % 1024 == 0 && OFF_P % 1024 == 0,
              "swizzle atoms need 1024-byte alignment");
static_assert(kH * kOS * 4 <= OFF_BAR - OFF_K, "the staged partial O fits in the tile and P buffers");
static_assert(SMEM <= 232448, "shared memory per block");

// Byte offset of (row, byte) in a [rows][128 B] block with the 128-byte
// swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz128(int row, int byte) {
  return (uint32_t)(row * 128 + ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
}
// ... and in a [rows][64 B] block with the 64-byte swizzle (chunk index XOR
// (row / 2) % 4: address bits 4-5 XOR bits 7-8).
__device__ __forceinline__ uint32_t swz64(int row, int byte) {
  return (uint32_t)(row * 64 + ((((byte >> 4) ^ ((row >> 1) & 3)) << 4) | (byte & 15)));
}

// 2^x on the MUFU unit (approximate, flush-to-zero), the base-2 exponential
// the softmax works in.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16-byte global -> shared copy (zero fill when !live; src must still be a
// valid address).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool live) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(live ? 16 : 0)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread has issued so far has
// landed (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// x = hi + lo + (error below the second term), hi and lo E4M3 (pairs).
__device__ __forceinline__ void e4m3_split2(float a, float b, uint16_t& hi, uint16_t& lo) {
  hi = e4m3x2_code(a, b);
  const float2 h = e4m3x2_val(hi);
  lo = e4m3x2_code(a - h.x, b - h.y);
}

// The same split from a pair rounded to f16 first, in f16x2 arithmetic (the
// softmax weights: both terms of an f16 pair hold its 11 bits to about 8).
__device__ __forceinline__ void e4m3_split2_h(float a, float b, uint16_t& hi, uint16_t& lo) {
  const __half2 x = __floats2half2_rn(a, b);
  hi = __nv_cvt_halfraw2_to_fp8x2(__half2_raw(x), __NV_SATFINITE, __NV_E4M3);
  const __half2 h(__nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3));
  lo = __nv_cvt_halfraw2_to_fp8x2(__half2_raw(__hsub2(x, h)), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  return (uint32_t)bf16_code(a) | ((uint32_t)bf16_code(b) << 16);
}

struct Rows {
  int64_t n_vis, n_ent_slots, w_lo, n_win;
  int64_t n_tok;  // 1: the stored position-0 row (sink token) follows the window
  bool ok;
};

__device__ __forceinline__ Rows rows_of(const AttnLaunch& a, int b, int t) {
  Rows r;
  const int64_t L = a.ctx_len[b];
  r.ok = L >= a.T && (a.kv.rows > 0 || L / a.m <= a.n_max);  // a shard holds a range: no limit
  const int64_t p = L - a.T + t;
  r.n_vis = r.ok ? (p + 1) / a.m : 0;
  r.n_ent_slots = a.idx ? a.k : a.kv.local_count(r.n_vis);
  r.w_lo = p - a.w + 1 > 0 ? p - a.w + 1 : 0;
  r.n_win = (r.ok && a.w > 0) ? p - r.w_lo + 1 : 0;
  r.n_tok = (r.ok && a.sink_token && !(r.n_win > 0 && r.w_lo == 0)) ? 1 : 0;
  return r;
}

// Bounded wait taken by a whole warp; false (for every lane) if any lane gave up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const AttnLaunch& a,
                                          volatile int* abort) {
  if (*abort) return false;
  bool ok = mbar_wait(bar, parity, a.status, a.waits.limit_ns);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) *abort = 1;
  return ok;
}

// 2^e as a float, e clamped to the normal range.
__device__ __forceinline__ float pow2(int e) {
  e = e < -126 ? -126 : (e > 127 ? 127 : e);
  return __int_as_float((e + 127) << 23);
}

// ---- The query image of one (sequence, token), built once and copied in by
// every CTA of its row splits.  Per head a power of two 2^-e brings the
// largest |q| into [128, 256); the 448 code dims become two E4M3 terms
// (64-byte-swizzled atoms of 64 dims), the 64 RoPE dims bf16 (128-byte
// swizzle); the image ends with 2^e per head, which the softmax multiplies
// back into the logits.
__global__ void __launch_bounds__(kThr) attn_qimage_kernel(const AttnLaunch a) {
  grid_dep_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* qsc_s = reinterpret_cast<float*>(sm + kQImg);  // per-head amax of q, then 2^e
  const int tid = threadIdx.x, lane = tid % 32;
  const int list = blockIdx.x;
  constexpr int kQChunks = kH * (kD / 8), kQIter = (kQChunks + kThr - 1) / kThr;
  static_assert(kThr % 64 == 0 && (kD / 8) == 64 && kQChunks % kThr == 0,
                "the lanes of a warp share one head per chunk round; every thread has kQIter chunks");
  auto q_mult = [&](int h) -> float {  // 2^-e from the head's amax (0: 1)
    const int bits = __float_as_int(qsc_s[h]);
    if (bits == 0) return 1.f;
    const int ex = ((bits >> 23) & 0xff) - 127 - 7;  // amax in [2^(ex+7), 2^(ex+8)) (normal amax)
    return pow2(-ex);
  };
  const bool q_bf = a.q_dtype == LCSC_DT_BF16;
  auto f32_chunk = [&](int i, float (&v)[8]) {
    const int64_t base = ((int64_t)list * a.H + i / (kD / 8)) * kD + (i % (kD / 8)) * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = load_elem(a.q, base + j, a.q_dtype);
  };
  if (tid < kH) qsc_s[tid] = 0.f;  // amax slots (non-negative: compared as integers)
  __syncthreads();
  uint4 raw[kQIter];  // bf16 queries stay in registers between the passes
  if (q_bf) {
#pragma unroll
    for (int u = 0; u < kQIter; ++u)
      raw[u] = reinterpret_cast<const uint4*>(a.q)[(int64_t)list * a.H * (kD / 8) + tid + u * kThr];
#pragma unroll
    for (int u = 0; u < kQIter; ++u) {
      const int i = tid + u * kThr;
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw[u]);
      uint32_t mb = 0;  // largest |bf16| bit pattern: the order of the magnitudes
#pragma unroll
      for (int j = 0; j < 4; ++j) mb = max(mb, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
      const float mx = warp_max(__uint_as_float(mb << 16));  // one head per warp and round
      if (lane == 0) atomicMax(reinterpret_cast<int*>(qsc_s) + i / (kD / 8), __float_as_int(mx));
    }
  } else {
    for (int u = 0; u < kQIter; ++u) {
      const int i = tid + u * kThr;
      float v[8], mx = 0.f;
      f32_chunk(i, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(v[j]));
      mx = warp_max(mx);
      if (lane == 0) atomicMax(reinterpret_cast<int*>(qsc_s) + i / (kD / 8), __float_as_int(mx));
    }
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kQIter; ++u) {
    const int i = tid + u * kThr;
    const int h = i / (kD / 8), d0 = (i % (kD / 8)) * 8;
    const float f = q_mult(h);
    float v[8];
    if (q_bf) {
      const uint16_t* bf = reinterpret_cast<const uint16_t*>(&raw[u]);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = bf16_val(bf[j]) * f;
    } else {
      f32_chunk(i, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] *= f;
    }
    if (d0 < kNope) {
      uint16_t hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) e4m3_split2(v[2 * j], v[2 * j + 1], hi[j], lo[j]);
      const uint32_t off = (d0 / 64) * kAtom + swz64(h, d0 % 64);
      *reinterpret_cast<uint2*>(sm + OFF_QHI + off) =
          make_uint2(hi[0] | ((uint32_t)hi[1] << 16), hi[2] | ((uint32_t)hi[3] << 16));
      *reinterpret_cast<uint2*>(sm + OFF_QLO + off) =
          make_uint2(lo[0] | ((uint32_t)lo[1] << 16), lo[2] | ((uint32_t)lo[3] << 16));
    } else {
      *reinterpret_cast<uint4*>(sm + OFF_QR + swz128(h, (d0 - kNope) * 2)) =
          make_uint4(bf16x2(v[0], v[1]), bf16x2(v[2], v[3]), bf16x2(v[4], v[5]), bf16x2(v[6], v[7]));
    }
  }
  __syncthreads();  // every multiplier was read: the slots now take 2^e
  if (tid < kH) qsc_s[tid] = 1.f / q_mult(tid);
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(a.q_img + (size_t)list * kAttnQImageBytes);
  const uint4* src = reinterpret_cast<const uint4*>(sm);
  for (int i = tid; i < (int)(kAttnQImageBytes / 16); i += kThr) dst[i] = src[i];
}

__global__ void __maxnreg__(128) attn_mma_kernel(const AttnLaunch a) {
  grid_dep_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* k_full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);  // [3] a tile's rows have landed
  uint64_t* k_free = k_full + 3;   // [3] the P V of a tile buffer is done
  uint64_t* s_full = k_full + 6;   // [2]
  uint64_t* p_full = k_full + 8;   // [2]
  uint64_t* pv_done = k_full + 10; // [2]
  uint64_t* drain = k_full + 12;   // every MMA issued has completed (before TMEM is freed)
  uint64_t* q_full = k_full + 13;  // the query image has landed
  int64_t* row_s = reinterpret_cast<int64_t*>(sm + OFF_ROW);
  float* scl_s = reinterpret_cast<float*>(sm + OFF_SCL);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(sm + OFF_MASK);
  uint32_t* tm_slot = reinterpret_cast<uint32_t*>(sm + OFF_TM);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_ABORT);
  volatile int* lstop = reinterpret_cast<volatile int*>(sm + OFF_LSTOP);  // loader-group decision
  float* qsc_s = reinterpret_cast<float*>(sm + OFF_QSC);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int list = blockIdx.y;
  const int b = list / a.T, t = list % a.T;
  const Rows qr = rows_of(a, b, t);
  if (!qr.ok && tid == 0 && blockIdx.x == 0 && a.status) atomicOr(a.status, LCSC_DEV_BAD_LENGTH);
  const int64_t total = qr.ok ? qr.n_ent_slots + qr.n_win + qr.n_tok : 0;
  const int64_t s_lo = (int64_t)blockIdx.x * a.rows_per_split;
  const int64_t s_hi = s_lo + a.rows_per_split < total ? s_lo + a.rows_per_split : total;
  const int ntiles = s_hi > s_lo ? (int)((s_hi - s_lo + kTR - 1) / kTR) : 0;

  if (tid == 0) {
    for (int i = 0; i < kNB; ++i) {
      mbar_init(&k_full[i], kLT + 1);  // every loader's copies + the tile's scales and row mask
      mbar_init(&k_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSW);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 2);
    mbar_init(q_full, 1);
    *abort = 0;
    *lstop = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tm_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tm_slot;
  if (tid == 0) {
    // the query image (attn_qimage_kernel): E4M3 terms, RoPE dims and
    // per-head scales, in this layout, by two bulk copies; waited for by the
    // Q K^T issuer and the softmax warps (this thread among them)
    const uint8_t* img = a.q_img + (size_t)list * kAttnQImageBytes;
    mbar_arrive_expect_tx(q_full, (uint32_t)kAttnQImageBytes);
    bulk_load(sm + OFF_QHI, img, kQImg, q_full);
    bulk_load(qsc_s, img + kQImg, kH * 4, q_full);
  }

  if (warp >= kSW && warp < kPvWarp) {
    // =================================================== loader warps
    const int lt = tid - kSW * 32;  // 0 .. kLT - 1
    // Copies of a tile, fixed per thread for the whole kernel.  Unit
    // u < 1792 is a 16-byte chunk of codes: q = u % 4 (chunk in the atom),
    // row-in-pair = (u / 4) % 2, then atom (7) and row pair (32), so that
    // the 8 lanes of a store phase fill 2 rows x 64 B of one atom (distinct
    // banks).  The rest are the 8 RoPE chunks of each row.  Table word:
    // destination offset in the buffer (16 bits) | row << 16 | chunk << 22;
    // all ones: no unit.
    uint32_t tab[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      const int u = lt + i * kLT;
      int r, c;
      uint32_t dst;
      if (u >= kUnits) {
        tab[i] = 0xFFFFFFFFu;
        continue;
      }
      if (u < kTR * kCodeChunks) {
        const int rest = u >> 3, at = rest % 7;
        r = 2 * (rest / 7) + ((u >> 2) & 1);
        c = 4 * at + (u & 3);
        dst = at * kAtom + swz64(r, (u & 3) * 16);
      } else {
        const int v = u - kTR * kCodeChunks;
        r = v >> 3;
        c = kCodeChunks + (v & 7);
        dst = KB_ROPE + swz128(r, (v & 7) * 16);
      }
      tab[i] = dst | ((uint32_t)r << 16) | ((uint32_t)c << 22);
    }
    auto slot_of = [&](int j) { return s_lo + (int64_t)j * kTR + lt; };
    auto load_idx = [&](int j) -> int32_t {
      const int64_t slot = slot_of(j);
      return (a.idx && slot < s_hi && slot < qr.n_ent_slots) ? a.idx[(int64_t)list * a.k + slot] : 0;
    };
    const int64_t win_cap = a.win_kv.capacity;
    const int64_t win_base = win_cap > 0 ? qr.w_lo % win_cap : 0;  // no window: never used
    // Row of tile j for this thread (lt < 64): pointer (null: no row) and scale address.
    auto locate = [&](int j, int32_t gi, const float*& scp) -> const uint8_t* {
      const int64_t slot = slot_of(j);
      scp = nullptr;
      if (slot >= s_hi) return nullptr;
      if (slot < qr.n_ent_slots) {
        const int64_t g = a.idx ? (int64_t)gi : slot + a.kv.row0;
        if (g >= 0 && g < qr.n_vis) {
          const int64_t r = a.kv.local(g);
          if (r < 0) return nullptr;  // another shard holds it
          scp = a.kv.fscale(b, r);
          return a.kv.row(b, r);
        }
        if ((g != -1 || !a.idx) && a.status) atomicOr(a.status, LCSC_DEV_BAD_INDEX);
        return nullptr;
      }
      if (slot >= qr.n_ent_slots + qr.n_win) {  // the sink token: position 0's stored row
        scp = a.tok_kv.fscale(b, 0);
        return a.tok_kv.row(b, 0);
      }
      int64_t row = win_base + (slot - qr.n_ent_slots);  // < 2 * capacity: the window is <= capacity rows
      if (row >= win_cap) row -= win_cap;
      scp = a.win_kv.fscale(b, row);
      return a.win_kv.row(b, row);
    };
    // tile j's row pointer and valid bit (slot j % 4); its scale is loaded
    // into `sc_pending` and stored a step later (0: no row)
    float sc_pending = 0.f;
    auto place = [&](int j, int32_t gi) {
      const float* scp;
      const uint8_t* p = locate(j, gi, scp);
      row_s[(j & 3) * kTR + lt] = reinterpret_cast<int64_t>(p);
      const uint32_t bits = __ballot_sync(0xffffffffu, p != nullptr);
      if (lane == 0) mask_s[(j & 3) * 2 + (lt >> 5)] = bits;
      sc_pending = p ? *scp : 0.f;
    };
    // tile j's copies into buffer j % 3; each thread's arrive on k_full
    // completes once its copies have landed
    auto issue = [&](int j) {
      const int64_t* rows = row_s + (j & 3) * kTR;
      const uint32_t kt = smem_u32(sm + OFF_K + (j % kNB) * KBUF);
#pragma unroll
      for (int i = 0; i < kLoads; ++i) {
        if (tab[i] == 0xFFFFFFFFu) continue;
        const uint8_t* ptr = reinterpret_cast<const uint8_t*>(rows[(tab[i] >> 16) & 63]);
        cp_async16(kt + (tab[i] & 0xFFFFu), ptr ? ptr + (tab[i] >> 22) * 16 : a.q, ptr != nullptr);
      }
      cp_async_arrive(&k_full[j % kNB]);
    };
    int32_t idx_next = 0;  // gather index of the next tile to place (in flight)
    // prologue: tiles 0 and 1 located, their scales stored, their copies issued
    if (lt < kTR) {
      for (int j = 0; j < 2 && j < ntiles; ++j) {
        place(j, load_idx(j));
        scl_s[(j & 3) * kTR + lt] = sc_pending;
      }
      if (ntiles > 2) idx_next = load_idx(2);
    }
    named_sync(1, kLT);
    if (lt == 0 && ntiles > 0) mbar_arrive(&k_full[0]);  // tile 0's scales and mask
    if (ntiles > 0) issue(0);
    if (ntiles > 1) issue(1);
    // Step j: tile j+1's scales published, tile j+2 located and (once the
    // P V of tile j-1 has freed its buffer) requested.  Nothing here waits
    // for copies: they complete their tiles' barriers by themselves.
    for (int j = 0; j < ntiles; ++j) {
      if (lt < kTR) {
        if (j >= 1 && j + 1 < ntiles) scl_s[((j + 1) & 3) * kTR + lt] = sc_pending;  // placed last step
        if (j + 2 < ntiles) {
          place(j + 2, idx_next);
          if (j + 3 < ntiles) idx_next = load_idx(j + 3);
        }
      }
      if (!a.idx && lt == 0 && j + 3 < ntiles) {
        // dense entries are contiguous: tile j+3's rows go to L2 now, in one
        // bulk prefetch, a step before their copies are issued (rows are
        // 576 B from a 16-byte-aligned base, so the start is aligned)
        const int64_t g0 = s_lo + (int64_t)(j + 3) * kTR;
        const int64_t hi = s_hi < qr.n_ent_slots ? s_hi : qr.n_ent_slots;
        if (g0 < hi) {
          const int64_t cnt = hi - g0 < kTR ? hi - g0 : kTR;
          prefetch_l2(a.kv.row(b, g0), (uint32_t)(cnt * a.kv.f.row_bytes));
        }
      }
      named_sync(1, kLT);
      if (lt == 0 && j + 1 < ntiles) mbar_arrive(&k_full[(j + 1) % kNB]);  // tile j+1's scales and mask
      if (j + 2 < ntiles) {
        // buffer (j+2) % 3 is free once the P V of tile j-1 is done; one
        // thread decides for the group (`lstop` is written only here,
        // between group barriers)
        if (lt == 0) {
          bool ok = !*abort;
          if (ok && j >= 1)
            ok = mbar_wait(&k_free[(j + 2) % kNB], (uint32_t)((j - 1) / kNB) & 1u, a.status, a.waits.limit_ns);
          if (!ok) *abort = 1;
          *lstop = ok ? 0 : 1;
        }
        named_sync(1, kLT);
        if (*lstop) break;
        issue(j + 2);
      }
    }
    cp_async_wait_all();  // no copy outlives the loop (the epilogue reuses the buffers)
  } else if (warp >= kPvWarp) {
    // =================================================== MMA warps
    // Two issuers, so that the per-instruction cost of issuing overlaps:
    // warp kMmaWarp issues Q K^T of each loaded tile into S[j % 2] once the
    // softmax of tile j-2 has published its P (S[j % 2] is then free); warp
    // kPvWarp issues P V of each tile whose P is out.  Each tracks its own
    // MMAs with tcgen05.commit.
    const uint32_t idesc_qk8 = idesc_dense(0, 0, 64, kTR);                 // E4M3 x E4M3
    const uint32_t idesc_qkr = idesc_dense(1, 1, 64, kTR);                 // bf16 x bf16
    const uint32_t idesc_pv8a = idesc_dense(0, 0, 64, 256, false, true);   // codes 0-255
    const uint32_t idesc_pv8b = idesc_dense(0, 0, 64, 192, false, true);   // codes 256-447
    const uint32_t idesc_pvr = idesc_dense(1, 1, 64, 64, false, true);     // RoPE dims
    const uint32_t qhi = smem_u32(sm + OFF_QHI), qlo = smem_u32(sm + OFF_QLO), qro = smem_u32(sm + OFF_QR);
    const uint32_t s_base = tmem + (16u << 16);
    auto issue_qk = [&](int j) {
      const int sb = j & 1;
      const uint32_t ka = smem_u32(sm + OFF_K + (j % kNB) * KBUF);
      const uint32_t dn = s_base + sb * kTR, dr = s_base + 2 * kTR + sb * kTR;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t qa = part ? qlo : qhi;
#pragma unroll
        for (int at = 0; at < 7; ++at) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t o = at * kAtom + kk * 32;
            mma_ss<1>(dn, smem_desc(qa + o, 16, 512, kSw64), smem_desc(ka + o, 16, 512, kSw64), idesc_qk8,
                      part > 0 || at > 0 || kk > 0);
          }
        }
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss<0>(dr, smem_desc(qro + kk * 32, 16, 1024, kSw128), smem_desc(ka + KB_ROPE + kk * 32, 16, 1024, kSw128),
                  idesc_qkr, kk > 0);
      tc_commit(&s_full[sb]);
    };
    auto issue_pv = [&](int j) {
      const int sb = j & 1;
      const uint32_t pa = smem_u32(sm + OFF_P + sb * PBUF);  // E4M3 weights [64][128 B]: terms at +0, +64
      const uint32_t pr = pa + kH * 128;                     // bf16 P [64][128 B]
      const uint32_t ka = smem_u32(sm + OFF_K + (j % kNB) * KBUF);
#pragma unroll
      for (int kk = 0; kk < kTR / 32; ++kk) {
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint64_t ad = smem_desc(pa + part * 64 + kk * 32, 16, 1024, kSw128);
          const bool acc = j > 0 || kk > 0 || part > 0;
          mma_ss<1>(tmem, ad, smem_desc(ka + kk * 2048, kAtom, 512, kSw64), idesc_pv8a, acc);
          mma_ss<1>(tmem + 256, ad, smem_desc(ka + 4 * kAtom + kk * 2048, kAtom, 512, kSw64), idesc_pv8b, acc);
        }
      }
#pragma unroll
      for (int kk = 0; kk < kTR / 16; ++kk)
        mma_ss<0>(tmem + kNope, smem_desc(pr + kk * 32, 16, 1024, kSw128),
                  smem_desc(ka + KB_ROPE + kk * 2048, 8192, 1024, kSw128), idesc_pvr, j > 0 || kk > 0);
      tc_commit(&pv_done[sb]);
      tc_commit(&k_free[j % kNB]);
    };
    if (warp == kMmaWarp) {
      // A test of the failure path (lcsc_set_wait_test): first wait on the
      // drain barrier, which cannot complete before this warp's own commit
      // below, so the wait runs out and the CTA aborts.
      const bool go = !a.waits.stall || warp_wait(drain, 0u, a, abort);
      for (int j = 0; go && j < ntiles; ++j) {
        if (j == 0 && !warp_wait(q_full, 0, a, abort)) break;
        if (!warp_wait(&k_full[j % kNB], (uint32_t)(j / kNB) & 1u, a, abort)) break;
        if (j >= 2 && !warp_wait(&p_full[j & 1], (uint32_t)((j - 2) >> 1) & 1u, a, abort)) break;
        tc_fence_after();
        if (lane == 0) issue_qk(j);
        __syncwarp();
      }
    } else {
      for (int j = 0; j < ntiles; ++j) {
        if (!warp_wait(&p_full[j & 1], (uint32_t)(j >> 1) & 1u, a, abort)) break;
        tc_fence_after();
        if (lane == 0) issue_pv(j);
        __syncwarp();
      }
    }
    // whether the loop ended or gave up, the MMAs of both issuers finish
    // before the CTA frees TMEM (bounded: a commit that never arrives is left
    // behind)
    if (lane == 0) {
      tc_commit(drain);
      mbar_wait(drain, 0, a.status, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // =================================================== softmax warps
    // Fragment layout (16x256b loads): thread t holds heads h0 = 16 w + t/4
    // and h1 = h0 + 8, at columns 8 g + 2 (t % 4) + {0, 1} of every 8-column
    // group g; register k: head (k / 2) % 2, group k / 4, column k % 2.
    const int q4 = lane & 3;
    const int hh[2] = {warp * 16 + (lane >> 2), warp * 16 + (lane >> 2) + 8};
    // the query's per-head scales (and, for warp 0's first thread, the end of
    // the copy it issued, before the CTA can exit)
    const bool q_in = warp_wait(q_full, 0, a, abort);
    const uint32_t o_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t s_addr = o_addr + (16u << 16);
    float c2[2], m_ref[2], l_part[2], gw[2];
    int g_exp[2];
    bool o_live[2], g_set[2];  // O may hold nonzero rows; g_h has been chosen
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      // this head's logit scale: sm_scale times the power of two q was divided by
      c2[e] = a.sm_scale * qsc_s[hh[e]] * kLog2e;
      m_ref[e] = -INFINITY;
      l_part[e] = 0.f;
      g_exp[e] = 0;
      gw[e] = 1.f;
      o_live[e] = g_set[e] = false;
    }
    for (int j = 0; q_in && j < ntiles; ++j) {
      const int sb = j & 1, slot = j & 3;
      // k_full orders the loaders' row mask and scales before these reads; s_full the TMEM S
      if (!warp_wait(&k_full[j % kNB], (uint32_t)(j / kNB) & 1u, a, abort)) break;
      if (!warp_wait(&s_full[sb], (uint32_t)(j >> 1) & 1u, a, abort)) break;
      tc_fence_after();
      uint32_t sn[32], sr[32];
      tmem_ld_16x256b_x8(s_addr + sb * kTR, sn);
      tmem_ld_16x256b_x8(s_addr + 2 * kTR + sb * kTR, sr);
      tmem_ld_wait(sn, sr);
      const float* scl = scl_s + slot * kTR;
      const uint32_t m0 = mask_s[slot * 2], m1 = mask_s[slot * 2 + 1];
      const bool full = (m0 & m1) == 0xFFFFFFFFu;  // every row of the tile valid (the common case)
      // logits (in units of the scaled query): s = c_r * codes part + RoPE part
      float v[32];
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float2 sc = *reinterpret_cast<const float2*>(scl + 8 * g + 2 * q4);
        const int col = 8 * g + 2 * q4;
        const uint32_t mw = col < 32 ? m0 : m1;
        const bool ok0 = full || ((mw >> (col & 31)) & 1u), ok1 = full || ((mw >> ((col + 1) & 31)) & 1u);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int k = 4 * g + 2 * e;
          v[k] = ok0 ? fmaf(__uint_as_float(sn[k]), sc.x, __uint_as_float(sr[k])) : -INFINITY;
          v[k + 1] = ok1 ? fmaf(__uint_as_float(sn[k + 1]), sc.y, __uint_as_float(sr[k + 1])) : -INFINITY;
          mx[e] = fmaxf(mx[e], fmaxf(v[k], v[k + 1]));
        }
      }
      float alpha[2] = {1.f, 1.f};
      bool moved[2] = {false, false};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 2));
        // reference max (natural-log units of the scaled logit): set on the
        // first rows seen, moved only by large jumps
        const float ms = mx[e] * (c2[e] * (1.f / kLog2e));  // sm_scale > 0 keeps the order
        if (mx[e] > -INFINITY && (m_ref[e] == -INFINITY || ms > m_ref[e] + kRescale)) {
          if (m_ref[e] > -INFINITY) {
            alpha[e] = __expf(m_ref[e] - ms);
            moved[e] = true;
            l_part[e] *= alpha[e];
          }
          m_ref[e] = ms;
        }
      }
      // p = exp(s * sm_scale - ref) = 2^(s * c2 - ref * log2 e): one FFMA and one EX2;
      // the code weight is p * c_r * g_h (formed again where it is stored)
      float wmax[2] = {0.f, 0.f};
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float2 sc = *reinterpret_cast<const float2*>(scl + 8 * g + 2 * q4);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int k = 4 * g + 2 * e;
          const float ref2 = m_ref[e] * kLog2e;
          const bool live = m_ref[e] > -INFINITY;
          const float p0 = live ? ex2(fmaf(v[k], c2[e], -ref2)) : 0.f;
          const float p1 = live ? ex2(fmaf(v[k + 1], c2[e], -ref2)) : 0.f;
          l_part[e] += p0 + p1;
          v[k] = p0;
          v[k + 1] = p1;
          wmax[e] = fmaxf(wmax[e], fmaxf(p0 * sc.x, p1 * sc.y));
        }
      }
      // g_h: re-chosen when the reference moved, on the first weights of the
      // head, or when a weight would leave the E4M3 range; the largest weight
      // of this tile then sits in [8, 16)
      float beta[2] = {1.f, 1.f};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        wmax[e] = fmaxf(wmax[e], __shfl_xor_sync(0xffffffffu, wmax[e], 1));
        wmax[e] = fmaxf(wmax[e], __shfl_xor_sync(0xffffffffu, wmax[e], 2)) * gw[e];
        if (wmax[e] > 0.f && (moved[e] || !g_set[e] || wmax[e] > kWeightHi)) {
          const int ex = ((__float_as_int(wmax[e]) >> 23) & 0xff) - 127;  // wmax in [2^ex, 2^(ex+1))
          int ge = g_exp[e] + (3 - ex);
          ge = ge < -120 ? -120 : (ge > 120 ? 120 : ge);
          beta[e] = pow2(ge - g_exp[e]);
          g_exp[e] = ge;
          gw[e] = pow2(ge);
        }
      }
      // P[sb] is free once the P V of tile j-2 is done
      if (j >= 2 && !warp_wait(&pv_done[sb], (uint32_t)((j - 2) >> 1) & 1u, a, abort)) break;
      uint8_t* pb = sm + OFF_P + sb * PBUF;
      const float gb[2] = {gw[0], gw[1]};  // g_h after the choice above
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int col = 8 * g + 2 * q4;
        const float2 sc = *reinterpret_cast<const float2*>(scl + col);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int k = 4 * g + 2 * e, h = hh[e];
          uint16_t hi, lo;
          e4m3_split2_h(v[k] * (sc.x * gb[e]), v[k + 1] * (sc.y * gb[e]), hi, lo);
          *reinterpret_cast<uint16_t*>(pb + swz128(h, col)) = hi;
          *reinterpret_cast<uint16_t*>(pb + swz128(h, 64 + col)) = lo;
          *reinterpret_cast<uint32_t*>(pb + kH * 128 + swz128(h, 2 * col)) = bf16x2(v[k], v[k + 1]);
        }
      }
      // O is rescaled in place (lanes 0-15) only after the previous P V is done
      const bool need[2] = {o_live[0] && (moved[0] || beta[0] != 1.f), o_live[1] && (moved[1] || beta[1] != 1.f)};
      if (__any_sync(0xffffffffu, need[0] || need[1])) {
        if (!warp_wait(&pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, a, abort)) break;
        tc_fence_after();
        const float fa[2] = {alpha[0] * beta[0], alpha[1] * beta[1]};  // code columns
        for (int c = 0; c < kD; c += 64) {
          uint32_t r[32];
          tmem_ld_16x256b_x8(o_addr + c, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int e = (q >> 1) & 1;
            const float f = c < kNope ? fa[e] : alpha[e];
            r[q] = __float_as_uint(__uint_as_float(r[q]) * f);
          }
          tmem_st_16x256b_x8(o_addr + c, r);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        o_live[e] = o_live[e] || m_ref[e] > -INFINITY;
        g_set[e] = g_set[e] || wmax[e] > 0.f;
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    // ---- partial results: wait for the last PV, then O (lanes 0-15) and (ref, sum)
    bool done = ntiles > 0 && !*abort;
    if (done) done = warp_wait(&pv_done[(ntiles - 1) & 1], (uint32_t)((ntiles - 1) >> 1) & 1u, a, abort);
    tc_fence_after();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 1);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 2);
    }
    // the 32x32b layout of the stores below: lane i < 16 holds head 16 w + i,
    // whose values sit with thread 4 (i % 8), as its head i / 8
    const int src = 4 * (lane & 7);
    const float m0v = __shfl_sync(0xffffffffu, m_ref[0], src), m1v = __shfl_sync(0xffffffffu, m_ref[1], src);
    const float l0v = __shfl_sync(0xffffffffu, l_part[0], src), l1v = __shfl_sync(0xffffffffu, l_part[1], src);
    const float g0v = __shfl_sync(0xffffffffu, gw[0], src), g1v = __shfl_sync(0xffffffffu, gw[1], src);
    const bool upper = (lane & 15) >= 8;
    const int head = warp * 16 + (lane & 15);
    const float m_h = done ? (upper ? m1v : m0v) : -INFINITY;
    const float l_h = done ? (upper ? l1v : l0v) : 0.f;
    const float inv_g = 1.f / (upper ? g1v : g0v);
    const int64_t pidx = ((int64_t)list * a.splits + blockIdx.x) * a.H + head;
    // One split per query: the merge with the sink happens here (the same
    // arithmetic as the split-combine kernel) and O leaves normalised.
    float o_scale = 1.f;
    if (a.splits == 1) {
      const float sigma = a.sink ? a.sink[head] : -INFINITY;
      float M = sigma, den = sigma > -INFINITY ? 1.f : 0.f;  // the sink's e^(sigma - M)
      if (m_h > M) {
        den *= M > -INFINITY ? expf(M - m_h) : 0.f;
        M = m_h;
      }
      float f = 0.f;
      if (m_h > -INFINITY) {
        f = expf(m_h - M);
        den = fmaf(l_h, f, den);
      }
      o_scale = den > 0.f ? f * (1.f / den) : 0.f;
      if (a.lse && lane < 16) a.lse[(int64_t)list * a.H + head] = den > 0.f ? M + logf(den) : -INFINITY;
    }
    // O -> shared memory (the tile buffers and P are dead: every P V is done),
    // padded rows so the 16-byte stores of a warp's heads hit distinct banks
    float* o_s = reinterpret_cast<float*>(sm + OFF_K);
    for (int c = 0; c < kD; c += 64) {  // two TMEM loads in flight
      uint32_t r0[32], r1[32];
      tmem_ld_32(o_addr + c, r0);
      tmem_ld_32(o_addr + c + 32, r1);
      tmem_ld_wait(r0, r1);
      const float f0 = done ? o_scale * (c < kNope ? inv_g : 1.f) : 0.f;
      const float f1 = done ? o_scale * (c + 32 < kNope ? inv_g : 1.f) : 0.f;
      if (lane < 16) {
        float* po = o_s + head * kOS + c;
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          *reinterpret_cast<float4*>(po + q) =
              make_float4(__uint_as_float(r0[q]) * f0, __uint_as_float(r0[q + 1]) * f0,
                          __uint_as_float(r0[q + 2]) * f0, __uint_as_float(r0[q + 3]) * f0);
          *reinterpret_cast<float4*>(po + 32 + q) =
              make_float4(__uint_as_float(r1[q]) * f1, __uint_as_float(r1[q + 1]) * f1,
                          __uint_as_float(r1[q + 2]) * f1, __uint_as_float(r1[q + 3]) * f1);
        }
      }
    }
    if (lane < 16 && a.splits > 1) {
      a.part_ml[pidx * 2] = m_h;
      a.part_ml[pidx * 2 + 1] = l_h;
    }
  }
  // the query image's copies have landed before the CTA can end (they have on
  // every path but an abort that came before them; bounded)
  if (tid == 0) mbar_wait(q_full, 0, nullptr, kDrainLimitNs);
  tc_fence_before();
  __syncthreads();
  {  // O of this split, [64 heads][512] contiguous: coalesced stores by every thread, of the
     // partial (several splits) or of the output in the query's type (one split)
    const float* o_s = reinterpret_cast<const float*>(sm + OFF_K);
    auto row4 = [&](int i) { return *reinterpret_cast<const float4*>(o_s + (i / (kD / 4)) * kOS + 4 * (i % (kD / 4))); };
    // one split: the output itself, rotated back by the query position where
    // asked (a thread's dims are the same in every row: kThr is a multiple
    // of kD / 4)
    static_assert(kThr % (kD / 4) == 0, "fixed dims per thread");
    RopePair2 rot;
    const bool turn = a.splits == 1 &&
                      inverse_rope_angles(4 * (tid % (kD / 4)), kD, a.out_rope_dim, a.out_rope_base,
                                          (int64_t)a.ctx_len[list / a.T] - a.T + list % a.T, &rot);
    auto out4 = [&](int i) { return turn ? rotate2(row4(i), rot) : row4(i); };
    if (a.splits > 1) {
      float4* dst = reinterpret_cast<float4*>(a.part_o + ((int64_t)list * a.splits + blockIdx.x) * a.H * kD);
      for (int i = tid; i < kH * (kD / 4); i += kThr) dst[i] = row4(i);
    } else if (a.q_dtype == LCSC_DT_BF16) {
      uint2* dst = reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.out) + (int64_t)list * a.H * kD);
      for (int i = tid; i < kH * (kD / 4); i += kThr) {
        const float4 v = out4(i);
        dst[i] = make_uint2(bf16x2(v.x, v.y), bf16x2(v.z, v.w));
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + (int64_t)list * a.H * kD);
      for (int i = tid; i < kH * (kD / 4); i += kThr) dst[i] = out4(i);
    }
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attn_mma_supported(const AttnLaunch& a) {
  return a.kv.f.fmt == LCSC_FMT_KV && a.D == 512 && a.Dv == 512 && a.H == 64 && a.v.data == nullptr &&
         a.kv.f.row_bytes == 576 && a.kv.f.rope == 64 && a.rows_per_split % kTR == 0;
}

cudaError_t launch_attn_qimage(const AttnLaunch& a, cudaStream_t stream) {
  constexpr int kImgSmem = (int)kAttnQImageBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_qimage_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kImgSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_qimage_kernel, dim3(a.B * a.T), dim3(kThr), kImgSmem, stream, a);
}

cudaError_t launch_attn_mma(const AttnLaunch& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  AttnLaunch la = a;
  la.waits = wait_test();
  return launch_pdl(attn_mma_kernel, dim3(a.splits, a.B * a.T), dim3(kThr), SMEM, stream, la);
}

}  // namespace lcsc
