// Joint attention on the 5th-generation tensor cores: all 64 query heads of
// one query against one shared 512-d KV row set (FP8 + BF16 RoPE storage).
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works" (exact attention over the selected
// compressed entries plus the uncompressed window, shared-KV multi-query
// layout; the sink enters in the combine step).
//
// One CTA owns (query, range of rows) and walks it in tiles of 64 rows with a
// warp-specialised pipeline:
//  * 11 loader warps resolve the tile's rows (gathered by index for CSA; dense
//    tiles are also prefetched into L2 two tiles ahead), read them and
//    dequantise them once into shared memory as f16, in a 128-byte-swizzled
//    layout that is both a K-major operand for Q K^T and an MN-major operand
//    for P V (the same bytes are K and V); two buffers, so tile t+1 is loaded
//    while tile t is being used;
//  * 1 MMA warp issues S = Q K^T (M = 64 heads, N = 64 rows, K = 512) for tile
//    t+1 as soon as it is loaded, and O += P V (N = 2 x 256 dims, K = 64) for
//    tile t once its probabilities are ready;
//  * 4 softmax warps, one thread per head, read S from TMEM, keep a running
//    reference max (O is rescaled only when the max grows by more than e^8),
//    and write P = exp(S - ref) as f16.
// Heads live on M = 64, so S and O use the half-lane TMEM layout: O at
// lanes 0-15 of each 32-lane sub-partition (all 512 columns), S (two
// 64-column buffers) at lanes 16-31.  With several splits per query the
// partial (ref max, sum, O) goes to the workspace the combine kernel merges;
// with one, the kernel merges the sink itself and writes the output.
#include "kernels.cuh"
#include "launches.h"
#include "rope.cuh"
#include "sm100.cuh"

namespace lcsc {
namespace {

using namespace sm100;

constexpr int kH = 64;       // heads (MMA M)
constexpr int kD = 512;      // row length (K of Q K^T, N of P V)
constexpr int kTR = 64;      // rows per tile
constexpr int kLW = 11;      // loader warps (16 warps in all: 4 per SM sub-partition)
constexpr int kSW = 4;       // softmax warps
constexpr int kThr = (kSW + kLW + 1) * 32;
constexpr int kMmaWarp = kSW + kLW;
constexpr int kFp8Chunks = 28;  // 16-byte FP8 chunks of a stored row (448 dims)
constexpr int kLT = kLW * 32;   // loader threads
constexpr int kFp8Units = kTR * kFp8Chunks, kBfUnits = kTR * 8;  // 16-byte chunks of a tile
constexpr int kFp8Loads = (kFp8Units + kLT - 1) / kLT;           // FP8 chunks per loader thread
constexpr int kLoads = kFp8Loads + (kBfUnits + kLT - 1) / kLT;   // + BF16 chunks
// the partial last FP8 and BF16 rounds are taken by whole warps
static_assert((kFp8Units % kLT) % 32 == 0 && (kBfUnits % kLT) % 32 == 0, "warp-uniform rounds");
constexpr float kRescale = 8.f;
constexpr float kLog2e = 1.4426950408889634f;  // log2(e), to work in base 2  // rescale O only when the max grows by more

// shared memory (offsets from a 1024-aligned base)
constexpr int kOS = kD + 4;       // row stride (floats) of the partial O staged in shared memory
constexpr int KB_Q = kH * 128;    // one 64-dim block of Q  (8 KB)
constexpr int KB_K = kTR * 128;   // one 64-dim block of a K tile (8 KB)
constexpr int OFF_Q = 0;                       // 8 blocks = 64 KB
constexpr int OFF_K = OFF_Q + 8 * KB_Q;        // 2 buffers x 8 blocks = 128 KB
constexpr int OFF_P = OFF_K + 2 * 8 * KB_K;    // 2 buffers x [64 heads][128 B] = 16 KB
constexpr int OFF_BAR = OFF_P + 2 * kH * 128;  // k_full[2] s_full[2] p_full[2] pv_done[2] drain
constexpr int OFF_ROW = OFF_BAR + 9 * 8;       // int64 [4][64] (row info of tiles j % 4)
constexpr int OFF_SRC = OFF_ROW + 4 * kTR * 8;  // int32 [4][64]
constexpr int OFF_SCL = OFF_SRC + 4 * kTR * 4;  // float [4][64]
constexpr int OFF_SCH = OFF_SCL + 4 * kTR * 4;  // f16x2 scale [4][64]
constexpr int OFF_NRM = OFF_SCH + 4 * kTR * 4;  // uint32 [4][2]: every scale of a tile a normal f16
constexpr int OFF_MASK = OFF_NRM + 32;          // uint32 [2][2] valid-row bits
constexpr int OFF_TM = OFF_MASK + 16;
constexpr int OFF_ABORT = OFF_TM + 4;
constexpr int OFF_LSTOP = OFF_ABORT + 4;
constexpr int OFF_QSC = OFF_LSTOP + 4;          // float [64]: per-head amax of q, then its power-of-two scale
constexpr int SMEM = OFF_QSC + kH * 4 + 1024;
// Largest row scale whose E4M3 codes (|code| <= 448) stay finite as f16.
constexpr float kMaxRowScale = 65504.f / 448.f;
static_assert(kH * kOS * 4 <= OFF_BAR - OFF_K, "the staged partial O fits in the K and P buffers");

// Byte offset of (row, byte) in a [rows][128 B] block with the 128-byte swizzle
// (16-byte chunk index XOR row % 8) that the tensor cores read.
__device__ __forceinline__ uint32_t swz(int row, int byte) {
  return (uint32_t)(row * 128 + ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 2^x on the MUFU unit (approximate, flush-to-zero), the base-2 exponential
// the softmax works in.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
  bool ok = mbar_wait(bar, parity, a.status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) *abort = 1;
  return ok;
}

__global__ void __maxnreg__(128) attn_mma_kernel(const AttnLaunch a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* k_full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* s_full = k_full + 2;
  uint64_t* p_full = k_full + 4;
  uint64_t* pv_done = k_full + 6;
  uint64_t* drain = k_full + 8;  // every MMA issued has completed (before TMEM is freed)
  int64_t* row_s = reinterpret_cast<int64_t*>(sm + OFF_ROW);
  int32_t* src_s = reinterpret_cast<int32_t*>(sm + OFF_SRC);
  float* scl_s = reinterpret_cast<float*>(sm + OFF_SCL);
  uint32_t* sch_s = reinterpret_cast<uint32_t*>(sm + OFF_SCH);
  volatile uint32_t* nrm_s = reinterpret_cast<volatile uint32_t*>(sm + OFF_NRM);
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

  if (tid < kH) qsc_s[tid] = 0.f;  // per-head amax of q (non-negative: compared as integers)
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSW);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    *lstop = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tm_slot, 512);

  // The rows of the first two tiles go to L2 before the query prologue, so
  // that the loaders' first gathers, issued after it, hit L2: one bulk
  // prefetch per dense tile of entries, one per gathered entry or window row.
  if (warp >= kSW && warp < kMmaWarp && tid - kSW * 32 < 2 * kTR) {
    const int lt = tid - kSW * 32, r = lt % kTR;
    const int64_t slot = s_lo + lt;
    const int64_t n_ent_here = s_hi < qr.n_ent_slots ? s_hi : qr.n_ent_slots;
    const uint32_t rb = (uint32_t)a.kv.f.row_bytes;
    if (slot < s_hi) {
      if (slot < qr.n_ent_slots) {
        if (a.idx) {
          const int64_t g = a.idx[(int64_t)list * a.k + slot];
          const int64_t lr = (g >= 0 && g < qr.n_vis) ? a.kv.local(g) : -1;
          if (lr >= 0) prefetch_l2(a.kv.row(b, lr), rb);
        } else if (r == 0) {
          const int64_t cnt = n_ent_here - slot < kTR ? n_ent_here - slot : kTR;
          prefetch_l2(a.kv.row(b, slot), (uint32_t)cnt * rb);
        }
      } else if (slot < qr.n_ent_slots + qr.n_win) {
        const int64_t cap = a.win_kv.capacity;
        prefetch_l2(a.win_kv.row(b, (qr.w_lo + (slot - qr.n_ent_slots)) % cap), rb);
      }
    }
  }

  // ---- Q (64 x 512) -> f16, K-major swizzled blocks of 64 dims (all threads;
  // bf16 rows: every 16-byte load of a thread in flight at once).  Each head
  // is multiplied by a power of two that puts its largest |q| in
  // [2^14, 2^15), so that any finite query keeps f16 precision; the softmax
  // multiplies that head's logits back (qsc_s holds 2^e per head).
  constexpr int kQChunks = kH * (kD / 8), kQIter = (kQChunks + kThr - 1) / kThr;
  static_assert(kThr % 64 == 0 && (kD / 8) == 64 && kQChunks % kThr == 0,
                "the lanes of a warp share one head per chunk round; every thread has kQIter chunks");
  // the multiplier 2^-e of head h from its amax (0: 1)
  auto q_mult = [&](int h) -> float {
    const int bits = __float_as_int(qsc_s[h]);
    if (bits == 0) return 1.f;
    int ex = ((bits >> 23) & 0xff) - 127 - 14;  // amax in [2^(ex+14), 2^(ex+15)) (normal amax)
    ex = ex < -126 ? -126 : (ex > 126 ? 126 : ex);
    return __int_as_float((127 - ex) << 23);
  };
  // Pass 1: each chunk's bf16 bits go to their final place in shared memory
  // (f16 and bf16 chunks have the same size) and its amax to the head's slot;
  // pass 2 converts every chunk in place once the head's scale is known.
  // fp32 rows are read from memory in both passes.
  const bool q_bf = a.q_dtype == LCSC_DT_BF16;
  auto q_addr = [&](int i) {
    const int h = i / (kD / 8), d0 = (i % (kD / 8)) * 8;
    return reinterpret_cast<uint4*>(sm + OFF_Q + (d0 / 64) * KB_Q + swz(h, (d0 % 64) * 2));
  };
  auto f32_chunk = [&](int i, float (&v)[8]) {
    const int64_t base = ((int64_t)list * a.H + i / (kD / 8)) * kD + (i % (kD / 8)) * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = load_elem(a.q, base + j, a.q_dtype);
  };
  __syncthreads();  // the amax slots are zero
  if (q_bf) {
    uint4 raw[kQIter];
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
      *q_addr(i) = raw[u];
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
  for (int u = 0; u < kQIter; ++u) {
    const int i = tid + u * kThr;
    const float f = q_mult(i / (kD / 8));
    float v[8];
    if (q_bf) {
      const uint4 r = *q_addr(i);
      const uint16_t* bf = reinterpret_cast<const uint16_t*>(&r);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = bf16_val(bf[j]) * f;
    } else {
      f32_chunk(i, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] *= f;
    }
    *q_addr(i) = make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]), pack_h2(v[6], v[7]));
  }
  __syncthreads();  // every multiplier was read: the slots now take 2^e
  if (tid < kH) qsc_s[tid] = 1.f / q_mult(tid);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tm_slot;

  if (warp >= kSW && warp < kMmaWarp) {
    // =================================================== loader warps
    // Software pipeline: the rows of tile j+1 are resolved and their bytes
    // requested (into a second register set) before tile j is dequantised.
    const int lt = tid - kSW * 32;  // 0 .. kLT - 1
    // Work units of a tile, fixed per thread for the whole kernel.  The
    // first kFp8Loads are 16-byte FP8 chunks (28 per row, 1792 in all): unit
    // u = lt + kLT i splits as q = u % 4, row-in-pair = (u / 4) % 2, then
    // 64-dim block (7) and row pair (32), so that the 8 lanes of a 128-bit
    // store phase cover 2 rows x 4 chunks of one block: distinct 16-byte bank
    // groups after the swizzle.  The rest are 16-byte BF16 chunks (8 per row,
    // 512 in all).  Table word: first f16 destination (16 bits) | row << 16 |
    // chunk << 22; all ones: no unit.
    uint32_t tab[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      int r, c;
      if (i < kFp8Loads) {
        const int u = lt + i * kLT, rest = u >> 3;
        if (u >= kFp8Units) {
          tab[i] = 0xFFFFFFFFu;
          continue;
        }
        r = 2 * (rest / 7) + ((u >> 2) & 1);
        c = 4 * (rest % 7) + (u & 3);
      } else {
        const int v = lt + (i - kFp8Loads) * kLT;
        if (v >= kBfUnits) {
          tab[i] = 0xFFFFFFFFu;
          continue;
        }
        r = v >> 3;
        c = kFp8Chunks + (v & 7);
      }
      const int dim = c < kFp8Chunks ? c * 16 : kFp8Chunks * 16 + (c - kFp8Chunks) * 8;
      const uint32_t d0 = (dim / 64) * KB_K + swz(r, (dim % 64) * 2);
      tab[i] = d0 | ((uint32_t)r << 16) | ((uint32_t)c << 22);
    }
    // Row-info threads (lt < 64, one per row of a tile) keep two global loads
    // in flight across steps: the gather index of the row one tile ahead of
    // the one being located, and the scale of the row just located.
    auto slot_of = [&](int j) { return s_lo + (int64_t)j * kTR + lt; };
    auto load_idx = [&](int j) -> int32_t {
      const int64_t slot = slot_of(j);
      return (a.idx && slot < s_hi && slot < qr.n_ent_slots) ? a.idx[(int64_t)list * a.k + slot] : 0;
    };
    // Row of tile j for this thread: pointer (null: no row) and scale address.
    // window ring row of window slot 0 (the ring index then only wraps once)
    const int64_t win_cap = a.win_kv.capacity;
    const int64_t win_base = win_cap > 0 ? qr.w_lo % win_cap : 0;  // no window: never used
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
    int32_t idx_next = 0;  // gather index of tile j+1's row (in flight)
    float sc_next = 1.f;   // scale of the row last located (in flight)
    auto place = [&](int j, int32_t gi) {  // tile j's row info -> row buffer j % 4
      const float* scp;
      const uint8_t* p = locate(j, gi, scp);
      row_s[(j & 3) * kTR + lt] = reinterpret_cast<int64_t>(p);
      src_s[(j & 3) * kTR + lt] = p != nullptr;
      sc_next = scp ? *scp : 1.f;
    };

    auto fetch = [&](int j, uint4 (&raw)[kLoads]) {
      const int64_t* rows = row_s + (j & 3) * kTR;
#pragma unroll
      for (int i = 0; i < kLoads; ++i) {
        raw[i] = make_uint4(0, 0, 0, 0);
        if (tab[i] == 0xFFFFFFFFu) continue;
        const uint8_t* ptr = reinterpret_cast<const uint8_t*>(rows[(tab[i] >> 16) & 63]);
        if (ptr) raw[i] = reinterpret_cast<const uint4*>(ptr)[tab[i] >> 22];
      }
    };
    auto convert = [&](int j, const uint4 (&raw)[kLoads]) {
      const float* scl = scl_s + (j & 3) * kTR;
      const uint32_t* sch = sch_s + (j & 3) * kTR;
      uint8_t* kt = sm + OFF_K + (j & 1) * (8 * KB_K);
      if (nrm_s[(j & 3) * 2] && nrm_s[(j & 3) * 2 + 1]) {
        // every row scale a normal f16 (the usual case): no per-unit branch,
        // so the units of a thread overlap
#pragma unroll
        for (int i = 0; i < kFp8Loads; ++i) {
          if (tab[i] == 0xFFFFFFFFu) continue;
          const uint32_t d0 = tab[i] & 0xFFFFu;
          const uint32_t s2u = sch[(tab[i] >> 16) & 63];
          const __half2 s2 = *reinterpret_cast<const __half2*>(&s2u);
          const uint16_t* c2 = reinterpret_cast<const uint16_t*>(&raw[i]);
          uint32_t h[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(c2[q], __NV_E4M3);
            const __half2 v = __hmul2(*reinterpret_cast<__half2*>(&hr), s2);
            h[q] = *reinterpret_cast<const uint32_t*>(&v);
          }
          *reinterpret_cast<uint4*>(kt + d0) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(kt + (d0 ^ 16u)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
      } else {
#pragma unroll
      for (int i = 0; i < kFp8Loads; ++i) {
        if (tab[i] == 0xFFFFFFFFu) continue;
        const uint32_t d0 = tab[i] & 0xFFFFu;
        const float sc = scl[(tab[i] >> 16) & 63];
        const uint16_t* c2 = reinterpret_cast<const uint16_t*>(&raw[i]);
        uint32_t h[8];
        if (sc >= 6.103515625e-05f && sc <= 65504.f) {  // a normal f16 scale: multiply in f16x2
          const __half2 s2 = __float2half2_rn(sc);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(c2[q], __NV_E4M3);
            const __half2 v = __hmul2(*reinterpret_cast<__half2*>(&hr), s2);
            h[q] = *reinterpret_cast<const uint32_t*>(&v);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float2 f = e4m3x2_val(c2[q]);
            h[q] = pack_h2(f.x * sc, f.y * sc);
          }
        }
        // the second 16 bytes are the next 16-byte chunk: swizzled position ^ 1
        *reinterpret_cast<uint4*>(kt + d0) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(kt + (d0 ^ 16u)) = make_uint4(h[4], h[5], h[6], h[7]);
      }
      }
#pragma unroll
      for (int i = kFp8Loads; i < kLoads; ++i) {
        if (tab[i] == 0xFFFFFFFFu) continue;
        const uint16_t* bf = reinterpret_cast<const uint16_t*>(&raw[i]);
        uint32_t h[4];
        float big = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float x0 = bf16_val(bf[2 * q]), x1 = bf16_val(bf[2 * q + 1]);
          big = fmaxf(big, fmaxf(fabsf(x0), fabsf(x1)));
          h[q] = pack_h2(x0, x1);
        }
        if (big > 65504.f && a.status) atomicOr(a.status, LCSC_DEV_RANGE);
        *reinterpret_cast<uint4*>(kt + (tab[i] & 0xFFFFu)) = make_uint4(h[0], h[1], h[2], h[3]);
      }
      if (lt < kTR) {  // valid-row bits of tile j, read by the softmax after k_full
        const uint32_t bits = __ballot_sync(0xffffffffu, src_s[(j & 3) * kTR + lt] != 0);
        if (lane == 0) mask_s[(j & 1) * 2 + (lt >> 5)] = bits;
      }
    };
    // One step: tile j+1 located and requested, tile j stored.  false: stop.
    auto step = [&](int j, const uint4 (&cur)[kLoads], uint4 (&nxt)[kLoads]) -> bool {
      if (!a.idx && lt == 0 && j + 2 < ntiles) {
        // dense entries are contiguous: tile j+2's rows go to L2 now, in one
        // bulk prefetch, a step before their loads are issued (rows are
        // 576 B from a 16-byte-aligned base, so the start is aligned)
        const int64_t g0 = slot_of(j + 2) - lt;
        const int64_t hi = s_hi < qr.n_ent_slots ? s_hi : qr.n_ent_slots;
        if (g0 < hi) {
          const int64_t cnt = hi - g0 < kTR ? hi - g0 : kTR;
          prefetch_l2(a.kv.row(b, g0), (uint32_t)(cnt * a.kv.f.row_bytes));
        }
      }
      if (lt < kTR) {
        scl_s[(j & 3) * kTR + lt] = sc_next;  // tile j's scale, loaded one step ago
        if (!(sc_next <= kMaxRowScale) && a.status) atomicOr(a.status, LCSC_DEV_RANGE);
        const bool nrm = sc_next >= 6.103515625e-05f && sc_next <= 65504.f;
        const __half2 s2 = __float2half2_rn(nrm ? sc_next : 0.f);
        sch_s[(j & 3) * kTR + lt] = *reinterpret_cast<const uint32_t*>(&s2);
        const uint32_t all = __ballot_sync(0xffffffffu, nrm);
        if (lane == 0) nrm_s[(j & 3) * 2 + (lt >> 5)] = all == 0xffffffffu;
        if (j + 1 < ntiles) {
          place(j + 1, idx_next);
          if (j + 2 < ntiles) idx_next = load_idx(j + 2);
        }
      }
      named_sync(1, kLW * 32);
      if (j + 1 < ntiles) fetch(j + 1, nxt);
      // One thread decides for the group (K[j % 2] is free once the PV of
      // tile j-2 is done); `lstop` is written only here, between group
      // barriers, so every loader reads the same value.
      if (lt == 0) {
        bool ok = !*abort;
        if (ok && j >= 2) ok = mbar_wait(&pv_done[j & 1], (uint32_t)((j - 2) >> 1) & 1u, a.status);
        if (!ok) *abort = 1;
        *lstop = ok ? 0 : 1;
      }
      named_sync(1, kLW * 32);
      if (*lstop) return false;
      convert(j, cur);
      fence_async_smem();
      named_sync(1, kLW * 32);
      if (lt == 0) mbar_arrive(&k_full[j & 1]);
      return true;
    };
    uint4 ra[kLoads], rb[kLoads];
    if (ntiles > 0) {
      if (lt < kTR) {
        place(0, load_idx(0));
        if (ntiles > 1) idx_next = load_idx(1);
      }
      named_sync(1, kLW * 32);
      fetch(0, ra);
    }
    for (int j = 0; j < ntiles; j += 2) {
      if (!step(j, ra, rb)) break;
      if (j + 1 < ntiles && !step(j + 1, rb, ra)) break;
    }
  } else if (warp == kMmaWarp) {
    // =================================================== MMA warp
    const uint32_t idesc_qk = idesc_dense(0, 0, 64, kTR);
    const uint32_t idesc_pv = idesc_dense(0, 0, 64, 256, false, true);
    const uint32_t qa = smem_u32(sm + OFF_Q);
    auto issue_qk = [&](int j) {
      const int buf = j & 1;
      const uint32_t ka = smem_u32(sm + OFF_K + buf * (8 * KB_K));
#pragma unroll 4
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t kb = kk / 4, ko = (kk % 4) * 32;
        mma_ss<0>(tmem + (16u << 16) + buf * kTR, smem_desc(qa + kb * KB_Q + ko, 16, 1024, kSw128),
                  smem_desc(ka + kb * KB_K + ko, 16, 1024, kSw128), idesc_qk, kk > 0);
      }
      tc_commit(&s_full[buf]);
    };
    auto issue_pv = [&](int j) {
      const int buf = j & 1;
      const uint32_t pa = smem_u32(sm + OFF_P + buf * (kH * 128));
      const uint32_t ka = smem_u32(sm + OFF_K + buf * (8 * KB_K));
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
        for (int kk = 0; kk < kTR / 16; ++kk) {
          const uint64_t adesc = smem_desc(pa + kk * 32, 16, 1024, kSw128);
          const uint64_t bdesc = smem_desc(ka + nh * 4 * KB_K + kk * 2048, KB_K, 1024, kSw128);
          mma_ss<0>(tmem + nh * 256, adesc, bdesc, idesc_pv, j > 0 || kk > 0);
        }
      }
      tc_commit(&pv_done[buf]);
    };
    // Q K^T of tile q and P V of tile v are issued in whichever order their
    // inputs become ready, so that a late tile load never holds back the P V
    // that frees a K buffer.  Q K^T of tile q also needs S[q % 2] free: the
    // softmax of tile q-2 has published its P (seen before P V of q-2 went out).
    int nq = 0, nv = 0;
    uint64_t t_last = global_timer_ns();
    while (nv < ntiles) {
      bool progressed = false;
      if (nq < ntiles && nq <= nv + 1) {
        const bool ready = __all_sync(0xffffffffu, mbar_test_wait(&k_full[nq & 1], (uint32_t)(nq >> 1) & 1u));
        if (ready) {
          tc_fence_after();
          if (lane == 0) issue_qk(nq);
          __syncwarp();
          ++nq;
          progressed = true;
        }
      }
      if (nv < nq) {
        const bool ready = __all_sync(0xffffffffu, mbar_test_wait(&p_full[nv & 1], (uint32_t)(nv >> 1) & 1u));
        if (ready) {
          tc_fence_after();
          if (lane == 0) issue_pv(nv);
          __syncwarp();
          ++nv;
          progressed = true;
        }
      }
      if (progressed) {
        t_last = global_timer_ns();
      } else {
        bool stop = *abort != 0;
        if (!stop && global_timer_ns() - t_last > kWaitLimitNs) {
          if (lane == 0 && a.status) atomicOr(a.status, LCSC_DEV_TIMEOUT);
          stop = true;
        }
        if (__any_sync(0xffffffffu, stop)) {
          if (lane == 0) *abort = 1;
          break;
        }
      }
    }
    // whether the loop ended or gave up, the MMAs it issued finish before the
    // CTA frees TMEM (bounded: a commit that never arrives is left behind)
    if (lane == 0) {
      tc_commit(drain);
      mbar_wait(drain, 0, a.status, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // =================================================== softmax warps
    const bool s_lane = lane >= 16;
    const int head = warp * 16 + (lane & 15);
    const uint32_t row_addr = tmem + ((uint32_t)(warp * 32) << 16);
    // this head's logit scale: sm_scale times the power of two q was divided by
    const float sm_h = a.sm_scale * qsc_s[head];
    float m_ref = -INFINITY, l_sum = 0.f;
    for (int j = 0; j < ntiles; ++j) {
      const int buf = j & 1;
      // k_full orders the loaders' row mask before this read; s_full the TMEM S
      if (!warp_wait(&k_full[buf], (uint32_t)(j >> 1) & 1u, a, abort)) break;
      if (!warp_wait(&s_full[buf], (uint32_t)(j >> 1) & 1u, a, abort)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld_32(row_addr + buf * kTR, r0);
      tmem_ld_32(row_addr + buf * kTR + 32, r1);
      tmem_ld_wait(r0, r1);
      const uint32_t m0 = mask_s[buf * 2], m1 = mask_s[buf * 2 + 1];
      const bool full = (m0 & m1) == 0xFFFFFFFFu;  // every row of the tile valid (the common case)
      float mx = -INFINITY;
      if (full) {
        float mm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mm[q] = fmaxf(__uint_as_float(r0[q]), __uint_as_float(r1[q]));
#pragma unroll
        for (int q = 8; q < 32; ++q) mm[q & 7] = fmaxf(mm[q & 7], fmaxf(__uint_as_float(r0[q]), __uint_as_float(r1[q])));
        mx = fmaxf(fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3])), fmaxf(fmaxf(mm[4], mm[5]), fmaxf(mm[6], mm[7])));
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          if ((m0 >> q) & 1u) mx = fmaxf(mx, __uint_as_float(r0[q]));
          if ((m1 >> q) & 1u) mx = fmaxf(mx, __uint_as_float(r1[q]));
        }
      }
      mx *= sm_h;  // sm_scale > 0 keeps the order
      // reference max: set on the first rows seen, moved only by large jumps
      float alpha = 1.f;
      bool moved = false;
      if (s_lane && mx > -INFINITY && (m_ref == -INFINITY || mx > m_ref + kRescale)) {
        if (m_ref > -INFINITY) {
          alpha = __expf(m_ref - mx);
          moved = true;
          l_sum *= alpha;
        }
        m_ref = mx;
      }
      // p = exp(s * sm_scale - ref) = 2^(s * c2 - ref * log2 e): one FFMA and one EX2
      const float ref = m_ref;
      const float c2 = sm_h * kLog2e, ref2 = ref * kLog2e;
      float sum = 0.f;
      uint32_t pk[32];
      if (full && ref > -INFINITY) {
        float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const float p0 = ex2(fmaf(__uint_as_float(r0[q]), c2, -ref2));
          const float p1 = ex2(fmaf(__uint_as_float(r0[q + 1]), c2, -ref2));
          const float p2 = ex2(fmaf(__uint_as_float(r1[q]), c2, -ref2));
          const float p3 = ex2(fmaf(__uint_as_float(r1[q + 1]), c2, -ref2));
          sp[0] += p0;
          sp[1] += p1;
          sp[2] += p2;
          sp[3] += p3;
          pk[q / 2] = pack_h2(p0, p1);
          pk[16 + q / 2] = pack_h2(p2, p3);
        }
        sum = (sp[0] + sp[1]) + (sp[2] + sp[3]);
      } else {
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const bool live = ref > -INFINITY;
          const float p0 = ((m0 >> q) & 1u) && live ? ex2(fmaf(__uint_as_float(r0[q]), c2, -ref2)) : 0.f;
          const float p1 = ((m0 >> (q + 1)) & 1u) && live ? ex2(fmaf(__uint_as_float(r0[q + 1]), c2, -ref2)) : 0.f;
          const float p2 = ((m1 >> q) & 1u) && live ? ex2(fmaf(__uint_as_float(r1[q]), c2, -ref2)) : 0.f;
          const float p3 = ((m1 >> (q + 1)) & 1u) && live ? ex2(fmaf(__uint_as_float(r1[q + 1]), c2, -ref2)) : 0.f;
          sum += (p0 + p1) + (p2 + p3);
          pk[q / 2] = pack_h2(p0, p1);
          pk[16 + q / 2] = pack_h2(p2, p3);
        }
      }
      if (s_lane) l_sum += sum;
      // O is rescaled in place (lanes 0-15) only after the previous PV is done
      const bool warp_moved = __any_sync(0xffffffffu, moved);
      if (warp_moved && j > 0) {
        if (!warp_wait(&pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, a, abort)) break;
        tc_fence_after();
        // O's 16 lanes only (the S lanes above them may be taking the next
        // tile's Q K^T): thread t holds heads t/4 and t/4 + 8 of the warp's 16
        const float a_lo = __shfl_sync(0xffffffffu, alpha, 16 + (lane >> 2));
        const float a_hi = __shfl_sync(0xffffffffu, alpha, 16 + (lane >> 2) + 8);
        for (int c = 0; c < kD; c += 64) {
          uint32_t r[32];
          tmem_ld_16x256b_x8(row_addr + c, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * (((q >> 1) & 1) ? a_hi : a_lo));
          tmem_st_16x256b_x8(row_addr + c, r);
        }
        tmem_st_wait();
      }
      // P[buf] is free once the PV of tile j-2 is done
      if (j >= 2 && !warp_wait(&pv_done[buf], (uint32_t)((j - 2) >> 1) & 1u, a, abort)) break;
      if (s_lane) {
        uint8_t* pb = sm + OFF_P + buf * (kH * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(pb + swz(head, q * 16)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[buf]);
    }
    // ---- partial results: wait for the last PV, then O (lanes 0-15) and (ref, sum)
    bool done = ntiles > 0 && !*abort;
    if (done) done = warp_wait(&pv_done[(ntiles - 1) & 1], (uint32_t)((ntiles - 1) >> 1) & 1u, a, abort);
    tc_fence_after();
    const int64_t pidx = ((int64_t)list * a.splits + blockIdx.x) * a.H + head;
    // One split per query: the merge with the sink happens here (the same
    // arithmetic as the split-combine kernel) and O leaves normalised.
    float o_scale = 1.f;
    if (a.splits == 1) {
      float f_own = 0.f;
      if (s_lane) {
        const float sigma = a.sink ? a.sink[head] : -INFINITY;
        const float m = done ? m_ref : -INFINITY, l = done ? l_sum : 0.f;
        float M = sigma, den = sigma > -INFINITY ? 1.f : 0.f;  // the sink's e^(sigma - M)
        if (m > M) {
          den *= M > -INFINITY ? expf(M - m) : 0.f;
          M = m;
        }
        float f = 0.f;
        if (m > -INFINITY) {
          f = expf(m - M);
          den = fmaf(l, f, den);
        }
        f_own = den > 0.f ? f * (1.f / den) : 0.f;
        if (a.lse) a.lse[(int64_t)list * a.H + head] = den > 0.f ? M + logf(den) : -INFINITY;
      }
      o_scale = __shfl_sync(0xffffffffu, f_own, (lane & 15) + 16);
    }
    // O -> shared memory (the K tiles and P are dead: every P V is done),
    // padded rows so the 16-byte stores of a warp's heads hit distinct banks
    float* o_s = reinterpret_cast<float*>(sm + OFF_K);
    for (int c = 0; c < kD; c += 64) {  // two TMEM loads in flight
      uint32_t r0[32], r1[32];
      tmem_ld_32(row_addr + c, r0);
      tmem_ld_32(row_addr + c + 32, r1);
      tmem_ld_wait(r0, r1);
      if (lane < 16) {
        float* po = o_s + head * kOS + c;
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          *reinterpret_cast<float4*>(po + q) =
              done ? make_float4(__uint_as_float(r0[q]) * o_scale, __uint_as_float(r0[q + 1]) * o_scale,
                                 __uint_as_float(r0[q + 2]) * o_scale, __uint_as_float(r0[q + 3]) * o_scale)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(po + 32 + q) =
              done ? make_float4(__uint_as_float(r1[q]) * o_scale, __uint_as_float(r1[q + 1]) * o_scale,
                                 __uint_as_float(r1[q + 2]) * o_scale, __uint_as_float(r1[q + 3]) * o_scale)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    if (s_lane && a.splits > 1) {
      a.part_ml[pidx * 2] = done ? m_ref : -INFINITY;
      a.part_ml[pidx * 2 + 1] = done ? l_sum : 0.f;
    }
  }
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
        dst[i] = make_uint2((uint32_t)bf16_code(v.x) | ((uint32_t)bf16_code(v.y) << 16),
                            (uint32_t)bf16_code(v.z) | ((uint32_t)bf16_code(v.w) << 16));
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

cudaError_t launch_attn_mma(const AttnLaunch& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  attn_mma_kernel<<<dim3(a.splits, a.B * a.T), kThr, SMEM, stream>>>(a);
  return counted(cudaGetLastError());
}

}  // namespace lcsc
