// Lightning-indexer scoring on the 5th-generation tensor cores.
//
// Method: "DeepSeek V4 Architecture Explained" (researchpapers.dev), "How
// compress-then-sparsify attention works"; "Inside DeepSeek-V4"
// (llmbytes.dev), section 1 (FP4 indexer):
//   s[g] = sum_h w[h] * ReLU(q~[h] . k~[g])
//
// GEMM view: S[g][(t, h)] = K[g][:] . Q[(t, h)][:], keys on M (128 per tile),
// the NQ queries' 64 heads on N, d_I = 128 on K.
//  * FP4 keys and queries: tcgen05.mma kind::mxf4nvf4 with one UE4M3 scale
//    per 16 values on both operands (the scales go smem -> TMEM with
//    tcgen05.cp); the accumulator holds the exact dequantised dot products.
//    The query scales are tiled by 128 rows, two queries to a tile: the
//    CTA of an odd query moves its rows' scales to the tile's first half
//    before the copy to TMEM.
//  * FP8 keys and queries: tcgen05.mma kind::f8f6f4 on the codes; the
//    per-row scales are positive, so the epilogue applies them outside ReLU:
//    s = sk[g] * sum_h (w[h] sq[h]) ReLU(acc[h]).
// Warp roles (one CTA per SM).  One thread's issue of TMA and
// tcgen05 instructions (tens of cycles each) is what limits a single
// pipeline, so tiles go to LANES lanes (warps 0 .. LANES-1, one thread each):
// round-robin over the CTA's share with four queries, claimed two at a time
// from a counter per list with one (the list's CTAs share its tiles).  Lane
// r loads its tiles with TMA (hardware swizzle) into a STAGES-deep ring,
// DIST of its tiles ahead, and issues their MMAs into NACC TMEM
// accumulators.  Groups of four epilogue warps drain the accumulators
// with tcgen05.ld, apply ReLU and the head weights, write one fp32 score per
// (query, key) and count it in the list's shared-memory histogram of the
// top-k's first digit.  One query (384 threads): two groups take alternate
// tiles.  Four queries (576 threads): four groups drain every tile, one query
// each, reading TMEM in the accumulator-fragment layout so that each
// thread's head weights stay in registers; the ReLU'd products of a key row
// are summed within a quad.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "launches.h"
#include "sm100.cuh"
#include "topk.cuh"

namespace lcsc {
namespace {

using namespace sm100;

struct MmaArgs {
  const void* key_scale;   // FP8: float [B][cap]; FP4: tiled UE4M3 block scales
  int64_t key_cap;         // rows per sequence (multiple of 128)
  const uint8_t* q_scale;  // FP8: float [B][T*64]; FP4: tiled block scales (capacity T*64)
  const float* w_idx;      // [B*T][64]
  const int32_t* ctx_len;
  int B, T, m;
  int64_t n_max;
  int64_t stride;          // score row stride
  float* scores;           // [B*T][stride]
  int chunks;              // CTAs per (sequence, query group)
  uint32_t* hist;          // top-k digit-1 histograms [B*T][2][4096] (zeroed)
  uint32_t* counters;      // top-k counters [B*T][8] (zeroed)
  int64_t k;               // top-k
  bool bins_in_collect;    // several CTAs per list: the collect pass sets the threshold bins
  int64_t shard_row0, shard_rows;  // keys of an entry shard: entries [row0, row0 + rows) in rows 0 ..
  int32_t* status;
  uint64_t wait_ns;        // limit of the bounded waits
  bool stall;              // a test of the failure path (lcsc_set_wait_test)
};

// A context length the call can serve (an unsharded call must have been sized
// for every entry the sequence has).
__device__ __forceinline__ bool length_ok(const MmaArgs& a, int64_t L) {
  return L >= a.T && (a.shard_rows > 0 || L / a.m <= a.n_max);
}

// Key rows the query at position p scores: its N(p) = floor((p + 1) / m)
// visible entries, or for a shard those of them it holds (at most n_max).
__device__ __forceinline__ int64_t rows_seen(const MmaArgs& a, int64_t p) {
  const int64_t n = (p + 1) / a.m;
  if (a.shard_rows <= 0) return n;
  int64_t c = n - a.shard_row0;
  c = c < a.shard_rows ? c : a.shard_rows;
  c = c < a.n_max ? c : a.n_max;
  return c > 0 ? c : 0;
}

template <int FMT, int NQ>
struct Cfg {
  static constexpr int ROW = FMT == LCSC_FMT_FP4 ? 64 : 128;   // bytes per 128-value row
  static constexpr int TILE = 128;                               // keys per tile (MMA M)
  static constexpr int N = 64 * NQ;                              // MMA N
  static constexpr int KSTEPS = 4 - (FMT == LCSC_FMT_FP4 ? 2 : 0);  // 32 bytes of K per MMA
  // Ring depth: enough bytes in flight to cover DRAM latency, and more than
  // half the shared memory so that a second CTA never shares the SM's TMEM.
  static constexpr int STAGES = FMT == LCSC_FMT_FP4 ? (NQ == 1 ? 20 : 16) : (NQ == 1 ? 8 : 6);
  // Accumulators in TMEM: the MMA runs up to NACC tiles ahead of the epilogue.
  static constexpr int NACC = NQ == 1 ? 4 : 2;
  // TMA + MMA lanes (warps 0 .. LANES-1) and how many of its own tiles each
  // loads ahead; LANES * DIST < STAGES keeps every wait on an earlier tile.
  static constexpr int LANES = FMT == LCSC_FMT_FP4 && NQ == 1 ? 4 : 2;
  static constexpr int DIST = STAGES / LANES - 1;
  // Lane r's tiles i = r, r + LANES, ... use accumulators i % NACC: each
  // accumulator belongs to one lane, whose waits on it then never fall two
  // phases behind.
  static_assert(NACC % LANES == 0, "one lane per accumulator");
  // Epilogue: GROUPS groups of four warps from warp EPI0 on (warp w reads
  // TMEM sub-partition w % 4).  Several queries: group g drains query g of
  // every tile.
  static constexpr int GROUPS = NQ == 1 ? 2 : NQ;
  static constexpr int EPI0 = NQ == 1 ? 4 : LANES;
  static constexpr int THREADS = (EPI0 + 4 * GROUPS) * 32;
  static_assert(NQ == 1 || GROUPS == NQ, "one query per epilogue group");
  static_assert(DIST >= 1 && LANES * DIST < STAGES, "lane prefetch distance");
  static constexpr int A_BYTES = TILE * ROW;
  static constexpr int SFA_BYTES = FMT == LCSC_FMT_FP4 ? 1024 : 0;
  static constexpr int Q_BYTES = N * ROW;
  static constexpr int SFB_BYTES = FMT == LCSC_FMT_FP4 ? ((N + 127) / 128) * 1024 : 0;
  static constexpr Swizzle SW = FMT == LCSC_FMT_FP4 ? kSw64 : kSw128;
  static constexpr int SBO = 8 * ROW;  // bytes between 8-row core-matrix groups
  // TMEM: accumulators [0, NACC*N); FP4 also SFA (one 8-column buffer per
  // accumulator) and SFB.
  static constexpr int SFA_COL = NACC * N;
  static constexpr int SFB_COL = NACC * N + 8 * NACC;
  static constexpr int COLS_USED = NACC * N + (FMT == LCSC_FMT_FP4 ? 8 * NACC + 8 * ((N + 127) / 128) : 0);
  static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                   : COLS_USED <= 256 ? 256 : 512;
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_Q = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SFA = OFF_Q + Q_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int OFF_BAR = OFF_SFB + SFB_BYTES;
  // One query per CTA (decode, draft tokens): the lanes claim their tiles
  // at run time, BL at a time, from a counter per list, so the CTAs of a
  // list on faster SMs take more (static equal shares ended up to 40%
  // apart).  A lane
  // publishes each claim to the epilogue through a ring of RING mbarriers.
  static constexpr bool DYN = NQ == 1;
  static constexpr int BL = 2;
  static constexpr int RING = 8;
  static_assert(!DYN || RING * BL >= BL + STAGES / LANES + 2, "a claim slot is reused only after its tiles are drained");
  static constexpr int NBARS = 2 * STAGES + 2 * NACC + 2 + (DYN ? LANES * RING : 0);
  static constexpr int OFF_W = OFF_BAR + NBARS * 8;
  static constexpr int OFF_HIST = OFF_W + N * 4;  // NQ x 4096 digit-1 counts of the scores written
  static constexpr int OFF_CLM = OFF_HIST + NQ * kTopkBins * 4;  // int32 [LANES][RING] claimed batches
  static constexpr int OFF_TMEM = OFF_CLM + LANES * RING * 4;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + slack to align the base
  static_assert(COLS_USED <= 512 && SFA_COL <= COLS_USED, "TMEM budget");
  static_assert(A_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(OFF_W % 16 == 0, "head weights are read as float4");
};

// Two fp32 lanes in one 64-bit register, and the packed fused multiply-add
// of sm_100 (each lane an IEEE fma, as fmaf).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int FMT, int NQ>
__global__ void __launch_bounds__(Cfg<FMT, NQ>::THREADS, 1)
    index_mma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                     const MmaArgs a) {
  grid_dep_wait();
  using C = Cfg<FMT, NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;  // [NACC] accumulator ready
  uint64_t* acce = accf + C::NACC;     // [NACC] accumulator drained
  uint64_t* qbar = acce + C::NACC;
  uint64_t* sfb_bar = qbar + 1;        // query scales in TMEM (FP4)
  uint64_t* clm_bar = sfb_bar + 1;     // [LANES][RING] claim published (DYN)
  int32_t* clm_s = reinterpret_cast<int32_t*>(sm + C::OFF_CLM);
  float* w_s = reinterpret_cast<float*>(sm + C::OFF_W);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_TMEM);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int groups = (a.T + NQ - 1) / NQ;  // the last may hold fewer than NQ queries
  const int b = blockIdx.y / groups;
  const int t0 = (blockIdx.y % groups) * NQ;
  const int nq_here = a.T - t0 < NQ ? a.T - t0 : NQ;  // queries this group holds
  const int64_t L = a.ctx_len[b];
  const bool ok = length_ok(a, L);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(sm + C::OFF_HIST);
  const int64_t list0 = (int64_t)b * a.T + t0;
  int64_t nvis[NQ];
#pragma unroll
  for (int l = 0; l < NQ; ++l) nvis[l] = ok && l < nq_here ? rows_seen(a, L - a.T + t0 + l) : 0;
  const int64_t n_last = ok ? rows_seen(a, L - a.T + t0 + nq_here - 1) : 0;  // rows the group's last query sees
  const int64_t tiles = (n_last + C::TILE - 1) / C::TILE;
  const int64_t per = (tiles + a.chunks - 1) / a.chunks;
  const int64_t tile_lo = C::DYN ? 0 : (int64_t)blockIdx.x * per;
  const int64_t tile_hi = C::DYN ? tiles : (tile_lo + per < tiles ? tile_lo + per : tiles);
  uint32_t* tile_ctr = a.counters + list0 * 8 + 4;  // claimed batches (DYN), zeroed with the histograms
  if (tile_hi <= tile_lo) {  // uniform over the CTA, before any barrier or TMEM use
    hist_finish(hist_s, false, nq_here, a.hist, a.counters, list0, list0, gridDim.x, nvis, a.k, !a.bins_in_collect);
    return;
  }
  for (int i = threadIdx.x; i < NQ * kTopkBins; i += blockDim.x) hist_s[i] = 0u;
  const int ntile = (int)(tile_hi - tile_lo);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < C::NACC; ++j) {
      mbar_init(&accf[j], 1);
      mbar_init(&acce[j], NQ == 1 ? 4 : 4 * C::GROUPS);  // the warps draining it
    }
    mbar_init(qbar, 1);
    mbar_init(sfb_bar, 1);
    if (C::DYN)
      for (int j = 0; j < C::LANES * C::RING; ++j) mbar_init(&clm_bar[j], 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < C::N; i += blockDim.x) {
    const int64_t list = (int64_t)b * a.T + t0 + i / 64;
    float wv = 0.f;  // a slot past the group's last query scores nothing
    if (i / 64 < nq_here) {
      wv = a.w_idx[list * 64 + (i % 64)];
      if (FMT == LCSC_FMT_FP8) wv *= reinterpret_cast<const float*>(a.q_scale)[list * 64 + (i % 64)];
    }
    w_s[i] = wv;
  }
  if (warp == 2) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < C::LANES) {
    // ------------------------------------------------------ TMA + MMA lanes
    // Lane r (warp r, one thread) takes tiles i = r, r + LANES, ...: it loads
    // tile i + LANES * DIST with TMA, then issues the MMAs of tile i.  Every
    // wait of the thread handling tile i is on an earlier tile (the TMA's
    // stage was freed by the MMAs of tile i + LANES * DIST - STAGES < i).
    const int r = warp;
    if (lane == 0) {
      const int64_t key_tiles = a.key_cap / 128;
      prefetch_tmap(&tm_k);
      if (r == 0) {
        prefetch_tmap(&tm_q);
        mbar_arrive_expect_tx(qbar, C::Q_BYTES + C::SFB_BYTES);
        tma_load_2d(sm + C::OFF_Q, &tm_q, 0, (int32_t)(((int64_t)b * a.T + t0) * 64), qbar);
        if (FMT == LCSC_FMT_FP4) {
          const int64_t q_tiles = ((int64_t)a.T * 64 + 127) / 128;
          const uint8_t* src = a.q_scale + ((int64_t)b * q_tiles + (t0 * 64) / 128) * 1024;
          bulk_load(sm + C::OFF_SFB, src, C::SFB_BYTES, qbar);
        }
      }
      bool live = true;
      int32_t cur = -1;  // the batch claimed for this lane's current BL tiles (DYN)
      // Global tile of this lane's t-th tile (local index i = r + LANES t), or
      // -1 past the end; DYN claims a batch on the first tile of each.
      auto tile_of = [&](int t) -> int64_t {
        if constexpr (C::DYN) {
          if (t % C::BL == 0) {
            const uint32_t gb = atomicAdd(tile_ctr, 1u);
            cur = (int64_t)gb * C::BL < tiles ? (int32_t)gb : -1;
            const int c = t / C::BL;
            clm_s[r * C::RING + c % C::RING] = cur;
            mbar_arrive(&clm_bar[r * C::RING + c % C::RING]);  // release: the epilogue reads the slot after it
          }
          const int64_t g = (int64_t)cur * C::BL + t % C::BL;
          return cur >= 0 && g < tiles ? g : -1;
        } else {
          const int i = r + C::LANES * t;
          return i < ntile ? tile_lo + i : -1;
        }
      };
      int my_n = 0;       // tiles of this lane whose copies were issued
      auto load = [&](int i, int64_t tile) {  // TMA of (local) tile i, global tile `tile`, into stage i % STAGES
        const int s = i % C::STAGES;
        const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, a.status, a.wait_ns)) {
          live = false;
          return;
        }
        ++my_n;
        mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::SFA_BYTES);
        tma_load_2d(sm + C::OFF_A + s * C::A_BYTES, &tm_k, 0, (int32_t)((int64_t)b * a.key_cap + tile * 128),
                    &full[s]);
        if (FMT == LCSC_FMT_FP4) {
          const uint8_t* src = reinterpret_cast<const uint8_t*>(a.key_scale) + ((int64_t)b * key_tiles + tile) * 1024;
          bulk_load(sm + C::OFF_SFA + s * 1024, src, 1024, &full[s]);
        }
      };
      bool more = true;   // whether a next one may exist
      auto load_next = [&]() {
        const int64_t tile = tile_of(my_n);
        if (tile < 0) {
          more = false;
          return;
        }
        load(r + C::LANES * my_n, tile);
      };
      for (int t = 0; t < C::DIST && more && live; ++t) load_next();
      live = live && mbar_wait(qbar, 0, a.status, a.wait_ns);
      tc_fence_after();
      const uint32_t q_addr = smem_u32(sm + C::OFF_Q);
      if (live && r == 0 && FMT == LCSC_FMT_FP4) {
        if (NQ == 1 && (t0 & 1)) {
          // an odd query's 64 rows are rows 64-127 of its 128-row scale
          // tile, whose bytes hold rows 64-95 and 96-127 at chunks 2 and 3
          // of each 16-byte lane entry: move them to chunks 0 and 1, where
          // an N = 64 MMA reads its B scales
          uint2* sfb = reinterpret_cast<uint2*>(sm + C::OFF_SFB);
          for (int e = 0; e < 64; ++e) sfb[2 * e] = sfb[2 * e + 1];
          fence_async_smem();
        }
        for (int j = 0; j < 2; ++j)
          for (int c = 0; c < (C::N + 127) / 128; ++c)
            tmem_cp_32x128b_x4(tmem + C::SFB_COL + 8 * c + 4 * j,
                               smem_desc(smem_u32(sm + C::OFF_SFB + c * 1024 + j * 512), 16, 128, kSwNone));
      }
      // the other lanes start once the query scales are in TMEM
      if (r == 0) tc_commit(sfb_bar);
      else live = live && mbar_wait(sfb_bar, 0, a.status, a.wait_ns);
      tc_fence_after();
      // A test of the failure path (lcsc_set_wait_test): the first lane
      // waits for the drain of its first accumulator, which it has not
      // filled, so the wait runs out and the lane stops.
      if (a.stall && r == 0) live = live && mbar_wait(&acce[0], 0u, a.status, a.wait_ns);
      const uint32_t idesc = FMT == LCSC_FMT_FP4 ? idesc_mxf4nvf4(128, C::N) : idesc_dense(0, 0, 128, C::N);
      int last = -1;
      int t = 0;  // this lane's first tile whose copies were not yet consumed
      for (; live && t < my_n; ++t) {
        if (more) {  // tile t + DIST
          load_next();
          if (!live) break;
        }
        const int i = r + C::LANES * t;
        const int s = i % C::STAGES;
        const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
        const int ab = i % C::NACC;
        const uint32_t au = (uint32_t)(i / C::NACC) & 1u;
        if (!mbar_wait(&full[s], ph, a.status, a.wait_ns)) break;
        if (!mbar_wait(&acce[ab], au ^ 1u, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sm + C::OFF_A + s * C::A_BYTES);
        const uint32_t d = tmem + ab * C::N;
        if constexpr (FMT == LCSC_FMT_FP4) {
          const uint32_t sfa = tmem + C::SFA_COL + 8 * ab;
          for (int j = 0; j < 2; ++j)
            tmem_cp_32x128b_x4(sfa + 4 * j, smem_desc(smem_u32(sm + C::OFF_SFA + s * 1024 + j * 512), 16, 128,
                                                      kSwNone));
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk)
            mma_mxf4nvf4(d, smem_desc(a_addr + kk * 32, 16, C::SBO, C::SW),
                         smem_desc(q_addr + kk * 32, 16, C::SBO, C::SW), idesc, sfa + 4 * kk,
                         tmem + C::SFB_COL + 4 * kk, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk)
            mma_ss<1>(d, smem_desc(a_addr + kk * 32, 16, C::SBO, C::SW), smem_desc(q_addr + kk * 32, 16, C::SBO, C::SW),
                      idesc, kk > 0);
        }
        tc_commit(&empty[s]);
        tc_commit(&accf[ab]);
        last = i;
      }
      if (last >= 0)  // the accumulator of the last tile is complete before TMEM is freed
        mbar_wait(&accf[last % C::NACC], (uint32_t)(last / C::NACC) & 1u, a.status, a.wait_ns);
      // After a wait gave up: the copies this lane issued and did not consume
      // (and the query's, on lane 0) land before the CTA's shared memory is
      // released; each wait is bounded again.  Nothing is left on the normal path.
      for (; t < my_n; ++t) {
        const int i = r + C::LANES * t;
        mbar_wait(&full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1u, a.status, kDrainLimitNs);
      }
      if (r == 0 && !live) mbar_wait(qbar, 0, a.status, kDrainLimitNs);
    }
  } else if (warp >= C::EPI0) {
    // ------------------------------------------------------ epilogue
    // Warp w reads TMEM sub-partition w % 4 (key rows 32 (w % 4) ..).  One
    // query: two groups of four warps take alternate tiles.  Several
    // queries: every group drains every tile, group g query g; a warp
    // copies its 64 columns to registers and hands the accumulator back
    // before summing, so the MMAs of the next tiles overlap the sums.
    const int grp = (warp - C::EPI0) >> 2;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const float* kscale = reinterpret_cast<const float*>(a.key_scale) + (int64_t)b * a.key_cap;
    if constexpr (NQ == 1) {
      uint64_t wr[32];  // head weight pairs (w[2j], w[2j + 1]) in registers
#pragma unroll
      for (int j = 0; j < 32; ++j) wr[j] = pack2(w_s[2 * j], w_s[2 * j + 1]);
      const int64_t n_p = ok ? rows_seen(a, L - a.T + t0) : 0;  // entries the query sees
      float* score_row = a.scores + ((int64_t)b * a.T + t0) * a.stride;
      // Local tile i = r + LANES t belongs to lane r = i % LANES; this group
      // takes the lanes r = grp, grp + 2, ... (their tiles in the order i).
      // Lane r's tiles end where its claims do (DYN) or at ntile.
      constexpr int NL = C::LANES / 2;
      int32_t cl[NL];  // lane grp + 2 jj's current claim
      bool dn[NL];     // and whether its tiles have ended
#pragma unroll
      for (int jj = 0; jj < NL; ++jj) {
        cl[jj] = -1;
        dn[jj] = false;
      }
      int n_dn = 0;
      for (int i = grp; n_dn < NL; i += 2) {
        const int r = i % C::LANES, jr = r / 2, tl = i / C::LANES;
        int64_t gtile;
        if constexpr (C::DYN) {
          bool d = false;
          int32_t c = -1;
#pragma unroll
          for (int jj = 0; jj < NL; ++jj)
            if (jj == jr) {
              d = dn[jj];
              c = cl[jj];
            }
          if (d) continue;
          if (tl % C::BL == 0) {  // the lane's next claim
            const int cb = tl / C::BL;
            if (!mbar_wait(&clm_bar[r * C::RING + cb % C::RING], (uint32_t)(cb / C::RING) & 1u, a.status,
                           a.wait_ns))
              break;
            c = clm_s[r * C::RING + cb % C::RING];
          }
          gtile = (int64_t)c * C::BL + tl % C::BL;
          if (c < 0 || gtile >= tiles) {
            d = true;
            ++n_dn;
          }
#pragma unroll
          for (int jj = 0; jj < NL; ++jj)
            if (jj == jr) {
              dn[jj] = d;
              cl[jj] = c;
            }
          if (d) continue;
        } else {
          if (i >= ntile) break;
          gtile = tile_lo + i;
        }
        const int ab = i % C::NACC;
        const int64_t g = gtile * 128 + row;
        const float sk = FMT == LCSC_FMT_FP8 ? kscale[g] : 1.f;
        if (!mbar_wait(&accf[ab], (uint32_t)(i / C::NACC) & 1u, a.status, a.wait_ns)) break;
        tc_fence_after();
        uint32_t r0[32], r1[32];
        const uint32_t taddr = tmem + ((uint32_t)(q4 * 32) << 16) + ab * C::N;
        tmem_ld_32(taddr, r0);
        tmem_ld_32(taddr + 32, r1);
        tmem_ld_wait();
        // head h of the row in lane pair (h & 7) / 2 of the packed sums
        uint64_t p2[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 16; ++j)
          p2[j & 3] = ffma2(wr[j], pack2(fmaxf(__uint_as_float(r0[2 * j]), 0.f), fmaxf(__uint_as_float(r0[2 * j + 1]), 0.f)),
                            p2[j & 3]);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          p2[j & 3] = ffma2(wr[16 + j], pack2(fmaxf(__uint_as_float(r1[2 * j]), 0.f), fmaxf(__uint_as_float(r1[2 * j + 1]), 0.f)),
                            p2[j & 3]);
        float p[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack2(p2[j]);
          p[2 * j] = f.x;
          p[2 * j + 1] = f.y;
        }
        const float acc = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        if (g < n_p) {
          const float v = acc * sk;
          score_row[g] = v;
          atomicAdd(&hist_s[float_key(v) >> 20], 1u);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[ab]);
      }
    } else {
      // TMEM is read in the mma accumulator-fragment layout (16 lanes x 64
      // columns per load): thread t holds key rows t/4 and t/4 + 8 of a
      // 16-row half and the 16 head columns 8c + 2 (t % 4) + {0, 1} of a
      // query, so its head weights stay in registers for the whole kernel.
      // The four threads of a quad share rows; a reduce-scatter over the quad
      // leaves thread t the score of row t/4 + 8 (t % 4) of the sub-partition.
      const int nq = grp;  // this group's query
      const int j4 = lane & 3;
      uint64_t wq[8];  // (w[8c + 2 (t % 4)], w[8c + 2 (t % 4) + 1]) pairs
#pragma unroll
      for (int c = 0; c < 8; ++c) wq[c] = pack2(w_s[nq * 64 + 8 * c + 2 * j4], w_s[nq * 64 + 8 * c + 2 * j4 + 1]);
      // entries the query sees (none past the group's last query)
      const int64_t n_q = ok && nq < nq_here ? rows_seen(a, L - a.T + t0 + nq) : 0;
      const int my_row = q4 * 32 + (lane >> 2) + 8 * j4;
      float* score_row = a.scores + ((int64_t)b * a.T + t0 + nq) * a.stride;
      uint32_t* hist_q = hist_s + nq * kTopkBins;
      // partial sums of rows (t/4, t/4 + 8) of a 16-row half over this
      // thread's columns (the column pair of each 8-column block in one
      // packed fma)
      auto half_sum = [&](const uint32_t (&r)[32], float& s0, float& s1) {
        uint64_t pa = 0, pb = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          pa = ffma2(wq[c], pack2(fmaxf(__uint_as_float(r[4 * c]), 0.f), fmaxf(__uint_as_float(r[4 * c + 1]), 0.f)), pa);
          pb = ffma2(wq[c], pack2(fmaxf(__uint_as_float(r[4 * c + 2]), 0.f), fmaxf(__uint_as_float(r[4 * c + 3]), 0.f)), pb);
        }
        const float2 a2 = unpack2(pa), b2 = unpack2(pb);
        s0 = a2.x + a2.y;
        s1 = b2.x + b2.y;
      };
      // v[j]: this thread's partial of row t/4 + 8 j; returns the quad's sum
      // of row t/4 + 8 (t % 4)
      auto quad_sum = [&](float v0, float v1, float v2, float v3) -> float {
        const bool hi = j4 & 2, odd = j4 & 1;
        float k0 = hi ? v2 : v0, k1 = hi ? v3 : v1;
        const float s0 = hi ? v0 : v2, s1 = hi ? v1 : v3;
        k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        float k = odd ? k1 : k0;
        const float s = odd ? k0 : k1;
        k += __shfl_xor_sync(0xffffffffu, s, 1);
        return k;
      };
      for (int i = 0; i < ntile; ++i) {
        const int ab = i % C::NACC;
        const int64_t g = (tile_lo + i) * 128 + my_row;
        const float sk = FMT == LCSC_FMT_FP8 ? kscale[g] : 1.f;
        if (!mbar_wait(&accf[ab], (uint32_t)(i / C::NACC) & 1u, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t base = tmem + ((uint32_t)(q4 * 32) << 16) + ab * C::N + nq * 64;
        // the query's 64 columns of this sub-partition's rows go to
        // registers and the accumulator is handed back before the sums, so
        // the next tile's MMAs overlap them
        uint32_t ra[32], rb[32];
        tmem_ld_16x256b_x8(base, ra);
        tmem_ld_16x256b_x8(base + (16u << 16), rb);  // rows 16..31 of the sub-partition
        tmem_ld_wait(ra, rb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[ab]);
        float v0, v1, v2, v3;
        half_sum(ra, v0, v1);
        half_sum(rb, v2, v3);
        const float acc = quad_sum(v0, v1, v2, v3);
        if (g < n_q) {
          const float v = acc * sk;
          score_row[g] = v;
          atomicAdd(&hist_q[float_key(v) >> 20], 1u);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  hist_finish(hist_s, true, nq_here, a.hist, a.counters, list0, list0, gridDim.x, nvis, a.k, !a.bins_in_collect);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major byte matrix [rows][row_bytes]; box = [box_rows][row_bytes].
bool map_rows(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows,
              CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Queries per CTA (the MMA's N = 64 per query): four FP8 queries when T is
// a multiple of four (chunked prefill), two FP4 queries whenever T > 1 (the
// two share one 128-row tile of block scales; an odd T leaves the last group
// one query), else one.
int queries_per_cta(const IndexLaunch& a) {
  if (a.keys.f.fmt == LCSC_FMT_FP8) return a.T % 4 == 0 ? 4 : 1;
  return a.T > 1 ? 2 : 1;
}

// CTAs per query group: as many as fit beside the other groups' on the SMs
// (one CTA per SM), at least one.  One query per CTA claims its tiles at run
// time, so it takes two as soon as the groups leave SMs idle: where both
// fit they share the list; a CTA that waits for an SM joins its list late
// and takes what is left.
int chunks_per_group(const IndexLaunch& a) {
  const int q = queries_per_cta(a);
  const int64_t ctas = (int64_t)a.B * ((a.T + q - 1) / q);
  if (ctas >= sm_count()) return 1;
  const int fit = (int)(sm_count() / ctas);
  return queries_per_cta(a) == 1 && fit < 2 ? 2 : fit;
}

template <int FMT, int NQ>
cudaError_t launch_mma(const IndexLaunch& a, cudaStream_t stream) {
  using C = Cfg<FMT, NQ>;
  CUtensorMap tk, tq;
  const CUtensorMapSwizzle sw = FMT == LCSC_FMT_FP4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!map_rows(&tk, a.keys.data, C::ROW, (uint64_t)a.B * a.keys.capacity, 128, sw)) return cudaErrorInvalidValue;
  if (!map_rows(&tq, a.q_store.data, C::ROW, (uint64_t)a.B * a.T * 64, C::N, sw)) return cudaErrorInvalidValue;
  MmaArgs m;
  m.key_scale = a.keys.scale;
  m.key_cap = a.keys.capacity;
  m.q_scale = reinterpret_cast<const uint8_t*>(a.q_store.scale);
  m.w_idx = a.w_idx;
  m.ctx_len = a.ctx_len;
  m.B = a.B;
  m.T = a.T;
  m.m = a.m;
  m.n_max = a.n_max;
  m.stride = a.stride;
  m.scores = a.scores;
  m.hist = a.hist;
  m.counters = a.counters;
  m.k = a.k;
  m.shard_row0 = a.keys.row0;
  m.shard_rows = a.keys.rows;
  m.status = a.status;
  const WaitTest wt = wait_test();
  m.wait_ns = wt.limit_ns;
  m.stall = wt.stall;
  const int groups = (a.T + NQ - 1) / NQ;
  const int64_t ctas = (int64_t)a.B * groups;
  m.chunks = chunks_per_group(a);
  m.bins_in_collect = index_bins_in_collect(a);
  auto kern = index_mma_kernel<FMT, NQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(m.chunks, (unsigned)ctas), dim3(C::THREADS), C::SMEM, stream, tk, tq, m);
}

}  // namespace

bool index_whole_lists(const IndexLaunch& a) {
  // one CTA per query group: its histograms never leave shared memory
  return index_mma_supported(a) && chunks_per_group(a) == 1;
}

bool index_bins_in_collect(const IndexLaunch& a) {
  // the one-query configuration with several CTAs per list
  return index_mma_supported(a) && queries_per_cta(a) == 1 && chunks_per_group(a) > 1;
}

bool index_mma_supported(const IndexLaunch& a) {
  const int fmt = a.keys.f.fmt;
  if (a.d_I != 128 || a.H_I != 64) return false;
  if (a.keys.capacity % 128 != 0) return false;
  if (fmt == LCSC_FMT_FP8) return true;
  if (fmt == LCSC_FMT_FP4) return true;
  return false;
}

cudaError_t launch_index_mma(const IndexLaunch& a, cudaStream_t stream) {
  if (a.keys.f.fmt == LCSC_FMT_FP4)
    return queries_per_cta(a) == 2 ? launch_mma<LCSC_FMT_FP4, 2>(a, stream) : launch_mma<LCSC_FMT_FP4, 1>(a, stream);
  if (queries_per_cta(a) == 4) return launch_mma<LCSC_FMT_FP8, 4>(a, stream);
  return launch_mma<LCSC_FMT_FP8, 1>(a, stream);
}

}  // namespace lcsc
