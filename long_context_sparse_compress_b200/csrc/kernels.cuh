// Internal launch interface between the C-ABI layer (api.cu) and the kernel
// translation units.  Every launcher enqueues on `stream` and returns the
// launch's cudaError_t.
#pragma once

#include "common.cuh"

namespace lcsc {

// Entry range of one call, per sequence:
//   fused step (ctx_len != nullptr): L = ctx_len[b], entries
//     [floor((L - T) / m), floor(L / m)), raw rows start at L - (T + G - 1),
//     window rows L - T .. L - 1;
//   bulk call (ctx_len == nullptr): entries [tok_begin / m, tok_end / m),
//     raw rows start at tok_begin - (G - m), window rows
//     max(tok_begin, tok_end - capacity) .. tok_end - 1.
struct Span {
  const int32_t* ctx_len;
  int T;
  int64_t tok_begin, tok_end;
  int m, G;
};

struct CompressLaunch {
  const void* x;        // [B][n_x][dim] raw rows
  int x_dtype;
  int64_t n_x;
  const void* w;        // [dim][dim] x_dtype, or (gate_logits) float32 [B][n_x][dim] logit rows
  int gate_logits;      // the gate logits are given (w) instead of computed as x W
  const float* bpos;    // [G][dim]
  int dim;
  int B;
  Span span;
  int n_new_max;        // max entries per sequence in this call
  float* pooled;        // [B][n_new_max][dim] scratch
  CacheView entries;
  CacheView window;     // data == nullptr: no window write
  int n_win_max;        // max window rows per sequence
  CacheView sink_tok;   // data != nullptr: the raw row of position 0 is also stored here (row 0)
  int32_t* status;
};

cudaError_t launch_compress(const CompressLaunch& a, cudaStream_t stream);

cudaError_t launch_encode_rows(const float* rows, int B, int64_t n, int64_t row0,
                               const CacheView& out, cudaStream_t stream);

// SMs of the current device (for sizing grids that fill it); 148 when the
// host has no device (sizes then only matter for workspace queries).
inline int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

// The bounded waits of the tensor-core kernels: their limit (2 s unless a
// test of the failure path shortened it) and whether one thread of each CTA
// first waits on a barrier that cannot complete (lcsc_set_wait_test).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
struct WaitTest {
  uint64_t limit_ns;
  bool stall;
};
void set_wait_test(int64_t limit_ns, int32_t stall);
WaitTest wait_test();

struct IndexLaunch {
  const void* q_idx;    // [B][T][H_I][d_I] q_dtype
  int q_dtype;
  const float* w_idx;   // [B][T][H_I]
  CacheView keys;       // idx_format, d_I
  CacheView q_store;    // workspace rows: [B][T*H_I] in the key format
  const int32_t* ctx_len;
  int B, T, H_I, d_I, m, k;
  int64_t n_max;
  int64_t stride;       // score / candidate row stride: n_max rounded up to 4
  float* scores;        // [B*T][stride]
  // top-k workspace
  uint32_t* hist;       // [B*T][2][4096]
  uint32_t* counters;   // [B*T][8]
  uint32_t* cand;       // [B*T][cand_cap][2] candidate (index, key) pairs
  int64_t cand_cap;     // min(stride, 65536)
  uint32_t* sel_bits;   // [B*T][bit_stride] selected-entry bitmap
  int64_t bit_stride;   // words per bitmap row: ceil(stride / 32) rounded up to 4
  int32_t* out_idx;     // [B*T][k]
  float* out_score;     // [B*T][k] or nullptr
  int32_t* status;
};

// Indexer scoring (query quantisation + scores) and top-k selection; the
// stand-alone call runs both.
cudaError_t launch_index_scores(const IndexLaunch& a, cudaStream_t stream);  // quantize + score
cudaError_t launch_index_quantize(const IndexLaunch& a, cudaStream_t stream);  // also zeroes top-k state
cudaError_t launch_index_score_only(const IndexLaunch& a, cudaStream_t stream);
cudaError_t launch_topk(const IndexLaunch& a, cudaStream_t stream);
cudaError_t launch_index_topk(const IndexLaunch& a, cudaStream_t stream);
// Tensor-core scoring (FP8 / FP4 keys, d_I = 128, H_I = 64, key capacity a
// multiple of 128); index_mma_supported() tells whether it applies.
bool index_mma_supported(const IndexLaunch& a);
cudaError_t launch_index_mma(const IndexLaunch& a, cudaStream_t stream);
// True when the tensor-core scoring runs several CTAs per list with one query
// each: its CTAs then only add up the digit-1 histograms, and the collect
// pass of the top-k sets each list's threshold bin while its slice loads.
bool index_bins_in_collect(const IndexLaunch& a);
// True when the tensor-core scoring runs one CTA per query group (each CTA
// builds its lists' histograms whole, in shared memory).
bool index_whole_lists(const IndexLaunch& a);

struct AttnLaunch {
  const void* q;        // [B][T][H][D]
  int q_dtype;
  CacheView kv, v, win_kv, win_v;  // v / win_v data == nullptr: V = K
  const int32_t* idx;   // [B][T][k] or nullptr (dense)
  const float* sink;    // [H] or nullptr
  int sink_token;       // the stored row of position 0 (tok_kv / tok_v, row 0) joins every row set
  CacheView tok_kv, tok_v;
  const int32_t* ctx_len;
  int B, T, H, D, Dv, m, w, k;
  int64_t n_max;
  float sm_scale;
  int out_rope_dim;     // > 0: the output's last dims rotated back by the query position
  float out_rope_base;
  int splits;           // row splits per query
  int rows_per_split;
  float* part_o;        // [B*T][splits][H][Dv]
  float* part_ml;       // [B*T][splits][H][2]
  uint8_t* q_img;       // [B*T][kAttnQImageBytes]: the tensor-core path's query images
  WaitTest waits;       // set by the tensor-core launcher
  void* out;            // [B][T][H][Dv] q_dtype
  float* lse;           // [B][T][H] or nullptr
  int32_t* status;
};

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream);

// Tensor-core attention (64 heads, 512-d FP8 + BF16 rows, V = K).  Its
// query images (launch_attn_qimage, or launch_attn_prepare, which launches
// it only for this path) must be built before the attention runs.
constexpr size_t kAttnQImageBytes = 64 * 1024 + 64 * 4;
bool attn_mma_supported(const AttnLaunch& a);
cudaError_t launch_attn_qimage(const AttnLaunch& a, cudaStream_t stream);
cudaError_t launch_attn_mma(const AttnLaunch& a, cudaStream_t stream);
cudaError_t launch_attn_prepare(const AttnLaunch& a, cudaStream_t stream);

// Merges of entry shards' results (shard.cu).
struct TopkMergeLaunch {
  int n_parts;
  int64_t lists, k;            // lists = B * T
  const int32_t* part_idx;     // [n_parts][lists][k] global entries, -1 pads
  const float* part_score;     // [n_parts][lists][k]
  int32_t* out_idx;            // [lists][k]
  float* out_score;            // [lists][k] or nullptr
};
cudaError_t launch_topk_merge(const TopkMergeLaunch& a, cudaStream_t stream);

struct AttnMergeLaunch {
  int n_parts;
  int64_t lists;               // B * T
  int T, H, Dv, dtype;
  const void* part_out;        // [n_parts][lists][H][Dv] dtype
  const float* part_lse;       // [n_parts][lists][H]
  const float* sink;           // [H] or nullptr
  const int32_t* ctx_len;      // [B]
  int out_rope_dim;
  float out_rope_base;
  void* out;                   // [lists][H][Dv] dtype
  float* lse;                  // [lists][H] or nullptr
};
cudaError_t launch_attn_merge(const AttnMergeLaunch& a, cudaStream_t stream);

// Attention split geometry: the rows of each query are cut into `splits`
// ranges of `rows_per_split` (a multiple of `granule`); n_ctas_per_split *
// splits CTAs run, target_ctas of them at a time, and the split count is
// the one that finishes them soonest.
void attention_splits(int64_t max_rows, int64_t n_ctas_per_split, int granule, int target_ctas, int* splits,
                      int* rows_per_split);

}  // namespace lcsc
