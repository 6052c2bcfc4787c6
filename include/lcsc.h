/*
 * lcsc.h -- C ABI of the B200 (sm_100a) compressed sparse attention library.
 *
 * One attention layer of DeepSeek-V4's hybrid compressed attention:
 *   CSA: groups of m = 4 tokens are pooled into compressed entries, a
 *        low-precision lightning indexer scores every entry, and exact
 *        attention runs over the top-k entries, a sliding window of raw
 *        tokens and a per-head attention sink.
 *   HCA: groups of m = 128 tokens are pooled and attended densely, with
 *        the same window and sink.
 * Sources: "DeepSeek V4 Architecture Explained" (researchpapers.dev), section
 * "How compress-then-sparsify attention works" and its Key numbers table;
 * "Inside DeepSeek-V4" (llmbytes.dev), sections 1 and 2; "How DeepSeek V4
 * Handles 1M Token Context" (docs.bswen.com), Components 2 and 3.
 *
 * Conventions for every call
 *  - Pointers marked (dev) are device pointers owned by the caller; the
 *    library never allocates device memory.  Pointers marked (host) are
 *    read before the call returns.
 *  - State the library keeps for the life of the process: a count of the
 *    kernels it has enqueued (lcsc_kernel_launches) and, per device, two
 *    streams and three events of its own, created by the first fused step
 *    on that device (lcsc_csa_decode runs the KV latent's pooling, the
 *    attention's query images and the query quantisation on them;
 *    lcsc_hca_decode the query images; each joined back to the caller's
 *    stream before the attention or the scoring).  Fused steps on one
 *    device share them, so steps issued on independent caller streams are
 *    ordered against each other's side work; issue independent layers'
 *    steps on one stream, or accept that ordering.  Make the first fused
 *    call on a device before any stream capture.  The no-allocation call
 *    below also keeps a fixed array per device.
 *  - Every call enqueues its kernels on `stream` (a cudaStream_t) and
 *    returns without synchronising.  Kernels are launched with programmatic
 *    stream serialisation and each waits (griddepcontrol.wait) for the
 *    stream's previous grid before touching memory, so results follow
 *    stream order as with plain launches; the environment variable
 *    LCSC_PDL=0, read once per process, launches without the attribute.
 *  - On a non-zero return nothing has been enqueued.
 *  - Data-dependent anomalies found on the device (an index in `idx` that
 *    is out of range, a window ring too small for the query positions) never
 *    trap: the offending row is skipped and a bit is OR-ed into `*status`
 *    (dev, nullable, int32): LCSC_DEV_BAD_INDEX, LCSC_DEV_BAD_LENGTH.
 *  - Batched arrays are dense: sequence b of a [B][n][...] array starts at
 *    b * n * (row bytes).  Every pointer must be 16-byte aligned.
 *  - Sequence lengths: `ctx_len` (dev, int32 [B]) gives, per sequence, the
 *    length L after the T new tokens of the step; the step's queries sit at
 *    positions p = L - T + i, i < T.
 *  - Entry g of a tensor pools the tokens [g*m + m - G, g*m + m) (positions
 *    below 0 are left out); a query at position p sees the entries
 *    g < N(p) = floor((p + 1) / m) and the raw window rows of positions
 *    max(0, p - w + 1) .. p.
 */
#ifndef LCSC_H_
#define LCSC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LCSC_ABI_VERSION 3

/* Return codes. */
#define LCSC_OK 0
#define LCSC_ERR_INVALID_ARG 1     /* null / misaligned pointer, bad size or parameter */
#define LCSC_ERR_UNSUPPORTED 2     /* a format / dimension combination that is not built */
#define LCSC_ERR_CUDA 3            /* a launch failed; see lcsc_last_cuda_error() */
#define LCSC_ERR_WORKSPACE 4       /* workspace smaller than the *_workspace_size() answer */

/* Bits OR-ed into *status on the device. */
#define LCSC_DEV_BAD_INDEX 1       /* an index outside [0, N(p)) was skipped */
#define LCSC_DEV_BAD_LENGTH 2      /* a ctx_len smaller than T, or past the sizes of the call */
#define LCSC_DEV_TIMEOUT 4         /* a kernel gave up a bounded wait (the call's results are not valid) */
#define LCSC_DEV_RANGE 8           /* reserved: no call of this version raises it */

/* What the sink of a layer is (lcsc_params.sink_mode); "DeepSeek V4
 * Architecture Explained", "How compress-then-sparsify attention works": a
 * sink term lets each head leave part of its weight on no row.
 *  LCSC_SINK_LOGIT: a learned logit sigma[h] per head whose value vector is
 *                   zero: exp(sigma[h]) joins the softmax denominator only
 *                   (the `sink` argument; NULL: no sink).
 *  LCSC_SINK_TOKEN: the raw row of position 0 is one more member of every
 *                   query's row set, once (nothing is added while the window
 *                   already holds position 0).  The row lives in a one-row
 *                   cache per sequence (`sink_kv`, and `sink_v` when V is
 *                   separate) that a fused step fills when position 0 is
 *                   one of its new tokens; `sink` must be NULL. */
#define LCSC_SINK_LOGIT 0
#define LCSC_SINK_TOKEN 1

/* Where the compression gate's logits come from (lcsc_params.gate_src).
 *  LCSC_GATE_PROJ:   z_j = x_j W + Bpos[place of j] with W [dim][dim].
 *  LCSC_GATE_LOGITS: z_j = u_j + Bpos[place of j], u_j a float32 logit row
 *                    per token given by the caller in place of x_j W (a
 *                    token of two overlapping groups gets the bias of its
 *                    place in each). */
#define LCSC_GATE_PROJ 0
#define LCSC_GATE_LOGITS 1

/* Row storage formats ("DeepSeek V4 Architecture Explained", Key numbers,
 * row "KV storage precision"; "Inside DeepSeek-V4", section 1, FP4 indexer).
 *  LCSC_FMT_F32: dim float32 values.                         row = 4*dim bytes
 *  LCSC_FMT_KV:  (dim - rope_dim) E4M3 values then rope_dim BF16 values;
 *                E4M3 part scaled by one float32 per row:
 *                s = amax / 448 (1 if amax = 0), code = E4M3_rne_sat(c / s).
 *                                                            row = dim + rope_dim bytes
 *  LCSC_FMT_FP8: dim E4M3 values, same per-row float32 scale rule.  row = dim bytes
 *  LCSC_FMT_FP4: dim E2M1 values, element 2i in the low nibble of byte i;
 *                one E4M3 scale byte per 16 values: b = amax / 6,
 *                scale = E4M3_rne_sat(b), code = E2M1_rne_sat(c / scale)
 *                (all-zero codes when the scale byte decodes to 0).
 *                                                            row = dim / 2 bytes
 * All encode decisions are taken in float32 with IEEE division. */
#define LCSC_FMT_F32 0
#define LCSC_FMT_KV 1
#define LCSC_FMT_FP8 2
#define LCSC_FMT_FP4 3

/* Element types of raw rows, gate weights, queries and outputs. */
#define LCSC_DT_F32 0
#define LCSC_DT_BF16 1

/* Which compressed tensor a compress / encode call writes. */
#define LCSC_TENSOR_KV 0    /* the shared KV latent (or K when V is separate) */
#define LCSC_TENSOR_V 1     /* a separate V */
#define LCSC_TENSOR_IDX 2   /* the indexer keys (CSA only) */

/* Layer parameters.  The pages fix m, k and w ("Inside DeepSeek-V4",
 * sections 1-2); the rest are this library's readings, kept as parameters. */
typedef struct lcsc_params {
  int32_t m;           /* compression ratio = entry stride: 4 (CSA), 128 (HCA) */
  int32_t group_len;   /* G, tokens pooled per entry: m, or 2m (overlapping groups) */
  int32_t window;      /* w, sliding-window length (raw tokens, query included) */
  int32_t top_k;       /* k, entries kept per query (CSA; <= 2048) */
  float sm_scale;      /* softmax scale of q.K (e.g. 1/sqrt(D)) */
  int32_t n_heads;     /* H query heads, all attending to one shared KV */
  int32_t head_dim;    /* D, query and key row length */
  int32_t rope_dim;    /* trailing dims stored BF16 in LCSC_FMT_KV */
  int32_t v_dim;       /* Dv: = D when V is the shared latent */
  int32_t idx_heads;   /* H_I indexer heads */
  int32_t idx_dim;     /* d_I indexer query / key length */
  int32_t kv_format;   /* LCSC_FMT_F32 or LCSC_FMT_KV (entries, V and the window ring) */
  int32_t idx_format;  /* LCSC_FMT_F32, LCSC_FMT_FP8 or LCSC_FMT_FP4 */
  int32_t x_dtype;     /* LCSC_DT_*: raw token rows and gate weights W */
  int32_t q_dtype;     /* LCSC_DT_*: queries, indexer queries and the output */
  /* Inverse RoPE of the output ("How DeepSeek V4 Handles 1M Token Context",
   * Component 1: K and V are one shared vector and inverse RoPE restores the
   * positional information).  out_rope_base > 0: the last out_rope_dim dims
   * of every output row, in pairs (2j, 2j+1), are turned by the angle
   * -p * out_rope_base^(-2j / out_rope_dim), p the query's position, so the
   * output carries the key positions relative to the query.  0: off.
   * out_rope_dim: a multiple of 4, <= v_dim, when on. */
  int32_t out_rope_dim;
  float out_rope_base;
  int32_t sink_mode;   /* LCSC_SINK_LOGIT or LCSC_SINK_TOKEN */
  int32_t gate_src;    /* LCSC_GATE_PROJ or LCSC_GATE_LOGITS */
} lcsc_params;

/* Stored rows of one tensor for B sequences (dev pointers).
 *   data:  [B][capacity][row bytes of the format]
 *   scale: [B][capacity] float32 (KV, FP8); NULL for F32; for FP4 uint8
 *          block scales tiled by 128 rows, the order the tensor cores read
 *          them: [B][ceil(capacity / 128)][dim / 64][32][4][4], the byte of
 *          row r, 16-value block k at
 *          [b][r / 128][k / 4][r % 32][(r % 128) / 32][k % 4].
 *   Indexer keys in FP8 / FP4 need a capacity that is a multiple of 128.
 * Compressed entries use row g for entry g.  A window ring uses row
 * (position mod capacity).
 * Entry shards (rows > 0; compressed entries only): the cache holds the
 *   entries [row0, row0 + rows) of each sequence, entry g in row g - row0
 *   (rows <= capacity), the way one GPU of several holds its range of a
 *   long sequence.  Entries outside the range belong to other shards:
 *   pooling does not write them, the indexer neither scores nor selects
 *   them (its out_idx still holds global entry numbers), the attention
 *   skips them without a status bit (an index outside [0, N(p)) still sets
 *   LCSC_DEV_BAD_INDEX).  The fused steps take unsharded caches only
 *   (rows = 0, row0 = 0: entry g in row g); lcsc_topk_merge and
 *   lcsc_attn_merge below combine the shards' results. */
typedef struct lcsc_cache {
  void* data;
  void* scale;
  int64_t capacity;
  int64_t row0;   /* first entry held (shards; else 0) */
  int64_t rows;   /* entries held from row0 (shards); 0: unsharded */
} lcsc_cache;

/* ---------------------------------------------------------------- misc */

int32_t lcsc_abi_version(void);
/* cudaError_t of the last LCSC_ERR_CUDA returned on this host thread. */
int32_t lcsc_last_cuda_error(void);
const char* lcsc_status_string(int32_t status);
/* Kernels this library has enqueued since it was loaded, over all host
 * threads and streams.  A kernel counts when its launch is enqueued, not when
 * it runs; read the count before and after a region to learn how many
 * launches that region issued. */
uint64_t lcsc_kernel_launches(void);
/* For tests of the failure path of the bounded waits (process-wide; affects
 * calls enqueued after it returns).  limit_ns > 0: the waits of the
 * tensor-core attention and scoring kernels give up after limit_ns instead
 * of 2 s.  stall != 0: in each CTA of those kernels one thread first waits on
 * a barrier that cannot complete at that point (the attention's Q K^T issuer
 * on the barrier it commits to at its end; the scoring's first lane on the
 * drain of its first accumulator, which it has not filled), so the wait runs
 * out, LCSC_DEV_TIMEOUT is set, and every role of the CTA stops, waits for
 * its copies and MMAs in flight and frees its tensor memory.  (0, 0)
 * restores the normal behaviour.  Returns LCSC_OK, or LCSC_ERR_INVALID_ARG for a
 * negative limit. */
int32_t lcsc_set_wait_test(int64_t limit_ns, int32_t stall);
/* Bytes of one stored row for a format and dimension (0 if invalid). */
int64_t lcsc_row_bytes(int32_t format, int32_t dim, int32_t rope_dim);

/* ------------------------------------------------------- compression (a1, a2)
 * lcsc_csa_compress / lcsc_hca_compress: softmax-gated pooling ("DeepSeek V4
 * Architecture Explained", "How compress-then-sparsify attention works":
 * trainable compression weights, a softmax over the group, learnable
 * positional biases).  For each entry g in [tok_begin/m, tok_end/m) and
 * each channel c:
 *     z_j[c] = sum_d x_j[d] W[d][c] + Bpos[j - (g*m + m - G)][c]
 *     e_g[c] = sum_j softmax_j(z[c])_j * x_j[c]
 * over the tokens j of the group; e_g is stored in the tensor's format.
 *   tensor:   LCSC_TENSOR_KV, _V or _IDX (IDX only for CSA); fixes the row
 *             length (D, Dv, d_I) and the format (kv_format / idx_format).
 *   x (dev):  [B][n_x][dim] x_dtype raw rows of positions
 *             tok_begin - (G - m) .. tok_end - 1, n_x = tok_end - tok_begin + G - m
 *             (rows at negative positions are never read).
 *   tok_begin % m == 0; every group that ends before tok_end is written.
 *   w_gate (dev): LCSC_GATE_PROJ: W [dim][dim] x_dtype; LCSC_GATE_LOGITS:
 *             the logit rows u [B][n_x][dim] float32 of the same positions
 *             as x.  b_pos (dev): [G][dim] float32.
 *   entries: written rows; window (nullable): the window ring, which also
 *   receives the raw rows of positions max(tok_begin, tok_end - capacity) ..
 *   tok_end - 1 (KV / V only).
 *   workspace: lcsc_compress_workspace_size() bytes (dev). */
int32_t lcsc_compress_workspace_size(const lcsc_params* p, int64_t B, int64_t n_tokens,
                                     size_t* bytes);
int32_t lcsc_csa_compress(const lcsc_params* p, int32_t tensor, const void* x, int64_t B,
                          int64_t tok_begin, int64_t tok_end, const void* w_gate,
                          const float* b_pos, const lcsc_cache* entries, const lcsc_cache* window,
                          void* workspace, size_t workspace_bytes, int32_t* status,
                          void* stream);
int32_t lcsc_hca_compress(const lcsc_params* p, int32_t tensor, const void* x, int64_t B,
                          int64_t tok_begin, int64_t tok_end, const void* w_gate,
                          const float* b_pos, const lcsc_cache* entries, const lcsc_cache* window,
                          void* workspace, size_t workspace_bytes, int32_t* status,
                          void* stream);

/* Store already-pooled float32 rows in a tensor's format, no pooling:
 * rows [B][n][dim] (dev, float32) go to rows row0 .. row0 + n - 1 of `out`.
 * For building caches from precomputed entry values and for tests. */
int32_t lcsc_encode_rows(const lcsc_params* p, int32_t tensor, const float* rows, int64_t B,
                         int64_t n, int64_t row0, const lcsc_cache* out, void* stream);

/* ---------------------------------------------------- indexer + top-k (a3, a4)
 * Lightning indexer ("DeepSeek V4 Architecture Explained", same section;
 * "How DeepSeek V4 Handles 1M Token Context", Component 3): every indexer
 * query row (t, h) is stored in the key format (FP8: per-row scale; FP4:
 * per-16 block scales; F32: as is), then for every visible entry g < N(p)
 *     s[g] = sum_h w[h] * ReLU(q~[h] . k~[g])
 * and the min(k, N(p)) entries with the largest s are kept.
 *   q_idx (dev): [B][T][H_I][d_I] q_dtype;  w_idx (dev): [B][T][H_I] float32.
 *   idx_keys: the stored indexer keys (idx_format, d_I).
 *   out_idx (dev): [B][T][k] int32; the set is unordered; rows beyond
 *   min(k, N(p)) are -1.  out_score (dev, nullable): [B][T][k] float32, the
 *   score of each kept index (-inf in padded rows). */
int32_t lcsc_index_topk_workspace_size(const lcsc_params* p, int64_t B, int64_t T, int64_t n_max,
                                       size_t* bytes);
int32_t lcsc_csa_index_topk(const lcsc_params* p, const void* q_idx, const float* w_idx,
                            const lcsc_cache* idx_keys, const int32_t* ctx_len, int64_t B,
                            int64_t T, int64_t n_max, int32_t* out_idx, float* out_score,
                            void* workspace, size_t workspace_bytes, int32_t* status,
                            void* stream);

/* The same indexer + top-k call for callers that cannot allocate device
 * memory: hosts that hand every byte of device memory to their own pool up
 * front, or callers reaching this library through a foreign-function
 * interface with no device allocator.  (No counterpart in the paper: it is
 * an interface of this library.)
 *  - Arguments and results are those of lcsc_csa_index_topk, minus the
 *    workspace; no call allocates or frees device memory.
 *  - Scratch: one static device array of LCSC_NOALLOC_SCRATCH_BYTES (40 MiB)
 *    inside the library, which every device that loads the library holds
 *    until the process exits.  A request whose scratch
 *    (lcsc_index_topk_workspace_size) exceeds it returns LCSC_ERR_WORKSPACE
 *    and enqueues nothing (B = 16, T = 1, n_max = 262144 fits).
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture.
 *  - Every call on a device shares the array, which keeps the last call's
 *    contents (each call clears what must start at zero): calls that overlap
 *    on the GPU (other streams, other host threads) race and give wrong
 *    results; serialise them. */
#define LCSC_NOALLOC_SCRATCH_BYTES (40ll << 20)
int32_t lcsc_csa_index_topk_noalloc(const lcsc_params* p, const void* q_idx, const float* w_idx,
                                    const lcsc_cache* idx_keys, const int32_t* ctx_len, int64_t B,
                                    int64_t T, int64_t n_max, int32_t* out_idx, float* out_score,
                                    int32_t* status, void* stream);

/* --------------------------------------------------------- attention (a5-a7)
 * One joint softmax per query head over a row set S (entries plus window
 * rows, plus the position-0 row with LCSC_SINK_TOKEN), with a per-head sink
 * logit sigma[h] (LCSC_SINK_LOGIT) that only adds exp(sigma) to the
 * denominator ("DeepSeek V4 Architecture Explained", "How
 * compress-then-sparsify attention works"):
 *     l_j = sm_scale * q[h] . K_j          (sm_scale > 0)
 *     o[h] = sum_j e^{l_j - M} V_j / (e^{sigma[h] - M} + sum_j e^{l_j - M})
 * K_j, V_j are dequantised stored rows; V = K unless `v` is given.
 *   q (dev): [B][T][H][D] q_dtype.   out (dev): [B][T][H][Dv] q_dtype.
 *   lse (dev, nullable): [B][T][H] float32 = M + log(denominator).
 *   sink (dev, nullable): [H] float32 sigma; NULL means no sink (must be
 *   NULL with LCSC_SINK_TOKEN).
 *   sink_kv, sink_v (LCSC_SINK_TOKEN only, else nullable and unread): the
 *   stored row of position 0 of each sequence, capacity 1 ([B][1] rows);
 *   sink_v only when V is separate.
 *   kv, v (v nullable): stored entries; win_kv, win_v (win_v nullable): the
 *   window rings, which must hold positions max(0, p - w + 1) .. p.
 * Range of the 512-dim FP8 + BF16 path (64 heads; its products run on the
 * tensor cores with float32 sums): stored rows enter as stored (E4M3 codes
 * x E4M3, BF16 RoPE dims x BF16) and the row scale is applied in float32,
 * so any finite row is used; every query is used at any finite magnitude
 * (each head is scaled by a power of two, its 448 code dims written as the
 * sum of two E4M3 numbers, and the scale is undone on its logits).  Query
 * values below 2^-10 of their head's largest |value| keep an absolute
 * precision of 2^-17 of it.
 * lcsc_csa_sparse_attn: S = {idx[b][t][j] >= 0} U window (idx (dev):
 *   [B][T][k] int32, e.g. from lcsc_csa_index_topk).
 * lcsc_hca_dense_attn: S = {all g < N(p)} U window. */
int32_t lcsc_attn_workspace_size(const lcsc_params* p, int64_t B, int64_t T, int64_t n_max,
                                 int32_t dense, size_t* bytes);
int32_t lcsc_csa_sparse_attn(const lcsc_params* p, const void* q, const lcsc_cache* kv,
                             const lcsc_cache* v, const lcsc_cache* win_kv,
                             const lcsc_cache* win_v, const int32_t* idx, const float* sink,
                             const lcsc_cache* sink_kv, const lcsc_cache* sink_v,
                             const int32_t* ctx_len, int64_t B, int64_t T, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, int32_t* status,
                             void* stream);
int32_t lcsc_hca_dense_attn(const lcsc_params* p, const void* q, const lcsc_cache* kv,
                            const lcsc_cache* v, const lcsc_cache* win_kv, const lcsc_cache* win_v,
                            const float* sink, const lcsc_cache* sink_kv, const lcsc_cache* sink_v,
                            const int32_t* ctx_len, int64_t B, int64_t T,
                            int64_t n_max, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, int32_t* status, void* stream);

/* ------------------------------------------------------------ fused steps
 * One step of a layer over T new tokens per sequence (T = 1 decode, a few
 * draft tokens, or a chunked-prefill block), each its own query: pool every
 * group that closes inside the T new tokens (entries
 * [floor((L - T) / m), floor(L / m))), store the T new raw rows in the
 * window rings, then (CSA) score + select + attend, or (HCA) attend densely.
 * Every sequence must have L >= T; raw rows x_* (dev) are
 * [B][T + G - 1][dim] x_dtype for positions L - (T + G - 1) .. L - 1.
 * The caches must already hold every entry below floor((L - T) / m) and the
 * rings the rows of positions L - T - w + 1 .. L - T - 1; the rings need at
 * least T + w - 1 rows.  With LCSC_SINK_TOKEN, sink_kv (and sink_v) must
 * hold the row of position 0 unless L - T <= 0, in which case the step
 * stores it there.  With LCSC_GATE_LOGITS, w_kv / w_v / w_idx are the
 * float32 gate logit rows [B][T + G - 1][dim] of the same positions as the
 * raw rows. */
typedef struct lcsc_step {
  int64_t B, T;
  int64_t n_max;                /* >= floor(L / m) for every sequence */
  const int32_t* ctx_len;       /* [B] L after the step */
  const void* x_kv;             /* raw rows of the KV latent (or K) */
  const void* x_v;              /* raw rows of a separate V, or NULL */
  const void* x_idx;            /* raw rows of the indexer keys (CSA) */
  const void* w_kv;  const float* b_kv;    /* gates of each tensor: W [dim][dim] (or logits), Bpos [G][dim] */
  const void* w_v;   const float* b_v;
  const void* w_idx; const float* b_idx;
  lcsc_cache kv, v, idx_keys;   /* entries (v.data NULL when V = K) */
  lcsc_cache win_kv, win_v;     /* window rings (win_v.data NULL when V = K) */
  const void* q;                /* [B][T][H][D] */
  const void* q_idx;            /* [B][T][H_I][d_I] (CSA) */
  const float* w_heads;         /* [B][T][H_I] indexer head weights (CSA) */
  const float* sink;            /* [H] or NULL */
  void* out;                    /* [B][T][H][Dv] */
  float* lse;                   /* [B][T][H] or NULL */
  int32_t* out_idx;             /* [B][T][k] selected entries (CSA), or NULL */
  float* out_score;             /* [B][T][k] their scores (CSA), or NULL */
  /* Optional stage timing (host array of cudaEvent_t, or NULL): event i is
   * recorded on `stream` at stage boundary i while i < n_events.
   * CSA: 0 start, 1 after the indexer keys' compression, 2 once the query
   * quantisation (on a stream of the library's) is also done, 3 after
   * indexer scoring, 4 after top-k, 5 after attention (the KV latent's
   * compression and window rows run on a second stream of the library's
   * from 0 and are joined before the attention).  HCA: 0 start, 1 after
   * compression, 2 after attention. */
  void* const* events;
  int32_t n_events;
  lcsc_cache sink_kv, sink_v;   /* LCSC_SINK_TOKEN: the position-0 rows ([B][1]); else unread */
} lcsc_step;

int32_t lcsc_step_workspace_size(const lcsc_params* p, int32_t csa, int64_t B, int64_t T,
                                 int64_t n_max, size_t* bytes);
int32_t lcsc_csa_decode(const lcsc_params* p, const lcsc_step* s, void* workspace,
                        size_t workspace_bytes, int32_t* status, void* stream);
int32_t lcsc_hca_decode(const lcsc_params* p, const lcsc_step* s, void* workspace,
                        size_t workspace_bytes, int32_t* status, void* stream);

/* ------------------------------------------------------ entry-shard merges
 * One long sequence split by entry range over G GPUs ("Inside DeepSeek-V4",
 * section 1: top-1,024 over the ~262K entries of a 1M-token context): GPU r
 * holds the entries [row0_r, row0_r + rows_r) in caches with those fields
 * set (lcsc_cache), and per step
 *   1. lcsc_csa_index_topk on its keys gives its own top-k (global entry
 *      numbers, with scores);
 *   2. the G lists are gathered (a collective of the caller's) and
 *      lcsc_topk_merge gives the top-k over all entries, the same list on
 *      every GPU;
 *   3. lcsc_csa_sparse_attn with that list, no sink and no output rotation
 *      (sink NULL, out_rope_base 0) attends to the listed entries this GPU
 *      holds; one GPU also takes the window rows (window w, the others 0);
 *      each writes its normalised output and lse (an empty share: lse -inf);
 *   4. the G (out, lse) pairs are gathered and lcsc_attn_merge folds them
 *      into the output a single GPU would give, with the sink and the
 *      inverse RoPE.
 * Both merges are pure functions of their inputs (dev pointers, caller
 * owned); parts are concatenated along the first dimension.
 *
 * lcsc_topk_merge: part_idx, part_score [n_parts][B*T][k] (k = top_k; pads
 *   -1); out_idx [B*T][k] (and out_score, nullable): the min(k, candidates)
 *   largest scores, ties to the lower entry, in the order of the parts
 *   (index order for parts given in range order), padded with -1.
 *   n_parts * k <= LCSC_MERGE_MAX_CANDIDATES.
 * lcsc_attn_merge: part_out [n_parts][B*T][H][Dv] q_dtype, part_lse
 *   [n_parts][B*T][H] float32; with M = max(sigma[h], lse_r) the output is
 *   sum_r e^{lse_r - M} out_r / (e^{sigma[h] - M} + sum_r e^{lse_r - M}),
 *   rotated back by the query position when out_rope_base > 0; lse
 *   (nullable) [B*T][H].  sink NULL: no sink (NULL with LCSC_SINK_TOKEN:
 *   the position-0 row is then one of the parts' rows). */
#define LCSC_MERGE_MAX_CANDIDATES 16384
int32_t lcsc_topk_merge(const lcsc_params* p, int32_t n_parts, const int32_t* part_idx,
                        const float* part_score, int64_t B, int64_t T, int32_t* out_idx,
                        float* out_score, void* stream);
int32_t lcsc_attn_merge(const lcsc_params* p, int32_t n_parts, const void* part_out, const float* part_lse,
                        const float* sink, const int32_t* ctx_len, int64_t B, int64_t T, void* out,
                        float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LCSC_H_ */
