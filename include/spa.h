/*
 * spa.h -- C ABI of libspa: one decode step of head-partitioned sparse attention
 * on an NVIDIA B200 (sm_100a).
 *
 * The method ("Full Attention Strikes Back" (RTPurbo summary), Methodology §1-§3,
 * §5) splits the KV heads of an attention layer in two:
 *   - streaming (local) heads attend to the attention sinks plus a sliding window;
 *   - retrieval heads score every cached token in a 16-dim index space built from
 *     the keys *before* RoPE, keep the smallest set of tokens whose index
 *     probability mass reaches p (top-p, not a fixed top-k), and run exact softmax
 *     attention over that set plus the sinks and window.
 * Conventions fixed by this library where the pages are silent:
 *   - index probabilities are computed per query head (softmax of idx_scale *
 *     <P_q[h] q_pre[h], idx_j>) and averaged over the heads of each GQA group
 *     ("Autonomy of Heads" summary, Deployment strategy: group mean), giving
 *     one selected set per (sequence, KV head);
 *   - tokens are ranked by (probability desc, position asc); the kept set is the
 *     shortest prefix whose mass reaches p (token kept iff the mass ranked ahead
 *     of it is < p); p >= 1 keeps every token;
 *   - sinks are positions [0, n_sink); the window is the last `window` positions,
 *     the current token (position seq_len-1) included; both are always attended;
 *   - RoPE is rotate-half with inv_freq_i = rope_theta^(-2i/128), applied by the
 *     library to the query at position seq_len-1.  k_cache holds post-RoPE keys
 *     written by the caller; the index cache is built from pre-RoPE keys.
 *
 * Memory and ownership
 *   Every tensor pointer is a DEVICE pointer owned by the caller, except
 *   `head_mask` (HOST memory, read during the call) and the handle.  Tensors are
 *   dense, row-major, 16-byte aligned.  Storage dtype of q/k/v is the handle's
 *   kv_dtype (SPA_BF16 or SPA_F32); the index cache is always bf16; outputs are
 *   float32.  The handle owns a device workspace allocated in spa_create.
 *
 * Execution
 *   Every compute call only enqueues kernels on `stream` (no host sync, no
 *   device->host copy), so a call can be captured in a CUDA graph.  Calls on one
 *   handle share its workspace: do not run two of them concurrently on
 *   different streams.  Argument errors are reported before anything is
 *   launched.  Values that live on the device (seq_lens, start_pos) are range
 *   checked by the kernels: an out-of-range value is clamped into range, a
 *   device status bit is set, and spa_device_status() reports it.
 *
 * Errors
 *   Every call returns SPA_OK (0) or a negative spa_status; spa_last_error()
 *   returns a thread-local message for the last failing call.  No C++ exception
 *   crosses this boundary.  There is no CPU fallback: without a usable CUDA
 *   device, calls that need one return SPA_ERR_CUDA.
 */
#ifndef SPA_H_
#define SPA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPA_API __attribute__((visibility("default")))
#else
#define SPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int spa_status;
#define SPA_OK 0
#define SPA_ERR_INVALID_ARG (-1)    /* null/misaligned pointer, bad size, p out of (0,1] ... */
#define SPA_ERR_UNSUPPORTED (-2)    /* head_dim != 128, idx_dim != 16, unsupported GQA ratio or dtype */
#define SPA_ERR_WORKSPACE (-3)      /* workspace allocation failed / request exceeds the handle's capacity */
#define SPA_ERR_CUDA (-4)           /* a CUDA runtime call or kernel launch failed */
#define SPA_ERR_DEVICE_TIMEOUT (-5) /* spa_device_status: a bounded device-side wait gave up */
#define SPA_ERR_DEVICE_RANGE (-6)   /* spa_device_status: a device-resident length/position was out of range */

/* storage dtypes of q / k / v */
#define SPA_BF16 0
#define SPA_F32 1

typedef struct spa_ctx* spa_handle;
/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* spa_stream;

typedef struct {
  int max_batch;      /* largest B a call may pass (>= 1) */
  int n_q_heads;      /* Hq */
  int n_kv_heads;     /* Hkv; Hq / Hkv (the GQA group size G) must be 1, 2, 4 or 8; Hkv <= 64 */
  int head_dim;       /* must be 128 */
  int idx_dim;        /* index dimension r; must be 16 */
  int kv_dtype;       /* SPA_BF16 or SPA_F32 */
  int64_t max_ctx;    /* Lmax: cache capacity in tokens per (sequence, KV head); 1 <= Lmax <= 2^24 */
  double rope_theta;  /* RoPE base (e.g. 500000) */
  float idx_scale;    /* index softmax temperature; <= 0 selects 1/sqrt(idx_dim) = 0.25 */
  int split_rows;     /* rows of K/V per attention split; 0 selects the default (a multiple of 64) */
  const float* P_q;   /* device [Hq][16][128] float32 query projectors; copied at create */
  const float* P_k;   /* device [Hkv][16][128] float32 key projectors; copied at create */
} spa_config;

/* Validate `cfg`, allocate the device workspace on the current device and copy
 * the projectors.  Synchronous.  On failure *out is NULL. */
SPA_API spa_status spa_create(spa_handle* out, const spa_config* cfg);

/* Free the workspace (synchronises the device first).  NULL is accepted. */
SPA_API spa_status spa_destroy(spa_handle h);

/* Bytes of device workspace spa_create would allocate for `cfg`. Host only. */
SPA_API spa_status spa_workspace_size(const spa_config* cfg, size_t* bytes);

/* Thread-local text of the last error ("" if none).  Valid until the next call
 * on this thread. */
SPA_API const char* spa_last_error(void);

/*
 * Index append ("Full Attention Strikes Back", Methodology §2: a 16-dim projector
 * applied to the key features before RoPE is injected).
 *   idx_cache[b][g][start_pos[b] + t][r] = bf16_rne( sum_d P_k[g][r][d] * k_pre[b][g][t][d] )
 * for b < B, g < Hkv, t < T, r < 16; each product is rounded to float32 and added
 * to a float32 running sum in ascending d (no fused multiply-add), so the code is
 * reproducible bit for bit.
 *   k_pre     device [B][Hkv][T][128], kv_dtype: pre-RoPE keys of T new tokens
 *   start_pos device int64 [B]: cache position of token t = 0 for each sequence
 *   idx_cache device bf16 [max_batch][Hkv][Lmax][16] (32 bytes per row), written
 * Rows whose position falls outside [0, Lmax) are skipped and flagged (device status).
 * Works for a prefill chunk (T large) and for the decode token (T = 1).
 */
SPA_API spa_status spa_index_append(spa_handle h, const void* k_pre, const int64_t* start_pos,
                            int B, int T, void* idx_cache, spa_stream stream);

/*
 * Top-p token selection for the retrieval heads ("Full Attention Strikes Back",
 * Methodology §2-§3, §5 histogram thresholding).  For each b < B and each KV head
 * g with head_mask[g] != 0, with L = seq_lens[b]:
 *   pi_j = mean_{h in group g} softmax_j( idx_scale * <P_q[h] q_pre[b][h], idx_cache[b][g][j]> ), j < L
 *   T    = shortest prefix of (pi desc, position asc) whose mass reaches p (all of [0,L) if p >= 1)
 *   sel_idx[b][g][0 .. count)  = T minus sinks/window, positions ascending
 *   sel_count[b * Hkv + g]     = count
 * Streaming heads get count 0.  Entries of sel_idx at or beyond the count are
 * left unspecified.
 *   q_pre      device [B][Hq][128], kv_dtype: pre-RoPE queries of the current token
 *   idx_cache  device bf16 [max_batch][Hkv][Lmax][16]
 *   head_mask  HOST uint8 [Hkv]: 1 = retrieval head, 0 = streaming head
 *   seq_lens   device int64 [B]: context length including the current token, 1..max_seq_len
 *   max_seq_len host upper bound on seq_lens for this call (sizes the launch); 0 = Lmax
 *   p          in (0, 1]; n_sink >= 0; window >= 0; n_sink + window >= 1
 *   sel_idx    device int32 [B][Hkv][Lmax]; sel_count device int32 [B * Hkv]
 * Selection is computed in float32 probabilities with exact integer mass sums
 * (each probability's mass taken exactly from its float32 bit pattern in units of
 * 2^-63; probabilities below 2^-40 count as 0) and is deterministic.
 */
SPA_API spa_status spa_select(spa_handle h, const void* q_pre, const void* idx_cache,
                      const uint8_t* head_mask, const int64_t* seq_lens, int B,
                      int64_t max_seq_len, float p, int n_sink, int window,
                      int32_t* sel_idx, int32_t* sel_count, spa_stream stream);

/*
 * One decode step ("Full Attention Strikes Back", Methodology §1-§3, §5;
 * exact token attention as in "Hierarchical Global Attention", §4).
 * For every b < B and query head h (KV head g = h / G), with L = seq_lens[b]:
 *   S   = sinks ∪ window                    (streaming head)
 *       = sinks ∪ window ∪ T               (retrieval head, T as in spa_select)
 *   out[b][h] = sum_{j in S} softmax_j( <RoPE(q_pre[b][h], L-1), k_cache[b][g][j]> / sqrt(128) ) v_cache[b][g][j]
 *   q_pre, idx_cache, head_mask, seq_lens, max_seq_len, p, n_sink, window: as in spa_select
 *   k_cache, v_cache device [max_batch][Hkv][Lmax][128], kv_dtype (k post-RoPE)
 *   out             device float32 [B][Hq][128], written
 *   sel_count_opt   NULL, or device int32 [B * Hkv] receiving the selected counts
 * Attention is split over rows (split-K), each split keeping an online-softmax
 * state (m, l, acc) merged with log-sum-exp weights (inside the attention kernel
 * for bf16 caches, by a combine kernel for float32 caches).
 */
SPA_API spa_status spa_decode(spa_handle h, const void* q_pre, const void* k_cache, const void* v_cache,
                      const void* idx_cache, const uint8_t* head_mask, const int64_t* seq_lens,
                      int B, int64_t max_seq_len, float p, int n_sink, int window,
                      float* out, int32_t* sel_count_opt, spa_stream stream);

/*
 * Top-k selector variant: the fixed budget that "Full Attention Strikes Back"
 * (RTPurbo summary), Methodology §3, contrasts with dynamic top-p.  T keeps the
 * first k tokens of the (pi desc, position asc) order over all L tokens (every
 * token when k >= L); sinks and window are attended anyway and the lists exclude
 * them, as for top-p.  Every other argument, output and error is that of
 * spa_select / spa_decode; k must be >= 1 (else SPA_ERR_INVALID_ARG).  The same
 * exact radix select runs with every token's mass set to 1 and the target k.
 */
SPA_API spa_status spa_select_topk(spa_handle h, const void* q_pre, const void* idx_cache,
                      const uint8_t* head_mask, const int64_t* seq_lens, int B, int64_t max_seq_len,
                      int64_t k, int n_sink, int window, int32_t* sel_idx, int32_t* sel_count,
                      spa_stream stream);
SPA_API spa_status spa_decode_topk(spa_handle h, const void* q_pre, const void* k_cache, const void* v_cache,
                      const void* idx_cache, const uint8_t* head_mask, const int64_t* seq_lens,
                      int B, int64_t max_seq_len, int64_t k, int n_sink, int window,
                      float* out, int32_t* sel_count_opt, spa_stream stream);

/*
 * Block-granular top-p variant.  The "Hierarchical Global Attention" summary
 * (Central mechanism §4) routes each query to whole chunks of the context rather
 * than to single tokens; here the chunks are blocks of 64 consecutive positions,
 * [64 c, min(64 c + 64, L)), and the mass threshold is that of "Full Attention
 * Strikes Back" (RTPurbo summary), Methodology §3:
 *   pi_c = sum of pi_j over block c's tokens (pi_j as in spa_select);
 *   blocks in (pi_c desc, c asc) order; block c is kept iff the mass of the blocks
 *   before it is < p (every block when p >= 1);
 *   T = every position of a kept block, minus sinks and window, ascending.
 * The mass test runs on pi_c quantised as in spa_select (exact integer sums).
 * Every other argument, output and error is that of spa_select / spa_decode.
 */
SPA_API spa_status spa_select_blocks(spa_handle h, const void* q_pre, const void* idx_cache,
                      const uint8_t* head_mask, const int64_t* seq_lens, int B, int64_t max_seq_len,
                      float p, int n_sink, int window, int32_t* sel_idx, int32_t* sel_count,
                      spa_stream stream);
SPA_API spa_status spa_decode_blocks(spa_handle h, const void* q_pre, const void* k_cache, const void* v_cache,
                      const void* idx_cache, const uint8_t* head_mask, const int64_t* seq_lens,
                      int B, int64_t max_seq_len, float p, int n_sink, int window,
                      float* out, int32_t* sel_count_opt, spa_stream stream);

/* ---- compact KV layout (streaming heads keep only sinks and window) ----
 *
 * "Autonomy of Heads" summary, Deployment strategy: retrieval heads keep their global
 * KV state, streaming heads keep only a fixed sink cache and a recent window.  The
 * head partition (head_mask) fixes the layout, so every call on the same caches must
 * pass the same head_mask, n_sink and window.  With n_ret retrieval and
 * n_str = Hkv - n_ret streaming heads, the rank of a head is its index among the heads
 * of its kind (ascending head index):
 *   k_ret, v_ret   device [max_batch][n_ret][Lmax][128], kv_dtype: every position
 *   k_ring, v_ring device [max_batch][n_str][n_sink + window][128], kv_dtype: position t
 *                  at row t for t < n_sink, else at row n_sink + (t - n_sink) mod window
 *   idx_ret        device bf16 [max_batch][n_ret][Lmax][16]: retrieval heads only
 * Streaming heads then use (n_sink + window) / Lmax of their full-layout memory.
 * Pointers are 16-byte aligned; errors as for the full-layout calls.
 */

/* Append T new positions start_pos[b] .. start_pos[b] + T - 1 of every (b, KV head):
 *   k_new, v_new  device [B][Hkv][T][128], kv_dtype (k post-RoPE)
 * Retrieval heads store every position; a streaming head stores position t iff
 * t < n_sink or t >= max(n_sink, start_pos[b] + T - window) (what it still attends
 * after the call; these never share a ring row).  Positions outside [0, Lmax) are
 * skipped and reported by spa_device_status. */
SPA_API spa_status spa_kv_append_compact(spa_handle h, const void* k_new, const void* v_new,
                      const int64_t* start_pos, int B, int T, const uint8_t* head_mask, int n_sink,
                      int window, void* k_ret, void* v_ret, void* k_ring, void* v_ring, spa_stream stream);

/* spa_index_append for the retrieval heads only, into idx_ret at their rank. */
SPA_API spa_status spa_index_append_compact(spa_handle h, const void* k_pre, const int64_t* start_pos,
                      int B, int T, const uint8_t* head_mask, void* idx_ret, spa_stream stream);

/* spa_select / spa_decode on the compact layout: the same selection and outputs
 * (bit for bit: the same rows in the same order) as on full-layout caches holding the
 * same values. */
SPA_API spa_status spa_select_compact(spa_handle h, const void* q_pre, const void* idx_ret,
                      const uint8_t* head_mask, const int64_t* seq_lens, int B, int64_t max_seq_len,
                      float p, int n_sink, int window, int32_t* sel_idx, int32_t* sel_count,
                      spa_stream stream);
SPA_API spa_status spa_decode_compact(spa_handle h, const void* q_pre, const void* k_ret, const void* v_ret,
                      const void* k_ring, const void* v_ring, const void* idx_ret, const uint8_t* head_mask,
                      const int64_t* seq_lens, int B, int64_t max_seq_len, float p, int n_sink, int window,
                      float* out, int32_t* sel_count_opt, spa_stream stream);

/* The compact-layout calls with any selector of the full layout:
 *   SPA_SELECT_TOP_P   p as in spa_select (k unused)
 *   SPA_SELECT_TOP_K   k as in spa_select_topk (p unused; k >= 1)
 *   SPA_SELECT_BLOCKS  p as in spa_select_blocks (k unused)
 * Results equal the full-layout call with the same selector on the same values. */
#define SPA_SELECT_TOP_P 0
#define SPA_SELECT_TOP_K 1
#define SPA_SELECT_BLOCKS 2
SPA_API spa_status spa_select_compact_sel(spa_handle h, const void* q_pre, const void* idx_ret,
                      const uint8_t* head_mask, const int64_t* seq_lens, int B, int64_t max_seq_len,
                      int selector, float p, int64_t k, int n_sink, int window, int32_t* sel_idx,
                      int32_t* sel_count, spa_stream stream);
SPA_API spa_status spa_decode_compact_sel(spa_handle h, const void* q_pre, const void* k_ret, const void* v_ret,
                      const void* k_ring, const void* v_ring, const void* idx_ret, const uint8_t* head_mask,
                      const int64_t* seq_lens, int B, int64_t max_seq_len, int selector, float p, int64_t k,
                      int n_sink, int window, float* out, int32_t* sel_count_opt, spa_stream stream);

/* ---- prefill ----
 *
 * Attention of a prefill chunk ("Full Attention Strikes Back" (RTPurbo summary),
 * Methodology §1: retrieval heads attend the full context, local heads a sliding
 * window with sinks; "Autonomy of Heads" summary, Deployment strategy).  Chunk row i
 * of sequence b is the query at absolute position t = start_pos[b] + i; it attends
 *   retrieval head (head_mask[g] = 1): keys j in [0, t]
 *   streaming head:                    keys j <= t with j < n_sink or j > t - window
 *   out[b][h][i] = sum_j softmax_j(<RoPE(q_chunk[b][h][i], t), k_cache[b][g][j]> / sqrt(128)) v_cache[b][g][j]
 * The caches must already hold every position < start_pos[b] + T (append the chunk's
 * rows first).  The rotated query and the probabilities are rounded to bf16 for the
 * tensor cores (tcgen05 MMA with float32 accumulators in tensor memory; float32
 * scores).  Requires kv_dtype = SPA_BF16.
 *   q_chunk    device bf16 [B][Hq][T][128] pre-RoPE queries
 *   k_cache, v_cache device bf16 [max_batch][Hkv][Lmax][128] (full layout)
 *   head_mask  host uint8 [Hkv]
 *   start_pos  device int64 [B]; start_pos[b] + T must not exceed Lmax (a CTA that
 *              finds otherwise writes nothing and spa_device_status reports it)
 *   out        device float32 [B][Hq][T][128], written
 * Errors: SPA_ERR_INVALID_ARG for NULL or misaligned pointers, B or T out of range,
 * n_sink < 0, window < 0, n_sink + window < 1, or float32 caches. */
SPA_API spa_status spa_prefill(spa_handle h, const void* q_chunk, const void* k_cache, const void* v_cache,
                      const uint8_t* head_mask, const int64_t* start_pos, int B, int T, int n_sink,
                      int window, float* out, spa_stream stream);

/* ---- context-parallel decode ----
 *
 * One decode step of long sequences whose positions are split over n_ranks ranks
 * (one process per GPU, or several handles on one GPU): rank r holds the contiguous run
 * of global positions [pos0, pos0 + max_ctx) of every sequence in its own caches, local
 * row i = global position pos0 + i (the usual split is pos0 = r * max_ctx, every rank's
 * handle created with the same configuration).  The result is the step spa_decode
 * computes over the whole context ("Full Attention Strikes Back" (RTPurbo summary),
 * Methodology §2, §3, §5; split over the context as in the context-parallel scaling of
 * the "Lighthouse Attention" summary, Experimental results): the top-p set of each
 * retrieval group is taken over all ranks' tokens, ties at the cut go to the lowest
 * positions, sinks and window are global positions.  Top-p with bf16 caches only.
 *
 * The step is five phases, SPA_CP_STATS .. SPA_CP_ATTEND, run in order on every rank,
 * each followed by an exchange of the buffer it wrote (NCCL or any other transport; on
 * one GPU, emulated ranks share the buffers and need none):
 *   SPA_CP_STATS   per-head (max, sum of exp) of the local index scores -> stats   (gather)
 *   SPA_CP_MASS    local probabilities; round-1 mass histogram           -> hist1   (sum)
 *   SPA_CP_ROUND2  cut of round 1 (summed hist1); round-2 histogram      -> hist2   (sum)
 *   SPA_CP_ROUND3  cut of round 2; round-3 histogram with counts         -> hist3   (gather)
 *   SPA_CP_ATTEND  final cut and this rank's share of the ties; attention over the
 *                  local kept rows                                -> out_all, lse_all (gather)
 * then spa_cp_combine merges the ranks' outputs.  A gathered buffer is [n_ranks][...]
 * with the rank's slot at index rank: the phase writes its own slot and reads the
 * others, which must hold the other ranks' data of the previous phase (an all-gather).
 * A summed buffer (hist1, hist2) has no slots: the phase adds this rank's masses into
 * it and the exchange must leave every rank's copy holding the sum over the ranks (an
 * all-reduce; the words are uint64 and an int64 sum gives the same bits, as two's
 * complement addition is unsigned addition modulo 2^64).  Histogram masses are
 * integers, so the sums are exact and every rank reaches the same cut.  The rows a
 * phase adds into are cleared by an earlier phase of the same rank (stats clears
 * hist1, mass clears hist2 and its hist3 slot), so emulated ranks that share the
 * buffers add into one sum.  Streaming heads never select, so stats and hist1..hist3
 * hold one row per retrieval slice only: row b * n_ret + j (in slot r for the gathered
 * ones) for the j-th retrieval KV head (in head order) of sequence b, n_ret the number
 * of retrieval heads.  spa_cp_exchange_sizes gives the byte size of each buffer (all
 * slots) for a head mask; the buffers must be sized with the same mask the phases get.  Every pointer
 * is a device pointer, 16-byte aligned.  Phases and combine only enqueue work on
 * `stream`; a phase called out of order computes garbage but stays in bounds. */
#define SPA_CP_STATS 0
#define SPA_CP_MASS 1
#define SPA_CP_ROUND2 2
#define SPA_CP_ROUND3 3
#define SPA_CP_ATTEND 4
#define SPA_CP_NBUF 6     /* stats, hist1, hist2, hist3, out_all, lse_all */
typedef struct {
  const void* q_pre;        /* bf16 [B][Hq][128] pre-RoPE queries, the same on every rank */
  const void* k_cache;      /* bf16 [max_batch][Hkv][max_ctx][128] local post-RoPE keys */
  const void* v_cache;      /* bf16 [max_batch][Hkv][max_ctx][128] local values */
  const void* idx_cache;    /* bf16 [max_batch][Hkv][max_ctx][16] local index rows */
  const uint8_t* head_mask; /* host [Hkv], 1 = retrieval head */
  const int64_t* seq_lens;  /* device [B] GLOBAL lengths (the current token at L - 1) */
  int B;
  float p;                  /* in (0, 1] */
  int n_sink, window;       /* >= 0, n_sink + window >= 1 */
  int n_ranks, rank;        /* 1 <= n_ranks <= 1024, 0 <= rank < n_ranks */
  int64_t pos0;             /* global position of local row 0, >= 0; must grow with rank (ties at
                               the cut are handed out rank by rank, lowest positions first) */
  int64_t max_seq_len;      /* bound on the global lengths (0: the larger of n_ranks * max_ctx
                               and pos0 + max_ctx) */
  void* stats;              /* [n_ranks][B][n_ret][ceil(max_ctx / 4096)][G] float2 (may be NULL, as
                               may hist1..hist3, when head_mask has no retrieval head) */
  void* hist1;              /* [B][n_ret][4096] uint64, summed over the ranks */
  void* hist2;              /* [B][n_ret][4096] uint64, summed over the ranks */
  void* hist3;              /* [n_ranks][B][n_ret][64][2] uint64 */
  float* out_all;           /* [n_ranks][B][Hq][128] float32 */
  float* lse_all;           /* [n_ranks][B][Hq] float32, log2 of the softmax denominator */
  int32_t* sel_count_opt;   /* NULL or device [B][Hkv]: local rows attended (SPA_CP_ATTEND) */
  int32_t* list_opt;        /* NULL or device [B][Hkv][max_ctx]: the local rows attended, ascending
                               (sinks and window included; global position = pos0 + row) */
} spa_cp_args;
/* bytes[i] for the SPA_CP_NBUF buffers in spa_cp_args order, for the host head mask
 * head_mask [Hkv] (1 = retrieval head; the statistics and histograms are sized for its
 * retrieval heads, 0 bytes when it has none).  Errors: NULL handle, head_mask or bytes,
 * B outside [1, max_batch], n_ranks outside [1, 1024]. */
SPA_API spa_status spa_cp_exchange_sizes(spa_handle h, int B, int n_ranks, const uint8_t* head_mask,
                                         size_t* bytes);
/* Runs one phase on this rank.  Errors: SPA_ERR_INVALID_ARG for a NULL or misaligned
 * pointer (stats and hist1..hist3 may be NULL only without retrieval heads), an
 * unknown phase, B / p / n_sink / window / rank / pos0 out of range, or max_ctx < 64;
 * SPA_ERR_UNSUPPORTED for float32 caches. */
SPA_API spa_status spa_cp_phase(spa_handle h, int phase, const spa_cp_args* a, spa_stream stream);
/* out[b][h] = sum_r 2^(lse_r - M) out_r / sum_r 2^(lse_r - M), M = max_r lse_r, over
 * the gathered out_all / lse_all (ranks in order; a rank with lse = -inf attended
 * nothing for that head).  out: device float32 [B][Hq][128]. */
SPA_API spa_status spa_cp_combine(spa_handle h, const float* out_all, const float* lse_all, int n_ranks, int B,
                      float* out, spa_stream stream);

/* ---- head labels from frozen weights ----
 *
 * "Autonomy of Heads" summary, Methodology §1-§4: the effective rank of each query
 * head's kernel operator M_h = W_K^{g T} W_Q^h (g = h / G, its key head),
 *   ER(h) = exp(-sum_k s_k ln s_k),  s_k = sigma_k / sum_j sigma_j,
 * sigma_k the singular values of M_h, taken as the square roots of the eigenvalues of
 * the d_head x d_head proxy (W_Q W_Q^T)(W_K W_K^T).  Per KV head the mean ER of its G
 * query heads; the n_retrieval KV heads of lowest mean ER (ties: lower index) get
 * head_mask = 1 (retrieval), the others 0 (streaming).  Everything runs in float64 on
 * the device; squaring the operator returns a zero singular value as about
 * sqrt(eps) sigma_max, so rank-deficient heads carry an ER error of up to ~5e-4
 * relative, full-rank heads about 1e-9.  Run once per model, off the decode path.
 *   W_Q          device float32 [n_q_heads][128][d_model] (q = W_Q^h x)
 *   W_K          device float32 [n_kv_heads][128][d_model]
 *   workspace    device scratch of spa_head_ranks_workspace_size bytes, 16-byte aligned
 *   er_q         device float64 [n_q_heads], written
 *   er_kv        device float64 [n_kv_heads], written
 *   head_mask    device uint8 [n_kv_heads], written
 *   sigma_opt    NULL, or device float64 [n_q_heads][128]: singular values, descending
 * Errors: SPA_ERR_INVALID_ARG for NULL or misaligned pointers, n_q_heads not a multiple
 * of n_kv_heads, n_kv_heads outside [1, 64], d_model < 1, n_retrieval outside
 * [0, n_kv_heads], or a workspace smaller than required.  The call only enqueues work. */
SPA_API spa_status spa_head_ranks_workspace_size(int n_q_heads, int n_kv_heads, size_t* bytes);
SPA_API spa_status spa_head_effective_ranks(const float* W_Q, const float* W_K, int n_q_heads, int n_kv_heads,
                      int d_model, int n_retrieval, void* workspace, size_t workspace_bytes, double* er_q,
                      double* er_kv, uint8_t* head_mask, double* sigma_opt, spa_stream stream);

/*
 * Synchronise `stream`, then read and clear the handle's device status word.
 * Returns SPA_ERR_DEVICE_RANGE (with the offending field named in
 * spa_last_error) if a kernel clamped an out-of-range seq_lens/start_pos value
 * since the last check, else SPA_OK.
 */
SPA_API spa_status spa_device_status(spa_handle h, spa_stream stream);

/* Failure-detection test hook (no fault, no hang): while enabled, the first CTA of the
 * selection kernel leaves before its first arrival at its slice's counter, so every
 * other CTA of that slice waits for an arrival that never comes until its bounded wait
 * (about 2 s) gives up; the call completes with meaningless lists and spa_device_status reports
 * SPA_ERR_DEVICE_TIMEOUT (and resets the synchronisation state, so the next call on the
 * handle is sound).  Off by default; for tests only. */
SPA_API spa_status spa_debug_drop_publish(spa_handle h, int enable);

/* ---- instrumentation (used by the benchmark; off by default) ---- */

/* Kernel ids for spa_profile_read / spa_kernel_name.  Selection (query prologue,
 * index scores, mass histogram, threshold, compaction) is one cooperative kernel. */
#define SPA_K_INDEX_APPEND 0
#define SPA_K_SELECT 1
#define SPA_K_ATTEND 2
#define SPA_K_COMBINE 3
#define SPA_K_KV_APPEND 4
#define SPA_K_PREFILL 5
#define SPA_K_CP_SELECT 6   /* context-parallel selection phases (every kernel of them) */
#define SPA_K_COUNT 7

/* kernel_mask = 0 disables timing.  Otherwise every launch of a kernel whose bit
 * (1 << SPA_K_...) is set is bracketed by two CUDA events recorded on the launch
 * stream (a bounded pool; launches beyond it are not timed).  Each event pair
 * adds a few microseconds of stream time, so time only what is needed.  Setting
 * a mask resets the pool. */
SPA_API spa_status spa_set_profiling(spa_handle h, unsigned kernel_mask);

/* Synchronise the recorded events and return, for kernel `kernel_id`, the
 * summed device time in milliseconds and the number of timed launches. */
SPA_API spa_status spa_profile_read(spa_handle h, int kernel_id, double* total_ms, int64_t* launches);

/* Name of a kernel id ("" if unknown). */
SPA_API const char* spa_kernel_name(int kernel_id);

/* Number of kernel launches this handle has issued since it was created. */
SPA_API spa_status spa_launch_count(spa_handle h, int64_t* launches);

/*
 * spa_select without a handle and without allocating anything, for callers that
 * cannot call cudaMalloc: code inside a host framework that has reserved the GPU's
 * memory for its own pool, or a decode loop that cannot afford the implicit device
 * synchronisation an allocation may cause.  The paper has no counterpart to this
 * entry point; it exists for those callers only.
 * Inputs, outputs and result are those of spa_select; the query projectors are
 * passed directly (P_q: device float32 [n_q_heads][16][128]) and max_ctx is the row
 * stride of idx_cache and sel_idx; idx_scale <= 0 selects 0.25.
 * All scratch is one static 12 MiB device array, held by every GPU that loads the
 * library until the process exits.  Limits: B*n_kv_heads <= 64, B*n_q_heads <= 512,
 * B*n_kv_heads*max_ctx <= 2^19 tokens; larger requests return SPA_ERR_WORKSPACE
 * before anything is launched.  The first call on a device looks up the array's
 * device address there (cudaGetSymbolAddress, with that device current): make that
 * first call before any stream capture.  Every call shares the array and the next
 * call overwrites it, so calls that overlap on the GPU race: serialise them.
 * Before each launch the call clears, with one cudaMemsetAsync on `stream` (which
 * allocates nothing), the fixed block at the head of the array that holds the
 * status word and the per-slice state (the selection kernel's arrival counters),
 * so no call inherits synchronisation state from an earlier one of another shape.
 * Device-side conditions are not reported by this entry point (there is no handle
 * to hold a status word): out-of-range seq_lens values are clamped, and a bounded
 * device wait that gives up (about 2 s; the kernel then leaves early and its lists
 * and counts are not valid) or an internal consistency check that fails is dropped.
 * In every such case the call has already returned SPA_OK; the next call starts
 * from cleared state.  Callers that need these conditions reported use
 * spa_create + spa_select + spa_device_status.
 */
SPA_API spa_status spa_select_noalloc(const float* P_q, int n_q_heads, int n_kv_heads, int kv_dtype,
                                      float idx_scale, int64_t max_ctx, const void* q_pre,
                                      const void* idx_cache, const uint8_t* head_mask,
                                      const int64_t* seq_lens, int B, int64_t max_seq_len, float p,
                                      int n_sink, int window, int32_t* sel_idx, int32_t* sel_count,
                                      spa_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* SPA_H_ */
