// Host side of the libspa C ABI: argument checks, workspace, launch sequencing.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/spa.h"
#include "spa_internal.cuh"

namespace {

thread_local std::string g_err;

spa_status fail(spa_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

spa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SPA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  size_t off[18];
  size_t total;
  int64_t max_items;
  int n_chunks_max;
};

// Sizes every workspace region for a configuration (offsets 256-byte aligned).
Layout plan(const spa_config& c, int split_rows) {
  Layout L{};
  const int G = c.n_q_heads / c.n_kv_heads;
  const size_t slices = (size_t)c.max_batch * c.n_kv_heads;
  const int64_t Lmax = c.max_ctx;
  L.n_chunks_max = (int)((Lmax + spa::kChunk - 1) / spa::kChunk);
  L.max_items = (int64_t)slices * ((Lmax + split_rows - 1) / split_rows);
  const int64_t part_slots = L.max_items > (int64_t)(spa::kMaxAttendCtas + slices + 1)
                                 ? L.max_items : (int64_t)(spa::kMaxAttendCtas + slices + 1);
  size_t sz[18] = {
      (size_t)c.n_q_heads * 16 * 128 * 4,                  // 0 P_q
      (size_t)c.n_kv_heads * 16 * 128 * 4,                 // 1 P_k
      64 * 8,                                              // 2 inv_freq
      (size_t)c.max_batch * c.n_q_heads * 128 * 4,         // 3 q_rot
      (size_t)c.max_batch * c.n_q_heads * 16 * 4,          // 4 q_idx
      (spa::kMaxSelectGrid + slices) * G * 8,              // 5 stats
      slices * (size_t)spa::pi_row_stride(Lmax) * 4,       // 6 pi
      slices * spa::kBins1 * 8,                            // 7 hist1
      slices * (size_t)Lmax * 8,                           // 8 cand
      slices * L.n_chunks_max * 4,                         // 9 chunk counts (context-parallel)
      slices * sizeof(spa::SliceState),                    // 10 st
      slices * (size_t)Lmax * 4,                           // 11 list
      (slices + 1) * 4,                                    // 12 item_base
      (size_t)part_slots * G * spa::kPartStride * 4,       // 13 split states
      256,                                                 // 14 dev_err
      slices * spa::kBins2 * 8,                            // 15 hist2
      slices * 4,                                          // 16 attention tickets
      (spa::kMaxSelectGrid + slices) * 4,                  // 17 per-range counts above the cut bin (selection)
  };
  size_t o = 0;
  for (int i = 0; i < 18; ++i) {
    L.off[i] = o;
    o += round_up(sz[i], 256);
  }
  L.total = o;
  return L;
}

}  // namespace

namespace spa {
// Records `msg` as the calling thread's spa_last_error() text; returns `code`.
int set_last_error(int code, const char* msg) {
  g_err = msg;
  return code;
}
}  // namespace spa

struct spa_ctx {
  spa_config cfg{};
  int G = 0;
  int split_rows = 0;
  float idx_scale = 0.f;
  int device = 0;
  int num_sms = 0;
  int attend_occ = 1;
  int select_max_grid = 1;   // co-resident CTAs of the cooperative selection kernel
  void* mem = nullptr;
  size_t mem_bytes = 0;
  spa::Workspace ws{};
  int n_chunks_max = 0;
  // instrumentation
  unsigned prof_mask = 0;
  std::vector<cudaEvent_t> ev;   // pairs: 2*i start, 2*i+1 stop
  std::vector<int> ev_kid;
  size_t ev_next = 0;
  int64_t launches = 0;
  int drop_publish = 0;   // failure-detection test hook (spa_debug_drop_publish)
};

namespace {

constexpr size_t kEventPairs = 1 << 14;

spa_status check_config(const spa_config* c) {
  if (!c) return fail(SPA_ERR_INVALID_ARG, "config is NULL");
  if (c->head_dim != 128) return fail(SPA_ERR_UNSUPPORTED, "head_dim must be 128 (got %d)", c->head_dim);
  if (c->idx_dim != 16) return fail(SPA_ERR_UNSUPPORTED, "idx_dim must be 16 (got %d)", c->idx_dim);
  if (c->kv_dtype != SPA_BF16 && c->kv_dtype != SPA_F32)
    return fail(SPA_ERR_UNSUPPORTED, "kv_dtype must be SPA_BF16 or SPA_F32 (got %d)", c->kv_dtype);
  if (c->n_kv_heads < 1 || c->n_kv_heads > spa::kMaxKvHeads)
    return fail(SPA_ERR_UNSUPPORTED, "n_kv_heads must be in [1, %d] (got %d)", spa::kMaxKvHeads, c->n_kv_heads);
  if (c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads != 0)
    return fail(SPA_ERR_INVALID_ARG, "n_q_heads (%d) must be a positive multiple of n_kv_heads (%d)",
                c->n_q_heads, c->n_kv_heads);
  const int G = c->n_q_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(SPA_ERR_UNSUPPORTED, "GQA group size must be 1, 2, 4 or 8 (got %d)", G);
  if (c->max_batch < 1 || (int64_t)c->max_batch * c->n_kv_heads > 65535)
    return fail(SPA_ERR_INVALID_ARG, "max_batch must be >= 1 with max_batch*n_kv_heads <= 65535 (got %d)",
                c->max_batch);
  if (c->max_ctx < 1 || c->max_ctx > spa::kMaxCtx)
    return fail(SPA_ERR_INVALID_ARG, "max_ctx must be in [1, 2^24] (got %lld)", (long long)c->max_ctx);
  if (!(c->rope_theta > 0.0) || !std::isfinite(c->rope_theta))
    return fail(SPA_ERR_INVALID_ARG, "rope_theta must be positive and finite");
  if (!std::isfinite(c->idx_scale)) return fail(SPA_ERR_INVALID_ARG, "idx_scale must be finite");
  if (c->split_rows < 0 || c->split_rows % spa::kTile != 0)
    return fail(SPA_ERR_INVALID_ARG, "split_rows must be 0 or a positive multiple of %d (got %d)", spa::kTile,
                c->split_rows);
  if (!c->P_q || !c->P_k) return fail(SPA_ERR_INVALID_ARG, "P_q and P_k must be device pointers");
  if (!aligned16(c->P_q) || !aligned16(c->P_k)) return fail(SPA_ERR_INVALID_ARG, "P_q/P_k must be 16-byte aligned");
  return SPA_OK;
}

template <class F>
spa_status run(spa_ctx* h, int kid, cudaStream_t st, const char* name, F&& f) {
  const bool timed = ((h->prof_mask >> kid) & 1u) && h->ev_next < kEventPairs;
  if (timed) cudaEventRecord(h->ev[2 * h->ev_next], st);
  cudaError_t e = f();
  if (timed) {
    cudaEventRecord(h->ev[2 * h->ev_next + 1], st);
    h->ev_kid[h->ev_next++] = kid;
  }
  ++h->launches;
  if (e != cudaSuccess) return cuda_fail(e, name);
  return SPA_OK;
}

struct StepArgs {
  const void* q_pre;
  const void* idx_cache;
  const uint8_t* head_mask;
  const int64_t* seq_lens;
  int B;
  int64_t max_seq_len;
  float p;
  int n_sink, window;
  int64_t k;   // > 0: top-k selection with budget k (p unused)
  int blocks;  // 1: block-granular top-p
};

spa_status check_step(spa_ctx* h, const StepArgs& a, spa::StepParams* P) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (!a.q_pre || !a.idx_cache || !a.seq_lens || !a.head_mask)
    return fail(SPA_ERR_INVALID_ARG, "q_pre, idx_cache, seq_lens and head_mask must be non-NULL");
  if (!aligned16(a.q_pre) || !aligned16(a.idx_cache) || ((uintptr_t)a.seq_lens & 7u))
    return fail(SPA_ERR_INVALID_ARG, "q_pre/idx_cache must be 16-byte aligned, seq_lens 8-byte aligned");
  if (a.B < 1 || a.B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, a.B);
  if (a.k < 0) return fail(SPA_ERR_INVALID_ARG, "k must be >= 1 (got %lld)", (long long)a.k);
  if (a.k == 0 && (!(a.p > 0.f) || !(a.p <= 1.f)))
    return fail(SPA_ERR_INVALID_ARG, "p must be in (0, 1] (got %g)", (double)a.p);
  if (a.n_sink < 0 || a.window < 0) return fail(SPA_ERR_INVALID_ARG, "n_sink and window must be >= 0");
  if ((int64_t)a.n_sink + a.window < 1)
    return fail(SPA_ERR_INVALID_ARG, "n_sink + window must be >= 1 (a streaming head needs a token)");
  if (a.max_seq_len < 0 || a.max_seq_len > h->cfg.max_ctx)
    return fail(SPA_ERR_INVALID_ARG, "max_seq_len must be in [0, max_ctx=%lld] (got %lld)",
                (long long)h->cfg.max_ctx, (long long)a.max_seq_len);
  std::memset(P, 0, sizeof *P);
  const int Hkv = h->cfg.n_kv_heads;
  for (int g = 0; g < Hkv; ++g) {
    P->is_ret[g] = a.head_mask[g] ? 1 : 0;
    if (P->is_ret[g]) P->ret_heads[P->n_ret++] = g;
  }
  P->q_pre = a.q_pre;
  P->idx_cache = static_cast<const uint16_t*>(a.idx_cache);
  P->seq_lens = a.seq_lens;
  P->B = a.B;
  P->Hq = h->cfg.n_q_heads;
  P->Hkv = Hkv;
  P->G = h->G;
  P->Lmax = h->cfg.max_ctx;
  P->Lcap = (int)(a.max_seq_len ? a.max_seq_len : h->cfg.max_ctx);
  P->n_chunks = (P->Lcap + spa::kChunk - 1) / spa::kChunk;
  P->n_slices = a.B * Hkv;
  P->p = a.k > 0 ? 1.f : a.p;
  P->keep_all = a.k == 0 && a.p >= 1.f ? 1 : 0;
  P->topk = a.k;
  P->blocks = a.blocks;
  P->n_sink = a.n_sink;
  P->window = a.window;
  P->idx_scale_log2 = h->idx_scale * 1.4426950408889634f;
  P->attn_scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  P->split_rows = h->split_rows;
  P->drop_publish = h->drop_publish;
  P->ws = h->ws;
  return SPA_OK;
}

// Compact layout: ring size and each head's rank among the heads of its kind.
spa_status setup_compact(spa::StepParams* P, const void* k_ring, const void* v_ring, bool need_ring) {
  P->compact = 1;
  P->n_str = P->Hkv - P->n_ret;
  P->ring = P->n_sink + P->window;
  int nr = 0, ns = 0;
  for (int g = 0; g < P->Hkv; ++g) P->head_rank[g] = P->is_ret[g] ? nr++ : ns++;
  if (need_ring && P->n_str > 0) {
    if (!k_ring || !v_ring) return fail(SPA_ERR_INVALID_ARG, "k_ring and v_ring must be non-NULL");
    if (!aligned16(k_ring) || !aligned16(v_ring)) return fail(SPA_ERR_INVALID_ARG, "k_ring/v_ring must be 16-byte aligned");
  }
  P->k_ring = k_ring;
  P->v_ring = v_ring;
  return SPA_OK;
}

spa_status run_selection(spa_ctx* h, spa::StepParams& P, cudaStream_t st) {
  return run(h, SPA_K_SELECT, st, "select",
             [&] { return spa::launch_select(P, h->cfg.kv_dtype, h->select_max_grid, st); });
}

spa_status select_with(spa_ctx* h, spa::StepParams& P, int32_t* sel_idx, int32_t* sel_count, spa_stream stream) {
  if (!sel_idx || !sel_count) return fail(SPA_ERR_INVALID_ARG, "sel_idx and sel_count must be non-NULL");
  if (!aligned16(sel_idx) || ((uintptr_t)sel_count & 3u))
    return fail(SPA_ERR_INVALID_ARG, "sel_idx must be 16-byte aligned, sel_count 4-byte aligned");
  P.sel_list = sel_idx;
  P.sel_count = sel_count;
  return run_selection(h, P, reinterpret_cast<cudaStream_t>(stream));
}


spa_status decode_with(spa_ctx* h, spa::StepParams& P, const void* k_cache, const void* v_cache, float* out,
                       int32_t* sel_count_opt, spa_stream stream) {
  spa_status r = SPA_OK;
  if (!k_cache || !v_cache || !out) return fail(SPA_ERR_INVALID_ARG, "k_cache, v_cache and out must be non-NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return fail(SPA_ERR_INVALID_ARG, "k_cache, v_cache and out must be 16-byte aligned");
  if (sel_count_opt && ((uintptr_t)sel_count_opt & 3u)) return fail(SPA_ERR_INVALID_ARG, "sel_count_opt misaligned");
  P.k_cache = k_cache;
  P.v_cache = v_cache;
  P.out = out;
  P.sel_list = h->ws.list;
  P.sel_count = nullptr;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((r = run_selection(h, P, st))) return r;
  // upper bound on splits: every slice has at most Lcap rows
  const int64_t per_slice = (P.Lcap + P.split_rows - 1) / P.split_rows;
  const int64_t max_items = per_slice * P.n_slices;
  int64_t cap = (int64_t)h->num_sms * h->attend_occ;
  if (cap > spa::kMaxAttendCtas) cap = spa::kMaxAttendCtas;
  const int grid = (int)(max_items < cap ? max_items : cap);
  // bf16 caches: the attention kernel combines the splits and reports the counts itself
  if (h->cfg.kv_dtype == 0) P.sel_count = sel_count_opt;
  if ((r = run(h, SPA_K_ATTEND, st, "attend", [&] { return spa::launch_attend(P, h->cfg.kv_dtype, grid, st); })))
    return r;
  if (h->cfg.kv_dtype == 0) return SPA_OK;
  P.sel_count = sel_count_opt;
  return run(h, SPA_K_COMBINE, st, "combine", [&] { return spa::launch_combine(P, st); });
}


// Selector arguments of the compact entry points: top-p (p), top-k (k), block top-p (p).
spa_status selector_args(int selector, float p, int64_t k, float* p_out, int64_t* k_out, int* blocks_out) {
  switch (selector) {
    case SPA_SELECT_TOP_P: *p_out = p; *k_out = 0; *blocks_out = 0; return SPA_OK;
    case SPA_SELECT_TOP_K:
      if (k < 1) return fail(SPA_ERR_INVALID_ARG, "k must be >= 1 (got %lld)", (long long)k);
      *p_out = 1.f; *k_out = k; *blocks_out = 0; return SPA_OK;
    case SPA_SELECT_BLOCKS: *p_out = p; *k_out = 0; *blocks_out = 1; return SPA_OK;
  }
  return fail(SPA_ERR_INVALID_ARG, "selector must be SPA_SELECT_TOP_P, _TOP_K or _BLOCKS (got %d)", selector);
}

spa_status select_compact_with(spa_ctx* h, const void* q_pre, const void* idx_ret, const uint8_t* head_mask,
                               const int64_t* seq_lens, int B, int64_t max_seq_len, int selector, float p, int64_t k,
                               int n_sink, int window, int32_t* sel_idx, int32_t* sel_count, spa_stream stream) {
  float pp;
  int64_t kk;
  int blocks;
  spa_status r = selector_args(selector, p, k, &pp, &kk, &blocks);
  if (r) return r;
  spa::StepParams P;
  r = check_step(h, StepArgs{q_pre, idx_ret, head_mask, seq_lens, B, max_seq_len, pp, n_sink, window, kk, blocks}, &P);
  if (r) return r;
  if ((r = setup_compact(&P, nullptr, nullptr, false))) return r;
  return select_with(h, P, sel_idx, sel_count, stream);
}

spa_status decode_compact_with(spa_ctx* h, const void* q_pre, const void* k_ret, const void* v_ret,
                               const void* k_ring, const void* v_ring, const void* idx_ret, const uint8_t* head_mask,
                               const int64_t* seq_lens, int B, int64_t max_seq_len, int selector, float p, int64_t k,
                               int n_sink, int window, float* out, int32_t* sel_count_opt, spa_stream stream) {
  float pp;
  int64_t kk;
  int blocks;
  spa_status r = selector_args(selector, p, k, &pp, &kk, &blocks);
  if (r) return r;
  spa::StepParams P;
  r = check_step(h, StepArgs{q_pre, idx_ret, head_mask, seq_lens, B, max_seq_len, pp, n_sink, window, kk, blocks}, &P);
  if (r) return r;
  if ((r = setup_compact(&P, k_ring, v_ring, true))) return r;
  if (P.n_ret == 0) {   // no retrieval head: the retrieval caches are never read
    static const uint4 dummy[1] = {};
    if (!k_ret) k_ret = dummy;
    if (!v_ret) v_ret = dummy;
  }
  return decode_with(h, P, k_ret, v_ret, out, sel_count_opt, stream);
}

// ---------------------------------------------------------------- context-parallel
constexpr int kMaxRanks = 1024;

int count_retrieval(const spa_ctx* h, const uint8_t* head_mask) {
  int n = 0;
  for (int g = 0; g < h->cfg.n_kv_heads; ++g) n += head_mask[g] ? 1 : 0;
  return n;
}

spa_status cp_check(spa_ctx* h, const spa_cp_args* a, spa::CpParams* C) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (!a) return fail(SPA_ERR_INVALID_ARG, "args is NULL");
  if (h->cfg.kv_dtype != SPA_BF16) return fail(SPA_ERR_UNSUPPORTED, "context-parallel decode needs bf16 caches");
  if (h->cfg.max_ctx < 64) return fail(SPA_ERR_INVALID_ARG, "context-parallel decode needs max_ctx >= 64");
  if (!a->q_pre || !a->k_cache || !a->v_cache || !a->idx_cache || !a->head_mask || !a->seq_lens || !a->out_all ||
      !a->lse_all)
    return fail(SPA_ERR_INVALID_ARG, "q_pre, the caches, head_mask, seq_lens, out_all and lse_all must be non-NULL");
  const int n_ret = count_retrieval(h, a->head_mask);
  if (n_ret > 0 && (!a->stats || !a->hist1 || !a->hist2 || !a->hist3))
    return fail(SPA_ERR_INVALID_ARG, "stats, hist1, hist2 and hist3 must be non-NULL when a head is a retrieval head");
  if (!aligned16(a->q_pre) || !aligned16(a->k_cache) || !aligned16(a->v_cache) || !aligned16(a->idx_cache) ||
      !aligned16(a->stats) || !aligned16(a->hist1) || !aligned16(a->hist2) || !aligned16(a->hist3) ||
      !aligned16(a->out_all) || !aligned16(a->lse_all) || ((uintptr_t)a->seq_lens & 7u) ||
      ((uintptr_t)a->sel_count_opt & 3u) || !aligned16(a->list_opt))
    return fail(SPA_ERR_INVALID_ARG, "spa_cp_args pointers must be 16-byte aligned (seq_lens 8, sel_count_opt 4)");
  if (a->B < 1 || a->B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, a->B);
  if (!(a->p > 0.f) || !(a->p <= 1.f)) return fail(SPA_ERR_INVALID_ARG, "p must be in (0, 1] (got %g)", (double)a->p);
  if (a->n_sink < 0 || a->window < 0 || (int64_t)a->n_sink + a->window < 1)
    return fail(SPA_ERR_INVALID_ARG, "n_sink, window must be >= 0 with n_sink + window >= 1");
  if (a->n_ranks < 1 || a->n_ranks > kMaxRanks || a->rank < 0 || a->rank >= a->n_ranks)
    return fail(SPA_ERR_INVALID_ARG, "need 1 <= n_ranks <= %d and 0 <= rank < n_ranks (got %d, %d)", kMaxRanks,
                a->n_ranks, a->rank);
  // default bound: the whole contiguous split (n_ranks * max_ctx), or this rank's end
  const int64_t split_end = (int64_t)a->n_ranks * h->cfg.max_ctx, rank_end = a->pos0 + h->cfg.max_ctx;
  const int64_t cap = a->max_seq_len ? a->max_seq_len : (split_end > rank_end ? split_end : rank_end);
  if (a->pos0 < 0 || a->pos0 + h->cfg.max_ctx > INT32_MAX || cap < 1 || cap > INT32_MAX)
    return fail(SPA_ERR_INVALID_ARG, "need pos0 >= 0, pos0 + max_ctx < 2^31 and max_seq_len in [1, 2^31) (got %lld, %lld)",
                (long long)a->pos0, (long long)cap);
  std::memset(C, 0, sizeof *C);
  const int Hkv = h->cfg.n_kv_heads;
  for (int g = 0; g < Hkv; ++g) {
    C->is_ret[g] = a->head_mask[g] ? 1 : 0;
    C->ret_ord[g] = C->is_ret[g] ? (signed char)C->n_ret++ : (signed char)-1;
  }
  C->n_xrows = a->B * C->n_ret;
  C->q_pre = a->q_pre;
  C->idx = static_cast<const uint16_t*>(a->idx_cache);
  C->seq_lens = a->seq_lens;
  C->B = a->B;
  C->Hq = h->cfg.n_q_heads;
  C->Hkv = Hkv;
  C->G = h->G;
  C->n_slices = a->B * Hkv;
  C->C = h->cfg.max_ctx;
  C->n_chunks = h->n_chunks_max;
  C->pos0 = a->pos0;
  C->rank = a->rank;
  C->n_ranks = a->n_ranks;
  C->Lcap = (int)cap;
  C->p = a->p;
  C->keep_all = a->p >= 1.f ? 1 : 0;
  C->n_sink = a->n_sink;
  C->window = a->window;
  C->idx_scale_log2 = h->idx_scale * 1.4426950408889634f;
  const spa::Workspace& w = h->ws;
  C->P_q = w.P_q;
  C->inv_freq_pi = w.inv_freq;
  C->q_rot = w.q_rot;
  C->q_idx = w.q_idx;
  C->pi = w.pi;
  C->pi_stride = w.pi_stride;
  C->stats = static_cast<float2*>(a->stats);
  C->hist1 = static_cast<unsigned long long*>(a->hist1);
  C->hist2 = static_cast<unsigned long long*>(a->hist2);
  C->hist3 = static_cast<unsigned long long*>(a->hist3);
  // the one-GPU selection's candidate buffer and round-2 histogram are free during a
  // context-parallel step: they hold the per-chunk round-3 counts and the cut states
  // (max_ctx >= 64 makes [slices][n_chunks][64] counts fit in [slices][max_ctx] uint2)
  C->tab3 = reinterpret_cast<unsigned*>(w.cand);
  C->cs = reinterpret_cast<spa::CpSlice*>(w.hist2);
  C->chunk_cnt = w.chunk_gt;
  C->list = a->list_opt ? a->list_opt : w.list;
  C->st = w.st;
  C->sel_count = a->sel_count_opt;
  C->out_rank = a->out_all + (size_t)a->rank * a->B * C->Hq * spa::kHeadDim;
  C->lse_rank = a->lse_all + (size_t)a->rank * a->B * C->Hq;
  C->err = w.dev_err;
  return SPA_OK;
}

// Attention over the rank's listed rows: every slice gathers (no contiguous rows).
spa_status cp_attend(spa_ctx* h, const spa_cp_args* a, const spa::CpParams& C, cudaStream_t st) {
  spa::StepParams P;
  std::memset(&P, 0, sizeof P);
  P.q_pre = a->q_pre;
  P.k_cache = a->k_cache;
  P.v_cache = a->v_cache;
  P.idx_cache = C.idx;
  P.seq_lens = a->seq_lens;
  P.out = C.out_rank;
  P.lse = C.lse_rank;
  P.sel_list = C.list;
  P.sel_count = nullptr;
  P.B = C.B;
  P.Hq = C.Hq;
  P.Hkv = C.Hkv;
  P.G = C.G;
  P.Lmax = h->cfg.max_ctx;
  P.Lcap = C.Lcap;
  P.n_slices = C.n_slices;
  P.p = 1.f;
  P.n_sink = 0;    // sinks and window are in the lists
  P.window = 0;
  P.attn_scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  P.split_rows = h->split_rows;
  for (int g = 0; g < C.Hkv; ++g) {
    P.is_ret[g] = 1;
    P.ret_heads[P.n_ret++] = g;
  }
  P.ws = h->ws;
  const int64_t per_slice = (h->cfg.max_ctx + P.split_rows - 1) / P.split_rows;
  const int64_t max_items = per_slice * P.n_slices;
  int64_t cap = (int64_t)h->num_sms * h->attend_occ;
  if (cap > spa::kMaxAttendCtas) cap = spa::kMaxAttendCtas;
  const int grid = (int)(max_items < cap ? max_items : cap);
  return run(h, SPA_K_ATTEND, st, "cp attend", [&] { return spa::launch_attend_bf16(P, grid, st); });
}

}  // namespace

extern "C" {

const char* spa_last_error(void) { return g_err.c_str(); }

spa_status spa_workspace_size(const spa_config* cfg, size_t* bytes) {
  spa_status r = check_config(cfg);
  if (r) return r;
  if (!bytes) return fail(SPA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = plan(*cfg, cfg->split_rows ? cfg->split_rows : spa::kDefaultSplitRows).total;
  return SPA_OK;
}

spa_status spa_create(spa_handle* out, const spa_config* cfg) {
  if (!out) return fail(SPA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  spa_status r = check_config(cfg);
  if (r) return r;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(SPA_ERR_UNSUPPORTED, "libspa is built for sm_100a (B200); device %d is sm_%d%d", dev, major, minor);

  spa_ctx* h = new (std::nothrow) spa_ctx;
  if (!h) return fail(SPA_ERR_WORKSPACE, "out of host memory");
  h->cfg = *cfg;
  h->G = cfg->n_q_heads / cfg->n_kv_heads;
  h->split_rows = cfg->split_rows ? cfg->split_rows : spa::kDefaultSplitRows;
  h->idx_scale = cfg->idx_scale > 0.f ? cfg->idx_scale : 0.25f;
  h->device = dev;
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  const Layout L = plan(*cfg, h->split_rows);
  e = cudaMalloc(&h->mem, L.total);
  if (e != cudaSuccess) {
    delete h;
    return fail(SPA_ERR_WORKSPACE, "cudaMalloc of %zu workspace bytes failed: %s", L.total, cudaGetErrorString(e));
  }
  h->mem_bytes = L.total;
  char* base = static_cast<char*>(h->mem);
  spa::Workspace& w = h->ws;
  w.P_q = (float*)(base + L.off[0]);
  w.P_k = (float*)(base + L.off[1]);
  w.inv_freq = (double*)(base + L.off[2]);
  w.q_rot = (float*)(base + L.off[3]);
  w.q_idx = (float*)(base + L.off[4]);
  w.stats = (float2*)(base + L.off[5]);
  w.pi = (float*)(base + L.off[6]);
  w.pi_stride = spa::pi_row_stride(cfg->max_ctx);
  w.hist1 = (unsigned long long*)(base + L.off[7]);
  w.cand = (uint2*)(base + L.off[8]);
  w.chunk_gt = (int*)(base + L.off[9]);
  w.st = (spa::SliceState*)(base + L.off[10]);
  w.list = (int*)(base + L.off[11]);
  w.item_base = (int*)(base + L.off[12]);
  w.part = (float*)(base + L.off[13]);
  w.dev_err = (unsigned*)(base + L.off[14]);
  w.hist2 = (unsigned long long*)(base + L.off[15]);
  w.attn_ticket = (unsigned*)(base + L.off[16]);
  w.seg_cnt = (int*)(base + L.off[17]);
  w.max_items = L.max_items;
  h->n_chunks_max = L.n_chunks_max;

  double invf[64];
  // inverse frequencies theta^(-2i/128), stored divided by pi (the device works in units of pi)
  const double kPi = 3.141592653589793238462643383279502884;
  for (int i = 0; i < 64; ++i) invf[i] = std::pow(cfg->rope_theta, -2.0 * i / 128.0) / kPi;
  const size_t pq = (size_t)cfg->n_q_heads * 16 * 128 * 4, pk = (size_t)cfg->n_kv_heads * 16 * 128 * 4;
  if ((e = cudaMemcpy(w.P_q, cfg->P_q, pq, cudaMemcpyDeviceToDevice)) != cudaSuccess ||
      (e = cudaMemcpy(w.P_k, cfg->P_k, pk, cudaMemcpyDeviceToDevice)) != cudaSuccess ||
      (e = cudaMemcpy(w.inv_freq, invf, sizeof invf, cudaMemcpyHostToDevice)) != cudaSuccess ||
      (e = cudaMemset(w.dev_err, 0, 4)) != cudaSuccess ||
      (e = cudaMemset(w.st, 0, L.off[11] - L.off[10])) != cudaSuccess ||
      (e = cudaMemset(w.attn_ticket, 0, (size_t)cfg->max_batch * cfg->n_kv_heads * 4)) != cudaSuccess ||
      (e = cudaDeviceSynchronize()) != cudaSuccess) {
    cudaFree(h->mem);
    delete h;
    return cuda_fail(e, "spa_create: copying projectors");
  }
  const int occ = spa::attend_setup(cfg->kv_dtype, h->G, cfg->max_batch * cfg->n_kv_heads);
  if (occ < 1) {
    cudaFree(h->mem);
    delete h;
    return fail(SPA_ERR_UNSUPPORTED, "attention kernel cannot be resident with this configuration");
  }
  h->attend_occ = occ;
  const int sel_occ = spa::select_resident_per_sm(cfg->kv_dtype, h->G);
  if (sel_occ < 1) {
    cudaFree(h->mem);
    delete h;
    return fail(SPA_ERR_UNSUPPORTED, "selection kernel cannot be resident with this configuration");
  }
  h->select_max_grid = sel_occ * h->num_sms;
  if (h->select_max_grid > spa::kMaxSelectGrid) h->select_max_grid = spa::kMaxSelectGrid;
  *out = h;
  return SPA_OK;
}

spa_status spa_destroy(spa_handle h) {
  if (!h) return SPA_OK;
  cudaDeviceSynchronize();
  for (cudaEvent_t ev : h->ev) cudaEventDestroy(ev);
  cudaError_t e = cudaFree(h->mem);
  delete h;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree");
  return SPA_OK;
}

spa_status spa_index_append(spa_handle h, const void* k_pre, const int64_t* start_pos, int B, int T,
                            void* idx_cache, spa_stream stream) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (!k_pre || !start_pos || !idx_cache) return fail(SPA_ERR_INVALID_ARG, "k_pre, start_pos, idx_cache must be non-NULL");
  if (!aligned16(k_pre) || !aligned16(idx_cache) || ((uintptr_t)start_pos & 7u))
    return fail(SPA_ERR_INVALID_ARG, "k_pre/idx_cache must be 16-byte aligned, start_pos 8-byte aligned");
  if (B < 1 || B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, B);
  if (T < 1 || (int64_t)T > h->cfg.max_ctx)
    return fail(SPA_ERR_INVALID_ARG, "T must be in [1, max_ctx] (got %d)", T);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return run(h, SPA_K_INDEX_APPEND, st, "index append", [&] {
    return spa::launch_index_append(k_pre, start_pos, B, T, h->cfg.n_kv_heads, h->cfg.max_ctx, h->cfg.kv_dtype,
                                    h->ws.P_k, static_cast<uint16_t*>(idx_cache), h->ws.dev_err, st);
  });
}

spa_status spa_select(spa_handle h, const void* q_pre, const void* idx_cache, const uint8_t* head_mask,
                      const int64_t* seq_lens, int B, int64_t max_seq_len, float p, int n_sink, int window,
                      int32_t* sel_idx, int32_t* sel_count, spa_stream stream) {
  spa::StepParams P;
  spa_status r = check_step(h, StepArgs{q_pre, idx_cache, head_mask, seq_lens, B, max_seq_len, p, n_sink, window, 0, 0}, &P);
  if (r) return r;
  return select_with(h, P, sel_idx, sel_count, stream);
}

spa_status spa_select_topk(spa_handle h, const void* q_pre, const void* idx_cache, const uint8_t* head_mask,
                           const int64_t* seq_lens, int B, int64_t max_seq_len, int64_t k, int n_sink, int window,
                           int32_t* sel_idx, int32_t* sel_count, spa_stream stream) {
  spa::StepParams P;
  if (k < 1) return fail(SPA_ERR_INVALID_ARG, "k must be >= 1 (got %lld)", (long long)k);
  spa_status r = check_step(h, StepArgs{q_pre, idx_cache, head_mask, seq_lens, B, max_seq_len, 1.f, n_sink, window, k, 0}, &P);
  if (r) return r;
  return select_with(h, P, sel_idx, sel_count, stream);
}

spa_status spa_decode(spa_handle h, const void* q_pre, const void* k_cache, const void* v_cache,
                      const void* idx_cache, const uint8_t* head_mask, const int64_t* seq_lens, int B,
                      int64_t max_seq_len, float p, int n_sink, int window, float* out, int32_t* sel_count_opt,
                      spa_stream stream) {
  spa::StepParams P;
  spa_status r = check_step(h, StepArgs{q_pre, idx_cache, head_mask, seq_lens, B, max_seq_len, p, n_sink, window, 0, 0}, &P);
  if (r) return r;
  return decode_with(h, P, k_cache, v_cache, out, sel_count_opt, stream);
}

spa_status spa_decode_topk(spa_handle h, const void* q_pre, const void* k_cache, const void* v_cache,
                           const void* idx_cache, const uint8_t* head_mask, const int64_t* seq_lens, int B,
                           int64_t max_seq_len, int64_t k, int n_sink, int window, float* out, int32_t* sel_count_opt,
                           spa_stream stream) {
  spa::StepParams P;
  if (k < 1) return fail(SPA_ERR_INVALID_ARG, "k must be >= 1 (got %lld)", (long long)k);
  spa_status r = check_step(h, StepArgs{q_pre, idx_cache, head_mask, seq_lens, B, max_seq_len, 1.f, n_sink, window, k, 0}, &P);
  if (r) return r;
  return decode_with(h, P, k_cache, v_cache, out, sel_count_opt, stream);
}

spa_status spa_select_blocks(spa_handle h, const void* q_pre, const void* idx_cache, const uint8_t* head_mask,
                             const int64_t* seq_lens, int B, int64_t max_seq_len, float p, int n_sink, int window,
                             int32_t* sel_idx, int32_t* sel_count, spa_stream stream) {
  spa::StepParams P;
  spa_status r = check_step(h, StepArgs{q_pre, idx_cache, head_mask, seq_lens, B, max_seq_len, p, n_sink, window, 0, 1}, &P);
  if (r) return r;
  return select_with(h, P, sel_idx, sel_count, stream);
}

spa_status spa_decode_blocks(spa_handle h, const void* q_pre, const void* k_cache, const void* v_cache,
                             const void* idx_cache, const uint8_t* head_mask, const int64_t* seq_lens, int B,
                             int64_t max_seq_len, float p, int n_sink, int window, float* out, int32_t* sel_count_opt,
                             spa_stream stream) {
  spa::StepParams P;
  spa_status r = check_step(h, StepArgs{q_pre, idx_cache, head_mask, seq_lens, B, max_seq_len, p, n_sink, window, 0, 1}, &P);
  if (r) return r;
  return decode_with(h, P, k_cache, v_cache, out, sel_count_opt, stream);
}

spa_status spa_kv_append_compact(spa_handle h, const void* k_new, const void* v_new, const int64_t* start_pos,
                                 int B, int T, const uint8_t* head_mask, int n_sink, int window, void* k_ret,
                                 void* v_ret, void* k_ring, void* v_ring, spa_stream stream) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (!k_new || !v_new || !start_pos || !head_mask)
    return fail(SPA_ERR_INVALID_ARG, "k_new, v_new, start_pos and head_mask must be non-NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || ((uintptr_t)start_pos & 7u))
    return fail(SPA_ERR_INVALID_ARG, "k_new/v_new must be 16-byte aligned, start_pos 8-byte aligned");
  if (B < 1 || B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, B);
  if (T < 1 || (int64_t)T > h->cfg.max_ctx)
    return fail(SPA_ERR_INVALID_ARG, "T must be in [1, max_ctx] (got %d)", T);
  if (n_sink < 0 || window < 0 || (int64_t)n_sink + window < 1)
    return fail(SPA_ERR_INVALID_ARG, "n_sink, window must be >= 0 with n_sink + window >= 1");
  const int Hkv = h->cfg.n_kv_heads;
  unsigned char is_ret[spa::kMaxKvHeads];
  int rank[spa::kMaxKvHeads];
  int n_ret = 0, n_str = 0;
  for (int g = 0; g < Hkv; ++g) {
    is_ret[g] = head_mask[g] ? 1 : 0;
    rank[g] = is_ret[g] ? n_ret++ : n_str++;
  }
  if (n_ret > 0 && (!k_ret || !v_ret || !aligned16(k_ret) || !aligned16(v_ret)))
    return fail(SPA_ERR_INVALID_ARG, "k_ret/v_ret must be non-NULL and 16-byte aligned");
  if (n_str > 0 && (!k_ring || !v_ring || !aligned16(k_ring) || !aligned16(v_ring)))
    return fail(SPA_ERR_INVALID_ARG, "k_ring/v_ring must be non-NULL and 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return run(h, SPA_K_KV_APPEND, st, "kv append", [&] {
    return spa::launch_kv_append_compact(k_new, v_new, start_pos, B, T, Hkv, h->cfg.max_ctx, h->cfg.kv_dtype, is_ret,
                                         rank, n_ret, n_str, n_sink, window, k_ret, v_ret, k_ring, v_ring,
                                         h->ws.dev_err, st);
  });
}

spa_status spa_index_append_compact(spa_handle h, const void* k_pre, const int64_t* start_pos, int B, int T,
                                    const uint8_t* head_mask, void* idx_ret, spa_stream stream) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (!k_pre || !start_pos || !idx_ret || !head_mask)
    return fail(SPA_ERR_INVALID_ARG, "k_pre, start_pos, head_mask, idx_ret must be non-NULL");
  if (!aligned16(k_pre) || !aligned16(idx_ret) || ((uintptr_t)start_pos & 7u))
    return fail(SPA_ERR_INVALID_ARG, "k_pre/idx_ret must be 16-byte aligned, start_pos 8-byte aligned");
  if (B < 1 || B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, B);
  if (T < 1 || (int64_t)T > h->cfg.max_ctx)
    return fail(SPA_ERR_INVALID_ARG, "T must be in [1, max_ctx] (got %d)", T);
  spa::HeadMap m;
  m.n = 0;
  for (int g = 0; g < h->cfg.n_kv_heads; ++g)
    if (head_mask[g]) {
      m.g[m.n] = g;
      m.slot[m.n] = m.n;
      ++m.n;
    }
  m.n_slots = m.n;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return run(h, SPA_K_INDEX_APPEND, st, "index append", [&] {
    return spa::launch_index_append(k_pre, start_pos, B, T, h->cfg.n_kv_heads, h->cfg.max_ctx, h->cfg.kv_dtype,
                                    h->ws.P_k, static_cast<uint16_t*>(idx_ret), h->ws.dev_err, st, &m);
  });
}

spa_status spa_select_compact(spa_handle h, const void* q_pre, const void* idx_ret, const uint8_t* head_mask,
                              const int64_t* seq_lens, int B, int64_t max_seq_len, float p, int n_sink, int window,
                              int32_t* sel_idx, int32_t* sel_count, spa_stream stream) {
  return select_compact_with(h, q_pre, idx_ret, head_mask, seq_lens, B, max_seq_len, SPA_SELECT_TOP_P, p, 0, n_sink,
                             window, sel_idx, sel_count, stream);
}

spa_status spa_decode_compact(spa_handle h, const void* q_pre, const void* k_ret, const void* v_ret,
                              const void* k_ring, const void* v_ring, const void* idx_ret, const uint8_t* head_mask,
                              const int64_t* seq_lens, int B, int64_t max_seq_len, float p, int n_sink, int window,
                              float* out, int32_t* sel_count_opt, spa_stream stream) {
  return decode_compact_with(h, q_pre, k_ret, v_ret, k_ring, v_ring, idx_ret, head_mask, seq_lens, B, max_seq_len,
                             SPA_SELECT_TOP_P, p, 0, n_sink, window, out, sel_count_opt, stream);
}

spa_status spa_select_compact_sel(spa_handle h, const void* q_pre, const void* idx_ret, const uint8_t* head_mask,
                                  const int64_t* seq_lens, int B, int64_t max_seq_len, int selector, float p,
                                  int64_t k, int n_sink, int window, int32_t* sel_idx, int32_t* sel_count,
                                  spa_stream stream) {
  return select_compact_with(h, q_pre, idx_ret, head_mask, seq_lens, B, max_seq_len, selector, p, k, n_sink, window,
                             sel_idx, sel_count, stream);
}

spa_status spa_decode_compact_sel(spa_handle h, const void* q_pre, const void* k_ret, const void* v_ret,
                                  const void* k_ring, const void* v_ring, const void* idx_ret,
                                  const uint8_t* head_mask, const int64_t* seq_lens, int B, int64_t max_seq_len,
                                  int selector, float p, int64_t k, int n_sink, int window, float* out,
                                  int32_t* sel_count_opt, spa_stream stream) {
  return decode_compact_with(h, q_pre, k_ret, v_ret, k_ring, v_ring, idx_ret, head_mask, seq_lens, B, max_seq_len,
                             selector, p, k, n_sink, window, out, sel_count_opt, stream);
}

spa_status spa_head_ranks_workspace_size(int n_q_heads, int n_kv_heads, size_t* bytes) {
  if (!bytes) return fail(SPA_ERR_INVALID_ARG, "bytes is NULL");
  if (n_kv_heads < 1 || n_kv_heads > spa::kMaxKvHeads || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads)
    return fail(SPA_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads in [1, %d]",
                spa::kMaxKvHeads);
  *bytes = spa::head_rank_workspace_bytes(n_q_heads, n_kv_heads);
  return SPA_OK;
}

spa_status spa_head_effective_ranks(const float* W_Q, const float* W_K, int n_q_heads, int n_kv_heads, int d_model,
                                    int n_retrieval, void* workspace, size_t workspace_bytes, double* er_q,
                                    double* er_kv, uint8_t* head_mask, double* sigma_opt, spa_stream stream) {
  size_t need = 0;
  spa_status r = spa_head_ranks_workspace_size(n_q_heads, n_kv_heads, &need);
  if (r) return r;
  if (!W_Q || !W_K || !workspace || !er_q || !er_kv || !head_mask)
    return fail(SPA_ERR_INVALID_ARG, "W_Q, W_K, workspace, er_q, er_kv and head_mask must be non-NULL");
  if (!aligned16(W_Q) || !aligned16(W_K) || !aligned16(workspace) || ((uintptr_t)er_q & 7u) ||
      ((uintptr_t)er_kv & 7u) || ((uintptr_t)sigma_opt & 7u))
    return fail(SPA_ERR_INVALID_ARG, "W_Q/W_K/workspace must be 16-byte aligned, outputs 8-byte aligned");
  if (d_model < 1) return fail(SPA_ERR_INVALID_ARG, "d_model must be >= 1 (got %d)", d_model);
  if (n_retrieval < 0 || n_retrieval > n_kv_heads)
    return fail(SPA_ERR_INVALID_ARG, "n_retrieval must be in [0, n_kv_heads] (got %d)", n_retrieval);
  if (workspace_bytes < need)
    return fail(SPA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  cudaError_t e = spa::launch_head_ranks(W_Q, W_K, n_q_heads, n_kv_heads, d_model, n_retrieval, workspace, er_q,
                                         er_kv, head_mask, sigma_opt, nullptr, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "head ranks");
  return SPA_OK;
}

spa_status spa_prefill(spa_handle h, const void* q_chunk, const void* k_cache, const void* v_cache,
                       const uint8_t* head_mask, const int64_t* start_pos, int B, int T, int n_sink, int window,
                       float* out, spa_stream stream) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (h->cfg.kv_dtype != 0) return fail(SPA_ERR_INVALID_ARG, "spa_prefill needs bf16 caches (kv_dtype = SPA_BF16)");
  if (!q_chunk || !k_cache || !v_cache || !head_mask || !start_pos || !out)
    return fail(SPA_ERR_INVALID_ARG, "q_chunk, k_cache, v_cache, head_mask, start_pos and out must be non-NULL");
  if (!aligned16(q_chunk) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      ((uintptr_t)start_pos & 7u))
    return fail(SPA_ERR_INVALID_ARG, "q_chunk/k_cache/v_cache/out must be 16-byte aligned, start_pos 8-byte aligned");
  if (B < 1 || B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, B);
  if (T < 1 || (int64_t)T > h->cfg.max_ctx)
    return fail(SPA_ERR_INVALID_ARG, "T must be in [1, max_ctx] (got %d)", T);
  if (n_sink < 0 || window < 0 || (int64_t)n_sink + window < 1)
    return fail(SPA_ERR_INVALID_ARG, "n_sink, window must be >= 0 with n_sink + window >= 1");
  unsigned char is_ret[spa::kMaxKvHeads];
  for (int g = 0; g < h->cfg.n_kv_heads; ++g) is_ret[g] = head_mask[g] ? 1 : 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return run(h, SPA_K_PREFILL, st, "prefill", [&] {
    return spa::launch_prefill_tc(q_chunk, k_cache, v_cache, out, start_pos, B, T, h->cfg.n_q_heads,
                               h->cfg.n_kv_heads, h->cfg.max_ctx, n_sink, window, is_ret, h->ws.inv_freq,
                               h->ws.dev_err, st);
  });
}

spa_status spa_cp_exchange_sizes(spa_handle h, int B, int n_ranks, const uint8_t* head_mask, size_t* bytes) {
  if (!h || !head_mask || !bytes) return fail(SPA_ERR_INVALID_ARG, "NULL argument");
  if (B < 1 || B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, B);
  if (n_ranks < 1 || n_ranks > kMaxRanks) return fail(SPA_ERR_INVALID_ARG, "n_ranks must be in [1, %d]", kMaxRanks);
  // histogram and statistics rows for the retrieval slices only; hist1 and hist2 are
  // summed over the ranks (no slot per rank)
  const size_t xrows = (size_t)B * count_retrieval(h, head_mask), rows = (size_t)B * h->cfg.n_q_heads;
  bytes[0] = (size_t)n_ranks * xrows * h->n_chunks_max * h->G * sizeof(float2);
  bytes[1] = xrows * spa::kBins1 * 8;
  bytes[2] = xrows * spa::kBins2 * 8;
  bytes[3] = (size_t)n_ranks * xrows * spa::kBins3 * 16;
  bytes[4] = (size_t)n_ranks * rows * spa::kHeadDim * 4;
  bytes[5] = (size_t)n_ranks * rows * 4;
  return SPA_OK;
}

spa_status spa_cp_phase(spa_handle h, int phase, const spa_cp_args* a, spa_stream stream) {
  spa::CpParams C;
  spa_status r = cp_check(h, a, &C);
  if (r) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (phase) {
    case SPA_CP_STATS:
      return run(h, SPA_K_CP_SELECT, st, "cp stats", [&] { return spa::launch_cp_stats(C, st); });
    case SPA_CP_MASS:   // (the stats phase cleared this rank's hist1 rows)
      return run(h, SPA_K_CP_SELECT, st, "cp mass", [&] { return spa::launch_cp_mass(C, st); });
    case SPA_CP_ROUND2:   // cut 1 + round 2 (the mass phase cleared this rank's hist2 and hist3 rows)
      return run(h, SPA_K_CP_SELECT, st, "cp round 2", [&] { return spa::launch_cp_hist(C, 2, st); });
    case SPA_CP_ROUND3:   // cut 2 + round 3
      return run(h, SPA_K_CP_SELECT, st, "cp round 3", [&] { return spa::launch_cp_hist(C, 3, st); });
    case SPA_CP_ATTEND:   // cut 3 + list count, list, attention
      if ((r = run(h, SPA_K_CP_SELECT, st, "cp list count", [&] { return spa::launch_cp_list(C, 0, st); }))) return r;
      if ((r = run(h, SPA_K_CP_SELECT, st, "cp list", [&] { return spa::launch_cp_list(C, 1, st); }))) return r;
      return cp_attend(h, a, C, st);
  }
  return fail(SPA_ERR_INVALID_ARG, "phase must be SPA_CP_STATS .. SPA_CP_ATTEND (got %d)", phase);
}

spa_status spa_cp_combine(spa_handle h, const float* out_all, const float* lse_all, int n_ranks, int B, float* out,
                          spa_stream stream) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (!out_all || !lse_all || !out) return fail(SPA_ERR_INVALID_ARG, "out_all, lse_all and out must be non-NULL");
  if (!aligned16(out_all) || !aligned16(lse_all) || !aligned16(out))
    return fail(SPA_ERR_INVALID_ARG, "out_all, lse_all and out must be 16-byte aligned");
  if (B < 1 || B > h->cfg.max_batch)
    return fail(SPA_ERR_INVALID_ARG, "B must be in [1, max_batch=%d] (got %d)", h->cfg.max_batch, B);
  if (n_ranks < 1 || n_ranks > kMaxRanks) return fail(SPA_ERR_INVALID_ARG, "n_ranks must be in [1, %d]", kMaxRanks);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int rows = B * h->cfg.n_q_heads;
  return run(h, SPA_K_COMBINE, st, "cp combine",
             [&] { return spa::launch_cp_combine(out_all, lse_all, n_ranks, rows, out, st); });
}

spa_status spa_debug_drop_publish(spa_handle h, int enable) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  h->drop_publish = enable ? 1 : 0;
  return SPA_OK;
}

spa_status spa_device_status(spa_handle h, spa_stream stream) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned flags = 0;
  if ((e = cudaMemcpy(&flags, h->ws.dev_err, 4, cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e, "read status");
  if (flags) {
    if ((e = cudaMemset(h->ws.dev_err, 0, 4)) != cudaSuccess) return cuda_fail(e, "clear status");
    if (flags & spa::kErrTimeout) {
      // a wait that gave up may have left arrival counters or attention tickets mid-way:
      // start the next call from clean ones (the prologue kernel also clears the counters)
      cudaMemset(h->ws.attn_ticket, 0, sizeof(unsigned) * (size_t)h->cfg.max_batch * h->cfg.n_kv_heads);
      cudaMemset(h->ws.st, 0, sizeof(spa::SliceState) * (size_t)h->cfg.max_batch * h->cfg.n_kv_heads);
      cudaDeviceSynchronize();
      return fail(SPA_ERR_DEVICE_TIMEOUT, "a bounded device-side wait gave up (flags 0x%x)", flags);
    }
    if (flags & spa::kErrInternal)
      return fail(SPA_ERR_CUDA, "internal consistency check failed in the selection kernels (flags 0x%x)", flags);
    return fail(SPA_ERR_DEVICE_RANGE, "device range check failed:%s%s",
                (flags & spa::kErrSeqLen) ? " seq_lens outside [1, max_seq_len]" : "",
                (flags & spa::kErrStartPos) ? " start_pos + t outside [0, max_ctx)" : "");
  }
  return SPA_OK;
}

spa_status spa_set_profiling(spa_handle h, unsigned kernel_mask) {
  if (!h) return fail(SPA_ERR_INVALID_ARG, "handle is NULL");
  if (kernel_mask && h->ev.empty()) {
    h->ev.resize(2 * kEventPairs);
    h->ev_kid.resize(kEventPairs);
    for (auto& ev : h->ev) {
      cudaError_t e = cudaEventCreate(&ev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
    }
  }
  h->prof_mask = kernel_mask;
  h->ev_next = 0;
  return SPA_OK;
}

spa_status spa_profile_read(spa_handle h, int kernel_id, double* total_ms, int64_t* launches) {
  if (!h || !total_ms || !launches) return fail(SPA_ERR_INVALID_ARG, "NULL argument");
  double sum = 0.0;
  int64_t n = 0;
  for (size_t i = 0; i < h->ev_next; ++i) {
    if (h->ev_kid[i] != kernel_id) continue;
    cudaError_t e = cudaEventSynchronize(h->ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, h->ev[2 * i], h->ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    sum += ms;
    ++n;
  }
  *total_ms = sum;
  *launches = n;
  return SPA_OK;
}

const char* spa_kernel_name(int kernel_id) {
  static const char* names[SPA_K_COUNT] = {"index_append", "select", "attend", "combine", "kv_append", "prefill",
                                            "cp_select"};
  return (kernel_id >= 0 && kernel_id < SPA_K_COUNT) ? names[kernel_id] : "";
}

spa_status spa_launch_count(spa_handle h, int64_t* launches) {
  if (!h || !launches) return fail(SPA_ERR_INVALID_ARG, "NULL argument");
  *launches = h->launches;
  return SPA_OK;
}

}  // extern "C"
