// Internal definitions shared by the libspa kernels and the host entry points.
// Not part of the public ABI (see include/spa.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spa {

constexpr int kHeadDim = 128;          // d
constexpr int kIdxDim = 16;            // r, the index dimension
constexpr int kMaxKvHeads = 64;
constexpr int kMaxGroup = 8;           // largest GQA group size G
constexpr int64_t kMaxCtx = int64_t(1) << 24;

// Selection works on chunks of kChunk consecutive tokens of one (b, kv head) slice.
constexpr int kChunk = 4096;
constexpr int kSelThreads = 512;   // threads of a selection CTA (2 CTAs per SM)
constexpr int kMaxChunks = int(kMaxCtx / kChunk);    // 4096
// Block-granular selection ranks blocks of kBlock consecutive positions of a slice.
constexpr int kBlock = 64;

// Radix digits of the fp32 bit pattern u of a probability in [0, 1]:
// bits 31..30 are zero, digit1 = u >> 18 (12 bits), digit2 = (u >> 6) & 0xfff
// (12 bits), digit3 = u & 0x3f (6 bits).
constexpr int kBins1 = 4096;
constexpr int kBins2 = 4096;
constexpr int kBins3 = 64;
// Masses are integers in units of 2^-63 (see mass_q): exact below 2^64 for any sum of
// probabilities that add up to at most 1 (plus fp32 rounding).
constexpr int kMassMinExp = 87;

// Largest grid of the selection kernel (sizes the per-range statistics, counts and
// offsets, and the per-range table of the per-slice refine step in shared memory).
constexpr int kMaxSelectGrid = 1024;
// Largest grid of the attention kernels (the bf16 kernel writes one split state per
// (CTA, slice) it touches: at most grid + slices of them).
constexpr int kMaxAttendCtas = 1024;

// Attention splits ("items") cover up to split_rows rows of one slice; rows are
// staged through shared memory kTile rows at a time.
constexpr int kTile = 64;
constexpr int kAttnThreads = 256;
constexpr int kDefaultSplitRows = 1024;
// One split's state per head: acc[128], m, l, 2 floats of padding (16-byte rows).
constexpr int kPartStride = kHeadDim + 4;

// Device status bits.
constexpr unsigned kErrSeqLen = 1u;
constexpr unsigned kErrStartPos = 2u;
constexpr unsigned kErrInternal = 4u;
constexpr unsigned kErrTimeout = 8u;   // a bounded device-side wait gave up

// Per (b, kv head) selection state, reset for every call by the selection's prologue
// kernel.  The arrival counters take one arrival per CTA range of the slice after each
// phase of the selection kernel; count is read by attention.
struct __align__(16) SliceState {
  unsigned long long target;    // cut target: ceil(p * total mass), or k for top-k
  unsigned long long m_above;   // mass of all tokens in round-1 bins above b1
  int b1;                       // round-1 bin holding the cut; -1 = keep everything
  int count;                    // listed tokens (kept, outside sinks/window)
  unsigned arr_score;           // ranges whose score statistics are stored
  unsigned arr_mass;            // ranges whose round-1 masses are added
  unsigned arr_thr;             // ranges whose candidates and counts above b1 are stored
  unsigned ncand;               // candidates of the round-1 cut bin (slots taken)
};

// Cut state of one (b, kv head) slice in a context-parallel step (each rank holds a
// contiguous run of the slice's positions).  Written by the cuts (chunk 0 of the slice
// in the launch that takes them), read by the histogram and list kernels of the
// following phases.
struct __align__(16) CpSlice {
  unsigned long long target;   // ceil(p * total mass), total over every rank
  unsigned long long above;    // mass of all tokens strictly above bin b1
  unsigned long long above2;   // mass of all tokens strictly above the prefix (b1, b2)
  int b1, b2;                  // round-1 / round-2 bins; b1 = -1 keeps every token
  unsigned tau;                // fp32 bits of the cut probability (after round 3)
  int quota;                   // tokens at tau this rank keeps (its lowest positions first)
};

// Arguments of the context-parallel kernels of one phase on one rank.
struct CpParams {
  const void* q_pre;              // [B][Hq][128] bf16, identical on every rank
  const uint16_t* idx;            // local index rows [Bm][Hkv][C][16]
  const int64_t* seq_lens;        // [B] global sequence lengths
  int B, Hq, Hkv, G, n_slices;
  int n_xrows;                    // exchange rows per rank: B * (retrieval KV heads)
  int n_ret;                      // retrieval KV heads
  signed char ret_ord[kMaxKvHeads];   // ordinal of KV head g among the retrieval heads (-1: streaming)
  int64_t C;                      // local row capacity (row stride of the local caches)
  int n_chunks;                   // ceil(C / kChunk): chunks of a slice's local rows
  int64_t pos0;                   // global position of local row 0
  int rank, n_ranks;
  int Lcap;                       // largest global sequence length accepted
  float p;
  int keep_all;                   // p >= 1
  int n_sink, window;
  float idx_scale_log2;
  unsigned char is_ret[kMaxKvHeads];
  const float* P_q;               // [Hq][16][128]
  const double* inv_freq_pi;      // [64] RoPE inverse frequencies / pi
  float* q_rot;                   // [Bm][Hq][128]
  float* q_idx;                   // [Bm][Hq][16]
  float* pi;                      // [Bm*Hkv][pi_stride] local probabilities
  int64_t pi_stride;
  // Exchange buffers: rows for the retrieval slices only (row b * n_ret + ret_ord[g]);
  // streaming slices never write or read them.  Gathered buffers have a slot per rank
  // (row r * n_xrows + ...); summed ones (all-reduced between the launches) do not.
  float2* stats;                  // gathered: [R][n_xrows][n_chunks][G] (m in log2 units, z)
  unsigned long long* hist1;      // summed: [n_xrows][kBins1] masses
  unsigned long long* hist2;      // summed: [n_xrows][kBins2] masses
  unsigned long long* hist3;      // gathered: [R][n_xrows][kBins3][2] (mass, count)
  unsigned* tab3;                 // [n_slices][n_chunks][kBins3] local round-3 counts per chunk
  int* chunk_cnt;                 // [n_slices][n_chunks] listed rows per chunk
  CpSlice* cs;                    // [n_slices]
  int* list;                      // [n_slices][C] listed local rows, ascending
  SliceState* st;                 // .count: listed rows of the slice (read by attention)
  int* sel_count;                 // optional [n_slices]
  float* out_rank;                // this rank's attention output slot [B][Hq][128]
  float* lse_rank;                // [B][Hq] log2-sum-exp of the rank's scores
  unsigned* err;
};

__host__ __device__ inline int64_t pi_row_stride(int64_t Lmax) { return (Lmax + 63) / 64 * 64; }

// Device workspace carved out of one allocation.
struct Workspace {
  float* P_q;            // [Hq][16][128]
  float* P_k;            // [Hkv][16][128]
  double* inv_freq;      // [64] RoPE inverse frequencies divided by pi
  float* q_rot;          // [Bm][Hq][128]
  float* q_idx;          // [Bm][Hq][16]
  float2* stats;         // [kMaxSelectGrid + Bm*Hkv][G] per-range (m in log2 units, z)
  float* pi;             // [Bm*Hkv][pi_stride]
  int64_t pi_stride;     // Lmax rounded up to 64 floats (256-byte rows)
  unsigned long long* hist1;  // [Bm*Hkv][kBins1]
  unsigned long long* hist2;  // [Bm*Hkv][kBins2] round-2 masses of the round-1 cut bin
  uint2* cand;           // [Bm*Hkv][Lmax]  (prob bits, position)
  int* chunk_gt;         // [Bm*Hkv][n_chunks_max]
  SliceState* st;        // [Bm*Hkv]
  int* list;             // [Bm*Hkv][Lmax]  selected positions (decode)
  int* item_base;        // [Bm*Hkv + 1]
  unsigned* attn_ticket; // [Bm*Hkv] pieces of each slice finished (bf16 attention; reset by its combiner)
  float* part;           // [max(max_items, kMaxAttendCtas + Bm*Hkv + 1)][G][kPartStride]
  int* seg_cnt;          // [kMaxSelectGrid + Bm*Hkv] per-range listed tokens above the cut bin
  unsigned* dev_err;     // [1]
  int64_t max_items;
};

// Arguments common to the selection / attention kernels of one call.
struct StepParams {
  const void* q_pre;
  const void* k_cache;
  const void* v_cache;
  const uint16_t* idx_cache;
  const int64_t* seq_lens;
  float* out;
  int* sel_list;         // [B*Hkv][Lmax] output list (workspace or caller's)
  int* sel_count;        // [B*Hkv] or null
  int B, Hq, Hkv, G;
  int64_t Lmax;          // cache row capacity (row stride of the caches)
  int Lcap;              // max_seq_len of this call
  int n_chunks;          // ceil(Lcap / kChunk)
  int n_slices;          // B * Hkv
  float p;
  int keep_all;          // p >= 1
  int64_t topk;          // > 0: keep the topk highest-probability tokens instead of top-p
  int blocks;            // 1: top-p over kBlock-token blocks, whole blocks kept
  int n_sink, window;
  float idx_scale_log2;  // idx_scale * log2(e)
  float attn_scale_log2; // log2(e) / sqrt(128)
  int split_rows;
  int n_ret;
  int ret_heads[kMaxKvHeads];
  unsigned char is_ret[kMaxKvHeads];
  // compact KV layout (0: every head keeps [Bm][Hkv][Lmax] rows, index rows likewise)
  int compact;
  int n_str;             // streaming heads (Hkv - n_ret)
  int ring;              // ring rows per streaming head: n_sink + window
  int head_rank[kMaxKvHeads];   // rank of head g among the retrieval or the streaming heads
  int drop_publish;      // failure-detection test hook: selection CTA 0 never arrives at its slice's counters
  int b_base;            // selection launches: first sequence of this launch's part of the batch
  const void* k_ring;    // [Bm][n_str][ring][128] streaming-head keys (compact layout)
  const void* v_ring;
  float* lse;            // optional [B][Hq]: log2-sum-exp of each head's attended scores
  Workspace ws;
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ int load_len(const int64_t* seq_lens, int b, int Lcap, unsigned* err) {
  int64_t L = seq_lens[b];
  if (L < 1 || L > Lcap) {
    atomicOr(err, kErrSeqLen);
    L = L < 1 ? 1 : Lcap;
  }
  return int(L);
}

// Sinks are [0, n_s); the window is [w_lo, L).  w_lo >= n_s so the two never overlap.
struct SinkWindow {
  int n_s, w_lo, L;
  __device__ __forceinline__ SinkWindow(int L_, int n_sink, int window) : L(L_) {
    n_s = n_sink < L_ ? n_sink : L_;
    long long lo = (long long)L_ - (long long)window;
    w_lo = lo > n_s ? int(lo) : n_s;
  }
  __device__ __forceinline__ int n_contig() const { return n_s + (L - w_lo); }
  __device__ __forceinline__ bool always(int j) const { return j < n_s || j >= w_lo; }
  __device__ __forceinline__ int contig_pos(int v) const { return v < n_s ? v : w_lo + (v - n_s); }
};

// Compact KV layout.  Retrieval heads keep every position in [Bm][n_ret][Lmax][128]
// (rank r of the head among the retrieval heads, ascending head index); streaming heads
// keep only what they attend, in a ring [Bm][n_str][n_sink + window][128]: position t
// at row t for t < n_sink, else at row n_sink + (t - n_sink) mod window.  Index rows of
// the retrieval heads live in [Bm][n_ret][Lmax][16].
__device__ __forceinline__ int ring_row(int pos, int n_sink, int window) {
  return pos < n_sink || window <= 0 ? pos : n_sink + (pos - n_sink) % window;
}
// K and V rows of slice s = b * Hkv + g, and whether its positions go through the ring.
template <typename T>
struct KvSlice {
  const T* k;
  const T* v;
  bool ring;
};
template <typename T>
__device__ __forceinline__ KvSlice<T> kv_slice(const StepParams& P, int s) {
  KvSlice<T> r;
  if (!P.compact) {
    const size_t off = (size_t)s * P.Lmax * kHeadDim;
    r.k = (const T*)P.k_cache + off;
    r.v = (const T*)P.v_cache + off;
    r.ring = false;
    return r;
  }
  const int b = s / P.Hkv, g = s % P.Hkv, rk = P.head_rank[g];
  if (P.is_ret[g]) {
    const size_t off = ((size_t)b * P.n_ret + rk) * P.Lmax * kHeadDim;
    r.k = (const T*)P.k_cache + off;
    r.v = (const T*)P.v_cache + off;
    r.ring = false;
  } else {
    const size_t off = ((size_t)b * P.n_str + rk) * P.ring * kHeadDim;
    r.k = (const T*)P.k_ring + off;
    r.v = (const T*)P.v_ring + off;
    r.ring = true;
  }
  return r;
}
// Index rows of retrieval slice y = b * n_ret + r (slice s = b * Hkv + g).
__device__ __forceinline__ const uint16_t* idx_rows(const StepParams& P, int y, int s) {
  return P.idx_cache + (size_t)(P.compact ? y : s) * P.Lmax * kIdxDim;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T> struct Elem;
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float get(const __nv_bfloat16* p, int i) { return __bfloat162float(p[i]); }
};
template <> struct Elem<float> {
  static __device__ __forceinline__ float get(const float* p, int i) { return p[i]; }
};

// Quantised mass of a probability from its fp32 bit pattern u: the exact value in units
// of 2^-63, M * 2^(E - 87) for the 24-bit significand M and exponent field E >= 87
// (values >= 2^-40); smaller values count as 0.  Integer sums of these masses are exact,
// so every total is independent of the order of accumulation.  Probabilities are at most
// 1 plus fp32 rounding (E <= 127), so one mass is below 2^64.
__device__ __forceinline__ unsigned long long mass_q(unsigned u) {
  int e = (int)((u >> 23) & 0xffu);
  if (e < kMassMinExp) return 0ull;
  e = e > 127 ? 127 : e;
  return (unsigned long long)((u & 0x7fffffu) | 0x800000u) << (e - kMassMinExp);
}

// Total mass_q of n probabilities of round-1 bin d (u >> 18 == d: same exponent and top
// five significand bits) whose low 18 bits sum to s_low.  Equal to the sum of their
// mass_q, which lets the per-chunk histograms count with 32-bit shared-memory atomics.
__device__ __forceinline__ unsigned long long bin1_mass(unsigned d, unsigned n, unsigned long long s_low) {
  int e = (int)(d >> 5);
  if (e < kMassMinExp || n == 0u) return 0ull;
  e = e > 127 ? 127 : e;
  const unsigned long long base = (unsigned long long)(32u | (d & 31u)) << 18;
  return (base * n + s_low) << (e - kMassMinExp);
}

// Merge two online-softmax states (m in log2 units).
__device__ __forceinline__ void merge_mz(float& m, float& z, float m2, float z2) {
  float mn = fmaxf(m, m2);
  if (mn == -INFINITY) { m = mn; z = 0.f; return; }
  z = z * exp2f(m - mn) + z2 * exp2f(m2 - mn);
  m = mn;
}

}  // namespace spa

// Launchers (defined in the kernel translation units).
namespace spa {
// Heads an append writes, with their destination slot (compact layout: rank).
struct HeadMap {
  int n;                    // heads written
  int g[kMaxKvHeads];       // source head
  int slot[kMaxKvHeads];    // destination head slot
  int n_slots;              // head slots per sequence in the destination
};
cudaError_t launch_index_append(const void* k_pre, const int64_t* start_pos, int B, int T, int Hkv,
                                int64_t Lmax, int kv_dtype, const float* P_k, uint16_t* idx_cache,
                                unsigned* dev_err, cudaStream_t st, const HeadMap* map = nullptr);
cudaError_t launch_kv_append_compact(const void* k_new, const void* v_new, const int64_t* start_pos, int B, int T,
                                     int Hkv, int64_t Lmax, int kv_dtype, const unsigned char* is_ret,
                                     const int* head_rank, int n_ret, int n_str, int n_sink, int window, void* k_ret,
                                     void* v_ret, void* k_ring, void* v_ring, unsigned* dev_err, cudaStream_t st);
// Selection of every slice of P (prologue + selection kernel).  Batches whose retrieval
// slices outnumber max_resident co-resident CTAs run as several launch pairs, each over
// as many whole sequences as fit.
cudaError_t launch_select(const StepParams& P, int kv_dtype, int max_resident, cudaStream_t st);
int select_grid(const StepParams& P, int max_resident);
int select_resident_per_sm(int kv_dtype, int G);
cudaError_t launch_attend(const StepParams& P, int kv_dtype, int grid, cudaStream_t st);
cudaError_t launch_combine(const StepParams& P, cudaStream_t st);
int attend_setup(int kv_dtype, int G, int max_slices);
cudaError_t launch_attend_bf16(const StepParams& P, int grid, cudaStream_t st);
int attend_bf16_setup(int G, int max_slices);
int set_last_error(int code, const char* msg);
size_t head_rank_workspace_bytes(int Hq, int Hkv);
cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, float* out, const int64_t* start, int B,
                              int T, int Hq, int Hkv, int64_t Lmax, int n_sink, int window,
                              const unsigned char* is_ret, const double* inv_freq_pi, unsigned* err, cudaStream_t st);
// Context-parallel phases (k_cp.cu).
cudaError_t launch_cp_stats(const CpParams& P, cudaStream_t st);
cudaError_t launch_cp_mass(const CpParams& P, cudaStream_t st);
cudaError_t launch_cp_hist(const CpParams& P, int round, cudaStream_t st);
cudaError_t launch_cp_list(const CpParams& P, int pass, cudaStream_t st);
cudaError_t launch_cp_combine(const float* out_all, const float* lse_all, int n_ranks, int rows, float* out,
                              cudaStream_t st);
cudaError_t launch_head_ranks(const float* W_Q, const float* W_K, int Hq, int Hkv, int d_model, int n_ret,
                              void* ws, double* er_q, double* er_kv, unsigned char* mask, double* sigma,
                              int* sweeps, cudaStream_t st);
}  // namespace spa
