// Context-parallel decode: the positions of every sequence are split over ranks (rank r
// holds the contiguous run [pos0, pos0 + C) in its own caches), and one decode step runs
// as phases of local launches with a small exchange between them.
//
// What is computed is the selection and attention of the one-GPU step:
//   "Full Attention Strikes Back" (RTPurbo summary), Methodology §2 (index scores in a
//   16-dim pre-RoPE subspace), §3 (dynamic top-p over the index attention mass), §5
//   (sort-free histogram thresholding); group mean of per-head probabilities as in the
//   "Autonomy of Heads" summary, Deployment strategy.  The split over the context follows
//   the context-parallel scaling of the "Lighthouse Attention" summary, Experimental
//   results (1M tokens on 32 GPUs).
//
// Phases (per rank; after each one an exchange: an all-gather of the rank's slot of
// stats, hist3 and the outputs, an all-reduce (sum) of hist1 and hist2; the histogram
// rows a phase adds into were cleared by an earlier phase of the same rank):
//   stats   q_rot = RoPE(q_pre, L-1); q_idx = P_q q_pre (float64 dots); per chunk of
//           local rows and head h: m = max_j l_hj, z = sum_j 2^(l_hj - m),
//           l_hj = log2(e) idx_scale <q_idx[h], idx_j>                    -> stats[rank]
//   mass    every rank merges all ranks' (m, z) in the same order -> (M_h, Z_h);
//           pi_j = sum_h 2^(l_hj - M_h) / (G Z_h) (fp32, kept locally); masses of the
//           round-1 digit (bits 31..18 of pi's pattern)                  -> hist1 (summed)
//   round 2 cut 1 over the summed round-1 histogram (target ceil(p * total)); masses
//           of the round-2 digit (bits 17..6) of the tokens in the cut bin -> hist2 (summed)
//   round 3 cut 2; masses and counts of the round-3 digit (bits 5..0)   -> hist3[rank]
//   attend  cut 3 -> tau; the tokens at tau that the selection still needs are taken
//           from the lowest positions first, i.e. rank by rank (their counts are in
//           hist3); the rank lists its kept rows (top-p set, sinks, window), attends
//           them and writes (out, log2-sum-exp)                      -> out[rank], lse[rank]
//   combine out = sum_r 2^(lse_r - M) out_r / sum_r 2^(lse_r - M).
// The exchange buffers hold one row per retrieval slice (xrow below): streaming heads
// never select, so they neither write nor read statistics or histograms.
// Masses are integers in units of 2^-63 (mass_q), so the summed histograms are exact
// whatever the order of the additions, and every rank takes the same cut decisions.
// The round-3 counts stay per rank: the tie quota hands ties out rank by rank.  Each cut is taken
// at the start of the launch that needs it, by every CTA of the slice (the summed
// histogram is a few KB to 32 KB per rank), so a rank's step is seven launches: stats,
// mass, round 2, round 3, list count, list, attention.  The kernels never wait on
// another launch or rank: the exchanges happen between launches.
#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kRun = kChunk / kThreads;   // 16 consecutive rows per thread in the list passes
// The two passes over the index rows run 512 threads per chunk, each with all of its
// 8 rows in flight at once (the passes are bound by memory latency, not bandwidth).
constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowsPer = kChunk / kRowThreads;   // 8

// 2^x with the hardware approximation (relative error about 2^-22; 2^-inf = 0), used by
// both passes over the index rows so that the sums and the probabilities agree.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ long long local_rows(const CpParams& P, int L) {
  long long n = (long long)L - P.pos0;
  return n < 0 ? 0 : (n > P.C ? P.C : n);
}

// Exchange row of retrieval slice s = (b, g): the exchange buffers hold the retrieval
// slices only, sequence-major.  xslot is the row of a summed buffer (hist1, hist2),
// xrow the row in rank r's slot of a gathered one (stats, hist3).
__device__ __forceinline__ size_t xslot(const CpParams& P, int s) {
  return (size_t)(s / P.Hkv) * P.n_ret + P.ret_ord[s % P.Hkv];
}
__device__ __forceinline__ size_t xrow(const CpParams& P, int r, int s) { return (size_t)r * P.n_xrows + xslot(P, s); }

// Length of sequence b, validated as in the one-GPU step; shared through *sh.
__device__ __forceinline__ int cta_len(const CpParams& P, int b, int* sh) {
  if (threadIdx.x == 0) {
    int64_t L = P.seq_lens[b];
    if (L < 1 || L > P.Lcap) {
      atomicOr(P.err, kErrSeqLen);
      L = L < 1 ? 1 : P.Lcap;
    }
    *sh = (int)L;
  }
  __syncthreads();
  return *sh;
}

// Exclusive prefix sum over the CTA in thread order; *total gets the sum.  Ends with a
// CTA barrier (scratch reusable afterwards).
template <typename T>
__device__ T block_excl_scan(T v, T* scratch, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  T before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarpsPerCta; ++w) {
    const T t = scratch[w];
    if (w < warp) before += t;
    all += t;
  }
  __syncthreads();
  *total = all;
  return before + x - v;
}

// Sum over the CTA (every thread gets it).
template <typename T>
__device__ T block_sum(T v, T* scratch) {
  T total;
  block_excl_scan<T>(v, scratch, &total);
  return total;
}

// ------------------------------------------------------------------ query prologue
// RoPE (rotate-half) of the G query heads of slice (b, g) at position L-1; the angle is
// carried in units of pi in float64 and reduced exactly modulo 2 before sincospi.
template <int G>
__device__ void rope_heads(const CpParams& P, const __nv_bfloat16* q, int b, int g, int L, double* cs, double* sn) {
  const int tid = threadIdx.x;
  if (tid < kHeadDim / 2) {
    const double t = (double)(L - 1) * P.inv_freq_pi[tid];
    const double r = t - 2.0 * rint(0.5 * t);
    sincospi(r, &sn[tid], &cs[tid]);
  }
  __syncthreads();
  for (int t = tid; t < G * (kHeadDim / 2); t += blockDim.x) {
    const int h = t / (kHeadDim / 2), i = t % (kHeadDim / 2);
    const double x1 = __bfloat162float(q[h * kHeadDim + i]);
    const double x2 = __bfloat162float(q[h * kHeadDim + i + kHeadDim / 2]);
    float* o = P.q_rot + ((size_t)b * P.Hq + (size_t)g * G + h) * kHeadDim;
    o[i] = (float)(x1 * cs[i] - x2 * sn[i]);
    o[i + kHeadDim / 2] = (float)(x2 * cs[i] + x1 * sn[i]);
  }
}

// q_idx[h] = P_q[g G + h] q_pre[h] for the G heads: output o = h * 16 + k is summed by
// four threads over 32 dims each in order (float64) and the quarters are added
// pairwise.  Every CTA runs the same code on the same data, so every CTA (and rank)
// gets the same bits.
template <int G>
__device__ void qidx_heads(const CpParams& P, const __nv_bfloat16* q, int g, float* qsm) {
  const int tid = threadIdx.x;
  for (int w = tid; w < G * kIdxDim * 4; w += blockDim.x) {   // whole warps (G * 64 = 64k)
    const int o = w >> 2, qd = w & 3, h = o / kIdxDim;
    const float4* prow = reinterpret_cast<const float4*>(P.P_q + ((size_t)g * G * kIdxDim + o) * kHeadDim + 32 * qd);
    const uint4* qrow = reinterpret_cast<const uint4*>(q + h * kHeadDim + 32 * qd);
    float4 pv[8];
    uint4 qw[4];
#pragma unroll
    for (int k = 0; k < 8; ++k) pv[k] = __ldg(prow + k);
#pragma unroll
    for (int k = 0; k < 4; ++k) qw[k] = __ldg(qrow + k);
    double acc = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 w4 = qw[k >> 1];
      const uint32_t wa = (k & 1) ? w4.z : w4.x, wb = (k & 1) ? w4.w : w4.y;
      acc += (double)pv[k].x * (double)bf16_lo(wa);
      acc += (double)pv[k].y * (double)bf16_hi(wa);
      acc += (double)pv[k].z * (double)bf16_lo(wb);
      acc += (double)pv[k].w * (double)bf16_hi(wb);
    }
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    if (qd == 0) qsm[o] = (float)acc;
  }
  __syncthreads();
}

// Log2-domain index logits of one row for the G heads.
template <int G>
__device__ __forceinline__ void row_logits(const uint4& a, const uint4& c, const float* qsm, float scale, float* l) {
  float x[16];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16_lo(w[i]);
    x[2 * i + 1] = bf16_hi(w[i]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) d = fmaf(qsm[h * kIdxDim + i], x[i], d);
    l[h] = d * scale;
  }
}

// ------------------------------------------------------------------ phase: stats
// Loads a thread's kRowsPer index rows of chunk c (row j0 + u * kRowThreads + tid).
__device__ __forceinline__ void load_rows(const uint16_t* rows, long long j0, long long n, uint4 (&ra)[kRowsPer],
                                          uint4 (&rc)[kRowsPer], bool last_use) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int u = 0; u < kRowsPer; ++u) {
    const long long j = j0 + (long long)u * kRowThreads + tid;
    if (j < n) {
      const uint4* r = reinterpret_cast<const uint4*>(rows + (size_t)j * kIdxDim);
      if (last_use) {
        ra[u] = __ldcs(r);
        rc[u] = __ldcs(r + 1);
      } else {
        ra[u] = __ldg(r);
        rc[u] = __ldg(r + 1);
      }
    }
  }
}

// grid (n_chunks, n_slices), kRowThreads threads.  Chunk 0 of every slice (streaming
// ones included) writes q_rot; the chunks of retrieval slices write their (m, z) to
// stats[rank].  The rows are requested before the query prologue so that the two
// overlap; this pass keeps their lines in L2 for the mass pass.
template <int G>
__global__ void __launch_bounds__(kRowThreads) k_cp_stats(CpParams P) {
  __shared__ float qsm[G * kIdxDim];
  __shared__ double cs[kHeadDim / 2], sn[kHeadDim / 2];
  __shared__ float2 wred[kRowWarps][G];
  __shared__ int sh_len;
  const int c = blockIdx.x, s = blockIdx.y, b = s / P.Hkv, g = s % P.Hkv, tid = threadIdx.x;
  const long long j0 = (long long)c * kChunk;
  uint4 ra[kRowsPer], rc[kRowsPer];
  // rows are requested before the sequence length is known: every row below C lies in
  // the shard; rows at or past the local length are ignored below
  if (P.is_ret[g]) load_rows(P.idx + (size_t)s * P.C * kIdxDim, j0, P.C, ra, rc, false);
  const int L = cta_len(P, b, &sh_len);
  const __nv_bfloat16* q = (const __nv_bfloat16*)P.q_pre + ((size_t)b * P.Hq + (size_t)g * G) * kHeadDim;
  const long long n = P.is_ret[g] ? local_rows(P, L) : 0;
  if (c == 0) rope_heads<G>(P, q, b, g, L, cs, sn);
  if (!P.is_ret[g]) return;
  if (c == 0) {   // the slice's round-1 histogram row in this rank's buffer, filled by the next phase
    unsigned long long* h1 = P.hist1 + xslot(P, s) * kBins1;
    for (int i = tid; i < kBins1; i += kRowThreads) h1[i] = 0ull;
  }
  qidx_heads<G>(P, q, g, qsm);
  if (c == 0 && tid < G * kIdxDim) P.q_idx[((size_t)b * P.Hq + (size_t)g * G) * kIdxDim + tid] = qsm[tid];

  float m[G], z[G];
#pragma unroll
  for (int h = 0; h < G; ++h) { m[h] = -INFINITY; z[h] = 0.f; }
#pragma unroll
  for (int u = 0; u < kRowsPer; ++u) {
    const long long j = j0 + (long long)u * kRowThreads + tid;
    if (j < n) {
      float l[G];
      row_logits<G>(ra[u], rc[u], qsm, P.idx_scale_log2, l);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (l[h] > m[h]) { z[h] = z[h] * ex2(m[h] - l[h]) + 1.f; m[h] = l[h]; }
        else z[h] += ex2(l[h] - m[h]);
      }
    }
  }
  // merge over the warp (butterfly), then over the warps in order
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float m2 = __shfl_xor_sync(kFull, m[h], o), z2 = __shfl_xor_sync(kFull, z[h], o);
      merge_mz(m[h], z[h], m2, z2);
    }
  }
  if ((tid & 31) == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) wred[tid >> 5][h] = make_float2(m[h], z[h]);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY, Z = 0.f;
    for (int w = 0; w < kRowWarps; ++w) merge_mz(M, Z, wred[w][tid].x, wred[w][tid].y);
    P.stats[(xrow(P, P.rank, s) * P.n_chunks + c) * G + tid] = make_float2(M, Z);
  }
}

// ------------------------------------------------------------------ phase: mass
// grid (n_chunks, n_slices), kRowThreads threads, retrieval slices only.  Shared
// histogram of the round-1 digit as a count and a sum of the low 18 significand bits
// per bin (32-bit atomics); bin1_mass turns them into the exact mass.
template <int G>
__global__ void __launch_bounds__(kRowThreads) k_cp_mass(CpParams P) {
  __shared__ unsigned hc[kBins1], hl[kBins1];
  __shared__ float qsm[G * kIdxDim];
  __shared__ float2 wred[kRowWarps];
  __shared__ float Msm[G], Wsm[G];
  __shared__ int sh_len;
  const int c = blockIdx.x, s = blockIdx.y, b = s / P.Hkv, g = s % P.Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  if (!P.is_ret[g]) return;
  const long long j0 = (long long)c * kChunk;
  uint4 ra[kRowsPer], rc[kRowsPer];
  // second and last read of the rows (requested before the length is known, as above)
  load_rows(P.idx + (size_t)s * P.C * kIdxDim, j0, P.C, ra, rc, true);
  const int L = cta_len(P, b, &sh_len);
  const long long n = local_rows(P, L);
  for (int i = tid; i < kBins1; i += kRowThreads) { hc[i] = 0u; hl[i] = 0u; }
  if (c == 0) {   // the slice's round-2 row and the rank's round-3 row, filled by later phases
    unsigned long long* h2 = P.hist2 + xslot(P, s) * kBins2;
    unsigned long long* h3 = P.hist3 + xrow(P, P.rank, s) * kBins3 * 2;
    for (int i = tid; i < kBins2; i += kRowThreads) h2[i] = 0ull;
    if (tid < kBins3 * 2) h3[tid] = 0ull;
  }
  if (tid < G * kIdxDim) qsm[tid] = P.q_idx[((size_t)b * P.Hq + (size_t)g * G) * kIdxDim + tid];
  // (M_h, Z_h): warp w merges head w % G over entries w / G, w / G + kWph, ... (all
  // ranks' chunks in rank-major order), then the warps of a head are merged in order.
  constexpr int kWph = kRowWarps / G;   // warps per head
  const int E = P.n_ranks * P.n_chunks;
  {
    const int h = warp % G, sub = warp / G;
    float m = -INFINITY, z = 0.f;
    for (int e = sub * 32 + lane; e < E; e += kWph * 32) {
      const int r = e / P.n_chunks, cc = e % P.n_chunks;
      const float2 v = P.stats[(xrow(P, r, s) * P.n_chunks + cc) * G + h];
      merge_mz(m, z, v.x, v.y);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float m2 = __shfl_xor_sync(kFull, m, o), z2 = __shfl_xor_sync(kFull, z, o);
      merge_mz(m, z, m2, z2);
    }
    if (lane == 0) wred[warp] = make_float2(m, z);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY, Z = 0.f;
    for (int k = 0; k < kWph; ++k) merge_mz(M, Z, wred[tid + G * k].x, wred[tid + G * k].y);
    Msm[tid] = M;
    Wsm[tid] = Z > 0.f ? 1.f / ((float)G * Z) : 0.f;
  }
  __syncthreads();

  float* pi = P.pi + (size_t)s * P.pi_stride;
  float Mh[G], Wh[G];
#pragma unroll
  for (int h = 0; h < G; ++h) { Mh[h] = Msm[h]; Wh[h] = Wsm[h]; }
#pragma unroll
  for (int u = 0; u < kRowsPer; ++u) {
    const long long j = j0 + (long long)u * kRowThreads + tid;
    if (j < n) {
      float l[G];
      row_logits<G>(ra[u], rc[u], qsm, P.idx_scale_log2, l);
      float v = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) v = fmaf(ex2(l[h] - Mh[h]), Wh[h], v);
      pi[j] = v;
      const unsigned bits = __float_as_uint(v);
      const unsigned d = min(bits >> 18, (unsigned)kBins1 - 1u);   // probabilities are <= 1: clamp is inert
      atomicAdd(&hc[d], 1u);
      atomicAdd(&hl[d], bits & 0x3ffffu);
    }
  }
  __syncthreads();
  unsigned long long* dst = P.hist1 + xslot(P, s) * kBins1;
  for (int d = tid; d < kBins1; d += kRowThreads) {
    const unsigned cnt = hc[d];
    if (cnt) {
      const unsigned long long ms = bin1_mass((unsigned)d, cnt, hl[d]);
      if (ms) atomicAdd(dst + d, ms);
    }
  }
}

// ------------------------------------------------------------------ cuts
// Shared-memory slot of bin d of a 4096-bin histogram: one pad word per 16 bins, so the
// 16 consecutive bins a thread scans in cut_desc do not share a bank with its neighbours'.
__device__ __forceinline__ int hslot(int d) { return d + (d >> 4); }
constexpr int kHistSlots = kBins1 + kBins1 / 16;

// Descending scan of NB bins h (shared memory, slot PAD ? hslot(d) : d): the bin d with
// above + mass(bins > d) < target <= above + mass(bins >= d).  Thread t owns bins
// NB-1-t*PER .. NB-PER-t*PER.  Result in *out_b / *out_above (untouched if target is
// never reached).  Ends with a CTA barrier.
template <int NB, bool PAD>
__device__ void cut_desc(const unsigned long long* h, unsigned long long above, unsigned long long target, int* out_b,
                         unsigned long long* out_above, unsigned long long* scratch) {
  constexpr int PER = NB >= kThreads ? NB / kThreads : 1;
  const int tid = threadIdx.x;
  const bool owns = tid * PER < NB;
  unsigned long long v[PER];
  unsigned long long mine = 0ull;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int d = NB - 1 - tid * PER - k;
    v[k] = owns ? h[PAD ? hslot(d) : d] : 0ull;
    mine += v[k];
  }
  unsigned long long total;
  const unsigned long long before = block_excl_scan<unsigned long long>(mine, scratch, &total);
  if (owns) {
    unsigned long long cum = above + before;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const unsigned long long nx = cum + v[k];
      if (cum < target && nx >= target) { *out_b = NB - 1 - tid * PER - k; *out_above = cum; }
      cum = nx;
    }
  }
  __syncthreads();
}

// Slice s's row of a summed [n_xrows][4096] histogram (every rank's masses added, by
// the all-reduce between the launches, or directly when emulated ranks share the
// buffer) into shared memory (padded slots); returns this thread's part of the total.
__device__ unsigned long long load_hist4096(const CpParams& P, const unsigned long long* hist, int s,
                                            unsigned long long* h) {
  constexpr int PER = kBins1 / kThreads;
  const int tid = threadIdx.x;
  const unsigned long long* src = hist + xslot(P, s) * kBins1 + tid;
  unsigned long long v[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) v[k] = __ldcg(src + k * kThreads);
  unsigned long long mine = 0ull;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    h[hslot(tid + k * kThreads)] = v[k];
    mine += v[k];
  }
  return mine;
}

// The cuts, taken at the start of the kernel that needs them by every CTA of the slice
// (the histograms were exchanged between the launches; every CTA reaches the same
// result from the same data).  Chunk 0 of the slice stores the cut state for the
// following phases.
//
// Cut 1: total mass and target from the summed round-1 histograms, then bin b1 (-1
// keeps every token).  h: kHistSlots words of shared memory.  Ends with a CTA barrier.
__device__ void cp_cut1(const CpParams& P, int s, bool store, unsigned long long* h, unsigned long long* scratch,
                        int* sb, unsigned long long* sabove, unsigned long long* starget) {
  const int tid = threadIdx.x;
  const unsigned long long mine = load_hist4096(P, P.hist1, s, h);
  const unsigned long long total = block_sum<unsigned long long>(mine, scratch);   // (barrier: h complete)
  unsigned long long target = (unsigned long long)ceil((double)P.p * (double)total);
  if (target < 1ull) target = 1ull;
  const bool keep = P.keep_all || target > total;
  if (tid == 0) { *sb = -1; *sabove = 0ull; *starget = target; }
  __syncthreads();
  if (!keep) cut_desc<kBins1, true>(h, 0ull, target, sb, sabove, scratch);
  if (store && tid == 0) {
    CpSlice* cs = P.cs + s;
    cs->target = target;
    cs->above = *sabove;
    cs->b1 = *sb;
    cs->b2 = -1;
    cs->tau = 0u;
    cs->quota = 0;
  }
  __syncthreads();
}

// Cut 2 (b1 >= 0): bin b2 inside b1 from the summed round-2 histograms; *sabove enters
// as the mass above b1 and leaves as the mass above (b1, b2) (stored as above2, so the
// launch's other CTAs still read the round-1 value).  Ends with a CTA barrier.
__device__ void cp_cut2(const CpParams& P, int s, bool store, unsigned long long target, unsigned long long* h,
                        unsigned long long* scratch, int* sb, unsigned long long* sabove) {
  const int tid = threadIdx.x;
  const unsigned long long above = *sabove;
  load_hist4096(P, P.hist2, s, h);
  if (tid == 0) *sb = -1;
  __syncthreads();
  cut_desc<kBins2, true>(h, above, target, sb, sabove, scratch);
  if (tid == 0) {
    if (*sb < 0) { atomicOr(P.err, kErrInternal); *sb = 0; }
    if (store) {
      CpSlice* cs = P.cs + s;
      cs->b2 = *sb;
      cs->above2 = *sabove;
    }
  }
  __syncthreads();
}

// Cut 3 (b1 >= 0): bin b3, tau and this rank's quota of the tokens at tau (lowest
// positions first, i.e. rank by rank) from the round-3 histograms.  Ends with a CTA
// barrier; results in *stau and *squota.
__device__ void cp_cut3(const CpParams& P, int s, bool store, unsigned long long* h, unsigned long long* cnt3,
                        unsigned long long* scratch, int* sb, unsigned long long* sabove, unsigned* stau, int* squota) {
  const int tid = threadIdx.x;
  const CpSlice* cs = P.cs + s;
  const int b1 = __ldcg(&cs->b1), b2 = __ldcg(&cs->b2);
  const unsigned long long target = __ldcg(&cs->target), above = __ldcg(&cs->above2);
  const int R = P.n_ranks;
  if (tid < kBins3) {
    unsigned long long v = 0ull, k = 0ull;
    for (int r = 0; r < R; ++r) {
      const unsigned long long* e = P.hist3 + (xrow(P, r, s) * kBins3 + tid) * 2;
      v += __ldcg(e);
      k += __ldcg(e + 1);
    }
    h[tid] = v;
    cnt3[tid] = k;
  }
  if (tid == 0) { *sb = -1; *sabove = above; }
  __syncthreads();
  cut_desc<kBins3, false>(h, above, target, sb, sabove, scratch);
  if (tid == 0) {
    int b3 = *sb;
    if (b3 < 0) { atomicOr(P.err, kErrInternal); b3 = 0; }
    const unsigned tau = ((unsigned)b1 << 18) | ((unsigned)b2 << 6) | (unsigned)b3;
    // tokens at tau, lowest positions first, while the mass before them is below target
    const unsigned long long mt = mass_q(tau);
    const unsigned long long need = target > *sabove ? target - *sabove : 0ull;
    const unsigned long long ties = mt ? (need + mt - 1ull) / mt : cnt3[b3];
    unsigned long long before = 0ull;
    for (int r = 0; r < P.rank; ++r) before += __ldcg(P.hist3 + (xrow(P, r, s) * kBins3 + b3) * 2 + 1);
    const unsigned long long mine = __ldcg(P.hist3 + (xrow(P, P.rank, s) * kBins3 + b3) * 2 + 1);
    unsigned long long q = ties > before ? ties - before : 0ull;
    if (q > mine) q = mine;
    *stau = tau;
    *squota = (int)q;
    if (store) {
      CpSlice* w = P.cs + s;
      w->tau = tau;
      w->quota = (int)q;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ rounds 2 and 3
// grid (n_chunks, n_slices), retrieval slices.  Round 2: cut 1, then the masses of the
// round-2 digit of the tokens in bin b1.  Round 3: cut 2, then the masses and counts of
// the round-3 digit of the tokens in (b1, b2), plus this chunk's counts per digit
// (tab3).  Slices whose cut keeps every token stop after the cut.
__global__ void __launch_bounds__(kThreads) k_cp_hist(CpParams P, int round) {
  __shared__ unsigned long long hm[kHistSlots];   // the cut's summed histogram, then this chunk's masses
  __shared__ unsigned hn[kBins3];
  __shared__ unsigned long long scratch[kWarpsPerCta];
  __shared__ unsigned long long sabove, starget;
  __shared__ int sb, sh_len;
  const int c = blockIdx.x, s = blockIdx.y, b = s / P.Hkv, g = s % P.Hkv, tid = threadIdx.x;
  if (!P.is_ret[g]) return;
  const CpSlice* cs = P.cs + s;
  int b1, b2 = 0;
  if (round == 2) {
    cp_cut1(P, s, c == 0, hm, scratch, &sb, &sabove, &starget);
    b1 = sb;
  } else {
    b1 = __ldcg(&cs->b1);
    if (b1 >= 0) {
      if (tid == 0) sabove = __ldcg(&cs->above);
      __syncthreads();
      cp_cut2(P, s, c == 0, __ldcg(&cs->target), hm, scratch, &sb, &sabove);
      b2 = sb;
    }
  }
  const int L = cta_len(P, b, &sh_len);
  if (b1 < 0) return;
  const long long n = local_rows(P, L);
  const long long j0 = (long long)c * kChunk;
  const unsigned* pb = reinterpret_cast<const unsigned*>(P.pi + (size_t)s * P.pi_stride);
  const unsigned pre2 = (unsigned)b1, pre3 = ((unsigned)b1 << 12) | (unsigned)b2;
  bool any = false;
  constexpr int PER = kChunk / kThreads;
  unsigned uv[PER];   // all of the thread's probabilities in flight at once; ~0u never matches a prefix
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const long long j = j0 + (long long)k * kThreads + tid;
    uv[k] = j < n ? __ldcg(pb + j) : ~0u;
  }
  const int nb = round == 2 ? kBins2 : kBins3;
  for (int i = tid; i < nb; i += kThreads) hm[i] = 0ull;
  if (round == 3 && tid < kBins3) hn[tid] = 0u;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const unsigned u = uv[k];
    if (round == 2) {
      if ((u >> 18) == pre2) {
        atomicAdd(&hm[(u >> 6) & 0xfffu], mass_q(u));
        any = true;
      }
    } else if ((u >> 6) == pre3) {
      atomicAdd(&hm[u & 0x3fu], mass_q(u));
      atomicAdd(&hn[u & 0x3fu], 1u);
      any = true;
    }
  }
  const bool cta_any = __syncthreads_or(any);
  if (round == 3 && tid < kBins3) P.tab3[((size_t)s * P.n_chunks + c) * kBins3 + tid] = hn[tid];
  if (!cta_any) return;
  if (round == 2) {
    unsigned long long* dst = P.hist2 + xslot(P, s) * kBins2;
    for (int d = tid; d < kBins2; d += kThreads)
      if (hm[d]) atomicAdd(dst + d, hm[d]);
  } else if (tid < kBins3 && hn[tid]) {
    unsigned long long* e = P.hist3 + (xrow(P, P.rank, s) * kBins3 + tid) * 2;
    atomicAdd(e, hm[tid]);
    atomicAdd(e + 1, (unsigned long long)hn[tid]);
  }
}

// ------------------------------------------------------------------ the rank's list
// Which of the 16 consecutive local rows of thread t in chunk c are attended: sinks and
// window of the global positions, plus (retrieval slices) the top-p set: probability
// above tau, or at tau within the rank's quota counted from its lowest position.
// Returns the 16-bit mask; needs the CTA (block scans of the tied rows).
__device__ unsigned list_mask(const CpParams& P, int s, int c, int L, int b1, unsigned tau, int quota,
                              unsigned* uscratch) {
  const int g = s % P.Hkv, tid = threadIdx.x;
  const bool ret = P.is_ret[g] != 0;
  const long long n = local_rows(P, L);
  const long long r0 = (long long)c * kChunk + (long long)tid * kRun;
  // issue the loads first: the thread's 16 probabilities (r0 is a multiple of 16 rows:
  // four aligned 16-byte words), the earlier chunks' tie counts
  uint4 pw[kRun / 4];
  if (ret) {
    const uint4* pv = reinterpret_cast<const uint4*>(P.pi + (size_t)s * P.pi_stride + r0);
#pragma unroll
    for (int q4 = 0; q4 < kRun / 4; ++q4) pw[q4] = r0 < n ? __ldcg(pv + q4) : make_uint4(0u, 0u, 0u, 0u);
  }
  const SinkWindow sw(L, P.n_sink, P.window);
  unsigned mask = 0u;
#pragma unroll
  for (int k = 0; k < kRun; ++k) {
    const long long r = r0 + k;
    if (r < n && sw.always((int)(P.pos0 + r))) mask |= 1u << k;
  }
  if (!ret) return mask;
  if (b1 < 0) {   // keep everything local
#pragma unroll
    for (int k = 0; k < kRun; ++k)
      if (r0 + k < n) mask |= 1u << k;
    return mask;
  }
  const unsigned b3 = tau & 0x3fu;
  // tied rows of the earlier chunks of this slice (local to the rank)
  unsigned earlier = 0u;
  for (int cc = tid; cc < c; cc += kThreads) earlier += __ldcg(P.tab3 + ((size_t)s * P.n_chunks + cc) * kBins3 + b3);
  unsigned gt = 0u, eq = 0u;
#pragma unroll
  for (int q4 = 0; q4 < kRun / 4; ++q4) {
    const unsigned v[4] = {pw[q4].x, pw[q4].y, pw[q4].z, pw[q4].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = 4 * q4 + i;
      if (r0 + k < n) {
        if (v[i] > tau) gt |= 1u << k;
        else if (v[i] == tau) eq |= 1u << k;
      }
    }
  }
  earlier = block_sum<unsigned>(earlier, uscratch);
  unsigned n_eq_total;
  const unsigned before = earlier + block_excl_scan<unsigned>((unsigned)__popc(eq), uscratch, &n_eq_total);
  unsigned kept_eq = 0u, seen = before;
#pragma unroll
  for (int k = 0; k < kRun; ++k) {
    if ((eq >> k) & 1u) {
      if (seen < (unsigned)quota) kept_eq |= 1u << k;
      ++seen;
    }
  }
  return mask | gt | kept_eq;
}

// pass 0: cut 3 (retrieval slices with a cut; chunk 0 stores tau and the quota), then
// the listed rows per chunk.  pass 1: the rows themselves (ascending), the slice's
// count, and (empty slices) the rank's zero output with log2-sum-exp -inf.
__global__ void __launch_bounds__(kThreads) k_cp_list(CpParams P, int pass) {
  __shared__ unsigned uscratch[kWarpsPerCta];
  __shared__ unsigned long long h3[kBins3], c3[kBins3], scratch[kWarpsPerCta], sabove;
  __shared__ unsigned stau;
  __shared__ int sb, squota, sh_len;
  const int c = blockIdx.x, s = blockIdx.y, b = s / P.Hkv, g = s % P.Hkv, tid = threadIdx.x;
  int b1 = -1, quota = 0;
  unsigned tau = 0u;
  if (P.is_ret[g]) {
    b1 = __ldcg(&P.cs[s].b1);
    if (b1 >= 0) {
      if (pass == 0) {
        cp_cut3(P, s, c == 0, h3, c3, scratch, &sb, &sabove, &stau, &squota);
        tau = stau;
        quota = squota;
      } else {
        tau = __ldcg(&P.cs[s].tau);
        quota = __ldcg(&P.cs[s].quota);
      }
    }
  }
  const int L = cta_len(P, b, &sh_len);
  const unsigned mask = list_mask(P, s, c, L, b1, tau, quota, uscratch);
  unsigned n_chunk;
  const unsigned off = block_excl_scan<unsigned>((unsigned)__popc(mask), uscratch, &n_chunk);
  if (pass == 0) {
    if (tid == 0) P.chunk_cnt[(size_t)s * P.n_chunks + c] = (int)n_chunk;
    return;
  }
  unsigned base = 0u;
  for (int cc = tid; cc < c; cc += kThreads) base += (unsigned)__ldcg(P.chunk_cnt + (size_t)s * P.n_chunks + cc);
  base = block_sum<unsigned>(base, uscratch);
  int* out = P.list + (size_t)s * P.C + base + off;
  const long long r0 = (long long)c * kChunk + (long long)tid * kRun;
  int w = 0;
#pragma unroll
  for (int k = 0; k < kRun; ++k)
    if ((mask >> k) & 1u) out[w++] = (int)(r0 + k);
  if (c == P.n_chunks - 1 && tid == 0) {
    const int total = (int)(base + n_chunk);
    P.st[s].count = total;
    if (P.sel_count) P.sel_count[s] = total;
  }
  if (c == P.n_chunks - 1 && base + n_chunk == 0u) {
    const int g = s % P.Hkv;
    for (int i = tid; i < P.G * kHeadDim; i += kThreads)
      P.out_rank[((size_t)b * P.Hq + (size_t)g * P.G) * kHeadDim + i] = 0.f;
    if (tid < P.G) P.lse_rank[(size_t)b * P.Hq + (size_t)g * P.G + tid] = -INFINITY;
  }
}

// ------------------------------------------------------------------ combine over ranks
// One warp per query head; lane l holds dims 4l..4l+3; ranks merged in order.
__global__ void __launch_bounds__(32) k_cp_combine(const float* out_all, const float* lse_all, int n_ranks, int rows,
                                                   float* out) {
  const int row = blockIdx.x, lane = threadIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < n_ranks; ++r) M = fmaxf(M, lse_all[(size_t)r * rows + row]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (M != -INFINITY) {
    for (int r = 0; r < n_ranks; ++r) {
      const float lr = lse_all[(size_t)r * rows + row];
      if (lr == -INFINITY) continue;
      const float w = exp2f(lr - M);
      const float4 v = reinterpret_cast<const float4*>(out_all + ((size_t)r * rows + row) * kHeadDim)[lane];
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
      den += w;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  reinterpret_cast<float4*>(out + (size_t)row * kHeadDim)[lane] =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

}  // namespace

cudaError_t launch_cp_stats(const CpParams& P, cudaStream_t st) {
  const dim3 grid(P.n_chunks, P.n_slices);
  switch (P.G) {
    case 1: k_cp_stats<1><<<grid, kRowThreads, 0, st>>>(P); break;
    case 2: k_cp_stats<2><<<grid, kRowThreads, 0, st>>>(P); break;
    case 4: k_cp_stats<4><<<grid, kRowThreads, 0, st>>>(P); break;
    case 8: k_cp_stats<8><<<grid, kRowThreads, 0, st>>>(P); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_cp_mass(const CpParams& P, cudaStream_t st) {
  const dim3 grid(P.n_chunks, P.n_slices);
  switch (P.G) {
    case 1: k_cp_mass<1><<<grid, kRowThreads, 0, st>>>(P); break;
    case 2: k_cp_mass<2><<<grid, kRowThreads, 0, st>>>(P); break;
    case 4: k_cp_mass<4><<<grid, kRowThreads, 0, st>>>(P); break;
    case 8: k_cp_mass<8><<<grid, kRowThreads, 0, st>>>(P); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_cp_hist(const CpParams& P, int round, cudaStream_t st) {
  k_cp_hist<<<dim3(P.n_chunks, P.n_slices), kThreads, 0, st>>>(P, round);
  return cudaGetLastError();
}

cudaError_t launch_cp_list(const CpParams& P, int pass, cudaStream_t st) {
  k_cp_list<<<dim3(P.n_chunks, P.n_slices), kThreads, 0, st>>>(P, pass);
  return cudaGetLastError();
}

cudaError_t launch_cp_combine(const float* out_all, const float* lse_all, int n_ranks, int rows, float* out,
                              cudaStream_t st) {
  k_cp_combine<<<rows, 32, 0, st>>>(out_all, lse_all, n_ranks, rows, out);
  return cudaGetLastError();
}

}  // namespace spa
