// Query prologue and top-p token selection for the retrieval heads.
//
// "Full Attention Strikes Back" (RTPurbo summary):
//   Methodology §2  index scores in a 16-dim pre-RoPE subspace;
//   Methodology §3  dynamic top-p: accumulate index attention mass until p;
//   Methodology §5  sort-free, histogram-based thresholding.
// Group mean of per-head probabilities: "Autonomy of Heads" summary, Deployment
// strategy (GQA scores aggregated to the group by their mean).
//
// Pipeline for every retrieval slice s = (b, g), over chunks of kChunk tokens:
//   k_prologue   q_rot = RoPE(q_pre, L-1) (float64 angles), q_idx = P_q q_pre,
//                reset of the slice's selection state;
//   k_score      per chunk and head h: m = max_j l_hj, z = sum_j 2^(l_hj - m),
//                l_hj = log2(e) * idx_scale * <q_idx[h], idx_j>   (idx read #1);
//   k_mass       merge (m, z) over chunks -> M_h, Z_h; recompute l_hj (idx read #2),
//                pi_j = sum_h 2^(l_hj - M_h) / (G Z_h), stored as fp32; a mass
//                histogram over the top 12 bits of pi_j's bit pattern, with
//                masses quantised to integer multiples of 2^-60 so every sum is
//                exact and order independent.  The last CTA of the slice finds
//                the bin b1 where the descending cumulative mass reaches p;
//   k_threshold  counts tokens above b1 per chunk and appends the tokens of bin
//                b1 to a candidate list; the last CTA resolves the exact cut value
//                tau (two more radix rounds over the candidates), the tie quota
//                at tau (lowest positions first) and per-chunk output offsets;
//   k_compact    writes kept positions outside sinks/window, ascending.
// No kernel waits on another CTA: cross-CTA steps use kernel boundaries or a
// "last CTA to finish" ticket.
#include <climits>

#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------------ block scans
template <typename V>
__device__ __forceinline__ V warp_incl_scan(V v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    V y = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Exclusive prefix sum across the block (blockDim.x a multiple of 32, <= 1024).
template <typename V>
__device__ V block_excl_scan(V x, V* sh, V* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  V v = warp_incl_scan(x);
  if (lane == 31) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    V w = lane < nw ? sh[lane] : V(0);
    w = warp_incl_scan(w);
    if (lane < nw) sh[lane] = w;
  }
  __syncthreads();
  V pre = warp ? sh[warp - 1] : V(0);
  if (total) *total = sh[nw - 1];
  __syncthreads();
  return pre + v - x;
}

template <typename V>
__device__ V block_sum(V x, V* sh) {
  V tot;
  block_excl_scan(x, sh, &tot);
  return tot;
}

// Bins are visited from the highest down; thread t owns bins [hi-15, hi], hi = 4095 - 16 t.
// Finds the bin where base + cumulative mass first reaches target.  Result in *out_bin /
// *out_above (mass strictly above that bin, base included); untouched if never reached.
__device__ void find_cut_desc_4096(const unsigned long long (&m)[16], unsigned long long base,
                                   unsigned long long target, unsigned long long* sh,
                                   int* out_bin, unsigned long long* out_above) {
  unsigned long long s = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) s += m[k];
  unsigned long long cum = base + block_excl_scan(s, sh, (unsigned long long*)nullptr);
  const int hi = 4095 - 16 * (int)threadIdx.x;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const unsigned long long nxt = cum + m[k];
    if (cum < target && nxt >= target) {
      *out_bin = hi - k;
      *out_above = cum;
    }
    cum = nxt;
  }
  __syncthreads();
}

// Ascending count search: thread t owns bins [16 t, 16 t + 15].  Finds the bin where the
// running count (starting at base) first reaches q.
__device__ void find_kth_asc_4096(const unsigned (&c)[16], unsigned base, unsigned q, unsigned* sh,
                                  int* out_bin, unsigned* out_before) {
  unsigned s = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) s += c[k];
  unsigned cum = base + block_excl_scan(s, sh, (unsigned*)nullptr);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const unsigned nxt = cum + c[k];
    if (cum < q && nxt >= q) {
      *out_bin = 16 * (int)threadIdx.x + k;
      *out_before = cum;
    }
    cum = nxt;
  }
  __syncthreads();
}

// ------------------------------------------------------------------ index scores
// Log2-domain logits of one index row (16 bf16 in two uint4) for the G heads.
template <int G>
__device__ __forceinline__ void row_logits(const uint4& a, const uint4& b, const float (&qi)[G][kIdxDim],
                                           float (&lg)[G]) {
  float x[16];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[2 * k] = bf16_lo(w[k]);
    x[2 * k + 1] = bf16_hi(w[k]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < kIdxDim; ++r) acc = fmaf(qi[h][r], x[r], acc);
    lg[h] = acc;
  }
}

struct SliceCoord {
  int s, b, g, c, L;
};

__device__ __forceinline__ SliceCoord slice_coord(const StepParams& P) {
  SliceCoord sc;
  const int y = blockIdx.y;
  sc.b = y / P.n_ret;
  sc.g = P.ret_heads[y % P.n_ret];
  sc.s = sc.b * P.Hkv + sc.g;
  sc.c = blockIdx.x;
  sc.L = load_len(P.seq_lens, sc.b, P.Lcap, P.ws.dev_err);
  return sc;
}

template <int G>
__device__ __forceinline__ void load_qidx(const StepParams& P, const SliceCoord& sc, float (&qi)[G][kIdxDim]) {
  const float* q = P.ws.q_idx + ((size_t)sc.b * P.Hq + (size_t)sc.g * G) * kIdxDim;
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int r = 0; r < kIdxDim; ++r) qi[h][r] = q[h * kIdxDim + r] * P.idx_scale_log2;
}

// ------------------------------------------------------------------ prologue
// One CTA per (b, kv head), 256 threads.  cos/sin of the 64 RoPE angles are formed
// once in float64 and shared; each warp owns index outputs (h, r) and reduces the
// 128-term float64 dot product P_q[h][r] . q_pre[h] across its lanes.
template <typename T>
__global__ void __launch_bounds__(256) k_prologue(StepParams P) {
  __shared__ double cs_s[kHeadDim / 2], sn_s[kHeadDim / 2];
  const int s = blockIdx.x;
  const int b = s / P.Hkv, g = s % P.Hkv, G = P.G;
  const int L = load_len(P.seq_lens, b, P.Lcap, P.ws.dev_err);
  const T* q = (const T*)P.q_pre + ((size_t)b * P.Hq + (size_t)g * G) * kHeadDim;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kHeadDim / 2) {
    // rotate-half RoPE at position L-1; the angle is formed and reduced in float64
    const double ang = (double)(L - 1) * P.ws.inv_freq[tid];
    sincos(ang, &sn_s[tid], &cs_s[tid]);
  }
  __syncthreads();
  for (int t = tid; t < G * (kHeadDim / 2); t += blockDim.x) {
    const int h = t / (kHeadDim / 2), i = t % (kHeadDim / 2);
    const double x1 = Elem<T>::get(q, h * kHeadDim + i);
    const double x2 = Elem<T>::get(q, h * kHeadDim + i + kHeadDim / 2);
    float* o = P.ws.q_rot + ((size_t)b * P.Hq + (size_t)g * G + h) * kHeadDim;
    o[i] = (float)(x1 * cs_s[i] - x2 * sn_s[i]);
    o[i + kHeadDim / 2] = (float)(x2 * cs_s[i] + x1 * sn_s[i]);
  }
  if (P.is_ret[g]) {
    for (int o = warp; o < G * kIdxDim; o += blockDim.x / 32) {
      const int h = o / kIdxDim, r = o % kIdxDim;
      const float* pq = P.ws.P_q + ((size_t)(g * G + h) * kIdxDim + r) * kHeadDim;
      double acc = 0.0;
#pragma unroll
      for (int k = 0; k < kHeadDim / 32; ++k) {
        const int d = lane + 32 * k;
        acc += (double)pq[d] * (double)Elem<T>::get(q, h * kHeadDim + d);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
      if (lane == 0) P.ws.q_idx[((size_t)b * P.Hq + (size_t)g * G + h) * kIdxDim + r] = (float)acc;
    }
    unsigned long long* h1 = P.ws.hist1 + (size_t)s * kBins1;
    for (int i = tid; i < kBins1; i += blockDim.x) h1[i] = 0ull;
    if (tid == 0) {
      SliceState z;
      z.q_total = z.target = z.m_above = 0ull;
      z.b1 = -1;
      z.tau_bits = 0u;
      z.pos_cut = INT_MAX;
      z.count = 0;
      z.ticket_mass = z.ticket_thr = z.cand_count = 0u;
      z.pad_ = 0;
      P.ws.st[s] = z;
    }
  } else if (tid == 0) {
    P.ws.st[s].count = 0;
    if (P.sel_count) P.sel_count[s] = 0;
  }
}

// ------------------------------------------------------------------ k_score
template <int G>
__global__ void __launch_bounds__(kSelThreads) k_score(StepParams P) {
  constexpr int U = G <= 4 ? 4 : 2;  // rows in flight per thread
  __shared__ float2 red[kSelThreads / 32][G];
  const SliceCoord sc = slice_coord(P);
  const int j0 = sc.c * kChunk;
  float2* out = P.ws.stats + ((size_t)sc.s * P.n_chunks + sc.c) * G;
  if (j0 >= sc.L) {
    if (threadIdx.x < G) out[threadIdx.x] = make_float2(-INFINITY, 0.f);
    return;
  }
  float qi[G][kIdxDim];
  load_qidx<G>(P, sc, qi);
  const int jend = min(sc.L, j0 + kChunk);
  const uint4* rows = reinterpret_cast<const uint4*>(P.idx_cache + (size_t)sc.s * P.Lmax * kIdxDim);
  float m[G], z[G];
#pragma unroll
  for (int h = 0; h < G; ++h) { m[h] = -INFINITY; z[h] = 0.f; }

  for (int i = 0; i < kTokPerThread; i += U) {
    uint4 ra[U], rb[U];
    int jj[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      jj[u] = j0 + threadIdx.x + kSelThreads * (i + u);
      if (jj[u] < jend) {
        ra[u] = __ldg(rows + 2 * (size_t)jj[u]);
        rb[u] = __ldg(rows + 2 * (size_t)jj[u] + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (jj[u] < jend) {
        float lg[G];
        row_logits<G>(ra[u], rb[u], qi, lg);
#pragma unroll
        for (int h = 0; h < G; ++h) merge_mz(m[h], z[h], lg[h], 1.f);
      }
    }
  }
  // reduce (m, z) over the block in a fixed order
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(kFull, m[h], o);
      const float z2 = __shfl_xor_sync(kFull, z[h], o);
      merge_mz(m[h], z[h], m2, z2);
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0)
#pragma unroll
    for (int h = 0; h < G; ++h) red[warp][h] = make_float2(m[h], z[h]);
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float mm = -INFINITY, zz = 0.f;
    for (int w = 0; w < kSelThreads / 32; ++w) merge_mz(mm, zz, red[w][h].x, red[w][h].y);
    out[h] = make_float2(mm, zz);
  }
}

// ------------------------------------------------------------------ k_mass
template <int G>
__global__ void __launch_bounds__(kSelThreads) k_mass(StepParams P) {
  constexpr int U = G <= 4 ? 4 : 2;
  __shared__ unsigned long long hist[kBins1];
  __shared__ float Mh[G], Wh[G];
  __shared__ unsigned long long sh[32];
  __shared__ int last_flag;
  __shared__ int cut_bin;
  __shared__ unsigned long long cut_above;
  const SliceCoord sc = slice_coord(P);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j0 = sc.c * kChunk;

  for (int i = tid; i < kBins1; i += kSelThreads) hist[i] = 0ull;
  // global (M_h, Z_h): warp h merges the chunk partials, in a fixed order
  if (warp < G) {
    const int nc = (sc.L + kChunk - 1) / kChunk;
    float m = -INFINITY, z = 0.f;
    for (int c = lane; c < nc; c += 32) {
      const float2 v = P.ws.stats[((size_t)sc.s * P.n_chunks + c) * G + warp];
      merge_mz(m, z, v.x, v.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(kFull, m, o);
      const float z2 = __shfl_xor_sync(kFull, z, o);
      merge_mz(m, z, m2, z2);
    }
    if (lane == 0) {
      Mh[warp] = m;
      Wh[warp] = 1.f / ((float)G * z);
    }
  }
  __syncthreads();

  if (j0 < sc.L) {
    float qi[G][kIdxDim];
    load_qidx<G>(P, sc, qi);
    float M[G], W[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { M[h] = Mh[h]; W[h] = Wh[h]; }
    const int jend = min(sc.L, j0 + kChunk);
    const uint4* rows = reinterpret_cast<const uint4*>(P.idx_cache + (size_t)sc.s * P.Lmax * kIdxDim);
    float* pi = P.ws.pi + (size_t)sc.s * P.Lmax;
    for (int i = 0; i < kTokPerThread; i += U) {
      uint4 ra[U], rb[U];
      int jj[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        jj[u] = j0 + tid + kSelThreads * (i + u);
        if (jj[u] < jend) {
          ra[u] = __ldg(rows + 2 * (size_t)jj[u]);
          rb[u] = __ldg(rows + 2 * (size_t)jj[u] + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (jj[u] < jend) {
          float lg[G];
          row_logits<G>(ra[u], rb[u], qi, lg);
          float pr = 0.f;
#pragma unroll
          for (int h = 0; h < G; ++h) pr = fmaf(exp2f(lg[h] - M[h]), W[h], pr);
          pi[jj[u]] = pr;
          const unsigned bits = __float_as_uint(pr);
          atomicAdd(&hist[min(bits >> 18, (unsigned)(kBins1 - 1))], mass_q(pr));
        }
      }
    }
  }
  __syncthreads();
  unsigned long long* g1 = P.ws.hist1 + (size_t)sc.s * kBins1;
  for (int i = tid; i < kBins1; i += kSelThreads)
    if (hist[i]) atomicAdd(g1 + i, hist[i]);
  __threadfence();
  __syncthreads();
  if (tid == 0) last_flag = (atomicAdd(&P.ws.st[sc.s].ticket_mass, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!last_flag) return;
  __threadfence();

  // ---- last CTA of this slice: total mass, target and the round-1 cut bin
  unsigned long long m16[16];
  unsigned long long tsum = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    m16[k] = __ldcg(g1 + (4095 - 16 * tid - k));
    tsum += m16[k];
  }
  const unsigned long long total = block_sum(tsum, sh);
  SliceState* st = P.ws.st + sc.s;
  if (P.keep_all || total == 0ull) {
    if (tid == 0) { st->q_total = total; st->target = total; st->b1 = -1; st->m_above = 0ull; }
    return;
  }
  unsigned long long target = (unsigned long long)ceil((double)P.p * (double)total);
  if (target < 1ull) target = 1ull;
  if (target > total) {  // cannot happen for p < 1; keep everything if it does
    if (tid == 0) { st->q_total = total; st->target = target; st->b1 = -1; st->m_above = 0ull; }
    return;
  }
  if (tid == 0) cut_bin = -1;
  __syncthreads();
  find_cut_desc_4096(m16, 0ull, target, sh, &cut_bin, &cut_above);
  if (tid == 0) {
    st->q_total = total;
    st->target = target;
    st->b1 = cut_bin;
    st->m_above = cut_above;
  }
}

// ------------------------------------------------------------------ k_threshold
__global__ void __launch_bounds__(kSelThreads) k_threshold(StepParams P) {
  __shared__ unsigned long long big[kBins2];    // round-2 masses; reused for counts
  __shared__ unsigned long long m3[kBins3];
  __shared__ unsigned c3[kBins3];
  __shared__ unsigned long long shl[32];
  __shared__ unsigned shu[32];
  __shared__ int shi[32];
  __shared__ int last_flag, b2, b3, kbin;
  __shared__ unsigned long long above2;
  __shared__ unsigned kbefore;
  const SliceCoord sc = slice_coord(P);
  const int tid = threadIdx.x, lane = tid & 31;
  const int j0 = sc.c * kChunk;
  SliceState* st = P.ws.st + sc.s;
  const int b1 = st->b1;
  const SinkWindow sw(sc.L, P.n_sink, P.window);
  const unsigned* pib = reinterpret_cast<const unsigned*>(P.ws.pi + (size_t)sc.s * P.Lmax);
  uint2* cand = P.ws.cand + (size_t)sc.s * P.Lmax;

  int cnt = 0;
  if (j0 < sc.L) {
    const int jend = min(sc.L, j0 + kChunk);
    for (int i = 0; i < kTokPerThread; ++i) {
      const int j = j0 + tid + kSelThreads * i;
      bool is_c = false;
      unsigned bits = 0;
      if (j < jend) {
        bits = __ldcg(pib + j);
        const int d1 = (int)min(bits >> 18, (unsigned)(kBins1 - 1));
        if (d1 > b1) cnt += sw.always(j) ? 0 : 1;
        else if (d1 == b1) is_c = true;
      }
      const unsigned mask = __ballot_sync(kFull, is_c);
      if (mask) {
        const int leader = __ffs(mask) - 1;
        unsigned base = 0;
        if (lane == leader) base = atomicAdd(&st->cand_count, (unsigned)__popc(mask));
        base = __shfl_sync(kFull, base, leader);
        if (is_c) cand[base + __popc(mask & ((1u << lane) - 1u))] = make_uint2(bits, (unsigned)j);
      }
    }
  }
  const int chunk_total = block_sum(cnt, shi);
  if (tid == 0) P.ws.chunk_gt[(size_t)sc.s * P.n_chunks + sc.c] = chunk_total;
  __threadfence();
  __syncthreads();
  if (tid == 0) last_flag = (atomicAdd(&st->ticket_thr, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!last_flag) return;
  __threadfence();

  // ---- last CTA: exact cut value, tie quota and per-chunk offsets
  unsigned tau = 0u;
  int pos_cut = INT_MAX;
  int* chunk_sel = reinterpret_cast<int*>(big);
  if (b1 >= 0) {
    const unsigned n = __ldcg(&st->cand_count);
    const unsigned long long target = __ldcg(&st->target);
    const unsigned long long mab = __ldcg(&st->m_above);
    // round 2: bits 17..6
    for (int i = tid; i < kBins2; i += kSelThreads) big[i] = 0ull;
    if (tid < kBins3) { m3[tid] = 0ull; c3[tid] = 0u; }
    if (tid == 0) { b2 = -1; b3 = -1; }
    __syncthreads();
    for (unsigned i = tid; i < n; i += kSelThreads) {
      const unsigned bits = __ldcg(&cand[i].x);
      atomicAdd(&big[(bits >> 6) & 0xfffu], mass_q(__uint_as_float(bits)));
    }
    __syncthreads();
    unsigned long long m16[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) m16[k] = big[4095 - 16 * tid - k];
    find_cut_desc_4096(m16, mab, target, shl, &b2, &above2);
    // round 3: bits 5..0 of the candidates in bin b2
    for (unsigned i = tid; i < n; i += kSelThreads) {
      const unsigned bits = __ldcg(&cand[i].x);
      if ((int)((bits >> 6) & 0xfffu) == b2) {
        atomicAdd(&m3[bits & 63u], mass_q(__uint_as_float(bits)));
        atomicAdd(&c3[bits & 63u], 1u);
      }
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long cum = above2;
      for (int k = kBins3 - 1; k >= 0; --k) {
        if (cum < target && cum + m3[k] >= target) { b3 = k; break; }
        cum += m3[k];
      }
      above2 = cum;  // mass strictly above tau
    }
    __syncthreads();
    // b2/b3 always exist (the candidates hold the mass of bin b1); if a search ever
    // failed, fall back to keeping every token rather than index a missing bin.
    const bool found = b2 >= 0 && b3 >= 0;
    tau = found ? (((unsigned)b1 << 18) | ((unsigned)b2 << 6) | (unsigned)b3) : 0u;
    const unsigned long long m_gt = above2;
    const unsigned n_eq = found ? c3[b3] : 0u;
    const unsigned long long q_tau = mass_q(__uint_as_float(tau));
    const unsigned long long need =
        (found && q_tau > 0ull && target > m_gt) ? (target - m_gt + q_tau - 1ull) / q_tau : ~0ull;
    if (found && need < (unsigned long long)n_eq) {
      // pos_cut = need-th smallest position among the tied candidates
      unsigned* cnt4k = reinterpret_cast<unsigned*>(big);
      const unsigned qk = (unsigned)need;
      for (int pass = 0; pass < 2; ++pass) {
        for (int i = tid; i < 4096; i += kSelThreads) cnt4k[i] = 0u;
        __syncthreads();
        for (unsigned i = tid; i < n; i += kSelThreads) {
          const uint2 cv = __ldcg(&cand[i]);
          if (cv.x != tau) continue;
          if (pass == 0) atomicAdd(&cnt4k[cv.y >> 12], 1u);
          else if ((int)(cv.y >> 12) == kbin) atomicAdd(&cnt4k[cv.y & 4095u], 1u);
        }
        __syncthreads();
        unsigned c16[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) c16[k] = cnt4k[16 * tid + k];
        __shared__ int fbin;
        __shared__ unsigned fbefore;
        if (tid == 0) fbin = -1;
        __syncthreads();
        find_kth_asc_4096(c16, pass == 0 ? 0u : kbefore, qk, shu, &fbin, &fbefore);
        if (tid == 0) {
          if (fbin < 0) kbin = -1;
          else if (pass == 0) { kbin = fbin; kbefore = fbefore; }
          else if (kbin >= 0) kbin = (kbin << 12) | fbin;
        }
        __syncthreads();
        if (kbin < 0) break;
      }
      pos_cut = kbin >= 0 ? kbin : INT_MAX;
    }
    // per-chunk count of kept, listed candidates
    for (int i = tid; i < P.n_chunks; i += kSelThreads) chunk_sel[i] = 0;
    __syncthreads();
    for (unsigned i = tid; i < n; i += kSelThreads) {
      const uint2 cv = __ldcg(&cand[i]);
      const bool keep = cv.x > tau || (cv.x == tau && (int)cv.y <= pos_cut);
      if (keep && !sw.always((int)cv.y)) atomicAdd(&chunk_sel[cv.y / kChunk], 1);
    }
    __syncthreads();
  } else {
    for (int i = tid; i < P.n_chunks; i += kSelThreads) chunk_sel[i] = 0;
    __syncthreads();
  }
  // offsets: exclusive scan over chunks of (above-b1 count + kept candidates)
  const int per = (P.n_chunks + kSelThreads - 1) / kSelThreads;
  const int c0 = tid * per;
  int loc = 0;
  for (int k = 0; k < per; ++k) {
    const int c = c0 + k;
    if (c < P.n_chunks) loc += __ldcg(&P.ws.chunk_gt[(size_t)sc.s * P.n_chunks + c]) + chunk_sel[c];
  }
  int total = 0;
  int run = block_excl_scan(loc, shi, &total);
  for (int k = 0; k < per; ++k) {
    const int c = c0 + k;
    if (c < P.n_chunks) {
      P.ws.chunk_off[(size_t)sc.s * P.n_chunks + c] = run;
      run += __ldcg(&P.ws.chunk_gt[(size_t)sc.s * P.n_chunks + c]) + chunk_sel[c];
    }
  }
  if (tid == 0) {
    st->tau_bits = tau;
    st->pos_cut = pos_cut;
    st->count = total;
    if (P.sel_count) P.sel_count[sc.s] = total;
  }
}

// ------------------------------------------------------------------ k_compact
__global__ void __launch_bounds__(kSelThreads) k_compact(StepParams P) {
  __shared__ int shi[32];
  const SliceCoord sc = slice_coord(P);
  const int j0 = sc.c * kChunk;
  if (j0 >= sc.L) return;
  const SliceState* st = P.ws.st + sc.s;
  const unsigned tau = st->tau_bits;
  const int pos_cut = st->pos_cut;
  const SinkWindow sw(sc.L, P.n_sink, P.window);
  const unsigned* pib = reinterpret_cast<const unsigned*>(P.ws.pi + (size_t)sc.s * P.Lmax);
  const int jb = j0 + threadIdx.x * kTokPerThread;  // this thread's 16 consecutive tokens
  unsigned keep = 0u;
#pragma unroll
  for (int i = 0; i < kTokPerThread; ++i) {
    const int j = jb + i;
    if (j < sc.L) {
      const unsigned bits = __ldcg(pib + j);
      const bool k = (bits > tau || (bits == tau && j <= pos_cut)) && !sw.always(j);
      keep |= (k ? 1u : 0u) << i;
    }
  }
  const int off = block_excl_scan(__popc(keep), shi, (int*)nullptr);
  const int64_t first = (int64_t)P.ws.chunk_off[(size_t)sc.s * P.n_chunks + sc.c] + off;
  int* dst = P.sel_list + (size_t)sc.s * P.Lmax;
  int k = 0;
#pragma unroll
  for (int i = 0; i < kTokPerThread; ++i) {
    if (keep >> i & 1u) {
      const int64_t o = first + k++;
      if (o < P.Lmax) dst[o] = jb + i;
      else atomicOr(P.ws.dev_err, kErrInternal);   // offsets and predicate disagree: never write past the list
    }
  }
}

template <int G>
cudaError_t launch_score_g(const StepParams& P, cudaStream_t st) {
  k_score<G><<<dim3(P.n_chunks, P.B * P.n_ret), kSelThreads, 0, st>>>(P);
  return cudaGetLastError();
}
template <int G>
cudaError_t launch_mass_g(const StepParams& P, cudaStream_t st) {
  k_mass<G><<<dim3(P.n_chunks, P.B * P.n_ret), kSelThreads, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prologue(const StepParams& P, int kv_dtype, cudaStream_t st) {
  if (kv_dtype == 0) k_prologue<__nv_bfloat16><<<P.n_slices, 256, 0, st>>>(P);
  else k_prologue<float><<<P.n_slices, 256, 0, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_score(const StepParams& P, cudaStream_t st) {
  switch (P.G) {
    case 1: return launch_score_g<1>(P, st);
    case 2: return launch_score_g<2>(P, st);
    case 4: return launch_score_g<4>(P, st);
    case 8: return launch_score_g<8>(P, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_mass(const StepParams& P, cudaStream_t st) {
  switch (P.G) {
    case 1: return launch_mass_g<1>(P, st);
    case 2: return launch_mass_g<2>(P, st);
    case 4: return launch_mass_g<4>(P, st);
    case 8: return launch_mass_g<8>(P, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_threshold(const StepParams& P, cudaStream_t st) {
  k_threshold<<<dim3(P.n_chunks, P.B * P.n_ret), kSelThreads, 0, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_compact(const StepParams& P, cudaStream_t st) {
  k_compact<<<dim3(P.n_chunks, P.B * P.n_ret), kSelThreads, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace spa
