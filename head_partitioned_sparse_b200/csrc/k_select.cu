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
// Scores of 16 tokens at a time on the tensor cores (mma.sync m16n8k16, bf16 in,
// float32 accumulate): A = the 16 tokens' bf16 index rows (16 x 16 dims), B = the
// group's query index vectors, each split exactly into three bf16 parts
// (hi + mid + lo = the float32 value), one part per column.  Summing the three
// part-columns in a fixed order gives the float32 score.  Lane (gid, t4) owns
// tokens gid and gid + 8 and head t4 (G <= 4) or heads t4, t4 + 4 (G = 8).
// Index dims are permuted consistently in A and B so that each lane loads one
// 8-byte word per token row: logical k {2t4, 2t4+1, 2t4+8, 2t4+9} <- physical
// dims {4t4 .. 4t4+3}.
template <int G>
struct IdxTiles {
  static constexpr int NT = G <= 4 ? 2 : 3;   // n-tiles of 8 columns
  static constexpr int NH = G <= 4 ? 1 : 2;   // heads per lane
};

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float x, float y) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Head owned by lane t4 in slot nh (may be >= G for G < 4: such lanes are ignored).
template <int G>
__device__ __forceinline__ int lane_head(int t4, int nh) { return G <= 4 ? t4 : t4 + 4 * nh; }

struct SliceCoord {
  int s, b, g, c, L;
};

template <int G>
__device__ __forceinline__ void load_qidx_frag(const StepParams& P, int b, int g,
                                               uint32_t (&qb)[IdxTiles<G>::NT][2]) {
  __shared__ float qsm[G * kIdxDim];
  const int lane = threadIdx.x & 31, gid = lane >> 2, t4 = lane & 3;
  if (threadIdx.x < G * kIdxDim) qsm[threadIdx.x] = P.ws.q_idx[((size_t)b * P.Hq + (size_t)g * G) * kIdxDim + threadIdx.x];
  __syncthreads();
  const float* qbase = qsm;
#pragma unroll
  for (int t = 0; t < IdxTiles<G>::NT; ++t) {
    int head, part;   // part 0 = hi, 1 = mid, 2 = lo, -1 = zero column
    if (G <= 4) {
      head = gid >> 1;
      part = t == 0 ? (gid & 1) : ((gid & 1) ? -1 : 2);
    } else {
      head = t < 2 ? 4 * t + (gid >> 1) : (gid >> 1) + 4 * (gid & 1);
      part = t < 2 ? (gid & 1) : 2;
    }
    if (head >= G) part = -1;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (part >= 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = qbase[head * kIdxDim + 4 * t4 + e];
        const float hi = __bfloat162float(__float2bfloat16_rn(x));
        const float mid = __bfloat162float(__float2bfloat16_rn(x - hi));
        const float lo = __bfloat162float(__float2bfloat16_rn((x - hi) - mid));
        v[e] = part == 0 ? hi : (part == 1 ? mid : lo);
      }
    }
    qb[t][0] = pack_bf16x2(v[0], v[1]);
    qb[t][1] = pack_bf16x2(v[2], v[3]);
  }
}

// Log2-domain logits of tokens gid (ra) and gid + 8 (rb) for the lane's heads.
template <int G>
__device__ __forceinline__ void group_logits(const uint2& ra, const uint2& rb,
                                             const uint32_t (&qb)[IdxTiles<G>::NT][2], float scale,
                                             float (&lg)[IdxTiles<G>::NH][2]) {
  const uint32_t a[4] = {ra.x, rb.x, ra.y, rb.y};
  float c[IdxTiles<G>::NT][4];
#pragma unroll
  for (int t = 0; t < IdxTiles<G>::NT; ++t) {
    c[t][0] = c[t][1] = c[t][2] = c[t][3] = 0.f;
    mma16816(c[t], a, qb[t][0], qb[t][1]);
  }
  if (G <= 4) {
    lg[0][0] = ((c[0][0] + c[0][1]) + c[1][0]) * scale;
    lg[0][1] = ((c[0][2] + c[0][3]) + c[1][2]) * scale;
  } else {
    lg[0][0] = ((c[0][0] + c[0][1]) + c[IdxTiles<G>::NT - 1][0]) * scale;
    lg[0][1] = ((c[0][2] + c[0][3]) + c[IdxTiles<G>::NT - 1][2]) * scale;
    lg[IdxTiles<G>::NH - 1][0] = ((c[1][0] + c[1][1]) + c[IdxTiles<G>::NT - 1][1]) * scale;
    lg[IdxTiles<G>::NH - 1][1] = ((c[1][2] + c[1][3]) + c[IdxTiles<G>::NT - 1][3]) * scale;
  }
}

// L2 eviction policies: the first index pass keeps its lines (the second pass reads
// the same rows right after), the second pass marks them first to go.
__device__ __forceinline__ uint64_t l2_policy_keep() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_drop() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint2 ld_hint(const uint2* ptr, uint64_t pol) {
  uint2 v;
  asm volatile("ld.global.nc.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;\n"
               : "=r"(v.x), "=r"(v.y)
               : "l"(ptr), "l"(pol));
  return v;
}

// One 16-token group: 8-byte slices of the two index rows a lane needs (zeros past jend).
__device__ __forceinline__ void load_group(const uint2* rows, int j, int jend, uint64_t pol, uint2& ra,
                                           uint2& rb) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, t4 = lane & 3;
  const int ja = j + gid, jb = j + gid + 8;
  ra = ja < jend ? ld_hint(rows + 4 * (size_t)ja + t4, pol) : make_uint2(0u, 0u);
  rb = jb < jend ? ld_hint(rows + 4 * (size_t)jb + t4, pol) : make_uint2(0u, 0u);
}

// Online max / sum-of-exp2 with one exp2 per value; -inf values are skipped.
__device__ __forceinline__ void online_add(float& m, float& z, float l) {
  if (l == -INFINITY) return;
  if (l > m) {
    z = z * exp2f(m - l) + 1.f;
    m = l;
  } else {
    z += exp2f(l - m);
  }
}


// Every CTA of a slice needs the same few scalars; one thread loads each of them and
// shares it, so thousands of warps do not queue on one L2 line.
__device__ __forceinline__ SliceCoord slice_coord(const StepParams& P) {
  __shared__ int s_len;
  SliceCoord sc;
  const int y = blockIdx.y;
  sc.b = y / P.n_ret;
  sc.g = P.ret_heads[y % P.n_ret];
  sc.s = sc.b * P.Hkv + sc.g;
  sc.c = blockIdx.x;
  if (threadIdx.x == 0) s_len = load_len(P.seq_lens, sc.b, P.Lcap, P.ws.dev_err);
  __syncthreads();
  sc.L = s_len;
  return sc;
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
    // rotate-half RoPE at position L-1.  The angle is carried in units of pi,
    // t = (L-1) * inv_freq / pi in float64, reduced exactly modulo 2 (|t| < 2^52), and
    // sincospi evaluates the reduced angle: no large-argument reduction on the device.
    const double t = (double)(L - 1) * P.ws.inv_freq[tid];
    const double r = t - 2.0 * rint(0.5 * t);
    sincospi(r, &sn_s[tid], &cs_s[tid]);
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
    // warp w owns outputs o = w + 8k (k < 2G); every projector load of the warp is issued
    // before the first reduction
    constexpr int kMaxOut = kMaxGroup * kIdxDim / 8;
    const int nw = blockDim.x / 32;
    float pv[kMaxOut][kHeadDim / 32];
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
      const int o = warp + nw * k;
      if (o < G * kIdxDim) {
        const float* pq = P.ws.P_q + ((size_t)g * G * kIdxDim + o) * kHeadDim;
#pragma unroll
        for (int e = 0; e < kHeadDim / 32; ++e) pv[k][e] = pq[lane + 32 * e];
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
      const int o = warp + nw * k;
      if (o < G * kIdxDim) {
        const int h = o / kIdxDim, r = o % kIdxDim;
        double acc = 0.0;
#pragma unroll
        for (int e = 0; e < kHeadDim / 32; ++e)
          acc += (double)pv[k][e] * (double)Elem<T>::get(q, h * kHeadDim + lane + 32 * e);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
        if (lane == 0) P.ws.q_idx[((size_t)b * P.Hq + (size_t)g * G + h) * kIdxDim + r] = (float)acc;
      }
    }
    unsigned long long* h1 = P.ws.hist1 + (size_t)s * kBins1;
    unsigned long long* h2 = P.ws.hist2 + (size_t)s * kBins2;
    for (int i = tid; i < kBins1; i += blockDim.x) h1[i] = 0ull;
    for (int i = tid; i < kBins2; i += blockDim.x) h2[i] = 0ull;
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
// Warp w of a chunk's CTA takes the 16-token groups w, w + 8, ... (4 in flight).
template <int G>
__global__ void __launch_bounds__(kSelThreads) k_score(StepParams P) {
  constexpr int NH = IdxTiles<G>::NH, U = 8;
  constexpr int kGroups = kChunk / 16, kWarps = kSelThreads / 32;
  __shared__ float2 red[kWarps][G];
  const SliceCoord sc = slice_coord(P);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, t4 = lane & 3;
  const int j0 = sc.c * kChunk;
  float2* out = P.ws.stats + ((size_t)sc.s * P.n_chunks + sc.c) * G;
  if (j0 >= sc.L) {
    if (threadIdx.x < G) out[threadIdx.x] = make_float2(-INFINITY, 0.f);
    return;
  }
  uint32_t qb[IdxTiles<G>::NT][2];
  load_qidx_frag<G>(P, sc.b, sc.g, qb);
  const float scale = P.idx_scale_log2;
  const int jend = min(sc.L, j0 + kChunk);
  const uint2* rows = reinterpret_cast<const uint2*>(P.idx_cache + (size_t)sc.s * P.Lmax * kIdxDim);
  // two independent online accumulators per head (tokens gid and gid + 8) keep the
  // exp2 dependency chains short; merged below
  float m[NH][2], z[NH][2];
#pragma unroll
  for (int h = 0; h < NH; ++h) { m[h][0] = m[h][1] = -INFINITY; z[h][0] = z[h][1] = 0.f; }
  const uint64_t pol = l2_policy_keep();
  const int gid = lane >> 2;
  for (int k = 0; k < kGroups / kWarps; k += U) {
    uint2 ra[U], rb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) load_group(rows, j0 + 16 * (warp + kWarps * (k + u)), jend, pol, ra[u], rb[u]);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + 16 * (warp + kWarps * (k + u));
      float lg[NH][2];
      group_logits<G>(ra[u], rb[u], qb, scale, lg);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        online_add(m[h][0], z[h][0], j + gid < jend ? lg[h][0] : -INFINITY);
        online_add(m[h][1], z[h][1], j + gid + 8 < jend ? lg[h][1] : -INFINITY);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < NH; ++h) merge_mz(m[h][0], z[h][0], m[h][1], z[h][1]);
  float mf[NH], zf[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) { mf[h] = m[h][0]; zf[h] = z[h][0]; }
  // lanes with the same t4 hold the same heads: merge over gid, then over warps
#pragma unroll
  for (int h = 0; h < NH; ++h) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const float m2 = __shfl_xor_sync(kFull, mf[h], o);
      const float z2 = __shfl_xor_sync(kFull, zf[h], o);
      merge_mz(mf[h], zf[h], m2, z2);
    }
    const int head = lane_head<G>(t4, h);
    if (lane < 4 && head < G) red[warp][head] = make_float2(mf[h], zf[h]);
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float mm = -INFINITY, zz = 0.f;
    for (int w = 0; w < kWarps; ++w) merge_mz(mm, zz, red[w][h].x, red[w][h].y);
    out[h] = make_float2(mm, zz);
  }
}

// ------------------------------------------------------------------ k_mass
template <int G>
__global__ void __launch_bounds__(kSelThreads) k_mass(StepParams P) {
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
    constexpr int NH = IdxTiles<G>::NH, U = 8;
    constexpr int kGroups = kChunk / 16, kWarps = kSelThreads / 32;
    uint32_t qb[IdxTiles<G>::NT][2];
    load_qidx_frag<G>(P, sc.b, sc.g, qb);
    const float scale = P.idx_scale_log2;
    const int gid = lane >> 2, t4 = lane & 3;
    float M[NH], W[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const int head = lane_head<G>(t4, h);
      M[h] = head < G ? Mh[head] : 0.f;
      W[h] = head < G ? Wh[head] : 0.f;   // lanes of absent heads contribute nothing
    }
    const int jend = min(sc.L, j0 + kChunk);
    const uint2* rows = reinterpret_cast<const uint2*>(P.idx_cache + (size_t)sc.s * P.Lmax * kIdxDim);
    float* pi = P.ws.pi + (size_t)sc.s * P.ws.pi_stride;
    const uint64_t pol = l2_policy_drop();
    for (int k = 0; k < kGroups / kWarps; k += U) {
      uint2 ra[U], rb[U];
#pragma unroll
      for (int u = 0; u < U; ++u) load_group(rows, j0 + 16 * (warp + kWarps * (k + u)), jend, pol, ra[u], rb[u]);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + 16 * (warp + kWarps * (k + u));
        float lg[NH][2];
        group_logits<G>(ra[u], rb[u], qb, scale, lg);
        // pi = sum over the group's heads of 2^(l - M_h) / (G Z_h): lane-local heads first,
        // then the 4 lanes of a token (fixed order, identical result in every lane)
        float pr[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float acc = 0.f;
#pragma unroll
          for (int h = 0; h < NH; ++h) acc += W[h] == 0.f ? 0.f : exp2f(lg[h][c] - M[h]) * W[h];
          acc += __shfl_xor_sync(kFull, acc, 1);
          acc += __shfl_xor_sync(kFull, acc, 2);
          pr[c] = acc;
        }
        if (t4 < 2) {   // lane t4 = 0 stores token gid, t4 = 1 token gid + 8
          const int jt = j + gid + 8 * t4;
          const float v = t4 == 0 ? pr[0] : pr[1];
          if (jt < jend) {
            pi[jt] = v;
            const unsigned bits = __float_as_uint(v);
            atomicAdd(&hist[min(bits >> 18, (unsigned)(kBins1 - 1))], mass_q(v));
          }
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
constexpr int kSmallCap = 1024;   // candidates of the round-2 cut bin held in shared memory
constexpr int kCandBatch = 8;     // candidates loaded per thread before any is used

// Calls f(bits, pos) for every candidate (in no particular order), kCandBatch
// independent loads per thread at a time.
template <class F>
__device__ __forceinline__ void for_each_candidate(const uint2* cand, unsigned n, F&& f) {
  for (unsigned i0 = 0; i0 < n; i0 += kSelThreads * kCandBatch) {
    uint2 cv[kCandBatch];
#pragma unroll
    for (int u = 0; u < kCandBatch; ++u) {
      const unsigned i = i0 + threadIdx.x + kSelThreads * u;
      cv[u] = i < n ? __ldcg(cand + i) : make_uint2(0u, 0xffffffffu);
    }
#pragma unroll
    for (int u = 0; u < kCandBatch; ++u)
      if (cv[u].y != 0xffffffffu) f(cv[u].x, (int)cv[u].y);
  }
}

// Number of positions of [lo, hi) outside sinks and window.
__device__ __forceinline__ int listed_in(const SinkWindow& sw, int lo, int hi) {
  if (hi <= lo) return 0;
  const int a = max(lo, sw.n_s), b = min(hi, sw.w_lo);
  return b > a ? b - a : 0;
}

__global__ void __launch_bounds__(kSelThreads) k_threshold(StepParams P) {
  __shared__ int chunk_sel[kMaxChunks];        // kept candidates per chunk (listed ones)
  __shared__ unsigned cnt4k[4096];             // position-select histogram
  __shared__ uint2 small[kSmallCap];           // candidates of the round-2 cut bin
  __shared__ unsigned long long m3[kBins3];
  __shared__ unsigned c3[kBins3];
  __shared__ unsigned long long shl[32];
  __shared__ unsigned shu[32];
  __shared__ int shi[32];
  __shared__ int last_flag, b2, b3, kbin, fbin;
  __shared__ unsigned small_n, kbefore, fbefore;
  __shared__ unsigned long long above2;
  const SliceCoord sc = slice_coord(P);
  const int tid = threadIdx.x, lane = tid & 31;
  const int j0 = sc.c * kChunk;
  SliceState* st = P.ws.st + sc.s;
  __shared__ int s_b1;
  if (tid == 0) s_b1 = st->b1;
  __syncthreads();
  const int b1 = s_b1;
  const SinkWindow sw(sc.L, P.n_sink, P.window);
  const unsigned* pib = reinterpret_cast<const unsigned*>(P.ws.pi + (size_t)sc.s * P.ws.pi_stride);
  uint2* cand = P.ws.cand + (size_t)sc.s * P.Lmax;
  unsigned long long* h2 = P.ws.hist2 + (size_t)sc.s * kBins2;

  // ---- every chunk: tokens above bin b1 (listed ones counted), tokens of bin b1
  // appended as candidates with their round-2 masses added to the slice histogram
  int cnt = 0;
  if (j0 < sc.L) {
    const int jend = min(sc.L, j0 + kChunk);
    unsigned bits[kTokPerThread];
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      const int j = j0 + tid + kSelThreads * i;
      bits[i] = j < jend ? __ldcg(pib + j) : 0u;
    }
    unsigned cflags = 0u;
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      const int j = j0 + tid + kSelThreads * i;
      if (j < jend) {
        const int d1 = (int)min(bits[i] >> 18, (unsigned)(kBins1 - 1));
        if (d1 > b1) cnt += sw.always(j) ? 0 : 1;
        else if (d1 == b1) cflags |= 1u << i;
      }
    }
    // one atomic per warp reserves the warp's candidate slots
    unsigned masks[kTokPerThread];
    unsigned warp_total = 0u;
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      masks[i] = __ballot_sync(kFull, (cflags >> i) & 1u);
      warp_total += __popc(masks[i]);
    }
    if (warp_total) {
      unsigned base = 0u;
      if (lane == 0) base = atomicAdd(&st->cand_count, warp_total);
      base = __shfl_sync(kFull, base, 0);
      const unsigned lt = (1u << lane) - 1u;
#pragma unroll
      for (int i = 0; i < kTokPerThread; ++i) {
        if ((cflags >> i) & 1u) {
          cand[base + __popc(masks[i] & lt)] = make_uint2(bits[i], (unsigned)(j0 + tid + kSelThreads * i));
          atomicAdd(&h2[(bits[i] >> 6) & 0xfffu], mass_q(__uint_as_float(bits[i])));
        }
        base += __popc(masks[i]);
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

  // ---- last CTA of the slice: exact cut value, tie quota, per-chunk output offsets
  unsigned tau = 0u;
  int pos_cut = INT_MAX;
  for (int c = tid; c < P.n_chunks; c += kSelThreads) chunk_sel[c] = 0;
  if (tid < kBins3) { m3[tid] = 0ull; c3[tid] = 0u; }
  if (tid == 0) { b2 = -1; b3 = -1; small_n = 0u; kbin = -1; }
  __syncthreads();
  bool found = b1 < 0;   // keep-everything mode needs no cut
  if (b1 >= 0) {
    const unsigned n = __ldcg(&st->cand_count);
    const unsigned long long target = __ldcg(&st->target);
    const unsigned long long mab = __ldcg(&st->m_above);
    // round 2 (bits 17..6): the chunks filled the slice histogram
    unsigned long long m16[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) m16[k] = __ldcg(h2 + (4095 - 16 * tid - k));
    find_cut_desc_4096(m16, mab, target, shl, &b2, &above2);
    const int cb2 = b2;
    // one pass over the candidates: above the round-2 bin they are kept; inside it
    // they feed round 3 (bits 5..0) and are parked in shared memory
    for_each_candidate(cand, n, [&](unsigned bits, int pos) {
      const int d2 = (int)((bits >> 6) & 0xfffu);
      if (d2 > cb2) {
        if (!sw.always(pos)) atomicAdd(&chunk_sel[pos / kChunk], 1);
      } else if (d2 == cb2) {
        atomicAdd(&m3[bits & 63u], mass_q(__uint_as_float(bits)));
        atomicAdd(&c3[bits & 63u], 1u);
        const unsigned slot = atomicAdd(&small_n, 1u);
        if (slot < kSmallCap) small[slot] = make_uint2(bits, (unsigned)pos);
      }
    });
    __syncthreads();
    if (tid == 0 && cb2 >= 0) {
      unsigned long long cum = above2;
      for (int k = kBins3 - 1; k >= 0; --k) {
        if (cum < target && cum + m3[k] >= target) { b3 = k; break; }
        cum += m3[k];
      }
      above2 = cum;   // mass strictly above tau
    }
    __syncthreads();
    // b2 and b3 always exist (the candidates carry the mass of bin b1); if a search ever
    // failed, every token is kept rather than a missing bin indexed
    found = cb2 >= 0 && b3 >= 0;
    const bool small_ok = small_n <= (unsigned)kSmallCap;
    const unsigned sn = small_ok ? small_n : 0u;
    if (found) {
      tau = ((unsigned)b1 << 18) | ((unsigned)cb2 << 6) | (unsigned)b3;
      const unsigned long long m_gt = above2;
      const unsigned n_eq = c3[b3];
      const unsigned long long q_tau = mass_q(__uint_as_float(tau));
      const unsigned long long need =
          (q_tau > 0ull && target > m_gt) ? (target - m_gt + q_tau - 1ull) / q_tau : ~0ull;
      if (need < (unsigned long long)n_eq) {
        // pos_cut = need-th smallest position among the candidates equal to tau
        const unsigned qk = (unsigned)need;
        for (int pass = 0; pass < 2; ++pass) {
          for (int i = tid; i < 4096; i += kSelThreads) cnt4k[i] = 0u;
          __syncthreads();
          const int kb = kbin;
          auto add = [&](unsigned bits, int pos) {
            if (bits != tau) return;
            if (pass == 0) atomicAdd(&cnt4k[(unsigned)pos >> 12], 1u);
            else if ((int)((unsigned)pos >> 12) == kb) atomicAdd(&cnt4k[(unsigned)pos & 4095u], 1u);
          };
          if (small_ok) {
            for (unsigned i = tid; i < sn; i += kSelThreads) add(small[i].x, (int)small[i].y);
          } else {
            for_each_candidate(cand, n, add);
          }
          __syncthreads();
          unsigned c16[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) c16[k] = cnt4k[16 * tid + k];
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
      // kept candidates of the round-2 cut bin
      const int pc = pos_cut;
      auto keep_bin = [&](unsigned bits, int pos) {
        if ((int)((bits >> 6) & 0xfffu) != cb2) return;
        if ((bits > tau || (bits == tau && pos <= pc)) && !sw.always(pos)) atomicAdd(&chunk_sel[pos / kChunk], 1);
      };
      if (small_ok) {
        for (unsigned i = tid; i < sn; i += kSelThreads) keep_bin(small[i].x, (int)small[i].y);
      } else {
        for_each_candidate(cand, n, keep_bin);
      }
    }
    __syncthreads();
  }
  if (!found) {
    // keep everything: every listed token of each chunk
    tau = 0u;
    pos_cut = INT_MAX;
    for (int c = tid; c < P.n_chunks; c += kSelThreads)
      chunk_sel[c] = listed_in(sw, c * kChunk, min(sc.L, (c + 1) * kChunk)) -
                     __ldcg(&P.ws.chunk_gt[(size_t)sc.s * P.n_chunks + c]);
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
  __shared__ unsigned s_tau;
  __shared__ int s_cut, s_off;
  if (threadIdx.x == 0) {
    const SliceState* st = P.ws.st + sc.s;
    s_tau = st->tau_bits;
    s_cut = st->pos_cut;
    s_off = P.ws.chunk_off[(size_t)sc.s * P.n_chunks + sc.c];
  }
  __syncthreads();
  const unsigned tau = s_tau;
  const int pos_cut = s_cut;
  const SinkWindow sw(sc.L, P.n_sink, P.window);
  const unsigned* pib = reinterpret_cast<const unsigned*>(P.ws.pi + (size_t)sc.s * P.ws.pi_stride);
  const int jb = j0 + threadIdx.x * kTokPerThread;  // this thread's 16 consecutive tokens
  unsigned keep = 0u;
  if (jb < sc.L) {
    // rows of the probability buffer are padded to 64 floats: four 16-byte loads stay in the row
    const uint4* v4 = reinterpret_cast<const uint4*>(pib + jb);
    unsigned bits[kTokPerThread];
#pragma unroll
    for (int q = 0; q < kTokPerThread / 4; ++q) {
      const uint4 v = __ldcg(v4 + q);
      bits[4 * q] = v.x;
      bits[4 * q + 1] = v.y;
      bits[4 * q + 2] = v.z;
      bits[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      const int j = jb + i;
      const bool k = j < sc.L && (bits[i] > tau || (bits[i] == tau && j <= pos_cut)) && !sw.always(j);
      keep |= (k ? 1u : 0u) << i;
    }
  }
  const int off = block_excl_scan(__popc(keep), shi, (int*)nullptr);
  const int64_t first = (int64_t)s_off + off;
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
