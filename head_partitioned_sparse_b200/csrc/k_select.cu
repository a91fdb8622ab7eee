// Query prologue and top-p token selection for the retrieval heads, as one
// cooperative persistent kernel.
//
// "Full Attention Strikes Back" (RTPurbo summary):
//   Methodology §2  index scores in a 16-dim pre-RoPE subspace;
//   Methodology §3  dynamic top-p: accumulate index attention mass until p;
//   Methodology §5  sort-free, histogram-based thresholding.
// Group mean of per-head probabilities: "Autonomy of Heads" summary, Deployment
// strategy (GQA scores aggregated to the group by their mean).
//
// Phases (units: retrieval slices s = (b, g); the score and mass phases split the
// slices' 16-token groups into equal ranges per CTA, the later phases work on chunks of
// kChunk tokens):
//   score     the leader CTA of each slice computes q_idx = P_q q_pre (float64 dot
//             products) and publishes it (flag); every range then forms, per head h,
//             m = max_j l_hj, z = sum_j 2^(l_hj - m),
//             l_hj = log2(e) * idx_scale * <q_idx[h], idx_j>   (index read #1);
//   -- grid barrier --
//   mass      merge (m, z) over ranges -> M_h, Z_h; recompute l_hj (index read #2),
//             pi_j = sum_h 2^(l_hj - M_h) / (G Z_h), stored as fp32; a mass histogram
//             over the top 12 bits of pi_j's bit pattern, masses quantised to integer
//             multiples of 2^-63 so every sum is exact and order independent (per range
//             as a count and a sum of low significand bits per bin, 32-bit atomics);
//   cut 1     per slice (last range, ticket): total mass, target ceil(p * total) (or k
//             for top-k) and the bin b1 where the descending cumulative mass reaches it;
//   -- grid barrier --
//   threshold per chunk: tokens above b1 counted, tokens of bin b1 appended as
//             candidates with their round-2 masses added to the slice histogram;
//   refine    per slice (last chunk, ticket): round-2 bin b2 from the histogram, one
//             pass over the candidates for round 3 (exact cut value tau), the tie quota
//             at tau (lowest positions first) and per-chunk output offsets; idle CTAs
//             compute q_rot = RoPE(q_pre, L-1) for every head as duties (angles in
//             float64, reduced exactly in units of pi);
//   -- grid barrier --
//   compact   per chunk: kept positions outside sinks/window, ascending.
// Block mode (the block-granular variant, a second instantiation): the ranges are cut at
// kBlock-token block boundaries, the mass phase stores and histograms each block's mass
// (the float32 sum of its tokens' pi) instead of the tokens', the threshold, refine and
// compact steps rank blocks and count their listed tokens, and compact lists every
// token of a kept block.  The blocks follow the chunk routing of the "Hierarchical
// Global Attention" summary, Central mechanism §4.
// One launch replaces a chain of small kernels whose fixed launch cost dominated.
// Grid barriers and the q_idx flags are polled with a clock budget; on timeout they set
// a device status bit and the kernel leaves or carries on without hanging.  The launch
// is cooperative, so all CTAs are resident together.
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

// Thread t's 16 coalesced histogram words (bins t + 256 k), issued before they are used.
__device__ __forceinline__ void hist_issue(const unsigned long long* g, unsigned long long (&v)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __ldcg(g + threadIdx.x + 256 * k);
}
// Redistributes them through shared memory so that thread t holds bins 4095 - 16 t - k,
// k = 0..15 (the layout of the descending cut search).  Ends with a CTA barrier.
__device__ __forceinline__ void hist_desc(unsigned long long* stage, const unsigned long long (&v)[16],
                                          unsigned long long (&m)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int i = (int)threadIdx.x + 256 * k;
    stage[i + (i >> 4)] = v[k];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int i = 4095 - 16 * (int)threadIdx.x - k;
    m[k] = stage[i + (i >> 4)];
  }
  __syncthreads();
}

// Mass of a token in the radix select: its quantised probability for top-p, 1 for
// top-k (the same select then counts tokens, and the target is k).
__device__ __forceinline__ unsigned long long sel_mass(const StepParams& P, unsigned bits) {
  return P.topk > 0 ? 1ull : mass_q(bits);
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


// The lane's B fragments of the group's query index vectors (qsm, G * 16 floats in
// shared memory).
template <int G>
__device__ __forceinline__ void qidx_frag(const float* qbase, uint32_t (&qb)[IdxTiles<G>::NT][2]) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, t4 = lane & 3;
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

// Stages the group's query index vectors (written by an earlier phase, read through L2)
// in shared memory and builds the fragments.  Called by every thread of the CTA.
template <int G>
__device__ __forceinline__ void load_qidx_frag(const StepParams& P, int b, int g, float* qsm,
                                               uint32_t (&qb)[IdxTiles<G>::NT][2]) {
  if (threadIdx.x < G * kIdxDim)
    qsm[threadIdx.x] = __ldcg(&P.ws.q_idx[((size_t)b * P.Hq + (size_t)g * G) * kIdxDim + threadIdx.x]);
  __syncthreads();
  qidx_frag<G>(qsm, qb);
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
__device__ __forceinline__ float4 ld_keep(const float4* ptr, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(ptr), "l"(pol));
  return v;
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

// 2^x with the hardware approximation (relative error about 2^-22, results below 2^-126
// flushed to 0), used by both index passes so that sums and probabilities agree.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Online max / sum-of-exp2 with one exp2 per value; -inf values are skipped.
__device__ __forceinline__ void online_add(float& m, float& z, float l) {
  if (l == -INFINITY) return;
  if (l > m) {
    z = z * ex2(m - l) + 1.f;
    m = l;
  } else {
    z += ex2(l - m);
  }
}



// ------------------------------------------------------------------ grid barrier
constexpr long long kBarrierCycles = 4000000000LL;   // ~2 s bound per barrier

// Barrier over all CTAs of a cooperative launch on one arrival word bar[0]: CTA 0
// adds 2^31 - (nb - 1), every other CTA adds 1, so the word's top bit flips exactly
// when the last CTA arrives and its low 31 bits return to their value (no reset, and
// the release is the last arrival itself).  Every CTA polls until the top bit differs
// from the one it saw on arrival.  The CTA whose arrival flips the bit also advances
// the generation word bar[32] (its own 128-byte line), which tags the q_idx flags of
// a call.  Returns false (on every thread of the CTA) if the wait gave up.
__device__ bool grid_barrier(unsigned* bar, unsigned* err, int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned add = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1u) : 1u;
    __threadfence();
    const unsigned old = atomicAdd(bar, add);
    if (((old + add) ^ old) & 0x80000000u) {
      atomicAdd(bar + 32, 1u);
    } else {
      volatile unsigned* word = bar;
      const long long t0 = clock64();
      unsigned ns = 32;
      while (((*word ^ old) & 0x80000000u) == 0u) {
        if (clock64() - t0 > kBarrierCycles) {
          atomicOr(err, kErrTimeout);
          ok = 0;
          break;
        }
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
      }
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

// "Last CTA of the slice" ticket: every unit of the slice takes one; the CTA that
// takes the last runs the per-slice step.  Called by every thread of the CTA.
__device__ bool last_of_slice(unsigned* ticket, unsigned n_units, int* s_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *s_flag = atomicAdd(ticket, 1u) == n_units - 1;
  __syncthreads();
  if (*s_flag) __threadfence();
  return *s_flag != 0;
}

// ------------------------------------------------------------------ shared memory
constexpr int kWarps = kSelThreads / 32;
constexpr int kGroupBatch = 4;                // groups per warp loaded together (8 spills at 64 registers)
constexpr int kSmallCap = 1024;   // candidates of the round-2 cut bin held in shared memory
constexpr int kCandBatch = 8;     // candidates loaded per thread before any is used

struct SmemPro { double cs[kHeadDim / 2], sn[kHeadDim / 2]; };
struct SmemScore { float2 red[kSelThreads / 32][kMaxGroup]; };
struct SmemMass { unsigned cnt[kBins1], low[kBins1]; float Mh[kMaxGroup], Wh[kMaxGroup]; };
struct SmemRefine {
  int chunk_sel[kMaxChunks];      // kept candidates per chunk (listed ones)
  unsigned cnt4k[4096];           // position-select histogram
  uint2 small[kSmallCap];         // candidates of the round-2 cut bin
  unsigned long long m3[kBins3];
  unsigned c3[kBins3];
};
// Round-1 / round-2 histogram staged for the cut search: loaded coalesced, read back as
// 16 consecutive bins per thread (index i stored at i + i / 16 against bank conflicts).
struct SmemStage { unsigned long long h[kBins1 + kBins1 / 16]; };
union SelSmem {
  SmemStage stage;
  SmemPro pro;
  SmemScore score;
  SmemMass mass;
  SmemRefine ref;
};
// Scalars shared by the threads of a CTA (outside the union: live across calls).
struct SelScalars {
  float qsm[kMaxGroup * kIdxDim];
  unsigned long long shl[32];
  unsigned shu[32];
  int shi[32];
  int L, b1, b2, b3, kbin, fbin, cut_bin, pos_cut, off, ok, duty;
  unsigned small_n, kbefore, fbefore, tau;
  unsigned long long above2, cut_above;
};

// Unit coordinates: retrieval slice y -> (b, g, s).
struct Unit {
  int b, g, s;
};
__device__ __forceinline__ Unit unit_of(const StepParams& P, int y) {
  Unit u;
  u.b = y / P.n_ret;
  u.g = P.ret_heads[y % P.n_ret];
  u.s = u.b * P.Hkv + u.g;
  return u;
}
// Sequence length of b, loaded by one thread and shared (every CTA of a slice needs it).
__device__ __forceinline__ int cta_len(const StepParams& P, int b, SelScalars& sc) {
  __syncthreads();   // previous readers of sc.L are done
  if (threadIdx.x == 0) sc.L = load_len(P.seq_lens, b, P.Lcap, P.ws.dev_err);
  __syncthreads();
  return sc.L;
}

// ------------------------------------------------------------------ query rotation
// RoPE of slice s's G query heads at position L-1 (streaming slices included), read by
// the attention kernels after this launch; a streaming slice's selection count is 0.
// Taken as a "duty" by CTAs that wait at the last barrier anyway.
template <typename T>
__device__ void qrot_slice(const StepParams& P, SmemPro& sm, SelScalars& sc, int s) {
  const int b = s / P.Hkv, g = s % P.Hkv, G = P.G;
  const int L = cta_len(P, b, sc);
  const T* q = (const T*)P.q_pre + ((size_t)b * P.Hq + (size_t)g * G) * kHeadDim;
  const int tid = threadIdx.x;
  if (tid < kHeadDim / 2) {
    // rotate-half RoPE at position L-1.  The angle is carried in units of pi,
    // t = (L-1) * inv_freq / pi in float64, reduced exactly modulo 2 (|t| < 2^52), and
    // sincospi evaluates the reduced angle: no large-argument reduction on the device.
    const double t = (double)(L - 1) * P.ws.inv_freq[tid];
    const double r = t - 2.0 * rint(0.5 * t);
    sincospi(r, &sm.sn[tid], &sm.cs[tid]);
  }
  __syncthreads();
  for (int t = tid; t < G * (kHeadDim / 2); t += blockDim.x) {
    const int h = t / (kHeadDim / 2), i = t % (kHeadDim / 2);
    const double x1 = Elem<T>::get(q, h * kHeadDim + i);
    const double x2 = Elem<T>::get(q, h * kHeadDim + i + kHeadDim / 2);
    float* o = P.ws.q_rot + ((size_t)b * P.Hq + (size_t)g * G + h) * kHeadDim;
    o[i] = (float)(x1 * sm.cs[i] - x2 * sm.sn[i]);
    o[i + kHeadDim / 2] = (float)(x2 * sm.cs[i] + x1 * sm.sn[i]);
  }
  if (!P.is_ret[g] && tid == 0) {
    P.ws.st[s].count = 0;
    if (P.sel_count) P.sel_count[s] = 0;
  }
  __syncthreads();   // sm.cs / sm.sn reused by the next duty
}

// Takes q_rot duties (slices) from a grid-wide ticket until none is left.
template <typename T>
__device__ void qrot_duties(const StepParams& P, SmemPro& sm, SelScalars& sc) {
  for (;;) {
    __syncthreads();
    if (threadIdx.x == 0) sc.duty = (int)atomicAdd(P.ws.bar + kBarDuty, 1u);
    __syncthreads();
    const int s = sc.duty;
    if (s >= P.n_slices) return;
    qrot_slice<T>(P, sm, sc, s);
  }
}

// ------------------------------------------------------------------ query index vectors
// q_idx[h] = P_q[g G + h] q_pre[h] for the G heads of slice (b, g): float64 dot products,
// thread w of G * 64 sums a quarter (32 dims) of output w / 4 in order, the quarters are
// added pairwise.  Result in sc.qsm (G * 16 floats) with the sequence length of b in
// sc.L (validated as load_len does), both visible after the call.
template <typename T, int G>
__device__ void compute_qidx(const StepParams& P, int b, int g, SelScalars& sc) {
  const int tid = threadIdx.x;
  float* qsm = sc.qsm;
  int64_t len_raw = 0;
  if (tid == 0) len_raw = P.seq_lens[b];   // validated after the dot products are issued
  const T* q = (const T*)P.q_pre + ((size_t)b * P.Hq + (size_t)g * G) * kHeadDim;
  const uint64_t keep = l2_policy_keep();   // projectors are reread by the next call
  for (int w = tid; w < G * kIdxDim * 4; w += kSelThreads) {   // whole warps (G * 64 = 64k)
    const int o = w >> 2, qd = w & 3, h = o / kIdxDim;
    const float4* prow = reinterpret_cast<const float4*>(P.ws.P_q + ((size_t)g * G * kIdxDim + o) * kHeadDim) + 8 * qd;
    const T* qrow = q + h * kHeadDim + 32 * qd;
    double acc = 0.0;
    if (sizeof(T) == 2) {
      // bf16 queries: all 32 projector values and the 32 query values in one round trip
      // (q_pre is 16-byte aligned and the quarter starts at a 64-byte offset)
      float4 pv[8];
      uint4 qw[4];
#pragma unroll
      for (int k = 0; k < 8; ++k) pv[k] = ld_keep(prow + k, keep);
#pragma unroll
      for (int k = 0; k < 4; ++k) qw[k] = __ldg(reinterpret_cast<const uint4*>(qrow) + k);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 w4 = qw[k >> 1];
        const uint32_t wa = (k & 1) ? w4.z : w4.x, wb = (k & 1) ? w4.w : w4.y;
        acc += (double)pv[k].x * (double)bf16_lo(wa);
        acc += (double)pv[k].y * (double)bf16_hi(wa);
        acc += (double)pv[k].z * (double)bf16_lo(wb);
        acc += (double)pv[k].w * (double)bf16_hi(wb);
      }
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float4 pv[4];
        float qv[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) pv[k] = ld_keep(prow + 4 * half + k, keep);
#pragma unroll
        for (int k = 0; k < 16; ++k) qv[k] = Elem<T>::get(qrow, 16 * half + k);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc += (double)pv[k].x * (double)qv[4 * k];
          acc += (double)pv[k].y * (double)qv[4 * k + 1];
          acc += (double)pv[k].z * (double)qv[4 * k + 2];
          acc += (double)pv[k].w * (double)qv[4 * k + 3];
        }
      }
    }
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    if (qd == 0) qsm[o] = (float)acc;
  }
  if (tid == 0) {
    if (len_raw < 1 || len_raw > P.Lcap) {
      atomicOr(P.ws.dev_err, kErrSeqLen);
      len_raw = len_raw < 1 ? 1 : P.Lcap;
    }
    sc.L = (int)len_raw;
  }
  __syncthreads();
}

// ------------------------------------------------------------------ work partition
// The score and mass phases split the retrieval slices' capacity (max_seq_len tokens
// each, as ngc 16-token groups; slice y = b * n_ret + r owns global groups
// [y ngc, (y+1) ngc)) into equal contiguous group ranges, one per CTA, so every SM of a
// full-occupancy grid gets the same share.  A range may span slices; groups past a
// sequence's length are empty.  Ranges are cut at multiples of q groups (q = 1, or
// kBlock / 16 in block mode so that no block is split; ngc is then a multiple of q):
// CTA c covers groups [q floor(c Q / nb), q floor((c+1) Q / nb)), Q = n_rs ngc / q.
template <bool BLK>
struct Ranges {
  static constexpr int q = BLK ? kBlock / 16 : 1;
  long long ngc, quanta;
  int nb;
  __device__ __forceinline__ Ranges(const StepParams& P) {
    ngc = ((long long)P.Lcap + 16 * q - 1) / (16 * q) * q;
    quanta = (long long)P.B * P.n_ret * (ngc / q);
    nb = (int)gridDim.x;
  }
  __device__ __forceinline__ long long begin(int c) const { return (long long)c * quanta / nb * q; }
  // CTA whose range holds global group g
  __device__ __forceinline__ int owner(long long g) const { return (int)(((g / q + 1) * nb - 1) / quanta); }
  __device__ __forceinline__ int first_cta(int y) const { return owner((long long)y * ngc); }
  __device__ __forceinline__ int last_cta(int y) const { return owner((long long)(y + 1) * ngc - 1); }
};
// Per-range statistics of slice y live at stats[(cta + y) * G]: the CTAs of slice y
// are consecutive and the last one of y may be the first one of y + 1, so the slots
// of different slices never overlap (at most nb + n_rs of them).
__device__ __forceinline__ size_t stats_slot(int cta, int y) { return (size_t)cta + (size_t)y; }

// Visits the CTA's range as segments f(y, l0, l1) of local groups [l0, l1) of slice y.
template <class RT, class F>
__device__ __forceinline__ void for_each_segment(const RT& R, F&& f) {
  const long long ge = R.begin(blockIdx.x + 1);
  for (long long g = R.begin(blockIdx.x); g < ge;) {
    const int y = (int)(g / R.ngc);
    const long long gend = min(ge, (long long)(y + 1) * R.ngc);
    f(y, (int)(g - (long long)y * R.ngc), (int)(gend - (long long)y * R.ngc));
    g = gend;
  }
}

// ------------------------------------------------------------------ score phase
// The leader of slice y (the CTA holding its first group) resets the slice state,
// computes the group's query index vectors, stores them and publishes them with a flag
// tagged with this call's barrier generation; every range of the slice reads them after
// the flag (bounded wait).  A CTA leads its slices before it scores any range, and only
// waits for lower-numbered CTAs, so the waits always end.
template <typename T, int G>
__device__ void lead_slice(const StepParams& P, SelScalars& sc, int y) {
  const Unit un = unit_of(P, y);
  SliceState* st = P.ws.st + un.s;
  unsigned gen = 0u;   // barrier generation (thread 0): constant while any CTA scores
  if (threadIdx.x == 0) gen = *reinterpret_cast<volatile unsigned*>(P.ws.bar + 32);
  __syncthreads();   // earlier readers of sc.qsm / sc.L are done
  if (threadIdx.x == 0) {
    SliceState z;
    z.q_total = z.target = z.m_above = 0ull;
    z.b1 = -1;
    z.tau_bits = 0u;
    z.pos_cut = INT_MAX;
    z.count = 0;
    z.cand_count = 0u;
    z.ticket_mass = z.ticket_thr = 0u;
    z.qidx_ready = 0u;
    *st = z;
  }
  compute_qidx<T, G>(P, un.b, un.g, sc);
  if (threadIdx.x < G * kIdxDim) {
    P.ws.q_idx[((size_t)un.b * P.Hq + (size_t)un.g * G) * kIdxDim + threadIdx.x] = sc.qsm[threadIdx.x];
    __threadfence();
  }
  __syncthreads();
  // (the failure-detection test hook leaves the flag unset: the other CTAs' bounded
  // waits then run out and report a timeout)
  if (threadIdx.x == 0 && !P.drop_publish) atomicExch(&st->qidx_ready, gen + 1u);
}

// Waits (thread 0, bounded) for slice s's q_idx flag of this call; the caller
// synchronises the CTA afterwards.  The barrier generation that tags the flag cannot
// change before this CTA reaches the first grid barrier.
__device__ __forceinline__ void wait_qidx(const StepParams& P, int s) {
  volatile unsigned* flag = &P.ws.st[s].qidx_ready;
  const unsigned want = *reinterpret_cast<volatile unsigned*>(P.ws.bar + 32) + 1u;
  const long long t0 = clock64();
  unsigned ns = 32;
  while (*flag != want) {
    if (clock64() - t0 > kBarrierCycles) {
      atomicOr(P.ws.dev_err, kErrTimeout);
      break;
    }
    __nanosleep(ns);
    if (ns < 128) ns <<= 1;
  }
  __threadfence();
}

// Clears the CTA's share of slice y's round-1 / round-2 histograms (read after a barrier).
template <class RT>
__device__ __forceinline__ void clear_hist_share(const StepParams& P, const RT& R, int y, int s) {
  static_assert(kBins1 == kBins2, "histogram reset assumes equal round-1 / round-2 bin counts");
  const int first = R.first_cta(y), n = R.last_cta(y) - first + 1, k = (int)blockIdx.x - first;
  unsigned long long* h1 = P.ws.hist1 + (size_t)s * kBins1;
  unsigned long long* h2 = P.ws.hist2 + (size_t)s * kBins2;
  for (int i = k * kSelThreads + (int)threadIdx.x; i < kBins1; i += n * kSelThreads) {
    h1[i] = 0ull;
    h2[i] = 0ull;
  }
}

// One range of slice y: per head m = max_j l_hj, z = sum_j 2^(l_hj - m) over the tokens
// of local groups [l0, l1), l_hj = log2(e) * idx_scale * <q_idx[h], idx_j>.  Warp w takes
// groups l0 + w, l0 + w + 8, ..., kGroupBatch at a time; the first batch is requested
// before the query vectors arrive (bounded by the call's max length; rows past the
// sequence are masked).
template <int G, class RT>
__device__ void score_segment(const StepParams& P, SmemScore& sm, SelScalars& sc, const RT& R, int y,
                              int l0, int l1) {
  constexpr int NH = IdxTiles<G>::NH, U = kGroupBatch;
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, t4 = lane & 3, gid = lane >> 2;
  clear_hist_share(P, R, y, un.s);
  const uint2* rows = reinterpret_cast<const uint2*>(idx_rows(P, y, un.s));
  const uint64_t pol = l2_policy_keep();
  uint2 ra[U], rb[U];
  {
    const int jpf = min(P.Lcap, 16 * l1);
#pragma unroll
    for (int u = 0; u < U; ++u) load_group(rows, 16 * (l0 + warp + kWarps * u), jpf, pol, ra[u], rb[u]);
  }
  __syncthreads();   // earlier readers of sc.L and sc.qsm are done
  if (tid == 0) {
    sc.L = load_len(P.seq_lens, un.b, P.Lcap, P.ws.dev_err);
    if (16 * l0 < sc.L) wait_qidx(P, un.s);
  }
  __syncthreads();
  const int L = sc.L;
  float2* out = P.ws.stats + stats_slot(blockIdx.x, y) * G;
  if (16 * l0 >= L) {
    if (tid < G) out[tid] = make_float2(-INFINITY, 0.f);
    return;
  }
  uint32_t qb[IdxTiles<G>::NT][2];
  load_qidx_frag<G>(P, un.b, un.g, sc.qsm, qb);
  const float scale = P.idx_scale_log2;
  const int jend = min(L, 16 * l1);
  // two independent online accumulators per head (tokens gid and gid + 8)
  float m[NH][2], z[NH][2];
#pragma unroll
  for (int h = 0; h < NH; ++h) { m[h][0] = m[h][1] = -INFINITY; z[h][0] = z[h][1] = 0.f; }
  for (int gb = l0; 16 * gb < jend; gb += kWarps * U) {
    if (gb > l0) {
#pragma unroll
      for (int u = 0; u < U; ++u) load_group(rows, 16 * (gb + warp + kWarps * u), jend, pol, ra[u], rb[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = 16 * (gb + warp + kWarps * u);
      float lg[NH][2];
      group_logits<G>(ra[u], rb[u], qb, scale, lg);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        online_add(m[h][0], z[h][0], j + gid < jend ? lg[h][0] : -INFINITY);
        online_add(m[h][1], z[h][1], j + gid + 8 < jend ? lg[h][1] : -INFINITY);
      }
    }
  }
  // lanes with the same t4 hold the same heads: merge over gid, then over warps
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    merge_mz(m[h][0], z[h][0], m[h][1], z[h][1]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const float m2 = __shfl_xor_sync(kFull, m[h][0], o);
      const float z2 = __shfl_xor_sync(kFull, z[h][0], o);
      merge_mz(m[h][0], z[h][0], m2, z2);
    }
    const int head = lane_head<G>(t4, h);
    if (lane < 4 && head < G) sm.red[warp][head] = make_float2(m[h][0], z[h][0]);
  }
  __syncthreads();
  if (tid < G) {
    float mm = -INFINITY, zz = 0.f;
    for (int w = 0; w < kWarps; ++w) merge_mz(mm, zz, sm.red[w][tid].x, sm.red[w][tid].y);
    out[tid] = make_float2(mm, zz);
  }
  __syncthreads();   // sm.red reused by the next range
}

template <typename T, int G, bool BLK>
__device__ void score_phase(const StepParams& P, SmemScore& sm, SelScalars& sc) {
  const Ranges<BLK> R(P);
  const long long ga = R.begin(blockIdx.x), ge = R.begin(blockIdx.x + 1);
  for (long long y = (ga + R.ngc - 1) / R.ngc; y * R.ngc < ge; ++y) lead_slice<T, G>(P, sc, (int)y);
  for_each_segment(R, [&](int y, int l0, int l1) { score_segment<G>(P, sm, sc, R, y, l0, l1); });
}

// ------------------------------------------------------------------ cut 1 (per slice)
__device__ void cut1_slice(const StepParams& P, SmemStage& sm, SelScalars& sc, int y) {
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x;
  unsigned long long v[16], m16[16];
  hist_issue(P.ws.hist1 + (size_t)un.s * kBins1, v);
  unsigned long long tsum = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) tsum += v[k];
  const unsigned long long total = block_sum(tsum, sc.shl);
  hist_desc(sm.h, v, m16);
  SliceState* st = P.ws.st + un.s;
  unsigned long long target = total;
  bool keep_all = P.keep_all || total == 0ull;
  if (!keep_all) {
    // top-k: the k-th token (total = the number of tokens); top-p: the mass ceil(p total)
    target = P.topk > 0 ? (unsigned long long)P.topk : (unsigned long long)ceil((double)P.p * (double)total);
    if (target < 1ull) target = 1ull;
    keep_all = target >= total && P.topk > 0 ? true : target > total;   // k >= L keeps all
  }
  if (tid == 0) sc.cut_bin = -1;
  __syncthreads();
  if (!keep_all) find_cut_desc_4096(m16, 0ull, target, sc.shl, &sc.cut_bin, &sc.cut_above);
  if (tid == 0) {
    st->q_total = total;
    st->target = target;
    st->b1 = keep_all ? -1 : sc.cut_bin;
    st->m_above = keep_all ? 0ull : sc.cut_above;
  }
  __syncthreads();
}

// ------------------------------------------------------------------ mass phase
// One range of slice y: M_h, Z_h merged from the slice's range statistics (fixed
// order), the logits recomputed (index read #2, mostly from L2),
// pi_j = sum_h 2^(l_hj - M_h) / (G Z_h) stored, and its mass added to the slice's
// round-1 histogram via a per-range shared histogram of counts and low significand
// bits (32-bit atomics; a range holds at most kMaxRangeGroups groups, so a bin's
// low-bit sum stays below 2^32).
// Block mode (BLK): warp w's batch is the four consecutive groups of one kBlock-token
// block; the block's mass (the float32 sum of its tokens' pi, in a fixed order) is
// stored at pi[block] and histogrammed instead of the tokens'.
constexpr int kMaxRangeGroups = 1024;   // 16384 tokens: 16384 * 2^18 = 2^32
static_assert(kGroupBatch * 16 == kBlock, "block mode: one warp batch is one block");
template <int G, bool BLK>
__device__ void mass_segment(const StepParams& P, SmemMass& sm, SelScalars& sc, const Ranges<BLK>& R, int y, int l0,
                             int l1) {
  constexpr int NH = IdxTiles<G>::NH, U = kGroupBatch;
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
  const uint2* rows = reinterpret_cast<const uint2*>(idx_rows(P, y, un.s));
  const uint64_t pol = l2_policy_drop();
  // local group of batch slot u at batch base gb
  auto grp = [&](int gb, int u) { return BLK ? gb + U * warp + u : gb + warp + kWarps * u; };
  uint2 ra[U], rb[U];
  {
    const int jpf = min(P.Lcap, 16 * l1);
#pragma unroll
    for (int u = 0; u < U; ++u) load_group(rows, 16 * grp(l0, u), jpf, pol, ra[u], rb[u]);
  }
  // the sequence length, the query index vectors and the slice statistics are
  // requested together; one CTA barrier publishes them
  __syncthreads();   // earlier readers of sc.L, sc.qsm and the histogram are done
  int64_t len_raw = 0;
  if (tid == 0) len_raw = P.seq_lens[un.b];
  float qv = 0.f;
  if (tid < G * kIdxDim) qv = __ldcg(&P.ws.q_idx[((size_t)un.b * P.Hq + (size_t)un.g * G) * kIdxDim + tid]);
  for (int i = tid; i < kBins1; i += kSelThreads) sm.cnt[i] = sm.low[i] = 0u;
  // global (M_h, Z_h): warp h merges the ranges' partials, in a fixed order
  if (warp < G) {
    const int c0 = R.first_cta(y), c1 = R.last_cta(y);
    float m = -INFINITY, z = 0.f;
    for (int c = c0 + lane; c <= c1; c += 32) {
      const float2 v = __ldcg(&P.ws.stats[stats_slot(c, y) * G + warp]);
      merge_mz(m, z, v.x, v.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(kFull, m, o);
      const float z2 = __shfl_xor_sync(kFull, z, o);
      merge_mz(m, z, m2, z2);
    }
    if (lane == 0) {
      sm.Mh[warp] = m;
      sm.Wh[warp] = 1.f / ((float)G * z);
    }
  }
  if (tid < G * kIdxDim) sc.qsm[tid] = qv;
  if (tid == 0) {
    if (len_raw < 1 || len_raw > P.Lcap) {
      atomicOr(P.ws.dev_err, kErrSeqLen);
      len_raw = len_raw < 1 ? 1 : P.Lcap;
    }
    sc.L = (int)len_raw;
  }
  __syncthreads();
  const int L = sc.L;
  if (16 * l0 >= L) return;
  uint32_t qb[IdxTiles<G>::NT][2];
  qidx_frag<G>(sc.qsm, qb);
  const float scale = P.idx_scale_log2;
  float M[NH], W[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const int head = lane_head<G>(t4, h);
    M[h] = head < G ? sm.Mh[head] : 0.f;
    W[h] = head < G ? sm.Wh[head] : 0.f;   // lanes of absent heads contribute nothing
  }
  const int jend = min(L, 16 * l1);
  float* pi = P.ws.pi + (size_t)un.s * P.ws.pi_stride;
  for (int gb = l0; 16 * gb < jend; gb += kWarps * U) {
    if (gb > l0) {
#pragma unroll
      for (int u = 0; u < U; ++u) load_group(rows, 16 * grp(gb, u), jend, pol, ra[u], rb[u]);
    }
    float bsum = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = 16 * grp(gb, u);
      float lg[NH][2];
      group_logits<G>(ra[u], rb[u], qb, scale, lg);
      // pi = sum over the group's heads of 2^(l - M_h) / (G Z_h): lane-local heads first,
      // then the 4 lanes of a token (fixed order, identical result in every lane)
      float pr[2];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (G < 4 && W[h] == 0.f) continue;   // lanes of absent heads (G < 4) add nothing
          acc += ex2(lg[h][cc] - M[h]) * W[h];
        }
        acc += __shfl_xor_sync(kFull, acc, 1);
        acc += __shfl_xor_sync(kFull, acc, 2);
        pr[cc] = acc;
      }
      if (BLK) {
        bsum += (j + gid < jend ? pr[0] : 0.f) + (j + gid + 8 < jend ? pr[1] : 0.f);
      } else if (t4 < 2) {   // lane t4 = 0 stores token gid, t4 = 1 token gid + 8
        const int jt = j + gid + 8 * t4;
        const float v = t4 == 0 ? pr[0] : pr[1];
        if (jt < jend) {
          pi[jt] = v;
          const unsigned bits = __float_as_uint(v);
          const unsigned d = min(bits >> 18, (unsigned)(kBins1 - 1));
          atomicAdd(&sm.cnt[d], 1u);
          atomicAdd(&sm.low[d], bits & 0x3ffffu);
        }
      }
    }
    if (BLK) {
      // every lane of a token quad holds the same sums: add over the 8 token rows
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) bsum += __shfl_xor_sync(kFull, bsum, o);
      const int jb = 16 * grp(gb, 0);
      if (lane == 0 && jb < jend) {
        pi[jb / kBlock] = bsum;
        const unsigned bits = __float_as_uint(bsum);
        const unsigned d = min(bits >> 18, (unsigned)(kBins1 - 1));
        atomicAdd(&sm.cnt[d], 1u);
        atomicAdd(&sm.low[d], bits & 0x3ffffu);
      }
    }
  }
  __syncthreads();
  unsigned long long* g1 = P.ws.hist1 + (size_t)un.s * kBins1;
  for (int i = tid; i < kBins1; i += kSelThreads)
    if (sm.cnt[i])
      atomicAdd(g1 + i, P.topk > 0 ? (unsigned long long)sm.cnt[i] : bin1_mass((unsigned)i, sm.cnt[i], sm.low[i]));
  __syncthreads();   // the histogram is reused by the next range
}

template <int G, bool BLK>
__device__ void mass_phase(const StepParams& P, SelSmem& sm_all, SelScalars& sc) {
  SmemMass& sm = sm_all.mass;
  const Ranges<BLK> R(P);
  for_each_segment(R, [&](int y, int l0, int l1) {
    for (int a = l0; a < l1; a += kMaxRangeGroups) mass_segment<G, BLK>(P, sm, sc, R, y, a, min(l1, a + kMaxRangeGroups));
    const int n = R.last_cta(y) - R.first_cta(y) + 1;
    if (last_of_slice(&P.ws.st[unit_of(P, y).s].ticket_mass, (unsigned)n, &sc.ok)) cut1_slice(P, sm_all.stage, sc, y);
  });
}

// ------------------------------------------------------------------ threshold phase
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

// Chunk of element e (a token, or a block in block mode).
template <bool BLK>
__device__ __forceinline__ int chunk_of(int e) {
  return BLK ? e / (kChunk / kBlock) : e / kChunk;
}

// Listed positions (outside sinks and window) of element e: token e, or block e in
// block mode.
template <bool BLK>
__device__ __forceinline__ int listed_of(const SinkWindow& sw, int L, int e) {
  if (!BLK) return sw.always(e) ? 0 : 1;
  return listed_in(sw, e * kBlock, min(L, (e + 1) * kBlock));
}

// Unit: one chunk.  Tokens above bin b1 counted (listed ones), tokens of bin b1
// appended as candidates with their round-2 masses added to the slice histogram.
// Block mode: the chunk's kChunk / kBlock blocks, one per thread of the first warps;
// a block above b1 counts its listed tokens, a block of bin b1 is a candidate.
template <bool BLK>
__device__ void threshold_unit(const StepParams& P, SelScalars& sc, int y, int c) {
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x, lane = tid & 31;
  const int j0 = c * kChunk;
  SliceState* st = P.ws.st + un.s;
  const unsigned* pib = reinterpret_cast<const unsigned*>(P.ws.pi + (size_t)un.s * P.ws.pi_stride);
  // the chunk's probabilities are requested with L and b1 (one round trip); rows hold
  // the call's capacity, and entries past L are masked below
  constexpr int kPer = kChunk / kBlock;
  static_assert(kPer % 32 == 0 && kPer <= kSelThreads, "block mode: whole warps of blocks per chunk");
  unsigned bits[kTokPerThread];
  if (BLK) {
    const int e = c * kPer + tid;
    bits[0] = tid < kPer && e * kBlock < P.Lcap ? __ldcg(pib + e) : 0u;
  } else {
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      const int j = j0 + tid + kSelThreads * i;
      bits[i] = j < P.Lcap ? __ldcg(pib + j) : 0u;
    }
  }
  __syncthreads();   // earlier readers of sc.L / sc.b1 are done
  if (tid == 0) {
    sc.L = load_len(P.seq_lens, un.b, P.Lcap, P.ws.dev_err);
    sc.b1 = __ldcg(&st->b1);
  }
  __syncthreads();
  const int L = sc.L, b1 = sc.b1;
  const SinkWindow sw(L, P.n_sink, P.window);
  uint2* cand = P.ws.cand + (size_t)un.s * P.Lmax;
  unsigned long long* h2 = P.ws.hist2 + (size_t)un.s * kBins2;
  int cnt = 0;
  if (BLK && j0 < L) {
    const int e = c * kPer + tid;
    bool is_cand = false;
    if (tid < kPer && e * kBlock < L) {
      const unsigned b = bits[0];
      const int d1 = (int)min(b >> 18, (unsigned)(kBins1 - 1));
      if (d1 > b1) cnt = listed_of<BLK>(sw, L, e);
      else is_cand = d1 == b1;
    }
    if (tid < kPer) {   // whole warps
      const unsigned mask = __ballot_sync(kFull, is_cand);
      if (mask) {
        unsigned base = 0u;
        if (lane == 0) base = atomicAdd(&st->cand_count, (unsigned)__popc(mask));
        base = __shfl_sync(kFull, base, 0);
        if (is_cand) {
          cand[base + __popc(mask & ((1u << lane) - 1u))] = make_uint2(bits[0], (unsigned)e);
          atomicAdd(&h2[(bits[0] >> 6) & 0xfffu], sel_mass(P, bits[0]));
        }
      }
    }
  } else if (j0 < L) {
    const int jend = min(L, j0 + kChunk);
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
          atomicAdd(&h2[(bits[i] >> 6) & 0xfffu], sel_mass(P, bits[i]));
        }
        base += __popc(masks[i]);
      }
    }
  }
  const int chunk_total = block_sum(cnt, sc.shi);
  if (tid == 0) P.ws.chunk_gt[(size_t)un.s * P.n_chunks + c] = chunk_total;
}

// ------------------------------------------------------------------ refine (per slice)
template <bool BLK>
__device__ void refine_slice(const StepParams& P, SelSmem& smu, SelScalars& sc, int y) {
  SmemRefine& sm = smu.ref;
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x;
  SliceState* st = P.ws.st + un.s;
  // every input of this step is requested at once: the round-2 histogram (bits 17..6,
  // filled by the chunks), the slice state and the sequence length
  unsigned long long v2[16];
  hist_issue(P.ws.hist2 + (size_t)un.s * kBins2, v2);
  const unsigned n = __ldcg(&st->cand_count);
  const unsigned long long target = __ldcg(&st->target);
  const unsigned long long mab = __ldcg(&st->m_above);
  const int b1 = __ldcg(&st->b1);
  int64_t len = P.seq_lens[un.b];
  __syncthreads();   // earlier readers of the scalars are done
  if (tid == 0) {
    if (len < 1 || len > P.Lcap) atomicOr(P.ws.dev_err, kErrSeqLen);
    sc.b2 = -1;
    sc.b3 = -1;
    sc.small_n = 0u;
    sc.kbin = -1;
  }
  __syncthreads();
  const int L = len < 1 ? 1 : (len > P.Lcap ? P.Lcap : (int)len);
  const SinkWindow sw(L, P.n_sink, P.window);
  const uint2* cand = P.ws.cand + (size_t)un.s * P.Lmax;
  if (b1 >= 0) {   // round 2 cut (the staging buffer aliases chunk_sel / cnt4k)
    unsigned long long m16[16];
    hist_desc(smu.stage.h, v2, m16);
    find_cut_desc_4096(m16, mab, target, sc.shl, &sc.b2, &sc.above2);
  }
  int* chunk_sel = sm.chunk_sel;
  unsigned* cnt4k = sm.cnt4k;
  uint2* small = sm.small;
  // exact cut value, tie quota, per-chunk output offsets
  unsigned tau = 0u;
  int pos_cut = INT_MAX;
  for (int c = tid; c < P.n_chunks; c += kSelThreads) chunk_sel[c] = 0;
  if (tid < kBins3) { sm.m3[tid] = 0ull; sm.c3[tid] = 0u; }
  __syncthreads();
  bool found = b1 < 0;   // keep-everything mode needs no cut
  if (b1 >= 0) {
    const int cb2 = sc.b2;
    // one pass over the candidates: above the round-2 bin they are kept; inside it
    // they feed round 3 (bits 5..0) and are parked in shared memory
    for_each_candidate(cand, n, [&](unsigned bits, int pos) {
      const int d2 = (int)((bits >> 6) & 0xfffu);
      if (d2 > cb2) {
        const int nl = listed_of<BLK>(sw, L, pos);
        if (nl) atomicAdd(&chunk_sel[chunk_of<BLK>(pos)], nl);
      } else if (d2 == cb2) {
        atomicAdd(&sm.m3[bits & 63u], sel_mass(P, bits));
        atomicAdd(&sm.c3[bits & 63u], 1u);
        const unsigned slot = atomicAdd(&sc.small_n, 1u);
        if (slot < kSmallCap) small[slot] = make_uint2(bits, (unsigned)pos);
      }
    });
    __syncthreads();
    if (tid < 32 && cb2 >= 0) {
      // round 3 (bits 5..0), descending: lane i holds bins 63 - 2i and 62 - 2i
      const unsigned long long ma = sm.m3[63 - 2 * tid], mb = sm.m3[62 - 2 * tid];
      unsigned long long x = ma + mb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long t = __shfl_up_sync(kFull, x, o);
        if (tid >= o) x += t;
      }
      const unsigned long long before = sc.above2 + x - (ma + mb);   // mass above bin 63 - 2i
      int hit = -1;
      unsigned long long above = 0ull;
      if (before < target && before + ma >= target) { hit = 63 - 2 * tid; above = before; }
      else if (before + ma < target && before + ma + mb >= target) { hit = 62 - 2 * tid; above = before + ma; }
      const unsigned who = __ballot_sync(kFull, hit >= 0);
      if (who != 0u && tid == __ffs(who) - 1) {
        sc.b3 = hit;
        sc.above2 = above;   // mass strictly above tau
      }
    }
    __syncthreads();
    // b2 and b3 always exist (the candidates carry the mass of bin b1); if a search ever
    // failed, every token is kept rather than a missing bin indexed
    found = cb2 >= 0 && sc.b3 >= 0;
    const bool small_ok = sc.small_n <= (unsigned)kSmallCap;
    const unsigned sn = small_ok ? sc.small_n : 0u;
    if (found) {
      tau = ((unsigned)b1 << 18) | ((unsigned)cb2 << 6) | (unsigned)sc.b3;
      const unsigned long long m_gt = sc.above2;
      const unsigned n_eq = sm.c3[sc.b3];
      const unsigned long long q_tau = sel_mass(P, tau);
      const unsigned long long need =
          (q_tau > 0ull && target > m_gt) ? (target - m_gt + q_tau - 1ull) / q_tau : ~0ull;
      if (need < (unsigned long long)n_eq) {
        // pos_cut = need-th smallest position among the candidates equal to tau
        const unsigned qk = (unsigned)need;
        for (int pass = 0; pass < 2; ++pass) {
          for (int i = tid; i < 4096; i += kSelThreads) cnt4k[i] = 0u;
          __syncthreads();
          const int kb = sc.kbin;
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
          if (tid == 0) sc.fbin = -1;
          __syncthreads();
          find_kth_asc_4096(c16, pass == 0 ? 0u : sc.kbefore, qk, sc.shu, &sc.fbin, &sc.fbefore);
          if (tid == 0) {
            if (sc.fbin < 0) sc.kbin = -1;
            else if (pass == 0) { sc.kbin = sc.fbin; sc.kbefore = sc.fbefore; }
            else if (sc.kbin >= 0) sc.kbin = (sc.kbin << 12) | sc.fbin;
          }
          __syncthreads();
          if (sc.kbin < 0) break;
        }
        pos_cut = sc.kbin >= 0 ? sc.kbin : INT_MAX;
      }
      // kept candidates of the round-2 cut bin
      const int pc = pos_cut;
      auto keep_bin = [&](unsigned bits, int pos) {
        if ((int)((bits >> 6) & 0xfffu) != cb2) return;
        if (bits > tau || (bits == tau && pos <= pc)) {
          const int nl = listed_of<BLK>(sw, L, pos);
          if (nl) atomicAdd(&chunk_sel[chunk_of<BLK>(pos)], nl);
        }
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
      chunk_sel[c] = listed_in(sw, c * kChunk, min(L, (c + 1) * kChunk)) -
                     __ldcg(&P.ws.chunk_gt[(size_t)un.s * P.n_chunks + c]);
    __syncthreads();
  }
  // offsets: exclusive scan over chunks of (above-b1 count + kept candidates); with one
  // chunk per thread (up to kSelThreads chunks) the count is loaded once
  const int per = (P.n_chunks + kSelThreads - 1) / kSelThreads;
  const int c0 = tid * per;
  const int* gt_row = P.ws.chunk_gt + (size_t)un.s * P.n_chunks;
  int loc = 0;
  for (int k = 0; k < per; ++k) {
    const int c = c0 + k;
    if (c < P.n_chunks) loc += __ldcg(gt_row + c) + chunk_sel[c];
  }
  int total = 0;
  int run = block_excl_scan(loc, sc.shi, &total);
  if (per == 1) {
    if (c0 < P.n_chunks) P.ws.chunk_off[(size_t)un.s * P.n_chunks + c0] = run;
  } else {
    for (int k = 0; k < per; ++k) {
      const int c = c0 + k;
      if (c < P.n_chunks) {
        P.ws.chunk_off[(size_t)un.s * P.n_chunks + c] = run;
        run += __ldcg(gt_row + c) + chunk_sel[c];
      }
    }
  }
  if (tid == 0) {
    st->tau_bits = tau;
    st->pos_cut = pos_cut;
    st->count = total;
    if (P.sel_count) P.sel_count[un.s] = total;
  }
  __syncthreads();   // shared memory reused by the next unit
}

// ------------------------------------------------------------------ compact phase
template <bool BLK>
__device__ void compact_unit(const StepParams& P, SelScalars& sc, int y, int c) {
  static_assert(kBlock % kTokPerThread == 0, "a thread's tokens must lie in one block");
  const Unit un = unit_of(P, y);
  const int j0 = c * kChunk;
  const unsigned* pib = reinterpret_cast<const unsigned*>(P.ws.pi + (size_t)un.s * P.ws.pi_stride);
  const int jb = j0 + threadIdx.x * kTokPerThread;  // this thread's 16 consecutive tokens
  // the probabilities are requested with L and the slice's cut (one round trip); rows
  // hold the call's capacity padded to 64 floats, so four 16-byte loads stay in the row
  unsigned bits[kTokPerThread] = {};
  if (BLK) {
    bits[0] = jb < P.Lcap ? __ldcg(pib + jb / kBlock) : 0u;   // the 16 tokens lie in one block
  } else if (jb < P.Lcap) {
    const uint4* v4 = reinterpret_cast<const uint4*>(pib + jb);
#pragma unroll
    for (int q = 0; q < kTokPerThread / 4; ++q) {
      const uint4 v = __ldcg(v4 + q);
      bits[4 * q] = v.x;
      bits[4 * q + 1] = v.y;
      bits[4 * q + 2] = v.z;
      bits[4 * q + 3] = v.w;
    }
  }
  __syncthreads();   // earlier readers of the scalars are done
  if (threadIdx.x == 0) {
    const SliceState* st = P.ws.st + un.s;
    sc.L = load_len(P.seq_lens, un.b, P.Lcap, P.ws.dev_err);
    sc.tau = __ldcg(&st->tau_bits);
    sc.pos_cut = __ldcg(&st->pos_cut);
    sc.off = __ldcg(&P.ws.chunk_off[(size_t)un.s * P.n_chunks + c]);
  }
  __syncthreads();
  const int L = sc.L;
  if (j0 >= L) return;
  const unsigned tau = sc.tau;
  const int pos_cut = sc.pos_cut;
  const SinkWindow sw(L, P.n_sink, P.window);
  unsigned keep = 0u;
  if (BLK && jb < L) {
    const int e = jb / kBlock;
    if (bits[0] > tau || (bits[0] == tau && e <= pos_cut)) {
#pragma unroll
      for (int i = 0; i < kTokPerThread; ++i) {
        const int j = jb + i;
        keep |= (j < L && !sw.always(j) ? 1u : 0u) << i;
      }
    }
  } else if (jb < L) {
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      const int j = jb + i;
      const bool k = j < L && (bits[i] > tau || (bits[i] == tau && j <= pos_cut)) && !sw.always(j);
      keep |= (k ? 1u : 0u) << i;
    }
  }
  const int off = block_excl_scan(__popc(keep), sc.shi, (int*)nullptr);
  const int64_t first = (int64_t)sc.off + off;
  int* dst = P.sel_list + (size_t)un.s * P.Lmax;
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

// ------------------------------------------------------------------ the kernel
template <typename T, int G, bool BLK>
__global__ void __launch_bounds__(kSelThreads, 4) k_select(StepParams P) {
  __shared__ SelSmem sm;
  __shared__ SelScalars sc;
  const int nb = gridDim.x;
  if (P.n_ret == 0) {   // nothing to select: only the query rotation
    for (int s = blockIdx.x; s < P.n_slices; s += nb) qrot_slice<T>(P, sm.pro, sc, s);
    return;
  }
  const int n_rs = P.B * P.n_ret;
  const int n_units = n_rs * P.n_chunks;
  if (blockIdx.x == 0 && threadIdx.x == 0) P.ws.bar[kBarDuty] = 0u;   // taken after two barriers
  score_phase<T, G, BLK>(P, sm.score, sc);
  if (!grid_barrier(P.ws.bar, P.ws.dev_err, &sc.ok)) return;
  mass_phase<G, BLK>(P, sm, sc);
  if (!grid_barrier(P.ws.bar, P.ws.dev_err, &sc.ok)) return;
  for (int u = blockIdx.x; u < n_units; u += nb) {
    const int y = u / P.n_chunks;
    threshold_unit<BLK>(P, sc, y, u % P.n_chunks);
    if (last_of_slice(&P.ws.st[unit_of(P, y).s].ticket_thr, P.n_chunks, &sc.ok)) refine_slice<BLK>(P, sm, sc, y);
  }
  qrot_duties<T>(P, sm.pro, sc);   // off the critical path: refine steps run meanwhile
  if (!grid_barrier(P.ws.bar, P.ws.dev_err, &sc.ok)) return;
  for (int u = blockIdx.x; u < n_units; u += nb) compact_unit<BLK>(P, sc, u / P.n_chunks, u % P.n_chunks);
}

template <typename T, int G>
cudaError_t launch_tg(const StepParams& P, int grid, cudaStream_t st) {
  StepParams local = P;
  void* args[] = {&local};
  const void* fn = P.blocks ? (const void*)k_select<T, G, true> : (const void*)k_select<T, G, false>;
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kSelThreads), args, 0, st);
}

// Co-resident CTAs per SM, the smaller of the token and block variants (one grid size
// serves both).
template <typename T, int G>
int resident_tg() {
  int n = 0, m = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_select<T, G, false>, kSelThreads, 0) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, k_select<T, G, true>, kSelThreads, 0) != cudaSuccess)
    return -1;
  return n < m ? n : m;
}

}  // namespace

// Grid of the selection launch: every resident CTA (the same count on every SM, so the
// range-partitioned score and mass phases are balanced per SM), but never more CTAs than
// range quanta (16-token groups, or kBlock-token blocks in block mode), so no CTA has an
// empty range.
int select_grid(const StepParams& P, int max_resident) {
  if (P.n_ret <= 0) return P.n_slices < max_resident ? P.n_slices : max_resident;
  const long long qt = P.blocks ? kBlock : 16;
  const long long groups = (long long)P.B * P.n_ret * (((long long)P.Lcap + qt - 1) / qt);
  long long want = max_resident;
  if (want > groups) want = groups;
  if (want < 1) want = 1;
  return (int)want;
}

cudaError_t launch_select(const StepParams& P, int kv_dtype, int grid, cudaStream_t st) {
  if (kv_dtype == 0) {
    switch (P.G) {
      case 1: return launch_tg<__nv_bfloat16, 1>(P, grid, st);
      case 2: return launch_tg<__nv_bfloat16, 2>(P, grid, st);
      case 4: return launch_tg<__nv_bfloat16, 4>(P, grid, st);
      case 8: return launch_tg<__nv_bfloat16, 8>(P, grid, st);
    }
  } else {
    switch (P.G) {
      case 1: return launch_tg<float, 1>(P, grid, st);
      case 2: return launch_tg<float, 2>(P, grid, st);
      case 4: return launch_tg<float, 4>(P, grid, st);
      case 8: return launch_tg<float, 8>(P, grid, st);
    }
  }
  return cudaErrorInvalidValue;
}

// Co-resident CTAs of the selection kernel per SM for (dtype, G), or -1.
int select_resident_per_sm(int kv_dtype, int G) {
  if (kv_dtype == 0) {
    switch (G) {
      case 1: return resident_tg<__nv_bfloat16, 1>();
      case 2: return resident_tg<__nv_bfloat16, 2>();
      case 4: return resident_tg<__nv_bfloat16, 4>();
      case 8: return resident_tg<__nv_bfloat16, 8>();
    }
  } else {
    switch (G) {
      case 1: return resident_tg<float, 1>();
      case 2: return resident_tg<float, 2>();
      case 4: return resident_tg<float, 4>();
      case 8: return resident_tg<float, 8>();
    }
  }
  return -1;
}

}  // namespace spa
