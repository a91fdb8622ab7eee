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
// Work partition: the retrieval slices' capacity, in 16-token groups, is split into
// equal contiguous ranges, one per CTA (a whole number of CTAs per slice when the grid
// holds at least one CTA per slice); a range may span slices (one segment per slice it
// touches).  Every phase works on the CTA's own range, and the probabilities of the range
// stay in shared memory from the mass phase to the compaction.  A prologue kernel
// (k_qprep) forms q_idx = P_q q_pre per slice (float64 dot products) and q_rot = RoPE(q,
// L-1) for the attention, and clears the slice's selection state and histograms.
// Phases of k_select (the CTAs of one slice meet at three per-slice arrival counters;
// there is no grid-wide barrier):
//   score     per head: m = max_j l_hj, z = sum_j 2^(l_hj - m) over the range,
//             l_hj = log2(e) * idx_scale * <q_idx[h], idx_j>   (index read #1, HBM);
//   -- the slice's score statistics are complete --
//   mass      merge (m, z) over the slice's ranges -> M_h, Z_h; recompute l_hj (index
//             read #2, from L2), pi_j = sum_h 2^(l_hj - M_h) / (G Z_h), kept on chip; a
//             mass histogram over the top 12 bits of pi_j's bit pattern, masses as
//             integer multiples of 2^-63 so every sum is exact and order independent
//             (per range as a count and a sum of low significand bits per bin); then an
//             L2 prefetch of the sink and window K/V rows the attention reads next;
//   -- the slice's histogram is complete --
//   cut 1     every CTA reads the slice's histogram: total mass, target ceil(p * total)
//             (or k for top-k) and the bin b1 where the descending cumulative mass
//             reaches it;
//   threshold per range: the listed tokens above b1 counted, the elements of bin b1
//             appended as candidates with their round-A masses added to the slice's
//             second histogram;
//   -- the slice's candidates are complete --
//   refine    every CTA takes the exact cut from the candidates - the value tau and the
//             position up to which tokens equal to tau are kept (lowest positions first)
//             - by an on-chip sort when they are few, else by more radix rounds, and its
//             range's offset in the list from the counts above b1 and the kept
//             candidates before it;
//   compact   per range: kept positions outside sinks/window, ascending.
// Block mode (the block-granular variant, a second instantiation): the ranges are cut at
// kBlock-token block boundaries, the mass phase keeps and histograms each block's mass
// (the float32 sum of its tokens' pi) instead of the tokens', the threshold and refine
// steps rank blocks and count their listed tokens, and compact lists every token of a
// kept block.  The blocks follow the chunk routing of the "Hierarchical Global
// Attention" summary, Central mechanism §4.
// One launch replaces a chain of small kernels whose fixed launch cost dominated.  The
// arrival waits are polled with a clock budget; on timeout they set a device status bit
// and the kernel leaves without hanging.  The launch is cooperative, so all CTAs are
// resident together.
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
// shared memory), each scaled by `scale` (log2(e) * idx_scale) in float32 before the
// split, so the tensor cores return log2-domain logits directly.
template <int G>
__device__ __forceinline__ void qidx_frag(const float* qbase, float scale, uint32_t (&qb)[IdxTiles<G>::NT][2]) {
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
        const float x = qbase[head * kIdxDim + 4 * t4 + e] * scale;
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

// Log2-domain logits of tokens gid (ra) and gid + 8 (rb) for the lane's heads (the
// scale is in the fragments).
template <int G>
__device__ __forceinline__ void group_logits(const uint2& ra, const uint2& rb,
                                             const uint32_t (&qb)[IdxTiles<G>::NT][2],
                                             float (&lg)[IdxTiles<G>::NH][2]) {
  const uint32_t a[4] = {ra.x, rb.x, ra.y, rb.y};
  float c[IdxTiles<G>::NT][4];
#pragma unroll
  for (int t = 0; t < IdxTiles<G>::NT; ++t) {
    c[t][0] = c[t][1] = c[t][2] = c[t][3] = 0.f;
    mma16816(c[t], a, qb[t][0], qb[t][1]);
  }
  if (G <= 4) {
    lg[0][0] = (c[0][0] + c[0][1]) + c[1][0];
    lg[0][1] = (c[0][2] + c[0][3]) + c[1][2];
  } else {
    lg[0][0] = (c[0][0] + c[0][1]) + c[IdxTiles<G>::NT - 1][0];
    lg[0][1] = (c[0][2] + c[0][3]) + c[IdxTiles<G>::NT - 1][2];
    lg[IdxTiles<G>::NH - 1][0] = (c[1][0] + c[1][1]) + c[IdxTiles<G>::NT - 1][1];
    lg[IdxTiles<G>::NH - 1][1] = (c[1][2] + c[1][3]) + c[IdxTiles<G>::NT - 1][3];
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



// ------------------------------------------------------------------ per-slice synchronisation
// The phases of a slice wait only for the CTA ranges of that slice: a range arrives at
// the slice's counter for a phase once its output of that phase is stored (the counters
// are reset by the prologue kernel before every launch), and a phase that needs the
// whole slice waits until every range of the slice has arrived.  The launch is
// cooperative, so every CTA that may be waited for is resident.
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s bound per wait

// This CTA's range arrives at counter ctr (called by every thread of the CTA): every
// thread fences its own writes of the phase, then one arrival for the CTA.
__device__ __forceinline__ void slice_arrive(unsigned* ctr) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) atomicAdd(ctr, 1u);
}

// Waits (thread 0, polled with back-off, bounded) until n ranges have arrived at ctr;
// returns false on every thread of the CTA if the wait gave up (the status word then
// holds kErrTimeout).
__device__ bool slice_wait(unsigned* ctr, unsigned n, unsigned* err, int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    volatile unsigned* w = ctr;
    if (*w < n) {
      const long long t0 = clock64();
      unsigned ns = 32;
      while (*w < n) {
        if (clock64() - t0 > kWaitCycles) {
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

// ------------------------------------------------------------------ shared memory
constexpr int kWarps = kSelThreads / 32;
constexpr int kGroupBatch = 4;    // groups per warp loaded together (8 spills at 64 registers)
constexpr int kPiCap = 16 * kSelThreads;   // probabilities of a range kept on chip (dynamic shared memory)
constexpr int kPiBytes = kPiCap * 4;
constexpr int kSmallList = 2048;  // candidates of the round-A cut digit kept on chip by the refine step
constexpr int kTieCap = 256;      // candidates equal to the cut value ranked directly
constexpr int kRefBatch = 8;      // candidate loads per thread issued together by the refine step

struct SmemPro { double cs[kHeadDim / 2], sn[kHeadDim / 2]; };
struct SmemScore { float2 red[kSelThreads / 32][kMaxGroup]; };
struct SmemMass { unsigned cnt[kBins1], low[kBins1]; float Mh[kMaxGroup]; };
struct SmemRefine {
  uint2 small[kSmallList];            // candidates of the round-A cut digit (bits, element)
  unsigned hc[512];                   // radix round: count per digit
  unsigned hl[512];                   // radix round: sum of the bits below the digit
  int tie[kTieCap];                   // positions of the candidates equal to the cut value
  int wcnt[kSelThreads / 32];         // per-warp counts
  int wabv[kSelThreads / 32];         // per-warp counts of listed tokens above the cut bin
};
union SelSmem {   // (compact_segment stages kThrRun * kSelThreads ints here)
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
  int L, b1, cut_bin, pos_cut, off, ok, digit, ntie;
  unsigned tau, ncand, nsmall, cbase;
  unsigned long long cut_above, above, target, m_above;
};

// Unit coordinates: retrieval slice y of this launch -> (b, g, s) and its retrieval
// slice index over the whole batch, yg (launches over part of a batch start at
// sequence P.b_base).
struct Unit {
  int b, g, s, yg;
};
__device__ __forceinline__ Unit unit_of(const StepParams& P, int y) {
  Unit u;
  u.b = P.b_base + y / P.n_ret;
  u.g = P.ret_heads[y % P.n_ret];
  u.s = u.b * P.Hkv + u.g;
  u.yg = P.b_base * P.n_ret + y;
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
// the attention kernels after this launch.
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
  __syncthreads();   // sm.cs / sm.sn and sc.L are reused
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

// Round-A histogram of slice s (candidates of its round-1 cut bin by bits 17..9): 512
// counts, then 512 sums of bits 8..0.  It lives in the slice's round-2 histogram row,
// which the one-GPU selection does not otherwise use.
__device__ __forceinline__ unsigned* hist_a(const StepParams& P, int s) {
  return reinterpret_cast<unsigned*>(P.ws.hist2 + (size_t)s * kBins2);
}


// ------------------------------------------------------------------ query prologue kernel
// Launched before the selection kernel: one CTA per (b, kv head) slice forms, for a
// retrieval slice, q_idx = P_q q_pre (float64 dot products) and resets its selection
// state (arrival counters included) and histograms (a streaming slice's selection count
// is 0); in decode calls a second CTA per slice forms q_rot for the slice's G heads at
// the same time.  Forming these once per slice lets every CTA of the selection kernel
// start streaming index rows at once.
template <typename T, int G>
__global__ void __launch_bounds__(kSelThreads) k_qprep(StepParams P) {
  __shared__ SmemPro sm;
  __shared__ SelScalars sc;
  // CTAs [0, n_slices) form q_idx and reset the selection state; decode calls add CTAs
  // [n_slices, 2 n_slices) for q_rot, so the two chains run side by side
  const bool rot = (int)blockIdx.x >= P.n_slices;
  const int s = P.b_base * P.Hkv + (int)blockIdx.x - (rot ? P.n_slices : 0), b = s / P.Hkv, g = s % P.Hkv,
            tid = threadIdx.x;
  // the selection kernel (launched with programmatic stream serialization) may start
  // its CTAs and their first index-row loads now; it waits for this grid's completion
  // before it reads anything written here
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  if (rot) {
    qrot_slice<T>(P, sm, sc, s);
    return;
  }
  if (P.is_ret[g]) {
    if (tid == 0) {
      SliceState z;
      z.target = z.m_above = 0ull;
      z.b1 = -1;
      z.count = 0;
      z.arr_score = z.arr_mass = z.arr_thr = 0u;
      z.ncand = 0u;
      P.ws.st[s] = z;
    }
    unsigned long long* h1 = P.ws.hist1 + (size_t)s * kBins1;
    for (int i = tid; i < kBins1; i += kSelThreads) h1[i] = 0ull;
    unsigned* ha = hist_a(P, s);
    for (int i = tid; i < 1024; i += kSelThreads) ha[i] = 0u;
    compute_qidx<T, G>(P, b, g, sc);
    if (tid < G * kIdxDim) P.ws.q_idx[((size_t)b * P.Hq + (size_t)g * G) * kIdxDim + tid] = sc.qsm[tid];
  } else if (tid == 0) {
    P.ws.st[s].count = 0;
    if (P.sel_count) P.sel_count[s] = 0;
  }
}

// ------------------------------------------------------------------ work partition
// The retrieval slices' capacity (max_seq_len tokens each, as ngc 16-token groups;
// slice y = b * n_ret + r owns global groups [y ngc, (y+1) ngc)) is split into equal
// contiguous group ranges, one per CTA, so every SM of a full-occupancy grid gets the
// same share.  A range may span slices; groups past a sequence's length are empty.
// Ranges are cut at multiples of q groups (q = 1, or kBlock / 16 in block mode so that
// no block is split; ngc is then a multiple of q): CTA c covers groups
// [q floor(c Q / nb), q floor((c+1) Q / nb)), Q = n_rs ngc / q.
// When the grid gives every retrieval slice the same whole number of CTAs, cps, the
// same partition reduces to 32-bit arithmetic computed once per CTA: CTA c = y cps + k
// covers local groups [q floor(k qs / cps), q floor((k+1) qs / cps)) of slice y,
// qs = ngc / q.  launch_select sizes every launch so (it splits larger batches); the
// general split stays correct for any grid.
template <bool BLK>
struct Ranges {
  static constexpr int q = BLK ? kBlock / 16 : 1;
  long long ngc, quanta;
  int nb;
  int cps;                 // CTAs per slice (0: ranges may span slices)
  int me;                  // this CTA's range index
  int y_me, l0_me, l1_me;  // with cps: this CTA's one segment
  __device__ __forceinline__ Ranges(const StepParams& P) {
    ngc = ((long long)P.Lcap + 16 * q - 1) / (16 * q) * q;
    const int n_rs = P.B * P.n_ret;
    quanta = (long long)n_rs * (ngc / q);
    nb = (int)gridDim.x;
    cps = (n_rs > 0 && nb % n_rs == 0) ? nb / n_rs : 0;
    me = (int)blockIdx.x;
    y_me = l0_me = l1_me = 0;
    if (cps) {
      const long long qs = ngc / q;
      y_me = me / cps;
      const int k = me - y_me * cps;
      l0_me = (int)((long long)k * qs / cps) * q;
      l1_me = (int)((long long)(k + 1) * qs / cps) * q;
    }
  }
  __device__ __forceinline__ long long begin(int c) const { return (long long)c * quanta / nb * q; }
  // CTA whose range holds global group g
  __device__ __forceinline__ int owner(long long g) const { return (int)(((g / q + 1) * nb - 1) / quanta); }
  __device__ __forceinline__ int first_cta(int y) const { return cps ? y * cps : owner((long long)y * ngc); }
  __device__ __forceinline__ int last_cta(int y) const {
    return cps ? y * cps + cps - 1 : owner((long long)(y + 1) * ngc - 1);
  }
  // range-relative group offset of slice y's group 0
  __device__ __forceinline__ long long seg_origin(int y) const {
    return cps ? -(long long)l0_me : (long long)y * ngc - begin(me);
  }
};
// Per-range values of slice y (statistics, counts, offsets) live at slot cta + y: the
// CTAs of slice y are consecutive and the last one of y may be the first one of y + 1,
// so the slots of different slices never overlap (at most nb + n_rs of them).
__device__ __forceinline__ size_t stats_slot(int cta, int y) { return (size_t)cta + (size_t)y; }

// Visits the CTA's range as segments f(y, l0, l1) of local groups [l0, l1) of slice y.
template <class RT, class F>
__device__ __forceinline__ void for_each_segment(const RT& R, F&& f) {
  if (R.cps) {   // one segment, no 64-bit division, no loop state kept live across f
    f(R.y_me, R.l0_me, R.l1_me);
    return;
  }
  const long long ge = R.begin(R.me + 1);
  for (long long g = R.begin(R.me); g < ge;) {
    const int y = (int)(g / R.ngc);
    const long long gend = min(ge, (long long)(y + 1) * R.ngc);
    f(y, (int)(g - (long long)y * R.ngc), (int)(gend - (long long)y * R.ngc));
    g = gend;
  }
}

// Probabilities of the CTA's range: element e of a segment's slice (token e, or block e
// in block mode) lives on chip at its offset from the range's first token (or block),
// or, past the first kPiCap elements of the range, in the global rows
// [slices][pi_stride].  One view per segment: t0 = the range-relative offset of the
// slice's element 0, s = the slice.
extern __shared__ float s_pi[];   // dynamic shared memory of the selection kernel: kPiCap floats
struct PiSeg {
  int t0, s;
};
template <bool BLK>
__device__ __forceinline__ PiSeg pi_seg(const Ranges<BLK>& R, int y, int s) {
  const long long t0 = 16 * R.seg_origin(y);
  PiSeg v;
  v.t0 = (int)(BLK ? t0 / kBlock : t0);
  v.s = s;
  return v;
}
__device__ __forceinline__ void pi_store(const StepParams& P, PiSeg ps, int e, float v) {
  const int loc = ps.t0 + e;
  if (loc < kPiCap) s_pi[loc] = v;
  else P.ws.pi[(size_t)ps.s * P.ws.pi_stride + e] = v;
}
__device__ __forceinline__ float pi_load(const StepParams& P, PiSeg ps, int e) {
  const int loc = ps.t0 + e;
  return loc < kPiCap ? s_pi[loc] : __ldcg(P.ws.pi + (size_t)ps.s * P.ws.pi_stride + e);
}
// elements e .. e + 3 (e a multiple of 4; token mode: t0 is a multiple of 16, so the
// four sit on one side of kPiCap and are 16-byte aligned on either side)
__device__ __forceinline__ float4 pi_load4(const StepParams& P, PiSeg ps, int e) {
  const int loc = ps.t0 + e;
  return loc < kPiCap ? *reinterpret_cast<const float4*>(s_pi + loc)
                      : __ldcg(reinterpret_cast<const float4*>(P.ws.pi + (size_t)ps.s * P.ws.pi_stride + e));
}

// ------------------------------------------------------------------ score phase
// One range of slice y: per head m = max_j l_hj, z = sum_j 2^(l_hj - m) over the tokens
// of local groups [l0, l1), l_hj = log2(e) * idx_scale * <q_idx[h], idx_j>.  Warp w takes
// groups l0 + w, l0 + w + 8, ..., kGroupBatch at a time; the first batch is requested
// before the query index vectors are read (bounded by the call's max length; rows past
// the sequence are masked).
template <int G>
__device__ void score_segment(const StepParams& P, SmemScore& sm, SelScalars& sc, int me, int y, int l0, int l1) {
  constexpr int NH = IdxTiles<G>::NH, U = kGroupBatch;
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, t4 = lane & 3, gid = lane >> 2;
  const uint2* rows = reinterpret_cast<const uint2*>(idx_rows(P, un.yg, un.s));
  const uint64_t pol = l2_policy_keep();
  uint2 ra[U], rb[U];
  {
    const int jpf = min(P.Lcap, 16 * l1);
#pragma unroll
    for (int u = 0; u < U; ++u) load_group(rows, 16 * (l0 + warp + kWarps * u), jpf, pol, ra[u], rb[u]);
  }
  // from here on the prologue kernel's writes (state reset, q_idx) are read: wait for
  // its completion (returns at once when this launch did not overlap it)
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // the sequence length and the query index vectors (formed by the prologue kernel)
  // are requested behind the first batch; one CTA barrier publishes them
  __syncthreads();   // earlier readers of sc.L and sc.qsm are done
  int64_t len_raw = 0;
  if (tid == 0) len_raw = P.seq_lens[un.b];
  if (tid < G * kIdxDim) sc.qsm[tid] = __ldcg(&P.ws.q_idx[((size_t)un.b * P.Hq + (size_t)un.g * G) * kIdxDim + tid]);
  if (tid == 0) {
    if (len_raw < 1 || len_raw > P.Lcap) {
      atomicOr(P.ws.dev_err, kErrSeqLen);
      len_raw = len_raw < 1 ? 1 : P.Lcap;
    }
    sc.L = (int)len_raw;
  }
  __syncthreads();
  const int L = sc.L;
  float2* out = P.ws.stats + stats_slot(me, y) * G;
  if (16 * l0 >= L) {
    if (tid < G) out[tid] = make_float2(-INFINITY, 0.f);
    return;
  }
  uint32_t qb[IdxTiles<G>::NT][2];
  qidx_frag<G>(sc.qsm, P.idx_scale_log2, qb);
  const int jend = min(L, 16 * l1);
  // two independent online accumulators per head (tokens gid and gid + 8)
  float m[NH][2], z[NH][2];
#pragma unroll
  for (int h = 0; h < NH; ++h) { m[h][0] = m[h][1] = -INFINITY; z[h][0] = z[h][1] = 0.f; }
  for (int gb = l0; 16 * gb < jend; gb += kWarps * U) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = 16 * (gb + warp + kWarps * u);
      float lg[NH][2];
      group_logits<G>(ra[u], rb[u], qb, lg);
      // refill the consumed slot with the same slot of the next batch
      load_group(rows, 16 * (gb + kWarps * U + warp + kWarps * u), jend, pol, ra[u], rb[u]);

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
  __syncthreads();   // sm.red, sc.L and sc.qsm are reused by the next segment
}

// ------------------------------------------------------------------ cut 1 (per range)
// Every CTA of a slice takes the slice's round-1 cut itself from the complete round-1
// histogram (32 KB, read from L2): thread t loads the kPer = 4096 / threads consecutive
// bins 4095 - kPer t - k (k = 0..kPer-1, descending), a warp scan and a scan of the warp
// totals give the mass ahead of each thread's bins, and the thread whose bins hold the
// crossing walks them: the
// total mass, the target ceil(p * total) (or k for top-k) and the bin b1 where the
// descending cumulative mass reaches it (-1: keep every token).  Results in sc.b1,
// sc.target, sc.m_above (the mass of all bins above b1) and sc.L (the sequence length,
// read in the same round trip); the slice's first CTA also stores the cut for the refine
// step of every range.
__device__ void cut1_range(const StepParams& P, SelScalars& sc, int y, bool lead) {
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPer = kBins1 / kSelThreads, kVec = kPer / 2;   // bins per thread, 16-byte words
  const ulonglong2* h = reinterpret_cast<const ulonglong2*>(P.ws.hist1 + (size_t)un.s * kBins1 + kBins1 - kPer * (tid + 1));
  ulonglong2 hv[kVec];
#pragma unroll
  for (int k = 0; k < kVec; ++k) hv[k] = __ldcg(h + k);   // bins 4096 - kPer (t + 1) .. 4095 - kPer t, ascending
  if (tid == 0) sc.L = load_len(P.seq_lens, un.b, P.Lcap, P.ws.dev_err);
  unsigned long long mine = 0ull;
#pragma unroll
  for (int k = 0; k < kVec; ++k) mine += hv[k].x + hv[k].y;
  unsigned long long x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) sc.shl[warp] = x;
  if (tid == 0) sc.cut_bin = -1;
  __syncthreads();
  unsigned long long wbase = 0ull, tot = 0ull;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned long long t = sc.shl[w];
    wbase += w < warp ? t : 0ull;
    tot += t;
  }
  unsigned long long target = tot;
  bool keep_all = P.keep_all || tot == 0ull;
  if (!keep_all) {
    // top-k: the k-th token (total = the number of tokens); top-p: the mass ceil(p total)
    target = P.topk > 0 ? (unsigned long long)P.topk : (unsigned long long)ceil((double)P.p * (double)tot);
    if (target < 1ull) target = 1ull;
    keep_all = target >= tot && P.topk > 0 ? true : target > tot;   // k >= L keeps all
  }
  if (!keep_all) {
    unsigned long long cum = wbase + x - mine;   // mass of the bins above this thread's
    if (cum < target && cum + mine >= target) {
#pragma unroll
      for (int k = kVec - 1; k >= 0; --k) {
        const unsigned long long b[2] = {hv[k].y, hv[k].x};   // descending: bin 2k + 1, then 2k
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (cum < target && cum + b[e] >= target) {
            sc.cut_bin = kBins1 - kPer * (tid + 1) + 2 * k + 1 - e;
            sc.cut_above = cum;
          }
          cum += b[e];
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    sc.b1 = keep_all ? -1 : sc.cut_bin;   // a search that fails keeps every token
    sc.target = target;
    sc.m_above = sc.b1 >= 0 ? sc.cut_above : 0ull;
    if (lead) {
      SliceState* st = P.ws.st + un.s;
      st->target = sc.target;
      st->b1 = sc.b1;
      st->m_above = sc.m_above;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ mass phase
// One range of slice y: M_h, Z_h merged from the slice's range statistics (fixed
// order), the logits recomputed (index read #2, mostly from L2),
// pi_j = sum_h 2^(l_hj - M_h) / (G Z_h), evaluated as sum_h 2^(l_hj - M'_h) with
// M'_h = M_h + log2(G Z_h), kept (PiSeg), and its mass added to the slice's
// round-1 histogram via a per-range shared histogram of counts and low significand
// bits (32-bit atomics; a range holds at most kMaxRangeGroups groups, so a bin's
// low-bit sum stays below 2^32).
// Block mode (BLK): warp w's batch is the four consecutive groups of one kBlock-token
// block; the block's mass (the float32 sum of its tokens' pi, in a fixed order) is
// kept for the block and histogrammed instead of the tokens'.
constexpr int kMaxRangeGroups = 1024;   // 16384 tokens: 16384 * 2^18 = 2^32
static_assert(kGroupBatch * 16 == kBlock, "block mode: one warp batch is one block");
template <int G, bool BLK>
__device__ bool mass_segment(const StepParams& P, SmemMass& sm, SelScalars& sc, const Ranges<BLK>& R,
                             int y, int l0, int l1, bool wait_scores, unsigned n_ranges) {
  constexpr int NH = IdxTiles<G>::NH, U = kGroupBatch;
  const Unit un = unit_of(P, y);
  const PiSeg ps = pi_seg<BLK>(R, y, un.s);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
  const uint2* rows = reinterpret_cast<const uint2*>(idx_rows(P, un.yg, un.s));
  const uint64_t pol = l2_policy_drop();
  // local group of batch slot u at batch base gb
  auto grp = [&](int gb, int u) { return BLK ? gb + U * warp + u : gb + warp + kWarps * u; };
  uint2 ra[U], rb[U];
  {
    const int jpf = min(P.Lcap, 16 * l1);
#pragma unroll
    for (int u = 0; u < U; ++u) load_group(rows, 16 * grp(l0, u), jpf, pol, ra[u], rb[u]);
  }
  // every range of the slice has stored its statistics (the first batch is in flight)
  if (wait_scores && !slice_wait(&P.ws.st[un.s].arr_score, n_ranges, P.ws.dev_err, &sc.ok)) return false;
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
      sm.Mh[warp] = m + log2f((float)G * z);
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
  if (16 * l0 >= L) return true;
  uint32_t qb[IdxTiles<G>::NT][2];
  qidx_frag<G>(sc.qsm, P.idx_scale_log2, qb);
  float M[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const int head = lane_head<G>(t4, h);
    M[h] = head < G ? sm.Mh[head] : INFINITY;   // lanes of absent heads contribute nothing
  }
  const int jend = min(L, 16 * l1);
  static_assert(kGroupBatch % 2 == 0, "token mode reduces the batch's groups in pairs");
  for (int gb = l0; 16 * gb < jend; gb += kWarps * U) {
    float bsum = 0.f;
    float pa[2] = {0.f, 0.f};   // token mode: the first group of the current pair
    int ja = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = 16 * grp(gb, u);
      float lg[NH][2];
      group_logits<G>(ra[u], rb[u], qb, lg);
      // refill the consumed slot with the same slot of the next batch
      load_group(rows, 16 * grp(gb + kWarps * U, u), jend, pol, ra[u], rb[u]);

      // pi = sum over the group's heads of 2^(l - M_h) / (G Z_h): lane-local heads first,
      // then the 4 lanes of a token (fixed order, identical result in every lane)
      float pr[2];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (G < 4 && M[h] == INFINITY) continue;   // lanes of absent heads (G < 4) add nothing
          acc += ex2(lg[h][cc] - M[h]);
        }
        pr[cc] = acc;
      }
      if (BLK) {
        // every lane ends with both tokens' sums
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          pr[cc] += __shfl_xor_sync(kFull, pr[cc], 1);
          pr[cc] += __shfl_xor_sync(kFull, pr[cc], 2);
        }
        bsum += (j + gid < jend ? pr[0] : 0.f) + (j + gid + 8 < jend ? pr[1] : 0.f);
      } else {
        // two groups (A = slot u - 1, B = slot u) reduced together over the 4 lanes of a
        // token row, so that every lane ends with one of the pair's 32 tokens: the
        // exchange with lane t4 ^ 2 leaves lanes t4 < 2 with group A's two partial sums
        // and lanes t4 >= 2 with group B's, the exchange with t4 ^ 1 leaves lane t4 with
        // token gid (t4 even) or gid + 8 (t4 odd) of its group, summed in a fixed order
        if ((u & 1) == 0) {
          pa[0] = pr[0];
          pa[1] = pr[1];
          ja = j;
        } else {
          const bool hi2 = (t4 & 2) != 0, odd = (t4 & 1) != 0;
          const float v0 = (hi2 ? pr[0] : pa[0]) + __shfl_xor_sync(kFull, hi2 ? pa[0] : pr[0], 2);
          const float v1 = (hi2 ? pr[1] : pa[1]) + __shfl_xor_sync(kFull, hi2 ? pa[1] : pr[1], 2);
          const float v = (odd ? v1 : v0) + __shfl_xor_sync(kFull, odd ? v0 : v1, 1);
          const int jt = (hi2 ? j : ja) + gid + 8 * (t4 & 1);
          if (jt < jend) {
            pi_store(P, ps, jt, v);
            const unsigned bits = __float_as_uint(v);
            const unsigned d = min(bits >> 18, (unsigned)(kBins1 - 1));
            atomicAdd(&sm.cnt[d], 1u);
            atomicAdd(&sm.low[d], bits & 0x3ffffu);
          }
        }
      }
    }
    if (BLK) {
      // every lane of a token quad holds the same sums: add over the 8 token rows
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) bsum += __shfl_xor_sync(kFull, bsum, o);
      const int jb = 16 * grp(gb, 0);
      if (lane == 0 && jb < jend) {
        pi_store(P, ps, jb / kBlock, bsum);
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
  return true;
}

// ------------------------------------------------------------------ L2 prefetch
// Bulk prefetch into L2 (no data returned to the SM): the rows are read again, from
// L2, by the attention kernel that follows this one.
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

// The sink and window K/V rows of every slice (streaming slices of the compact layout:
// their ring), which the attention reads whatever the selection keeps, prefetched in
// pieces of up to 64 KB.  Thread t of CTA c takes piece c + t nb, so the pieces spread
// over every CTA.  Decode calls only (select-only calls pass no caches).
template <typename T>
__device__ void prefetch_attended_rows(const StepParams& P) {
  if (!P.k_cache) return;
  constexpr long long kRow = kHeadDim * sizeof(T);
  constexpr long long kPiece = 65536;
  const long long span = (long long)(P.compact ? max(P.window, P.ring) : P.window) * kRow;
  const int per_slice = 2 * (1 + (int)((span + kPiece - 1) / kPiece));   // K and V: sinks + window pieces
  const long long total = (long long)P.n_slices * per_slice;
  for (long long p = blockIdx.x + (long long)threadIdx.x * gridDim.x; p < total;
       p += (long long)gridDim.x * blockDim.x) {
    const int s = P.b_base * P.Hkv + (int)(p / per_slice), r = (int)(p % per_slice), piece = r >> 1;
    int64_t L = P.seq_lens[s / P.Hkv];
    L = L < 1 ? 1 : (L > P.Lcap ? P.Lcap : L);
    const KvSlice<T> sl = kv_slice<T>(P, s);
    const char* base = reinterpret_cast<const char*>((r & 1) ? sl.v : sl.k);
    long long lo, hi;   // byte range in the slice's rows
    if (sl.ring) {      // ring rows [0, min(L, ring))
      if (piece == 0) continue;
      lo = (long long)(piece - 1) * kPiece;
      hi = min((long long)min((int64_t)P.ring, L) * kRow, lo + kPiece);
    } else {
      const SinkWindow sw((int)L, P.n_sink, P.window);
      if (piece == 0) {
        lo = 0;
        hi = (long long)sw.n_s * kRow;
      } else {
        lo = (long long)sw.w_lo * kRow + (long long)(piece - 1) * kPiece;
        hi = min(L * kRow, lo + kPiece);
      }
    }
    if (hi > lo) prefetch_l2(base + lo, (unsigned)(hi - lo));
  }
}

// ------------------------------------------------------------------ threshold phase
// Number of positions of [lo, hi) outside sinks and window.
__device__ __forceinline__ int listed_in(const SinkWindow& sw, int lo, int hi) {
  if (hi <= lo) return 0;
  const int a = max(lo, sw.n_s), b = min(hi, sw.w_lo);
  return b > a ? b - a : 0;
}

// Listed positions (outside sinks and window) of element e: token e, or block e in
// block mode.
template <bool BLK>
__device__ __forceinline__ int listed_of(const SinkWindow& sw, int L, int e) {
  if (!BLK) return sw.always(e) ? 0 : 1;
  return listed_in(sw, e * kBlock, min(L, (e + 1) * kBlock));
}

// Elements (tokens, or blocks in block mode) of the segment of local groups [l0, l1) of
// a slice of length L: [e0, e1).
template <bool BLK>
__device__ __forceinline__ void seg_elems(int L, int l0, int l1, int& e0, int& e1) {
  const int j0 = 16 * l0, j1 = min(L, 16 * l1);
  e0 = BLK ? j0 / kBlock : j0;
  e1 = j1 <= j0 ? e0 : (BLK ? (j1 + kBlock - 1) / kBlock : j1);
}

// One range of slice y (after cut1_range of y): the elements of bin b1 are the slice's
// candidates; the listed tokens of the elements above b1 (every element when b1 < 0) are
// kept whatever the exact cut, and their count is stored at the range's slot.  Rounds
// of kThrRun consecutive elements per thread (token mode; one block per thread in block
// mode), held in registers: one CTA scan gives each thread's candidate offset and the
// round's totals, one atomic per round reserves the candidates' slots in the slice's
// candidate array, and the candidates (bits, element) are written in range order and
// added to the slice's round-A histogram (bits 17..9: count and sum of bits 8..0).
constexpr int kThrRun = 16;
template <bool BLK>
__device__ void threshold_segment(const StepParams& P, SelScalars& sc, SmemRefine& sm, const Ranges<BLK>& R, int y,
                                  int l0, int l1) {
  (void)sm;
  const Unit un = unit_of(P, y);
  const PiSeg ps = pi_seg<BLK>(R, y, un.s);
  const int tid = threadIdx.x;
  const int L = sc.L, b1 = sc.b1;   // from cut1_range (b1 < 0: keep everything)
  const SinkWindow sw(L, P.n_sink, P.window);
  int e0, e1;
  seg_elems<BLK>(L, l0, l1, e0, e1);
  constexpr int kPer = BLK ? 1 : kThrRun;
  uint2* cand = P.ws.cand + (size_t)un.s * P.Lmax;
  unsigned* ha = hist_a(P, un.s);
  int above_all = 0;
  for (int k0 = e0; k0 < e1; k0 += kSelThreads * kPer) {   // whole CTA: the scan below
    const int eb = k0 + kPer * tid;
    unsigned bits[kPer];
    unsigned cmask = 0u;
    int above = 0;
    if (eb < e1) {
      if (BLK) {
        bits[0] = __float_as_uint(pi_load(P, ps, eb));
      } else {
#pragma unroll
        for (int q4 = 0; q4 < kPer / 4; ++q4) {   // eb is a multiple of 16: aligned 16-byte words
          const float4 v = pi_load4(P, ps, eb + 4 * q4);
          bits[4 * q4] = __float_as_uint(v.x);
          bits[4 * q4 + 1] = __float_as_uint(v.y);
          bits[4 * q4 + 2] = __float_as_uint(v.z);
          bits[4 * q4 + 3] = __float_as_uint(v.w);
        }
      }
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        if (eb + q < e1) {
          const int bin = (int)min(bits[q] >> 18, (unsigned)(kBins1 - 1));
          if (bin == b1) cmask |= 1u << q;
          if (bin > b1) above += listed_of<BLK>(sw, L, eb + q);
        }
      }
    }
    // candidates before this thread (low half) and the round's totals (candidates low,
    // listed tokens above b1 high)
    unsigned long long tot;
    const unsigned long long pre =
        block_excl_scan<unsigned long long>(((unsigned long long)above << 32) | (unsigned)__popc(cmask), sc.shl, &tot);
    above_all += (int)(tot >> 32);
    const unsigned n_round = (unsigned)tot;
    if (n_round == 0u) continue;   // uniform: the totals are the CTA's
    if (tid == 0) sc.cbase = atomicAdd(&P.ws.st[un.s].ncand, n_round);
    __syncthreads();
    unsigned slot = sc.cbase + (unsigned)pre;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      if (cmask >> q & 1u) {
        cand[slot++] = make_uint2(bits[q], (unsigned)(eb + q));
        const unsigned d = (bits[q] >> 9) & 511u;
        atomicAdd(ha + d, 1u);
        atomicAdd(ha + 512 + d, bits[q] & 511u);
      }
    }
    __syncthreads();   // sc.cbase is rewritten by the next round
  }
  if (tid == 0) P.ws.seg_cnt[stats_slot(R.me, y)] = above_all;
}

// ------------------------------------------------------------------ refine (per range)
// Mass of the round-A/B digit d of the cut bin b1: count c, sum l of the bits below the
// digit, significand bits above them sig (implicit bit included).  Every candidate
// shares b1's exponent field, so the digit's mass is the exact sum of its candidates'
// mass_q: (sig * c + l) << (e - 87) (0 for e < 87), or c for top-k.
__device__ __forceinline__ unsigned long long digit_mass(const StepParams& P, int b1, unsigned sig, unsigned c,
                                                         unsigned l) {
  if (P.topk > 0) return c;
  int e = b1 >> 5;
  if (e < kMassMinExp || c == 0u) return 0ull;
  e = e > 127 ? 127 : e;
  return ((unsigned long long)sig * c + l) << (e - kMassMinExp);
}

// The digit d of [0, 512) (visited from 511 down) where base plus the cumulative mass of
// the digits above it first reaches target; sc.digit (left as it was if never; callers
// set -1 first) and sc.above (the mass ahead of d).  sig_of(d) gives the digit's
// significand bits.  Called by every thread of the CTA: thread t takes digits
// 511 - kDPer t - k, one CTA scan orders them.
template <class SIG>
__device__ void digit_cut_desc(const StepParams& P, const SmemRefine& sm, SelScalars& sc, int b1, SIG sig_of,
                               unsigned long long base, unsigned long long target) {
  constexpr int kDPer = 512 / kSelThreads;
  static_assert(kDPer * kSelThreads == 512, "the CTA covers the 512 digits");
  const int tid = threadIdx.x;
  unsigned long long m[kDPer], sum = 0ull;
#pragma unroll
  for (int k = 0; k < kDPer; ++k) {
    const int d = 511 - kDPer * tid - k;
    m[k] = digit_mass(P, b1, sig_of(d), sm.hc[d], sm.hl[d]);
    sum += m[k];
  }
  unsigned long long tot;
  unsigned long long cum = base + block_excl_scan<unsigned long long>(sum, sc.shl, &tot);
  if (cum < target && cum + sum >= target) {   // the crossing is in this thread's digits
#pragma unroll
    for (int k = 0; k < kDPer; ++k) {
      if (cum < target && cum + m[k] >= target) {
        sc.digit = 511 - kDPer * tid - k;
        sc.above = cum;
      }
      cum += m[k];
    }
  }
}

// Warp 0: the digit of [0, 256) (visited from 0 up) where base plus the count of the
// digits below it first reaches need; sc.digit (-1 if never) and sc.above (the count
// before it).
__device__ void digit_kth_asc(const SmemRefine& sm, SelScalars& sc, unsigned long long base,
                              unsigned long long need) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  unsigned sum = 0u;
  for (int k = 0; k < 8; ++k) sum += sm.hc[8 * lane + k];
  unsigned x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned t = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += t;
  }
  unsigned long long cum = base + x - sum;
  if (cum < need && cum + sum >= need) {
    for (int k = 0; k < 8; ++k) {
      const unsigned c = sm.hc[8 * lane + k];
      if (cum < need && cum + c >= need) {
        sc.digit = 8 * lane + k;
        sc.above = cum;
      }
      cum += c;
    }
  }
}

// Whether element e (token e, or block e) is kept by the cut (tau, pos_cut).
__device__ __forceinline__ bool kept_by_cut(unsigned bits, int e, unsigned tau, int pos_cut) {
  return bits > tau || (bits == tau && e <= pos_cut);
}

// The slice's exact cut and this range's place in the slice's list, taken by every CTA of
// the slice for itself once every range has stored its candidates and its count of
// listed tokens above the round-1 bin b1.  All tokens above b1 are kept; among the
// candidates of b1, in (pi desc, position asc) order, a candidate is kept while the mass
// ranked ahead of it (m_above plus the candidates before it) is below the target.
// Round A: the round-A histogram (bits 17..9, exact masses from counts and sums of the
// lower bits) gives the digit dA holding the cut.  One pass over the slice's candidate
// array gathers the candidates of dA on chip; round B over those (bits 8..0) gives the
// cut value tau and the mass above it; if only some of the candidates equal to tau are
// needed, the lowest positions are kept: ranked directly when they are few, else by
// three 8-bit rounds over their positions.  The kept candidates' listed tokens, those
// before this range and all of them, added to the ranges' counts above b1, give the
// range's offset and the slice's total.  A search that finds no cut (inconsistent
// masses) keeps every candidate of the last digit it reached and above, so the counts
// and the compaction's predicate still agree.  Results in sc.tau, sc.pos_cut, sc.L and
// sc.off; the slice's first CTA (lead) stores the total.
template <bool BLK>
__device__ void refine_range(const StepParams& P, SmemRefine& sm, SelScalars& sc, const Ranges<BLK>& R, int y,
                             int l0, int l1, bool lead) {
  const Unit un = unit_of(P, y);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SliceState* st = P.ws.st + un.s;
  const int first = R.first_cta(y), n_seg = R.last_cta(y) - first + 1, mine = R.me - first;
  const int* abv_row = P.ws.seg_cnt + stats_slot(first, y);
  constexpr int kSegPer = kMaxSelectGrid / kSelThreads;
  // one round trip: the cut state, the ranges' counts above b1, the round-A histogram
  // (1024 words over the CTA) and the first kRefBatch candidates per thread (read up to the
  // row's capacity, used below n)
  const unsigned long long target = __ldcg(&st->target);
  const unsigned long long mab = __ldcg(&st->m_above);
  const int b1 = __ldcg(&st->b1);
  const unsigned n_raw = __ldcg(&st->ncand);
  const int L = load_len(P.seq_lens, un.b, P.Lcap, P.ws.dev_err);
  const uint2* cand = P.ws.cand + (size_t)un.s * P.Lmax;
  const unsigned* ha = hist_a(P, un.s);
  int av[kSegPer];
#pragma unroll
  for (int k = 0; k < kSegPer; ++k) {
    const int c = tid + kSelThreads * k;
    av[k] = c < n_seg ? __ldcg(abv_row + c) : 0;
  }
  constexpr int kHaPer = 1024 / kSelThreads;
  unsigned hav[kHaPer];
#pragma unroll
  for (int k = 0; k < kHaPer; ++k) hav[k] = __ldcg(ha + tid + kSelThreads * k);
  uint2 c0[kRefBatch];
#pragma unroll
  for (int u = 0; u < kRefBatch; ++u) {
    const unsigned i = tid + kSelThreads * u;
    c0[u] = i < (unsigned)P.Lmax ? __ldcg(cand + i) : make_uint2(0u, 0u);
  }
  const unsigned n = b1 >= 0 ? n_raw : 0u;
  {
    int before = 0, all = 0;
#pragma unroll
    for (int k = 0; k < kSegPer; ++k) {
      all += av[k];
      before += tid + kSelThreads * k < mine ? av[k] : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(kFull, before, o);
      all += __shfl_xor_sync(kFull, all, o);
    }
    if (lane == 0) {
      sm.wcnt[warp] = before;
      sm.wabv[warp] = all;
    }
  }
#pragma unroll
  for (int k = 0; k < kHaPer; ++k) {   // words 0..511 counts, 512..1023 low sums
    const int w = tid + kSelThreads * k;
    if (w < 512) sm.hc[w] = hav[k]; else sm.hl[w - 512] = hav[k];
  }
  if (tid == 0) {
    sc.digit = -1;
    sc.pos_cut = INT_MAX;
    sc.ntie = 0;
    sc.nsmall = 0u;
  }
  __syncthreads();
  int ab_before = 0, ab_all = 0;   // listed tokens above b1: ranges before this one, all
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    ab_before += sm.wcnt[w];
    ab_all += sm.wabv[w];
  }
  // listed tokens of the kept candidates: before this range's first element, all
  int e0, e1;
  seg_elems<BLK>(L, l0, l1, e0, e1);
  const SinkWindow sw(L, P.n_sink, P.window);
  int pb = 0, pt = 0;
  auto kept_cand = [&](uint2 v) {
    const int c = listed_of<BLK>(sw, L, (int)v.y);
    pt += c;
    pb += (int)v.y < e0 ? c : 0;
  };
  // f(v) for every candidate, kRefBatch coalesced loads per thread issued together (the
  // first batch is the one already loaded)
  auto for_each_cand = [&](auto&& f) {
#pragma unroll
    for (int u = 0; u < kRefBatch; ++u)
      if (tid + kSelThreads * u < n) f(c0[u]);
    for (unsigned i0 = kSelThreads * kRefBatch; i0 < n; i0 += kSelThreads * kRefBatch) {
      uint2 v[kRefBatch];
#pragma unroll
      for (int u = 0; u < kRefBatch; ++u) {
        const unsigned i = i0 + tid + kSelThreads * u;
        v[u] = i < n ? __ldcg(cand + i) : make_uint2(0u, 0xffffffffu);
      }
#pragma unroll
      for (int u = 0; u < kRefBatch; ++u)
        if (v[u].y != 0xffffffffu) f(v[u]);
    }
  };
  unsigned tau = 0u;     // keep everything (b1 < 0)
  int pos_cut = INT_MAX;
  if (b1 >= 0) {
    const unsigned sig1 = (((unsigned)b1 & 31u) << 18) | 0x800000u;   // significand bits above bit 18
    digit_cut_desc(P, sm, sc, b1, [&](int d) { return sig1 | ((unsigned)d << 9); }, mab, target);
    __syncthreads();
    const int dA = sc.digit;
    const unsigned long long aboveA = sc.above;
    if (dA < 0) {
      tau = (unsigned)b1 << 18;   // no cut found: every candidate of b1 is kept
      for_each_cand(kept_cand);
    } else {
      const unsigned preB = ((unsigned)b1 << 9) | (unsigned)dA;
      tau = preB << 9;   // until the cut is found: every candidate of dA and above is kept
      // the candidates of digit dA gathered on chip; those above it are kept
      for_each_cand([&](uint2 v) {
        const unsigned d9 = v.x >> 9;
        if (d9 == preB) {
          const unsigned k = atomicAdd(&sc.nsmall, 1u);
          if (k < (unsigned)kSmallList) sm.small[k] = v;
        } else if (d9 > preB) {
          kept_cand(v);
        }
      });
      for (int d = tid; d < 512; d += kSelThreads) sm.hc[d] = sm.hl[d] = 0u;
      if (tid == 0) sc.digit = -1;
      __syncthreads();
      const unsigned ns = sc.nsmall;
      const bool fits = ns <= (unsigned)kSmallList;
      // f(v) for every candidate of digit dA: from the on-chip list, or (if it overflowed)
      // from the candidate array
      auto for_each_small = [&](auto&& f) {
        if (fits) {
          for (unsigned i = tid; i < ns; i += kSelThreads) f(sm.small[i]);
        } else {
          for_each_cand([&](uint2 v) { if ((v.x >> 9) == preB) f(v); });
        }
      };
      if (ns <= 32u) {
        // few: warp 0 sorts them by (pi desc, position asc) and keeps the prefix whose
        // mass ahead stays below the target; the last kept gives tau and pos_cut
        if (tid < 32) {
          unsigned long long key = 0ull, m = 0ull;
          if (lane < (int)ns) {
            const uint2 v = sm.small[lane];
            key = ((unsigned long long)v.x << 32) | (0xffffffffu - v.y);
            m = sel_mass(P, v.x);
          }
#pragma unroll
          for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
              const unsigned long long ok_ = __shfl_xor_sync(kFull, key, j);
              const unsigned long long om = __shfl_xor_sync(kFull, m, j);
              const bool desc = (lane & k) == 0, lower = (lane & j) == 0;
              // lower lane of the pair keeps the larger key in a descending run
              const bool take = lower == desc ? ok_ > key : ok_ < key;
              if (take) { key = ok_; m = om; }
            }
          }
          unsigned long long x = m;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long t = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += t;
          }
          const unsigned long long before = aboveA + x - m;
          const bool kept = key != 0ull && before < target;
          const unsigned kmask = __ballot_sync(kFull, kept);
          if (kmask != 0u && lane == 31 - __clz(kmask)) {   // the last kept
            sc.tau = (unsigned)(key >> 32);
            sc.pos_cut = (int)(0xffffffffu - (unsigned)key);
            sc.digit = 1;
          }
        }
        __syncthreads();
        if (sc.digit >= 0) {
          tau = sc.tau;
          pos_cut = sc.pos_cut;
        }
      } else {
        // round B: bits 8..0 of the candidates of digit dA
        for_each_small([&](uint2 v) { atomicAdd(&sm.hc[v.x & 511u], 1u); });
        __syncthreads();
        const unsigned sigA = sig1 | ((unsigned)dA << 9);
        digit_cut_desc(P, sm, sc, b1, [&](int d) { return sigA | (unsigned)d; }, aboveA, target);
        __syncthreads();
        if (sc.digit >= 0) {
          const int dB = sc.digit;
          tau = preB << 9 | (unsigned)dB;                 // fp32 bits of the cut value
          const unsigned long long m_gt = sc.above;       // mass strictly above tau
          const unsigned n_eq = sm.hc[dB];                 // candidates equal to tau
          const unsigned long long q_tau = sel_mass(P, tau);
          const unsigned long long need =
              (q_tau > 0ull && target > m_gt) ? (target - m_gt + q_tau - 1ull) / q_tau : ~0ull;
          __syncthreads();   // every read of sm.hc is done
          if (need < (unsigned long long)n_eq) {
            // keep the need lowest positions among the candidates equal to tau
            if (n_eq <= (unsigned)kTieCap) {
              for_each_small([&](uint2 v) {
                if (v.x == tau) sm.tie[atomicAdd(&sc.ntie, 1)] = (int)v.y;
              });
              __syncthreads();
              if (tid < (int)n_eq) {
                const int pmine = sm.tie[tid];
                unsigned r = 0u;
                for (unsigned k = 0; k < n_eq; ++k) r += sm.tie[k] < pmine ? 1u : 0u;
                if (r == (unsigned)need - 1u) sc.pos_cut = pmine;
              }
              __syncthreads();
            } else {
              unsigned pp = 0u;
              unsigned long long before = 0ull;
              bool ok = true;
              for (int sh = 16; sh >= 0 && ok; sh -= 8) {   // positions < 2^24
                for (int d = tid; d < 256; d += kSelThreads) sm.hc[d] = 0u;
                if (tid == 0) sc.digit = -1;
                __syncthreads();
                for_each_small([&](uint2 v) {
                  if (v.x == tau && (v.y >> (sh + 8)) == pp) atomicAdd(&sm.hc[(v.y >> sh) & 255u], 1u);
                });
                __syncthreads();
                digit_kth_asc(sm, sc, before, need);
                __syncthreads();
                ok = sc.digit >= 0;
                if (ok) {
                  pp = (pp << 8) | (unsigned)sc.digit;
                  before = sc.above;
                }
              }
              if (tid == 0) sc.pos_cut = ok ? (int)pp : INT_MAX;
              __syncthreads();
            }
            pos_cut = sc.pos_cut;
          }
        }
      }
      // the kept candidates of digit dA
      for_each_small([&](uint2 v) {
        if (kept_by_cut(v.x, (int)v.y, tau, pos_cut)) kept_cand(v);
      });
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    pb += __shfl_xor_sync(kFull, pb, o);
    pt += __shfl_xor_sync(kFull, pt, o);
  }
  __syncthreads();   // earlier readers of the scalars and of the per-warp counts are done
  if (lane == 0) {
    sm.wcnt[warp] = pb;
    sm.wabv[warp] = pt;
  }
  __syncthreads();
  if (tid == 0) {
    int kb = 0, kt = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      kb += sm.wcnt[w];
      kt += sm.wabv[w];
    }
    sc.tau = tau;
    sc.pos_cut = pos_cut;
    sc.L = L;
    sc.off = ab_before + kb;
    if (lead) {   // the slice's listed count, for the attention kernel
      const int total = ab_all + kt;
      P.ws.st[un.s].count = total;
      if (P.sel_count) P.sel_count[un.s] = total;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ compact phase
// One range of slice y (after refine_range of y): its kept positions outside
// sinks/window, ascending, written at the range's offset in the slice's list.  Rounds of
// kThrRun consecutive tokens per thread: the thread's keep mask from its probabilities
// (16-byte reads in token mode, its block's one in block mode), one CTA scan of the
// counts for the thread's offset, the kept positions staged in order in shared memory
// (`stage`, kThrRun * threads ints), then copied to the list with coalesced stores.
template <bool BLK>
__device__ void compact_segment(const StepParams& P, SelScalars& sc, int* stage, const Ranges<BLK>& R, int y, int l0,
                                int l1) {
  const Unit un = unit_of(P, y);
  const PiSeg ps = pi_seg<BLK>(R, y, un.s);
  const int tid = threadIdx.x;
  const int L = sc.L;   // sc.L, sc.tau, sc.pos_cut and sc.off from refine_range of this slice
  const unsigned tau = sc.tau;
  const int pos_cut = sc.pos_cut;
  const SinkWindow sw(L, P.n_sink, P.window);
  const int j0 = 16 * l0, j1 = min(L, 16 * l1);
  int* dst = P.sel_list + (size_t)un.s * P.Lmax;
  int run = sc.off;
  static_assert(kBlock % kThrRun == 0, "a thread's run lies in one block");
  static_assert(sizeof(SelSmem) >= sizeof(int) * kThrRun * kSelThreads, "a round's positions fit the stage");
  for (int k0 = j0; k0 < j1; k0 += kThrRun * kSelThreads) {   // whole CTA: the scan below
    const int jb = k0 + kThrRun * tid;
    unsigned keep = 0u;
    if (jb < j1) {
      unsigned bits[kThrRun];
      if (BLK) {
        const unsigned v = __float_as_uint(pi_load(P, ps, jb / kBlock));
#pragma unroll
        for (int q = 0; q < kThrRun; ++q) bits[q] = v;
      } else {
#pragma unroll
        for (int q4 = 0; q4 < kThrRun / 4; ++q4) {   // jb is a multiple of 16: aligned 16-byte words
          const float4 v = pi_load4(P, ps, jb + 4 * q4);
          bits[4 * q4] = __float_as_uint(v.x);
          bits[4 * q4 + 1] = __float_as_uint(v.y);
          bits[4 * q4 + 2] = __float_as_uint(v.z);
          bits[4 * q4 + 3] = __float_as_uint(v.w);
        }
      }
#pragma unroll
      for (int q = 0; q < kThrRun; ++q) {
        const int j = jb + q;
        const int e = BLK ? j / kBlock : j;
        if (j < j1 && !sw.always(j) && kept_by_cut(bits[q], e, tau, pos_cut)) keep |= 1u << q;
      }
    }
    int total;
    int o = block_excl_scan<int>(__popc(keep), sc.shi, &total);   // (ends with a CTA barrier)
    // the round's kept positions in order in shared memory, then one coalesced copy
#pragma unroll
    for (int q = 0; q < kThrRun; ++q)
      if (keep >> q & 1u) stage[o++] = jb + q;
    __syncthreads();
    if (run + total > P.Lmax) {   // offsets and predicate disagree: never write past the list
      if (tid == 0) atomicOr(P.ws.dev_err, kErrInternal);
      total = P.Lmax - run;
    }
    for (int i = tid; i < total; i += kSelThreads) dst[run + i] = stage[i];
    __syncthreads();   // the stage is rewritten by the next round
    run += total;
  }
}

// ------------------------------------------------------------------ the kernel
template <typename T, int G, bool BLK>
__global__ void __launch_bounds__(kSelThreads, 1024 / kSelThreads) k_select(StepParams P) {
  __shared__ SelSmem sm;
  __shared__ SelScalars sc;
  const Ranges<BLK> R(P);
  auto n_ranges = [&](int y) { return (unsigned)(R.last_cta(y) - R.first_cta(y) + 1); };
  for_each_segment(R, [&](int y, int l0, int l1) {
    score_segment<G>(P, sm.score, sc, R.me, y, l0, l1);
    // failure-detection test hook: CTA 0 never arrives, so the other CTAs of its slice
    // give up their bounded waits for the slice's statistics
    if (!(P.drop_publish && blockIdx.x == 0)) slice_arrive(&P.ws.st[unit_of(P, y).s].arr_score);
  });
  if (P.drop_publish && blockIdx.x == 0) return;
  bool ok = true;
  for_each_segment(R, [&](int y, int l0, int l1) {
    for (int a = l0; a < l1 && ok; a += kMaxRangeGroups)
      ok = mass_segment<G, BLK>(P, sm.mass, sc, R, y, a, min(l1, a + kMaxRangeGroups), a == l0, n_ranges(y));
    if (ok) slice_arrive(&P.ws.st[unit_of(P, y).s].arr_mass);
  });
  if (!ok) return;
  prefetch_attended_rows<T>(P);
  for_each_segment(R, [&](int y, int l0, int l1) {
    if (!ok) return;
    SliceState* st = P.ws.st + unit_of(P, y).s;
    ok = slice_wait(&st->arr_mass, n_ranges(y), P.ws.dev_err, &sc.ok);
    if (!ok) return;
    cut1_range(P, sc, y, R.me == R.first_cta(y));
    threshold_segment<BLK>(P, sc, sm.ref, R, y, l0, l1);
    slice_arrive(&st->arr_thr);
  });
  if (!ok) return;
  for_each_segment(R, [&](int y, int l0, int l1) {
    if (!ok) return;
    SliceState* st = P.ws.st + unit_of(P, y).s;
    ok = slice_wait(&st->arr_thr, n_ranges(y), P.ws.dev_err, &sc.ok);
    if (!ok) return;
    refine_range<BLK>(P, sm.ref, sc, R, y, l0, l1, R.me == R.first_cta(y));
    compact_segment<BLK>(P, sc, reinterpret_cast<int*>(&sm), R, y, l0, l1);
  });
}

template <typename T, int G>
cudaError_t launch_tg(const StepParams& P, int grid, cudaStream_t st) {
  k_qprep<T, G><<<P.k_cache ? 2 * P.n_slices : P.n_slices, kSelThreads, 0, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || P.n_ret == 0) return e;   // nothing to select
  StepParams local = P;
  void* args[] = {&local};
  const void* fn = P.blocks ? (const void*)k_select<T, G, true> : (const void*)k_select<T, G, false>;
  // cooperative (every CTA resident: the arrival waits need it) and allowed to start
  // before the prologue kernel ends (programmatic stream serialization; the score phase
  // waits for the prologue's completion after requesting its first index rows)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = kPiBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// Co-resident CTAs per SM, the smaller of the token and block variants (one grid size
// serves both).  Also raises the variants' dynamic shared memory limit to kPiBytes.
template <typename T, int G>
int resident_tg() {
  int n = 0, m = 0;
  if (cudaFuncSetAttribute(k_select<T, G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPiBytes) !=
          cudaSuccess ||
      cudaFuncSetAttribute(k_select<T, G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPiBytes) !=
          cudaSuccess)
    return -1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_select<T, G, false>, kSelThreads, kPiBytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, k_select<T, G, true>, kSelThreads, kPiBytes) != cudaSuccess)
    return -1;
  return n < m ? n : m;
}

}  // namespace

// Grid of the selection launch: as many resident CTAs as give every retrieval slice the
// same whole number of CTAs (all of them when the slices do not divide the resident
// count), but never more CTAs than range quanta (16-token groups, or kBlock-token blocks
// in block mode), so no CTA has an empty range.
int select_grid(const StepParams& P, int max_resident) {
  if (max_resident > kMaxSelectGrid) max_resident = kMaxSelectGrid;
  if (P.n_ret <= 0) return P.n_slices < max_resident ? P.n_slices : max_resident;
  const long long qt = P.blocks ? kBlock : 16;
  const long long n_rs = (long long)P.B * P.n_ret, per_slice = ((long long)P.Lcap + qt - 1) / qt;
  // a whole number of CTAs per retrieval slice when there are at least as many CTAs as
  // slices: every range then lies inside one slice (the range split places the
  // boundaries of equal shares there), so no CTA serves two slices' phases
  if (n_rs <= max_resident) {
    long long cps = max_resident / n_rs;
    if (cps > per_slice) cps = per_slice;
    return (int)(n_rs * cps);
  }
  long long want = max_resident;
  if (want > n_rs * per_slice) want = n_rs * per_slice;
  if (want < 1) want = 1;
  return (int)want;
}

namespace {
cudaError_t launch_part(const StepParams& P, int kv_dtype, int grid, cudaStream_t st) {
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
}  // namespace

cudaError_t launch_select(const StepParams& P, int kv_dtype, int max_resident, cudaStream_t st) {
  if (max_resident > kMaxSelectGrid) max_resident = kMaxSelectGrid;
  if (max_resident < 1 || P.n_ret > max_resident) return cudaErrorInvalidValue;
  // sequences per launch: all, unless their retrieval slices outnumber the co-resident
  // CTAs (then every launch still gets a whole number of CTAs per slice)
  const int per = P.n_ret > 0 ? (max_resident / P.n_ret > 0 ? max_resident / P.n_ret : 1) : P.B;
  for (int b0 = 0; b0 < P.B; b0 += per) {
    StepParams Q = P;
    Q.b_base = P.b_base + b0;
    Q.B = P.B - b0 < per ? P.B - b0 : per;
    Q.n_slices = Q.B * P.Hkv;
    const cudaError_t e = launch_part(Q, kv_dtype, select_grid(Q, max_resident), st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
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
