// Prefill chunk attention: dense causal for retrieval heads, sinks + sliding window for
// streaming heads.
//
// "Full Attention Strikes Back" (RTPurbo summary), Methodology §1: retrieval heads keep
// the full context (the sparse selection is a decode step), local heads attend a
// sliding window with attention sinks; "Autonomy of Heads" summary, Deployment
// strategy: streaming heads keep sinks and a recent window from the first token on.
//
// A query at absolute position t (chunk row i, t = start[b] + i) attends keys j <= t:
// every j on a retrieval head, j < n_sink or j > t - window on a streaming head.  The
// query is rotated to position t (rotate-half RoPE, angles in float64 in units of pi)
// and rounded to bf16; scores and the softmax run in float32 (log2 domain), the
// probabilities are rounded to bf16 for P V, accumulation is float32.
//
// Layout: a CTA takes one (b, KV head) and 128 query rows packed as G heads x 128/G
// positions, so the group's G query heads share every K/V tile (GQA).  Eight warps
// own 16 rows each (one head, 16 consecutive positions).  K/V tiles of 64 keys stream
// through a two-stage cp.async ring in shared memory (rows padded to 272 bytes, so
// ldmatrix reads are conflict-free); S = Q K^T and O += P V run on mma.sync
// m16n8k16 (bf16 in, float32 accumulate) with an online softmax per row.  Key tiles
// outside a warp's causal or window range are skipped by that warp; the CTAs are
// issued heaviest first.
#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kKT = 64;                 // keys per tile
constexpr int kRowsPerCta = 128;        // query rows (heads x positions)
constexpr int kPWarps = 8;
constexpr int kPThreads = kPWarps * 32;
constexpr int kLdS = kHeadDim + 8;      // padded smem row (bf16 elements): 272 bytes

struct PrefillParams {
  const __nv_bfloat16* q;   // [B][Hq][T][128] pre-RoPE
  const __nv_bfloat16* k;   // [Bm][Hkv][Lmax][128] post-RoPE
  const __nv_bfloat16* v;
  float* out;               // [B][Hq][T][128]
  const int64_t* start;     // [B]
  const double* inv_freq_pi;   // [64] inv_freq / pi
  unsigned* err;
  int T, Hq, Hkv, n_sink, window, n_qblocks;
  int64_t Lmax;
  float scale_log2;
  unsigned char is_ret[kMaxKvHeads];
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16-byte async copy; src_bytes = 0 fills the destination with zeros (no read)
__device__ __forceinline__ void cp16(void* dst, const void* src, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" :: "r"(d), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" :: "n"(N)); }
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Key tiles a CTA visits, ascending: tiles of [0, n_sink) and tiles of [lo, hi) (the
// window of the CTA's rows), or every tile of [0, hi) for a retrieval head.
struct TileRange {
  int sink_tiles, w_first, w_last;   // sink tiles [0, sink_tiles); window tiles [w_first, w_last]
  __device__ __forceinline__ int count() const { return sink_tiles + (w_last >= w_first ? w_last - w_first + 1 : 0); }
  __device__ __forceinline__ int tile(int i) const { return i < sink_tiles ? i : w_first + (i - sink_tiles); }
};

template <int G>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill_bf16(const PrefillParams P) {
  constexpr int QB = kRowsPerCta / G;   // positions per CTA
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem_raw);              // [128][kLdS]
  __nv_bfloat16* kvs = qs + kRowsPerCta * kLdS;                                 // [2][K|V][64][kLdS]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
  const int qblk = P.n_qblocks - 1 - (int)blockIdx.x;   // heaviest first
  const int bg = blockIdx.y, b = bg / P.Hkv, g = bg % P.Hkv;
  const bool ret = P.is_ret[g] != 0;
  const int64_t start = P.start[b];
  const int i0 = qblk * QB;                       // first chunk row of the CTA
  if (start < 0 || start + P.T > P.Lmax) {
    if (tid == 0) atomicOr(P.err, kErrStartPos);
    return;
  }
  const int t_first = (int)start + i0;                       // first position of the CTA
  const int t_end = (int)start + min(i0 + QB, P.T);          // one past its last valid position
  // warp rows: head hl, positions pw .. pw + 15
  const int hl = warp % G, pw = t_first + 16 * (warp / G);
  const int h = g * G + hl;

  // ---- Q: rotate to each row's position, round to bf16, stage in shared memory
  {
    const __nv_bfloat16* qsrc = P.q + ((size_t)b * P.Hq + h) * P.T * kHeadDim;
    __nv_bfloat16* qdst = qs + (size_t)warp * 16 * kLdS;
    for (int e = lane; e < 16 * (kHeadDim / 2); e += 32) {
      const int r = e / (kHeadDim / 2), i = e % (kHeadDim / 2);
      const int t = pw + r, row = t - (int)start;
      float o1 = 0.f, o2 = 0.f;
      if (row < P.T) {
        const float x1 = __bfloat162float(qsrc[(size_t)row * kHeadDim + i]);
        const float x2 = __bfloat162float(qsrc[(size_t)row * kHeadDim + i + kHeadDim / 2]);
        const double a = (double)t * P.inv_freq_pi[i];
        double sn, cs;
        sincospi(a - 2.0 * rint(0.5 * a), &sn, &cs);
        o1 = (float)((double)x1 * cs - (double)x2 * sn);
        o2 = (float)((double)x2 * cs + (double)x1 * sn);
      }
      qdst[r * kLdS + i] = __float2bfloat16_rn(o1);
      qdst[r * kLdS + i + kHeadDim / 2] = __float2bfloat16_rn(o2);
    }
  }

  // ---- key tiles of the CTA
  TileRange tr;
  if (ret) {
    tr.sink_tiles = 0;
    tr.w_first = 0;
    tr.w_last = (t_end - 1) / kKT;
  } else {
    const int ns = min(P.n_sink, t_end);
    tr.sink_tiles = (ns + kKT - 1) / kKT;
    const int wlo = max(ns, t_first - P.window + 1);   // lowest window key of the CTA's rows
    tr.w_first = max(wlo / kKT, tr.sink_tiles);
    tr.w_last = (t_end - 1) / kKT;
    if (wlo >= t_end) tr.w_last = tr.w_first - 1;      // no window keys
  }
  const int n_tiles = tr.count();
  const __nv_bfloat16* kg = P.k + ((size_t)b * P.Hkv + g) * (size_t)P.Lmax * kHeadDim;
  const __nv_bfloat16* vg = P.v + ((size_t)b * P.Hkv + g) * (size_t)P.Lmax * kHeadDim;
  auto issue = [&](int it) {
    if (it < n_tiles) {
      const int j0 = tr.tile(it) * kKT;
      __nv_bfloat16* dst = kvs + (size_t)(it & 1) * 2 * kKT * kLdS;
#pragma unroll
      for (int u = 0; u < (2 * kKT * kHeadDim / 8) / kPThreads; ++u) {   // 16-byte pieces
        const int e = tid + kPThreads * u;
        const int tv = e / (kKT * kHeadDim / 8), rem = e % (kKT * kHeadDim / 8);
        const int r = rem / (kHeadDim / 8), c = rem % (kHeadDim / 8);
        const int j = j0 + r;
        const bool ok = j < t_end;
        const __nv_bfloat16* src = (tv ? vg : kg) + (size_t)(ok ? j : 0) * kHeadDim + c * 8;
        cp16(dst + (size_t)tv * kKT * kLdS + r * kLdS + c * 8, src, ok ? 16 : 0);
      }
    }
    cp_commit();
  };
  issue(0);
  __syncthreads();   // Q staged

  // Q fragments (A operand), kept in registers: 8 k-steps of 16 dims
  uint32_t qa[kHeadDim / 16][4];
  {
    const __nv_bfloat16* qw = qs + (size_t)warp * 16 * kLdS;
#pragma unroll
    for (int kk = 0; kk < kHeadDim / 16; ++kk) ldsm_x4(qa[kk], qw + (lane % 16) * kLdS + kk * 16 + (lane / 16) * 8);
  }

  float o[kHeadDim / 8][4];
#pragma unroll
  for (int n = 0; n < kHeadDim / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int t_row[2] = {pw + gid, pw + gid + 8};
  const int t_hi = min(pw + 15, t_end - 1);   // the warp's last valid position
  const float sl2 = P.scale_log2;

  for (int it = 0; it < n_tiles; ++it) {
    issue(it + 1);
    cp_wait<1>();
    __syncthreads();
    const int j0 = tr.tile(it) * kKT;
    // does any key of this tile reach any row of the warp?
    bool active = pw <= t_hi && j0 <= t_hi;
    if (active && !ret) {
      const bool sink_part = j0 < P.n_sink;
      const bool win_part = j0 + kKT - 1 > pw - P.window;
      active = sink_part || win_part;
    }
    if (active) {
      const __nv_bfloat16* ks = kvs + (size_t)(it & 1) * 2 * kKT * kLdS;
      const __nv_bfloat16* vs = ks + kKT * kLdS;
      // S = Q K^T: 8 n-tiles of 8 keys
      float s[kKT / 8][4];
#pragma unroll
      for (int n = 0; n < kKT / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kHeadDim / 16; ++kk) {
#pragma unroll
        for (int n = 0; n < kKT / 8; n += 2) {
          uint32_t bk[4];
          const int i = lane / 8, r = lane % 8;
          ldsm_x4(bk, ks + (n * 8 + (i / 2) * 8 + r) * kLdS + kk * 16 + (i % 2) * 8);
          mma_bf16(s[n], qa[kk], bk[0], bk[1]);
          mma_bf16(s[n + 1], qa[kk], bk[2], bk[3]);
        }
      }
      // mask, scale, online softmax (rows gid and gid + 8 of the warp)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < kKT / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rr = e >> 1, j = j0 + n * 8 + 2 * t4 + (e & 1), t = t_row[rr];
          const bool ok = j <= t && t < t_end && (ret || j < P.n_sink || j > t - P.window);
          s[n][e] = ok ? s[n][e] * sl2 : -INFINITY;
          mx[rr] = fmaxf(mx[rr], s[n][e]);
        }
      }
      float corr[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(kFull, mx[rr], 1));
        mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(kFull, mx[rr], 2));
        const float mn = fmaxf(m_r[rr], mx[rr]);
        corr[rr] = mn == -INFINITY ? 1.f : ex2f(m_r[rr] - mn);
        m_r[rr] = mn;
      }
      float ls[2] = {0.f, 0.f};
#pragma unroll
      for (int n = 0; n < kKT / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rr = e >> 1;
          const float p = m_r[rr] == -INFINITY ? 0.f : ex2f(s[n][e] - m_r[rr]);
          s[n][e] = p;
          ls[rr] += p;
        }
      }
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        ls[rr] += __shfl_xor_sync(kFull, ls[rr], 1);
        ls[rr] += __shfl_xor_sync(kFull, ls[rr], 2);
        l_r[rr] = l_r[rr] * corr[rr] + ls[rr];
      }
#pragma unroll
      for (int n = 0; n < kHeadDim / 8; ++n) {
        o[n][0] *= corr[0];
        o[n][1] *= corr[0];
        o[n][2] *= corr[1];
        o[n][3] *= corr[1];
      }
      // O += P V: 4 k-steps of 16 keys, 16 n-tiles of 8 dims
#pragma unroll
      for (int kk = 0; kk < kKT / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = pack2(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack2(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int n = 0; n < kHeadDim / 8; n += 2) {
          uint32_t bv[4];
          const int i = lane / 8, r = lane % 8;
          ldsm_x4_t(bv, vs + (kk * 16 + (i % 2) * 8 + r) * kLdS + n * 8 + (i / 2) * 8);
          mma_bf16(o[n], pa, bv[0], bv[1]);
          mma_bf16(o[n + 1], pa, bv[2], bv[3]);
        }
      }
    }
    __syncthreads();   // the stage is refilled by the next issue
  }
  cp_wait<0>();

  // ---- output rows: O / l
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int t = t_row[rr], row = t - (int)start;
    if (t >= t_end) continue;
    const float inv = l_r[rr] > 0.f ? 1.f / l_r[rr] : 0.f;
    float* dst = P.out + (((size_t)b * P.Hq + h) * P.T + row) * kHeadDim;
#pragma unroll
    for (int n = 0; n < kHeadDim / 8; ++n) {
      const float2 v2 = make_float2(o[n][2 * rr] * inv, o[n][2 * rr + 1] * inv);
      *reinterpret_cast<float2*>(dst + n * 8 + 2 * t4) = v2;
    }
  }
}

template <int G>
cudaError_t launch_g(const PrefillParams& P, int B, cudaStream_t st) {
  const int smem = (kRowsPerCta + 2 * 2 * kKT) * kLdS * (int)sizeof(__nv_bfloat16);
  cudaError_t e = cudaFuncSetAttribute(k_prefill_bf16<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(P.n_qblocks, B * P.Hkv);
  k_prefill_bf16<G><<<grid, kPThreads, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const void* q, const void* k, const void* v, float* out, const int64_t* start, int B,
                           int T, int Hq, int Hkv, int64_t Lmax, int n_sink, int window, const unsigned char* is_ret,
                           const double* inv_freq_pi, unsigned* err, cudaStream_t st) {
  PrefillParams P;
  P.q = (const __nv_bfloat16*)q;
  P.k = (const __nv_bfloat16*)k;
  P.v = (const __nv_bfloat16*)v;
  P.out = out;
  P.start = start;
  P.inv_freq_pi = inv_freq_pi;
  P.err = err;
  P.T = T;
  P.Hq = Hq;
  P.Hkv = Hkv;
  P.n_sink = n_sink;
  P.window = window;
  P.Lmax = Lmax;
  P.scale_log2 = (float)(1.4426950408889634 / 11.313708498984761);   // log2(e) / sqrt(128)
  for (int g = 0; g < kMaxKvHeads; ++g) P.is_ret[g] = g < Hkv ? is_ret[g] : 0;
  const int G = Hq / Hkv;
  P.n_qblocks = (T + kRowsPerCta / G - 1) / (kRowsPerCta / G);
  switch (G) {
    case 1: return launch_g<1>(P, B, st);
    case 2: return launch_g<2>(P, B, st);
    case 4: return launch_g<4>(P, B, st);
    case 8: return launch_g<8>(P, B, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace spa
