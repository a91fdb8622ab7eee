// Split-K attention for bf16 caches on the tensor cores (mma.sync m16n8k16).
//
// Same computation as the float32 kernel in k_attend.cu ("Full Attention Strikes
// Back" (RTPurbo summary), Methodology §1; exact token attention as in
// "Hierarchical Global Attention", Central mechanism §4): for every split of a
// slice's attended rows, the online-softmax state (m, l, acc) of each query head
// of the GQA group.
//
// Work layout.  One CTA per SM, 8 warps.  The attended rows of all slices form one
// virtual row space (per slice: sinks, window, then the gathered list); each CTA takes
// an equal contiguous share of it, i.e. one piece per slice it touches, so every SM gets
// the same number of rows whatever the slices' lengths.  Inside a piece, warp w takes
// the 16-row chunks w, w + 8, ...  Each warp streams its chunks through its own 3-stage
// ring in shared memory with 16-byte cp.async (one K row = 256 bytes = 16 lanes), keeps
// prefetching across pieces, loads the row positions of the next chunk one issue ahead
// (no copy waits on a list load), and keeps its own online softmax.
// (One 256-byte TMA bulk copy per row was measured 4.6x slower than this: the
// per-request cost of the bulk-copy engine dominates at row granularity.)  At the
// end of a piece the 8 warp states are merged in a fixed 3-round tree and warp 0
// writes the split state of (CTA, slice); the last CTA to finish a piece of a slice
// (a per-slice ticket) combines the slice's states into the output, so a decode step
// needs no separate combine launch.
//
// Tensor-core mapping (G <= 8 heads of the group, M = 16 rows):
//   S[16 x 16 tokens] = Q[16 x 128] . K^T:  A rows 0..7 = bf16 high parts of the
//       G rotated queries, rows 8..15 = the bf16 residuals (q - hi), so the two
//       halves of the accumulator sum to the score at ~2^-17 relative precision;
//       B = K rows straight from shared memory (ldmatrix, rows are tokens).
//   O[16 x 128] += P[16 x 16 tokens] . V:  the probabilities, split the same way
//       into bf16 high parts (rows 0..7) and residuals (rows 8..15), come from the
//       score accumulators without a shuffle; B = V via ldmatrix.trans.
// Rows of a stage are padded to 272 bytes so the 8 row addresses of an ldmatrix
// fall in 8 different bank groups.
#include <climits>

#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarps = 8;
constexpr int kChunkRows = 16;
constexpr int kStages = 3;
constexpr int kRowPad = kHeadDim + 8;                               // 136 bf16 = 272 bytes
constexpr int kStageElems = 2 * kChunkRows * kRowPad;               // K then V
constexpr size_t kRingBytes = (size_t)kWarps * kStages * kStageElems * 2;

// K/V rows are read once per step: their L2 lines are marked first to go, so the
// stream does not push out the small tensors the next call reads first.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint64_t pol) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "l"(pol) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_stages() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(kStages - 2) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// bf16 pair: x in the low half (lower column), y in the high half.
__device__ __forceinline__ uint32_t pack2(float x, float y) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float bf16r(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
// 2^x with the hardware approximation (relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Where an item's rows come from.
struct ItemInfo {
  int s;          // slice b * Hkv + g
  int v0, v1;     // virtual rows [v0, v1)
  int nc;         // contiguous (sink + window) rows of the slice
  int n_s, w_lo;  // sinks [0, n_s), window [w_lo, L)
  int nch;        // 16-row chunks
};

// Slice holding virtual row r of the concatenated row space (binary search over the
// row prefix: the largest s with rpre[s] <= r).
__device__ __forceinline__ int slice_of_row(const long long* rpre, int n_slices, long long r) {
  int lo = 0, hi = n_slices - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (rpre[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The piece of slice s inside the CTA's row range [r_lo, r_hi), from shared memory only:
// the row prefix over slices and each slice's (sequence length, listed rows).
__device__ __forceinline__ ItemInfo piece_info(const StepParams& P, const long long* rpre, const int2* sinfo,
                                              long long r_lo, long long r_hi, int s) {
  ItemInfo it;
  it.s = s;
  const int2 si = sinfo[s];
  const SinkWindow sw(si.x, P.n_sink, P.window);
  it.nc = sw.n_contig();
  it.n_s = sw.n_s;
  it.w_lo = sw.w_lo;
  const long long a = r_lo > rpre[s] ? r_lo : rpre[s];
  const long long e = r_hi < rpre[s + 1] ? r_hi : rpre[s + 1];
  it.v0 = (int)(a - rpre[s]);
  it.v1 = (int)(e - rpre[s]);
  it.nch = it.v1 > it.v0 ? (it.v1 - it.v0 + kChunkRows - 1) / kChunkRows : 0;
  return it;
}

// Combines slice s's split states (slots c + s for CTAs c0..c1) into out[b][g G + h]:
// warp w takes head w % G and the slots c0 + w / G, c0 + w / G + 8 / G, ... (merged in
// order), then the warps of a head are merged in warp order through shared memory.
// Lane l holds dims 4l..4l+3.  Called by every thread of the CTA.
template <int G>
__device__ void combine_slice(const StepParams& P, int s, int c0, int c1, float* cbuf) {
  constexpr int kPer = kWarps / G;   // warps per head
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = warp % G, sub = warp / G;
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int kB = 4;
  for (int c = c0 + sub; c <= c1; c += kPer * kB) {
    float4 a[kB];
    float mi[kB], li[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int cc = c + u * kPer;
      if (cc <= c1) {
        const float* pp = P.ws.part + ((size_t)(cc + s) * G + h) * kPartStride;
        a[u] = __ldcg(reinterpret_cast<const float4*>(pp) + lane);
        mi[u] = __ldcg(pp + kHeadDim);
        li[u] = __ldcg(pp + kHeadDim + 1);
      } else {
        a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        mi[u] = -INFINITY;
        li[u] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const float mn = fmaxf(m, mi[u]);
      if (mn == -INFINITY) continue;
      const float sa = exp2f(m - mn), sb = exp2f(mi[u] - mn);
      l = l * sa + li[u] * sb;
      acc.x = acc.x * sa + a[u].x * sb;
      acc.y = acc.y * sa + a[u].y * sb;
      acc.z = acc.z * sa + a[u].z * sb;
      acc.w = acc.w * sa + a[u].w * sb;
      m = mn;
    }
  }
  float* mine = cbuf + (size_t)warp * kPartStride;
  *reinterpret_cast<float4*>(mine + 4 * lane) = acc;
  if (lane == 0) { mine[kHeadDim] = m; mine[kHeadDim + 1] = l; }
  __syncthreads();
  if (warp < G) {
    float M = -INFINITY, Ls = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < kPer; ++k) {
      const float* src = cbuf + (size_t)(h + G * k) * kPartStride;
      const float m2 = src[kHeadDim], l2 = src[kHeadDim + 1];
      const float mn = fmaxf(M, m2);
      if (mn == -INFINITY) continue;
      const float sa = exp2f(M - mn), sb = exp2f(m2 - mn);
      const float4 v = *reinterpret_cast<const float4*>(src + 4 * lane);
      Ls = Ls * sa + l2 * sb;
      num.x = num.x * sa + v.x * sb;
      num.y = num.y * sa + v.y * sb;
      num.z = num.z * sa + v.z * sb;
      num.w = num.w * sa + v.w * sb;
      M = mn;
    }
    const float inv = 1.f / Ls;
    const int b = s / P.Hkv, g = s % P.Hkv;
    *reinterpret_cast<float4*>(P.out + ((size_t)b * P.Hq + (size_t)g * G + h) * kHeadDim + 4 * lane) =
        make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
    if (P.lse && lane == 0) P.lse[(size_t)b * P.Hq + (size_t)g * G + h] = M + log2f(Ls);
  }
  if (threadIdx.x == 0 && P.sel_count) {
    const int g = s % P.Hkv;
    P.sel_count[s] = P.is_ret[g] ? P.ws.st[s].count : 0;
  }
  __syncthreads();   // cbuf reused by the next combine
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32, 1) k_attend_bf16(StepParams P) {
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* ring = reinterpret_cast<__nv_bfloat16*>(smem);
  float* mbuf = reinterpret_cast<float*>(smem + kRingBytes);         // [4][G][kPartStride]
  long long* rpre = reinterpret_cast<long long*>(mbuf + 4 * G * kPartStride);   // [n_slices + 1] row prefix
  int2* sinfo = reinterpret_cast<int2*>(rpre + P.n_slices + 1);                  // [n_slices] (L, listed rows)
  // [8 warps][kPartStride], 16-byte aligned (float4 accesses)
  float* cbuf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(sinfo + P.n_slices) + 15) & ~uintptr_t(15));
  __shared__ int s_merge;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, t4 = lane & 3;
  const int NS = P.n_slices;

  // ---- row prefix over slices: slice s owns virtual rows [rpre[s], rpre[s + 1]) of the
  // concatenated row space (its sinks, window, then its gathered list)
  {
    __shared__ long long shl[32];
    long long carry = 0;
    for (int base = 0; base < NS; base += kWarps * 32) {
      const int s = base + tid;
      long long rows = 0;
      if (s < NS) {
        const int b = s / P.Hkv, g = s % P.Hkv;
        const int L = load_len(P.seq_lens, b, P.Lcap, P.ws.dev_err);
        const SinkWindow sw(L, P.n_sink, P.window);
        const int cnt = P.is_ret[g] ? P.ws.st[s].count : 0;
        sinfo[s] = make_int2(L, cnt);
        rows = sw.n_contig() + cnt;
      }
      long long v = rows;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += y;
      }
      if (lane == 31) shl[warp] = v;
      __syncthreads();
      if (warp == 0) {
        long long w = lane < kWarps ? shl[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long y = __shfl_up_sync(kFull, w, o);
          if (lane >= o) w += y;
        }
        if (lane < kWarps) shl[lane] = w;
      }
      __syncthreads();
      if (s < NS) rpre[s] = carry + (warp ? shl[warp - 1] : 0) + v - rows;
      carry += shl[kWarps - 1];
      __syncthreads();
    }
    if (tid == 0) rpre[NS] = carry;
    __syncthreads();
  }
  // ---- the CTA's equal share of the row space, as one piece per slice it touches.  The
  // split state of the piece of slice s goes to partial slot blockIdx.x + s, so each
  // slice's slots are consecutive; CTA 0 publishes where they start for the combine.  A
  // CTA whose range starts exactly at a slice boundary writes an empty state into the one
  // slot (its index + s - 1) that the previous slice's range would otherwise skip.
  const long long T = rpre[NS];
  if (T == 0) return;   // nothing to attend (a context-parallel rank past every sequence)
  const int nb = (long long)gridDim.x < T ? (int)gridDim.x : (int)T;   // active CTAs: >= 1 row each
  const long long r_lo = (long long)blockIdx.x * T / nb, r_hi = blockIdx.x < nb ? (long long)(blockIdx.x + 1) * T / nb : r_lo;
  auto owner = [&](long long r) { return (int)(((r + 1) * nb - 1) / T); };
  const int s_first = r_lo < r_hi ? slice_of_row(rpre, NS, r_lo) : 1;
  const int s_last = r_lo < r_hi ? slice_of_row(rpre, NS, r_hi - 1) : 0;

  __nv_bfloat16* myring = ring + (size_t)warp * kStages * kStageElems;

  // ---- prefetch cursor over this warp's (item, chunk) units.  The row positions of
  // the unit to issue next are loaded one issue ahead (apos, lane r < 16 holds row r),
  // so no copy address waits on a load from the selected list.
  int pf_item = s_first, pf_ch = warp;   // pf_item: the slice of the piece
  ItemInfo pf = {};
  if (pf_item <= s_last) pf = piece_info(P, rpre, sinfo, r_lo, r_hi, pf_item);
  auto pf_normalise = [&]() {
    while (pf_item <= s_last && pf_ch >= pf.nch) {
      ++pf_item;
      pf_ch = warp;
      if (pf_item <= s_last) pf = piece_info(P, rpre, sinfo, r_lo, r_hi, pf_item);
    }
  };
  auto load_pos = [&]() -> int {
    int pos = 0;
    if (pf_item <= s_last && lane < kChunkRows) {
      const int r0 = pf.v0 + pf_ch * kChunkRows;
      int v = r0 + lane;
      if (v >= pf.v1) v = r0;   // rows past the item repeat row 0 (finite, masked later)
      if (v < pf.nc) {
        pos = v < pf.n_s ? v : pf.w_lo + (v - pf.n_s);
        // compact layout: a streaming head's rows sit in its ring
        if (P.compact && !P.is_ret[pf.s % P.Hkv]) pos = ring_row(pos, P.n_sink, P.window);
      } else {
        pos = P.sel_list[(size_t)pf.s * P.Lmax + (v - pf.nc)];
      }
    }
    return pos;
  };
  pf_normalise();
  int apos = load_pos();
  int issued = 0;  // units issued so far (selects the ring slot)
  const uint64_t kv_pol = l2_evict_first();
  auto issue_next = [&]() {
    __nv_bfloat16* dst = myring + (size_t)(issued % kStages) * kStageElems;
    if (pf_item <= s_last) {
      const KvSlice<__nv_bfloat16> kv = kv_slice<__nv_bfloat16>(P, pf.s);
      const __nv_bfloat16* kb = kv.k;
      const __nv_bfloat16* vb = kv.v;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int idx = i * 32 + lane;   // 512 pieces of 16 bytes: [K|V][row][piece]
        const int tv = idx >> 8, rem = idx & 255, r = rem >> 4, c = rem & 15;
        const int prow = __shfl_sync(kFull, apos, r);
        const __nv_bfloat16* src = (tv ? vb : kb) + (size_t)prow * kHeadDim + c * 8;
        cp_async16(dst + tv * kChunkRows * kRowPad + r * kRowPad + c * 8, src, kv_pol);
      }
      pf_ch += kWarps;
      pf_normalise();
      apos = load_pos();
    }
    cp_async_commit();
    ++issued;
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) issue_next();

  int consumed = 0;
  int cur_slice = -1;
  uint32_t qa[8][4];   // A fragments of Q (hi rows 0..7, residual rows 8..15), per 16-dim k-step
  const float scale = P.attn_scale_log2;

  for (int ps = s_first; ps <= s_last; ++ps) {
    const ItemInfo it = piece_info(P, rpre, sinfo, r_lo, r_hi, ps);
    // a slice with no rows (only in context-parallel steps) has no split state, no
    // ticket and no output here: the list kernel wrote its empty result
    if (it.v1 <= it.v0) continue;
    if (it.s != cur_slice) {
      cur_slice = it.s;
      const int b = it.s / P.Hkv, g = it.s % P.Hkv;
      const float* q = P.ws.q_rot + ((size_t)b * P.Hq + (size_t)g * G + (gid < G ? gid : 0)) * kHeadDim;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        float x[4];
        x[0] = q[16 * kk + 2 * t4];
        x[1] = q[16 * kk + 2 * t4 + 1];
        x[2] = q[16 * kk + 2 * t4 + 8];
        x[3] = q[16 * kk + 2 * t4 + 9];
        if (gid >= G) x[0] = x[1] = x[2] = x[3] = 0.f;
        float hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          hi[j] = bf16r(x[j]);
          lo[j] = x[j] - hi[j];
        }
        qa[kk][0] = pack2(hi[0], hi[1]);
        qa[kk][1] = pack2(lo[0], lo[1]);
        qa[kk][2] = pack2(hi[2], hi[3]);
        qa[kk][3] = pack2(lo[2], lo[3]);
      }
    }
    {
      // the next piece of this CTA: bring its slice's rotated query rows into L1 now
      // (lane (gid, t4): 128-byte line t4 of head gid)
      const int ns = ps + 1;
      if (ns <= s_last && gid < G) {
        const float* qn = P.ws.q_rot + ((size_t)(ns / P.Hkv) * P.Hq + (size_t)(ns % P.Hkv) * G + gid) * kHeadDim + 32 * t4;
        asm volatile("prefetch.global.L1 [%0];\n" ::"l"(qn));
      }
    }
    float m = -INFINITY, l = 0.f;
    float acc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

    for (int ch = warp; ch < it.nch; ch += kWarps) {
      cp_async_wait_stages();
      __syncwarp();
      const __nv_bfloat16* ks = myring + (size_t)(consumed % kStages) * kStageElems;
      const __nv_bfloat16* vs = ks + kChunkRows * kRowPad;
      ++consumed;
      issue_next();   // refill the slot consumed last time
      const int nr = min(kChunkRows, it.v1 - (it.v0 + ch * kChunkRows));

      // S = Q K^T for 16 tokens (two n-tiles of 8); two accumulators per n-tile
      // (even / odd k-steps) halve the dependent mma chain
      float sc[2][2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int e = 0; e < 2; ++e) sc[a][e][0] = sc[a][e][1] = sc[a][e][2] = sc[a][e][3] = 0.f;
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t bk[4];
        ldsm_x4(bk, ks + (8 * (mi >> 1) + rr) * kRowPad + 16 * kk + 8 * (mi & 1));
        mma16816(sc[0][kk & 1], qa[kk], bk[0], bk[1]);
        mma16816(sc[1][kk & 1], qa[kk], bk[2], bk[3]);
      }
      // scores of head gid for tokens 8j + 2 t4 + c (hi row + residual row)
      float s[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int tok = 8 * j + 2 * t4 + c;
          const float v = ((sc[j][0][c] + sc[j][1][c]) + (sc[j][0][2 + c] + sc[j][1][2 + c])) * scale;
          s[j][c] = tok < nr ? v : -INFINITY;
          mx = fmaxf(mx, s[j][c]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      const float mn = fmaxf(m, mx);
      const float alpha = ex2(m - mn);   // m = -inf on the first chunk: alpha = 0
      m = mn;
      if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          acc[nt][0] *= alpha;
          acc[nt][1] *= alpha;
          acc[nt][2] *= alpha;
          acc[nt][3] *= alpha;
        }
        l *= alpha;
      }
      float p[2][2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          p[j][c] = ex2(s[j][c] - mn);
          l += p[j][c];
        }
      // P as the A operand: rows gid = bf16(p), rows gid + 8 = p - bf16(p)
      uint32_t pa[4];
      {
        const float h00 = bf16r(p[0][0]), h01 = bf16r(p[0][1]), h10 = bf16r(p[1][0]), h11 = bf16r(p[1][1]);
        pa[0] = pack2(h00, h01);
        pa[1] = pack2(p[0][0] - h00, p[0][1] - h01);
        pa[2] = pack2(h10, h11);
        pa[3] = pack2(p[1][0] - h10, p[1][1] - h11);
      }
      // O += P V over 128 dims (16 n-tiles of 8)
#pragma unroll
      for (int nt = 0; nt < 16; nt += 2) {
        uint32_t bv[4];
        ldsm_x4_t(bv, vs + (8 * (mi & 1) + rr) * kRowPad + 8 * (nt + (mi >> 1)));
        mma16816(acc[nt], pa, bv[0], bv[1]);
        mma16816(acc[nt + 1], pa, bv[2], bv[3]);
      }
    }

    // ---- warp state: row sums over the 4 lanes of a head, hi + residual rows combined
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    float o[16][2];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] = acc[nt][0] + acc[nt][2];
      o[nt][1] = acc[nt][1] + acc[nt][3];
    }
    // ---- merge the 8 warp states: 8 -> 4 -> 2 -> 1
#pragma unroll
    for (int half = kWarps / 2; half >= 1; half >>= 1) {
      if (warp >= half && warp < 2 * half && gid < G) {
        float* dst = mbuf + ((size_t)(warp - half) * G + gid) * kPartStride;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
          *reinterpret_cast<float2*>(dst + 8 * nt + 2 * t4) = make_float2(o[nt][0], o[nt][1]);
        if (t4 == 0) { dst[kHeadDim] = m; dst[kHeadDim + 1] = l; }
      }
      __syncthreads();
      if (warp < half && gid < G) {
        const float* src = mbuf + ((size_t)warp * G + gid) * kPartStride;
        const float m2 = src[kHeadDim], l2 = src[kHeadDim + 1];
        const float mn = fmaxf(m, m2);
        if (mn != -INFINITY) {
          const float sa = exp2f(m - mn), sb = exp2f(m2 - mn);
          l = l * sa + l2 * sb;
#pragma unroll
          for (int nt = 0; nt < 16; ++nt) {
            const float2 v = *reinterpret_cast<const float2*>(src + 8 * nt + 2 * t4);
            o[nt][0] = o[nt][0] * sa + v.x * sb;
            o[nt][1] = o[nt][1] * sa + v.y * sb;
          }
          m = mn;
        }
      }
      __syncthreads();
    }
    if (warp == 0 && gid < G) {
      float* dst = P.ws.part + ((size_t)(blockIdx.x + it.s) * G + gid) * kPartStride;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<float2*>(dst + 8 * nt + 2 * t4) = make_float2(o[nt][0], o[nt][1]);
      if (t4 == 0) { dst[kHeadDim] = m; dst[kHeadDim + 1] = l; }
      __threadfence();
    }
    // ---- the last CTA to finish a piece of this slice combines its split states
    __syncthreads();
    const int c0 = owner(rpre[it.s]), c1 = owner(rpre[it.s + 1] - 1);
    if (tid == 0) s_merge = atomicAdd(&P.ws.attn_ticket[it.s], 1u) == (unsigned)(c1 - c0);
    __syncthreads();
    if (s_merge) {
      __threadfence();
      combine_slice<G>(P, it.s, c0, c1, cbuf);
      if (tid == 0) P.ws.attn_ticket[it.s] = 0u;   // ready for the next call
    }
  }
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

size_t smem_bytes(int G, int max_slices) {
  return kRingBytes + (size_t)4 * G * kPartStride * 4 + (size_t)(max_slices + 1) * 8 + (size_t)max_slices * 8 +
         16 + (size_t)kWarps * kPartStride * 4;
}

template <int G>
int setup_g(int max_slices) {
  const size_t sm = smem_bytes(G, max_slices);
  if (cudaFuncSetAttribute(k_attend_bf16<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
    return -1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_attend_bf16<G>, kWarps * 32, sm) != cudaSuccess) return -1;
  return n;
}

}  // namespace

cudaError_t launch_attend_bf16(const StepParams& P, int grid, cudaStream_t st) {
  const size_t sm = smem_bytes(P.G, P.n_slices);
  switch (P.G) {
    case 1: k_attend_bf16<1><<<grid, kWarps * 32, sm, st>>>(P); break;
    case 2: k_attend_bf16<2><<<grid, kWarps * 32, sm, st>>>(P); break;
    case 4: k_attend_bf16<4><<<grid, kWarps * 32, sm, st>>>(P); break;
    case 8: k_attend_bf16<8><<<grid, kWarps * 32, sm, st>>>(P); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int attend_bf16_setup(int G, int max_slices) {
  switch (G) {
    case 1: return setup_g<1>(max_slices);
    case 2: return setup_g<2>(max_slices);
    case 4: return setup_g<4>(max_slices);
    case 8: return setup_g<8>(max_slices);
  }
  return -1;
}

}  // namespace spa
