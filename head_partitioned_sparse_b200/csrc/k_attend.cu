// Exact split-K attention over the attended rows of every (b, kv head) slice, and
// the log-sum-exp combine of the splits.
//
// "Full Attention Strikes Back" (RTPurbo summary), Methodology §1: local heads see
// sinks plus a sliding window; retrieval heads additionally see their top-p set.
// "Hierarchical Global Attention" summary, Central mechanism §4: plain softmax over
// the exact selected tokens.  The per-split state (m, l, acc) and its merge follow
// the cached online-softmax state of the S2O summary (Kernel implementation,
// pass 1).
//
// Rows of a slice are numbered virtually: v < n_contig are the sinks then the
// window (contiguous in the cache), v >= n_contig index the slice's selected list.
// A split ("item") covers split_rows consecutive virtual rows.  A persistent grid
// walks the items; each CTA stages kTile rows of K and V per step in shared memory
// with cp.async (double buffered), scores them against the G query heads of the
// group, keeps an online softmax per head, and writes (m, l, acc) for the split.
#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ int slice_items(const StepParams& P, int s, int* n_rows_out) {
  const int b = s / P.Hkv, g = s % P.Hkv;
  const int L = load_len(P.seq_lens, b, P.Lcap, P.ws.dev_err);
  const SinkWindow sw(L, P.n_sink, P.window);
  const int n = sw.n_contig() + (P.is_ret[g] ? P.ws.st[s].count : 0);
  if (n_rows_out) *n_rows_out = n;
  return (n + P.split_rows - 1) / P.split_rows;
}

template <typename T, int G>
struct AttnSmem {
  static constexpr int kRowElems = kHeadDim;
  static constexpr size_t kKV = (size_t)kTile * kRowElems * sizeof(T);  // one K (or V) tile
  static size_t bytes(int n_slices) {
    return 2 * 2 * kKV + (size_t)G * kHeadDim * 4 + (size_t)G * kTile * 4 + 4 * G * 4 +
           (size_t)(n_slices + 1) * 4 + 64;
  }
};

template <typename T, int G>
__global__ void __launch_bounds__(kAttnThreads) k_attend(StepParams P) {
  extern __shared__ __align__(16) unsigned char smem[];
  using S = AttnSmem<T, G>;
  T* kv = reinterpret_cast<T*>(smem);                       // [2 buf][K|V][kTile][128]
  float* qs = reinterpret_cast<float*>(smem + 4 * S::kKV);  // [G][128]
  float* ps = qs + G * kHeadDim;                            // [G][kTile]
  float* mrun = ps + G * kTile;                             // [G]
  float* lrun = mrun + G;                                   // [G]
  float* alpha = lrun + G;                                  // [G]
  int* pref = reinterpret_cast<int*>(alpha + 2 * G);        // [n_slices + 1]
  __shared__ int shi[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = P.n_slices;

  // item prefix over slices (every CTA computes it; CTA 0 publishes it for the combine)
  int carry = 0;
  for (int base = 0; base < NS; base += kAttnThreads) {
    const int s = base + tid;
    const int it = s < NS ? slice_items(P, s, nullptr) : 0;
    int tot;
    // block exclusive scan
    int v = it;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(kFull, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) shi[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = lane < kAttnThreads / 32 ? shi[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(kFull, w, o);
        if (lane >= o) w += y;
      }
      if (lane < kAttnThreads / 32) shi[lane] = w;
    }
    __syncthreads();
    const int pre = (warp ? shi[warp - 1] : 0) + v - it;
    tot = shi[kAttnThreads / 32 - 1];
    if (s < NS) pref[s] = carry + pre;
    carry += tot;
    __syncthreads();
  }
  if (tid == 0) pref[NS] = carry;
  __syncthreads();
  const int total_items = pref[NS];
  if (blockIdx.x == 0)
    for (int s = tid; s <= NS; s += kAttnThreads) P.ws.item_base[s] = pref[s];

  constexpr int kCpr = kHeadDim * sizeof(T) / 16;  // 16-byte chunks per row
  int cur_slice = -1;
  for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
    // locate the slice: largest s with pref[s] <= item
    int lo = 0, hi = NS - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pref[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int b = s / P.Hkv, g = s % P.Hkv;
    int n_rows;
    slice_items(P, s, &n_rows);
    const int L = load_len(P.seq_lens, b, P.Lcap, P.ws.dev_err);
    const SinkWindow sw(L, P.n_sink, P.window);
    const int nc = sw.n_contig();
    const int v0 = (item - pref[s]) * P.split_rows;
    const int v1 = min(v0 + P.split_rows, n_rows);
    const KvSlice<T> kvs = kv_slice<T>(P, s);
    const T* kbase = kvs.k;
    const T* vbase = kvs.v;
    const bool ring = kvs.ring;
    const int* list = P.sel_list + (size_t)s * P.Lmax;

    __syncthreads();  // previous item done with qs / buffers
    if (s != cur_slice) {
      for (int i = tid; i < G * kHeadDim; i += kAttnThreads)
        qs[i] = P.ws.q_rot[((size_t)b * P.Hq + (size_t)g * G) * kHeadDim + i];
      cur_slice = s;
    }
    if (tid < G) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; }

    auto issue = [&](int t, int buf) {
      const int r0 = v0 + t * kTile;
      const int nr = min(kTile, v1 - r0);
      T* kd = kv + (size_t)buf * 2 * kTile * kHeadDim;
      T* vd = kd + kTile * kHeadDim;
      for (int i = tid; i < nr * kCpr; i += kAttnThreads) {
        const int r = i / kCpr, c = i % kCpr;
        const int v = r0 + r;
        int pos = v < nc ? sw.contig_pos(v) : list[v - nc];
        if (ring) pos = ring_row(pos, P.n_sink, P.window);   // streaming head, compact layout
        cp_async16(kd + r * kHeadDim + c * (16 / sizeof(T)), kbase + (size_t)pos * kHeadDim + c * (16 / sizeof(T)));
        cp_async16(vd + r * kHeadDim + c * (16 / sizeof(T)), vbase + (size_t)pos * kHeadDim + c * (16 / sizeof(T)));
      }
      cp_async_commit();
    };

    // PV ownership: dim d, heads [h0, h0 + HP)
    constexpr int HP = G >= 2 ? G / 2 : 1;
    const int d = tid & (kHeadDim - 1);
    const int h0 = G >= 2 ? (tid >> 7) * HP : 0;
    const bool pv_active = G >= 2 || tid < kHeadDim;
    float acc[HP];
#pragma unroll
    for (int k = 0; k < HP; ++k) acc[k] = 0.f;
    // score ownership: lane holds dims [4 lane, 4 lane + 4) of q for every head
    float qreg[G][4];
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) qreg[h][i] = qs[h * kHeadDim + 4 * lane + i];

    const int ntiles = (v1 - v0 + kTile - 1) / kTile;
    issue(0, 0);
    for (int t = 0; t < ntiles; ++t) {
      if (t + 1 < ntiles) { issue(t + 1, (t + 1) & 1); cp_async_wait<1>(); }
      else cp_async_wait<0>();
      __syncthreads();
      const int nr = min(kTile, v1 - (v0 + t * kTile));
      const T* kd = kv + (size_t)(t & 1) * 2 * kTile * kHeadDim;
      const T* vd = kd + kTile * kHeadDim;
      // scores, log2 units
      for (int r = warp; r < kTile; r += kAttnThreads / 32) {
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
        if (r < nr) {
          float kx[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) kx[i] = Elem<T>::get(kd + r * kHeadDim, 4 * lane + i);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) a = fmaf(qreg[h][i], kx[i], a);
            part[h] = a;
          }
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part[h] += __shfl_xor_sync(kFull, part[h], o);
        }
        float mine = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h)
          if (lane == h) mine = part[h];
        if (lane < G) ps[lane * kTile + r] = r < nr ? mine * P.attn_scale_log2 : -INFINITY;
      }
      __syncthreads();
      // online softmax update, one warp per head
      if (warp < G) {
        const int h = warp;
        const float s0 = ps[h * kTile + lane], s1 = ps[h * kTile + lane + 32];
        float mx = fmaxf(s0, s1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        const float mold = mrun[h];
        const float mnew = fmaxf(mold, mx);
        const float p0 = exp2f(s0 - mnew), p1 = exp2f(s1 - mnew);
        ps[h * kTile + lane] = p0;
        ps[h * kTile + lane + 32] = p1;
        float sum = p0 + p1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
        if (lane == 0) {
          const float a = exp2f(mold - mnew);
          alpha[h] = a;
          lrun[h] = lrun[h] * a + sum;
          mrun[h] = mnew;
        }
      }
      __syncthreads();
      if (pv_active) {
#pragma unroll
        for (int k = 0; k < HP; ++k) acc[k] *= alpha[h0 + k];
        for (int r = 0; r < nr; ++r) {
          const float vv = Elem<T>::get(vd + r * kHeadDim, d);
#pragma unroll
          for (int k = 0; k < HP; ++k) acc[k] = fmaf(ps[(h0 + k) * kTile + r], vv, acc[k]);
        }
      }
      __syncthreads();
    }
    // write the split's state: [acc 128][m][l][pad 2] per head
    float* dst = P.ws.part + (size_t)item * G * kPartStride;
    if (pv_active)
#pragma unroll
      for (int k = 0; k < HP; ++k) dst[(h0 + k) * kPartStride + d] = acc[k];
    if (tid < G) {
      dst[tid * kPartStride + kHeadDim] = mrun[tid];
      dst[tid * kPartStride + kHeadDim + 1] = lrun[tid];
    }
  }
}

// One CTA per (slice, head): warp w merges the splits w, w + kCombWarps, ... of the
// slice (lane = 4 dims), loading kCombBatch splits before merging any, then warp
// states are merged in warp order.  Deterministic.
constexpr int kCombWarps = 16;
constexpr int kCombBatch = 4;

template <int G>
__global__ void __launch_bounds__(kCombWarps * 32) k_combine(StepParams P) {
  __shared__ float wm[kCombWarps], wl[kCombWarps];
  __shared__ __align__(16) float wacc[kCombWarps][kHeadDim];
  const int s = blockIdx.x / G, h = blockIdx.x % G;
  const int b = s / P.Hkv, g = s % P.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i0 = P.ws.item_base[s], i1 = P.ws.item_base[s + 1];
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int ib = i0 + warp; ib < i1; ib += kCombWarps * kCombBatch) {
    float4 a[kCombBatch];
    float mi[kCombBatch], li[kCombBatch];
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
      const int i = ib + u * kCombWarps;
      if (i < i1) {
        const float* pp = P.ws.part + ((size_t)i * G + h) * kPartStride;
        a[u] = *reinterpret_cast<const float4*>(pp + 4 * lane);
        mi[u] = pp[kHeadDim];
        li[u] = pp[kHeadDim + 1];
      } else {
        a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        mi[u] = -INFINITY;
        li[u] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
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
  if (lane == 0) { wm[warp] = m; wl[warp] = l; }
  *reinterpret_cast<float4*>(&wacc[warp][4 * lane]) = acc;
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
    for (int w = 0; w < kCombWarps; ++w) M = fmaxf(M, wm[w]);
    float den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w = 0; w < kCombWarps; ++w) {
      if (wm[w] == -INFINITY) continue;
      const float sc = exp2f(wm[w] - M);
      den = fmaf(sc, wl[w], den);
      const float4 v = *reinterpret_cast<const float4*>(&wacc[w][4 * lane]);
      num.x = fmaf(sc, v.x, num.x);
      num.y = fmaf(sc, v.y, num.y);
      num.z = fmaf(sc, v.z, num.z);
      num.w = fmaf(sc, v.w, num.w);
    }
    const float inv = 1.f / den;
    const float4 o = make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
    *reinterpret_cast<float4*>(P.out + ((size_t)b * P.Hq + (size_t)g * G + h) * kHeadDim + 4 * lane) = o;
  }
  if (threadIdx.x == 0 && h == 0 && P.sel_count) P.sel_count[s] = P.is_ret[g] ? P.ws.st[s].count : 0;
}

template <typename T, int G>
cudaError_t launch_attend_tg(const StepParams& P, int grid, cudaStream_t st) {
  const size_t sm = AttnSmem<T, G>::bytes(P.n_slices);
  k_attend<T, G><<<grid, kAttnThreads, sm, st>>>(P);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_attend_t(const StepParams& P, int grid, cudaStream_t st) {
  switch (P.G) {
    case 1: return launch_attend_tg<T, 1>(P, grid, st);
    case 2: return launch_attend_tg<T, 2>(P, grid, st);
    case 4: return launch_attend_tg<T, 4>(P, grid, st);
    case 8: return launch_attend_tg<T, 8>(P, grid, st);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int G>
int setup_tg(int max_slices) {
  const size_t sm = AttnSmem<T, G>::bytes(max_slices);
  if (cudaFuncSetAttribute(k_attend<T, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
    return -1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_attend<T, G>, kAttnThreads, sm) != cudaSuccess) return -1;
  return n;
}

}  // namespace

cudaError_t launch_attend(const StepParams& P, int kv_dtype, int grid, cudaStream_t st) {
  // bf16 caches: tensor-core kernel (k_attend_mma.cu); float32 caches: this file's kernel
  return kv_dtype == 0 ? launch_attend_bf16(P, grid, st) : launch_attend_t<float>(P, grid, st);
}

cudaError_t launch_combine(const StepParams& P, cudaStream_t st) {
  switch (P.G) {
    case 1: k_combine<1><<<P.n_slices * 1, kCombWarps * 32, 0, st>>>(P); break;
    case 2: k_combine<2><<<P.n_slices * 2, kCombWarps * 32, 0, st>>>(P); break;
    case 4: k_combine<4><<<P.n_slices * 4, kCombWarps * 32, 0, st>>>(P); break;
    case 8: k_combine<8><<<P.n_slices * 8, kCombWarps * 32, 0, st>>>(P); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Sets the dynamic shared-memory limit for the (dtype, G) instantiation and returns
// resident CTAs per SM (or -1).
int attend_setup(int kv_dtype, int G, int max_slices) {
  if (kv_dtype == 0) return attend_bf16_setup(G, max_slices);
  switch (G) {
    case 1: return setup_tg<float, 1>(max_slices);
    case 2: return setup_tg<float, 2>(max_slices);
    case 4: return setup_tg<float, 4>(max_slices);
    case 8: return setup_tg<float, 8>(max_slices);
  }
  return -1;
}

}  // namespace spa
