// Index append: bf16 16-dim index rows from pre-RoPE keys.
//
// "Full Attention Strikes Back" (RTPurbo summary), Methodology §2: a 16-dim
// projector is applied to the key features before RoPE is injected; relevance is
// then estimated in that compact subspace.  Each row is
//   idx[r] = bf16_rne( sum_d P_k[g][r][d] * k_pre[d] ),  r < 16,
// the sum accumulated in float32.
//
// bf16 keys (k_index_append_mma): the projection is a dense [tokens x 128] x [128 x 16]
// contraction, 14 flops per byte moved, more than the float32 pipes sustain at HBM
// rate, so it runs on the tensor cores (mma.sync m16n8k16, bf16 in, float32
// accumulate).  The projector is split exactly into three bf16 parts (hi + mid + lo =
// the float32 value), so every product is exact and the three parts accumulate into
// the same float32 sums.  A warp takes 16-token tiles; each lane loads 64 contiguous
// bytes of two key rows straight from global memory (16-byte loads; the next tile's
// rows are requested before the current tile is computed), because the
// 128 dims are permuted consistently in A and B: k-step s, lane t4 covers physical
// dims 32 t4 + 4 s .. + 3.  Output columns are permuted so that a lane ends with four
// consecutive outputs of a row and writes them as one 8-byte store.  The B fragments
// of the head's projector are built once per CTA (2048 tokens) in shared memory, in
// fragment order.
//
// float32 keys (k_index_append): a CTA takes 64 consecutive tokens of one (b, kv head);
// the key tile (rows padded to 129 floats so a warp's 8 rows hit 8 banks) and the
// head's projector sit in shared memory; each thread produces 4 of a row's 16 outputs
// (float32 products and sums in ascending d) and writes them as one 8-byte store.
//
// Both run over the head map: all heads in place, or the retrieval heads only at their
// rank for the compact layout.
#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr int kRowsPerCta = 64;
constexpr int kPad = kHeadDim + 1;

template <typename T>
__global__ void __launch_bounds__(256)
k_index_append(const T* __restrict__ k_pre, const int64_t* __restrict__ start_pos, int T_, int Hkv,
               int64_t Lmax, const float* __restrict__ P_k, uint16_t* __restrict__ idx,
               unsigned* __restrict__ err, const HeadMap map) {
  __shared__ float ks[kRowsPerCta][kPad];
  __shared__ float ps[kIdxDim][kPad];
  const int b = blockIdx.y / map.n, m = blockIdx.y % map.n;
  const int g = map.g[m];
  const int s = b * Hkv + g;                      // source (b, head)
  const int sd = b * map.n_slots + map.slot[m];   // destination (b, slot)
  const int t0 = blockIdx.x * kRowsPerCta;
  const int nrows = min(kRowsPerCta, T_ - t0);
  const int tid = threadIdx.x;

  for (int i = tid; i < kIdxDim * kHeadDim; i += blockDim.x)
    ps[i / kHeadDim][i % kHeadDim] = P_k[(size_t)g * kIdxDim * kHeadDim + i];
  const T* src = k_pre + ((size_t)s * T_ + t0) * kHeadDim;
  for (int i = tid; i < nrows * kHeadDim; i += blockDim.x)
    ks[i / kHeadDim][i % kHeadDim] = Elem<T>::get(src, i);
  __syncthreads();

  const int row = tid >> 2;
  const int r0 = (tid & 3) * 4;
  if (row >= nrows) return;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // float32 product, then float32 add, in ascending d
#pragma unroll 4
  for (int d = 0; d < kHeadDim; ++d) {
    const float x = ks[row][d];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(ps[r0 + i][d], x));
  }
  const int64_t pos = start_pos[b] + t0 + row;
  if (pos < 0 || pos >= Lmax) {
    atomicOr(err, kErrStartPos);
    return;
  }
  uint2 packed;
  packed.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[0])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[1])) << 16);
  packed.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[3])) << 16);
  *reinterpret_cast<uint2*>(idx + ((size_t)sd * Lmax + pos) * kIdxDim + r0) = packed;
}

// ---------------------------------------------------------------- tensor-core variant
constexpr int kIaWarps = 8;
constexpr int kIaTiles = 16;                              // 16-token tiles per warp
constexpr int kIaTok = kIaWarps * kIaTiles * 16;          // 2048 tokens per CTA

__device__ __forceinline__ void ia_mma(float (&d)[4], const uint32_t (&a)[4], uint2 b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y));
}

__device__ __forceinline__ uint32_t ia_pack(float x, float y) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Part p (0 hi, 1 mid, 2 lo) of the exact three-way bf16 split of x.
__device__ __forceinline__ float ia_part(float x, int p) {
  const float hi = __bfloat162float(__float2bfloat16_rn(x));
  if (p == 0) return hi;
  const float mid = __bfloat162float(__float2bfloat16_rn(x - hi));
  if (p == 1) return mid;
  return __bfloat162float(__float2bfloat16_rn((x - hi) - mid));
}

__global__ void __launch_bounds__(kIaWarps * 32)
k_index_append_mma(const __nv_bfloat16* __restrict__ k_pre, const int64_t* __restrict__ start_pos, int T_, int Hkv,
                   int64_t Lmax, const float* __restrict__ P_k, uint16_t* __restrict__ idx, unsigned* __restrict__ err,
                   const HeadMap map) {
  // B fragments [k-step][n-tile][part][lane]: column c of n-tile t is output
  // r = 4 (c >> 1) + 2 t + (c & 1); k-step s, logical k -> physical dim
  // 32 ((k & 7) >> 1) + 4 s + 2 (k >> 3) + (k & 1).
  __shared__ uint2 bfrag[8][2][3][32];
  const int b = blockIdx.y / map.n, m = blockIdx.y % map.n;
  const int g = map.g[m];
  const int s_src = b * Hkv + g;
  const int sd = b * map.n_slots + map.slot[m];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
  const int64_t base_pos = start_pos[b];
  const __nv_bfloat16* src = k_pre + (size_t)s_src * T_ * kHeadDim;
  // warp w takes tiles w, w + 8, ... of the CTA's 2048 tokens; the next tile's rows are
  // requested before the current tile is computed (two tiles in flight per warp)
  auto load_tile = [&](int tile, uint4 (&qa)[4], uint4 (&qb)[4]) {
    const int tok0 = blockIdx.x * kIaTok + tile * 16;
    const int ra = tok0 + gid, rb = ra + 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qa[i] = ra < T_ ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)ra * kHeadDim + 32 * t4) + i)
                      : make_uint4(0u, 0u, 0u, 0u);
      qb[i] = rb < T_ ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)rb * kHeadDim + 32 * t4) + i)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  const float* Pg = P_k + (size_t)g * kIdxDim * kHeadDim;
  for (int i = tid; i < 8 * 2 * 3 * 32; i += blockDim.x) {
    const int ln = i & 31, part = (i >> 5) % 3, t = (i / 96) & 1, ks = i / 192;
    const int c = ln >> 2, q4 = ln & 3;
    const int r = 4 * (c >> 1) + 2 * t + (c & 1);
    const int d0 = 32 * q4 + 4 * ks;
    const float* pr = Pg + (size_t)r * kHeadDim + d0;
    uint2 v;
    v.x = ia_pack(ia_part(pr[0], part), ia_part(pr[1], part));
    v.y = ia_pack(ia_part(pr[2], part), ia_part(pr[3], part));
    bfrag[ks][t][part][ln] = v;
  }
  __syncthreads();
  uint4 qa[4], qb[4], na[4], nb[4];
  int tile = warp;
  if (blockIdx.x * kIaTok + tile * 16 < T_) load_tile(tile, qa, qb);
  for (; tile < kIaWarps * kIaTiles && blockIdx.x * kIaTok + tile * 16 < T_; tile += kIaWarps) {
    const int next = tile + kIaWarps;
    const bool more = next < kIaWarps * kIaTiles && blockIdx.x * kIaTok + next * 16 < T_;
    if (more) load_tile(next, na, nb);
    const int ra = blockIdx.x * kIaTok + tile * 16 + gid, rb = ra + 8;
    float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint4 wa = qa[ks >> 1], wb = qb[ks >> 1];
      uint32_t a[4];
      a[0] = (ks & 1) ? wa.z : wa.x;   // row gid, dims 4s + 0, 1 of the lane's 32
      a[1] = (ks & 1) ? wb.z : wb.x;   // row gid + 8
      a[2] = (ks & 1) ? wa.w : wa.y;   // row gid, dims 4s + 2, 3
      a[3] = (ks & 1) ? wb.w : wb.y;
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int part = 0; part < 3; ++part) ia_mma(c[t], a, bfrag[ks][t][part][lane]);
    }
    // lane t4 holds outputs 4 t4 .. 4 t4 + 3 of rows gid and gid + 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = h ? rb : ra;
      if (row >= T_) continue;
      const int64_t pos = base_pos + row;
      if (pos < 0 || pos >= Lmax) {
        atomicOr(err, kErrStartPos);
        continue;
      }
      uint2 packed;
      packed.x = ia_pack(c[0][2 * h], c[0][2 * h + 1]);
      packed.y = ia_pack(c[1][2 * h], c[1][2 * h + 1]);
      *reinterpret_cast<uint2*>(idx + ((size_t)sd * Lmax + pos) * kIdxDim + 4 * t4) = packed;
    }
    if (more) {
#pragma unroll
      for (int i = 0; i < 4; ++i) { qa[i] = na[i]; qb[i] = nb[i]; }
    }
  }
}

}  // namespace

cudaError_t launch_index_append(const void* k_pre, const int64_t* start_pos, int B, int T, int Hkv,
                                int64_t Lmax, int kv_dtype, const float* P_k, uint16_t* idx_cache,
                                unsigned* dev_err, cudaStream_t st, const HeadMap* map) {
  HeadMap m;
  if (map) {
    m = *map;
  } else {
    m.n = m.n_slots = Hkv;
    for (int g = 0; g < Hkv; ++g) m.g[g] = m.slot[g] = g;
  }
  if (m.n == 0) return cudaSuccess;
  dim3 grid((T + kRowsPerCta - 1) / kRowsPerCta, B * m.n);
  if (kv_dtype == 0) {
    const dim3 grid_mma((T + kIaTok - 1) / kIaTok, B * m.n);
    k_index_append_mma<<<grid_mma, kIaWarps * 32, 0, st>>>((const __nv_bfloat16*)k_pre, start_pos, T, Hkv, Lmax,
                                                           P_k, idx_cache, dev_err, m);
  } else
    k_index_append<float><<<grid, 256, 0, st>>>((const float*)k_pre, start_pos, T, Hkv, Lmax, P_k,
                                                 idx_cache, dev_err, m);
  return cudaGetLastError();
}

}  // namespace spa
