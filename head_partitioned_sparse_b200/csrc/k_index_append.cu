// Index append: bf16 16-dim index rows from pre-RoPE keys.
//
// "Full Attention Strikes Back" (RTPurbo summary), Methodology §2: a 16-dim
// projector is applied to the key features before RoPE is injected; relevance is
// then estimated in that compact subspace.  Each row is
//   idx[r] = bf16_rne( sum_d P_k[g][r][d] * k_pre[d] ),  r < 16,
// the sum accumulated in float32.
//
// bf16 keys (k_index_append_bulk): the projection is a dense [tokens x 128] x [128 x 16]
// contraction, 14 flops per byte moved, more than the float32 pipes sustain at HBM
// rate, so it runs on the tensor cores (mma.sync m16n8k16, bf16 in, float32
// accumulate).  The projector is split exactly into three bf16 parts (hi + mid + lo =
// the float32 value), so every product is exact and the three parts accumulate into
// the same float32 sums.  The key rows reach shared memory through the copy engine
// (one 256-byte bulk copy per row, completion counted on an mbarrier), two 16-token
// tiles per warp in flight; the 128 dims are permuted consistently in A and B so that
// each lane's 16-byte shared loads are conflict-free.  Output columns are permuted so
// that a lane ends with four consecutive outputs of a row and writes them as one 8-byte
// store.  The B fragments of the head's projector are built once per CTA (2048 tokens)
// in shared memory, in fragment order, while the first tiles are in flight.
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

// ---------------------------------------------------------------- bulk-copy variant
// The same contraction with the key rows staged in shared memory by the copy engine:
// each warp owns a ring of kIbStages 16-row tiles, and lane r < 16 requests row r of a
// tile with one bulk copy (cp.async.bulk, 256 B, completion counted on the stage's
// mbarrier), so a tile's bytes stay in flight without holding registers.  Rows sit
// kIbRowB = 320 bytes apart, so the two rows a quarter-warp reads with one 16-byte
// shared load fall into disjoint banks.  Lane t4 reads the 16-byte chunks t4, t4 + 4,
// t4 + 8, t4 + 12 of its rows: k-step s, lane t4 covers physical dims
// 32 (s >> 1) + 8 t4 + 4 (s & 1) .. + 3.  The stage is handed back to the copy engine
// as soon as the warp holds the tile in registers (after a proxy fence), then the
// tile is contracted.  Every mbarrier wait is bounded; a wait that gives up sets the
// status word, waits (bounded) for this warp's other copies and stops.
constexpr int kIbWarps = 8;
constexpr int kIbStages = 2;
constexpr int kIbTiles = 16;                              // 16-token tiles per warp
constexpr int kIbTok = kIbWarps * kIbTiles * 16;          // 2048 tokens per CTA
constexpr int kIbRowB = 320;                              // shared-memory row stride, bytes
constexpr int kIbTileB = 16 * kIbRowB;
constexpr int kIbFragB = 8 * 2 * 3 * 32 * 8;              // B fragments
constexpr int kIbSmem = kIbFragB + kIbWarps * kIbStages * kIbTileB + kIbWarps * kIbStages * 8;
constexpr long long kIbWaitCycles = 4000000000LL;         // ~2 s per wait

__device__ __forceinline__ uint32_t ib_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool ib_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  for (int n = 0;; ++n) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}\n"
        : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    if (done) return true;
    if ((n & 255) == 255 && clock64() - t0 > kIbWaitCycles) return false;
  }
}

__global__ void __launch_bounds__(kIbWarps * 32, 2)
k_index_append_bulk(const __nv_bfloat16* __restrict__ k_pre, const int64_t* __restrict__ start_pos, int T_, int Hkv,
                    int64_t Lmax, const float* __restrict__ P_k, uint16_t* __restrict__ idx,
                    unsigned* __restrict__ err, const HeadMap map) {
  extern __shared__ __align__(128) unsigned char ib_sm[];
  uint2 (*bfrag)[2][3][32] = reinterpret_cast<uint2 (*)[2][3][32]>(ib_sm);
  unsigned char* ring = ib_sm + kIbFragB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kIbWarps * kIbStages * kIbTileB);
  const int b = blockIdx.y / map.n, m = blockIdx.y % map.n;
  const int g = map.g[m];
  const int s_src = b * Hkv + g;
  const int sd = b * map.n_slots + map.slot[m];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
  const __nv_bfloat16* src = k_pre + (size_t)s_src * T_ * kHeadDim;
  const int tok_cta = blockIdx.x * kIbTok;
  // this warp's tiles: warp, warp + 8, ... while they start before T_
  int n_w = 0;
  if (tok_cta + warp * 16 < T_) n_w = min(kIbTiles, (T_ - tok_cta - warp * 16 + 16 * kIbWarps - 1) / (16 * kIbWarps));
  unsigned char* wring = ring + warp * kIbStages * kIbTileB;
  const uint32_t wbar = ib_smem(bars + warp * kIbStages);
  if (lane == 0) {
    for (int st = 0; st < kIbStages; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" :: "r"(wbar + 8 * st) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncwarp();
  // tile j of this warp into stage j % kIbStages: lane 0 announces the bytes, lane r < 16
  // copies row r
  auto issue = [&](int j) {
    const int tok0 = tok_cta + (warp + kIbWarps * j) * 16;
    const int nrows = min(16, T_ - tok0);
    const uint32_t bar = wbar + 8 * (j % kIbStages);
    if (lane == 0)
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" :: "r"(bar), "r"(nrows * 256) : "memory");
    __syncwarp();
    if (lane < nrows) {
      const uint32_t dst = ib_smem(wring + (j % kIbStages) * kIbTileB + lane * kIbRowB);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 256, [%2];\n"
          :: "r"(dst), "l"(src + (size_t)(tok0 + lane) * kHeadDim), "r"(bar) : "memory");
    }
  };
  for (int j = 0; j < kIbStages && j < n_w; ++j) issue(j);
  // the projector's B fragments, built while the first tiles are in flight
  const float* Pg = P_k + (size_t)g * kIdxDim * kHeadDim;
  for (int i = tid; i < 8 * 2 * 3 * 32; i += blockDim.x) {
    const int ln = i & 31, part = (i >> 5) % 3, t = (i / 96) & 1, ks = i / 192;
    const int c = ln >> 2, q4 = ln & 3;
    const int r = 4 * (c >> 1) + 2 * t + (c & 1);
    const int d0 = 32 * (ks >> 1) + 8 * q4 + 4 * (ks & 1);
    const float* pr = Pg + (size_t)r * kHeadDim + d0;
    uint2 v;
    v.x = ia_pack(ia_part(pr[0], part), ia_part(pr[1], part));
    v.y = ia_pack(ia_part(pr[2], part), ia_part(pr[3], part));
    bfrag[ks][t][part][ln] = v;
  }
  __syncthreads();
  const int64_t base_pos = start_pos[b];
  int j = 0;
  for (; j < n_w; ++j) {
    const int st = j % kIbStages;
    if (!ib_wait(wbar + 8 * st, (uint32_t)(j / kIbStages) & 1u)) {
      atomicOr(err, kErrTimeout);
      break;
    }
    const unsigned char* tb = wring + st * kIbTileB;
    uint4 qa[4], qb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qa[i] = *reinterpret_cast<const uint4*>(tb + gid * kIbRowB + 64 * i + 16 * t4);
      qb[i] = *reinterpret_cast<const uint4*>(tb + (gid + 8) * kIbRowB + 64 * i + 16 * t4);
    }
    // the warp's reads of the stage are done before the copy engine refills it
    __syncwarp();
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    if (j + kIbStages < n_w) issue(j + kIbStages);
    const int ra = tok_cta + (warp + kIbWarps * j) * 16 + gid, rb = ra + 8;
    float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint4 wa = qa[ks >> 1], wb = qb[ks >> 1];
      uint32_t a[4];
      a[0] = (ks & 1) ? wa.z : wa.x;
      a[1] = (ks & 1) ? wb.z : wb.x;
      a[2] = (ks & 1) ? wa.w : wa.y;
      a[3] = (ks & 1) ? wb.w : wb.y;
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int part = 0; part < 3; ++part) ia_mma(c[t], a, bfrag[ks][t][part][lane]);
    }
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
  }
  if (j < n_w) {
    // a wait gave up: let this warp's copies still in flight land before leaving
    for (int k = j; k < n_w && k < j + kIbStages; ++k) ib_wait(wbar + 8 * (k % kIbStages), (uint32_t)(k / kIbStages) & 1u);
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
    // the copies need 16-byte aligned rows: the entry points reject other k_pre pointers
    if ((reinterpret_cast<uintptr_t>(k_pre) & 15u) != 0u) return cudaErrorMisalignedAddress;
    static bool smem_set[64] = {};   // per device: the shared-memory limit is raised once
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !smem_set[dev]) {
      e = cudaFuncSetAttribute(k_index_append_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, kIbSmem);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) smem_set[dev] = true;
    }
    const dim3 grid_b((T + kIbTok - 1) / kIbTok, B * m.n);
    k_index_append_bulk<<<grid_b, kIbWarps * 32, kIbSmem, st>>>((const __nv_bfloat16*)k_pre, start_pos, T, Hkv,
                                                                Lmax, P_k, idx_cache, dev_err, m);
  } else
    k_index_append<float><<<grid, 256, 0, st>>>((const float*)k_pre, start_pos, T, Hkv, Lmax, P_k,
                                                 idx_cache, dev_err, m);
  return cudaGetLastError();
}

}  // namespace spa
