// Prefill chunk attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// Semantics are those of the prefill oracle ("Full Attention Strikes Back" (RTPurbo
// summary), Methodology §1; "Autonomy of Heads" summary, Deployment strategy): a query
// at absolute position t attends keys j <= t, every one on a retrieval head and the
// sinks (j < n_sink) plus the window (j > t - window) on a streaming head.  The query
// is rotated to its position (float64 angles in units of pi) and rounded to bf16; the
// probabilities are rounded to bf16 for P V; scores and accumulators are float32.
//
// One CTA: one (b, KV head) and 128 query rows (the group's G heads x 128/G positions,
// so the G heads share every K/V tile).  Warp specialised, 9 warps:
//   control warp (its lane 0): TMA loads of the K and V tiles (128 keys x 128 dims,
//     two 64-column boxes each, 128-byte swizzle) into two-stage rings, and the MMAs:
//     S_it = Q K_it^T (8 tcgen05.mma, M = N = 128, K = 16) into one of two TMEM S
//     buffers as soon as the tile before has been consumed, and O += P_it V_it once
//     the softmax warps have written P_it;
//   8 softmax warps: row r (TMEM lane r) belongs to lane r % 32 of warps r / 32 and
//     r / 32 + 4 (a warp may only touch its own quarter of the TMEM lanes), which take
//     its column halves; they read S from TMEM, mask it (tiles every row attends whole
//     skip the mask), agree on the row maximum through shared memory at a named barrier
//     of the two warps, keep the running maximum unless a score exceeds it by more than
//     2^8 (then the O row in TMEM is rescaled), and write P = 2^(s - m) as bf16.
// Hand-offs are mbarriers (TMA transaction counts, tcgen05.commit, 256 softmax
// arrivals); no CTA-wide barrier runs per tile.  Q, K, V and P sit in shared memory in
// the 128-byte swizzled layout (two 64-column halves; row r of a half at (r/8)*1024 +
// (r%8)*128, 16-byte chunk c at (c ^ r%8)*16): K-major operands for Q, K and P, and an
// MN-major operand (N = head dim) for V.  Keys past the chunk's last position are
// masked, and their V rows zeroed (the TMA reads real cache rows there).  Every
// mbarrier wait is bounded and gives up at once when another warp has aborted; a
// failed CTA sets the device status, frees its tensor memory and leaves.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr int kT = 128;                       // rows per CTA = keys per tile = head dim
constexpr int kTileBytes = kT * kT * 2;       // one bf16 128 x 128 tile (32 KB)
constexpr int kHalf = kTileBytes / 2;         // one 64-column half
constexpr int kSoftWarps = 8;                 // softmax warps: two per TMEM lane group
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kThreads = kSoftThreads + 32;   // plus one control warp (TMA and MMA issue)
constexpr long long kWaitCycles = 2000000000LL;   // ~1 s at 2 GHz
constexpr uint32_t kTmemCols = 512;           // S0 [0, 128), S1 [128, 256), O [256, 384)
constexpr int kKStages = 2, kVStages = 2;   // with Q and P: 6 tiles of 32 KB (+ alignment)

struct TcParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  float* out;
  const int64_t* start;
  const double* inv_freq_pi;
  unsigned* err;
  int T, Hq, Hkv, G, n_sink, window, n_qblocks;
  int64_t Lmax;
  float scale_log2;
  unsigned char is_ret[kMaxKvHeads];
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of (row r, 16-byte chunk c16 in [0, 16)) in a swizzled 128 x 128 bf16 tile.
__device__ __forceinline__ uint32_t sw_off(int r, int c16) {
  const int half = c16 >> 3, c = c16 & 7;
  return (uint32_t)(half * kHalf + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor (sm_100): start, LBO, SBO in 16-byte units, version 1,
// 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: bf16 A and B, float32 D, M = N = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(kT >> 3) << 17) |
         ((uint32_t)(kT >> 4) << 24);
}

__device__ __forceinline__ void mma_tc(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
               :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
// 32 consecutive float32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
         "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
         "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
         "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
         "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
         "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
         "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
         "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
         "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
         "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
         "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Packed float32 pairs (one instruction for two lanes of arithmetic).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Bounded mbarrier wait that also gives up as soon as another warp has aborted.
__device__ __forceinline__ bool mbar_wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const uint32_t a = smem_u32(bar);
  const long long t0 = clock64();
  for (int n = 0;; ++n) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}\n"
        : "=r"(done) : "r"(a), "r"(parity) : "memory");
    if (done) return true;
    if ((n & 255) == 255 && (*abort || clock64() - t0 > kWaitCycles)) return false;
  }
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// 3-D tiled TMA load (128-byte swizzle) of box {64, 128, 1} at (x, y, z) into dst.
__device__ __forceinline__ void tma_load3(uint32_t dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;\n" :: "r"(id), "r"(n) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
k_prefill_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const TcParams P) {
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned tiles: Q | P | K0 K1 | V0 V1
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qs = base;
  unsigned char* ps = base + kTileBytes;
  unsigned char* kst = base + 2 * kTileBytes;
  unsigned char* vst = kst + kKStages * kTileBytes;
  __shared__ uint64_t bar_s[2], bar_o, bar_p, bar_k[kKStages], bar_v[kVStages];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ float xch[2][2][kT];   // [iteration parity][column half][row]: row maxima
  __shared__ float xl[2][kT];       // row sums of the two halves

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool control = warp == kSoftWarps;   // TMA and MMA issue (its lane 0)
  const int lg = warp & 3, ch = (warp >> 2) & 1;
  const int r = 32 * lg + lane;
  const int QB = kT / P.G;
  const int qblk = P.n_qblocks - 1 - (int)blockIdx.x;   // heaviest first
  const int bg = blockIdx.y, b = bg / P.Hkv, g = bg % P.Hkv;
  const bool ret = P.is_ret[g] != 0;
  const int64_t start = P.start[b];
  if (start < 0 || start + P.T > P.Lmax) {
    if (tid == 0) atomicOr(P.err, kErrStartPos);
    return;
  }
  const int i0 = qblk * QB;
  const int t_first = (int)start + i0;
  const int t_end = (int)start + min(i0 + QB, P.T);
  const int t_last = t_end - 1;
  const int hl = r / QB, t = t_first + r % QB, h = g * P.G + hl;
  const bool row_ok = t < t_end;

  // key tiles (CTA-uniform)
  int sink_tiles, w_first, w_last;
  if (ret) {
    sink_tiles = 0;
    w_first = 0;
    w_last = t_last / kT;
  } else {
    const int ns = min(P.n_sink, t_end);
    sink_tiles = (ns + kT - 1) / kT;
    const int wlo = max(ns, t_first - P.window + 1);
    w_first = max(wlo / kT, sink_tiles);
    w_last = wlo >= t_end ? w_first - 1 : t_last / kT;
  }
  const int n_tiles = sink_tiles + (w_last >= w_first ? w_last - w_first + 1 : 0);
  auto tile_of = [&](int it) { return it < sink_tiles ? it : w_first + (it - sink_tiles); };
  auto k_stage = [&](int it) { return smem_u32(kst) + (uint32_t)((it % kKStages) * kTileBytes); };
  auto v_stage = [&](int it) { return smem_u32(vst) + (uint32_t)((it % kVStages) * kTileBytes); };
  const int zslice = b * P.Hkv + g;
  auto issue_k = [&](int it) {
    if (it >= n_tiles) return;
    uint64_t* bar = &bar_k[it % kKStages];
    mbar_expect_tx(bar, kTileBytes);
    const int j0 = tile_of(it) * kT;
    tma_load3(k_stage(it), &tm_k, 0, j0, zslice, bar);
    tma_load3(k_stage(it) + kHalf, &tm_k, 64, j0, zslice, bar);
  };
  auto issue_v = [&](int it) {
    if (it >= n_tiles) return;
    uint64_t* bar = &bar_v[it % kVStages];
    mbar_expect_tx(bar, kTileBytes);
    const int j0 = tile_of(it) * kT;
    tma_load3(v_stage(it), &tm_v, 0, j0, zslice, bar);
    tma_load3(v_stage(it) + kHalf, &tm_v, 64, j0, zslice, bar);
  };

  if (control && lane == 0) {
    mbar_init(&bar_s[0], 1);
    mbar_init(&bar_s[1], 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_p, kSoftThreads);
    for (int i = 0; i < kKStages; ++i) mbar_init(&bar_k[i], 1);
    for (int i = 0; i < kVStages; ++i) mbar_init(&bar_v[i], 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    for (int i = 0; i < kKStages; ++i) issue_k(i);
    for (int i = 0; i < kVStages; ++i) issue_v(i);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 :: "r"(smem_u32(&tmem_base)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }

  // ---- Q row r, dims [32 ch, 32 ch + 32) and their rotation partners: rotate to t, bf16
  if (!control) {
    const __nv_bfloat16* src = P.q + (((size_t)b * P.Hq + h) * P.T + (t - (int)start)) * kHeadDim;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int c16 = 4 * ch + cc;   // dims 8 c16 .. 8 c16 + 7 and 64 + 8 c16 ..
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        float r1[2], r2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = 8 * c16 + e + u;
          float x1 = 0.f, x2 = 0.f;
          if (row_ok) {
            x1 = __bfloat162float(src[i]);
            x2 = __bfloat162float(src[i + kHeadDim / 2]);
          }
          const double a = (double)t * P.inv_freq_pi[i];
          double sn, cs;
          sincospi(a - 2.0 * rint(0.5 * a), &sn, &cs);
          r1[u] = (float)((double)x1 * cs - (double)x2 * sn);
          r2[u] = (float)((double)x2 * cs + (double)x1 * sn);
        }
        lo[e / 2] = pk2(r1[0], r1[1]);
        hi[e / 2] = pk2(r2[0], r2[1]);
      }
      *reinterpret_cast<uint4*>(qs + sw_off(r, c16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(qs + sw_off(r, c16 + 8)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
    fence_proxy_async();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_base;
  constexpr uint32_t kIdK = idesc_bf16(false), kIdV = idesc_bf16(true);
  volatile int* ab = &abort_flag;
  auto fail = [&]() {
    atomicOr(&abort_flag, 1);
    atomicOr(P.err, kErrTimeout);
  };

  if (control) {
    // ------------------------------------------------------------ TMA and MMA issue
    if (lane == 0) {
      auto issue_qk = [&](int it) {
        const uint32_t ks = k_stage(it);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_tc(tmem + kT * (it & 1), sdesc(smem_u32(qs) + off, 16, 1024), sdesc(ks + off, 16, 1024), kIdK,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_s[it & 1]);
      };
      bool okc = mbar_wait_ab(&bar_k[0], 0, ab);
      if (okc) {
        fence_after();
        issue_qk(0);
      }
      for (int it = 0; okc && it < n_tiles; ++it) {
        if (it >= 1) {   // P V_{it-1} done: its V stage takes V_{it+1}
          if (!(okc = mbar_wait_ab(&bar_o, (uint32_t)((it - 1) & 1), ab))) break;
          issue_v(it + 1);
        }
        if (it + 1 < n_tiles) {   // S_{it+1}: its buffer was read by softmax_{it-1} (done: P V_{it-1} ran)
          if (!(okc = mbar_wait_ab(&bar_k[(it + 1) % kKStages], (uint32_t)(((it + 1) / kKStages) & 1), ab))) break;
          fence_after();
          issue_qk(it + 1);
        }
        // O += P_it V_it once every softmax thread has written P_it
        if (!(okc = mbar_wait_ab(&bar_p, (uint32_t)(it & 1), ab))) break;
        if (!(okc = mbar_wait_ab(&bar_v[it % kVStages], (uint32_t)((it / kVStages) & 1), ab))) break;
        fence_after();
        const uint32_t vs = v_stage(it);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          // A = P (K-major, keys 16 kk ..), B = V (MN-major: 16 keys = two 8-key groups)
          const uint32_t aoff = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_tc(tmem + 2 * kT, sdesc(smem_u32(ps) + aoff, 16, 1024), sdesc(vs + kk * 2048, kHalf, 1024), kIdV,
                 (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_o);
        issue_k(it + kKStages);   // K_it was consumed by S_it (its softmax has finished)
      }
      if (!okc) fail();
    }
    __syncwarp();   // lanes 1..31 wait for lane 0 before the final CTA barrier
  } else {
    // ------------------------------------------------------------ softmax warps
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t t_o = tmem + lane_off + 2 * kT + 64 * ch;   // this thread's 64 O columns
    float m_run = -INFINITY, l_half = 0.f;
    const float sl2 = P.scale_log2;
    // No early exit: a pair of warps meets at a named barrier every tile, so after a
    // failed wait (the abort flag makes every later wait return at once) a warp runs the
    // remaining tiles without touching tensor memory and still meets its partner.
    bool failed = false;
    for (int it = 0; it < n_tiles; ++it) {
      const int j0 = tile_of(it) * kT;
      bool ok = mbar_wait_ab(&bar_s[it & 1], (uint32_t)((it >> 1) & 1), ab);
      __syncwarp();
      const bool warp_ok = __all_sync(0xffffffffu, ok) && !failed;   // uniform in the warp
      failed = !warp_ok;
      fence_after();
      float s[64];
      if (warp_ok) {
        const uint32_t t_s = tmem + lane_off + kT * (it & 1) + 64 * ch;
        float v32[32];
        tmem_ld32(t_s, v32);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = v32[i];
        tmem_ld32(t_s + 32, v32);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 + i] = v32[i];
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = 0.f;
      }
      const bool full = j0 + kT - 1 <= t_first && (ret || j0 + kT - 1 < P.n_sink || j0 > t_last - P.window);
      if (!full) {
        const int jb = j0 + 64 * ch;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int j = jb + i;
          const bool okj = row_ok && j <= t && (ret || j < P.n_sink || j > t - P.window);
          s[i] = okj ? s[i] : -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; i += 2) mx = max3(mx, s[i], s[i + 1]);
      xch[it & 1][ch][r] = mx;
      named_sync(1 + lg, 64);   // the two warps of lane group lg
      mx = fmaxf(xch[it & 1][0][r], xch[it & 1][1][r]) * sl2;
      // O and P are free once P V_{it-1} has run
      ok = it == 0 || mbar_wait_ab(&bar_o, (uint32_t)((it - 1) & 1), ab);
      __syncwarp();
      failed = failed || !__all_sync(0xffffffffu, ok);
      fence_after();
      const bool raise = mx > m_run + 8.f;
      const float corr = raise ? (m_run == -INFINITY ? 0.f : ex2a(m_run - mx)) : 1.f;
      const bool rescale = raise && m_run != -INFINITY;
      if (!failed && __any_sync(0xffffffffu, rescale)) {
        const float f = rescale ? corr : 1.f;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float v32[32];
          tmem_ld32(t_o + 32 * c, v32);
#pragma unroll
          for (int i = 0; i < 32; ++i) v32[i] *= f;
          tmem_st32(t_o + 32 * c, v32);
        }
      }
      if (raise) {
        l_half *= corr;
        m_run = mx;
      }
      const float nm = m_run == -INFINITY ? 0.f : -m_run;
      const bool live = m_run != -INFINITY;
      const uint64_t sl2x2 = f2pack(sl2, sl2), nmx2 = f2pack(nm, nm);
      uint64_t acc2 = f2pack(0.f, 0.f);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float z0, z1;
          f2unpack(f2fma(f2pack(s[8 * cc + 2 * e], s[8 * cc + 2 * e + 1]), sl2x2, nmx2), z0, z1);
          const float p0 = live ? ex2a(z0) : 0.f;
          const float p1 = live ? ex2a(z1) : 0.f;
          acc2 = f2add(acc2, f2pack(p0, p1));
          w[e] = pk2(p0, p1);
        }
        *reinterpret_cast<uint4*>(ps + sw_off(r, 8 * ch + cc)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      {
        float a0, a1;
        f2unpack(acc2, a0, a1);
        l_half += a0 + a1;
      }
      // keys past the chunk's last position: zero their V rows (the TMA read real cache
      // rows there, which may hold anything; a zero weight times a NaN is NaN)
      if (j0 + kT > t_end) {
        ok = mbar_wait_ab(&bar_v[it % kVStages], (uint32_t)((it / kVStages) & 1), ab);
        if (ok && r >= t_end - j0) {
          unsigned char* vrow = vst + (size_t)((it % kVStages) * kTileBytes);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(vrow + sw_off(r, 8 * ch + c)) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        failed = failed || !__all_sync(0xffffffffu, ok);
      }
      fence_before();
      fence_proxy_async();
      mbar_arrive(&bar_p);
    }
    if (failed) fail();
    // ---- epilogue: O / l once the last P V has run
    bool okf = !failed && !*ab && mbar_wait_ab(&bar_o, (uint32_t)((n_tiles - 1) & 1), ab);
    xl[ch][r] = l_half;
    named_sync(1 + lg, 64);
    __syncwarp();
    if (__all_sync(0xffffffffu, okf)) {
      fence_after();
      const float l = xl[0][r] + xl[1][r];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* dst = P.out + (((size_t)b * P.Hq + h) * P.T + (t - (int)start)) * kHeadDim + 64 * ch;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v32[32];
        tmem_ld32(t_o + 32 * c, v32);
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + i) =
                make_float4(v32[i] * inv, v32[i + 1] * inv, v32[i + 2] * inv, v32[i + 3] * inv);
        }
      }
    } else {
      fail();
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

int prefill_tc_smem_bytes() { return (2 + kKStages + kVStages) * kTileBytes + 1024; }

namespace {
// A 3-D view [slices][Lmax][128] bf16 of a cache, boxes of 128 rows x 64 columns, 128-byte
// swizzle (rows past Lmax read as zeros).
cudaError_t make_cache_map(CUtensorMap* tm, const void* base, int64_t slices, int64_t Lmax) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return e != cudaSuccess ? e : cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)Lmax, (cuuint64_t)slices};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)Lmax * kHeadDim * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kT, 1};
  const cuuint32_t elem[3] = {1, 1, 1};
  const CUresult r = encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, float* out, const int64_t* start, int B,
                              int T, int Hq, int Hkv, int64_t Lmax, int n_sink, int window,
                              const unsigned char* is_ret, const double* inv_freq_pi, unsigned* err, cudaStream_t st) {
  TcParams P;
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
  P.G = Hq / Hkv;
  P.n_sink = n_sink;
  P.window = window;
  P.Lmax = Lmax;
  P.scale_log2 = (float)(1.4426950408889634 / 11.313708498984761);   // log2(e) / sqrt(128)
  for (int g = 0; g < kMaxKvHeads; ++g) P.is_ret[g] = g < Hkv ? is_ret[g] : 0;
  const int QB = kT / P.G;
  P.n_qblocks = (T + QB - 1) / QB;
  CUtensorMap tmk, tmv;
  cudaError_t e = make_cache_map(&tmk, k, (int64_t)B * Hkv, Lmax);
  if (e == cudaSuccess) e = make_cache_map(&tmv, v, (int64_t)B * Hkv, Lmax);
  if (e != cudaSuccess) return e;
  const int smem = prefill_tc_smem_bytes();
  e = cudaFuncSetAttribute(k_prefill_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k_prefill_tc<<<dim3(P.n_qblocks, B * Hkv), kThreads, smem, st>>>(tmk, tmv, P);
  return cudaGetLastError();
}

}  // namespace spa
