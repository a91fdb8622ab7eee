// Index append: bf16 16-dim index rows from pre-RoPE keys.
//
// "Full Attention Strikes Back" (RTPurbo summary), Methodology §2: a 16-dim
// projector is applied to the key features before RoPE is injected; relevance is
// then estimated in that compact subspace.  Each row is
//   idx[r] = bf16_rne( sum_d P_k[g][r][d] * k_pre[d] ),  r < 16,
// with each product rounded to float32 and added to a float32 running sum in
// ascending d.
//
// Layout: a CTA takes 64 consecutive tokens of one (b, kv head) of the head map (all
// heads in place, or the retrieval heads only at their rank for the compact layout);
// the key tile
// (as float32, rows padded to 129 floats so a warp's 8 rows hit 8 banks) and the
// head's projector sit in shared memory; each thread produces 4 of a row's 16
// outputs and writes them as one 8-byte store (a row is 32 contiguous bytes).
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
  // float32 product, then float32 add, in ascending d (no fused multiply-add): the
  // bf16 code is decided by exactly this sequence of roundings.
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
  if (kv_dtype == 0)
    k_index_append<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)k_pre, start_pos, T, Hkv, Lmax,
                                                          P_k, idx_cache, dev_err, m);
  else
    k_index_append<float><<<grid, 256, 0, st>>>((const float*)k_pre, start_pos, T, Hkv, Lmax, P_k,
                                                 idx_cache, dev_err, m);
  return cudaGetLastError();
}

}  // namespace spa
