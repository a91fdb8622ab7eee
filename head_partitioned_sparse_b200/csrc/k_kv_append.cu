// Compact KV append: new key/value rows scattered into the compact layout.
//
// Retrieval heads keep every position (global context); streaming heads keep only
// what they attend: the sink tokens and a recent window ("Autonomy of Heads" summary,
// Deployment strategy: streaming heads retain a fixed sink cache and a recent window;
// "Full Attention Strikes Back" (RTPurbo summary), Methodology §1: local heads attend a
// sliding window with sinks).  Streaming rows live in a ring of n_sink + window rows:
// position t at row t for t < n_sink, else at row n_sink + (t - n_sink) mod window.
//
// One call appends positions start[b] + i, i < T, of every (b, head).  A streaming head
// writes position t iff t < n_sink or t >= max(n_sink, start[b] + T - window): the
// positions still attended after the call.  Those are at most window consecutive
// positions past the sinks, so no two of them share a ring row and the result does
// not depend on the order of the writes.
//
// Layout: a CTA takes kRows consecutive positions of one (b, head); its threads copy
// 16-byte pieces of the K and V rows (coalesced reads and writes of whole rows).
#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr int kRows = 32;

struct KvAppendArgs {
  unsigned char is_ret[kMaxKvHeads];
  int head_rank[kMaxKvHeads];
  int n_ret, n_str, n_sink, window;
  void* k_ret;
  void* v_ret;
  void* k_ring;
  void* v_ring;
};

template <typename T>
__global__ void __launch_bounds__(256)
k_kv_append_compact(const T* __restrict__ k_new, const T* __restrict__ v_new, const int64_t* __restrict__ start_pos,
                    int T_, int Hkv, int64_t Lmax, const KvAppendArgs a, unsigned* __restrict__ err) {
  constexpr int kCpr = kHeadDim * (int)sizeof(T) / 16;   // 16-byte pieces per row
  const int s = blockIdx.y, b = s / Hkv, g = s % Hkv;
  const int t0 = blockIdx.x * kRows;
  const int nrows = min(kRows, T_ - t0);
  const int64_t start = start_pos[b];
  const bool ret = a.is_ret[g] != 0;
  const int rk = a.head_rank[g];
  const int64_t keep_lo = a.window > 0 ? max((int64_t)a.n_sink, start + T_ - a.window) : INT64_MAX;
  const uint4* ksrc = reinterpret_cast<const uint4*>(k_new + ((size_t)s * T_ + t0) * kHeadDim);
  const uint4* vsrc = reinterpret_cast<const uint4*>(v_new + ((size_t)s * T_ + t0) * kHeadDim);
  uint4* kdst;
  uint4* vdst;
  if (ret) {
    const size_t off = ((size_t)b * a.n_ret + rk) * (size_t)Lmax * kHeadDim;
    kdst = reinterpret_cast<uint4*>((T*)a.k_ret + off);
    vdst = reinterpret_cast<uint4*>((T*)a.v_ret + off);
  } else {
    const size_t off = ((size_t)b * a.n_str + rk) * (size_t)(a.n_sink + a.window) * kHeadDim;
    kdst = reinterpret_cast<uint4*>((T*)a.k_ring + off);
    vdst = reinterpret_cast<uint4*>((T*)a.v_ring + off);
  }
  for (int i = threadIdx.x; i < nrows * 2 * kCpr; i += blockDim.x) {
    const int r = i / (2 * kCpr), rem = i % (2 * kCpr), tv = rem / kCpr, c = rem % kCpr;
    const int64_t pos = start + t0 + r;
    if (pos < 0 || pos >= Lmax) {
      if (rem == 0) atomicOr(err, kErrStartPos);
      continue;
    }
    int64_t row = pos;
    if (!ret) {
      if (pos >= a.n_sink && pos < keep_lo) continue;   // not attended after this call
      row = ring_row((int)pos, a.n_sink, a.window);
    }
    const uint4 v = (tv ? vsrc : ksrc)[(size_t)r * kCpr + c];
    (tv ? vdst : kdst)[(size_t)row * kCpr + c] = v;
  }
}

}  // namespace

cudaError_t launch_kv_append_compact(const void* k_new, const void* v_new, const int64_t* start_pos, int B, int T,
                                     int Hkv, int64_t Lmax, int kv_dtype, const unsigned char* is_ret,
                                     const int* head_rank, int n_ret, int n_str, int n_sink, int window, void* k_ret,
                                     void* v_ret, void* k_ring, void* v_ring, unsigned* dev_err, cudaStream_t st) {
  KvAppendArgs a;
  for (int g = 0; g < kMaxKvHeads; ++g) {
    a.is_ret[g] = g < Hkv ? is_ret[g] : 0;
    a.head_rank[g] = g < Hkv ? head_rank[g] : 0;
  }
  a.n_ret = n_ret;
  a.n_str = n_str;
  a.n_sink = n_sink;
  a.window = window;
  a.k_ret = k_ret;
  a.v_ret = v_ret;
  a.k_ring = k_ring;
  a.v_ring = v_ring;
  dim3 grid((T + kRows - 1) / kRows, B * Hkv);
  if (kv_dtype == 0)
    k_kv_append_compact<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)k_new,
                                                              (const __nv_bfloat16*)v_new, start_pos, T, Hkv, Lmax,
                                                              a, dev_err);
  else
    k_kv_append_compact<float><<<grid, 256, 0, st>>>((const float*)k_new, (const float*)v_new, start_pos, T, Hkv,
                                                      Lmax, a, dev_err);
  return cudaGetLastError();
}

}  // namespace spa
