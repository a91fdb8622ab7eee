// spa_select_noalloc: the top-p selection of spa_select for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code embedded in a host framework
// that has already reserved the GPU's memory for its own pool and forbids other
// allocations, code that must not trigger the implicit device synchronisation an
// allocation may cause in the middle of a latency-critical decode loop, or code
// that cannot own a library handle's lifetime.  This entry point needs no handle
// and allocates nothing: every scratch buffer of the selection kernels lives in one
// file-scope static device array of fixed size, which every GPU that loads the
// library holds until the process exits.  The caller passes inputs and outputs.
//
// The array's name is only a host-side stand-in in host code, so its device address
// is looked up once per device with cudaGetSymbolAddress, with that device current,
// on the first call made on that device (do that first call before any stream
// capture).  Every call shares the array and it keeps the last call's contents.  The
// words that must start at zero on every call (the device status word and the
// per-slice state with the selection kernel's arrival counters) sit at fixed offsets
// at the head of the array and are cleared with one cudaMemsetAsync on the call's
// stream before the launch, so a call never inherits a half-counted arrival, whatever
// the shapes of earlier calls or whether one of their bounded waits gave up; the
// kernels clear the rest (histograms, counters) themselves.  Calls that overlap on the GPU (other streams, other host
// threads) race on the array: serialise them.
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/spa.h"
#include "spa_internal.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(12) << 20;   // 12 MiB per device
constexpr int64_t kMaxTokens = int64_t(1) << 19;     // B * n_kv_heads * max_ctx
constexpr int kMaxSlices = 64;                        // B * n_kv_heads
constexpr int kMaxQueryRows = 512;                    // B * n_q_heads
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

spa_status err(spa_status code, const char* msg) { return spa::set_last_error(code, msg); }

// Device address of g_scratch on the current device (looked up on first use).
spa_status scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return err(SPA_ERR_CUDA, "spa_select_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return err(SPA_ERR_UNSUPPORTED, "spa_select_noalloc: device ordinal >= 64");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) return err(SPA_ERR_CUDA, "spa_select_noalloc: cudaGetSymbolAddress of the scratch failed");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SPA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" SPA_API spa_status spa_select_noalloc(const float* P_q, int n_q_heads, int n_kv_heads, int kv_dtype,
                                                 float idx_scale, int64_t max_ctx, const void* q_pre,
                                                 const void* idx_cache, const uint8_t* head_mask,
                                                 const int64_t* seq_lens, int B, int64_t max_seq_len, float p,
                                                 int n_sink, int window, int32_t* sel_idx, int32_t* sel_count,
                                                 spa_stream stream) {
  if (!P_q || !q_pre || !idx_cache || !head_mask || !seq_lens || !sel_idx || !sel_count)
    return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: a required pointer is NULL");
  if (!aligned16(P_q) || !aligned16(q_pre) || !aligned16(idx_cache) || !aligned16(sel_idx) ||
      ((uintptr_t)seq_lens & 7u) || ((uintptr_t)sel_count & 3u))
    return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: misaligned pointer");
  if (kv_dtype != SPA_BF16 && kv_dtype != SPA_F32) return err(SPA_ERR_UNSUPPORTED, "spa_select_noalloc: bad kv_dtype");
  if (n_kv_heads < 1 || n_kv_heads > spa::kMaxKvHeads || n_q_heads < 1 || n_q_heads % n_kv_heads)
    return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: bad head counts");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return err(SPA_ERR_UNSUPPORTED, "spa_select_noalloc: G must be 1, 2, 4 or 8");
  if (B < 1 || max_ctx < 1 || max_seq_len < 0 || max_seq_len > max_ctx)
    return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: bad B, max_ctx or max_seq_len");
  if (!(p > 0.f) || !(p <= 1.f)) return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: p must be in (0, 1]");
  if (n_sink < 0 || window < 0 || (int64_t)n_sink + window < 1)
    return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: need n_sink, window >= 0 and n_sink + window >= 1");
  if (!std::isfinite(idx_scale)) return err(SPA_ERR_INVALID_ARG, "spa_select_noalloc: idx_scale must be finite");
  const int64_t slices = (int64_t)B * n_kv_heads;
  if (slices > kMaxSlices || (int64_t)B * n_q_heads > kMaxQueryRows || slices * max_ctx > kMaxTokens)
    return err(SPA_ERR_WORKSPACE,
               "spa_select_noalloc: request exceeds the static scratch (limits: B*n_kv_heads <= 64, "
               "B*n_q_heads <= 512, B*n_kv_heads*max_ctx <= 2^19 tokens); use spa_create + spa_select");

  spa::StepParams P;
  std::memset(&P, 0, sizeof P);
  for (int g = 0; g < n_kv_heads; ++g) {
    P.is_ret[g] = head_mask[g] ? 1 : 0;
    if (P.is_ret[g]) P.ret_heads[P.n_ret++] = g;
  }
  P.q_pre = q_pre;
  P.idx_cache = static_cast<const uint16_t*>(idx_cache);
  P.seq_lens = seq_lens;
  P.sel_list = sel_idx;
  P.sel_count = sel_count;
  P.B = B;
  P.Hq = n_q_heads;
  P.Hkv = n_kv_heads;
  P.G = G;
  P.Lmax = max_ctx;
  P.Lcap = (int)(max_seq_len ? max_seq_len : max_ctx);
  P.n_chunks = (P.Lcap + spa::kChunk - 1) / spa::kChunk;
  P.n_slices = (int)slices;
  P.p = p;
  P.keep_all = p >= 1.f ? 1 : 0;
  P.n_sink = n_sink;
  P.window = window;
  P.idx_scale_log2 = (idx_scale > 0.f ? idx_scale : 0.25f) * 1.4426950408889634f;
  P.attn_scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  P.split_rows = spa::kDefaultSplitRows;

  int dev = 0, sms = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return err(SPA_ERR_CUDA, cudaGetErrorString(ce));
  ce = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (ce != cudaSuccess) return err(SPA_ERR_CUDA, cudaGetErrorString(ce));
  const int per_sm = spa::select_resident_per_sm(kv_dtype, G);
  if (per_sm < 1 || sms < 1) return err(SPA_ERR_UNSUPPORTED, "spa_select_noalloc: selection kernel cannot be resident");
  const int max_grid = per_sm * sms < spa::kMaxSelectGrid ? per_sm * sms : spa::kMaxSelectGrid;

  void* base_v = nullptr;
  spa_status r = scratch_on_current_device(&base_v);
  if (r) return r;
  char* base = static_cast<char*>(base_v);
  // Fixed head block, cleared before every launch: the status word and the per-slice
  // state (arrival counters included) of up to kMaxSlices slices.
  const size_t off_err = 0, off_st = 256;
  const size_t head_bytes = up256(off_st + (size_t)kMaxSlices * sizeof(spa::SliceState));
  const size_t sz[] = {
      64 * 8,                                                  // inv_freq (unused by selection; zero)
      (size_t)B * n_q_heads * spa::kHeadDim * 4,               // q_rot
      (size_t)B * n_q_heads * spa::kIdxDim * 4,                // q_idx
      (size_t)(max_grid + slices) * G * 8,                     // per-range statistics
      (size_t)slices * spa::pi_row_stride(max_ctx) * 4,        // pi
      (size_t)slices * spa::kBins1 * 8,                        // hist1
      (size_t)slices * max_ctx * 8,                            // candidates
      (size_t)slices * spa::kBins2 * 8,                        // hist2
      (size_t)(spa::kMaxSelectGrid + slices) * 4,              // per-range counts above the cut bin
  };
  size_t off[sizeof sz / sizeof sz[0]];
  size_t o = head_bytes;
  for (size_t i = 0; i < sizeof sz / sizeof sz[0]; ++i) {
    off[i] = o;
    o += up256(sz[i]);
  }
  if (o > kScratchBytes) return err(SPA_ERR_WORKSPACE, "spa_select_noalloc: request exceeds the 12 MiB static scratch");
  spa::Workspace& w = P.ws;
  w.P_q = const_cast<float*>(P_q);
  w.inv_freq = (double*)(base + off[0]);
  w.q_rot = (float*)(base + off[1]);
  w.q_idx = (float*)(base + off[2]);
  w.stats = (float2*)(base + off[3]);
  w.pi = (float*)(base + off[4]);
  w.pi_stride = spa::pi_row_stride(max_ctx);
  w.hist1 = (unsigned long long*)(base + off[5]);
  w.cand = (uint2*)(base + off[6]);
  w.hist2 = (unsigned long long*)(base + off[7]);
  w.seg_cnt = (int*)(base + off[8]);
  w.dev_err = (unsigned*)(base + off_err);
  w.st = (spa::SliceState*)(base + off_st);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(base, 0, head_bytes, st);   // stream-ordered; allocates nothing
  if (e != cudaSuccess) return err(SPA_ERR_CUDA, cudaGetErrorString(e));
  e = spa::launch_select(P, kv_dtype, max_grid, st);
  if (e != cudaSuccess) return err(SPA_ERR_CUDA, cudaGetErrorString(e));
  return SPA_OK;
}
