// Data-free head labels: the effective rank of each head's query-key operator.
//
// "Autonomy of Heads" summary, Methodology:
//   §1 M_h = W_K^{hT} W_Q^h, the frozen query-key matching directions of head h;
//   §2 effective rank exp(-sum_k s_k ln s_k), s_k = sigma_k / sum_j sigma_j;
//   §3 the nonzero sigma_k^2 are the eigenvalues of the d_head x d_head proxy
//      C_h = (W_Q W_Q^T)(W_K W_K^T) (Sylvester's determinant theorem);
//   §4 the k KV groups of lowest mean effective rank are the retrieval heads.
//
// Steps, all in float64 on the device (run once per model, off the decode path):
//   1. Gram matrices A_h = W_Q^h W_Q^hT (every query head) and B_g = W_K^g W_K^gT
//      (every key head): products of float32 inputs are exact in float64;
//   2. B_g = L_g L_g^T (Cholesky; a pivot at or below 128 eps max_i B_ii leaves its
//      column at zero, which keeps a rank-deficient B_g semi-definite);
//   3. S_h = L_g^T A_h L_g: symmetric positive semi-definite with the eigenvalues of
//      C_h (eig(A B) = eig(A L L^T) = eig(L^T A L));
//   4. cyclic Jacobi on S_h (two-sided, round-robin order: 64 disjoint rotations per
//      step, each chosen to zero its off-diagonal pair as in the symmetric 2x2 Schur
//      step of Golub and Van Loan) until the off-diagonal part is negligible; then
//      sigma = sqrt(max(diag, 0)) and the effective rank;
//   5. per KV head the mean over its G query heads, and the k lowest (ties: lower
//      index) are marked retrieval.
// Squaring the operator (steps 1-3) returns a zero singular value as about
// sqrt(eps) sigma_max; full-rank heads keep near float64 accuracy.
#include <cfloat>

#include "../../include/spa.h"
#include "spa_internal.cuh"

namespace spa {
namespace {

constexpr int kD = kHeadDim;       // d_head = 128
constexpr int kDD = kD * kD;
constexpr int kLd = kD + 1;        // padded row stride (doubles) of a matrix in shared memory
constexpr int kGramBand = 16;      // rows of a Gram matrix per CTA
constexpr int kGramK = 64;         // d_model columns staged per step
constexpr int kMaxSweeps = 40;

// ---- 1. Gram matrices: out[z] = W_z W_z^T, W_z = w + z * 128 * d_model (row-major)
__global__ void __launch_bounds__(256) k_gram(const float* __restrict__ w, int d_model, double* __restrict__ out) {
  __shared__ float ws[kD][kGramK + 1];
  const int z = blockIdx.y, band = blockIdx.x, tid = threadIdx.x;
  const float* W = w + (size_t)z * kD * d_model;
  const int i = band * kGramBand + (tid >> 4);   // output row
  const int j0 = tid & 15;                       // output columns j0 + 16 m
  double acc[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) acc[m] = 0.0;
  for (int k0 = 0; k0 < d_model; k0 += kGramK) {
    const int nk = min(kGramK, d_model - k0);
    __syncthreads();
    for (int e = tid; e < kD * kGramK; e += blockDim.x) {
      const int r = e / kGramK, c = e % kGramK;
      ws[r][c] = c < nk ? W[(size_t)r * d_model + k0 + c] : 0.f;
    }
    __syncthreads();
    for (int k = 0; k < nk; ++k) {
      const double wi = ws[i][k];
#pragma unroll
      for (int m = 0; m < 8; ++m) acc[m] = fma(wi, (double)ws[j0 + 16 * m][k], acc[m]);
    }
  }
  double* O = out + (size_t)z * kDD;
#pragma unroll
  for (int m = 0; m < 8; ++m) O[(size_t)i * kD + j0 + 16 * m] = acc[m];
}

// ---- 2. Cholesky B = L L^T in place (lower triangle; the upper part is zeroed)
__global__ void __launch_bounds__(256) k_cholesky(double* __restrict__ mats) {
  extern __shared__ double a[];   // [kD][kLd]
  __shared__ double piv;
  double* M = mats + (size_t)blockIdx.x * kDD;
  const int tid = threadIdx.x;
  for (int e = tid; e < kDD; e += blockDim.x) a[(e / kD) * kLd + e % kD] = M[e];
  __syncthreads();
  if (tid == 0) {
    double mx = 0.0;
    for (int i = 0; i < kD; ++i) mx = fmax(mx, a[i * kLd + i]);
    piv = 128.0 * DBL_EPSILON * mx;   // pivots at or below this count as zero
  }
  __syncthreads();
  const double tol = piv;
  for (int k = 0; k < kD; ++k) {
    if (tid == 0) {
      const double d = a[k * kLd + k];
      a[k * kLd + k] = d > tol ? sqrt(d) : 0.0;
    }
    __syncthreads();
    const double r = a[k * kLd + k];
    for (int i = k + 1 + tid; i < kD; i += blockDim.x) a[i * kLd + k] = r > 0.0 ? a[i * kLd + k] / r : 0.0;
    __syncthreads();
    // trailing update of the lower triangle: a_ij -= l_ik l_jk, k < j <= i
    const int n = kD - k - 1;
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int i = k + 1 + e / n, j = k + 1 + e % n;
      if (j <= i) a[i * kLd + j] -= a[i * kLd + k] * a[j * kLd + k];
    }
    __syncthreads();
  }
  for (int e = tid; e < kDD; e += blockDim.x) {
    const int i = e / kD, j = e % kD;
    M[e] = j <= i ? a[i * kLd + j] : 0.0;
  }
}

// ---- 3. batched 128 x 128 float64 products: C_z = op(X_z) Y_z, op = transpose or not.
// X_z = x + (z / x_div) * kDD, Y_z = y + (z / y_div) * kDD (query head z, key head z / G).
// A CTA computes a 32 x 32 tile.
__global__ void __launch_bounds__(256) k_gemm128(const double* __restrict__ x, int x_div, int trans_x,
                                                 const double* __restrict__ y, int y_div, double* __restrict__ c) {
  __shared__ double xs[32][33], ys[32][33];
  const int z = blockIdx.z, ti = blockIdx.y * 32, tj = blockIdx.x * 32, tid = threadIdx.x;
  const double* X = x + (size_t)(z / x_div) * kDD;
  const double* Y = y + (size_t)(z / y_div) * kDD;
  const int r = tid >> 3, c4 = (tid & 7) * 4;   // row r, columns c4 .. c4 + 3 of the tile
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int k0 = 0; k0 < kD; k0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * 32; e += blockDim.x) {
      const int a = e / 32, b = e % 32;
      // xs[a][b] = op(X)[ti + a][k0 + b]
      xs[a][b] = trans_x ? X[(size_t)(k0 + b) * kD + ti + a] : X[(size_t)(ti + a) * kD + k0 + b];
      ys[a][b] = Y[(size_t)(k0 + a) * kD + tj + b];
    }
    __syncthreads();
    for (int k = 0; k < 32; ++k) {
      const double xv = xs[r][k];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = fma(xv, ys[k][c4 + m], acc[m]);
    }
  }
  double* C = c + (size_t)z * kDD;
#pragma unroll
  for (int m = 0; m < 4; ++m) C[(size_t)(ti + r) * kD + tj + c4 + m] = acc[m];
}

// ---- 4. Jacobi eigenvalues of symmetric S_z, singular values and effective rank
__device__ __forceinline__ void round_robin_pair(int round, int k, int& p, int& q) {
  // circle method over kD players: player kD-1 is fixed, the others rotate
  if (k == 0) {
    p = kD - 1;
    q = round;
  } else {
    p = (round + k) % (kD - 1);
    q = (round - k + kD - 1) % (kD - 1);
  }
  if (p > q) { const int t = p; p = q; q = t; }
}

__device__ double block_sum_f64(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];   // fixed order
  return t;
}

__global__ void __launch_bounds__(256) k_jacobi_er(const double* __restrict__ S, double* __restrict__ er,
                                                   double* __restrict__ sigma_out, int* __restrict__ sweeps_out) {
  extern __shared__ double a[];   // [kD][kLd]
  __shared__ double cs[kD / 2], sn[kD / 2];
  __shared__ double red[32];
  __shared__ double sig[kD];
  const int tid = threadIdx.x;
  const double* M = S + (size_t)blockIdx.x * kDD;
  for (int e = tid; e < kDD; e += blockDim.x) {
    const int i = e / kD, j = e % kD;
    a[i * kLd + j] = 0.5 * (M[(size_t)i * kD + j] + M[(size_t)j * kD + i]);   // exact symmetry
  }
  __syncthreads();
  int sweep = 0;
  for (; sweep < kMaxSweeps; ++sweep) {
    double off = 0.0, dg = 0.0;
    for (int e = tid; e < kDD; e += blockDim.x) {
      const int i = e / kD, j = e % kD;
      const double v = a[i * kLd + j];
      if (i != j) off += v * v; else dg += v * v;
    }
    off = block_sum_f64(off, red);
    dg = block_sum_f64(dg, red);
    if (!(off > 1e-28 * dg)) break;   // off-diagonal part below 1e-14 of the diagonal (or a NaN: stop)
    for (int round = 0; round < kD - 1; ++round) {
      if (tid < kD / 2) {
        int p, q;
        round_robin_pair(round, tid, p, q);
        const double apq = a[p * kLd + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (a[q * kLd + q] - a[p * kLd + p]) / (2.0 * apq);
          const double t = tau >= 0.0 ? 1.0 / (tau + sqrt(1.0 + tau * tau)) : -1.0 / (-tau + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        cs[tid] = c;
        sn[tid] = s;
      }
      __syncthreads();
      // rows: row_p <- c row_p - s row_q, row_q <- s row_p + c row_q
      for (int e = tid; e < (kD / 2) * kD; e += blockDim.x) {
        const int k = e / kD, j = e % kD;
        int p, q;
        round_robin_pair(round, k, p, q);
        const double c = cs[k], s = sn[k];
        const double xp = a[p * kLd + j], xq = a[q * kLd + j];
        a[p * kLd + j] = c * xp - s * xq;
        a[q * kLd + j] = s * xp + c * xq;
      }
      __syncthreads();
      // columns: col_p <- c col_p - s col_q, col_q <- s col_p + c col_q
      for (int e = tid; e < (kD / 2) * kD; e += blockDim.x) {
        const int k = e / kD, i = e % kD;
        int p, q;
        round_robin_pair(round, k, p, q);
        const double c = cs[k], s = sn[k];
        const double xp = a[i * kLd + p], xq = a[i * kLd + q];
        a[i * kLd + p] = c * xp - s * xq;
        a[i * kLd + q] = s * xp + c * xq;
      }
      __syncthreads();
    }
  }
  // singular values (clamped rounding residue), effective rank
  double sv = 0.0;
  if (tid < kD) {
    sv = sqrt(fmax(a[tid * kLd + tid], 0.0));
    sig[tid] = sv;
  }
  const double total = block_sum_f64(tid < kD ? sv : 0.0, red);
  double h = 0.0;
  if (tid < kD && sv > 0.0 && total > 0.0) {
    const double p = sv / total;
    h = -p * log(p);
  }
  const double H = block_sum_f64(h, red);
  if (tid == 0) {
    er[blockIdx.x] = total > 0.0 ? exp(H) : 0.0;
    if (sweeps_out) sweeps_out[blockIdx.x] = sweep;
  }
  if (sigma_out && tid < kD) {   // descending order (equal values by index)
    int rank = 0;
    for (int j = 0; j < kD; ++j) rank += (sig[j] > sv || (sig[j] == sv && j < tid)) ? 1 : 0;
    sigma_out[(size_t)blockIdx.x * kD + rank] = sv;
  }
}

// ---- 5. group means and labels
__global__ void k_labels(const double* __restrict__ er_q, int Hq, int Hkv, int n_ret, double* __restrict__ er_kv,
                         unsigned char* __restrict__ mask) {
  __shared__ double m[kMaxKvHeads];
  const int g = threadIdx.x, G = Hq / Hkv;
  if (g < Hkv) {
    double s = 0.0;
    for (int i = 0; i < G; ++i) s += er_q[g * G + i];   // fixed order
    m[g] = s / G;
    er_kv[g] = m[g];
  }
  __syncthreads();
  if (g < Hkv) {
    int rank = 0;
    for (int j = 0; j < Hkv; ++j) rank += (m[j] < m[g] || (m[j] == m[g] && j < g)) ? 1 : 0;
    mask[g] = rank < n_ret ? 1 : 0;
  }
}

}  // namespace

// Workspace layout (doubles): A [Hq][kDD] | B, then L [Hkv][kDD] | T [Hq][kDD] | S [Hq][kDD].
size_t head_rank_workspace_bytes(int Hq, int Hkv) { return (size_t)(3 * Hq + Hkv) * kDD * sizeof(double); }

cudaError_t launch_head_ranks(const float* W_Q, const float* W_K, int Hq, int Hkv, int d_model, int n_ret,
                              void* ws, double* er_q, double* er_kv, unsigned char* mask, double* sigma,
                              int* sweeps, cudaStream_t st) {
  const int smem = kD * kLd * (int)sizeof(double);   // one padded 128 x 128 float64 matrix
  cudaError_t e = cudaFuncSetAttribute(k_cholesky, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_jacobi_er, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  double* A = (double*)ws;
  double* L = A + (size_t)Hq * kDD;
  double* T = L + (size_t)Hkv * kDD;
  double* S = T + (size_t)Hq * kDD;
  const int G = Hq / Hkv;
  k_gram<<<dim3(kD / kGramBand, Hq), 256, 0, st>>>(W_Q, d_model, A);
  k_gram<<<dim3(kD / kGramBand, Hkv), 256, 0, st>>>(W_K, d_model, L);
  k_cholesky<<<Hkv, 256, smem, st>>>(L);
  // T_h = A_h L_g(h);  S_h = L_g(h)^T T_h
  k_gemm128<<<dim3(kD / 32, kD / 32, Hq), 256, 0, st>>>(A, 1, 0, L, G, T);
  k_gemm128<<<dim3(kD / 32, kD / 32, Hq), 256, 0, st>>>(L, G, 1, T, 1, S);
  k_jacobi_er<<<Hq, 256, smem, st>>>(S, er_q, sigma, sweeps);
  k_labels<<<1, kMaxKvHeads, 0, st>>>(er_q, Hq, Hkv, n_ret, er_kv, mask);
  return cudaGetLastError();
}

}  // namespace spa
