// lowrank_svd.cuh — load-time rank-r truncated SVD of W^T on the GPU, all in
// float64, giving the factors of the 16-bit low-rank branch.
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
// "Background: SVDQuant and Nunchaku": the hardest part of each weight matrix
// is kept in a small 16-bit low-rank branch obtained from its singular value
// decomposition. With A = W^T (K x N) = U S V^T the branch is
// L1 = bf16(U_r S_r) (K x r) and L2 = bf16(V_r^T) (r x N).
//
// Method: randomized subspace iteration (range finder with power iterations,
// Halko, Martinsson and Tropp, "Finding structure with randomness", SIAM
// Review 2011, algorithms 4.3/4.4 and 5.1):
//   Y = A Omega (Omega: N x p Gaussian, p = r + oversampling)
//   q times: Y = orth(Y); Z = orth(A^T Y); Y = A Z
//   Q = orth(Y); Z = A^T Q (= B^T with B = Q^T A)
//   B B^T = Z^T Z = U_B diag(lambda) U_B^T (two-sided Jacobi)
//   sigma = sqrt(lambda); U_r = Q U_B,r; V_r^T = diag(1/sigma_r) U_B,r^T B
// orth() is CholeskyQR2 with a diagonal shift in the first pass (Fukaya,
// Kannan, Nakatsukasa, Yamamoto, Yanagisawa, "Shifted Cholesky QR for
// computing the QR factorization of ill-conditioned matrices", SIAM J. Sci.
// Comput. 2020), so rank-deficient inputs do not break down.
//
// Kernels: a Gaussian fill from a counter-based generator (splitmix64, Steele,
// Lea and Flood 2014, and the Box-Muller transform); a tall-skinny GEMM family
// whose partial sums over the long dimension are added in a fixed order
// (deterministic); and one-CTA kernels for the p x p Cholesky factor, its
// inverse and the Jacobi eigensolver (p <= 160).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace svdq {

constexpr int kSvdMaxP = 160;     // r + 32 oversampling columns (r <= 128), multiple of 16
constexpr int kTsRows = 32;       // output rows per CTA of the tall-skinny GEMM
constexpr int kTsL = 32;          // long-dimension slice staged in shared memory
constexpr int kTsThreads = 256;

// ------------------------------------------------------------------ Gaussian fill
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// out[i] ~ N(0, 1), i < n: pair j = i / 2 uses the 53-bit uniforms of counters
// 2j and 2j + 1 (in (0, 1]) and the Box-Muller transform.
__global__ void gauss_fill_kernel(double* __restrict__ out, int64_t n, uint64_t seed) {
  const int64_t pairs = (n + 1) / 2;
  for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < pairs;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t a = splitmix64(seed ^ splitmix64(2 * static_cast<uint64_t>(j)));
    const uint64_t b = splitmix64(seed ^ splitmix64(2 * static_cast<uint64_t>(j) + 1));
    const double u1 = static_cast<double>((a >> 11) + 1) * 0x1.0p-53;
    const double u2 = static_cast<double>(b >> 11) * 0x1.0p-53;
    const double rad = sqrt(-2.0 * log(u1));
    double sn, cs;
    sincospi(2.0 * u2, &sn, &cs);
    out[2 * j] = rad * cs;
    if (2 * j + 1 < n) out[2 * j + 1] = rad * sn;
  }
}

// ------------------------------------------------------------------ tall-skinny GEMM
__device__ __forceinline__ double to_f64(double x) { return x; }
__device__ __forceinline__ double to_f64(__nv_bfloat16 x) { return static_cast<double>(__bfloat162float(x)); }

// Partial products over one slice of the long dimension L:
//   TRANS_A = false: C[m][j] = sum_l A[m][l] B[l][j]   (A: M x L, row-major, lda)
//   TRANS_A = true:  C[m][j] = sum_l A[l][m] B[l][j]   (A: L x M, row-major, lda)
// B: L x P float64 (ldb = P). colscale (or nullptr) multiplies each element
// of the row-major A by the factor of its column: A[.][c] * colscale[c] (the
// smoothing of W's input channels). Grid (ceil(M / 32), splits); split s covers
// l in [s*lchunk, min(L, (s+1)*lchunk)) in ascending order and writes
// part[s][m][j]. P <= kSvdMaxP and a multiple of 16; dynamic shared memory
// holds the B slice (kTsL x P doubles).
template <bool TRANS_A, typename TA>
__global__ void __launch_bounds__(kTsThreads) ts_gemm_kernel(int M, int L, int P, const TA* __restrict__ A,
                                                            int64_t lda, const float* __restrict__ colscale,
                                                            const double* __restrict__ B,
                                                            double* __restrict__ part, int lchunk) {
  __shared__ double a_s[kTsL][kTsRows + 1];
  extern __shared__ double ts_dyn[];
  double* b_s = ts_dyn;  // [kTsL][P]
  const int m0 = blockIdx.x * kTsRows;
  const int s = blockIdx.y;
  const int l_begin = s * lchunk;
  const int l_end = min(L, l_begin + lchunk);
  // thread -> 2 rows x (P/16) columns: rows rr, rr + 16; columns cq + 16 c
  const int rr = threadIdx.x & 15;
  const int cq = threadIdx.x >> 4;  // 0..15
  const int ncol = P / 16;
  double acc0[kSvdMaxP / 16], acc1[kSvdMaxP / 16];
#pragma unroll
  for (int c = 0; c < kSvdMaxP / 16; ++c) acc0[c] = acc1[c] = 0.0;
  for (int l0 = l_begin; l0 < l_end; l0 += kTsL) {
    const int lt = min(kTsL, l_end - l0);
    for (int i = threadIdx.x; i < kTsL * kTsRows; i += kTsThreads) {
      const int li = TRANS_A ? i / kTsRows : i % kTsL;
      const int mi = TRANS_A ? i % kTsRows : i / kTsL;
      double v = 0.0;
      if (li < lt && m0 + mi < M) {
        v = TRANS_A ? to_f64(A[static_cast<int64_t>(l0 + li) * lda + m0 + mi])
                    : to_f64(A[static_cast<int64_t>(m0 + mi) * lda + l0 + li]);
        if (colscale != nullptr) v *= static_cast<double>(colscale[TRANS_A ? m0 + mi : l0 + li]);
      }
      a_s[li][mi] = v;
    }
    for (int i = threadIdx.x; i < kTsL * P; i += kTsThreads) {
      const int li = i / P, j = i % P;
      b_s[li * P + j] = li < lt ? B[static_cast<int64_t>(l0 + li) * P + j] : 0.0;
    }
    __syncthreads();
    for (int li = 0; li < lt; ++li) {
      const double a0 = a_s[li][rr], a1 = a_s[li][rr + 16];
#pragma unroll
      for (int c = 0; c < kSvdMaxP / 16; ++c) {
        if (c < ncol) {
          const double bv = b_s[li * P + cq + 16 * c];
          acc0[c] = fma(a0, bv, acc0[c]);
          acc1[c] = fma(a1, bv, acc1[c]);
        }
      }
    }
    __syncthreads();
  }
  double* out = part + static_cast<int64_t>(s) * M * P;
#pragma unroll
  for (int c = 0; c < kSvdMaxP / 16; ++c) {
    if (c < ncol) {
      const int j = cq + 16 * c;
      if (m0 + rr < M) out[static_cast<int64_t>(m0 + rr) * P + j] = acc0[c];
      if (m0 + rr + 16 < M) out[static_cast<int64_t>(m0 + rr + 16) * P + j] = acc1[c];
    }
  }
}

// C[i] = sum_s part[s][i] in ascending s (n elements per split).
__global__ void split_sum_kernel(const double* __restrict__ part, int splits, int64_t n, double* __restrict__ C) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double acc = part[i];
    for (int s = 1; s < splits; ++s) acc += part[static_cast<int64_t>(s) * n + i];
    C[i] = acc;
  }
}

// ------------------------------------------------------------------ p x p kernels (one CTA)
// R (upper, p x p) with R^T R = G + shift I, then Rinv = R^-1 (upper). G, R,
// Rinv row-major p x p in global memory. shift = rel * max_i G_ii, at least
// the smallest normal double. A pivot not above shift / 1000 (a breakdown)
// is replaced by sqrt(shift).
__global__ void __launch_bounds__(1024) chol_inv_kernel(const double* __restrict__ G, int p, double rel,
                                                        double* __restrict__ R, double* __restrict__ Rinv) {
  __shared__ double shift;
  if (threadIdx.x == 0) {
    double mx = 0.0;
    for (int i = 0; i < p; ++i) mx = fmax(mx, G[i * p + i]);
    shift = fmax(rel * mx, 2.2250738585072014e-308);
  }
  for (int i = threadIdx.x; i < p * p; i += blockDim.x) {
    const int r = i / p, c = i % p;
    R[i] = (r <= c) ? G[i] : 0.0;
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int i = 0; i < p; ++i) R[i * p + i] += shift;
  __syncthreads();
  // right-looking Cholesky on the upper triangle: row k of R
  for (int k = 0; k < p; ++k) {
    __shared__ double d;
    if (threadIdx.x == 0) {
      const double v = R[k * p + k];
      d = v > shift * 1e-3 ? sqrt(v) : sqrt(shift);
      R[k * p + k] = d;
    }
    __syncthreads();
    for (int j = k + 1 + threadIdx.x; j < p; j += blockDim.x) R[k * p + j] /= d;
    __syncthreads();
    const int rem = p - k - 1;
    for (int t = threadIdx.x; t < rem * rem; t += blockDim.x) {
      const int i = k + 1 + t / rem, j = k + 1 + t % rem;
      if (j >= i) R[i * p + j] -= R[k * p + i] * R[k * p + j];
    }
    __syncthreads();
  }
  // Rinv column j (thread j): back substitution of R x = e_j
  for (int j = threadIdx.x; j < p; j += blockDim.x) {
    for (int i = p - 1; i >= 0; --i) {
      double v = (i == j) ? 1.0 : 0.0;
      if (i <= j) {
        for (int k = i + 1; k <= j; ++k) v -= R[i * p + k] * Rinv[k * p + j];
        v /= R[i * p + i];
      } else {
        v = 0.0;
      }
      Rinv[i * p + j] = v;
    }
  }
}

// Eigen-decomposition of the symmetric p x p matrix C (overwritten; row-major)
// by the two-sided cyclic Jacobi method with the parallel round-robin ordering
// of Brent and Luk (p even, p/2 disjoint rotations per round). V (p x p)
// receives the eigenvectors as columns, lam[i] = C[i][i] at the end. Sweeps
// stop when the off-diagonal Frobenius norm is below 1e-15 of the total, or
// after max_sweeps.
__global__ void __launch_bounds__(1024) jacobi_eig_kernel(double* __restrict__ C, int p, double* __restrict__ V,
                                                          double* __restrict__ lam, int max_sweeps) {
  __shared__ double cs_[kSvdMaxP / 2], sn_[kSvdMaxP / 2];
  __shared__ int pi_[kSvdMaxP / 2], pj_[kSvdMaxP / 2];
  __shared__ int perm[kSvdMaxP];
  __shared__ double red[32];
  __shared__ int stop;
  const int half = p / 2;
  for (int i = threadIdx.x; i < p * p; i += blockDim.x) V[i] = (i / p == i % p) ? 1.0 : 0.0;
  for (int i = threadIdx.x; i < p; i += blockDim.x) perm[i] = i;
  __syncthreads();
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    // convergence test: off-diagonal vs total Frobenius norm
    double off = 0.0, tot = 0.0;
    for (int i = threadIdx.x; i < p * p; i += blockDim.x) {
      const double v = C[i] * C[i];
      tot += v;
      if (i / p != i % p) off += v;
    }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = off;
    __syncthreads();
    if (threadIdx.x == 0) {
      double o2 = 0.0;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) o2 += red[w];
      red[0] = o2;
    }
    __syncthreads();
    const double off_all = red[0];
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = tot;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t2 = 0.0;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t2 += red[w];
      stop = !(off_all > 1e-30 * t2);
    }
    __syncthreads();
    if (stop) break;
    for (int round = 0; round < p - 1; ++round) {
      // pairs (perm[k], perm[p-1-k])
      for (int k = threadIdx.x; k < half; k += blockDim.x) {
        int i = perm[k], j = perm[p - 1 - k];
        if (i > j) { const int t = i; i = j; j = t; }
        pi_[k] = i;
        pj_[k] = j;
        const double aij = C[i * p + j];
        double c = 1.0, s = 0.0;
        if (aij != 0.0) {
          const double tau = (C[j * p + j] - C[i * p + i]) / (2.0 * aij);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        cs_[k] = c;
        sn_[k] = s;
      }
      __syncthreads();
      // rows: C <- J^T C  (row i' = c row_i - s row_j, row j' = s row_i + c row_j)
      for (int t = threadIdx.x; t < half * p; t += blockDim.x) {
        const int k = t / p, col = t % p;
        const int i = pi_[k], j = pj_[k];
        const double c = cs_[k], s = sn_[k];
        const double xi = C[i * p + col], xj = C[j * p + col];
        C[i * p + col] = c * xi - s * xj;
        C[j * p + col] = s * xi + c * xj;
      }
      __syncthreads();
      // columns: C <- C J, V <- V J
      for (int t = threadIdx.x; t < half * p; t += blockDim.x) {
        const int k = t / p, row = t % p;
        const int i = pi_[k], j = pj_[k];
        const double c = cs_[k], s = sn_[k];
        const double xi = C[row * p + i], xj = C[row * p + j];
        C[row * p + i] = c * xi - s * xj;
        C[row * p + j] = s * xi + c * xj;
        const double vi = V[row * p + i], vj = V[row * p + j];
        V[row * p + i] = c * vi - s * vj;
        V[row * p + j] = s * vi + c * vj;
      }
      __syncthreads();
      for (int k = threadIdx.x; k < half; k += blockDim.x) {
        const int i = pi_[k], j = pj_[k];
        C[i * p + j] = 0.0;
        C[j * p + i] = 0.0;
      }
      // next round-robin arrangement: perm[0] fixed, the rest rotate by one
      __syncthreads();
      if (threadIdx.x == 0) {
        const int last = perm[p - 1];
        for (int k = p - 1; k > 1; --k) perm[k] = perm[k - 1];
        perm[1] = last;
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < p; i += blockDim.x) lam[i] = C[i * p + i];
}

// Sort the eigenpairs by decreasing eigenvalue and form, for the leading r,
//   M1[j][i] = V[j][o_i] sigma_i   and   M2[j][i] = V[j][o_i] / sigma_i (0 if sigma_i = 0)
// (p x r, row-major), sigma_i = sqrt(max(lam[o_i], 0)); sigma_out[i] = sigma_i.
__global__ void svd_coeff_kernel(const double* __restrict__ lam, const double* __restrict__ V, int p, int r,
                                 double* __restrict__ M1, double* __restrict__ M2, double* __restrict__ sigma_out) {
  __shared__ int order[kSvdMaxP];
  __shared__ double sig[kSvdMaxP];
  if (threadIdx.x == 0) {
    for (int i = 0; i < p; ++i) order[i] = i;
    for (int i = 0; i < p; ++i) {  // selection sort, ties keep the lower index
      int best = i;
      for (int k = i + 1; k < p; ++k)
        if (lam[order[k]] > lam[order[best]]) best = k;
      const int t = order[i];
      order[i] = order[best];
      order[best] = t;
    }
    for (int i = 0; i < r; ++i) sig[i] = sqrt(fmax(lam[order[i]], 0.0));
  }
  __syncthreads();
  for (int t = threadIdx.x; t < p * r; t += blockDim.x) {
    const int j = t / r, i = t % r;
    const double v = V[j * p + order[i]];
    M1[t] = v * sig[i];
    M2[t] = sig[i] > 0.0 ? v / sig[i] : 0.0;
  }
  for (int i = threadIdx.x; i < r; i += blockDim.x)
    if (sigma_out != nullptr) sigma_out[i] = sig[i];
}

// bf16 outputs: L1[k][i] = bf16(U1[k][i] / lambda_k) (K x r; the division in
// float64, none when smooth is nullptr) and L2[i][n] = bf16(V2[n][i]) (r x N).
__global__ void svd_store_kernel(const double* __restrict__ U1, int K, const double* __restrict__ V2, int N, int r,
                                 const float* __restrict__ smooth, __nv_bfloat16* __restrict__ L1,
                                 __nv_bfloat16* __restrict__ L2) {
  const int64_t n1 = static_cast<int64_t>(K) * r, n2 = static_cast<int64_t>(N) * r;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < n1 + n2;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (t < n1) {
      L1[t] = __double2bfloat16(smooth != nullptr ? U1[t] / static_cast<double>(smooth[t / r]) : U1[t]);
    } else {
      const int64_t u = t - n1;  // output index in L2 (r x N)
      const int64_t i = u / N, n = u % N;
      L2[u] = __double2bfloat16(V2[n * r + i]);
    }
  }
}

}  // namespace svdq
