// moments.cuh — moment-based row statistics and thresholds.
//
// "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification", method: query-dependent threshold routing (Eq. 4-5).  The
// proxy row ŝ_i = K̄ Q̄_i / sqrt(d) is a linear projection of the pooled keys,
// so its mean and variance follow from their first and second moments:
//   m   = (1/N) Σ_j K̄_j,   Σ_K = (1/N) Σ_j (K̄_j - m)(K̄_j - m)^T,
//   μ_i = Q̄_i · m / sqrt(d),   σ_i² = Q̄_i^T Σ_K Q̄_i / d,   τ_i = μ_i + β σ_i,
// in O(Ld + Nd²) time and O(d²) memory, without the N x N proxy map.
//
// Two kernels, both accumulating in fp64:
//   moments_kernel   one CTA per (batch, head): m, then the centred covariance
//                    (two passes, so a large common key offset does not cancel).
//   threshold_kernel Σ_K staged in shared memory; each warp evaluates the
//                    quadratic form for four query blocks at a time.
#pragma once

#include <cstdint>

namespace solattn {

enum ThresholdMode : int { kThresholdBeta = 0, kThresholdSelectAll = 1, kThresholdSelectNone = 2 };

template <int D>
__global__ void __launch_bounds__(256) moments_kernel(const float* __restrict__ kbar, int N,
                                                      double* __restrict__ mean_out,
                                                      double* __restrict__ cov_out) {
  constexpr int TPROW = 256 / D;   // threads sharing one covariance row
  constexpr int CPT = D / TPROW;   // covariance entries per thread
  constexpr int JB = 16;           // pooled keys staged per round
  __shared__ double s_m[D];
  __shared__ double s_kc[JB][D];

  const size_t bh = blockIdx.x;
  const int tid = threadIdx.x;
  const float* kb = kbar + bh * static_cast<size_t>(N) * D;

  // pass 1: mean of the pooled keys
  if (tid < D) {
    double acc = 0.0;
    for (int j = 0; j < N; ++j) acc += static_cast<double>(kb[static_cast<size_t>(j) * D + tid]);
    s_m[tid] = acc / N;
  }
  __syncthreads();

  // pass 2: centred second moment
  const int r = tid / TPROW;
  const int c0 = (tid % TPROW) * CPT;
  double acc[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) acc[c] = 0.0;

  for (int j0 = 0; j0 < N; j0 += JB) {
    const int nj = min(JB, N - j0);
    for (int e = tid; e < JB * D; e += 256) {
      const int jj = e / D, cc = e % D;
      s_kc[jj][cc] = (jj < nj) ? static_cast<double>(kb[static_cast<size_t>(j0 + jj) * D + cc]) - s_m[cc] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < JB; ++jj) {
      const double a = s_kc[jj][r];
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[c] = fma(a, s_kc[jj][c0 + c], acc[c]);
    }
    __syncthreads();
  }
  double* cov = cov_out + bh * D * D;
#pragma unroll
  for (int c = 0; c < CPT; ++c) cov[r * D + c0 + c] = acc[c] / N;
  if (tid < D) mean_out[bh * D + tid] = s_m[tid];
}

// Each CTA handles 32 query blocks of one (batch, head): 8 warps x 4 blocks.
template <int D>
__global__ void __launch_bounds__(256) threshold_kernel(const float* __restrict__ qbar,
                                                        const double* __restrict__ mean_in,
                                                        const double* __restrict__ cov_in, int N,
                                                        float beta, int mode, float* __restrict__ tau,
                                                        float* __restrict__ mu_dbg,
                                                        float* __restrict__ sigma_dbg) {
  constexpr int QW = 4;            // query blocks per warp
  constexpr int RPL = D / 32;      // quadratic-form rows per lane
  extern __shared__ __align__(16) double s_dyn[];
  double* s_cov = s_dyn;                 // [D][D]
  double* s_mean = s_cov + D * D;        // [D]
  double* s_q = s_mean + D;              // [8 warps][QW][D]

  const size_t bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const double* cov = cov_in + bh * D * D;
  for (int e = tid; e < D * D; e += 256) s_cov[e] = cov[e];
  if (tid < D) s_mean[tid] = mean_in[bh * D + tid];

  const int i_base = blockIdx.x * (8 * QW) + warp * QW;
  double* sq = s_q + warp * QW * D;
  for (int e = lane; e < QW * D; e += 32) {
    const int qq = e / D, cc = e % D;
    const int i = i_base + qq;
    sq[e] = (i < N) ? static_cast<double>(qbar[(bh * N + i) * D + cc]) : 0.0;
  }
  __syncthreads();

  // y = Σ_K q for QW query blocks; lane owns rows r = lane + 32*t.  Σ_K is
  // symmetric, so row r of Σ_K q reads column r of s_cov (conflict-free).
  double quad[QW], mu[QW];
#pragma unroll
  for (int qq = 0; qq < QW; ++qq) quad[qq] = mu[qq] = 0.0;
#pragma unroll
  for (int t = 0; t < RPL; ++t) {
    const int rr = lane + 32 * t;
    double y[QW];
#pragma unroll
    for (int qq = 0; qq < QW; ++qq) y[qq] = 0.0;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const double s = s_cov[c * D + rr];
#pragma unroll
      for (int qq = 0; qq < QW; ++qq) y[qq] = fma(s, sq[qq * D + c], y[qq]);
    }
#pragma unroll
    for (int qq = 0; qq < QW; ++qq) {
      quad[qq] = fma(sq[qq * D + rr], y[qq], quad[qq]);
      mu[qq] = fma(sq[qq * D + rr], s_mean[rr], mu[qq]);
    }
  }
#pragma unroll
  for (int qq = 0; qq < QW; ++qq) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      quad[qq] += __shfl_xor_sync(0xffffffffu, quad[qq], o);
      mu[qq] += __shfl_xor_sync(0xffffffffu, mu[qq], o);
    }
  }
  if (lane < QW) {
    double qd = 0.0, m = 0.0;
#pragma unroll
    for (int qq = 0; qq < QW; ++qq)
      if (qq == lane) { qd = quad[qq]; m = mu[qq]; }
    const int i = i_base + lane;
    if (i < N) {
      const double inv_sqrt_d = 1.0 / sqrt(static_cast<double>(D));
      const double mean_i = m * inv_sqrt_d;
      const double sd_i = sqrt(fmax(qd / D, 0.0));
      double t;
      if (mode == kThresholdSelectAll) t = -INFINITY;
      else if (mode == kThresholdSelectNone) t = INFINITY;
      else t = mean_i + static_cast<double>(beta) * sd_i;
      const size_t o = bh * N + i;
      tau[o] = static_cast<float>(t);
      if (mu_dbg) mu_dbg[o] = static_cast<float>(mean_i);
      if (sigma_dbg) sigma_dbg[o] = static_cast<float>(sd_i);
    }
  }
}

}  // namespace solattn
