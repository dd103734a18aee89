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
//   moments_kernel   one CTA per (batch, head, 64 x 64 piece of the upper
//                    triangle of Σ_K): one pass over the pooled keys, shifted
//                    by the first of them so a large common offset does not
//                    cancel; register tiles of 4 x 4 entries per thread.
//   threshold_kernel Σ_K staged in shared memory; each warp evaluates the
//                    quadratic form for eight query blocks at a time.
#pragma once

#include <cstdint>

namespace solattn {

enum ThresholdMode : int { kThresholdBeta = 0, kThresholdSelectAll = 1, kThresholdSelectNone = 2 };

constexpr int kThresholdBlocksPerWarp = 8;
constexpr int kThresholdBlocksPerCta = 8 * kThresholdBlocksPerWarp;

// Shared memory of threshold_kernel<D>: Σ_K, the key mean and the warps' query blocks (fp64).
constexpr size_t threshold_smem_bytes(int D) {
  return (static_cast<size_t>(D) * D + D + static_cast<size_t>(8) * kThresholdBlocksPerWarp * D) * sizeof(double);
}

template <int D>
__global__ void __launch_bounds__(256) moments_kernel(const float* __restrict__ kbar, int N,
                                                      double* __restrict__ mean_out,
                                                      double* __restrict__ cov_out) {
  constexpr int T = D / 64;   // 64 x 64 pieces per side of the d x d matrix
  constexpr int JB = 32;      // pooled keys staged per round
  __shared__ double s_r[JB][64];   // shifted key values, the piece's rows
  __shared__ double s_c[JB][64];   // shifted key values, the piece's columns
  __shared__ double s_sum[2][128];
  __shared__ float s_shift[128];

  // blockIdx.x enumerates the pieces (ti, tj) with ti <= tj; Σ_K is symmetric.
  int ti = 0, t = blockIdx.x;
  while (t >= T - ti) { t -= T - ti; ++ti; }
  const int tj = ti + t;
  const int R0 = 64 * ti, C0 = 64 * tj;

  const size_t bh = blockIdx.y;
  const int tid = threadIdx.x;
  const float* kb = kbar + bh * static_cast<size_t>(N) * D;

  // Shifted-data accumulation: with the shift c = K̄_0 (a sample of the keys),
  //   Σ_K = (1/N) Σ_j (K̄_j - c)(K̄_j - c)^T - (m - c)(m - c)^T,  m = c + (1/N) Σ_j (K̄_j - c),
  // and the terms stay of the size of the keys' spread, so a large common
  // offset does not cancel (one pass over the keys).
  const int e = tid & 127;                 // staged value: rows (e < 64) or columns
  const int col = (e < 64) ? R0 + e : C0 + (e - 64);
  const int sub = tid >> 7;                // staging threads take every other key
  if (tid < 128) s_shift[tid] = kb[col];
  __syncthreads();
  const float shift = s_shift[e];
  double run = 0.0;                        // Σ_j (K̄_j - c) for this thread's keys and column

  const int a = tid >> 4, b = tid & 15;    // rows a + 16p, columns b + 16q of the piece
  double acc[4][4];
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[p][q] = 0.0;

  for (int j0 = 0; j0 < N; j0 += JB) {
    float v[JB / 2];   // all of a round's loads in flight at once
#pragma unroll
    for (int u = 0; u < JB / 2; ++u) {
      const int j = j0 + sub + 2 * u;
      v[u] = (j < N) ? kb[static_cast<size_t>(j) * D + col] : shift;
    }
#pragma unroll
    for (int u = 0; u < JB / 2; ++u) {
      const double x = static_cast<double>(v[u]) - static_cast<double>(shift);
      run += x;
      if (e < 64) s_r[sub + 2 * u][e] = x;
      else s_c[sub + 2 * u][e - 64] = x;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < JB; ++jj) {
      double r[4], c[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) r[p] = s_r[jj][a + 16 * p];
#pragma unroll
      for (int q = 0; q < 4; ++q) c[q] = s_c[jj][b + 16 * q];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fma(r[p], c[q], acc[p][q]);
    }
    __syncthreads();
  }
  s_sum[sub][e] = run;
  __syncthreads();
  const double inv_n = 1.0 / N;
  double* cov = cov_out + bh * D * D;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int rr = a + 16 * p;
    const double dr = (s_sum[0][rr] + s_sum[1][rr]) * inv_n;               // (m - c) at row R0 + rr
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int cc = b + 16 * q;
      const double dc = (s_sum[0][64 + cc] + s_sum[1][64 + cc]) * inv_n;   // (m - c) at column C0 + cc
      const double v = acc[p][q] * inv_n - dr * dc;
      cov[(R0 + rr) * D + C0 + cc] = v;
      if (ti != tj) cov[(C0 + cc) * D + R0 + rr] = v;
    }
  }
  if (ti == tj && tid < 64)
    mean_out[bh * D + R0 + tid] = static_cast<double>(s_shift[tid]) + (s_sum[0][tid] + s_sum[1][tid]) * inv_n;
}

// Each CTA handles 64 query blocks of one (batch, head): 8 warps x 8 blocks.
template <int D>
__global__ void __launch_bounds__(256, 1) threshold_kernel(const float* __restrict__ qbar,
                                                        const double* __restrict__ mean_in,
                                                        const double* __restrict__ cov_in, int N,
                                                        float beta, int mode, float* __restrict__ tau,
                                                        float* __restrict__ mu_dbg,
                                                        float* __restrict__ sigma_dbg) {
  constexpr int QW = kThresholdBlocksPerWarp;   // query blocks per warp
  constexpr int RPL = D / 32;                   // rows of Σ_K q per lane
  extern __shared__ __align__(16) double s_dyn[];
  double* s_cov = s_dyn;                 // [D][D]
  double* s_mean = s_cov + D * D;        // [D]
  double* s_q = s_mean + D;              // [8 warps][QW][D]

  const size_t bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Staging: eight 16-byte loads in flight per thread before their stores.
  const double2* cov2 = reinterpret_cast<const double2*>(cov_in + bh * D * D);
  constexpr int kCovIters = D * D / 2 / 256;
  static_assert(kCovIters % 8 == 0, "covariance staging unrolls by 8");
  for (int u0 = 0; u0 < kCovIters; u0 += 8) {
    double2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = cov2[(u0 + u) * 256 + tid];
#pragma unroll
    for (int u = 0; u < 8; ++u) reinterpret_cast<double2*>(s_cov)[(u0 + u) * 256 + tid] = v[u];
  }
  if (tid < D) s_mean[tid] = mean_in[bh * D + tid];

  const int i_base = blockIdx.x * (8 * QW) + warp * QW;
  double* sq = s_q + warp * QW * D;
  {
    float v[QW * D / 32];
#pragma unroll
    for (int u = 0; u < QW * D / 32; ++u) {
      const int e = lane + 32 * u, qq = e / D, cc = e % D;
      const int i = i_base + qq;
      v[u] = (i < N) ? qbar[(bh * N + i) * D + cc] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < QW * D / 32; ++u) sq[lane + 32 * u] = static_cast<double>(v[u]);
  }
  __syncthreads();

  // y = Σ_K q for QW query blocks; lane owns rows r = lane + 32*t.  Σ_K is
  // symmetric, so row r of Σ_K q reads column r of s_cov (conflict-free); the
  // query values are warp-wide broadcasts, two columns per load.
  double y[RPL][QW];
#pragma unroll
  for (int t = 0; t < RPL; ++t)
#pragma unroll
    for (int qq = 0; qq < QW; ++qq) y[t][qq] = 0.0;
#pragma unroll 2
  for (int c = 0; c < D; c += 2) {
    double2 qv[QW];
#pragma unroll
    for (int qq = 0; qq < QW; ++qq) qv[qq] = *reinterpret_cast<const double2*>(&sq[qq * D + c]);
#pragma unroll
    for (int t = 0; t < RPL; ++t) {
      const double s0 = s_cov[c * D + lane + 32 * t];
      const double s1 = s_cov[(c + 1) * D + lane + 32 * t];
#pragma unroll
      for (int qq = 0; qq < QW; ++qq) y[t][qq] = fma(s1, qv[qq].y, fma(s0, qv[qq].x, y[t][qq]));
    }
  }
  double quad[QW], mu[QW];
#pragma unroll
  for (int qq = 0; qq < QW; ++qq) {
    quad[qq] = mu[qq] = 0.0;
#pragma unroll
    for (int t = 0; t < RPL; ++t) {
      const int rr = lane + 32 * t;
      quad[qq] = fma(sq[qq * D + rr], y[t][qq], quad[qq]);
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
