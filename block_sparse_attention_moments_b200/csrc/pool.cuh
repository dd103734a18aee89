// pool.cuh — block pooling of Q, K and V (one HBM pass over the inputs).
//
// "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification", method: threshold routing (block-proxy logits, Eq. 3) and
// proxy-score reuse (summed value V̂_j before Eq. 9; KC/VC of Alg. 3.2):
//   Q̄_j = mean of block j's valid query tokens, K̄_j = mean of its valid keys,
//   V̂_j = sum of its valid values; a ragged last block is pooled over its
//   valid tokens only.
//
// The fused kernel's approximation multiplies probabilities that already carry
// the block's token count n_j by the block mean V̂_j / n_j, so V is also written
// as that mean in bf16 (V̂ itself is only exported for checks).
//
// K̄ is also written as a bf16 pair (hi, lo = bf16(K̄ - hi)): the approximation
// tile multiplies Q by both, so its logits carry K̄ to ~16 significant bits
// rather than bf16's 8 (the exact path's K is bf16 input and needs no split).
//
// One CTA of 256 threads pools one 64-token block of all three tensors.  Each
// thread streams 16-byte vectors (8 bf16) with no-allocate loads and keeps fp32
// partial sums; a shared-memory tree finishes the column sums.  The kernel is
// HBM-bound: 3 * n_j * d * 2 bytes read per block.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace solattn {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += __uint_as_float(w[i] << 16);
    a[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                   const uint16_t* __restrict__ v, int L, int N,
                                                   float* __restrict__ qbar, float* __restrict__ kbar,
                                                   __nv_bfloat16* __restrict__ kbar_bf,
                                                   __nv_bfloat16* __restrict__ kbar_lo,
                                                   __nv_bfloat16* __restrict__ vbar_bf,
                                                   float* __restrict__ vhat_f32 /* nullable */) {
  constexpr int TPR = D / 8;      // threads per token row (16 bytes each)
  constexpr int RPP = 256 / TPR;  // token rows per pass
  __shared__ float red[3][RPP][D];

  const int j = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int c8 = tid % TPR;
  const int rsub = tid / TPR;
  const int n = min(64, L - 64 * j);
  const size_t base = (bh * static_cast<size_t>(L) + 64u * static_cast<size_t>(j)) * D + 8 * c8;

  float aq[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float ak[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float av[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int r = rsub; r < 64; r += RPP) {
    if (r < n) {
      const size_t off = base + static_cast<size_t>(r) * D;
      const uint4 xq = ld_stream_v4(q + off);
      const uint4 xk = ld_stream_v4(k + off);
      const uint4 xv = ld_stream_v4(v + off);
      acc_bf16x8(aq, xq);
      acc_bf16x8(ak, xk);
      acc_bf16x8(av, xv);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red[0][rsub][8 * c8 + i] = aq[i];
    red[1][rsub][8 * c8 + i] = ak[i];
    red[2][rsub][8 * c8 + i] = av[i];
  }
  __syncthreads();
  if (tid < D) {
    float sq = 0.f, sk = 0.f, sv = 0.f;
#pragma unroll
    for (int r = 0; r < RPP; ++r) {
      sq += red[0][r][tid];
      sk += red[1][r][tid];
      sv += red[2][r][tid];
    }
    const float fn = static_cast<float>(n);
    const size_t o = (bh * static_cast<size_t>(N) + j) * D + tid;
    const float mk = sk / fn;
    qbar[o] = sq / fn;
    kbar[o] = mk;
    const __nv_bfloat16 hi = __float2bfloat16_rn(mk);
    kbar_bf[o] = hi;
    kbar_lo[o] = __float2bfloat16_rn(mk - __bfloat162float(hi));
    vbar_bf[o] = __float2bfloat16_rn(sv / fn);
    if (vhat_f32) vhat_f32[o] = sv;
  }
}

}  // namespace solattn
