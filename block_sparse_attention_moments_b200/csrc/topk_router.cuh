// topk_router.cuh — a materialised top-k block router, the kind of routing the
// method is compared with (experiments: routing latency against top-k and
// top-p routers that materialise and traverse the proxy map, Fig. 5b/5c).  It
// is a measurement aid, not a step of the method:
//   proxy_map_kernel  writes the whole proxy map ŝ_ij = Q̄_i·K̄_j/sqrt(d) of
//                     every head to HBM (fp32, B*H*N*N values);
//   topk_mask_kernel  reads each row back and keeps its k largest entries
//                     (ties broken towards the lower block index) as mask
//                     bits, by a radix select on the order-preserving bit
//                     pattern of the fp32 values.
#pragma once

#include <cstdint>

namespace solattn {

constexpr int kMapTile = 64;   // proxy-map tile (query blocks x key blocks) per CTA

// One CTA of 256 threads computes a 64 x 64 tile of one head's map in fp32;
// each thread 4 x 4 entries.  Shared memory: the tile's pooled queries and
// keys, D + 1 floats a row (the pad spreads the column accesses over banks).
template <int D>
__global__ void __launch_bounds__(256) proxy_map_kernel(const float* __restrict__ qbar,
                                                        const float* __restrict__ kbar, int N, float inv_sqrt_d,
                                                        float* __restrict__ map) {
  extern __shared__ float sm[];
  float* sq = sm;                          // [64][D + 1]
  float* sk = sm + kMapTile * (D + 1);     // [64][D + 1]
  const int i0 = blockIdx.y * kMapTile, j0 = blockIdx.x * kMapTile;
  const size_t bh = blockIdx.z;
  const float* qb = qbar + bh * static_cast<size_t>(N) * D;
  const float* kb = kbar + bh * static_cast<size_t>(N) * D;
  for (int e = threadIdx.x; e < kMapTile * D; e += 256) {
    const int r = e / D, c = e % D;
    sq[r * (D + 1) + c] = (i0 + r < N) ? qb[static_cast<size_t>(i0 + r) * D + c] : 0.f;
    sk[r * (D + 1) + c] = (j0 + r < N) ? kb[static_cast<size_t>(j0 + r) * D + c] : 0.f;
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;   // rows ty + 16 a, columns tx + 16 b
  float acc[4][4] = {};
  for (int c = 0; c < D; ++c) {
    float a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a[u] = sq[(ty + 16 * u) * (D + 1) + c];
      b[u] = sk[(tx + 16 * u) * (D + 1) + c];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
  }
  float* mrow = map + bh * static_cast<size_t>(N) * N;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty + 16 * u;
    if (i >= N) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int j = j0 + tx + 16 * v;
      if (j < N) mrow[static_cast<size_t>(i) * N + j] = acc[u][v] * inv_sqrt_d;
    }
  }
}

// fp32 bit pattern -> unsigned key with the same order (larger value, larger key)
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One CTA of 256 threads per (head, query block) row: the row's N keys in
// shared memory, four 8-bit radix passes (most significant first) find the
// k-th largest key; entries above it are kept, and of the entries equal to it
// the lowest-indexed ones until k are kept.  mask: [B*H][N][ceil(N/32)].
__global__ void __launch_bounds__(256) topk_mask_kernel(const float* __restrict__ map, int N, int k,
                                                        uint32_t* __restrict__ mask) {
  extern __shared__ uint32_t keys[];       // [N]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_need, s_eqbase;
  __shared__ uint32_t s_wcount[8];
  const size_t row = blockIdx.x;           // bh * N + i
  const float* mrow = map + row * N;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int j = tid; j < N; j += 256) keys[j] = order_key(mrow[j]);
  if (tid == 0) {
    s_prefix = 0u;
    s_need = static_cast<uint32_t>(k);     // how many of the still-undecided entries to take
  }
  __syncthreads();
  uint32_t prefix = 0u, pmask = 0u;
  for (int pass = 0; pass < 4 && k > 0 && k < N; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = tid; b < 256; b += 256) hist[b] = 0u;
    __syncthreads();
    for (int j = tid; j < N; j += 256) {
      const uint32_t x = keys[j];
      if ((x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (tid == 0) {   // digit of the k-th largest among the candidates
      uint32_t need = s_need, b = 255u;
      for (;; --b) {
        if (hist[b] >= need || b == 0u) break;
        need -= hist[b];
      }
      s_prefix = prefix | (b << shift);
      s_need = need;
    }
    __syncthreads();
    prefix = s_prefix;
    pmask |= 0xFFu << shift;
  }
  // threshold key: prefix (after the passes every bit is fixed); s_need of the
  // entries equal to it are taken, lowest index first
  const uint32_t thr = prefix;
  const uint32_t take_eq = (k <= 0) ? 0u : (k >= N ? 0xFFFFFFFFu : s_need);
  const int NW = (N + 31) >> 5;
  uint32_t* mr = mask + row * NW;
  if (tid == 0) s_eqbase = 0u;
  __syncthreads();
  // walk the row in chunks of 256 so that ties are ranked by index
  for (int base = 0; base < N; base += 256) {
    const int j = base + tid;
    const uint32_t x = (j < N) ? keys[j] : 0u;
    const bool valid = j < N;
    const bool gt = valid && (k >= N || (k > 0 && x > thr));
    const bool eq = valid && k > 0 && k < N && x == thr;
    const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
    if (lane == 0) s_wcount[warp] = __popc(eqb);
    __syncthreads();
    uint32_t before = s_eqbase;
    for (int w = 0; w < warp; ++w) before += s_wcount[w];
    before += __popc(eqb & ((1u << lane) - 1u));
    const bool take = gt || (eq && before < take_eq);
    const uint32_t bits = __ballot_sync(0xFFFFFFFFu, take);
    if (lane == 0 && base + 32 * warp < N) mr[(base >> 5) + warp] = bits;
    __syncthreads();
    if (tid == 0) {
      uint32_t tot = 0u;
      for (int w = 0; w < 8; ++w) tot += s_wcount[w];
      s_eqbase += tot;
    }
    __syncthreads();
  }
}

}  // namespace solattn
