// fused.cuh — the fused Sol-Attn kernel for sm_100a: on-the-fly routing, the
// exact inner loop over selected K/V blocks and the zeroth-order approximation
// of the unselected ones, in one online-softmax pass.
//
// "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification", method: chunk-wise streaming thresholding (Eq. 6-7, the
// nested-loop structure), proxy-score reuse (Eq. 8-10), the batched
// token-to-block tile (Eq. 11) and the kernel of Fig. 4 / Alg. 3.2.
//
// Work item = (batch*head, pair of adjacent query blocks).  The two 64-token
// query blocks i0 = 2p and i1 = 2p+1 form one 128-row tile, the M of a full
// rate cta_group::1 tcgen05 MMA.  Each half keeps its own selection S_i; the
// pair streams the union of the two selections through the exact path and
// masks, per half, the columns of blocks that half did not select (those
// blocks reach that half through the approximation instead).  The result is
// the same as processing the blocks one by one.
//
// For each chunk t of C pooled keys (outer loop):
//   route   ŝ_ij = Q̄_i·K̄_j/sqrt(d) in fp32 on CUDA cores, compared with τ_i;
//           a warp ballot turns 32 tests into one mask word (both halves).
//   approx  A = Q·K̄^(t)ᵀ (tcgen05, 128 x W, fp32 in TMEM, K̄ as a bf16 hi/lo
//           pair so the logits keep K̄ to ~16 bits); per row and per
//           column not selected by the row's half: running max m, running sum
//           l += n_j 2^(a-m), and O += 2^(a-m) V̂_j (tcgen05, P from smem).
//   exact   for the selected blocks of the chunk, two at a time: S = Q·[K_a;K_b]ᵀ
//           (128 x 128), mask per half and for keys >= L, online-softmax update,
//           O += P·[V_a;V_b].
// Epilogue: O / l in bf16 for rows < L; per-row counts |S_i|.
//
// Shared memory (1024-byte aligned, 128-byte swizzled K-major tiles):
//   Q 128 x d | K-side 128 x d | V-side 128 x d | P 128 x 128 | control block.
// TMEM: columns [0, 128) hold O (fp32, lane = row), [128, 256) hold S / A.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace solattn {

constexpr int kMaxMaskWords = 512;       // N <= 16384 pooled blocks per head
constexpr unsigned kFlagSelectAll = 1u;
constexpr unsigned kFlagExactOnly = 2u;
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusDevice = 2u;

struct FusedParams {
  int BH, L, N, W;          // W: approximation tile width (MMA N), 32 or 64
  int chunk;                // C
  int num_pairs, num_items;
  unsigned flags;
  float scale_log2;         // log2(e) / sqrt(d)
  float inv_sqrt_d;
  const float* qbar;        // [BH][N][d] fp32
  const float* kbar;        // [BH][N][d] fp32
  const float* tau;         // [BH][N] fp32
  int* counts;              // [BH][N]
  uint32_t* mask_out;       // nullable [BH][N][ceil(N/32)]
  uint16_t* out;            // [BH][L][d] bf16 bits
  unsigned* work_counter;   // zeroed before launch
  unsigned* status;         // sticky error word
  unsigned long long timeout_ns;
};

struct __align__(16) FusedCtl {
  float qbar[2][128];               // pooled queries of the pair (read as float4)
  uint32_t mask[2][kMaxMaskWords];  // selection bits of both halves
  uint64_t bar_q;
  uint64_t bar_kv;
  uint64_t bar_mma;
  uint32_t tmem_base;
  int item;
  int abort;
  int cnt[2];
};
static_assert(offsetof(FusedCtl, qbar) % 16 == 0, "float4 access to qbar");
static_assert(offsetof(FusedCtl, bar_q) % 8 == 0, "mbarrier alignment");

constexpr uint32_t kTileBytes = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0, kSmemK = 32768, kSmemV = 65536, kSmemP = 98304, kSmemCtl = 131072;
constexpr uint32_t kFusedSmemBytes = kSmemCtl + sizeof(FusedCtl) + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 0, kTmemS = 128;

__device__ __forceinline__ bool mask_bit(const uint32_t* m, int j) { return (m[j >> 5] >> (j & 31)) & 1u; }

// First j in [from, hi) selected by either half, or hi.
__device__ __forceinline__ int next_union(const FusedCtl& ctl, int from, int hi) {
  int j = from;
  while (j < hi) {
    const int w = j >> 5;
    const uint32_t u = (ctl.mask[0][w] | ctl.mask[1][w]) & (0xFFFFFFFFu << (j & 31));
    if (u) {
      const int jj = (w << 5) + __ffs(u) - 1;
      return jj < hi ? jj : hi;
    }
    j = (w + 1) << 5;
  }
  return hi;
}

// Write one row's 32 probabilities (columns [c0, c0+32)) as bf16 into the
// 128B-swizzled K-major P tile.
__device__ __forceinline__ void store_p32(uint8_t* sP, int row, int c0, const float (&p)[32]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {  // four 16-byte chunks of 8 columns
    const int c = c0 + 8 * g;
    const int cb = c >> 6;                      // 64-column block
    const int chunk = (c & 63) >> 3;            // 16-byte chunk within the 128-byte row
    const uint32_t off = cb * 16384u + row * 128u + (((chunk ^ (row & 7)) & 7) << 4);
    uint4 v;
    v.x = pack_bf16x2(p[8 * g + 0], p[8 * g + 1]);
    v.y = pack_bf16x2(p[8 * g + 2], p[8 * g + 3]);
    v.z = pack_bf16x2(p[8 * g + 4], p[8 * g + 5]);
    v.w = pack_bf16x2(p[8 * g + 6], p[8 * g + 7]);
    *reinterpret_cast<uint4*>(sP + off) = v;
  }
}

template <int D>
__global__ void __launch_bounds__(128, 1)
    sol_attn_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
                          const __grid_constant__ CUtensorMap tm_kl, const __grid_constant__ CUtensorMap tm_vb,
                          const FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sK = smem + kSmemK;
  uint8_t* sV = smem + kSmemV;
  uint8_t* sP = smem + kSmemP;
  FusedCtl& ctl = *reinterpret_cast<FusedCtl*>(smem + kSmemCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int KSTEPS = D / 16;           // MMA K-steps over the head dimension
  constexpr uint32_t CB = 16384;           // bytes per 64-column block of a 128-row tile
  const int NW = (p.N + 31) >> 5;
  volatile int* abort_flag = &ctl.abort;

  if (tid == 0) {
    mbar_init(&ctl.bar_q, 1);
    mbar_init(&ctl.bar_kv, 1);
    mbar_init(&ctl.bar_mma, 1);
    ctl.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_kb);
    tma_prefetch_desc(&tm_kl);
    tma_prefetch_desc(&tm_vb);
  }
  if (warp == 0) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tO = tmem + kTmemO + lane_base;
  const uint32_t tS = tmem + kTmemS + lane_base;

  uint32_t ph_q = 0, ph_kv = 0, ph_mma = 0;
  const uint32_t idesc_pv = idesc_bf16_f32(128, D, 1);
  const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
  const int row = tid;                     // this thread's row of the 128-row tile
  const int half = row >> 6;
  const int tail_n = p.L - 64 * (p.N - 1);

  // Wait for one mbarrier phase.  On a timeout the thread raises the CTA's
  // abort flag and the status word; from then on every wait returns at once,
  // thread 0 issues no more copies or MMAs, and all threads run the same
  // (now empty) control flow to the end of the item, so no barrier is missed.
  auto wait_all = [&](uint64_t* bar, uint32_t& ph) {
    const bool ok = mbar_wait(bar, ph, abort_flag, p.timeout_ns);
    ph ^= 1u;
    if (!ok) {
      *abort_flag = 1;
      atomicOr(p.status, kStatusTimeout);
    }
  };
  auto issuer = [&]() -> bool { return tid == 0 && *abort_flag == 0; };

  for (;;) {
    if (tid == 0) ctl.item = *abort_flag ? p.num_items : static_cast<int>(atomicAdd(p.work_counter, 1u));
    __syncthreads();
    const int item = ctl.item;
    if (item >= p.num_items) break;
    const int bh = item / p.num_pairs;
    const int pair = item - bh * p.num_pairs;
    const int i0 = 2 * pair, i1 = 2 * pair + 1;
    const bool has1 = i1 < p.N;

    // ---- load the 128-row query tile (TMA, zero-filled past L)
    if (issuer()) {
      mbar_arrive_expect_tx(&ctl.bar_q, 128u * D * 2u);
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb) tma_load_3d(sQ + cb * CB, &tm_q, &ctl.bar_q, cb * 64, 128 * pair, bh);
    }

    // ---- routing for the whole pair (method: Eq. 6-7; tested as ŝ >= τ)
    const float* qb = p.qbar + static_cast<size_t>(bh) * p.N * D;
    const float* kb = p.kbar + static_cast<size_t>(bh) * p.N * D;
    for (int e = tid; e < 2 * D; e += 128) {
      const int h = e / D, c = e % D;
      const int i = h ? i1 : i0;
      ctl.qbar[h][c] = (i < p.N) ? qb[static_cast<size_t>(i) * D + c] : 0.f;
    }
    if (tid < 2) ctl.cnt[tid] = 0;
    __syncthreads();
    const float tau0 = p.tau[static_cast<size_t>(bh) * p.N + i0];
    const float tau1 = has1 ? p.tau[static_cast<size_t>(bh) * p.N + i1] : INFINITY;
    int my_cnt0 = 0, my_cnt1 = 0;
    for (int g = warp; g < NW; g += 4) {
      const int j = 32 * g + lane;
      bool s0 = false, s1 = false;
      if (j < p.N) {
        const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D);
        float d0 = 0.f, d1 = 0.f;
#pragma unroll 8
        for (int c4 = 0; c4 < D / 4; ++c4) {
          const float4 x = __ldg(kr + c4);
          const float4 a = *reinterpret_cast<const float4*>(&ctl.qbar[0][4 * c4]);
          const float4 b = *reinterpret_cast<const float4*>(&ctl.qbar[1][4 * c4]);
          d0 = fmaf(a.x, x.x, d0); d0 = fmaf(a.y, x.y, d0); d0 = fmaf(a.z, x.z, d0); d0 = fmaf(a.w, x.w, d0);
          d1 = fmaf(b.x, x.x, d1); d1 = fmaf(b.y, x.y, d1); d1 = fmaf(b.z, x.z, d1); d1 = fmaf(b.w, x.w, d1);
        }
        s0 = d0 * p.inv_sqrt_d >= tau0;
        s1 = has1 && (d1 * p.inv_sqrt_d >= tau1);
      }
      const uint32_t m0 = __ballot_sync(0xFFFFFFFFu, s0);
      const uint32_t m1 = __ballot_sync(0xFFFFFFFFu, s1);
      if (lane == 0) {
        ctl.mask[0][g] = m0;
        ctl.mask[1][g] = m1;
        my_cnt0 += __popc(m0);
        my_cnt1 += __popc(m1);
      }
    }
    if (lane == 0) {
      atomicAdd(&ctl.cnt[0], my_cnt0);
      atomicAdd(&ctl.cnt[1], my_cnt1);
    }
    __syncthreads();
    if (tid == 0) {
      p.counts[static_cast<size_t>(bh) * p.N + i0] = ctl.cnt[0];
      if (has1) p.counts[static_cast<size_t>(bh) * p.N + i1] = ctl.cnt[1];
    }
    if (p.mask_out) {
      for (int e = tid; e < 2 * NW; e += 128) {
        const int h = e / NW, g = e % NW;
        const int i = h ? i1 : i0;
        if (i < p.N) p.mask_out[(static_cast<size_t>(bh) * p.N + i) * NW + g] = ctl.mask[h][g];
      }
    }

    // ---- online-softmax state of this thread's row (log2 domain)
    float m_run = -INFINITY, l_run = 0.f;
    bool o_init = false;
    wait_all(&ctl.bar_q, ph_q);

    const uint32_t* own = ctl.mask[half];
    const bool exact_only = (p.flags & kFlagExactOnly) != 0;

    // One tile: issue S MMA (tid 0), online-softmax on this thread's row,
    // issue PV MMA.  kind 0 = approximation, 1 = exact.
    auto process_tile = [&](int kind, int ncols_mma, int ja, int jb, int a_valid) {
      // S / A = Q · Kside^T
      if (issuer()) {
        tc_fence_after();
        const uint32_t idesc_s = idesc_bf16_f32(128, ncols_mma, 0);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t koff = (kk >> 2) * CB + (kk & 3) * 32;
          umma_ss(tmem + kTmemS, sdesc_sw128(sQa + koff, 16, 1024), sdesc_sw128(sKa + koff, 16, 1024), idesc_s,
                  kk > 0 ? 1u : 0u);
        }
        if (kind == 0) {  // + Q · K̄_lo^T (rows 64.. of the K-side tile)
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            const uint32_t koff = (kk >> 2) * CB + (kk & 3) * 32;
            umma_ss(tmem + kTmemS, sdesc_sw128(sQa + koff, 16, 1024), sdesc_sw128(sKa + 8192 + koff, 16, 1024),
                    idesc_s, 1u);
          }
        }
        umma_commit(&ctl.bar_mma);
      }
      wait_all(&ctl.bar_mma, ph_mma);
      tc_fence_after();

      // masked logits of this row
      float x[128];
#pragma unroll
      for (int c32 = 0; c32 < 4; ++c32) {
        if (c32 * 32 < ncols_mma) {
          uint32_t r[32];
          tmem_ld_x32(tS + c32 * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c32 * 32 + e] = __uint_as_float(r[e]) * p.scale_log2;
        }
      }
      // validity bitmap of the row's columns: vm[c32] bit e <-> column 32*c32 + e
      uint32_t vm[4];
#pragma unroll
      for (int c32 = 0; c32 < 4; ++c32) {
        uint32_t bits = 0u;
        if (c32 * 32 < ncols_mma) {
          if (kind == 0) {
            const int c0 = 32 * c32;
            const int nv = min(max(a_valid - c0, 0), 32);
            const uint32_t range = (nv >= 32) ? 0xFFFFFFFFu : ((1u << nv) - 1u);
            const int j0 = ja + c0;
            const int w = j0 >> 5, sh = j0 & 31;
            uint32_t sel = (w < NW) ? (own[w] >> sh) : 0u;
            if (sh && w + 1 < NW) sel |= own[w + 1] << (32 - sh);
            bits = range & ~sel;
          } else {
            const int jx = (c32 < 2) ? ja : jb;
            const int key0 = 64 * jx + 32 * (c32 & 1);
            const int nv = min(max(p.L - key0, 0), 32);
            const uint32_t range = (nv >= 32) ? 0xFFFFFFFFu : ((1u << nv) - 1u);
            bits = mask_bit(own, jx) ? range : 0u;
          }
        }
        vm[c32] = bits;
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if ((vm[c >> 5] >> (c & 31)) & 1u) tmax = fmaxf(tmax, x[c]);
      // lazy rescale: move the reference max only when it grows by > 8 (x256).
      // TMEM loads/stores are warp-collective, so the O update runs for the
      // whole warp when any of its rows needs it (alpha = 1 for the others).
      const bool need = tmax > m_run + 8.f || (m_run == -INFINITY && tmax != -INFINITY);
      float alpha = 1.f;
      if (need) {
        const float m_new = fmaxf(m_run, tmax);
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      if (o_init && __any_sync(0xFFFFFFFFu, need)) {
#pragma unroll
        for (int c32 = 0; c32 < D / 32; ++c32) {
          uint32_t r[32];
          tmem_ld_x32(tO + c32 * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st_x32(tO + c32 * 32, r);
        }
        tmem_st_wait();
      }
      const float m_ref = (m_run == -INFINITY) ? 0.f : m_run;
      // tail block weight for the approximation (n_j of the ragged last block)
      const int tail_col = (kind == 0) ? (p.N - 1 - ja) : -1;
      float ps = 0.f;
#pragma unroll
      for (int c32 = 0; c32 < 4; ++c32) {
        if (c32 * 32 < ncols_mma) {
          float pr[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = c32 * 32 + e;
            const bool valid = (vm[c32] >> e) & 1u;
            const float pv = valid ? ex2_approx(x[c] - m_ref) : 0.f;
            const float w = (kind == 0) ? ((c == tail_col) ? static_cast<float>(tail_n) : 64.f) : 1.f;
            ps = fmaf(w, pv, ps);
            pr[e] = pv;
          }
          store_p32(sP, row, c32 * 32, pr);
        }
      }
      l_run += ps;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // O += P · Vside
      if (issuer()) {
        tc_fence_after();
        const int ksteps = ncols_mma / 16;
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint32_t poff = (kk >> 2) * CB + (kk & 3) * 32;
          umma_ss(tmem + kTmemO, sdesc_sw128(sPa + poff, 16, 1024), sdesc_sw128(sVa + kk * 2048, CB, 1024),
                  idesc_pv, (o_init || kk > 0) ? 1u : 0u);
        }
        umma_commit(&ctl.bar_mma);
      }
      wait_all(&ctl.bar_mma, ph_mma);
      tc_fence_after();
      o_init = true;
    };

    const int C = p.chunk;
    for (int lo = 0; lo < p.N; lo += C) {
      const int hi = min(lo + C, p.N);
      // -- approximation sub-tiles of this chunk (Eq. 9-11)
      if (!exact_only) {
        for (int a0 = lo; a0 < hi; a0 += p.W) {
          const int a1 = min(a0 + p.W, hi);
          // skip when every column is selected by both halves (nothing to approximate)
          bool any = false;
          for (int j = a0; j < a1 && !any; ++j)
            any = !mask_bit(ctl.mask[0], j) || (has1 && !mask_bit(ctl.mask[1], j));
          if (!any) continue;
          if (issuer()) {
            mbar_arrive_expect_tx(&ctl.bar_kv, 3u * p.W * D * 2u);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
              tma_load_3d(sK + cb * CB, &tm_kb, &ctl.bar_kv, cb * 64, a0, bh);
              tma_load_3d(sK + cb * CB + 8192, &tm_kl, &ctl.bar_kv, cb * 64, a0, bh);
              tma_load_3d(sV + cb * CB, &tm_vb, &ctl.bar_kv, cb * 64, a0, bh);
            }
          }
          wait_all(&ctl.bar_kv, ph_kv);
          process_tile(0, p.W, a0, 0, a1 - a0);
        }
      }
      // -- exact inner loop over the selected blocks of this chunk (Eq. 7)
      int j = next_union(ctl, lo, hi);
      while (j < hi) {
        const int jb = next_union(ctl, j + 1, hi);
        const int nblk = (jb < hi) ? 2 : 1;
        if (issuer()) {
          mbar_arrive_expect_tx(&ctl.bar_kv, static_cast<uint32_t>(nblk) * 2u * 64u * D * 2u);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            tma_load_3d(sK + cb * CB, &tm_k, &ctl.bar_kv, cb * 64, 64 * j, bh);
            tma_load_3d(sV + cb * CB, &tm_v, &ctl.bar_kv, cb * 64, 64 * j, bh);
            if (nblk == 2) {
              tma_load_3d(sK + cb * CB + 8192, &tm_k, &ctl.bar_kv, cb * 64, 64 * jb, bh);
              tma_load_3d(sV + cb * CB + 8192, &tm_v, &ctl.bar_kv, cb * 64, 64 * jb, bh);
            }
          }
        }
        wait_all(&ctl.bar_kv, ph_kv);
        process_tile(1, 64 * nblk, j, nblk == 2 ? jb : -1, 0);
        j = (nblk == 2) ? next_union(ctl, jb + 1, hi) : hi;
      }
    }
    // ---- epilogue: O / l for rows < L (Eq. 10 normalisation)
    {
      const int token = 128 * pair + row;
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      uint16_t* orow = p.out + (static_cast<size_t>(bh) * p.L + token) * D;
#pragma unroll
      for (int c32 = 0; c32 < D / 32; ++c32) {
        uint32_t r[32];
        if (o_init) {
          tmem_ld_x32(tO + c32 * 32, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (token < p.L) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]) * inv_l, __uint_as_float(r[8 * g + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]) * inv_l, __uint_as_float(r[8 * g + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]) * inv_l, __uint_as_float(r[8 * g + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]) * inv_l, __uint_as_float(r[8 * g + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + c32 * 32 + 8 * g) = v;
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // After a timeout, give copies or MMAs that may still be in flight a bounded
  // time to land before the shared memory and TMEM are released.
  if (*abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace solattn
