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
// For each window of pooled keys (the chunk C, widened to at least 64) the
// item's tile sequence holds
//   exact   the selected blocks of the chunk, two per tile: S = Q·[K_a;K_b]ᵀ
//           (128 x 128), per-half / key >= L masks, online-softmax update,
//           O += P·[V_a;V_b];
//   approx  A = Q·K̄ᵀ over the chunk's pooled keys (128 x W, W = 32 or 64; K̄
//           as a bf16 hi/lo pair so the logits keep K̄ to ~16 bits); per row,
//           columns not selected by the row's half get p = n_j 2^(a-m) (n_j
//           folded into the logit as + log2 n_j), l += p and O += p V̄_j with
//           V̄_j = V̂_j / n_j, which is Eq. 9-10's n_j e^a in the denominator
//           and e^a V̂_j above.
// The walk starts at the chunk holding the item's own query blocks (see
// TileIter).  Epilogue: O / l in bf16 for rows < L.
//
// Warp roles (384 threads, one persistent CTA per SM, atomic work counter):
//   warps 0-7  softmax, two warpgroups: each thread owns one tile row and one
//              half of every tile's columns; masks, lazy-rescaled one-pass
//              online softmax, P into TMEM, epilogue.
//   warp 8     TMA producers: lane 0 loads Q and the K side (K blocks, or K̄
//              hi/lo), lane 1 the V side (V blocks, or V̄).
//   warp 9     tcgen05 MMA issuer: S runs up to two tiles ahead of the PVs.
//   warp 10    routing: fetches the next item, computes ŝ_ij = Q̄_i·K̄_j/sqrt(d)
//              in fp32 for both halves, compares with τ_i (warp ballot -> mask
//              words), one item ahead (double-buffered mask slots).
//   warp 11    scheduler: walks each item's tile sequence from its masks and
//              publishes one descriptor per tile (blocks, column validity per
//              half, first/last flags) into a shared-memory ring that the
//              producers, the MMA issuer and the softmax warps consume.
//
// The two threads of a row (one per warpgroup) share one reference maximum,
// agreed per tile through shared memory, so a single O accumulates the whole
// row.  P is written back into TMEM over the thread's own part of its S tile
// (bf16 pairs) and fed to the PV MMA as its A operand, so the only
// shared-memory operand traffic is Q, K and V.
//
// Shared memory (1024-byte aligned, 128-byte swizzled tiles):
//   Q 32 KB | K ring 2 x 32 KB | V ring 2 x 32 KB | control.
// TMEM (512 columns): O [0,128), S/P buffers b = t mod 3 at [128 + 128 b, 256 + 128 b).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace solattn {

constexpr int kMaxMaskWords = 512;       // N <= 16384 pooled blocks per head

// Optional per-role cycle accounting (build with -DSOL_ATTN_PROFILE): every
// bounded wait and the softmax phases add their clock64() cycles to a slot;
// the per-CTA totals are summed into g_profile at exit.
enum ProfSlot : int {
  kPrRouteWait, kPrKDesc, kPrKQEmpty, kPrKEmpty, kPrVDesc, kPrVEmpty,
  kPrMmaP, kPrMmaV, kPrMmaDesc, kPrMmaQ, kPrMmaSEmpty, kPrMmaK,
  kPrSmDesc, kPrSmS, kPrSmO, kPrSmX,
  kPrTotRoute, kPrTotK, kPrTotV, kPrTotMma, kPrTotSm,
  kPrSmPass1, kPrSmRescale, kPrSmPass2, kPrSmEpi, kPrSmTiles, kPrSmRescales, kPrSchedItem, kPrSchedRing,
  kPrTotSched, kPrSmRedo, kPrMmaIssueS, kPrMmaIssuePV, kPrSlots
};
constexpr int kProfileSlots = 48;
static_assert(kPrSlots <= kProfileSlots, "profile slots");
#ifdef SOL_ATTN_PROFILE
__device__ unsigned long long g_profile[kProfileSlots];
#define SA_PROF(x) x
#else
#define SA_PROF(x)
#endif
constexpr unsigned kFlagSelectAll = 1u;
constexpr unsigned kFlagExactOnly = 2u;
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusDevice = 2u;

struct FusedParams {
  int BH, L, N, W;          // W: approximation tile width (MMA N), 32 or 64
  int chunk;                // window of the tile walk: max(C, 64) pooled keys
  int num_pairs, num_items;
  unsigned flags;
  float scale_log2;         // log2(e) / sqrt(d)
  float inv_sqrt_d;
  float tail_raw;           // (log2(n_tail) - 6) / scale_log2: logit shift of the ragged block's approximation
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

constexpr int kStages = 2;

// One entry of the tile sequence, published by the scheduler warp.
struct __align__(16) TileDesc {
  uint32_t bits[2][4];  // [half][32-column group]: columns that take part for that half's rows
  int ja, jb;           // approximation: first pooled key; exact: key blocks (jb = -1: one block)
  int bh, pair;         // work item
  int ncols;            // 32, 64 or 128 (MMA N of S, K of PV)
  int flags;            // kDesc* bits
  int tail;             // column of the ragged block's approximation (weight n_tail), or -1
  int pad;
};
constexpr int kDescFirst = 1;    // first tile of its item (PV overwrites O)
constexpr int kDescLast = 2;     // last tile of its item
constexpr int kDescApprox = 4;   // approximation tile (else exact)
constexpr int kDescEmpty = 8;    // item without any tile (exact-only, nothing selected)
constexpr int kDescEnd = 16;     // no more work
constexpr int kRing = 8;         // descriptor ring entries

struct __align__(16) ItemSlot {
  uint32_t mask[2][kMaxMaskWords];  // selection bits of both halves
  int item;                         // work item index, or -1 = no more work
  int no_tiles;                     // exact-only item with nothing selected: no tile at all
  int pad[2];
};

struct __align__(16) FusedCtl {
  ItemSlot slot[2];
  TileDesc ring[kRing];             // scheduler -> producers, MMA issuer, softmax
  float qbar[2][128];               // routing: pooled queries of the pair
  uint64_t item_full[2], item_empty[2];
  uint64_t ring_full[kRing], ring_empty[kRing];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages];         // K-side stage loaded (its reuse waits for the S MMA: s_full)
  uint64_t v_full[kStages];         // V-side stage loaded (its reuse waits for the PV MMA: pv_done)
  uint64_t s_full[3], p_full[3];    // per TMEM S buffer (tile index % 3)
  uint64_t pv_done[3];              // per TMEM S buffer: its PV completed
  uint64_t xchg;                    // softmax warpgroups: partial row max / sum exchange
  float xval[2][2][128];            // [phase parity][warpgroup][row]
  uint32_t tmem_base;
  int abort;
};
static_assert(offsetof(FusedCtl, qbar) % 16 == 0, "float4 access to qbar");
static_assert(offsetof(FusedCtl, item_full) % 8 == 0, "mbarrier alignment");

constexpr uint32_t kTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kTile;
constexpr uint32_t kSmemV = kSmemK + kStages * kTile;
constexpr uint32_t kSmemCtl = kSmemV + kStages * kTile;
constexpr uint32_t kFusedSmemBytes = kSmemCtl + sizeof(FusedCtl) + 1024;  // + alignment slack
static_assert(kFusedSmemBytes <= 227u * 1024u, "dynamic shared memory of one CTA on sm_100");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS0 = 128;    // O at [0, 128), S / P buffer b at 128 + 128 b (b < 3)
constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;   // two warpgroups, each owning half of every tile's columns
constexpr uint32_t kRingEmptyCount = 8 + 3;  // softmax warps (lane 0 each) + K producer + V producer + MMA

__device__ __forceinline__ bool mask_bit(const uint32_t* m, int j) { return (m[j >> 5] >> (j & 31)) & 1u; }

// 32 selection bits starting at block j0 (bits past nw words read as 0).
__device__ __forceinline__ uint32_t mask_bits32(const uint32_t* m, int j0, int nw) {
  const int w = j0 >> 5, sh = j0 & 31;
  uint32_t r = (w < nw) ? (m[w] >> sh) : 0u;
  if (sh && w + 1 < nw) r |= m[w + 1] << (32 - sh);
  return r;
}

struct Tile {
  int kind;    // 0 approximation, 1 exact
  int ja, jb;  // approx: first pooled key; exact: the one or two key blocks (jb = -1: one)
  int ncols;   // MMA N of S / K of PV
  int avalid;  // approx: valid columns (rest of the tile belongs to no chunk)
  bool first;  // first tile of its item (PV overwrites O)
};

// Walks an item's tile sequence, one chunk of C pooled keys at a time: the
// union of the selected blocks, two per tile, then the chunk's approximation
// sub-tiles (skipped when both halves selected every block in them).  The walk
// starts at the chunk that holds the item's own query blocks, and inside that
// chunk at block i0, then wraps around.  The online softmax is independent of
// the order of its tiles up to rounding; starting near the diagonal makes the
// first tiles carry each row's largest logits, so the running maximum rarely
// moves afterwards.  Run by the scheduler warp.
struct TileIter {
  const uint32_t* m0;
  const uint32_t* m1;
  int N, C, W;
  int nw;           // mask words per half
  bool has1, exact_only, first;
  int lo, hi;       // current chunk [lo, hi)
  int jstart;       // the chunk's exact blocks run over [jstart, hi) then [lo, jstart)
  int seg;          // 0, 1: position in those two ranges; 2: exact blocks done
  int j;            // next candidate block of the current range
  int a0;           // next approximation sub-tile start
  int chunks_left;

  // First block of the union of both selections in [from, lim), or lim.
  __device__ __forceinline__ int next_union(int from, int lim) const {
    int x = from;
    while (x < lim) {
      const int w = x >> 5;
      const uint32_t u = (m0[w] | m1[w]) & (0xFFFFFFFFu << (x & 31));
      if (u) {
        const int jj = (w << 5) + __ffs(u) - 1;
        return jj < lim ? jj : lim;
      }
      x = (w + 1) << 5;
    }
    return lim;
  }
  // Next selected block of the current chunk in its exact order, or -1.
  __device__ __forceinline__ int next_exact() {
    while (seg < 2) {
      const int lim = seg == 0 ? hi : jstart;
      const int jj = next_union(j, lim);
      if (jj < lim) {
        j = jj + 1;
        return jj;
      }
      ++seg;
      j = lo;
    }
    return -1;
  }
  __device__ __forceinline__ void start_chunk(int start) {
    hi = min(lo + C, N);
    jstart = start;
    seg = 0;
    j = start;
    a0 = exact_only ? hi : lo;
  }
  __device__ __forceinline__ void init(const ItemSlot& s, int N_, int C_, int W_, int i0, bool has1_,
                                       bool exact_only_) {
    m0 = s.mask[0];
    m1 = s.mask[1];
    N = N_;
    C = C_;
    W = W_;
    nw = (N_ + 31) >> 5;
    has1 = has1_;
    exact_only = exact_only_;
    first = true;
    chunks_left = (N_ + C_ - 1) / C_;
    lo = (i0 / C_) * C_;
    start_chunk(i0);
  }
  __device__ __forceinline__ bool next(Tile& t) {
    while (chunks_left > 0) {
      const int ja = next_exact();
      if (ja >= 0) {
        const int jb = next_exact();
        t = (jb >= 0) ? Tile{1, ja, jb, 128, 0, first} : Tile{1, ja, -1, 64, 0, first};
        first = false;
        return true;
      }
      while (a0 < hi) {
        const int a1 = min(a0 + W, hi);
        const int s = a0;
        a0 = a1;
        bool any = false;
        for (int x = s; x < a1 && !any; x += 32) {
          const int n = min(32, a1 - x);
          const uint32_t range = (n >= 32) ? 0xFFFFFFFFu : ((1u << n) - 1u);
          uint32_t unsel = ~mask_bits32(m0, x, nw);
          if (has1) unsel |= ~mask_bits32(m1, x, nw);
          any = (unsel & range) != 0u;
        }
        if (any) {
          t = Tile{0, s, -1, W, a1 - s, first};
          first = false;
          return true;
        }
      }
      if (--chunks_left > 0) {
        lo = (hi >= N) ? 0 : hi;
        start_chunk(lo);
      }
    }
    return false;
  }
};


// Bounded wait for an mbarrier phase after a failed first probe; on a timeout
// it raises the abort flag and the status word.
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned* status,
                                       unsigned long long timeout_ns) {
  if (mbar_wait(bar, parity, abort, timeout_ns)) return true;
  *abort = 1;
  atomicOr(status, kStatusTimeout);
  return false;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sol_attn_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
                          const __grid_constant__ CUtensorMap tm_kl, const __grid_constant__ CUtensorMap tm_vb,
                          const FusedParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled tiles.  Offsetting the shared array
  // itself (not a round trip through an integer) keeps every pointer below in
  // the shared state space, so accesses compile to shared-memory instructions.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sK = smem + kSmemK;
  uint8_t* sV = smem + kSmemV;
  FusedCtl& ctl = *reinterpret_cast<FusedCtl*>(smem + kSmemCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int KSTEPS = D / 16;           // MMA K-steps over the head dimension
  constexpr uint32_t CB = 16384;           // bytes per 64-column block of a 128-row tile
  volatile int* abort_flag = &ctl.abort;
  const bool exact_only = (p.flags & kFlagExactOnly) != 0;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl.item_full[s], 1);
      mbar_init(&ctl.item_empty[s], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&ctl.s_full[b], 1);
      mbar_init(&ctl.p_full[b], kSoftmaxThreads);
    }
    for (int b = 0; b < 3; ++b) mbar_init(&ctl.pv_done[b], 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&ctl.ring_full[r], 1);
      mbar_init(&ctl.ring_empty[r], kRingEmptyCount);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.k_full[s], 1);
      mbar_init(&ctl.v_full[s], 1);
    }
    mbar_init(&ctl.q_full, 1);
    mbar_init(&ctl.q_empty, 1);
    mbar_init(&ctl.xchg, kSoftmaxThreads / 32);   // one arrival per softmax warp
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  // Bounded wait; on a timeout raise the abort flag and the status word.  All
  // later waits return false at once, every role leaves its loop, and the CTA
  // meets at the final barrier.
  SA_PROF(unsigned long long prof[kPrSlots]; for (int i = 0; i < kPrSlots; ++i) prof[i] = 0;
          const unsigned long long prof_t0 = clock64();)
  // The first probe is inline; the sleeping loop behind it is out of line,
  // which keeps every wait site small.
  auto wait = [&](uint64_t* bar, uint32_t parity, int slot) -> bool {
    SA_PROF(const unsigned long long tw = clock64();)
    const bool okw = mbar_try_wait(bar, parity) || wait_slow(bar, parity, abort_flag, p.status, p.timeout_ns);
    SA_PROF(prof[slot] += clock64() - tw;)
    (void)slot;
    return okw;
  };
  // Consumer side of the descriptor ring: descriptor r lives in slot r % kRing.
  auto ring_get = [&](uint32_t r, int slot) -> bool {
    return wait(&ctl.ring_full[r % kRing], (r / kRing) & 1, slot);
  };

  if (warp == 10) {
    // =========================================================== routing
    for (int seq = 0;; ++seq) {
      const int s = seq & 1;
      if (seq >= 2 && !wait(&ctl.item_empty[s], ((seq >> 1) - 1) & 1, kPrRouteWait)) break;
      int item = 0;
      if (lane == 0) item = static_cast<int>(atomicAdd(p.work_counter, 1u));
      item = __shfl_sync(0xFFFFFFFFu, item, 0);
      ItemSlot& sl = ctl.slot[s];
      if (item >= p.num_items) {
        if (lane == 0) {
          sl.item = -1;
          mbar_arrive(&ctl.item_full[s]);
        }
        break;
      }
      const int bh = item / p.num_pairs;
      const int pair = item - bh * p.num_pairs;
      const int i0 = 2 * pair, i1 = 2 * pair + 1;
      const bool has1 = i1 < p.N;
      const float* qb = p.qbar + static_cast<size_t>(bh) * p.N * D;
      const float* kb = p.kbar + static_cast<size_t>(bh) * p.N * D;
      for (int e = lane; e < 2 * D; e += 32) {
        const int h = e / D, c = e % D;
        const int i = h ? i1 : i0;
        ctl.qbar[h][c] = (i < p.N) ? qb[static_cast<size_t>(i) * D + c] : 0.f;
      }
      __syncwarp();
      const float tau0 = p.tau[static_cast<size_t>(bh) * p.N + i0];
      const float tau1 = has1 ? p.tau[static_cast<size_t>(bh) * p.N + i1] : INFINITY;
      const int NW = (p.N + 31) >> 5;
      int cnt0 = 0, cnt1 = 0;
      for (int g = 0; g < NW; ++g) {
        const int j = 32 * g + lane;
        bool s0 = false, s1 = false;
        if (j < p.N) {
          const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D);
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll 2
          for (int c4 = 0; c4 < D / 4; ++c4) {
            const float4 x = __ldg(kr + c4);
            const float4 qa = *reinterpret_cast<const float4*>(&ctl.qbar[0][4 * c4]);
            const float4 qb4 = *reinterpret_cast<const float4*>(&ctl.qbar[1][4 * c4]);
            a0 = fmaf(qa.x, x.x, a0); a1 = fmaf(qa.y, x.y, a1); a2 = fmaf(qa.z, x.z, a2); a3 = fmaf(qa.w, x.w, a3);
            b0 = fmaf(qb4.x, x.x, b0); b1 = fmaf(qb4.y, x.y, b1); b2 = fmaf(qb4.z, x.z, b2); b3 = fmaf(qb4.w, x.w, b3);
          }
          const float d0 = (a0 + a1) + (a2 + a3);
          const float d1 = (b0 + b1) + (b2 + b3);
          s0 = d0 * p.inv_sqrt_d >= tau0;
          s1 = has1 && (d1 * p.inv_sqrt_d >= tau1);
        }
        const uint32_t m0 = __ballot_sync(0xFFFFFFFFu, s0);
        const uint32_t m1 = __ballot_sync(0xFFFFFFFFu, s1);
        if (lane == 0) {
          sl.mask[0][g] = m0;
          sl.mask[1][g] = m1;
        }
        cnt0 += __popc(m0);
        cnt1 += __popc(m1);
      }
      if (lane == 0) {
        p.counts[static_cast<size_t>(bh) * p.N + i0] = cnt0;
        if (has1) p.counts[static_cast<size_t>(bh) * p.N + i1] = cnt1;
        sl.item = item;
        sl.no_tiles = exact_only && (cnt0 + cnt1 == 0);
      }
      __syncwarp();
      if (p.mask_out) {
        for (int e = lane; e < 2 * NW; e += 32) {
          const int h = e / NW, g = e % NW;
          const int i = h ? i1 : i0;
          if (i < p.N) p.mask_out[(static_cast<size_t>(bh) * p.N + i) * NW + g] = sl.mask[h][g];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.item_full[s]);   // release: masks and item visible
    }
  } else if (warp == 11) {
    // =========================================================== scheduler
    uint32_t r = 0;   // descriptors published
    const int NW = (p.N + 31) >> 5;
    // Claim ring slot r (all consumers are done with descriptor r - kRing).
    auto claim = [&]() -> TileDesc* {
      if (r >= kRing && !wait(&ctl.ring_empty[r % kRing], ((r / kRing) - 1) & 1, kPrSchedRing)) return nullptr;
      return &ctl.ring[r % kRing];
    };
    auto publish = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.ring_full[r % kRing]);   // release: descriptor visible
      ++r;
    };
    for (int seq = 0;; ++seq) {
      const int s = seq & 1;
      if (!wait(&ctl.item_full[s], (seq >> 1) & 1, kPrSchedItem)) break;
      const ItemSlot& sl = ctl.slot[s];
      const int item = sl.item;
      TileDesc* dsc = claim();
      if (!dsc) break;
      if (item < 0) {
        if (lane == 0) dsc->flags = kDescEnd;
        publish();
        break;
      }
      const int bh = item / p.num_pairs;
      const int pair = item - bh * p.num_pairs;
      if (sl.no_tiles) {
        if (lane == 0) {
          dsc->bh = bh;
          dsc->pair = pair;
          dsc->flags = kDescEmpty;
        }
        publish();
      } else {
        TileIter it;
        it.init(sl, p.N, p.chunk, p.W, 2 * pair, 2 * pair + 1 < p.N, exact_only);
        Tile t, tn;
        bool have = it.next(t);
        bool first_desc = true;
        while (have) {
          const bool have_next = it.next(tn);
          if (!first_desc && !(dsc = claim())) break;
          first_desc = false;
          // lanes 0-7 each compute one (half, 32-column group) validity word
          if (lane < 8) {
            const int g = lane >> 1, h = lane & 1;
            uint32_t bits = 0u;
            if (32 * g < t.ncols) {
              if (t.kind == 0) {
                const int nv = min(max(t.avalid - 32 * g, 0), 32);
                const uint32_t range = (nv >= 32) ? 0xFFFFFFFFu : ((1u << nv) - 1u);
                bits = range & ~mask_bits32(sl.mask[h], t.ja + 32 * g, NW);
              } else {
                const int jx = (g < 2) ? t.ja : t.jb;
                const int nv = min(max(p.L - (64 * jx + 32 * (g & 1)), 0), 32);
                const uint32_t range = (nv >= 32) ? 0xFFFFFFFFu : ((1u << nv) - 1u);
                bits = mask_bit(sl.mask[h], jx) ? range : 0u;
              }
            }
            dsc->bits[h][g] = bits;
          } else if (lane == 8) {
            const int tail_col = (t.kind == 0 && p.L - 64 * (p.N - 1) != 64) ? (p.N - 1 - t.ja) : -1;
            dsc->ja = t.ja;
            dsc->jb = t.jb;
            dsc->bh = bh;
            dsc->pair = pair;
            dsc->ncols = t.ncols;
            dsc->flags = (t.first ? kDescFirst : 0) | (have_next ? 0 : kDescLast) | (t.kind == 0 ? kDescApprox : 0);
            dsc->tail = (tail_col >= 0 && tail_col < t.ncols) ? tail_col : -1;
          }
          publish();
          t = tn;
          have = have_next;
        }
        if (have) break;   // left early on a timeout
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.item_empty[s]);   // the item's masks are no longer read
    }
  } else if (warp == 8) {
    // =========================================================== TMA producers
    const bool kside = (lane == 0);
    if (lane < 2) {
      int stage = 0;
      uint32_t tl = 0;     // tiles loaded
      uint32_t qseq = 0;   // items with tiles seen (K side loads their Q tiles)
      for (uint32_t r = 0;; ++r) {
        if (!ring_get(r, kside ? kPrKDesc : kPrVDesc)) break;
        const TileDesc& dsc = ctl.ring[r % kRing];
        const int flags = dsc.flags, ja = dsc.ja, jb = dsc.jb, bh = dsc.bh, pair = dsc.pair;
        mbar_arrive(&ctl.ring_empty[r % kRing]);
        if (flags & kDescEnd) break;
        if (flags & kDescEmpty) continue;
        if (kside && (flags & kDescFirst)) {  // the item's query tile (the previous item's S MMAs must be done)
          if (qseq > 0 && !wait(&ctl.q_empty, (qseq - 1) & 1, kPrKQEmpty)) break;
          mbar_arrive_expect_tx(&ctl.q_full, 128u * D * 2u);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(sQ + cb * CB, &tm_q, &ctl.q_full, cb * 64, 128 * pair, bh);
          ++qseq;
        }
        // The stage was last used by tile tl - kStages; it is free once that
        // tile's S MMA (K side) or PV MMA (V side) has completed, which the
        // barriers of its TMEM buffer (tl - kStages) % 3 record.
        uint64_t* full = kside ? &ctl.k_full[stage] : &ctl.v_full[stage];
        if (tl >= kStages) {
          const uint32_t tp = tl - kStages;
          uint64_t* done = kside ? &ctl.s_full[tp % 3u] : &ctl.pv_done[tp % 3u];
          if (!wait(done, (tp / 3u) & 1u, kside ? kPrKEmpty : kPrVEmpty)) break;
        }
        ++tl;
        uint8_t* dst = (kside ? sK : sV) + stage * kTile;
        if (flags & kDescApprox) {
          mbar_arrive_expect_tx(full, (kside ? 2u : 1u) * p.W * D * 2u);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            if (kside) {
              tma_load_3d(dst + cb * CB, &tm_kb, full, cb * 64, ja, bh);
              tma_load_3d(dst + cb * CB + 8192, &tm_kl, full, cb * 64, ja, bh);
            } else {
              tma_load_3d(dst + cb * CB, &tm_vb, full, cb * 64, ja, bh);
            }
          }
        } else {
          const int nblk = (jb >= 0) ? 2 : 1;
          mbar_arrive_expect_tx(full, static_cast<uint32_t>(nblk) * 64u * D * 2u);
          const CUtensorMap* map = kside ? &tm_k : &tm_v;
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            tma_load_3d(dst + cb * CB, map, full, cb * 64, 64 * ja, bh);
            if (nblk == 2) tma_load_3d(dst + cb * CB + 8192, map, full, cb * 64, 64 * jb, bh);
          }
        }
        if (++stage == kStages) stage = 0;
      }
    }
  } else if (warp == 9) {
    // =========================================================== MMA issuer
    // S(t) goes into TMEM buffer t % 3 and runs up to two tiles ahead of the
    // PVs: for tile t this thread issues PV(t-2), then S(t) once PV(t-3), the
    // last reader of the buffer, has completed.  PV(t-2) and S(t-1) sit
    // between the two in the tensor pipe, so that wait rarely stalls it.
    if (lane == 0) {
      const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 1);
      int kstage = 0, vstage = 0;
      uint32_t kphase = 0, vphase = 0;
      uint32_t tcount = 0;           // tiles whose S MMA is issued
      uint32_t qseq = 0;             // items with tiles seen
      struct PendingPv {
        uint32_t t, vphase;
        int ncols, vstage;
        bool first;
      };
      PendingPv pend[2];
      int npend = 0;
      bool ok = true;
      // O (+)= P(t) · Vside(t), P read from TMEM buffer t % 3.  Softmax warpgroup
      // w wrote the P of the tile's columns [w h, (w + 1) h), h = ncols / 2 (all
      // 32 columns of a 32-column tile: warpgroup 0), as bf16 pairs starting at
      // the buffer's column w h.
      auto issue_pv = [&](const PendingPv& pv) -> bool {
        const uint32_t b = pv.t % 3u;
        if (!wait(&ctl.p_full[b], (pv.t / 3u) & 1u, kPrMmaP)) return false;
        if (!wait(&ctl.v_full[pv.vstage], pv.vphase, kPrMmaV)) return false;
        tc_fence_after();
        SA_PROF(const unsigned long long tis = clock64();)
        // descriptors are linear in the address: + (bytes >> 4) moves them
        const uint64_t vdesc = sdesc_sw128(sVa + pv.vstage * kTile, CB, 1024);
        const uint32_t pbase = tmem + kTmemS0 + 128u * b;
        const uint32_t acc0 = pv.first ? 0u : 1u;
        // K-step kk (keys 16 kk ..): P column 8 kk, + ncols / 4 for the second
        // warpgroup's keys (a 32-column tile has only the first's)
        if (pv.ncols == 128) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tmem + kTmemO, pbase + 8 * kk + (kk >= 4 ? 32 : 0), vdesc + 128 * kk, idesc_pv,
                    kk == 0 ? acc0 : 1u);
        } else if (pv.ncols == 64) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + kTmemO, pbase + 8 * kk + (kk >= 2 ? 16 : 0), vdesc + 128 * kk, idesc_pv,
                    kk == 0 ? acc0 : 1u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_ts(tmem + kTmemO, pbase + 8 * kk, vdesc + 128 * kk, idesc_pv, kk == 0 ? acc0 : 1u);
        }
        umma_commit(&ctl.pv_done[b]);
        SA_PROF(prof[kPrMmaIssuePV] += clock64() - tis;)
        return true;
      };
      auto pop_pv = [&]() -> bool {
        const bool r = issue_pv(pend[0]);
        pend[0] = pend[1];
        --npend;
        return r;
      };
      for (uint32_t r = 0;; ++r) {
        if (!ring_get(r, kPrMmaDesc)) { ok = false; break; }
        const TileDesc& dsc = ctl.ring[r % kRing];
        const int flags = dsc.flags, ncols = dsc.ncols;
        mbar_arrive(&ctl.ring_empty[r % kRing]);
        if (flags & kDescEnd) break;
        if (flags & kDescEmpty) continue;
        if (npend == 2 && !pop_pv()) { ok = false; break; }   // PV(t-2)
        const uint32_t b = tcount % 3u;
        if (tcount >= 3 && !wait(&ctl.pv_done[b], ((tcount / 3u) - 1u) & 1u, kPrMmaSEmpty)) { ok = false; break; }
        if (flags & kDescFirst) {
          if (!wait(&ctl.q_full, qseq & 1, kPrMmaQ)) { ok = false; break; }
        }
        if (!wait(&ctl.k_full[kstage], kphase, kPrMmaK)) { ok = false; break; }
        tc_fence_after();
        SA_PROF(const unsigned long long tis = clock64();)
        // S(t) = Q · Kside^T into buffer t % 3
        const uint32_t dS = tmem + kTmemS0 + 128u * b;
        const uint64_t kdesc = sdesc_sw128(sKa + kstage * kTile, 16, 1024);
        const uint32_t idesc_s = idesc_bf16_f32(128, ncols, 0);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t koff = ((kk >> 2) * CB + (kk & 3) * 32) >> 4;
          umma_ss(dS, qdesc + koff, kdesc + koff, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (flags & kDescApprox) {  // + Q · K̄_lo^T (rows 64.. of the K-side tile)
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            const uint32_t koff = ((kk >> 2) * CB + (kk & 3) * 32) >> 4;
            umma_ss(dS, qdesc + koff, kdesc + (8192 >> 4) + koff, idesc_s, 1u);
          }
        }
        umma_commit(&ctl.s_full[b]);
        SA_PROF(prof[kPrMmaIssueS] += clock64() - tis;)
        if (++kstage == kStages) {
          kstage = 0;
          kphase ^= 1u;
        }
        if (flags & kDescLast) {  // every S MMA of this item is issued: Q is free once they complete
          umma_commit(&ctl.q_empty);
          ++qseq;
        }
        pend[npend++] = PendingPv{tcount, vphase, ncols, vstage, (flags & kDescFirst) != 0};
        if (++vstage == kStages) {
          vstage = 0;
          vphase ^= 1u;
        }
        ++tcount;
      }
      while (ok && npend > 0) ok = pop_pv();
    }
  } else {
    // =========================================================== softmax (warps 0-7)
    // Both warpgroups work on every tile: the thread of warpgroup wg and TMEM
    // lane `row` owns tile row `row` and the tile's columns [wg h, (wg + 1) h),
    // h = ncols / 2 (a 32-column tile belongs to warpgroup 0 alone).  The two
    // threads of a row share one reference maximum m (log2 units) and keep
    // partial row sums l; P of the tile accumulates into the single O.
    const int wg = warp >> 2;
    const int row = tid & 127;        // tile row = TMEM lane
    const int half = row >> 6;        // query block of the pair the row belongs to
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + kTmemO + lane_base;
    uint32_t tcount = 0;     // tiles processed (S buffer tcount % 3, PV index tcount)
    uint32_t xc = 0;         // exchanges done
    // Exchange one value per row with the other warpgroup's thread of the row.
    auto exchange = [&](float a) -> float {
      const int ph = xc & 1;
      ctl.xval[ph][wg][row] = a;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.xchg);
      wait(&ctl.xchg, ph, kPrSmX);
      ++xc;
      return ctl.xval[ph][wg ^ 1][row];
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool item_tiles = false;  // the current item had a tile
    for (uint32_t r = 0;; ++r) {
      if (!ring_get(r, kPrSmDesc)) break;
      const TileDesc& dsc = ctl.ring[r % kRing];
      const uint4 bw = *reinterpret_cast<const uint4*>(dsc.bits[half]);
      const int ncols = dsc.ncols, dflags = dsc.flags, tail_col = dsc.tail, dbh = dsc.bh, dpair = dsc.pair;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.ring_empty[r % kRing]);
      if (dflags & kDescEnd) break;
      if (!(dflags & kDescEmpty)) {
        const uint32_t t = tcount++;
        const uint32_t b = t % 3u;
        wait(&ctl.s_full[b], (t / 3u) & 1u, kPrSmS);
        tc_fence_after();
        SA_PROF(unsigned long long tph = clock64(); prof[kPrSmTiles] += 1;)
        const bool first = (dflags & kDescFirst) != 0;
        if (first) {
          m_run = -INFINITY;
          l_run = 0.f;
        }
        item_tiles = true;
        const int hw = (ncols == 32) ? (wg == 0 ? 32 : 0) : (ncols >> 1);   // this thread's columns
        const int c0 = (ncols == 32) ? 0 : wg * hw;                           // their first column
        const int ng = hw >> 5;                                               // 32-column groups: 0, 1, 2
        const uint32_t tS = tmem + kTmemS0 + 128u * b + lane_base;
        auto gb = [&](int i) -> uint32_t { return i == 0 ? bw.x : i == 1 ? bw.y : i == 2 ? bw.z : bw.w; };
        // Column adjustments, only where needed: invalid columns become -inf,
        // the ragged block's approximation column gets log2(n_tail / 64).
        const int tail_g = tail_col >= 0 ? (tail_col >> 5) : -1;
        auto adjust = [&](float* xv, int g) {
          const uint32_t bits = gb(g);
          const int et = (g == tail_g) ? (tail_col & 31) : -1;
          if (bits != 0xFFFFFFFFu || et >= 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e == et) xv[e] += p.tail_raw;
              if (!((bits >> e) & 1u)) xv[e] = -INFINITY;
            }
          }
        };
        // In log2 units.  An approximation column stands for its n_j tokens:
        // its weight n_j is folded into the logit as + log2(n_j) (6 for a full
        // block) and the value side uses the block mean V̂_j / n_j.
        const float boost = (dflags & kDescApprox) ? 6.f : 0.f;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        // p = 2^y, y = x * scale_log2 + off, for 32 adjusted columns, packed as
        // 16 bf16 pairs; the fp32 values go into the row sum (ra, rb) and the
        // largest y into ym.
        auto probs32 = [&](const float* xv, float2 of2, uint32_t* pk, float2& ra, float2& rb, float& ym) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const float2 y0 = __ffma2_rn(make_float2(xv[e], xv[e + 1]), sc2, of2);
            const float2 y1 = __ffma2_rn(make_float2(xv[e + 2], xv[e + 3]), sc2, of2);
            const float2 y2 = __ffma2_rn(make_float2(xv[e + 4], xv[e + 5]), sc2, of2);
            const float2 y3 = __ffma2_rn(make_float2(xv[e + 6], xv[e + 7]), sc2, of2);
            ym = max3f(ym, max3f(y0.x, y0.y, y1.x), max3f(y1.y, y2.x, y2.y));
            ym = max3f(ym, y3.x, y3.y);
            const float2 q0 = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
            const float2 q1 = make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
            const float2 q2 = make_float2(ex2_approx(y2.x), ex2_approx(y2.y));
            const float2 q3 = make_float2(ex2_approx(y3.x), ex2_approx(y3.y));
            ra = __fadd2_rn(ra, __fadd2_rn(q0, q2));
            rb = __fadd2_rn(rb, __fadd2_rn(q1, q3));
            pk[e >> 1] = pack_bf16x2(q0.x, q0.y);
            pk[(e >> 1) + 1] = pack_bf16x2(q1.x, q1.y);
            pk[(e >> 1) + 2] = pack_bf16x2(q2.x, q2.y);
            pk[(e >> 1) + 3] = pack_bf16x2(q3.x, q3.y);
          }
        };
        // This thread's columns, against the reference maximum mref: P into
        // pk[0, 16 ng), the row sum into (ra, rb); returns the largest y.
        auto own_cols = [&](float mref, uint32_t* pk, float2& ra, float2& rb) -> float {
          const float2 of2 = make_float2(boost - mref, boost - mref);
          float ym = -INFINITY;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (i < ng) {
              float xv[32];
              tmem_ld_x32f(tS + c0 + 32 * i, xv);
              tmem_ld_wait();
              reg_fence32(xv);
              adjust(xv, (c0 >> 5) + i);
              probs32(xv, of2, pk + 16 * i, ra, rb, ym);
            }
          }
          return ym;
        };
        // One pass against the row's reference maximum m (0 while the row has
        // seen no valid column), P held in registers.  Each thread proposes the
        // m it needs: m itself while its y stay <= 8 (the lazy rescale rule),
        // else m raised by a whole number k of doublings (so that everything
        // accumulated so far scales by 2^-k exactly, even P already in bf16),
        // or its maximum rounded up on the row's first valid column.  The two
        // threads of the row agree on the larger proposal; where it moved, l
        // and this thread's half of O scale by 2^(m - m') and the columns are
        // recomputed from S, which no P store has reached yet.
        uint32_t pk[32];
        float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
        const float ym = own_cols(m_run == -INFINITY ? 0.f : m_run, pk, sa, sb);
        // m stays a whole number (its first value is rounded up), so that every
        // later step m' - m is exact in fp32
        const float prop = (m_run == -INFINITY) ? ceilf(ym) : (ym > 8.f ? m_run + ceilf(ym) : m_run);
        const float m_new = fmaxf(prop, exchange(prop));
        const bool moved = !(m_new == m_run);
        if (__any_sync(0xFFFFFFFFu, moved)) {
          SA_PROF(prof[kPrSmRedo] += 1;)
          float alpha = 1.f;
          if (moved) {
            if (m_run == -INFINITY) {
              alpha = 0.f;   // nothing valid accumulated yet
            } else {
              const int k = __float2int_rn(m_new - m_run);
              alpha = (k >= 126) ? 0.f : __int_as_float((127 - k) << 23);
            }
            l_run *= alpha;
            m_run = m_new;
          }
          __syncwarp();
          if (!first) {
            // O holds PV(0 .. t-1) of the item; wait for PV(t-1), then scale this
            // thread's half of the row
            wait(&ctl.pv_done[(t - 1u) % 3u], ((t - 1u) / 3u) & 1u, kPrSmO);
            tc_fence_after();
#pragma unroll 1
            for (int c16 = wg * (D / 2); c16 < (wg + 1) * (D / 2); c16 += 16) {
              float rr[16];
              tmem_ld_x16f(tO + c16, rr);
              tmem_ld_wait();
              reg_fence16(rr);
              uint32_t pw[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) pw[e] = __float_as_uint(rr[e] * alpha);
              tmem_st_x16(tO + c16, pw);
            }
            SA_PROF(prof[kPrSmRescales] += 1;)
          }
          sa = make_float2(0.f, 0.f);
          sb = make_float2(0.f, 0.f);
          (void)own_cols(m_run == -INFINITY ? 0.f : m_run, pk, sa, sb);
        }
        // P of this thread's columns lands in TMEM columns [c0, c0 + hw / 2),
        // inside its own part of S, which it has read
        if (ng > 0) tmem_st_x16(tS + c0, pk);
        if (ng > 1) tmem_st_x16(tS + c0 + 16, pk + 16);
        l_run += (sa.x + sa.y) + (sb.x + sb.y);
        tmem_st_wait();
        SA_PROF(prof[kPrSmPass2] += clock64() - tph;)
        tc_fence_before();
        mbar_arrive(&ctl.p_full[b]);
      }
      if (!(dflags & (kDescLast | kDescEmpty))) continue;
      // ---- epilogue: O / (l_0 + l_1) for this thread's half of the row's columns
      SA_PROF(const unsigned long long tep = clock64();)
      if (item_tiles) {   // the item's last PV
        wait(&ctl.pv_done[(tcount - 1u) % 3u], ((tcount - 1u) / 3u) & 1u, kPrSmO);
        tc_fence_after();
      }
      const float my_l = item_tiles ? l_run : 0.f;
      const float l_tot = my_l + exchange(my_l);
      const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
      const int token = 128 * dpair + row;
      uint16_t* orow = p.out + (static_cast<size_t>(dbh) * p.L + token) * D;
#pragma unroll 1
      for (int c16 = wg * (D / 2); c16 < (wg + 1) * (D / 2); c16 += 16) {
        float a[16];
        if (item_tiles) {
          tmem_ld_x16f(tO + c16, a);
          tmem_ld_wait();
          reg_fence16(a);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) a[e] = 0.f;
        }
        if (token < p.L) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c16);
          dst[0] = make_uint4(pack_bf16x2(a[0] * inv_l, a[1] * inv_l), pack_bf16x2(a[2] * inv_l, a[3] * inv_l),
                              pack_bf16x2(a[4] * inv_l, a[5] * inv_l), pack_bf16x2(a[6] * inv_l, a[7] * inv_l));
          dst[1] = make_uint4(pack_bf16x2(a[8] * inv_l, a[9] * inv_l), pack_bf16x2(a[10] * inv_l, a[11] * inv_l),
                              pack_bf16x2(a[12] * inv_l, a[13] * inv_l), pack_bf16x2(a[14] * inv_l, a[15] * inv_l));
        }
      }
      // O is read; the next item's first PV (which overwrites O) waits for this
      // thread's next P arrival, which comes after these reads
      tc_fence_before();
      item_tiles = false;
      SA_PROF(prof[kPrSmEpi] += clock64() - tep;)
    }
  }

  SA_PROF({
    const int tslot = warp == 10 ? kPrTotRoute : warp == 11 ? kPrTotSched : warp == 9 ? kPrTotMma
                    : warp == 8 ? (lane == 0 ? kPrTotK : kPrTotV) : kPrTotSm;
    if ((lane == 0 && (warp >= 8 || warp == 0)) || (warp == 8 && lane == 1)) {
      prof[tslot] = clock64() - prof_t0;
      for (int i = 0; i < kPrSlots; ++i) if (prof[i]) atomicAdd(&g_profile[i], prof[i]);
    }
  })
  // After a timeout, give copies or MMAs that may still be in flight a bounded
  // time to land before the shared memory and TMEM are released.
  __syncwarp();
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
