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
// Warp roles (416 threads, one persistent CTA per SM, atomic work counter):
//   warps 0-7  softmax, two warpgroups that take the tiles in turns (tile t
//              belongs to warpgroup t & 1); the thread of TMEM lane r owns row
//              r of its warpgroup's tiles, all columns: row maximum, the
//              lazy-rescale decision, P = 2^(y - m) into TMEM, row sums.
//   warp 8     TMA producers: lane 0 loads Q and the K side (K blocks, or K̄
//              hi/lo), lane 1 the V side (V blocks, or V̄).
//   warp 9     tcgen05 issuer of the S MMAs (up to three tiles in flight).
//   warp 10    routing: fetches the next item, computes ŝ_ij = Q̄_i·K̄_j/sqrt(d)
//              in fp32 for both halves, compares with τ_i (warp ballot -> mask
//              words), one item ahead (double-buffered mask slots).
//   warp 11    scheduler: walks each item's tile sequence from its masks (the
//              union blocks of a chunk listed by all 32 lanes at once) and
//              publishes one descriptor per tile (blocks, column validity per
//              half, first/last flags) into a shared-memory ring that the
//              producers, both MMA issuers and the softmax warps consume.
//   warp 12    tcgen05 issuer of the PV MMAs (O += P·V, in tile order).
// S and PV have an issuer each: an MMA occupies its issuing thread for about
// its execution time, so one thread alternating between waiting for P and
// issuing leaves the tensor pipe idle between the two batches.
//
// Both warpgroups accumulate into one O per row, so they share the row's
// reference maximum m (log2 units, a whole number).  The owner of tile t
// computes P in one pass over its row, 32 columns at a time, against the m
// its own previous tile of the item settled on, raising it (lazy rescale)
// only when a group's maximum exceeds it by more than 8 (the groups already
// stored are scaled by the exact power of two).  At the end of the tile it
// meets the m that tile t - 1 settled on (shared memory, one mbarrier per
// hand-off slot): the larger wins, and this tile's P or O (after PV(t - 1)
// has completed), whichever is behind, is scaled by 2^-k.  Each thread keeps
// its partial row sum with the m it was accumulated at, and the two partials
// meet in the epilogue.  P is written back into TMEM over the consumed
// columns of its S tile (bf16 pairs) and fed to the PV MMA as its A operand,
// so the only shared-memory operand traffic is Q, K and V.
//
// Shared memory (1024-byte aligned, 128-byte swizzled tiles):
//   Q 32 KB | K ring 2 x 32 KB | V ring 3 x 32 KB | control.
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
  kPrSDesc, kPrSQ, kPrSBuf, kPrSK, kPrSIssue,
  kPrPvDesc, kPrPvP, kPrPvV, kPrPvIssue,
  kPrSmDesc, kPrSmS, kPrSmHand, kPrSmO, kPrSmX, kPrSmPass, kPrSmMeet, kPrSmEpi, kPrSmTiles, kPrSmRescales,
  kPrSchedItem, kPrSchedRing,
  kPrTotRoute, kPrTotK, kPrTotV, kPrTotS, kPrTotPv, kPrTotSm, kPrTotSched, kPrSmLd, kPrSmExp, kPrSchedNext, kPrSchedDesc, kPrRouteItem, kPrSlots
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
constexpr unsigned kFlagTestStall = 8u;    // routing publishes nothing: every role's wait runs out
constexpr unsigned kFlagFirstOrder = 16u;  // unselected blocks: first-order expansion on exact tiles
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusDevice = 2u;     // a tile descriptor failed its range check

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
constexpr int kStagesV = 3;   // V ring: a stage is free once the PV of its tile completed

// One entry of the tile sequence, published by the scheduler warp.
struct __align__(16) TileDesc {
  uint32_t bits[2][4];  // [half][32-column group]: columns that take part for that half's rows
  int ja, jb;           // approximation: first pooled key; exact: key blocks (jb = -1: one block)
  int bh, pair;         // work item
  int ncols;            // 32, 64 or 128 (MMA N of S, K of PV)
  int flags;            // kDesc* bits
  int tail;             // column of the ragged block's approximation (weight n_tail), or -1
  int selbits;          // first-order mode: bit 2 h + b set when half h selected block b of the tile
};
constexpr int kDescFirst = 1;    // first tile of its item (PV overwrites O)
constexpr int kDescLast = 2;     // last tile of its item
constexpr int kDescApprox = 4;   // approximation tile (else exact)
constexpr int kDescEmpty = 8;    // item without any tile (exact-only, nothing selected)
constexpr int kDescEnd = 16;     // no more work
constexpr int kRing = 8;         // descriptor ring entries
constexpr int kListPass = 1024;                 // blocks examined per listing pass
constexpr int kListCap = kListPass + 32;        // listed blocks held (a pass plus a leftover)


struct __align__(16) ItemSlot {
  uint32_t mask[2][kMaxMaskWords];  // selection bits of both halves
  int item;                         // work item index, or -1 = no more work
  int no_tiles;                     // exact-only item with nothing selected: no tile at all
  int pad[2];
};

struct __align__(16) FusedCtl {
  ItemSlot slot[2];
  TileDesc ring[kRing];             // scheduler -> producers, MMA issuers, softmax
  float qbar[2][128];               // routing: pooled queries of the pair
  uint16_t ulist[kListCap];         // scheduler: union blocks of the current chunk in walk order
  float hand[3][128];               // [tile % 3][row]: the m tile t settled on, read by tile t + 1
  float2 xval[2][2][128];           // epilogue: [parity][warpgroup][row] partial (row sum, its m)
  uint64_t item_full[2], item_empty[2];
  uint64_t ring_full[kRing], ring_empty[kRing];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages];         // K-side stage loaded (its reuse waits for the S MMA: s_full)
  uint64_t v_full[kStagesV];        // V-side stage loaded (its reuse waits for the PV MMA: pv_done)
  uint64_t s_full[3], p_full[3];    // per TMEM S buffer (tile index % 3)
  uint64_t pv_done[3];              // per TMEM S buffer: its PV completed
  uint64_t mready[3];               // per TMEM S buffer: hand[] of that tile written
  uint64_t xchg;                    // softmax warpgroups: epilogue exchange
  uint32_t tmem_base;
  int abort;
};
static_assert(offsetof(FusedCtl, qbar) % 16 == 0, "float4 access to qbar");
static_assert(offsetof(FusedCtl, item_full) % 8 == 0, "mbarrier alignment");

constexpr uint32_t kTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kTile;
constexpr uint32_t kSmemV = kSmemK + kStages * kTile;
constexpr uint32_t kSmemCtl = kSmemV + kStagesV * kTile;
constexpr uint32_t kFusedSmemBytes = kSmemCtl + sizeof(FusedCtl) + 1024;  // + alignment slack
static_assert(kFusedSmemBytes <= 227u * 1024u, "dynamic shared memory of one CTA on sm_100");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS0 = 128;    // O at [0, 128), S / P buffer b at 128 + 128 b (b < 3)
constexpr int kThreads = 416;                    // 13 warps
// Registers: the 13 warps sit 4-3-3-3 on the SM's four sub-partitions, each
// with a quarter of the register file, so a thread may hold at most 128.
constexpr int kLaunchBoundThreads = 512;
constexpr int kWarpLoad = 8, kWarpS = 9, kWarpRoute = 10, kWarpSched = 11, kWarpPv = 12;
constexpr uint32_t kRingEmptyCount = 8 + 4;      // softmax warps (lane 0 each) + K, V producers + S, PV issuers
constexpr uint32_t kPFullCount = 8;              // owner warps arrive 2 each; on an item's first tile all 8 arrive 1

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
// moves afterwards.  Run by the whole scheduler warp (warp-collective): the
// union blocks of a chunk are listed 1024 at a time, each lane taking 32
// blocks, with a warp prefix sum of their counts placing them in order.
struct TileIter {
  const uint32_t* m0;
  const uint32_t* m1;
  uint16_t* list;   // shared memory, kListCap entries
  int N, C, W;
  int nw;           // mask words per half
  bool has1, exact_only, first;
  bool all_blocks;  // walk every block as exact (first-order mode), whatever the selection
  int lo, hi;       // current chunk [lo, hi)
  int jstart;       // the chunk's exact blocks run over [jstart, hi) then [lo, jstart)
  int seg;          // 0, 1: position in those two ranges; 2: exact blocks listed
  int scan;         // next block of the current range not yet listed
  int n, k;         // blocks listed, next one to emit
  int a0;           // next approximation sub-tile start
  int chunks_left;

  // Lists further union blocks in walk order until at least two wait to be
  // emitted or the chunk's ranges are exhausted.
  __device__ __forceinline__ void refill(int lane) {
    if (k > 0) {   // keep a leftover block at the front
      const int keep = n - k;
      const uint16_t v = (keep > 0) ? list[k] : 0;
      __syncwarp();
      if (keep > 0 && lane == 0) list[0] = v;
      __syncwarp();
      n = keep;
      k = 0;
    }
    while (seg < 2 && n < 2) {
      const int lim = seg == 0 ? hi : jstart;
      if (scan >= lim) {
        ++seg;
        scan = lo;
        continue;
      }
      const int wb = scan + 32 * lane;
      uint32_t u = 0u;
      if (wb < lim) {
        u = all_blocks ? 0xFFFFFFFFu : (mask_bits32(m0, wb, nw) | mask_bits32(m1, wb, nw));
        const int nv = lim - wb;
        if (nv < 32) u &= (1u << nv) - 1u;
      }
      const int c = __popc(u);
      int pre = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, pre, o);
        if (lane >= o) pre += v;
      }
      const int tot = __shfl_sync(0xFFFFFFFFu, pre, 31);
      int pos = n + pre - c;
      while (u) {
        const int bb = __ffs(u) - 1;
        u &= u - 1u;
        list[pos++] = static_cast<uint16_t>(wb + bb);
      }
      __syncwarp();
      n += tot;
      scan = min(scan + kListPass, lim);
    }
  }
  __device__ __forceinline__ void start_chunk(int start) {
    hi = min(lo + C, N);
    jstart = start;
    seg = 0;
    scan = start;
    n = 0;
    k = 0;
    a0 = exact_only ? hi : lo;
  }
  __device__ __forceinline__ void init(const ItemSlot& s, uint16_t* list_, int N_, int C_, int W_, int i0,
                                       bool has1_, bool exact_only_) {
    m0 = s.mask[0];
    m1 = s.mask[1];
    list = list_;
    N = N_;
    C = C_;
    W = W_;
    nw = (N_ + 31) >> 5;
    has1 = has1_;
    exact_only = exact_only_;
    all_blocks = false;
    first = true;
    chunks_left = (N_ + C_ - 1) / C_;
    lo = (i0 / C_) * C_;
    start_chunk(i0);
  }
  __device__ __forceinline__ bool next(Tile& t, int lane) {
    while (chunks_left > 0) {
      if (n - k < 2 && seg < 2) refill(lane);
      if (k < n) {
        const int ja = list[k];
        const int jb = (k + 1 < n) ? static_cast<int>(list[k + 1]) : -1;
        k += (jb >= 0) ? 2 : 1;
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
          const int nn = min(32, a1 - x);
          const uint32_t range = (nn >= 32) ? 0xFFFFFFFFu : ((1u << nn) - 1u);
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

// Largest of 32 values (three-input max, a tree of depth 4).
__device__ __forceinline__ float max32(const float* x) {
  float a[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) a[i] = max3f(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
  a[10] = fmaxf(x[30], x[31]);
  const float b0 = max3f(a[0], a[1], a[2]), b1 = max3f(a[3], a[4], a[5]), b2 = max3f(a[6], a[7], a[8]);
  return max3f(max3f(b0, b1, b2), a[9], a[10]);
}

// Multiplies the bf16 P values already stored in the first n 16-column groups
// of a row's S/P buffer by f (a power of two: exact).  Warp-wide.
__device__ __noinline__ void scale_p(uint32_t tS, int n, float f) {
  tmem_st_wait();   // the groups' stores have landed
  const __nv_bfloat162 f2 = __floats2bfloat162_rn(f, f);
#pragma unroll 1
  for (int g = 0; g < n; ++g) {
    float r[16];
    tmem_ld_x16f(tS + 16 * g, r);
    tmem_ld_wait();
    reg_fence16(r);
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&r[e]);
      h = __hmul2(h, f2);
      w[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    tmem_st_x16(tS + 16 * g, w);
  }
}

// 2^-k for a whole number k >= 0 given as a float difference of two whole
// numbers (0 below the fp32 range), exact.
__device__ __forceinline__ float exp2_neg_int(float k) {
  const int ki = __float2int_rn(k);
  return (ki >= 126) ? 0.f : __int_as_float((127 - ki) << 23);
}

// Out-of-line pieces of the softmax path that run rarely (once per item, or on
// a rescale), so that the per-tile code stays small.
// The row's O (its first d columns) times alpha, a power of two.  Warp-wide.
__device__ __noinline__ void scale_o(uint32_t tO, float alpha, int d) {
#pragma unroll 1
  for (int c = 0; c < d; c += 32) {
    float o[32];
    tmem_ld_x32f(tO + c, o);
    tmem_ld_wait();
    reg_fence32(o);
    uint32_t ow[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) ow[e] = __float_as_uint(o[e] * alpha);
    tmem_st_x32(tO + c, ow);
  }
}
__device__ __noinline__ void store_o_rows(uint32_t tO, int c_lo, int c_hi, bool have, float inv_l, uint16_t* orow) {
#pragma unroll 1
  for (int c16 = c_lo; c16 < c_hi; c16 += 16) {
    float a[16];
    if (have) {
      tmem_ld_x16f(tO + c16, a);
      tmem_ld_wait();
      reg_fence16(a);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) a[e] = 0.f;
    }
    if (orow) {
      uint4* dst = reinterpret_cast<uint4*>(orow + c16);
      dst[0] = make_uint4(pack_bf16x2(a[0] * inv_l, a[1] * inv_l), pack_bf16x2(a[2] * inv_l, a[3] * inv_l),
                          pack_bf16x2(a[4] * inv_l, a[5] * inv_l), pack_bf16x2(a[6] * inv_l, a[7] * inv_l));
      dst[1] = make_uint4(pack_bf16x2(a[8] * inv_l, a[9] * inv_l), pack_bf16x2(a[10] * inv_l, a[11] * inv_l),
                          pack_bf16x2(a[12] * inv_l, a[13] * inv_l), pack_bf16x2(a[14] * inv_l, a[15] * inv_l));
    }
  }
}
// FO: the first-order mode (kFlagFirstOrder) is a separate instantiation, so
// that its extra per-tile work does not enter the default kernel's code.
template <int D, bool FO>
__global__ void __launch_bounds__(kLaunchBoundThreads, 1)
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
  constexpr bool first_order = FO;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl.item_full[s], 1);
      mbar_init(&ctl.item_empty[s], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&ctl.s_full[b], 1);
      mbar_init(&ctl.p_full[b], kPFullCount);
      mbar_init(&ctl.pv_done[b], 1);
      mbar_init(&ctl.mready[b], 4);   // the four warps of the tile's warpgroup
    }
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&ctl.ring_full[r], 1);
      mbar_init(&ctl.ring_empty[r], kRingEmptyCount);
    }
    for (int s = 0; s < kStages; ++s) mbar_init(&ctl.k_full[s], 1);
    for (int s = 0; s < kStagesV; ++s) mbar_init(&ctl.v_full[s], 1);
    mbar_init(&ctl.q_full, 1);
    mbar_init(&ctl.q_empty, 1);
    mbar_init(&ctl.xchg, 8);   // one arrival per softmax warp
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

  SA_PROF(unsigned long long prof[kPrSlots]; for (int i = 0; i < kPrSlots; ++i) prof[i] = 0;
          const unsigned long long prof_t0 = clock64();)
  // Bounded wait; on a timeout raise the abort flag and the status word.  All
  // later waits return false at once, every role leaves its loop, and the CTA
  // meets at the final barrier.  The first probe is inline; the sleeping loop
  // behind it is out of line, which keeps every wait site small.
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
  // A descriptor that points outside the head's blocks or items is a bug in
  // the walk: record it, stop every role, never issue the copy.
  auto bad_desc = [&]() {
    *abort_flag = 1;
    atomicOr(p.status, kStatusDevice);
  };

  if (warp >= 8 && warp < 12) {
  if (warp == kWarpRoute) {
    // =========================================================== routing
    // (kFlagTestStall: publish nothing, so that every other role's bounded
    // wait runs out; used only to exercise the timeout path.)
    for (int seq = 0; !(p.flags & kFlagTestStall); ++seq) {
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
      SA_PROF(const unsigned long long tr0 = clock64();)
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
          // the key's 128 floats (L2-resident) in batches of 8 x 16 bytes, all
          // loads of a batch in flight before its products
          const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D);
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll 1
          for (int c0 = 0; c0 < D / 4; c0 += 8) {
            float4 xs[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) xs[u] = __ldg(kr + c0 + u);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float4 x = xs[u];
              const float4 qa = *reinterpret_cast<const float4*>(&ctl.qbar[0][4 * (c0 + u)]);
              const float4 qb4 = *reinterpret_cast<const float4*>(&ctl.qbar[1][4 * (c0 + u)]);
              a0 = fmaf(qa.x, x.x, a0); a1 = fmaf(qa.y, x.y, a1); a2 = fmaf(qa.z, x.z, a2); a3 = fmaf(qa.w, x.w, a3);
              b0 = fmaf(qb4.x, x.x, b0); b1 = fmaf(qb4.y, x.y, b1); b2 = fmaf(qb4.z, x.z, b2); b3 = fmaf(qb4.w, x.w, b3);
            }
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
      SA_PROF(prof[kPrRouteItem] += clock64() - tr0;)
      if (lane == 0) mbar_arrive(&ctl.item_full[s]);   // release: masks and item visible
    }
  } else if (warp == kWarpSched) {
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
        it.init(sl, ctl.ulist, p.N, p.chunk, p.W, 2 * pair, 2 * pair + 1 < p.N, exact_only || first_order);
        it.all_blocks = first_order;
        Tile t, tn;
        bool have = it.next(t, lane);
        bool first_desc = true;
        while (have) {
          SA_PROF(const unsigned long long tn0 = clock64();)
          const bool have_next = it.next(tn, lane);
          SA_PROF(prof[kPrSchedNext] += clock64() - tn0;)
          if (!first_desc && !(dsc = claim())) break;
          first_desc = false;
          SA_PROF(const unsigned long long td0 = clock64();)
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
                bits = (first_order || mask_bit(sl.mask[h], jx)) ? range : 0u;
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
            int sb = 0xF;
            if (first_order && t.kind == 1) {
              sb = 0;
              for (int h = 0; h < 2; ++h) {
                if (mask_bit(sl.mask[h], t.ja)) sb |= 1 << (2 * h);
                if (t.jb >= 0 && mask_bit(sl.mask[h], t.jb)) sb |= 2 << (2 * h);
              }
            }
            dsc->selbits = sb;
          }
          publish();
          SA_PROF(prof[kPrSchedDesc] += clock64() - td0;)
          t = tn;
          have = have_next;
        }
        if (have) break;   // left early on a timeout
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.item_empty[s]);   // the item's masks are no longer read
    }
  } else if (warp == kWarpLoad) {
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
        // range check of the coordinates this tile's copies use
        if (bh < 0 || bh >= p.BH || pair < 0 || pair >= p.num_pairs || ja < 0 || ja >= p.N || jb >= p.N ||
            ((flags & kDescApprox) && jb != -1)) {
          bad_desc();
          break;
        }
        if (kside && (flags & kDescFirst)) {  // the item's query tile (the previous item's S MMAs must be done)
          if (qseq > 0 && !wait(&ctl.q_empty, (qseq - 1) & 1, kPrKQEmpty)) break;
          mbar_arrive_expect_tx(&ctl.q_full, 128u * D * 2u);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(sQ + cb * CB, &tm_q, &ctl.q_full, cb * 64, 128 * pair, bh);
          ++qseq;
        }
        // The stage was last used by tile tl - nst (nst stages on this side);
        // it is free once that tile's S MMA (K side) or PV MMA (V side) has
        // completed, which the barriers of its TMEM buffer (tl - nst) % 3
        // record.
        uint64_t* full = kside ? &ctl.k_full[stage] : &ctl.v_full[stage];
        const uint32_t nst = kside ? kStages : kStagesV;
        if (tl >= nst) {
          const uint32_t tp = tl - nst;
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
        if (++stage == static_cast<int>(nst)) stage = 0;
      }
    }
  } else {
    // =========================================================== S issuer
    // S(t) = Q · Kside(t)ᵀ into TMEM buffer t % 3, once PV(t - 3), the last
    // reader of that buffer, has completed.
    if (lane == 0) {
      const uint32_t sKa = smem_u32(sK);
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      int kstage = 0;
      uint32_t kphase = 0, tcount = 0, qseq = 0;
      for (uint32_t r = 0;; ++r) {
        if (!ring_get(r, kPrSDesc)) break;
        const TileDesc& dsc = ctl.ring[r % kRing];
        const int flags = dsc.flags, ncols = dsc.ncols;
        mbar_arrive(&ctl.ring_empty[r % kRing]);
        if (flags & kDescEnd) break;
        if (flags & kDescEmpty) continue;
        const uint32_t t = tcount++;
        const uint32_t b = t % 3u;
        if (t >= 3 && !wait(&ctl.pv_done[b], ((t / 3u) - 1u) & 1u, kPrSBuf)) break;
        if ((flags & kDescFirst) && !wait(&ctl.q_full, qseq & 1, kPrSQ)) break;
        if (!wait(&ctl.k_full[kstage], kphase, kPrSK)) break;
        tc_fence_after();
        SA_PROF(const unsigned long long tis = clock64();)
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
        SA_PROF(prof[kPrSIssue] += clock64() - tis;)
        if (++kstage == kStages) {
          kstage = 0;
          kphase ^= 1u;
        }
        if (flags & kDescLast) {  // every S MMA of this item is issued: Q is free once they complete
          umma_commit(&ctl.q_empty);
          ++qseq;
        }
      }
    }
  }
  } else if (warp >= 12) {
  if (warp == kWarpPv) {
    // =========================================================== PV issuer
    // O (+)= P(t) · Vside(t) in tile order, P read from TMEM buffer t % 3: the
    // P of the tile's 16 kk .. 16 kk + 15 keys sits in the buffer's columns
    // 8 kk .. 8 kk + 7 (bf16 pairs).
    if (lane == 0) {
      const uint32_t sVa = smem_u32(sV);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 1);
      int vstage = 0;
      uint32_t vphase = 0, tcount = 0;
      for (uint32_t r = 0;; ++r) {
        if (!ring_get(r, kPrPvDesc)) break;
        const TileDesc& dsc = ctl.ring[r % kRing];
        const int flags = dsc.flags, ncols = dsc.ncols;
        mbar_arrive(&ctl.ring_empty[r % kRing]);
        if (flags & kDescEnd) break;
        if (flags & kDescEmpty) continue;
        const uint32_t t = tcount++;
        const uint32_t b = t % 3u;
        if (!wait(&ctl.p_full[b], (t / 3u) & 1u, kPrPvP)) break;
        if (!wait(&ctl.v_full[vstage], vphase, kPrPvV)) break;
        tc_fence_after();
        SA_PROF(const unsigned long long tis = clock64();)
        // descriptors are linear in the address: + (bytes >> 4) moves them
        const uint64_t vdesc = sdesc_sw128(sVa + vstage * kTile, CB, 1024);
        const uint32_t pbase = tmem + kTmemS0 + 128u * b;
        const uint32_t acc0 = (flags & kDescFirst) ? 0u : 1u;
        if (ncols == 128) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tmem + kTmemO, pbase + 8 * kk, vdesc + 128 * kk, idesc_pv, kk == 0 ? acc0 : 1u);
        } else if (ncols == 64) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + kTmemO, pbase + 8 * kk, vdesc + 128 * kk, idesc_pv, kk == 0 ? acc0 : 1u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_ts(tmem + kTmemO, pbase + 8 * kk, vdesc + 128 * kk, idesc_pv, kk == 0 ? acc0 : 1u);
        }
        umma_commit(&ctl.pv_done[b]);
        SA_PROF(prof[kPrPvIssue] += clock64() - tis;)
        if (++vstage == kStagesV) {
          vstage = 0;
          vphase ^= 1u;
        }
      }
    }
  }
  } else {
    // =========================================================== softmax (warps 0-7)
    // Tile t belongs to warpgroup t & 1; the thread of TMEM lane `row` owns row
    // `row` of it, every column.  m and the row sums are in log2 units.
    const int wg = warp >> 2;
    const int row = tid & 127;        // tile row = TMEM lane
    const int half = row >> 6;        // query block of the pair the row belongs to
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + kTmemO + lane_base;
    uint32_t tcount = 0;     // tiles seen (S buffer tcount % 3, PV index tcount)
    uint32_t xc = 0;         // epilogue exchanges done
    float l_run = 0.f;       // this thread's partial row sum ...
    float m_l = -INFINITY;   // ... accumulated at this reference maximum
    float m_own = -INFINITY; // the m this warpgroup's latest tile of the item settled on
    bool item_tiles = false; // the current item had a tile
    // The warp leaves together: its TMEM loads and stores are warp-wide.
    auto wait_w = [&](uint64_t* bar, uint32_t parity, int slot) -> bool {
      return __all_sync(0xFFFFFFFFu, wait(bar, parity, slot));
    };
    for (uint32_t r = 0;; ++r) {
      if (!wait_w(&ctl.ring_full[r % kRing], (r / kRing) & 1, kPrSmDesc)) break;
      const TileDesc& dsc = ctl.ring[r % kRing];
      const uint4 bw = *reinterpret_cast<const uint4*>(dsc.bits[half]);
      const int ncols = dsc.ncols, dflags = dsc.flags, tail_col = dsc.tail, dbh = dsc.bh, dpair = dsc.pair;
      const int selbits = dsc.selbits;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.ring_empty[r % kRing]);
      if (dflags & kDescEnd) break;
      if (!(dflags & kDescEmpty)) {
        const uint32_t t = tcount++;
        const uint32_t b = t % 3u;
        const bool first = (dflags & kDescFirst) != 0;
        if (first) {
          l_run = 0.f;
          m_l = -INFINITY;
          m_own = -INFINITY;
        }
        item_tiles = true;
        if (static_cast<int>(t & 1u) != wg) {
          // Not this warpgroup's tile.  On an item's first tile both warpgroups
          // arrive, so that its PV (which overwrites O) waits for this
          // warpgroup's epilogue reads of the previous item's O.
          if (first) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cnt(&ctl.p_full[b], 1u);
          }
        } else {
          if (!wait_w(&ctl.s_full[b], (t / 3u) & 1u, kPrSmS)) break;
          tc_fence_after();
          SA_PROF(unsigned long long tph = clock64(); prof[kPrSmTiles] += 1;)
          const int ng = ncols >> 5;                 // 32-column groups: 1, 2 or 4
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
          // One pass over the row's columns, 32 at a time, against a running
          // reference m_cur that starts at the m this warpgroup's previous tile
          // of the item settled on.  A group whose largest y exceeds m_cur by
          // more than 8 raises m_cur to a whole number (the groups already
          // stored are scaled by the exact power of two).  Afterwards m_cur
          // meets the m that tile t - 1 settled on; the larger wins, and P or
          // O, whichever is behind, is scaled to it (both are rare).
          const float boost = (dflags & kDescApprox) ? 6.f : 0.f;
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          float m_cur = m_own;
          float2 ra = make_float2(0.f, 0.f), rb = make_float2(0.f, 0.f);
          // First-order mode: a block this row's half did not select is
          // expanded around its row-wise mean score c (the mean of the exact
          // scores over the block's valid keys, equal to q.K̄_j/sqrt(d)):
          // weight 2^(c - m) (1 + (s - c)) in natural-log units of s and c.
          const bool lin0 = first_order && !((selbits >> (2 * half)) & 1);
          const bool lin1 = first_order && ncols == 128 && !((selbits >> (2 * half + 1)) & 1);
          float xc0 = 0.f, xc1 = 0.f;   // raw-score means of the tile's two blocks
          if (__any_sync(0xFFFFFFFFu, lin0 || lin1)) {
#pragma unroll 1
            for (int g = 0; g < ng; ++g) {
              float xv[32];
              tmem_ld_x32f(tS + 32 * g, xv);
              tmem_ld_wait();
              reg_fence32(xv);
              const uint32_t bits = gb(g);
              float sum = 0.f;
#pragma unroll
              for (int e = 0; e < 32; ++e) sum += ((bits >> e) & 1u) ? xv[e] : 0.f;
              if (g < 2) xc0 += sum; else xc1 += sum;
            }
            const int n0 = __popc(gb(0)) + (ng > 1 ? __popc(gb(1)) : 0);
            const int n1 = (ng > 2) ? __popc(gb(2)) + __popc(gb(3)) : 0;
            xc0 = n0 ? xc0 / static_cast<float>(n0) : 0.f;
            xc1 = n1 ? xc1 / static_cast<float>(n1) : 0.f;
          }
#pragma unroll 1
          for (int g = 0; g < ng; ++g) {
            float xv[32];
            SA_PROF(const unsigned long long tl0 = clock64();)
            tmem_ld_x32f(tS + 32 * g, xv);
            tmem_ld_wait();
            reg_fence32(xv);
            SA_PROF(prof[kPrSmLd] += clock64() - tl0;)
            adjust(xv, g);
            const float ym = max32(xv) * p.scale_log2 + boost;   // -inf: no valid column here
            const bool up = ym > m_cur + 8.f;
            if (__any_sync(0xFFFFFFFFu, up)) {
              const float m_new = up ? ceilf(ym) : m_cur;
              const float f = (m_cur == -INFINITY) ? 0.f : exp2_neg_int(m_new - m_cur);
              scale_p(tS, g, f);
              ra.x *= f; ra.y *= f; rb.x *= f; rb.y *= f;
              m_cur = m_new;
            }
            const float mref = (m_cur == -INFINITY) ? 0.f : m_cur;
            const float2 of2 = make_float2(boost - mref, boost - mref);
            SA_PROF(const unsigned long long te0 = clock64();)
            uint32_t pk[16];
            const bool lin = (g < 2) ? lin0 : lin1;
            if (lin) {   // first-order weights of an unselected block (warp-uniform: a warp's rows share a half)
              const float xc = (g < 2) ? xc0 : xc1;
              const float ec = ex2_approx(fmaf(xc, p.scale_log2, boost - mref));
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float w0 = (xv[e] == -INFINITY) ? 0.f : ec * fmaf(xv[e] - xc, p.inv_sqrt_d, 1.f);
                const float w1 = (xv[e + 1] == -INFINITY) ? 0.f : ec * fmaf(xv[e + 1] - xc, p.inv_sqrt_d, 1.f);
                ra.x += w0;
                ra.y += w1;
                pk[e >> 1] = pack_bf16x2(w0, w1);
              }
            } else {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              const float2 y0 = __ffma2_rn(make_float2(xv[e], xv[e + 1]), sc2, of2);
              const float2 y1 = __ffma2_rn(make_float2(xv[e + 2], xv[e + 3]), sc2, of2);
              const float2 y2 = __ffma2_rn(make_float2(xv[e + 4], xv[e + 5]), sc2, of2);
              const float2 y3 = __ffma2_rn(make_float2(xv[e + 6], xv[e + 7]), sc2, of2);
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
            }
            tmem_st_x16(tS + 16 * g, pk);
            SA_PROF(prof[kPrSmExp] += clock64() - te0;)
          }
          SA_PROF(prof[kPrSmPass] += clock64() - tph; tph = clock64();)
          // ---- meet the m of tile t - 1 (its owner published it at its end)
          float m_hand = -INFINITY;
          if (!first) {
            const uint32_t tp = t - 1u;
            if (!wait_w(&ctl.mready[tp % 3u], (tp / 3u) & 1u, kPrSmHand)) break;
            m_hand = ctl.hand[tp % 3u][row];
          }
          const float m_fin = fmaxf(m_cur, m_hand);
          const bool p_behind = (m_fin != m_cur) && (m_cur != -INFINITY);
          if (__any_sync(0xFFFFFFFFu, p_behind)) {   // tile t - 1 raised m: scale this tile's P
            const float f = p_behind ? exp2_neg_int(m_fin - m_cur) : 1.f;
            scale_p(tS, ng, f);
            ra.x *= f; ra.y *= f; rb.x *= f; rb.y *= f;
          }
          const bool o_behind = (m_fin != m_hand) && (m_hand != -INFINITY);
          if (__any_sync(0xFFFFFFFFu, o_behind)) {   // this tile raised m: scale O (PV(0 .. t - 1))
            if (!wait_w(&ctl.pv_done[(t - 1u) % 3u], ((t - 1u) / 3u) & 1u, kPrSmO)) break;
            tc_fence_after();
            const float alpha = o_behind ? exp2_neg_int(m_fin - m_hand) : 1.f;
            scale_o(tO, alpha, D);
            SA_PROF(prof[kPrSmRescales] += 1;)
          }
          ctl.hand[b][row] = m_fin;
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.mready[b]);
          m_own = m_fin;
          // this thread's partial row sum follows the reference
          const float tile_sum = (ra.x + ra.y) + (rb.x + rb.y);
          l_run = (m_l == -INFINITY || m_l == m_fin) ? l_run : l_run * exp2_neg_int(m_fin - m_l);
          l_run += tile_sum;
          m_l = m_fin;
          tmem_st_wait();
          SA_PROF(prof[kPrSmMeet] += clock64() - tph;)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cnt(&ctl.p_full[b], first ? 1u : 2u);
        }
      }
      if (!(dflags & (kDescLast | kDescEmpty))) continue;
      // ---- epilogue: O / (l_0 + l_1) for this warpgroup's half of the row's columns
      SA_PROF(const unsigned long long tep = clock64();)
      if (item_tiles) {   // the item's last PV
        if (!wait_w(&ctl.pv_done[(tcount - 1u) % 3u], ((tcount - 1u) / 3u) & 1u, kPrSmO)) break;
        tc_fence_after();
      }
      const float2 mine = item_tiles ? make_float2(l_run, m_l) : make_float2(0.f, -INFINITY);
      float2 other;
      {
        const int ph = xc & 1;
        ctl.xval[ph][wg][row] = mine;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.xchg);
        if (!wait_w(&ctl.xchg, ph, kPrSmX)) break;
        ++xc;
        other = ctl.xval[ph][wg ^ 1][row];
      }
      // O was accumulated at the item's last reference maximum, the larger of
      // the two partials' (m never falls)
      const float m_f = fmaxf(mine.y, other.y);
      float l_tot = 0.f;
      if (mine.y != -INFINITY) l_tot += mine.x * exp2_neg_int(m_f - mine.y);
      if (other.y != -INFINITY) l_tot += other.x * exp2_neg_int(m_f - other.y);
      const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
      const int token = 128 * dpair + row;
      uint16_t* orow = p.out + (static_cast<size_t>(dbh) * p.L + token) * D;
      store_o_rows(tO, wg * (D / 2), (wg + 1) * (D / 2), item_tiles, inv_l, token < p.L ? orow : nullptr);
      // O is read; the next item's first PV (which overwrites O) waits for this
      // warp's arrival on that tile, which comes after these reads
      tc_fence_before();
      item_tiles = false;
      SA_PROF(prof[kPrSmEpi] += clock64() - tep;)
    }
  }

  SA_PROF({
    const int tslot = warp == kWarpRoute ? kPrTotRoute : warp == kWarpSched ? kPrTotSched
                    : warp == kWarpS ? kPrTotS : warp == kWarpPv ? kPrTotPv
                    : warp == kWarpLoad ? (lane == 0 ? kPrTotK : kPrTotV) : kPrTotSm;
    // one thread per role; the softmax slots come from the first warp of each
    // warpgroup, so they cover every tile once
    if ((lane == 0 && (warp >= 8 || warp == 0 || warp == 4)) || (warp == kWarpLoad && lane == 1)) {
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
