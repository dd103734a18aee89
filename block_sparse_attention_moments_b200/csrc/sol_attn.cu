// sol_attn.cu — C ABI of the Sol-Attn forward (declared in include/sol_attn.h):
// argument checks, the per-device workspace, TMA descriptor set-up and the
// launches of the three kernels (pool, moments + thresholds, fused attention).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "fused.cuh"
#include "moments.cuh"
#include "pool.cuh"
#include "sol_attn.h"
#include "topk_router.cuh"

using namespace solattn;

namespace {

constexpr int kBlock = 64;
constexpr int kMaxL = 1 << 20;
constexpr int kMaxBH = 65535;
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // bounded device waits: 2 s
constexpr unsigned long long kTestTimeoutNs = 1000000ull;  // with SOL_ATTN_FLAG_TEST_STALL: 1 ms

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                        \
  do {                                                                                        \
    cudaError_t e_ = (expr);                                                                  \
    if (e_ != cudaSuccess) return fail(SOL_ATTN_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

// ------------------------------------------------------------------ workspace
struct Shape {
  int B = 0, H = 0, L = 0, d = 0;
  bool operator==(const Shape& o) const { return B == o.B && H == o.H && L == o.L && d == o.d; }
};

struct Workspace {
  void* base = nullptr;
  size_t bytes = 0;
  // carved views
  float* qbar = nullptr;
  float* kbar = nullptr;
  __nv_bfloat16* kbar_bf = nullptr;
  __nv_bfloat16* kbar_lo = nullptr;
  __nv_bfloat16* vbar_bf = nullptr;
  double* mom_mean = nullptr;
  double* mom_cov = nullptr;
  float* tau = nullptr;
  int* counts = nullptr;
  unsigned* counter = nullptr;   // fixed 256-byte block, allocated once per device:
  unsigned* status = nullptr;    // [0] work counter, [32] sticky status word
  void* ctl_block = nullptr;
  Shape shape;        // shape the views are carved for
  int stage = 0;      // 0 none, 1 pooled, 2 thresholds, 3 fused done
  Shape last_fused;   // shape of the last completed forward (for stats)
  // host-buffer entry point: two staging slots, three streams (copy in,
  // compute, copy out) and the events that order them
  void* topk_map = nullptr;   // proxy map of the comparison top-k router (grown on demand)
  size_t topk_map_bytes = 0;
  void* host_stage = nullptr;
  size_t host_stage_bytes = 0;
  cudaStream_t host_stream = nullptr;   // copies in
  cudaStream_t host_comp = nullptr;     // kernels
  cudaStream_t host_out = nullptr;      // copies out
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr}, ev_out[2] = {nullptr, nullptr};
};

constexpr int kMaxDevices = 64;
Workspace g_ws[kMaxDevices];
std::mutex g_mu;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t layout(const Shape& s, Workspace* w, char* base) {
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t N = (static_cast<size_t>(s.L) + kBlock - 1) / kBlock;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return base ? base + o : nullptr;
  };
  char* p_qbar = take(BH * N * s.d * 4);
  char* p_kbar = take(BH * N * s.d * 4);
  char* p_kbf = take(BH * N * s.d * 2);
  char* p_klo = take(BH * N * s.d * 2);
  char* p_vbf = take(BH * N * s.d * 2);
  char* p_mean = take(BH * s.d * 8);
  char* p_cov = take(BH * s.d * s.d * 8);
  char* p_tau = take(BH * N * 4);
  char* p_cnt = take(BH * N * 4);
  if (w && base) {
    w->qbar = reinterpret_cast<float*>(p_qbar);
    w->kbar = reinterpret_cast<float*>(p_kbar);
    w->kbar_bf = reinterpret_cast<__nv_bfloat16*>(p_kbf);
    w->kbar_lo = reinterpret_cast<__nv_bfloat16*>(p_klo);
    w->vbar_bf = reinterpret_cast<__nv_bfloat16*>(p_vbf);
    w->mom_mean = reinterpret_cast<double*>(p_mean);
    w->mom_cov = reinterpret_cast<double*>(p_cov);
    w->tau = reinterpret_cast<float*>(p_tau);
    w->counts = reinterpret_cast<int*>(p_cnt);
  }
  return off;
}

int current_device(int* dev) {
  CUDA_TRY(cudaGetDevice(dev));
  if (*dev < 0 || *dev >= kMaxDevices) return fail(SOL_ATTN_ERR_UNSUPPORTED, "device index %d too large", *dev);
  return SOL_ATTN_OK;
}

int check_arch(int dev) {
  static int checked[kMaxDevices] = {0};
  if (checked[dev] == 1) return SOL_ATTN_OK;
  int major = 0, minor = 0;
  CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0)
    return fail(SOL_ATTN_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, major,
                minor);
  checked[dev] = 1;
  return SOL_ATTN_OK;
}

// Make the workspace of the current device fit shape s (grow-only allocation).
int ensure_ws(const Shape& s, Workspace** out) {
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  if ((rc = check_arch(dev))) return rc;
  Workspace& w = g_ws[dev];
  if (!w.ctl_block) {
    CUDA_TRY(cudaMalloc(&w.ctl_block, 256));
    CUDA_TRY(cudaMemset(w.ctl_block, 0, 256));
    w.counter = static_cast<unsigned*>(w.ctl_block);
    w.status = static_cast<unsigned*>(w.ctl_block) + 32;
  }
  const size_t need = layout(s, nullptr, nullptr);
  if (need > w.bytes) {
    if (w.base) CUDA_TRY(cudaFree(w.base));
    w.base = nullptr;
    w.bytes = 0;
    CUDA_TRY(cudaMalloc(&w.base, need));
    w.bytes = need;
    CUDA_TRY(cudaMemset(w.base, 0, need));
  }
  if (!(w.shape == s)) {
    layout(s, &w, static_cast<char*>(w.base));
    w.shape = s;
    w.stage = 0;
  }
  *out = &w;
  return SOL_ATTN_OK;
}

int check_shape(int B, int H, int L, int d, int block) {
  if (B <= 0 || H <= 0 || L <= 0) return fail(SOL_ATTN_ERR_ARG, "B, H, L must be positive (got %d, %d, %d)", B, H, L);
  if (block != kBlock) return fail(SOL_ATTN_ERR_UNSUPPORTED, "block must be 64 (got %d)", block);
  if (d != 64 && d != 128) return fail(SOL_ATTN_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  if (L > kMaxL) return fail(SOL_ATTN_ERR_UNSUPPORTED, "L = %d exceeds the supported maximum %d", L, kMaxL);
  // pool, moments and threshold kernels put B*H on gridDim.y (at most 65535)
  if (static_cast<long long>(B) * H > kMaxBH)
    return fail(SOL_ATTN_ERR_UNSUPPORTED, "B*H = %lld exceeds the supported maximum %d",
                static_cast<long long>(B) * H, kMaxBH);
  return SOL_ATTN_OK;
}

int check_ptr(const void* p, const char* name) {
  if (!p) return fail(SOL_ATTN_ERR_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return fail(SOL_ATTN_ERR_ALIGN, "%s is not 16-byte aligned", name);
  return SOL_ATTN_OK;
}

// ------------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return fail(SOL_ATTN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *fn = cached;
  return SOL_ATTN_OK;
}

// 3-D bf16 map over [BH][rows][d] with a {64, box_rows, 1} box and 128-byte swizzle.
// Rows past `rows` read as zero.
int make_map(CUtensorMap* m, const void* ptr, int d, long long rows, long long BH, int box_rows) {
  EncodeTiledFn enc;
  int rc = get_encoder(&enc);
  if (rc) return rc;
  cuuint64_t gdim[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
  cuuint64_t gstride[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), gdim, gstride, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SOL_ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return SOL_ATTN_OK;
}

// ------------------------------------------------------------------ stages
int run_pool(Workspace& w, const void* q, const void* k, const void* v, const sol_attn_debug* dbg,
             cudaStream_t st) {
  const Shape& s = w.shape;
  const int N = (s.L + kBlock - 1) / kBlock;
  dim3 grid(N, s.B * s.H);
  float* vdbg = dbg ? dbg->vhat : nullptr;
  auto qq = static_cast<const uint16_t*>(q);
  auto kk = static_cast<const uint16_t*>(k);
  auto vv = static_cast<const uint16_t*>(v);
  if (s.d == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(qq, kk, vv, s.L, N, w.qbar, w.kbar, w.kbar_bf, w.kbar_lo, w.vbar_bf,
                                           vdbg);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(qq, kk, vv, s.L, N, w.qbar, w.kbar, w.kbar_bf, w.kbar_lo, w.vbar_bf,
                                          vdbg);
  CUDA_TRY(cudaGetLastError());
  const size_t nbytes = static_cast<size_t>(s.B) * s.H * N * s.d * 4;
  if (dbg && dbg->qbar) CUDA_TRY(cudaMemcpyAsync(dbg->qbar, w.qbar, nbytes, cudaMemcpyDeviceToDevice, st));
  if (dbg && dbg->kbar) CUDA_TRY(cudaMemcpyAsync(dbg->kbar, w.kbar, nbytes, cudaMemcpyDeviceToDevice, st));
  w.stage = 1;
  return SOL_ATTN_OK;
}

template <int D>
int launch_threshold(Workspace& w, int N, float beta, int mode, const sol_attn_debug* dbg, cudaStream_t st) {
  const int BH = w.shape.B * w.shape.H;
  constexpr int T = D / 64;
  moments_kernel<D><<<dim3(T * (T + 1) / 2, BH), 256, 0, st>>>(w.kbar, N, w.mom_mean, w.mom_cov);
  CUDA_TRY(cudaGetLastError());
  constexpr size_t smem = threshold_smem_bytes(D);
  static bool attr_set[kMaxDevices] = {false};   // the attribute is set per device
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_ATTN_ERR_UNSUPPORTED, "device index %d too large", dev);
  if (!attr_set[dev]) {
    CUDA_TRY(cudaFuncSetAttribute(threshold_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem)));
    attr_set[dev] = true;
  }
  dim3 grid((N + kThresholdBlocksPerCta - 1) / kThresholdBlocksPerCta, BH);
  threshold_kernel<D><<<grid, 256, smem, st>>>(w.qbar, w.mom_mean, w.mom_cov, N, beta, mode, w.tau,
                                                dbg ? dbg->mu : nullptr, dbg ? dbg->sigma : nullptr);
  CUDA_TRY(cudaGetLastError());
  return SOL_ATTN_OK;
}

int run_threshold(Workspace& w, float beta, unsigned flags, const sol_attn_debug* dbg, cudaStream_t st) {
  const Shape& s = w.shape;
  const int N = (s.L + kBlock - 1) / kBlock;
  int mode = kThresholdBeta;
  if ((flags & SOL_ATTN_FLAG_SELECT_ALL) || (std::isinf(beta) && beta < 0)) mode = kThresholdSelectAll;
  else if (std::isinf(beta)) mode = kThresholdSelectNone;
  int rc = (s.d == 128) ? launch_threshold<128>(w, N, beta, mode, dbg, st)
                        : launch_threshold<64>(w, N, beta, mode, dbg, st);
  if (rc) return rc;
  if (dbg && dbg->tau)
    CUDA_TRY(cudaMemcpyAsync(dbg->tau, w.tau, static_cast<size_t>(s.B) * s.H * N * 4, cudaMemcpyDeviceToDevice, st));
  w.stage = 2;
  return SOL_ATTN_OK;
}

template <int D>
int launch_fused(Workspace& w, const void* q, const void* k, const void* v, void* out, int chunk, unsigned flags,
                 const sol_attn_debug* dbg, cudaStream_t st) {
  const Shape& s = w.shape;
  const int N = (s.L + kBlock - 1) / kBlock;
  const long long BH = static_cast<long long>(s.B) * s.H;
  if ((N + 31) / 32 > kMaxMaskWords)
    return fail(SOL_ATTN_ERR_UNSUPPORTED, "N = %d pooled blocks exceeds the fused kernel's %d", N, kMaxMaskWords * 32);
  // The tile walk goes through windows of max(C, 64) pooled keys.  The
  // selection does not depend on C (the union of the chunk-wise selections is
  // the global one) and the online softmax does not depend on the order of its
  // tiles, so C only shapes the walk; windows narrower than 64 blocks would
  // only make the approximation tiles narrower and the exact tiles single-block.
  const int win = std::max(chunk, 64);
  const int W = std::min(64, (std::min(win, N) + 31) / 32 * 32);
  CUtensorMap tq, tk, tv, tkb, tkl, tvb;
  int rc;
  if ((rc = make_map(&tq, q, D, s.L, BH, 128))) return rc;
  if ((rc = make_map(&tk, k, D, s.L, BH, 64))) return rc;
  if ((rc = make_map(&tv, v, D, s.L, BH, 64))) return rc;
  if ((rc = make_map(&tkb, w.kbar_bf, D, N, BH, W))) return rc;
  if ((rc = make_map(&tkl, w.kbar_lo, D, N, BH, W))) return rc;
  if ((rc = make_map(&tvb, w.vbar_bf, D, N, BH, W))) return rc;

  FusedParams p{};
  p.BH = static_cast<int>(BH);
  p.L = s.L;
  p.N = N;
  p.W = W;
  p.chunk = win;
  p.num_pairs = (N + 1) / 2;
  p.num_items = static_cast<int>(BH * p.num_pairs);
  p.flags = flags;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  {
    const int tail_n = s.L - 64 * (N - 1);
    p.tail_raw = static_cast<float>((std::log2(static_cast<double>(tail_n)) - 6.0) / static_cast<double>(p.scale_log2));
  }
  p.qbar = w.qbar;
  p.kbar = w.kbar;
  p.tau = w.tau;
  p.counts = w.counts;
  p.mask_out = dbg ? dbg->mask : nullptr;
  p.out = static_cast<uint16_t*>(out);
  p.work_counter = w.counter;
  p.status = w.status;
  // SOL_ATTN_FLAG_TEST_STALL: the routing warp publishes nothing and every
  // wait gives up after 1 ms (exercises the timeout path; no output is written)
  p.timeout_ns = (flags & SOL_ATTN_FLAG_TEST_STALL) ? kTestTimeoutNs : kTimeoutNs;

  int dev = 0, nsm = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  static bool attr_set[kMaxDevices] = {false};   // the attribute is set per device
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_ATTN_ERR_UNSUPPORTED, "device index %d too large", dev);
  if (!attr_set[dev]) {
    CUDA_TRY(cudaFuncSetAttribute(sol_attn_fused_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kFusedSmemBytes)));
    CUDA_TRY(cudaFuncSetAttribute(sol_attn_fused_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kFusedSmemBytes)));
    attr_set[dev] = true;
  }
  CUDA_TRY(cudaMemsetAsync(w.counter, 0, sizeof(unsigned), st));
  const int grid = std::min(p.num_items, nsm);
  if (flags & SOL_ATTN_FLAG_FIRST_ORDER)
    sol_attn_fused_kernel<D, true><<<grid, kThreads, kFusedSmemBytes, st>>>(tq, tk, tv, tkb, tkl, tvb, p);
  else
    sol_attn_fused_kernel<D, false><<<grid, kThreads, kFusedSmemBytes, st>>>(tq, tk, tv, tkb, tkl, tvb, p);
  CUDA_TRY(cudaGetLastError());
  return SOL_ATTN_OK;
}

int run_fused(Workspace& w, const void* q, const void* k, const void* v, void* out, int chunk, unsigned flags,
              const sol_attn_debug* dbg, cudaStream_t st) {
  int rc = (w.shape.d == 128) ? launch_fused<128>(w, q, k, v, out, chunk, flags, dbg, st)
                              : launch_fused<64>(w, q, k, v, out, chunk, flags, dbg, st);
  if (rc) return rc;
  w.stage = 3;
  w.last_fused = w.shape;
  return SOL_ATTN_OK;
}

int read_status(Workspace& w, cudaStream_t st) {
  CUDA_TRY(cudaStreamSynchronize(st));
  unsigned h = 0;
  CUDA_TRY(cudaMemcpy(&h, w.status, sizeof(h), cudaMemcpyDeviceToHost));
  if (h) {
    CUDA_TRY(cudaMemset(w.status, 0, sizeof(unsigned)));
    if (h & kStatusTimeout) return fail(SOL_ATTN_ERR_TIMEOUT, "a bounded device wait gave up (status 0x%x)", h);
    return fail(SOL_ATTN_ERR_DEVICE, "device-side check failed: a tile descriptor was out of range (status 0x%x)", h);
  }
  return SOL_ATTN_OK;
}

int check_io(const void* q, const void* k, const void* v, const void* out, int B, int H, int L, int d) {
  int rc;
  if ((rc = check_ptr(q, "q")) || (rc = check_ptr(k, "k")) || (rc = check_ptr(v, "v"))) return rc;
  if (out) {
    if ((rc = check_ptr(out, "out"))) return rc;
    const size_t n = static_cast<size_t>(B) * H * L * d * 2;
    const char* o = static_cast<const char*>(out);
    for (const void* x : {q, k, v}) {
      const char* xc = static_cast<const char*>(x);
      if (o < xc + n && xc < o + n) return fail(SOL_ATTN_ERR_ARG, "out overlaps an input tensor");
    }
  }
  return SOL_ATTN_OK;
}

// ------------------------------------------------------------------ allocation-free forward
// Some callers cannot call cudaMalloc: code running inside a custom or
// pre-reserved memory pool that forbids outside allocations, latency-critical
// serving loops where an allocation could synchronise the device, and hosts
// that hand this library only the tensors it reads and writes.  For them the
// scratch of sol_attn_forward_noalloc lives in this fixed device array,
// reserved once per GPU when the library is loaded and held until exit.
constexpr size_t kNoAllocScratchBytes = size_t(96) << 20;   // 96 MiB
constexpr size_t kNoAllocCtlBytes = 256;                    // work counter + status word
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device with that
// device current (the host-side symbol is only a stand-in, not an address).
char* g_noalloc_base[kMaxDevices] = {nullptr};

int noalloc_base(int dev, char** out) {
  if (!g_noalloc_base[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return fail(SOL_ATTN_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    // the status word must start at zero; the work counter is cleared before every launch
    CUDA_TRY(cudaMemset(ptr, 0, kNoAllocCtlBytes));
    g_noalloc_base[dev] = static_cast<char*>(ptr);
  }
  *out = g_noalloc_base[dev];
  return SOL_ATTN_OK;
}

int check_flags(unsigned flags) {
  if ((flags & SOL_ATTN_FLAG_FIRST_ORDER) && (flags & SOL_ATTN_FLAG_EXACT_ONLY))
    return fail(SOL_ATTN_ERR_ARG, "FIRST_ORDER and EXACT_ONLY exclude each other");
  if (flags & ~(SOL_ATTN_FLAG_SELECT_ALL | SOL_ATTN_FLAG_EXACT_ONLY | SOL_ATTN_FLAG_SYNC_CHECK |
                SOL_ATTN_FLAG_TEST_STALL | SOL_ATTN_FLAG_FIRST_ORDER))
    return fail(SOL_ATTN_ERR_ARG, "unknown flag bits 0x%x", flags);
  return SOL_ATTN_OK;
}

}  // namespace

extern "C" {

int sol_attn_forward_ex(const void* q, const void* k, const void* v, void* out, int B, int H, int L, int d, int block,
                        int chunk, float beta, unsigned flags, const sol_attn_debug* dbg, void* stream) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if ((rc = check_flags(flags))) return rc;
  if (chunk < 1) return fail(SOL_ATTN_ERR_ARG, "chunk must be >= 1 (got %d)", chunk);
  if (std::isnan(beta)) return fail(SOL_ATTN_ERR_ARG, "beta is NaN");
  if (!out) return fail(SOL_ATTN_ERR_ARG, "out is NULL");
  if ((rc = check_io(q, k, v, out, B, H, L, d))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace* w;
  if ((rc = ensure_ws(Shape{B, H, L, d}, &w))) return rc;
  auto st = static_cast<cudaStream_t>(stream);
  if ((rc = run_pool(*w, q, k, v, dbg, st))) return rc;
  if ((rc = run_threshold(*w, beta, flags, dbg, st))) return rc;
  if ((rc = run_fused(*w, q, k, v, out, chunk, flags, dbg, st))) return rc;
  if (flags & SOL_ATTN_FLAG_SYNC_CHECK) return read_status(*w, st);
  return SOL_ATTN_OK;
}

int sol_attn_forward(const void* q, const void* k, const void* v, void* out, int B, int H, int L, int d, int block,
                     int chunk, float beta, void* stream) {
  return sol_attn_forward_ex(q, k, v, out, B, H, L, d, block, chunk, beta, 0u, nullptr, stream);
}

int sol_attn_stage_pool(const void* q, const void* k, const void* v, int B, int H, int L, int d, int block,
                        const sol_attn_debug* dbg, void* stream) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if ((rc = check_io(q, k, v, nullptr, B, H, L, d))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace* w;
  if ((rc = ensure_ws(Shape{B, H, L, d}, &w))) return rc;
  return run_pool(*w, q, k, v, dbg, static_cast<cudaStream_t>(stream));
}

int sol_attn_stage_threshold(int B, int H, int L, int d, int block, float beta, unsigned flags,
                             const sol_attn_debug* dbg, void* stream) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if (std::isnan(beta)) return fail(SOL_ATTN_ERR_ARG, "beta is NaN");
  std::lock_guard<std::mutex> lk(g_mu);
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Workspace& w = g_ws[dev];
  if (!(w.shape == Shape{B, H, L, d}) || w.stage < 1)
    return fail(SOL_ATTN_ERR_STATE, "stage_threshold needs a stage_pool of the same shape first");
  return run_threshold(w, beta, flags, dbg, static_cast<cudaStream_t>(stream));
}

int sol_attn_stage_fused(const void* q, const void* k, const void* v, void* out, int B, int H, int L, int d, int block,
                         int chunk, unsigned flags, const sol_attn_debug* dbg, void* stream) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if ((rc = check_flags(flags))) return rc;
  if (chunk < 1) return fail(SOL_ATTN_ERR_ARG, "chunk must be >= 1 (got %d)", chunk);
  if (!out) return fail(SOL_ATTN_ERR_ARG, "out is NULL");
  if ((rc = check_io(q, k, v, out, B, H, L, d))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Workspace& w = g_ws[dev];
  if (!(w.shape == Shape{B, H, L, d}) || w.stage < 2)
    return fail(SOL_ATTN_ERR_STATE, "stage_fused needs stage_pool and stage_threshold of the same shape first");
  auto st = static_cast<cudaStream_t>(stream);
  if ((rc = run_fused(w, q, k, v, out, chunk, flags, dbg, st))) return rc;
  if (flags & SOL_ATTN_FLAG_SYNC_CHECK) return read_status(w, st);
  return SOL_ATTN_OK;
}

int sol_attn_stats(int32_t* counts, int B, int H, int L, int block, void* stream) {
  if (!counts) return fail(SOL_ATTN_ERR_ARG, "counts is NULL");
  if (B <= 0 || H <= 0 || L <= 0) return fail(SOL_ATTN_ERR_ARG, "B, H, L must be positive");
  if (block != kBlock) return fail(SOL_ATTN_ERR_UNSUPPORTED, "block must be 64 (got %d)", block);
  std::lock_guard<std::mutex> lk(g_mu);
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  Workspace& w = g_ws[dev];
  const Shape& f = w.last_fused;
  if (w.stage < 3 || f.B != B || f.H != H || f.L != L || !(w.shape == f))
    return fail(SOL_ATTN_ERR_STATE, "no forward of shape (B=%d, H=%d, L=%d) to report on", B, H, L);
  const size_t N = (static_cast<size_t>(L) + kBlock - 1) / kBlock;
  CUDA_TRY(cudaMemcpyAsync(counts, w.counts, static_cast<size_t>(B) * H * N * sizeof(int32_t),
                           cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return SOL_ATTN_OK;
}

int sol_attn_forward_host(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int B, int H, int L,
                          int d, int block, int chunk, float beta, unsigned flags) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if (!q || !k || !v || !out) return fail(SOL_ATTN_ERR_ARG, "a host pointer is NULL");
  if (chunk < 1) return fail(SOL_ATTN_ERR_ARG, "chunk must be >= 1 (got %d)", chunk);
  if (std::isnan(beta)) return fail(SOL_ATTN_ERR_ARG, "beta is NaN");
  int dev;
  if ((rc = current_device(&dev))) return rc;
  // The (batch, head) slices are independent and contiguous: they go through in
  // up to kHostChunks groups, the copy in of group c + 1 and the copy out of
  // group c - 1 overlapping the kernels of group c.
  constexpr int kHostChunks = 16;
  const int BH = B * H;
  const int hc = (BH + kHostChunks - 1) / kHostChunks;     // heads per group
  const int ngroups = (BH + hc - 1) / hc;
  const size_t head_elems = static_cast<size_t>(L) * d;
  const size_t slot = align_up(static_cast<size_t>(hc) * head_elems * 2, 256);   // one tensor of a group
  Workspace* w;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    w = &g_ws[dev];
    if (!w->host_stream) {
      CUDA_TRY(cudaStreamCreateWithFlags(&w->host_stream, cudaStreamNonBlocking));
      CUDA_TRY(cudaStreamCreateWithFlags(&w->host_comp, cudaStreamNonBlocking));
      CUDA_TRY(cudaStreamCreateWithFlags(&w->host_out, cudaStreamNonBlocking));
      for (int i = 0; i < 2; ++i) {
        CUDA_TRY(cudaEventCreateWithFlags(&w->ev_in[i], cudaEventDisableTiming));
        CUDA_TRY(cudaEventCreateWithFlags(&w->ev_comp[i], cudaEventDisableTiming));
        CUDA_TRY(cudaEventCreateWithFlags(&w->ev_out[i], cudaEventDisableTiming));
      }
    }
    if (w->host_stage_bytes < 8 * slot) {   // 2 slots x (q, k, v, out)
      if (w->host_stage) CUDA_TRY(cudaFree(w->host_stage));
      w->host_stage = nullptr;
      w->host_stage_bytes = 0;
      CUDA_TRY(cudaMalloc(&w->host_stage, 8 * slot));
      w->host_stage_bytes = 8 * slot;
    }
  }
  char* stage = static_cast<char*>(w->host_stage);
  cudaStream_t s_in = w->host_stream, s_comp = w->host_comp, s_out = w->host_out;
  for (int c = 0; c < ngroups; ++c) {
    const int sl = c & 1;
    const int h0 = c * hc, cnt = std::min(hc, BH - h0);
    const size_t off = static_cast<size_t>(h0) * head_elems, bytes = static_cast<size_t>(cnt) * head_elems * 2;
    char* dq = stage + (4 * sl) * slot;
    char* dk = dq + slot;
    char* dv = dq + 2 * slot;
    char* dout = dq + 3 * slot;
    // inputs of slot sl are free once the kernels of group c - 2 have run
    if (c >= 2) CUDA_TRY(cudaStreamWaitEvent(s_in, w->ev_comp[sl], 0));
    CUDA_TRY(cudaMemcpyAsync(dq, q + off, bytes, cudaMemcpyHostToDevice, s_in));
    CUDA_TRY(cudaMemcpyAsync(dk, k + off, bytes, cudaMemcpyHostToDevice, s_in));
    CUDA_TRY(cudaMemcpyAsync(dv, v + off, bytes, cudaMemcpyHostToDevice, s_in));
    CUDA_TRY(cudaEventRecord(w->ev_in[sl], s_in));
    CUDA_TRY(cudaStreamWaitEvent(s_comp, w->ev_in[sl], 0));
    // the output of slot sl is free once group c - 2 has been copied out
    if (c >= 2) CUDA_TRY(cudaStreamWaitEvent(s_comp, w->ev_out[sl], 0));
    rc = sol_attn_forward_ex(dq, dk, dv, dout, 1, cnt, L, d, block, chunk, beta, flags & ~SOL_ATTN_FLAG_SYNC_CHECK,
                             nullptr, s_comp);
    if (rc) return rc;
    CUDA_TRY(cudaEventRecord(w->ev_comp[sl], s_comp));
    CUDA_TRY(cudaStreamWaitEvent(s_out, w->ev_comp[sl], 0));
    CUDA_TRY(cudaMemcpyAsync(out + off, dout, bytes, cudaMemcpyDeviceToHost, s_out));
    CUDA_TRY(cudaEventRecord(w->ev_out[sl], s_out));
  }
  CUDA_TRY(cudaStreamSynchronize(s_out));
  CUDA_TRY(cudaStreamSynchronize(s_comp));
  if (flags & SOL_ATTN_FLAG_SYNC_CHECK) {
    std::lock_guard<std::mutex> lk(g_mu);
    return read_status(g_ws[dev], s_comp);
  }
  return SOL_ATTN_OK;
}

size_t sol_attn_workspace_bytes(int B, int H, int L, int d, int block) {
  if (check_shape(B, H, L, d, block)) return 0;
  return layout(Shape{B, H, L, d}, nullptr, nullptr);
}

int sol_attn_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  Workspace& w = g_ws[dev];
  if (w.base) CUDA_TRY(cudaFree(w.base));
  if (w.ctl_block) CUDA_TRY(cudaFree(w.ctl_block));
  if (w.host_stage) CUDA_TRY(cudaFree(w.host_stage));
  if (w.topk_map) CUDA_TRY(cudaFree(w.topk_map));
  if (w.host_stream) CUDA_TRY(cudaStreamDestroy(w.host_stream));
  if (w.host_comp) CUDA_TRY(cudaStreamDestroy(w.host_comp));
  if (w.host_out) CUDA_TRY(cudaStreamDestroy(w.host_out));
  for (int i = 0; i < 2; ++i) {
    if (w.ev_in[i]) CUDA_TRY(cudaEventDestroy(w.ev_in[i]));
    if (w.ev_comp[i]) CUDA_TRY(cudaEventDestroy(w.ev_comp[i]));
    if (w.ev_out[i]) CUDA_TRY(cudaEventDestroy(w.ev_out[i]));
  }
  w = Workspace{};
  return SOL_ATTN_OK;
}

const char* sol_attn_error_string(int code) {
  static thread_local std::string msg;
  const char* base = "unknown status";
  switch (code) {
    case SOL_ATTN_OK: base = "ok"; break;
    case SOL_ATTN_ERR_ARG: base = "invalid argument"; break;
    case SOL_ATTN_ERR_UNSUPPORTED: base = "unsupported configuration"; break;
    case SOL_ATTN_ERR_ALIGN: base = "misaligned pointer"; break;
    case SOL_ATTN_ERR_CUDA: base = "CUDA error"; break;
    case SOL_ATTN_ERR_TIMEOUT: base = "device wait timed out"; break;
    case SOL_ATTN_ERR_STATE: base = "invalid call order / state"; break;
    case SOL_ATTN_ERR_DEVICE: base = "device-side check failed"; break;
  }
  msg = base;
  if (code != SOL_ATTN_OK && !g_last_error.empty()) msg += ": " + g_last_error;
  return msg.c_str();
}

int sol_attn_kernels_per_forward(void) { return 4; }

int sol_attn_profile_read(uint64_t* cycles, int n, int reset) {
#ifdef SOL_ATTN_PROFILE
  if (!cycles || n < 1) return fail(SOL_ATTN_ERR_ARG, "cycles is NULL or n < 1");
  unsigned long long h[kProfileSlots];
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpyFromSymbol(h, g_profile, sizeof(h)));
  for (int i = 0; i < n && i < kProfileSlots; ++i) cycles[i] = h[i];
  if (reset) {
    unsigned long long z[kProfileSlots] = {0};
    CUDA_TRY(cudaMemcpyToSymbol(g_profile, z, sizeof(z)));
  }
  return SOL_ATTN_OK;
#else
  (void)cycles; (void)n; (void)reset;
  return fail(SOL_ATTN_ERR_UNSUPPORTED, "library built without SOL_ATTN_PROFILE");
#endif
}

int sol_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B, int H, int L, int d,
                             int block, int chunk, float beta, void* stream) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if (chunk < 1) return fail(SOL_ATTN_ERR_ARG, "chunk must be >= 1 (got %d)", chunk);
  if (std::isnan(beta)) return fail(SOL_ATTN_ERR_ARG, "beta is NaN");
  if (!out) return fail(SOL_ATTN_ERR_ARG, "out is NULL");
  if ((rc = check_io(q, k, v, out, B, H, L, d))) return rc;
  const Shape s{B, H, L, d};
  const size_t need = layout(s, nullptr, nullptr);
  if (need > kNoAllocScratchBytes - kNoAllocCtlBytes)
    return fail(SOL_ATTN_ERR_UNSUPPORTED,
                "shape (B=%d, H=%d, L=%d, d=%d) needs %zu bytes of scratch; the allocation-free entry point "
                "holds %zu",
                B, H, L, d, need, kNoAllocScratchBytes - kNoAllocCtlBytes);
  std::lock_guard<std::mutex> lk(g_mu);
  int dev;
  if ((rc = current_device(&dev))) return rc;
  if ((rc = check_arch(dev))) return rc;
  char* base;
  if ((rc = noalloc_base(dev, &base))) return rc;
  Workspace w;   // a view over the fixed array; nothing is allocated
  w.counter = reinterpret_cast<unsigned*>(base);
  w.status = reinterpret_cast<unsigned*>(base) + 32;
  w.base = base + kNoAllocCtlBytes;
  w.bytes = kNoAllocScratchBytes - kNoAllocCtlBytes;
  layout(s, &w, static_cast<char*>(w.base));
  w.shape = s;
  auto st = static_cast<cudaStream_t>(stream);
  // the status word reports on this call only (read by sol_attn_noalloc_status)
  CUDA_TRY(cudaMemsetAsync(w.status, 0, sizeof(unsigned), st));
  if ((rc = run_pool(w, q, k, v, nullptr, st))) return rc;
  if ((rc = run_threshold(w, beta, 0u, nullptr, st))) return rc;
  return run_fused(w, q, k, v, out, chunk, 0u, nullptr, st);
}

int sol_attn_noalloc_status(void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  if (!g_noalloc_base[dev])
    return fail(SOL_ATTN_ERR_STATE, "no allocation-free forward has run on device %d", dev);
  auto st = static_cast<cudaStream_t>(stream);
  unsigned* status = reinterpret_cast<unsigned*>(g_noalloc_base[dev]) + 32;
  unsigned h = 0;
  CUDA_TRY(cudaMemcpyAsync(&h, status, sizeof(h), cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (h) {
    CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(unsigned), st));
    CUDA_TRY(cudaStreamSynchronize(st));
    if (h & kStatusTimeout) return fail(SOL_ATTN_ERR_TIMEOUT, "a bounded device wait gave up (status 0x%x)", h);
    return fail(SOL_ATTN_ERR_DEVICE, "device-side check failed: a tile descriptor was out of range (status 0x%x)",
                h);
  }
  return SOL_ATTN_OK;
}

int sol_attn_topk_route(int B, int H, int L, int d, int block, int k, uint32_t* mask, void* stream) {
  int rc;
  if ((rc = check_shape(B, H, L, d, block))) return rc;
  if (!mask) return fail(SOL_ATTN_ERR_ARG, "mask is NULL");
  std::lock_guard<std::mutex> lk(g_mu);
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Workspace& w = g_ws[dev];
  if (!(w.shape == Shape{B, H, L, d}) || w.stage < 1)
    return fail(SOL_ATTN_ERR_STATE, "topk_route needs a stage_pool or forward of the same shape first");
  const int N = (L + kBlock - 1) / kBlock;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t bytes = BH * N * N * sizeof(float);
  if (w.topk_map_bytes < bytes) {
    if (w.topk_map) CUDA_TRY(cudaFree(w.topk_map));
    w.topk_map = nullptr;
    w.topk_map_bytes = 0;
    CUDA_TRY(cudaMalloc(&w.topk_map, bytes));
    w.topk_map_bytes = bytes;
  }
  auto st = static_cast<cudaStream_t>(stream);
  float* map = static_cast<float*>(w.topk_map);
  const float isd = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  const dim3 grid((N + kMapTile - 1) / kMapTile, (N + kMapTile - 1) / kMapTile, static_cast<unsigned>(BH));
  const size_t msm = 2u * kMapTile * (d + 1) * sizeof(float);
  static bool attr_set[kMaxDevices] = {false};
  if (!attr_set[dev]) {
    CUDA_TRY(cudaFuncSetAttribute(proxy_map_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(2u * kMapTile * 129 * sizeof(float))));
    CUDA_TRY(cudaFuncSetAttribute(proxy_map_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(2u * kMapTile * 65 * sizeof(float))));
    CUDA_TRY(cudaFuncSetAttribute(topk_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kMaxMaskWords * 32 * sizeof(uint32_t))));
    attr_set[dev] = true;
  }
  if (d == 128)
    proxy_map_kernel<128><<<grid, 256, msm, st>>>(w.qbar, w.kbar, N, isd, map);
  else
    proxy_map_kernel<64><<<grid, 256, msm, st>>>(w.qbar, w.kbar, N, isd, map);
  CUDA_TRY(cudaGetLastError());
  topk_mask_kernel<<<static_cast<unsigned>(BH * N), 256, static_cast<size_t>(N) * sizeof(uint32_t), st>>>(map, N, k,
                                                                                                        mask);
  CUDA_TRY(cudaGetLastError());
  return SOL_ATTN_OK;
}

}  // extern "C"
