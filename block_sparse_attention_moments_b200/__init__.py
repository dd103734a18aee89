"""Sol-Attn single-pass sparse attention forward for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/sol_attn.h`` (libsol_attn.so):
it only checks tensor properties and marshals pointers; every step of the
forward runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing or fails to load, every call raises.

Method: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
Attention Sparsification" (block pooling, moment-based thresholds
τ_i = μ_i + β σ_i, chunk-wise streaming routing, exact attention on the
selected blocks and zeroth-order proxy-score reuse for the rest).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "FLAG_SELECT_ALL", "FLAG_EXACT_ONLY", "FLAG_SYNC_CHECK", "FLAG_TEST_STALL", "FLAG_FIRST_ORDER", "SolAttnError", "lib", "lib_path",
    "forward", "stats", "forward_host", "stage_pool", "stage_threshold", "stage_fused",
    "workspace_bytes", "release", "kernels_per_forward", "DebugBuffers", "EXPORTED_SYMBOLS", "topk_route",
    "executed_flops", "BLOCK",
]

FLAG_SELECT_ALL = 0x1
FLAG_EXACT_ONLY = 0x2
FLAG_SYNC_CHECK = 0x4
FLAG_TEST_STALL = 0x8   # failure-path test only: every bounded device wait runs out (see sol_attn.h)
FLAG_FIRST_ORDER = 0x10  # first-order expansion for unselected blocks (extension; see sol_attn.h)
BLOCK = 64

_PKG = os.path.dirname(os.path.abspath(__file__))
# SOL_ATTN_PROFILE=1 selects the build with per-role cycle accounting.
_LIB_PATH = os.path.join(_PKG, "libsol_attn_profile.so" if os.environ.get("SOL_ATTN_PROFILE") == "1"
                         else "libsol_attn.so")
_lib = None

# Every entry point declared in include/sol_attn.h.
EXPORTED_SYMBOLS = (
    "sol_attn_forward", "sol_attn_forward_ex", "sol_attn_stats", "sol_attn_forward_host",
    "sol_attn_stage_pool", "sol_attn_stage_threshold", "sol_attn_stage_fused",
    "sol_attn_workspace_bytes", "sol_attn_release", "sol_attn_error_string",
    "sol_attn_kernels_per_forward", "sol_attn_forward_noalloc", "sol_attn_profile_read",
    "sol_attn_noalloc_status", "sol_attn_topk_route",
)


class SolAttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"sol_attn error {code}: {msg}")
        self.code = code


class _Debug(ctypes.Structure):
    _fields_ = [("qbar", ctypes.c_void_p), ("kbar", ctypes.c_void_p), ("vhat", ctypes.c_void_p),
                ("mu", ctypes.c_void_p), ("sigma", ctypes.c_void_p), ("tau", ctypes.c_void_p),
                ("mask", ctypes.c_void_p)]


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """Load libsol_attn.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing; build it with "
                           "`python -m block_sparse_attention_moments_b200._build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i, f, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint
    L.sol_attn_forward.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.sol_attn_forward_ex.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, u, ctypes.POINTER(_Debug), vp]
    L.sol_attn_stats.argtypes = [vp, i, i, i, i, vp]
    L.sol_attn_forward_host.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, u]
    L.sol_attn_stage_pool.argtypes = [vp, vp, vp, i, i, i, i, i, ctypes.POINTER(_Debug), vp]
    L.sol_attn_stage_threshold.argtypes = [i, i, i, i, i, f, u, ctypes.POINTER(_Debug), vp]
    L.sol_attn_stage_fused.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, u, ctypes.POINTER(_Debug), vp]
    L.sol_attn_workspace_bytes.argtypes = [i, i, i, i, i]
    L.sol_attn_workspace_bytes.restype = ctypes.c_size_t
    L.sol_attn_release.argtypes = []
    L.sol_attn_error_string.argtypes = [i]
    L.sol_attn_error_string.restype = ctypes.c_char_p
    L.sol_attn_kernels_per_forward.argtypes = []
    L.sol_attn_forward_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.sol_attn_profile_read.argtypes = [vp, i, i]
    L.sol_attn_noalloc_status.argtypes = [vp]
    L.sol_attn_topk_route.argtypes = [i, i, i, i, i, i, vp, vp]
    for name in ("sol_attn_forward", "sol_attn_forward_ex", "sol_attn_stats", "sol_attn_forward_host",
                 "sol_attn_stage_pool", "sol_attn_stage_threshold", "sol_attn_stage_fused", "sol_attn_release",
                 "sol_attn_kernels_per_forward", "sol_attn_forward_noalloc", "sol_attn_profile_read",
                 "sol_attn_noalloc_status", "sol_attn_topk_route"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(rc: int):
    if rc != 0:
        raise SolAttnError(rc, lib().sol_attn_error_string(rc).decode())


def _stream_handle(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check_qkv(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bfloat16")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dim() != 4 or t.shape != q.shape:
            raise ValueError("q, k, v must share one [B, H, L, d] shape")
    return tuple(q.shape)


class DebugBuffers:
    """Device buffers for the debug exports of sol_attn_forward_ex."""

    def __init__(self, B: int, H: int, L: int, d: int, device=None):
        import torch
        N = -(-L // BLOCK)
        nw = -(-N // 32)
        kw = dict(device=device or "cuda", dtype=torch.float32)
        self.qbar = torch.empty(B, H, N, d, **kw)
        self.kbar = torch.empty(B, H, N, d, **kw)
        self.vhat = torch.empty(B, H, N, d, **kw)
        self.mu = torch.empty(B, H, N, **kw)
        self.sigma = torch.empty(B, H, N, **kw)
        self.tau = torch.empty(B, H, N, **kw)
        self.mask = torch.zeros(B, H, N, nw, device=device or "cuda", dtype=torch.int32)

    def struct(self) -> _Debug:
        return _Debug(self.qbar.data_ptr(), self.kbar.data_ptr(), self.vhat.data_ptr(), self.mu.data_ptr(),
                      self.sigma.data_ptr(), self.tau.data_ptr(), self.mask.data_ptr())

    def selection(self):
        """Selection mask as a [B, H, N, N] bool tensor."""
        import torch
        B, H, N, nw = self.mask.shape
        w = self.mask.to(torch.int64) & 0xFFFFFFFF
        bits = (w[..., None] >> torch.arange(32, device=w.device)) & 1
        return bits.reshape(B, H, N, nw * 32)[..., :N].bool()


def forward(q, k, v, beta: float, chunk: int, *, flags: int = 0, out=None, debug: Optional[DebugBuffers] = None,
            stream=None):
    """Sol-Attn forward on bf16 CUDA tensors [B, H, L, d]; returns out (bf16)."""
    import torch
    B, H, L, d = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    dbg = ctypes.pointer(debug.struct()) if debug is not None else None
    _check(lib().sol_attn_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, L, d, BLOCK,
                                     int(chunk), float(beta), int(flags), dbg, _stream_handle(stream)))
    return out


def stats(B: int, H: int, L: int, stream=None):
    """Per-row selected-block counts |S_i| of the last forward, as int32 [B, H, N]."""
    import torch
    N = -(-L // BLOCK)
    counts = torch.empty(B, H, N, device="cuda", dtype=torch.int32)
    _check(lib().sol_attn_stats(counts.data_ptr(), B, H, L, BLOCK, _stream_handle(stream)))
    return counts


def forward_host(q, k, v, beta: float, chunk: int, *, flags: int = 0, out=None):
    """Forward on host arrays (numpy uint16 bf16 bits or CPU bf16 tensors); copies are
    done by the library (host -> device -> host) and the call is synchronous."""
    import numpy as np

    def ptr(x):
        if hasattr(x, "data_ptr"):
            if not x.is_contiguous() or x.is_cuda:
                raise ValueError("host tensors must be contiguous CPU tensors")
            return x.data_ptr(), tuple(x.shape)
        if not isinstance(x, np.ndarray) or x.dtype != np.uint16 or not x.flags.c_contiguous:
            raise ValueError("host arrays must be C-contiguous numpy uint16 arrays of raw bf16 bits")
        return x.ctypes.data, x.shape

    (pq, shape), (pk, sk), (pv, sv) = ptr(q), ptr(k), ptr(v)
    if not (shape == sk == sv) or len(shape) != 4:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    B, H, L, d = shape
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    po, so = ptr(out)
    if so != shape:
        raise ValueError("out has the wrong shape")
    _check(lib().sol_attn_forward_host(pq, pk, pv, po, B, H, L, d, BLOCK, int(chunk), float(beta), int(flags)))
    return out


def stage_pool(q, k, v, *, debug: Optional[DebugBuffers] = None, stream=None):
    B, H, L, d = _check_qkv(q, k, v)
    dbg = ctypes.pointer(debug.struct()) if debug is not None else None
    _check(lib().sol_attn_stage_pool(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L, d, BLOCK, dbg,
                                     _stream_handle(stream)))


def stage_threshold(B: int, H: int, L: int, d: int, beta: float, *, flags: int = 0,
                    debug: Optional[DebugBuffers] = None, stream=None):
    dbg = ctypes.pointer(debug.struct()) if debug is not None else None
    _check(lib().sol_attn_stage_threshold(B, H, L, d, BLOCK, float(beta), int(flags), dbg, _stream_handle(stream)))


def stage_fused(q, k, v, out, chunk: int, *, flags: int = 0, debug: Optional[DebugBuffers] = None, stream=None):
    B, H, L, d = _check_qkv(q, k, v)
    dbg = ctypes.pointer(debug.struct()) if debug is not None else None
    _check(lib().sol_attn_stage_fused(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, L, d, BLOCK,
                                      int(chunk), int(flags), dbg, _stream_handle(stream)))
    return out


def topk_route(B: int, H: int, L: int, d: int, k: int, stream=None):
    """Comparison top-k router (measurement aid): from the pooled Q̄, K̄ of the
    last pooling of this shape, materialise every head's proxy map in HBM and
    keep each row's k largest blocks; returns the [B, H, N] selection as a bool
    tensor view of the mask bits (see sol_attn_topk_route)."""
    import torch
    N = -(-L // BLOCK)
    nw = -(-N // 32)
    mask = torch.zeros(B, H, N, nw, device="cuda", dtype=torch.int32)
    _check(lib().sol_attn_topk_route(B, H, L, d, BLOCK, int(k), mask.data_ptr(), _stream_handle(stream)))
    return mask


def workspace_bytes(B: int, H: int, L: int, d: int) -> int:
    return int(lib().sol_attn_workspace_bytes(B, H, L, d, BLOCK))


# Slot names of the profiling build's counters, in the order of the ProfSlot
# enum in csrc/fused.cuh.
PROFILE_SLOTS = (
    "route.wait_item_empty", "k.wait_desc", "k.wait_q_empty", "k.wait_stage", "v.wait_desc", "v.wait_stage",
    "s.wait_desc", "s.wait_q", "s.wait_buffer", "s.wait_k", "s.issue",
    "pv.wait_desc", "pv.wait_p", "pv.wait_v", "pv.issue",
    "softmax.wait_desc", "softmax.wait_s", "softmax.wait_handoff", "softmax.wait_o", "softmax.wait_exchange",
    "softmax.pass", "softmax.meet", "softmax.epilogue", "softmax.tiles", "softmax.rescales",
    "sched.wait_item", "sched.wait_ring",
    "total.route", "total.k", "total.v", "total.s", "total.pv", "total.softmax", "total.sched",
    "softmax.tmem_load", "softmax.exp_block", "sched.walk", "sched.descriptor", "route.item",
)


def profile_read(reset: bool = True) -> dict:
    """Cycle counters of the profiling build, summed over CTAs (see sol_attn_profile_read)."""
    buf = (ctypes.c_uint64 * 48)()
    _check(lib().sol_attn_profile_read(buf, 48, 1 if reset else 0))
    return {name: int(buf[k]) for k, name in enumerate(PROFILE_SLOTS)}


def release():
    _check(lib().sol_attn_release())


def kernels_per_forward() -> int:
    return int(lib().sol_attn_kernels_per_forward())


def executed_flops(selected_pairs: int, B: int, H: int, L: int, d: int, *, approx: bool = True) -> float:
    """FLOPs of one forward by the method's accounting: 4*64*64*d per selected
    (query block, key block) pair (QK^T and PV of the exact inner loop), plus the
    proxy work: 4*64*d per (query block, pooled key) for the token-to-block tile
    and its value product (when the approximation runs), and 2*d per routing dot
    product Q̄_i·K̄_j."""
    N = -(-L // BLOCK)
    exact = 4.0 * BLOCK * BLOCK * d * float(selected_pairs)
    proxy = 4.0 * BLOCK * d * N * N * B * H if approx else 0.0
    route = 2.0 * d * N * N * B * H
    return exact + proxy + route
