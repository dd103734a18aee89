"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the fp64 CPU oracle and the CUDA path read the
exact bf16 values produced here.

Workloads stand in for the activations of the video/image diffusion
transformers measured in "Sol-Attn: Accelerating Video Generation Inference via
On-the-Fly Attention Sparsification" (experiments: setup), whose activations
and weights are not available.  Tokens sit in raster order on a
(frames x height x width) latent grid; Q and K share a smooth positional
signal built from random Fourier features of the normalised grid coordinates,
plus independent unit Gaussian noise; V is unit Gaussian.

Recipe (one reading of the workload text, stated here and in the design notes):
  * F = 64 frequencies w_k ~ N(0, 3^2 I_3) and phases b_k ~ U[0, 2*pi).
  * g_k(p) = sqrt(2) * cos(w_k . p + b_k)   (unit variance per feature).
  * Q = A * [g, 0_{d-64}] + N(0,1),  K = A * [g, 0_{d-64}] + N(0,1),  V ~ N(0,1),
    the same g for Q and K and for every (batch, head).
  * A = 2.0 for the two small shapes, 3.0 for the large ones.
  * numpy PCG64: the Fourier frequencies and phases come from the stream seeded
    with (1000 + shape index); each (batch, head) slice b*H + h draws its Q noise,
    K noise and V, in that order, from its own stream seeded with
    SeedSequence([1000 + shape index, b*H + h]), so any subset of heads can be
    generated alone.
  * values are rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "grid_coords", "fourier_inputs", "gauss_inputs", "ramp_inputs", "offset_inputs",
    "near_block_constant_keys", "bf16_round", "bf16_bits_to_f64", "f32_to_bf16_bits", "f32_to_bf16_bits_np",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: tuple            # (frames, height, width); L = prod(grid)
    d: int
    chunk: int
    betas: tuple            # finite betas; -inf marks the select-all run
    amp: float
    seed: int
    block: int = 64

    @property
    def L(self) -> int:
        f, h, w = self.grid
        return f * h * w

    @property
    def N(self) -> int:
        return -(-self.L // self.block)


NEG_INF = float("-inf")

# The five shapes of the workload list: a tiny check, a small bf16 case, an
# image-generation shape, and Wan-2.1-14B-like / HunyuanVideo-13B-like
# self-attention with a ragged 16-token final block.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, (4, 16, 16), 64, 4, (1.0,), 2.0, 1000),
    "small": Workload("small", 1, 2, (4, 32, 32), 128, 16, (0.5, 1.0, 1.5, NEG_INF), 2.0, 1001),
    "image": Workload("image", 2, 24, (1, 128, 128), 128, 32, (1.0,), 3.0, 1002),
    "wan": Workload("wan", 1, 40, (21, 45, 80), 128, 64, (0.75, 1.0, 1.5), 3.0, 1003),
    "hunyuan": Workload("hunyuan", 1, 24, (33, 45, 80), 128, 64, (0.75, 1.0, 1.5, NEG_INF), 3.0, 1004),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even) and return the raw uint16 bits.

    Uses torch's float32 -> bfloat16 cast (round-to-nearest-even, multithreaded)
    when torch is importable; ``f32_to_bf16_bits_np`` is the plain numpy form
    and the tests check that the two agree bit for bit."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        return f32_to_bf16_bits_np(x)
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32_to_bf16_bits_np(x: np.ndarray) -> np.ndarray:
    """numpy round-to-nearest-even float32 -> bf16 bits (finite inputs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # Finite inputs only (the generators make no NaN/Inf): RNE on the bit
    # pattern; the largest finite pattern plus the rounding bias stays < 2^32.
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to float64 exactly."""
    u = bits.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value and return it as float64."""
    return bf16_bits_to_f64(f32_to_bf16_bits(x))


def grid_coords(grid) -> np.ndarray:
    """Normalised (f, y, x) coordinates of every token in raster order; [L, 3] float64.
    A dimension of size 1 maps to 0."""
    axes = [np.zeros(1) if n == 1 else np.arange(n, dtype=np.float64) / (n - 1) for n in grid]
    f, y, x = np.meshgrid(*axes, indexing="ij")
    return np.stack([f.ravel(), y.ravel(), x.ravel()], axis=1)


def _fourier_features(rng: np.random.Generator, grid, n_feat: int = 64) -> np.ndarray:
    w = rng.normal(0.0, 3.0, size=(n_feat, 3))
    b = rng.uniform(0.0, 2.0 * math.pi, size=(n_feat,))
    p = grid_coords(grid)
    return (math.sqrt(2.0) * np.cos(p @ w.T + b)).astype(np.float32)  # [L, n_feat]


def fourier_inputs(wl: Workload, heads: Optional[list] = None):
    """bf16 Q, K, V bits for a workload as uint16 arrays of shape [B, H, L, d].

    ``heads`` restricts generation to a list of flattened (b*H + h) indices.
    Every head has its own stream, so a head's values do not depend on which
    heads were requested.  Skipped heads are returned as zeros (callers that
    ask for a subset only read that subset).
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    g = _fourier_features(rng, wl.grid)                      # [L, 64]
    L, d = wl.L, wl.d
    nf = g.shape[1]
    signal = np.zeros((L, d), dtype=np.float32)
    signal[:, :min(nf, d)] = wl.amp * g[:, :min(nf, d)]
    shape = (wl.B, wl.H, L, d)
    q = np.zeros(shape, np.uint16)
    k = np.zeros(shape, np.uint16)
    v = np.zeros(shape, np.uint16)
    todo = [bh for bh in range(wl.B * wl.H) if heads is None or bh in set(heads)]

    def one(bh):
        b, h = divmod(bh, wl.H)
        hr = np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.seed, bh])))
        nz = hr.standard_normal(size=(3, L, d), dtype=np.float32)
        q[b, h] = f32_to_bf16_bits(signal + nz[0])
        k[b, h] = f32_to_bf16_bits(signal + nz[1])
        v[b, h] = f32_to_bf16_bits(nz[2])

    # Heads are independent streams, so threads only change the wall time.
    import concurrent.futures as cf
    import os
    with cf.ThreadPoolExecutor(max_workers=min(len(todo), os.cpu_count() or 1) or 1) as ex:
        list(ex.map(one, todo))
    return q, k, v


def gauss_inputs(B: int, H: int, L: int, d: int, seed: int):
    """iid N(0,1) bf16 Q, K, V bits of shape [B, H, L, d] (the Gaussian-logit case)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=(3, B, H, L, d), dtype=np.float32)
    return f32_to_bf16_bits(x[0]), f32_to_bf16_bits(x[1]), f32_to_bf16_bits(x[2])


def ramp_inputs(B: int, H: int, L: int, d: int, q_amp: float, k_lo: float, k_hi: float, seed: int,
                v_amp: float = 1.0):
    """bf16 Q, K, V bits [B, H, L, d]: Q ~ N(0, q_amp^2), V ~ N(0, v_amp^2), and K ~ N(0, s_t^2)
    with the scale s_t rising linearly from k_lo (first token) to k_hi (last), so a row's
    largest logits sit late in the sequence."""
    rng = np.random.default_rng(seed)
    s = (k_lo + (k_hi - k_lo) * np.arange(L, dtype=np.float64) / max(L - 1, 1)).astype(np.float32)
    q = rng.standard_normal((B, H, L, d), dtype=np.float32) * np.float32(q_amp)
    k = rng.standard_normal((B, H, L, d), dtype=np.float32) * s[None, None, :, None]
    v = rng.standard_normal((B, H, L, d), dtype=np.float32) * np.float32(v_amp)
    return f32_to_bf16_bits_np(q), f32_to_bf16_bits_np(k), f32_to_bf16_bits_np(v)


def offset_inputs(B: int, H: int, L: int, d: int, a: float, sign: float, noise: float, seed: int):
    """bf16 Q, K, V bits [B, H, L, d] whose logits all sit near sign * a^2 / sqrt(d):
    Q = a e_0 + noise N(0, I), K = sign a e_0 + noise N(0, I), V ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, d), dtype=np.float32) * np.float32(noise)
    k = rng.standard_normal((B, H, L, d), dtype=np.float32) * np.float32(noise)
    q[..., 0] += np.float32(a)
    k[..., 0] += np.float32(sign * a)
    v = rng.standard_normal((B, H, L, d), dtype=np.float32)
    return f32_to_bf16_bits_np(q), f32_to_bf16_bits_np(k), f32_to_bf16_bits_np(v)


def custom_fourier(B: int, H: int, grid, d: int, amp: float, seed: int):
    """Fourier-feature inputs for an arbitrary grid (edge-case shapes in tests)."""
    wl = Workload("custom", B, H, tuple(grid), d, 1, (1.0,), amp, seed)
    return fourier_inputs(wl)


def near_block_constant_keys(kb: np.ndarray, eps: float, seed: int, block: int = 64) -> np.ndarray:
    """bf16 key bits [B, H, L, d] in which every key of a 64-token block is the
    block's first key of ``kb`` plus eps * N(0, 1) noise: keys nearly constant
    within a block, the regime in which the approximation of unselected blocks
    carries a large share of each row's softmax mass."""
    k = bf16_bits_to_f64(kb).astype(np.float32)
    L = k.shape[2]
    for j in range(0, L, block):
        k[:, :, j:j + block, :] = k[:, :, j:j + 1, :]
    rng = np.random.default_rng(seed)
    k = k + np.float32(eps) * rng.standard_normal(size=k.shape, dtype=np.float32)
    return f32_to_bf16_bits(k)

