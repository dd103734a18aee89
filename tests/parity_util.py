"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same seeded bf16 inputs.

Tolerances (the workload statement): selection masks bit-exact except for
blocks whose proxy logit lies within 1e-4 of the row threshold (counted and
reported); outputs within max-abs 2e-2 and relative-l2 5e-3.
"""
import math

import numpy as np

from oracle import proxy_row, sol_attn_head
from synth import bf16_bits_to_f64

BAND = 1e-4
MAX_ABS = 2e-2
REL_L2 = 5e-3


def to_device(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(qb, kb, vb, beta, chunk, flags=0, debug=True):
    """Run the forward on bf16 bits; returns (out float32 numpy, DebugBuffers or None, counts numpy)."""
    import torch

    import block_sparse_attention_moments_b200 as sa
    B, H, L, d = qb.shape
    q, k, v = to_device(qb), to_device(kb), to_device(vb)
    dbg = sa.DebugBuffers(B, H, L, d) if debug else None
    out = sa.forward(q, k, v, beta, chunk, flags=flags | sa.FLAG_SYNC_CHECK, debug=dbg)
    counts = sa.stats(B, H, L)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), dbg, counts.cpu().numpy()


class Report:
    def __init__(self):
        self.band_mismatch = 0
        self.rows = 0
        self.max_abs = 0.0
        self.num = 0.0
        self.den = 0.0

    @property
    def rel_l2(self):
        return math.sqrt(self.num / self.den) if self.den > 0 else 0.0

    def check(self):
        assert self.max_abs <= MAX_ABS, f"max-abs {self.max_abs:.3e} > {MAX_ABS}"
        assert self.rel_l2 <= REL_L2, f"rel-l2 {self.rel_l2:.3e} > {REL_L2}"

    def __str__(self):
        return (f"rows={self.rows} max_abs={self.max_abs:.3e} rel_l2={self.rel_l2:.3e} "
                f"band_mismatches={self.band_mismatch}")


def compare_head(rep, qb, kb, vb, b, h, beta, gpu_out, gpu_sel, gpu_counts, rows=None, exact_only=False,
                 dbg=None):
    """Compare one (b, h) slice on the given query blocks (default all)."""
    q = bf16_bits_to_f64(qb[b, h])
    k = bf16_bits_to_f64(kb[b, h])
    v = bf16_bits_to_f64(vb[b, h])
    L = q.shape[0]
    N = -(-L // 64)
    rows = list(range(N)) if rows is None else list(rows)
    ref = sol_attn_head(q, k, v, beta, exact_only=exact_only, rows=rows)
    sel_gpu = np.asarray(gpu_sel[b, h], dtype=bool)
    override_rows = []
    for i in rows:
        diff = np.nonzero(sel_gpu[i] != ref["sel"][i])[0]
        if len(diff):
            s = proxy_row(ref["qbar"][i], ref["kbar"])
            gap = np.abs(s[diff] - ref["tau"][i])
            assert (gap < BAND).all(), (f"mask mismatch outside the {BAND} band at head ({b},{h}) row {i}: "
                                        f"blocks {diff[gap >= BAND].tolist()} gap {gap[gap >= BAND].tolist()}")
            rep.band_mismatch += len(diff)
            override_rows.append(i)
        assert gpu_counts[b, h, i] == sel_gpu[i].sum()
    O = ref["O"]
    if override_rows:   # evaluate those rows with the GPU's (equally valid) selection
        alt = sol_attn_head(q, k, v, beta, exact_only=exact_only, rows=override_rows, sel_override=sel_gpu)
        for i in override_rows:
            lo, hi = 64 * i, min(64 * i + 64, L)
            O[lo:hi] = alt["O"][lo:hi]
    if dbg is not None:   # pooled statistics and thresholds
        # fp32 pooling of bf16 inputs vs fp64: a few fp32 ulps of the block sums
        np.testing.assert_allclose(dbg["qbar"][b, h], ref["qbar"], rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(dbg["kbar"][b, h], ref["kbar"], rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(dbg["vhat"][b, h], ref["vhat"], rtol=1e-5, atol=1e-4)
        if not math.isinf(beta):
            # fp64 moments of fp32 pooled values, rounded to fp32: well inside the mask band
            np.testing.assert_allclose(dbg["tau"][b, h], ref["tau"], rtol=2e-6, atol=BAND / 2)
            np.testing.assert_allclose(dbg["mu"][b, h], ref["mu"], rtol=2e-6, atol=BAND / 2)
            np.testing.assert_allclose(dbg["sigma"][b, h], ref["sigma"], rtol=2e-6, atol=BAND / 2)
    for i in rows:
        lo, hi = 64 * i, min(64 * i + 64, L)
        g = gpu_out[b, h, lo:hi].astype(np.float64)
        r = O[lo:hi]
        rep.max_abs = max(rep.max_abs, float(np.abs(g - r).max()))
        rep.num += float(((g - r) ** 2).sum())
        rep.den += float((r ** 2).sum())
        rep.rows += 1
    return rep


def debug_numpy(dbg):
    return dict(qbar=dbg.qbar.cpu().numpy(), kbar=dbg.kbar.cpu().numpy(), vhat=dbg.vhat.cpu().numpy(),
                tau=dbg.tau.cpu().numpy(), mu=dbg.mu.cpu().numpy(), sigma=dbg.sigma.cpu().numpy())
