"""The allocation-free entry point, sol_attn_forward_noalloc.

It serves callers that must not allocate device memory themselves or have the
library allocate it for them (a fixed memory pool, a serving loop in which a
cudaMalloc could synchronise the device).  Its scratch is a fixed array inside
the library.  These tests call it through the C ABI and check that two calls
in a row, with different inputs, match the regular sol_attn_forward within the
parity tolerance, so nothing left in the shared array from one call leaks
into the next.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_moments_b200 as sa
from synth import WORKLOADS, custom_fourier, fourier_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(q, k, v, beta, chunk):
    import torch
    B, H, L, d = q.shape
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream().cuda_stream
    rc = sa.lib().sol_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, L, d,
                                           64, chunk, ctypes.c_float(beta), stream)
    assert rc == 0, sa.lib().sol_attn_error_string(rc).decode()
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def _regular(q, k, v, beta, chunk):
    import torch
    out = sa.forward(q, k, v, beta, chunk, flags=sa.FLAG_SYNC_CHECK)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def _close(a, b):
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert err <= MAX_ABS and rel <= REL_L2, (err, rel)


def test_two_calls_in_a_row_match_the_regular_forward():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    wl = WORKLOADS["small"]
    first = [_dev(x) for x in fourier_inputs(wl)]
    second = [_dev(x) for x in custom_fourier(2, 3, (1, 1, 3000), 128, 3.0, seed=77)]
    a1 = _noalloc(*first, 1.0, wl.chunk)
    a2 = _noalloc(*second, 0.75, 32)
    _close(a1, _regular(*first, 1.0, wl.chunk))
    _close(a2, _regular(*second, 0.75, 32))
    # and once more after the regular path ran, with the first inputs again
    _close(_noalloc(*first, 1.0, wl.chunk), a1)


def test_large_shape_is_rejected_without_touching_the_device():
    fake = ctypes.c_void_p(0x100000)
    out = ctypes.c_void_p(0x100000 + (1 << 40))
    rc = sa.lib().sol_attn_forward_noalloc(fake, fake, fake, out, 1, 64, 1 << 20, 128, 64, 64,
                                           ctypes.c_float(1.0), None)
    assert rc == -2
    msg = sa.lib().sol_attn_error_string(rc).decode()
    assert "allocation-free" in msg and "scratch" in msg
