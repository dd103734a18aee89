"""The allocation-free entry point, sol_attn_forward_noalloc.

It serves callers that must not allocate device memory themselves or have the
library allocate it for them (a fixed memory pool, a serving loop in which a
cudaMalloc could synchronise the device).  Its scratch is a fixed array inside
the library.  These tests call it through the C ABI: it runs the same kernels
on the same inputs as the regular sol_attn_forward, so its output must equal
that forward's bit for bit, on two calls in a row with different inputs (so
nothing left in the shared array from one call leaks into the next) and on a
shape whose scratch nearly fills the array.  One call is also checked against
the fp64 oracle, and the status query is exercised.  The file is named to be
collected last.
"""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_moments_b200 as sa
from synth import WORKLOADS, bf16_bits_to_f64, custom_fourier, fourier_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3
SCRATCH_BYTES = 96 << 20   # the fixed array; 256 bytes of it hold the work counter and status word


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
    rc = sa.lib().sol_attn_noalloc_status(stream)
    assert rc == 0, sa.lib().sol_attn_error_string(rc).decode()
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def _regular(q, k, v, beta, chunk):
    import torch
    out = sa.forward(q, k, v, beta, chunk, flags=sa.FLAG_SYNC_CHECK)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")


def test_two_calls_in_a_row_equal_the_regular_forward():
    wl = WORKLOADS["small"]
    first = [_dev(x) for x in fourier_inputs(wl)]
    second = [_dev(x) for x in custom_fourier(2, 3, (1, 1, 3000), 128, 3.0, seed=77)]
    a1 = _noalloc(*first, 1.0, wl.chunk)
    a2 = _noalloc(*second, 0.75, 32)
    assert np.array_equal(a1, _regular(*first, 1.0, wl.chunk))
    assert np.array_equal(a2, _regular(*second, 0.75, 32))
    # and once more after the regular path ran, with the first inputs again
    assert np.array_equal(_noalloc(*first, 1.0, wl.chunk), a1)


def test_matches_the_oracle():
    from oracle import sol_attn_head
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    got = _noalloc(_dev(qb), _dev(kb), _dev(vb), 1.0, wl.chunk)
    for h in range(wl.H):
        ref = sol_attn_head(bf16_bits_to_f64(qb[0, h]), bf16_bits_to_f64(kb[0, h]), bf16_bits_to_f64(vb[0, h]), 1.0)
        g = got[0, h].astype(np.float64)
        assert np.abs(g - ref["O"]).max() <= MAX_ABS
        assert np.linalg.norm(g - ref["O"]) / np.linalg.norm(ref["O"]) <= REL_L2


def test_shape_near_the_scratch_limit():
    # the Wan-like shape: B*H*N*d*14 + B*H*d*d*8 bytes, about 86 of the 96 MiB
    wl = WORKLOADS["wan"]
    need = sa.workspace_bytes(wl.B, wl.H, wl.L, wl.d)
    assert 0.85 * SCRATCH_BYTES < need <= SCRATCH_BYTES - 256
    q, k, v = (_dev(x) for x in fourier_inputs(wl))
    a = _noalloc(q, k, v, 1.0, wl.chunk)
    assert np.array_equal(a, _regular(q, k, v, 1.0, wl.chunk))


def test_shape_one_block_past_the_limit_is_rejected_without_touching_the_device():
    # the largest H at L = 4096, d = 128 whose scratch fits, then one head more
    fake = ctypes.c_void_p(0x100000)
    out = ctypes.c_void_p(0x100000 + (1 << 40))
    L, d = 4096, 128
    H = 1
    while sa.workspace_bytes(1, H + 1, L, d) <= SCRATCH_BYTES - 256:
        H += 1
    assert sa.workspace_bytes(1, H + 1, L, d) > SCRATCH_BYTES - 256
    rc = sa.lib().sol_attn_forward_noalloc(fake, fake, fake, out, 1, H + 1, L, d, 64, 64, ctypes.c_float(1.0), None)
    assert rc == -2
    msg = sa.lib().sol_attn_error_string(rc).decode()
    assert "allocation-free" in msg and "scratch" in msg
    rc = sa.lib().sol_attn_forward_noalloc(fake, fake, fake, out, 1, 64, 1 << 20, 128, 64, 64,
                                           ctypes.c_float(1.0), None)
    assert rc == -2
