"""Host-side checks of the C ABI: the library loads without a GPU, exports
every entry point declared in include/sol_attn.h, and rejects bad arguments
before touching the device."""
import ctypes
import math
import os
import re

import pytest

import block_sparse_attention_moments_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sol_attn.h")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_moments_b200 import _build
    _build.build()
    return sa.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sol_attn_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_symbols() == sorted(sa.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # the shared object really is the in-tree build
    assert os.path.dirname(sa.lib_path()) == os.path.join(ROOT, "block_sparse_attention_moments_b200")


def test_argument_errors_without_gpu(lib):
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
    mis = ctypes.c_void_p(0x10008)
    f = lib.sol_attn_forward_ex
    assert f(None, fake, fake, fake, 1, 1, 128, 128, 64, 4, 1.0, 0, None, None) == -1       # null q
    assert f(fake, fake, fake, fake, 0, 1, 128, 128, 64, 4, 1.0, 0, None, None) == -1       # B = 0
    assert f(fake, fake, fake, fake, 1, 1, 128, 96, 64, 4, 1.0, 0, None, None) == -2        # d = 96
    assert f(fake, fake, fake, fake, 1, 1, 128, 128, 32, 4, 1.0, 0, None, None) == -2       # block = 32
    assert f(fake, fake, fake, fake, 1, 1, 1 << 21, 128, 64, 4, 1.0, 0, None, None) == -2   # L too large
    assert f(fake, fake, fake, fake, 1, 1, 128, 128, 64, 0, 1.0, 0, None, None) == -1       # chunk = 0
    # B*H beyond 65535 (gridDim.y of the pooling and moment kernels)
    assert f(fake, fake, fake, ctypes.c_void_p(1 << 44), 1, 65536, 64, 64, 64, 4, 1.0, 0, None, None) == -2
    assert f(fake, fake, fake, ctypes.c_void_p(1 << 44), 256, 257, 64, 64, 64, 4, 1.0, 0, None, None) == -2
    assert "65535" in lib.sol_attn_error_string(-2).decode()
    assert f(fake, fake, fake, fake, 1, 1, 128, 128, 64, 4, math.nan, 0, None, None) == -1  # NaN beta
    assert f(mis, fake, fake, ctypes.c_void_p(0x90000), 1, 1, 128, 128, 64, 4, 1.0, 0, None, None) == -3
    assert f(fake, fake, fake, fake, 1, 1, 128, 128, 64, 4, 1.0, 0, None, None) == -1       # out aliases q
    msg = lib.sol_attn_error_string(-1).decode()
    assert "invalid argument" in msg and "overlap" in msg
    assert lib.sol_attn_stats(None, 1, 1, 128, 64, None) == -1
    assert lib.sol_attn_forward_host(None, None, None, None, 1, 1, 128, 128, 64, 4, 1.0, 0) == -1


def test_workspace_size_is_host_arithmetic(lib):
    B, H, L, d = 1, 40, 75600, 128
    N = -(-L // 64)
    expect_min = B * H * N * d * (4 + 4 + 2 + 2) + B * H * d * d * 8
    got = sa.workspace_bytes(B, H, L, d)
    assert expect_min <= got <= expect_min + 64 * 1024 * 1024
    assert sa.workspace_bytes(1, 1, 128, 96) == 0
    # the longest sequence is 2^20 tokens (16384 pooled blocks, the fused kernel's mask capacity)
    assert sa.workspace_bytes(1, 1, 1 << 20, 64) > 0
    assert sa.workspace_bytes(1, 1, (1 << 20) + 1, 64) == 0
    assert sa.kernels_per_forward() == 4


def test_executed_flops_accounting():
    # 4*64*64*d per selected pair, 4*64*d per (query block, pooled key), 2*d per routing dot
    B, H, L, d = 1, 1, 64 * 10, 128
    assert sa.executed_flops(7, B, H, L, d) == 4 * 64 * 64 * d * 7 + 4 * 64 * d * 100 + 2 * d * 100
    assert sa.executed_flops(7, B, H, L, d, approx=False) == 4 * 64 * 64 * d * 7 + 2 * d * 100
