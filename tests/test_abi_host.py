"""Host-only checks of the C-ABI library: it builds, loads, exports every
symbol include/nvfp4_gemm.h declares, and rejects bad arguments before any
CUDA work (none of these calls reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

from nvfp4_block_scaled_gemm_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    import nvfp4_block_scaled_gemm_b200 as nv
    return nv.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "nvfp4_gemm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 9
    import nvfp4_block_scaled_gemm_b200 as nv
    assert set(names) == set(nv.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert L.nvfp4_version() == 100
    for code, name in [(0, b"NVFP4_OK"), (1, b"NVFP4_ERR_INVALID_ARG"), (5, b"NVFP4_ERR_TIMEOUT"), (99, b"NVFP4_ERR_UNKNOWN")]:
        assert L.nvfp4_status_string(code) == name


def test_swizzled_bytes(L):
    assert L.nvfp4_swizzled_scale_bytes(1, 64) == 512
    assert L.nvfp4_swizzled_scale_bytes(128, 6144) == 96 * 512
    assert L.nvfp4_swizzled_scale_bytes(129, 6144) == 2 * 96 * 512
    assert L.nvfp4_swizzled_scale_bytes(10, 48) == 0


def test_gemm_argument_validation(L):
    p = ctypes.c_void_p(0x1000)      # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x1001)
    # shapes
    assert L.nvfp4_gemm(p, p, p, p, 1.0, p, 4, 8, 96, None) == 2     # K % 64
    assert L.nvfp4_gemm(p, p, p, p, 1.0, p, 4, 12, 128, None) == 2   # N % 8
    assert L.nvfp4_gemm(p, p, p, p, 1.0, p, -1, 8, 128, None) == 1
    assert L.nvfp4_gemm(p, p, p, p, 1.0, p, 4, 8, 0, None) == 1
    # empty problems are a no-op
    assert L.nvfp4_gemm(None, None, None, None, 1.0, None, 0, 8, 128, None) == 0
    assert L.nvfp4_gemm(None, None, None, None, 1.0, None, 4, 0, 128, None) == 0
    # null / misaligned pointers
    assert L.nvfp4_gemm(None, p, p, p, 1.0, p, 4, 8, 128, None) == 1
    assert L.nvfp4_gemm(p, p, p, p, 1.0, None, 4, 8, 128, None) == 1
    assert L.nvfp4_gemm(odd, p, p, p, 1.0, p, 4, 8, 128, None) == 1
    # gemm_ex flags
    assert L.nvfp4_gemm_ex(p, p, p, p, 1.0, p, 4, 8, 96, 1, None) == 2
    assert L.nvfp4_gemm_ex(p, p, p, p, 1.0, p, 4, 8, 128, 2, None) == 1
    # grouped
    assert L.nvfp4_grouped_gemm(p, p, p, p, p, p, 0, p, 4, 8, 128, None) == 1
    assert L.nvfp4_grouped_gemm(p, p, p, p, None, p, 2, p, 4, 8, 128, None) == 1
    assert L.nvfp4_grouped_gemm(p, p, p, p, p, p, 2, p, 4, 8, 80, None) == 2
    # quantize / swizzle / diagnostics
    assert L.nvfp4_quantize(p, 2, 24, p, p, p, None) == 2
    assert L.nvfp4_quantize(p, 2, 32, p, p, None, None) == 1
    assert L.nvfp4_swizzle_scales(p, 2, 48, p, None) == 2
    assert L.nvfp4_debug_wait_timeout(10, None) == 1
