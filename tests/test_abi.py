"""The C ABI library loads without a GPU, exports every symbol include/mxfp4.h
declares, and rejects invalid arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import quantize_block_scaled_rht_b200 as mx
from conftest import ROOT


def _declared():
    with open(os.path.join(ROOT, "include", "mxfp4.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"MXFP4_API\s+[\w\s\*]*?\b(mxfp4_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    from quantize_block_scaled_rht_b200 import build
    build.build()
    names = _declared()
    assert len(names) >= 10
    L = mx.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(mx.ABI_FUNCTIONS)


def test_status_strings_and_layout_helpers():
    assert mx.status_string(mx.MXFP4_OK) == "MXFP4_OK"
    assert mx.status_string(mx.MXFP4_ERR_TIMEOUT) == "MXFP4_ERR_TIMEOUT"
    assert mx.lib().mxfp4_version() == 103
    # 128 rows x 4 K-blocks per 512-byte atom
    assert mx.mma_scales_bytes(128, 128) == 512
    assert mx.mma_scales_bytes(129, 2880) == 2 * 23 * 512
    assert mx.mma_scale_offset(0, 0, 256) == 0
    assert mx.mma_scale_offset(1, 0, 256) == 16
    assert mx.mma_scale_offset(32, 0, 256) == 4
    assert mx.mma_scale_offset(0, 5, 256) == 512 + 1
    assert mx.mma_scale_offset(128, 0, 256) == 2 * 512


def test_invalid_arguments_rejected_without_gpu():
    L = mx.lib()
    fake = ctypes.c_void_p(0x10000)    # never dereferenced: validation fails first
    # null pointers
    assert L.mxfp4_quantize(None, 32, 32, 32, 0, 0, 0, 0, 0, fake, 16, fake, 1, 0, None, 0, None, 0, None) == 1
    # block axis not a multiple of 32
    assert L.mxfp4_quantize(fake, 32, 48, 48, 0, 0, 0, 0, 0, fake, 32, fake, 2, 0, None, 0, None, 0, None) == 1
    # bad RHT size
    assert L.mxfp4_quantize(fake, 32, 64, 64, 0, 8, 0, 0, 0, fake, 32, fake, 2, 0, None, 0, None, 0, None) == 1
    # transposed copy only for 2D
    assert L.mxfp4_quantize(fake, 32, 64, 64, 0, 0, 0, 0, 0, fake, 32, fake, 2, 0, fake, 16, None, 0, None) == 1
    # misaligned leading dimension
    assert L.mxfp4_quantize(fake, 32, 64, 68, 0, 0, 0, 0, 0, fake, 32, fake, 2, 0, None, 0, None, 0, None) == 2
    # rounding: unknown rounding mode, unknown scale rule, stray bits
    for bad in (2, 0x30, 0x40, 0x101):
        assert L.mxfp4_quantize(fake, 32, 64, 64, 0, 0, bad, 0, 0, fake, 32, fake, 2, 0, None, 0, None, 0,
                                None) == 1
    # GEMM: K not a multiple of 64 -> unsupported; not of 32 -> invalid
    assert L.mxfp4_gemm(fake, 16, fake, fake, 16, fake, 128, 128, 96, fake, 128, None) == 3
    assert L.mxfp4_gemm(fake, 16, fake, fake, 16, fake, 128, 128, 80, fake, 128, None) == 1
    assert L.mxfp4_gemm(fake, 40, fake, fake, 32, fake, 128, 128, 64, fake, 128, None) == 2
    # bf16-output GEMM: ldc must give 16-byte rows (8 bf16), K rules as for FP32
    assert L.mxfp4_gemm_bf16(fake, 32, fake, fake, 32, fake, 128, 132, 64, fake, 132, None) == 2
    assert L.mxfp4_gemm_bf16(fake, 16, fake, fake, 16, fake, 128, 128, 96, fake, 128, None) == 3
    assert L.mxfp4_gemm_bf16(fake, 32, fake, fake, 32, fake, 0, 128, 64, fake, 128, None) == 1
    assert L.mxfp4_grouped_gemm_bf16(fake, 32, fake, 128, fake, fake, 5000, fake, 32, fake, 128, 64, fake, 128,
                                     None) == 3
    assert L.mxfp4_grouped_gemm_bf16(fake, 32, fake, 128, fake, fake, 2, fake, 32, fake, 132, 64, fake, 132,
                                     None) == 2
    # MXFP4-output GEMM: N a multiple of 32, 16-byte code rows, a known scale layout
    assert L.mxfp4_gemm_mxfp4(fake, 32, fake, fake, 32, fake, 128, 200, 64, fake, 112, fake, 8, 0, None) == 1
    assert L.mxfp4_gemm_mxfp4(fake, 32, fake, fake, 32, fake, 128, 192, 64, fake, 104, fake, 6, 0, None) == 2
    assert L.mxfp4_gemm_mxfp4(fake, 32, fake, fake, 32, fake, 128, 192, 64, fake, 96, fake, 6, 7, None) == 1
    assert L.mxfp4_gemm_mxfp4(fake, 16, fake, fake, 16, fake, 128, 192, 96, fake, 96, fake, 6, 0, None) == 3
    # bf16 grouped wgrad: ldc must give 16-byte rows
    assert L.mxfp4_grouped_gemm_wgrad_bf16(fake, 64, fake, fake, 64, fake, fake, 2, 128, 132, 128, fake, 132,
                                           None) == 2
    # grouped wgrad: K not a multiple of 128, too many groups
    assert L.mxfp4_grouped_gemm_wgrad(fake, 32, fake, fake, 32, fake, fake, 2, 128, 128, 64, fake, 128, None) == 1
    assert L.mxfp4_grouped_gemm_wgrad(fake, 64, fake, fake, 64, fake, fake, 5000, 128, 128, 128, fake, 128,
                                      None) == 3
    # grouped: too many groups
    assert L.mxfp4_grouped_gemm(fake, 32, fake, 128, fake, fake, 5000, fake, 32, fake, 128, 64, fake, 128,
                                None) == 3
