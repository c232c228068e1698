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
    assert mx.lib().mxfp4_version() == 105
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


def test_dual_quantize_rejects_misaligned_mma_scales_without_gpu():
    """GEMM-ready scales are written in 4- and 16-byte pieces: an offset scale
    pointer is an alignment error before launch, not a misaligned store."""
    L = mx.lib()
    fake = ctypes.c_void_p(0x10000)
    off = ctypes.c_void_p(0x10004)
    args = lambda rs, cs: (fake, 64, 64, 64, 0, 0, 0, 0, 0, fake, 32, rs, 2, fake, 32, cs, 2, mx.SCALES_MMA, None)
    assert L.mxfp4_quantize_dual(*args(off, fake)) == mx.MXFP4_ERR_ALIGNMENT
    assert L.mxfp4_quantize_dual(*args(fake, off)) == mx.MXFP4_ERR_ALIGNMENT
    # row-major scales are single bytes: any address is fine (the check passes
    # and the call would launch, so only the failing forms are called here)


def test_scales_to_mma_rejects_invalid_arguments_without_gpu():
    L = mx.lib()
    fake = ctypes.c_void_p(0x10000)
    assert L.mxfp4_scales_to_mma(None, 4, 128, 128, 0, fake, None) == mx.MXFP4_ERR_INVALID_ARG
    assert L.mxfp4_scales_to_mma(fake, 4, 128, 96 + 8, 0, fake, None) == mx.MXFP4_ERR_INVALID_ARG   # k % 32
    assert L.mxfp4_scales_to_mma(fake, 4, 48, 128, 1, fake, None) == mx.MXFP4_ERR_INVALID_ARG       # 2D rows % 32
    assert L.mxfp4_scales_to_mma(fake, 3, 128, 128, 0, fake, None) == mx.MXFP4_ERR_INVALID_ARG      # ld < k/32
    assert L.mxfp4_scales_to_mma(fake, 4, 128, 128, 2, fake, None) == mx.MXFP4_ERR_INVALID_ARG      # two_d flag
    assert L.mxfp4_scales_to_mma(fake, 4, 128, 128, 0, ctypes.c_void_p(0x10002), None) == mx.MXFP4_ERR_ALIGNMENT


def test_gemm_wrappers_reject_rowmajor_scales_before_the_abi():
    """The binding checks scale sizes the C library cannot see: row-major scales
    (or too-short codes) raise ValueError before any pointer is taken."""
    import torch
    M, N, K = 256, 192, 512
    a = torch.zeros((M, K // 2), dtype=torch.uint8)
    b = torch.zeros((N, K // 2), dtype=torch.uint8)
    a_rm = torch.zeros((M, K // 32), dtype=torch.uint8)
    b_rm = torch.zeros((N, K // 32), dtype=torch.uint8)
    b_2d = torch.zeros((N // 32, K // 32), dtype=torch.uint8)
    a_mma = torch.zeros(mx.mma_scales_bytes(M, K), dtype=torch.uint8)
    b_mma = torch.zeros(mx.mma_scales_bytes(N, K), dtype=torch.uint8)
    for fn in (mx.mxfp4_gemm, mx.mxfp4_gemm_bf16, mx.mxfp4_gemm_mxfp4):
        with pytest.raises(ValueError, match="SCALES_MMA"):
            fn(a, a_rm, b, b_mma, K)
        with pytest.raises(ValueError, match="SCALES_MMA"):
            fn(a, a_mma, b, b_2d, K)
        with pytest.raises(ValueError, match="elements per row"):
            fn(a[:, :100], a_mma, b, b_mma, K)
    G = 4
    offs = torch.zeros(G + 1, dtype=torch.int32)
    sizes = torch.zeros(G, dtype=torch.int32)
    bg = torch.zeros((G, N, K // 2), dtype=torch.uint8)
    for fn in (mx.mxfp4_grouped_gemm, mx.mxfp4_grouped_gemm_bf16):
        with pytest.raises(ValueError, match="SCALES_MMA"):       # one expert's scales for G experts
            fn(a, a_mma, offs, sizes, bg, b_mma, N, K)
        with pytest.raises(ValueError, match="SCALES_MMA"):
            fn(a, a_rm, offs, sizes, bg, torch.zeros(G * mx.mma_scales_bytes(N, K), dtype=torch.uint8), N, K)
    for fn in (mx.mxfp4_grouped_gemm_wgrad, mx.mxfp4_grouped_gemm_wgrad_bf16):
        with pytest.raises(ValueError, match="SCALES_MMA"):
            fn(a, a_mma, b, b_rm, offs, K)


def test_quantize_dual_rows_rejects_bad_slices_without_gpu():
    L = mx.lib()
    fake = ctypes.c_void_p(0x10000)
    call = lambda row0, total, rows=64: L.mxfp4_quantize_dual_rows(fake, rows, 64, 64, row0, total, 32, 1, 42, fake,
                                                                   32, fake, 2, fake, 32, fake, 2, 0, None)
    assert call(16, 256) == mx.MXFP4_ERR_INVALID_ARG        # slice start off a 32-token boundary
    assert call(0, 240) == mx.MXFP4_ERR_INVALID_ARG         # whole tensor not a multiple of 32 rows
    assert call(224, 256) == mx.MXFP4_ERR_INVALID_ARG       # slice past the end
    assert call(-32, 256) == mx.MXFP4_ERR_INVALID_ARG
