"""quantize_block_scaled_rht_b200 -- MXFP4 quantization and block-scaled GEMMs on B200.

A thin Python binding over the C ABI of libmxfp4.so (include/mxfp4.h): every
function here only marshals arguments (torch tensors -> device pointers, the
current CUDA stream) and calls the library; all arithmetic runs in the CUDA
kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: without the built library or a CUDA device these calls raise.

The method is the one on "MXFP4" (aiwiki.ai) -- "Format specification",
"Conversion rules", "Training with MXFP4" -- as used by the ALTO recipe
("Training an MoE LLM in MXFP4", abstract): 1D blocks for activations and
gradients, 2D 32x32 blocks for weights, randomized Hadamard transform and
stochastic rounding.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxfp4.so")

# enums (include/mxfp4.h)
MXFP4_OK = 0
MXFP4_ERR_INVALID_ARG = 1
MXFP4_ERR_ALIGNMENT = 2
MXFP4_ERR_UNSUPPORTED = 3
MXFP4_ERR_CUDA = 4
MXFP4_ERR_TIMEOUT = 5
LAYOUT_1D_ROW, LAYOUT_1D_COL, LAYOUT_2D = 0, 1, 2
ROUND_RNE, ROUND_SR = 0, 1
# scale rules, OR-ed into the rounding argument (MXFP4_SCALE_* in include/mxfp4.h)
SCALE_FLOOR, SCALE_ROUNDUP, SCALE_PRESCALE_34 = 0x00, 0x10, 0x20
SCALES_ROWMAJOR, SCALES_MMA = 0, 1
OUT_BF16, OUT_F32 = 0, 1

ABI_FUNCTIONS = (
    "mxfp4_status_string", "mxfp4_version", "mxfp4_mma_scales_bytes", "mxfp4_mma_scale_offset",
    "mxfp4_quantize", "mxfp4_quantize_dual", "mxfp4_dequantize", "mxfp4_gemm", "mxfp4_grouped_gemm",
    "mxfp4_gemm_bf16", "mxfp4_grouped_gemm_bf16", "mxfp4_gemm_mxfp4", "mxfp4_grouped_gemm_wgrad",
    "mxfp4_grouped_gemm_wgrad_bf16", "mxfp4_nvfp4_quantize", "mxfp4_nvfp4_dequantize", "mxfp4_nvfp4_gemm",
    "mxfp4_get_error",
    "mxfp4_set_wait_limit_ns", "mxfp4_wait_probe", "mxfp4_scales_to_mma",
    "mxfp4_quantize_dual_rows",
)


class MXFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmxfp4.so from the package directory (built by build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmxfp4.so not built: run `python -m quantize_block_scaled_rht_b200.build` ({LIB_PATH})")
        L = ctypes.CDLL(LIB_PATH)
        i64, u64, i32, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p
        L.mxfp4_status_string.argtypes = [i32]
        L.mxfp4_status_string.restype = ctypes.c_char_p
        L.mxfp4_version.restype = i32
        L.mxfp4_mma_scales_bytes.argtypes = [i64, i64]
        L.mxfp4_mma_scales_bytes.restype = i64
        L.mxfp4_mma_scale_offset.argtypes = [i64, i64, i64]
        L.mxfp4_mma_scale_offset.restype = i64
        L.mxfp4_quantize.argtypes = [vp, i64, i64, i64, i32, i32, i32, u64, u64, vp, i64, vp, i64, i32,
                                     vp, i64, vp, i64, vp]
        L.mxfp4_quantize.restype = i32
        L.mxfp4_quantize_dual.argtypes = [vp, i64, i64, i64, i32, i32, u64, u64, u64, vp, i64, vp, i64, vp, i64,
                                          vp, i64, i32, vp]
        L.mxfp4_quantize_dual.restype = i32
        L.mxfp4_quantize_dual_rows.argtypes = [vp, i64, i64, i64, i64, i64, i32, i32, u64, vp, i64, vp, i64, vp,
                                               i64, vp, i64, i32, vp]
        L.mxfp4_quantize_dual_rows.restype = i32
        L.mxfp4_dequantize.argtypes = [vp, i64, vp, i64, i32, i64, i64, i32, i32, u64, vp, i64, i32, vp]
        L.mxfp4_dequantize.restype = i32
        L.mxfp4_gemm.argtypes = [vp, i64, vp, vp, i64, vp, i64, i64, i64, vp, i64, vp]
        L.mxfp4_gemm.restype = i32
        L.mxfp4_grouped_gemm.argtypes = [vp, i64, vp, i64, vp, vp, i32, vp, i64, vp, i64, i64, vp, i64, vp]
        L.mxfp4_grouped_gemm.restype = i32
        L.mxfp4_gemm_bf16.argtypes = [vp, i64, vp, vp, i64, vp, i64, i64, i64, vp, i64, vp]
        L.mxfp4_gemm_bf16.restype = i32
        L.mxfp4_grouped_gemm_bf16.argtypes = [vp, i64, vp, i64, vp, vp, i32, vp, i64, vp, i64, i64, vp, i64, vp]
        L.mxfp4_grouped_gemm_bf16.restype = i32
        L.mxfp4_gemm_mxfp4.argtypes = [vp, i64, vp, vp, i64, vp, i64, i64, i64, vp, i64, vp, i64, i32, vp]
        L.mxfp4_gemm_mxfp4.restype = i32
        L.mxfp4_grouped_gemm_wgrad.argtypes = [vp, i64, vp, vp, i64, vp, vp, i32, i64, i64, i64, vp, i64, vp]
        L.mxfp4_grouped_gemm_wgrad.restype = i32
        L.mxfp4_grouped_gemm_wgrad_bf16.argtypes = [vp, i64, vp, vp, i64, vp, vp, i32, i64, i64, i64, vp, i64, vp]
        L.mxfp4_grouped_gemm_wgrad_bf16.restype = i32
        L.mxfp4_nvfp4_quantize.argtypes = [vp, i64, i64, i64, i32, i32, u64, u64, vp, vp, i64, vp, i64, i32, vp]
        L.mxfp4_nvfp4_quantize.restype = i32
        L.mxfp4_nvfp4_dequantize.argtypes = [vp, i64, vp, i64, i32, vp, i64, i64, i32, vp, i64, vp]
        L.mxfp4_nvfp4_dequantize.restype = i32
        L.mxfp4_nvfp4_gemm.argtypes = [vp, i64, vp, vp, vp, i64, vp, vp, i64, i64, i64, vp, i64, vp]
        L.mxfp4_nvfp4_gemm.restype = i32
        L.mxfp4_scales_to_mma.argtypes = [vp, i64, i64, i64, i32, vp, vp]
        L.mxfp4_scales_to_mma.restype = i32
        L.mxfp4_get_error.argtypes = [vp]
        L.mxfp4_get_error.restype = i32
        L.mxfp4_set_wait_limit_ns.argtypes = [u64]
        L.mxfp4_set_wait_limit_ns.restype = u64
        L.mxfp4_wait_probe.argtypes = [i32, vp]
        L.mxfp4_wait_probe.restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mxfp4_status_string(int(status)).decode()


def _check(rc: int, what: str) -> None:
    if rc != MXFP4_OK:
        raise MXFP4Error(rc, what)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmxfp4 takes CUDA tensors (device pointers)")
    return t.data_ptr()


def mma_scales_bytes(rows: int, k: int) -> int:
    """Bytes of the GEMM-ready scale layout of a (rows x k) operand."""
    return int(lib().mxfp4_mma_scales_bytes(rows, k))


def mma_scale_offset(row: int, kb: int, k: int) -> int:
    return int(lib().mxfp4_mma_scale_offset(row, kb, k))


def _check_operand(codes: torch.Tensor, scales: torch.Tensor, rows: int, K: int, what: str, groups: int = 1,
                   scale_bytes=None) -> None:
    """Host-side check of one GEMM operand before its pointers cross the ABI:
    the C library cannot see buffer sizes, so a row-major scale tensor passed
    where the GEMM-ready layout is read (32x smaller for 2D weights) is caught
    here instead of becoming reads past the allocation."""
    if codes.dtype != torch.uint8 or scales.dtype != torch.uint8:
        raise ValueError(f"{what}: codes and scales must be uint8 tensors")
    if codes.shape[-1] * 2 < K:
        raise ValueError(f"{what}: codes hold {codes.shape[-1] * 2} elements per row, K = {K}")
    need = groups * (scale_bytes or mma_scales_bytes)(rows, K)
    if scales.dim() != 1 or scales.numel() < need:
        raise ValueError(f"{what}: scales must be the GEMM-ready (SCALES_MMA) layout, a 1-D tensor of at least "
                         f"{need} bytes; got shape {tuple(scales.shape)} (quantize with scale_layout=SCALES_MMA "
                         f"or convert with mxfp4_scales_to_mma)")
    if codes.device != scales.device:
        raise ValueError(f"{what}: codes and scales on different devices")


def _check_same_device(*ts: torch.Tensor) -> None:
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError(f"GEMM operands on different devices: {sorted(map(str, devs))}")


@dataclass
class Quantized:
    """Output of mxfp4_quantize: codes/scales (and the 2D transposed copy)."""
    codes: torch.Tensor
    scales: torch.Tensor
    rows: int            # rows of the quantized operand (output view)
    k: int               # elements per row of the quantized operand
    layout: int
    scale_layout: int
    codes_t: Optional[torch.Tensor] = None
    scales_t: Optional[torch.Tensor] = None


def _scale_tensor(rows, k, scale_layout, device, two_d=False):
    if scale_layout == SCALES_MMA:
        return torch.empty(mma_scales_bytes(rows, k), dtype=torch.uint8, device=device)
    if two_d:
        return torch.empty((rows // 32, k // 32), dtype=torch.uint8, device=device)
    return torch.empty((rows, k // 32), dtype=torch.uint8, device=device)


def mxfp4_quantize(x: torch.Tensor, layout: int = LAYOUT_1D_ROW, rht_size: int = 0, rounding: int = ROUND_RNE,
                   seed: int = 0, elem_offset: int = 0, scale_layout: int = SCALES_ROWMAJOR,
                   transposed_copy: bool = False, stream=None, out: Optional[Quantized] = None,
                   scale_rule: int = SCALE_FLOOR) -> Quantized:
    """Quantize a 2-D bf16 CUDA tensor to MXFP4 (see mxfp4_quantize in include/mxfp4.h)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    if out is None:
        dev = x.device
        if layout == LAYOUT_1D_COL:
            orows, k = cols, rows
        else:
            orows, k = rows, cols
        codes = torch.empty((orows, k // 2), dtype=torch.uint8, device=dev)
        scales = _scale_tensor(orows, k, scale_layout, dev, two_d=(layout == LAYOUT_2D))
        codes_t = scales_t = None
        if transposed_copy:
            codes_t = torch.empty((cols, rows // 2), dtype=torch.uint8, device=dev)
            scales_t = _scale_tensor(cols, rows, scale_layout, dev, two_d=True)
        out = Quantized(codes, scales, orows, k, layout, scale_layout, codes_t, scales_t)
    ld_sc = out.scales.shape[1] if out.scales.dim() == 2 else 0
    ld_sct = out.scales_t.shape[1] if (out.scales_t is not None and out.scales_t.dim() == 2) else 0
    rc = lib().mxfp4_quantize(
        _ptr(x), rows, cols, x.stride(0), layout, rht_size, rounding | scale_rule, seed & 0xFFFFFFFFFFFFFFFF, elem_offset,
        _ptr(out.codes), out.codes.stride(0), _ptr(out.scales), ld_sc, scale_layout,
        _ptr(out.codes_t), out.codes_t.stride(0) if out.codes_t is not None else 0,
        _ptr(out.scales_t), ld_sct, _stream(stream))
    _check(rc, "mxfp4_quantize")
    return out


def mxfp4_quantize_dual(x: torch.Tensor, col_rht_size: int = 0, rounding: int = ROUND_RNE, seed: int = 0,
                        row_elem_offset: int = 0, col_elem_offset: int = 0, scale_layout: int = SCALES_ROWMAJOR,
                        row: bool = True, col: bool = True, stream=None, out_row: Optional[Quantized] = None,
                        out_col: Optional[Quantized] = None, scale_rule: int = SCALE_FLOOR):
    """Row blocks and column blocks (RHT along rows) of one bf16 tensor from a
    single read (see mxfp4_quantize_dual in include/mxfp4.h).  Returns
    (row Quantized or None, column Quantized or None)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    dev = x.device
    if row and out_row is None:
        out_row = Quantized(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                            _scale_tensor(rows, cols, scale_layout, dev), rows, cols, LAYOUT_1D_ROW, scale_layout)
    if col and out_col is None:
        out_col = Quantized(torch.empty((cols, rows // 2), dtype=torch.uint8, device=dev),
                            _scale_tensor(cols, rows, scale_layout, dev), cols, rows, LAYOUT_1D_COL, scale_layout)
    r = out_row if row else None
    c = out_col if col else None
    ld = lambda q: (q.scales.shape[1] if q.scales.dim() == 2 else 0) if q is not None else 0
    rc = lib().mxfp4_quantize_dual(
        _ptr(x), rows, cols, x.stride(0), col_rht_size, rounding | scale_rule, seed & 0xFFFFFFFFFFFFFFFF, row_elem_offset,
        col_elem_offset, _ptr(r.codes) if r else None, r.codes.stride(0) if r else 0, _ptr(r.scales) if r else None,
        ld(r), _ptr(c.codes) if c else None, c.codes.stride(0) if c else 0, _ptr(c.scales) if c else None, ld(c),
        scale_layout, _stream(stream))
    _check(rc, "mxfp4_quantize_dual")
    return r, c


def mxfp4_quantize_dual_rows(x: torch.Tensor, row0: int, total_rows: int, col_rht_size: int = 0,
                             rounding: int = ROUND_RNE, seed: int = 0, scale_layout: int = SCALES_ROWMAJOR,
                             row: bool = True, col: bool = True, stream=None, out_row: Optional[Quantized] = None,
                             out_col: Optional[Quantized] = None, scale_rule: int = SCALE_FLOOR):
    """mxfp4_quantize_dual of rows [row0, row0 + x.shape[0]) of a tensor with
    total_rows rows: the slice's part of the whole tensor's quantization, SR
    included (see mxfp4_quantize_dual_rows in include/mxfp4.h).  The column
    output is [cols, rows/2], the slice's columns of the whole [cols,
    total_rows] view."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    dev = x.device
    if row and out_row is None:
        out_row = Quantized(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                            _scale_tensor(rows, cols, scale_layout, dev), rows, cols, LAYOUT_1D_ROW, scale_layout)
    if col and out_col is None:
        out_col = Quantized(torch.empty((cols, rows // 2), dtype=torch.uint8, device=dev),
                            _scale_tensor(cols, rows, scale_layout, dev), cols, rows, LAYOUT_1D_COL, scale_layout)
    r = out_row if row else None
    c = out_col if col else None
    ld = lambda q: (q.scales.shape[1] if q.scales.dim() == 2 else 0) if q is not None else 0
    rc = lib().mxfp4_quantize_dual_rows(
        _ptr(x), rows, cols, x.stride(0), row0, total_rows, col_rht_size, rounding | scale_rule,
        seed & 0xFFFFFFFFFFFFFFFF, _ptr(r.codes) if r else None, r.codes.stride(0) if r else 0,
        _ptr(r.scales) if r else None, ld(r), _ptr(c.codes) if c else None, c.codes.stride(0) if c else 0,
        _ptr(c.scales) if c else None, ld(c), scale_layout, _stream(stream))
    _check(rc, "mxfp4_quantize_dual_rows")
    return r, c


def mxfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, rows: int, cols: int, layout: int = LAYOUT_1D_ROW,
                     rht_size: int = 0, seed: int = 0, scale_layout: int = SCALES_ROWMAJOR,
                     out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Decode MXFP4 codes/scales of a [rows, cols] tensor (inverse RHT if rht_size)."""
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype, device=codes.device)
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    ld_sc = scales.shape[1] if scales.dim() == 2 else 0
    rc = lib().mxfp4_dequantize(_ptr(codes), codes.stride(0), _ptr(scales), ld_sc, scale_layout, rows, cols,
                                layout, rht_size, seed & 0xFFFFFFFFFFFFFFFF, _ptr(out), out.stride(0), od,
                                _stream(stream))
    _check(rc, "mxfp4_dequantize")
    return out


def mxfp4_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor,
               K: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """C[M, N] = A[M, K] B[N, K]^T in FP32; scales in the GEMM-ready (MMA) layout."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    _check_operand(a_codes, a_scales, M, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B")
    _check_same_device(a_codes, b_codes, out)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=a_codes.device)
    rc = lib().mxfp4_gemm(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), _ptr(b_codes), b_codes.stride(0),
                          _ptr(b_scales), M, N, K, _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_gemm")
    return out


def mxfp4_grouped_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, group_offsets: torch.Tensor,
                       group_sizes: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor, N: int, K: int,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per group g: C[rows of g] = A[rows of g] B_g^T.  b_codes is [G, N, K/2]."""
    a_rows = a_codes.shape[0]
    G = group_sizes.numel()
    _check_operand(a_codes, a_scales, a_rows, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B", groups=G)
    _check_same_device(a_codes, b_codes, group_offsets, group_sizes, out)
    if out is None:
        out = torch.empty((a_rows, N), dtype=torch.float32, device=a_codes.device)
    rc = lib().mxfp4_grouped_gemm(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), a_rows, _ptr(group_offsets),
                                  _ptr(group_sizes), G, _ptr(b_codes), b_codes.stride(-2), _ptr(b_scales), N, K,
                                  _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_grouped_gemm")
    return out


def mxfp4_gemm_bf16(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor,
                    K: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxfp4_gemm with the FP32 accumulators rounded to a bf16 output."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    _check_operand(a_codes, a_scales, M, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B")
    _check_same_device(a_codes, b_codes, out)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    if out.dtype != torch.bfloat16:
        raise ValueError("out must be bfloat16")
    rc = lib().mxfp4_gemm_bf16(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), _ptr(b_codes), b_codes.stride(0),
                               _ptr(b_scales), M, N, K, _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_gemm_bf16")
    return out


def mxfp4_gemm_mxfp4(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor,
                     K: int, scale_layout: int = SCALES_ROWMAJOR, out: Optional[Quantized] = None,
                     stream=None) -> Quantized:
    """mxfp4_gemm with C requantized to MXFP4 (1D row blocks, reference scale
    rule, RNE) in the epilogue; returns C as a Quantized [M, N]."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    _check_operand(a_codes, a_scales, M, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B")
    dev = a_codes.device
    if out is None:
        out = Quantized(torch.empty((M, N // 2), dtype=torch.uint8, device=dev), _scale_tensor(M, N, scale_layout, dev),
                        M, N, LAYOUT_1D_ROW, scale_layout)
    ld_sc = out.scales.shape[1] if out.scales.dim() == 2 else 0
    rc = lib().mxfp4_gemm_mxfp4(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), _ptr(b_codes), b_codes.stride(0),
                                _ptr(b_scales), M, N, K, _ptr(out.codes), out.codes.stride(0), _ptr(out.scales), ld_sc,
                                scale_layout, _stream(stream))
    _check(rc, "mxfp4_gemm_mxfp4")
    return out


def mxfp4_grouped_gemm_bf16(a_codes: torch.Tensor, a_scales: torch.Tensor, group_offsets: torch.Tensor,
                            group_sizes: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor, N: int, K: int,
                            out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxfp4_grouped_gemm with a bf16 output."""
    a_rows = a_codes.shape[0]
    G = group_sizes.numel()
    _check_operand(a_codes, a_scales, a_rows, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B", groups=G)
    _check_same_device(a_codes, b_codes, group_offsets, group_sizes, out)
    if out is None:
        out = torch.empty((a_rows, N), dtype=torch.bfloat16, device=a_codes.device)
    if out.dtype != torch.bfloat16:
        raise ValueError("out must be bfloat16")
    rc = lib().mxfp4_grouped_gemm_bf16(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), a_rows,
                                       _ptr(group_offsets), _ptr(group_sizes), G, _ptr(b_codes), b_codes.stride(-2),
                                       _ptr(b_scales), N, K, _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_grouped_gemm_bf16")
    return out


def mxfp4_grouped_gemm_wgrad(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor,
                             b_scales: torch.Tensor, group_offsets: torch.Tensor, K: int,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per group g: C_g = A[:, K range g] B[:, K range g]^T (the MoE weight
    gradient).  a_codes [M, K/2], b_codes [N, K/2]; group_offsets is a device
    int32 tensor of G + 1 offsets along K; returns [G * M, N] FP32."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    G = group_offsets.numel() - 1
    _check_operand(a_codes, a_scales, M, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B")
    _check_same_device(a_codes, b_codes, group_offsets, out)
    if out is None:
        out = torch.empty((G * M, N), dtype=torch.float32, device=a_codes.device)
    rc = lib().mxfp4_grouped_gemm_wgrad(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), _ptr(b_codes),
                                        b_codes.stride(0), _ptr(b_scales), _ptr(group_offsets), G, M, N, K,
                                        _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_grouped_gemm_wgrad")
    return out


def mxfp4_grouped_gemm_wgrad_bf16(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor,
                                  b_scales: torch.Tensor, group_offsets: torch.Tensor, K: int,
                                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxfp4_grouped_gemm_wgrad with a bf16 output; returns [G * M, N] bf16."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    G = group_offsets.numel() - 1
    _check_operand(a_codes, a_scales, M, K, "A")
    _check_operand(b_codes, b_scales, N, K, "B")
    _check_same_device(a_codes, b_codes, group_offsets, out)
    if out is None:
        out = torch.empty((G * M, N), dtype=torch.bfloat16, device=a_codes.device)
    if out.dtype != torch.bfloat16:
        raise ValueError("out must be bfloat16")
    rc = lib().mxfp4_grouped_gemm_wgrad_bf16(_ptr(a_codes), a_codes.stride(0), _ptr(a_scales), _ptr(b_codes),
                                             b_codes.stride(0), _ptr(b_scales), _ptr(group_offsets), G, M, N, K,
                                             _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_grouped_gemm_wgrad_bf16")
    return out


@dataclass
class NvQuantized:
    """NVFP4 codes, E4M3 block scales and the device tensor amax (a 1-element
    float32 tensor) of one tensor."""
    codes: torch.Tensor
    scales: torch.Tensor
    amax: torch.Tensor
    rows: int
    k: int
    layout: int
    scale_layout: int


def nv_mma_scales_bytes(rows: int, k: int) -> int:
    """Bytes of NVFP4 scales in the MMA layout: 512-byte atoms of 128 rows x 4 blocks of 16."""
    return ((rows + 127) // 128) * ((k // 16 + 3) // 4) * 512


def mxfp4_nvfp4_quantize(x: torch.Tensor, layout: int = LAYOUT_1D_ROW, rounding: int = ROUND_RNE, seed: int = 0,
                         elem_offset: int = 0, scale_layout: int = SCALES_ROWMAJOR, stream=None,
                         out: Optional[NvQuantized] = None) -> NvQuantized:
    """NVFP4 quantization (see mxfp4_nvfp4_quantize in include/mxfp4.h)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    orows, k = (cols, rows) if layout == LAYOUT_1D_COL else (rows, cols)
    if out is None:
        dev = x.device
        codes = torch.empty((orows, k // 2), dtype=torch.uint8, device=dev)
        if scale_layout == SCALES_MMA:
            scales = torch.zeros((nv_mma_scales_bytes(orows, k),), dtype=torch.uint8, device=dev)
        else:
            scales = torch.empty((orows, k // 16), dtype=torch.uint8, device=dev)
        out = NvQuantized(codes, scales, torch.empty(1, dtype=torch.float32, device=dev), orows, k, layout,
                          scale_layout)
    ld_sc = out.scales.shape[1] if out.scales.dim() == 2 else 0
    rc = lib().mxfp4_nvfp4_quantize(_ptr(x), rows, cols, x.stride(0), layout, rounding, seed & 0xFFFFFFFFFFFFFFFF,
                                    elem_offset, _ptr(out.amax), _ptr(out.codes), out.codes.stride(0),
                                    _ptr(out.scales), ld_sc, scale_layout, _stream(stream))
    _check(rc, "mxfp4_nvfp4_quantize")
    return out


def mxfp4_nvfp4_dequantize(q: NvQuantized, rows: int, cols: int, out: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=q.codes.device)
    ld_sc = q.scales.shape[1] if q.scales.dim() == 2 else 0
    rc = lib().mxfp4_nvfp4_dequantize(_ptr(q.codes), q.codes.stride(0), _ptr(q.scales), ld_sc, q.scale_layout,
                                      _ptr(q.amax), rows, cols, q.layout, _ptr(out), out.stride(0), _stream(stream))
    _check(rc, "mxfp4_nvfp4_dequantize")
    return out


def mxfp4_nvfp4_gemm(a: NvQuantized, b: NvQuantized, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """C = A B^T for NVFP4 operands quantized with SCALES_MMA."""
    M, N, K = a.rows, b.rows, a.k
    if a.scale_layout != SCALES_MMA or b.scale_layout != SCALES_MMA or b.k != K:
        raise ValueError("mxfp4_nvfp4_gemm: both operands need SCALES_MMA scales and the same K")
    _check_operand(a.codes, a.scales, M, K, "A", scale_bytes=nv_mma_scales_bytes)
    _check_operand(b.codes, b.scales, N, K, "B", scale_bytes=nv_mma_scales_bytes)
    _check_same_device(a.codes, b.codes, a.amax, b.amax, out)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=a.codes.device)
    rc = lib().mxfp4_nvfp4_gemm(_ptr(a.codes), a.codes.stride(0), _ptr(a.scales), _ptr(a.amax), _ptr(b.codes),
                                b.codes.stride(0), _ptr(b.scales), _ptr(b.amax), M, N, K, _ptr(out), out.stride(0),
                                _stream(stream))
    _check(rc, "mxfp4_nvfp4_gemm")
    return out


def mxfp4_scales_to_mma(scales: torch.Tensor, rows: int, k: int, two_d: bool = False,
                        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Canonical row-major scales ([rows, k/32], or [rows/32, k/32] tile scales
    with two_d) to the GEMM-ready layout the GEMMs read (see
    mxfp4_scales_to_mma in include/mxfp4.h)."""
    if scales.dtype != torch.uint8 or scales.dim() != 2:
        raise ValueError("scales must be a 2-D uint8 tensor (canonical row-major)")
    want = ((rows // 32) if two_d else rows, k // 32)
    if tuple(scales.shape) != want or scales.stride(1) != 1:
        raise ValueError(f"scales must be {want} row-major; got {tuple(scales.shape)}")
    if out is None:
        out = torch.empty(mma_scales_bytes(rows, k), dtype=torch.uint8, device=scales.device)
    if out.dim() != 1 or out.numel() < mma_scales_bytes(rows, k):
        raise ValueError("out must be a 1-D uint8 tensor of mma_scales_bytes(rows, k) bytes")
    rc = lib().mxfp4_scales_to_mma(_ptr(scales), scales.stride(0), rows, k, 1 if two_d else 0, _ptr(out),
                                   _stream(stream))
    _check(rc, "mxfp4_scales_to_mma")
    return out


def mxfp4_get_error(stream=None) -> int:
    """Synchronize the stream; return and clear the first device-side error."""
    return int(lib().mxfp4_get_error(_stream(stream)))


def mxfp4_set_wait_limit_ns(limit_ns: int) -> int:
    return int(lib().mxfp4_set_wait_limit_ns(limit_ns))


def mxfp4_wait_probe(arrive: bool, stream=None) -> None:
    _check(lib().mxfp4_wait_probe(1 if arrive else 0, _stream(stream)), "mxfp4_wait_probe")
