"""Python handle on the C oracle (oracle/mxfp4_oracle.c) for the MXFP4 path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check in
__graft_entry__.py and by the CPU-baseline leg of bench.py -- never by the
product package.  All arrays are host numpy arrays; nothing here touches a GPU.

Every function follows the page "MXFP4" (aiwiki.ai): "Format specification"
(E2M1/E8M0 encodings, 32-element blocks), "Conversion rules" (scale and
round-to-nearest-even with saturation, block dot products) and "Training with
MXFP4" (stochastic rounding, random Hadamard transform); the readings taken
where those sections are silent are listed at the top of the C file.
"""
import ctypes
import os

import numpy as np

from . import build as _build

LAYOUT_1D_ROW, LAYOUT_1D_COL, LAYOUT_2D = 0, 1, 2
ROUND_RNE, ROUND_SR = 0, 1
SCALE_FLOOR, SCALE_ROUNDUP, SCALE_PRESCALE_34 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        # MXFP4_ORACLE_LIB points the mutation tests at an oracle built with a
        # planted mistake; otherwise the regular build is used.
        path = os.environ.get("MXFP4_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i64 = ctypes.c_int64
        L.orc_philox4x32_10.argtypes = [ctypes.POINTER(ctypes.c_uint32)] * 3
        L.orc_sr_word.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.orc_sr_word.restype = ctypes.c_uint32
        L.orc_sr_words.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                   ctypes.POINTER(ctypes.c_uint32)]
        L.orc_rht_sign_mask.argtypes = [ctypes.c_uint64]
        L.orc_rht_sign_mask.restype = ctypes.c_uint32
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint32]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e8m0_decode.argtypes = [ctypes.c_uint32]
        L.orc_e8m0_decode.restype = ctypes.c_double
        L.orc_scale_code.argtypes = [ctypes.c_float]
        L.orc_scale_code.restype = ctypes.c_uint32
        L.orc_e2m1_rne.argtypes = [ctypes.c_float]
        L.orc_e2m1_rne.restype = ctypes.c_uint32
        L.orc_e2m1_sr.argtypes = [ctypes.c_float, ctypes.c_uint32]
        L.orc_e2m1_sr.restype = ctypes.c_uint32
        fp = ctypes.POINTER(ctypes.c_float)
        L.orc_fwht_f32.argtypes = [fp, ctypes.c_int]
        L.orc_rht_forward.argtypes = [fp, ctypes.c_int, ctypes.c_uint32]
        L.orc_rht_inverse.argtypes = [fp, ctypes.c_int, ctypes.c_uint32]
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint32]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_rne.argtypes = [ctypes.c_double]
        L.orc_e4m3_rne.restype = ctypes.c_uint32
        L.orc_nvfp4_tensor_scale.argtypes = [ctypes.c_float]
        L.orc_nvfp4_tensor_scale.restype = ctypes.c_float
        L.orc_nvfp4_quantize.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                         ctypes.c_uint64, u8p, i64, u8p, i64, ctypes.POINTER(ctypes.c_float)]
        L.orc_nvfp4_quantize.restype = ctypes.c_int
        L.orc_nvfp4_dequantize.argtypes = [u8p, i64, u8p, i64, i64, i64, ctypes.c_int, ctypes.c_float,
                                           ctypes.POINTER(ctypes.c_float), i64]
        L.orc_nvfp4_dequantize.restype = ctypes.c_int
        L.orc_nvfp4_gemm_entry.argtypes = [u8p, i64, u8p, i64, ctypes.c_float, u8p, i64, u8p, i64, ctypes.c_float,
                                           i64, i64, i64, ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_double)]
        L.orc_scale_code_rule.argtypes = [ctypes.c_float, ctypes.c_int]
        L.orc_scale_code_rule.restype = ctypes.c_uint32
        L.orc_quantize.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_uint64, ctypes.c_uint64, u8p, i64, u8p, i64, ctypes.c_void_p, i64]
        L.orc_quantize.restype = ctypes.c_int
        L.orc_quantize_view.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64, i64, u8p, i64, u8p, i64,
                                        ctypes.c_void_p, i64]
        L.orc_quantize_view.restype = ctypes.c_int
        L.orc_dequantize.argtypes = [u8p, i64, u8p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                     fp, ctypes.c_void_p, i64]
        L.orc_dequantize.restype = ctypes.c_int
        dp = ctypes.POINTER(ctypes.c_double)
        L.orc_gemm.argtypes = [u8p, i64, u8p, i64, ctypes.c_int, u8p, i64, u8p, i64, ctypes.c_int,
                               i64, i64, i64, dp, i64, ctypes.c_void_p, i64]
        L.orc_gemm_entry.argtypes = [u8p, i64, u8p, i64, ctypes.c_int, u8p, i64, u8p, i64, ctypes.c_int,
                                     i64, i64, i64, dp, dp]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


# ---- scalar primitives -------------------------------------------------------

def philox4x32_10(ctr, key):
    """Philox4x32-10 (Salmon et al., SC'11) on one 128-bit counter."""
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (ctypes.c_uint32 * 4)()
    lib().orc_philox4x32_10(c, k, o)
    return [int(v) for v in o]


def sr_word(seed: int, g: int) -> int:
    return int(lib().orc_sr_word(seed, g))


def sr_words(seed: int, g0: int, n: int) -> np.ndarray:
    out = np.zeros(n, np.uint32)
    lib().orc_sr_words(seed, g0, n, _ptr(out, ctypes.c_uint32))
    return out


def rht_sign_mask(seed: int) -> int:
    return int(lib().orc_rht_sign_mask(seed))


def e2m1_decode(code: int) -> float:
    return float(lib().orc_e2m1_decode(code))


def e8m0_decode(code: int) -> float:
    return float(lib().orc_e8m0_decode(code))


def scale_code(amax: float) -> int:
    return int(lib().orc_scale_code(ctypes.c_float(amax)))


def e2m1_rne(v: float) -> int:
    return int(lib().orc_e2m1_rne(ctypes.c_float(v)))


def e2m1_sr(v: float, r: int) -> int:
    return int(lib().orc_e2m1_sr(ctypes.c_float(v), r & 0xFFFFFFFF))


def fwht_f32(v: np.ndarray) -> np.ndarray:
    out = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().orc_fwht_f32(_ptr(out, ctypes.c_float), out.size)
    return out


def rht_forward(v: np.ndarray, sign_mask: int) -> np.ndarray:
    out = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().orc_rht_forward(_ptr(out, ctypes.c_float), out.size, sign_mask)
    return out


def rht_inverse(v: np.ndarray, sign_mask: int) -> np.ndarray:
    out = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().orc_rht_inverse(_ptr(out, ctypes.c_float), out.size, sign_mask)
    return out


# ---- tensor level ------------------------------------------------------------

def scale_code_rule(amax: float, rule: int) -> int:
    """E8M0 code of a block with the given amax under scale rule `rule`."""
    return int(lib().orc_scale_code_rule(amax, rule))


def quantize(x_bf16: np.ndarray, layout: int, rht: int = 0, rnd: int = ROUND_RNE, seed: int = 0,
             elem_offset: int = 0, transposed_copy: bool = False, scale_rule: int = SCALE_FLOOR,
             sr_ld: int = 0):
    """Quantize a bf16 tensor given as uint16 bit patterns [rows, cols].

    Returns (codes, scales) or (codes, scales, codes_t) in the canonical
    layouts described in the C file (row-major scales).  sr_ld (with
    elem_offset) places the tensor as a slice of a larger one for the SR
    stream: the row length of the whole tensor's quantized output view
    (0 = this tensor's own).
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    if layout == LAYOUT_1D_COL:
        codes = np.zeros((cols, rows // 2), np.uint8)
        scales = np.zeros((cols, rows // 32), np.uint8)
    elif layout == LAYOUT_2D:
        codes = np.zeros((rows, cols // 2), np.uint8)
        scales = np.zeros((rows // 32, cols // 32), np.uint8)
    else:
        codes = np.zeros((rows, cols // 2), np.uint8)
        scales = np.zeros((rows, cols // 32), np.uint8)
    codes_t = np.zeros((cols, rows // 2), np.uint8) if (layout == LAYOUT_2D and transposed_copy) else None
    rc = lib().orc_quantize_view(x.ctypes.data, rows, cols, cols, layout, rht, rnd, scale_rule, seed, elem_offset,
                                 sr_ld, _ptr(codes, ctypes.c_uint8), codes.shape[1], _ptr(scales, ctypes.c_uint8),
                                 scales.shape[1], codes_t.ctypes.data if codes_t is not None else None,
                                 codes_t.shape[1] if codes_t is not None else 0)
    if rc != 0:
        raise ValueError("oracle: shape not defined for this layout")
    return (codes, scales, codes_t) if codes_t is not None else (codes, scales)


def dequantize(codes: np.ndarray, scales: np.ndarray, rows: int, cols: int, layout: int,
               rht: int = 0, seed: int = 0):
    """Decode to (fp32 [rows, cols], bf16 bit patterns [rows, cols])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), np.float32)
    outb = np.zeros((rows, cols), np.uint16)
    rc = lib().orc_dequantize(_ptr(codes, ctypes.c_uint8), codes.shape[1], _ptr(scales, ctypes.c_uint8),
                              scales.shape[1], rows, cols, layout, rht, seed, _ptr(out, ctypes.c_float),
                              outb.ctypes.data, cols)
    if rc != 0:
        raise ValueError("oracle: shape not defined for this layout")
    return out, outb


def gemm(a_codes, a_scales, b_codes, b_scales, K: int, a_mode: int = 0, b_mode: int = 0, want_abs=True):
    """C = A * B^T in fp64 (both operands K-major), plus sum |a b| if asked."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    M, N = a_codes.shape[0], b_codes.shape[0]
    c = np.zeros((M, N), np.float64)
    s = np.zeros((M, N), np.float64) if want_abs else None
    lib().orc_gemm(_ptr(a_codes, ctypes.c_uint8), a_codes.shape[1], _ptr(a_scales, ctypes.c_uint8),
                   a_scales.shape[1], a_mode, _ptr(b_codes, ctypes.c_uint8), b_codes.shape[1],
                   _ptr(b_scales, ctypes.c_uint8), b_scales.shape[1], b_mode, M, N, K,
                   _ptr(c, ctypes.c_double), N, s.ctypes.data if s is not None else None, N)
    return (c, s) if want_abs else c


def gemm_entries(a_codes, a_scales, b_codes, b_scales, K: int, pairs, a_mode: int = 0, b_mode: int = 0):
    """C[m, n] and sum|a b| for the listed (m, n) pairs only."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    out_c = np.zeros(len(pairs), np.float64)
    out_s = np.zeros(len(pairs), np.float64)
    c = ctypes.c_double()
    s = ctypes.c_double()
    L = lib()
    pa, pas = _ptr(a_codes, ctypes.c_uint8), _ptr(a_scales, ctypes.c_uint8)
    pb, pbs = _ptr(b_codes, ctypes.c_uint8), _ptr(b_scales, ctypes.c_uint8)
    for i, (m, n) in enumerate(pairs):
        L.orc_gemm_entry(pa, a_codes.shape[1], pas, a_scales.shape[1], a_mode, pb, b_codes.shape[1], pbs,
                         b_scales.shape[1], b_mode, K, int(m), int(n), ctypes.byref(c), ctypes.byref(s))
        out_c[i], out_s[i] = c.value, s.value
    return out_c, out_s


# ---- NVFP4 (reading R16 of the C file) ------------------------------------------------

def e4m3_decode(code: int) -> float:
    return float(lib().orc_e4m3_decode(code))


def e4m3_rne(a: float) -> int:
    """Nearest non-negative E4M3 code (ties to even), saturating at 448."""
    return int(lib().orc_e4m3_rne(a))


def nvfp4_tensor_scale(amax: float) -> float:
    return float(lib().orc_nvfp4_tensor_scale(amax))


def nvfp4_quantize(x_bf16: np.ndarray, layout: int, rnd: int = ROUND_RNE, seed: int = 0, elem_offset: int = 0):
    """NVFP4 of a bf16 tensor [rows, cols] (uint16 bit patterns): returns
    (codes, scales (E4M3 bytes, row-major), tensor_amax)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    orows, k = (cols, rows) if layout == LAYOUT_1D_COL else (rows, cols)
    codes = np.zeros((orows, k // 2), np.uint8)
    scales = np.zeros((orows, k // 16), np.uint8)
    amax = ctypes.c_float()
    rc = lib().orc_nvfp4_quantize(x.ctypes.data, rows, cols, cols, layout, rnd, seed, elem_offset,
                                  _ptr(codes, ctypes.c_uint8), codes.shape[1], _ptr(scales, ctypes.c_uint8),
                                  scales.shape[1], ctypes.byref(amax))
    if rc != 0:
        raise ValueError("oracle: shape not defined for NVFP4")
    return codes, scales, float(amax.value)


def nvfp4_dequantize(codes, scales, rows: int, cols: int, layout: int, tensor_amax: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    out = np.zeros((rows, cols), np.float32)
    rc = lib().orc_nvfp4_dequantize(_ptr(codes, ctypes.c_uint8), codes.shape[1], _ptr(scales, ctypes.c_uint8),
                                    scales.shape[1], rows, cols, layout, tensor_amax,
                                    _ptr(out, ctypes.c_float), cols)
    if rc != 0:
        raise ValueError("oracle: shape not defined for NVFP4")
    return out


def nvfp4_gemm_entries(a_codes, a_scales, a_amax: float, b_codes, b_scales, b_amax: float, K: int, pairs):
    """NVFP4 C[m, n] = A[m, :] B[n, :]^T and sum |terms| for the listed pairs."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    out_c = np.zeros(len(pairs), np.float64)
    out_s = np.zeros(len(pairs), np.float64)
    c, s = ctypes.c_double(), ctypes.c_double()
    L = lib()
    for i, (m, n) in enumerate(pairs):
        L.orc_nvfp4_gemm_entry(_ptr(a_codes, ctypes.c_uint8), a_codes.shape[1], _ptr(a_scales, ctypes.c_uint8),
                               a_scales.shape[1], a_amax, _ptr(b_codes, ctypes.c_uint8), b_codes.shape[1],
                               _ptr(b_scales, ctypes.c_uint8), b_scales.shape[1], b_amax, K, int(m), int(n),
                               ctypes.byref(c), ctypes.byref(s))
        out_c[i], out_s[i] = c.value, s.value
    return out_c, out_s


def f32_to_bf16(values) -> np.ndarray:
    """The oracle's fp32 -> bf16 rounding (nearest even) of each value, as bit
    patterns; used for bf16 outputs of dequantize."""
    L = lib()
    v = np.ascontiguousarray(values, np.float32).ravel()
    return np.fromiter((L.orc_f32_to_bf16(float(x)) for x in v), dtype=np.uint16, count=v.size)
