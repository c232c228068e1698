"""Helpers shared by the GPU parity tests (index permutations and transfers only)."""
import numpy as np
import torch


def mma_offsets(rows: int, nkb: int, k: int) -> np.ndarray:
    """Byte offsets of (row, kb) in the GEMM-ready scale layout (include/mxfp4.h)."""
    katoms = (k // 32 + 3) // 4
    r = np.arange(rows, dtype=np.int64)[:, None]
    kb = np.arange(nkb, dtype=np.int64)[None, :]
    return ((r // 128) * katoms + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4


def mma_bytes(rows: int, k: int) -> int:
    return ((rows + 127) // 128) * ((k // 32 + 3) // 4) * 512


def to_mma(scales_rowmajor: np.ndarray, k: int) -> np.ndarray:
    rows, nkb = scales_rowmajor.shape
    out = np.zeros(mma_bytes(rows, k), np.uint8)
    out[mma_offsets(rows, nkb, k)] = scales_rowmajor
    return out


def from_mma(flat: np.ndarray, rows: int, k: int) -> np.ndarray:
    return flat[mma_offsets(rows, k // 32, k)]


def expand_2d(scales_2d: np.ndarray, rows: int) -> np.ndarray:
    """2D tile scales [rows/32, k/32] -> one scale per row [rows, k/32]."""
    return np.repeat(scales_2d, 32, axis=0)[:rows]


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 CUDA tensor (bit-exact)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_gemm_close(c_gpu: np.ndarray, c_ref: np.ndarray, s_ref: np.ndarray, rel: float = 1e-5):
    """|C_gpu - C_fp64| <= rel * sum_k |a_k b_k| element-wise; NaN where the reference is NaN."""
    nan_ref = np.isnan(c_ref)
    assert np.array_equal(np.isnan(c_gpu), nan_ref), "NaN pattern differs"
    ok = ~nan_ref
    err = np.abs(c_gpu[ok].astype(np.float64) - c_ref[ok])
    bound = rel * s_ref[ok]
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} entries outside {rel}*S; worst ratio "
                           f"{float(np.max(err / np.maximum(bound, 1e-300)))}")
    return float(np.max(err / np.maximum(s_ref[ok], 1e-300))) if ok.any() else 0.0
