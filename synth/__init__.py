"""Seeded synthetic inputs for the MXFP4 path (shared by tests and bench.py).

This module holds no arithmetic of the method: it draws random numbers,
rounds them to bf16 (round-to-nearest-even on the fp32 bit pattern) and builds
the MoE routing.  Both the oracle side and the CUDA side read its outputs.

Workloads stand in for the ones named on "Training an MoE LLM in MXFP4" (the
ALTO brief: GPT-OSS-20B, MLPerf Small MoE, C4), whose data and weights are not
available here: shapes follow GPT-OSS-20B (hidden 2880, expert intermediate
5760, 32 experts, top-4), values are drawn from the stated distributions.
"""
from __future__ import annotations

import numpy as np

HIDDEN = 2880
INTERMEDIATE = 5760
EXPERTS = 32
TOPK = 4
TOKENS = 4096
MOE_TOKENS = 16384
GROUP_ALIGN = 128


def bf16_bits(f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.  No NaNs expected."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(seed))
    return bf16_bits(g.standard_normal(shape, dtype=np.float32) * np.float32(std))


# ---- configurations ------------------------------------------------------------

def pr1_inputs(n: int = 256):
    """PR1: X, Y [n, n] ~ N(0, 1), seeds 0 and 1."""
    return normal_bf16((n, n), 0), normal_bf16((n, n), 1)


def activations_with_outliers(rows: int = TOKENS, cols: int = HIDDEN, seed: int = 2,
                              frac: float = 0.01, factor: float = 50.0) -> np.ndarray:
    """N(0, 1) activations with round(frac*cols) seeded outlier columns scaled by factor."""
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal((rows, cols), dtype=np.float32)
    n_out = int(round(frac * cols))
    cols_out = g.choice(cols, size=n_out, replace=False)
    x[:, cols_out] *= np.float32(factor)
    return bf16_bits(x)


def fprop_inputs(tokens: int = TOKENS):
    """Expert gate_up fprop: X [tokens, 2880] (1% outlier columns x50, seed 2),
    W [5760, 2880] ~ N(0, 0.02^2) (seed 3)."""
    x = activations_with_outliers(tokens, HIDDEN, seed=2)
    w = normal_bf16((INTERMEDIATE, HIDDEN), 3, 0.02)
    return x, w


def backward_inputs(tokens: int = TOKENS):
    """Expert backward: dY [tokens, 5760] ~ N(0, 1e-3^2), seed 4."""
    return normal_bf16((tokens, INTERMEDIATE), 4, 1e-3)


SR_SEED = 42


def zipf_probs(n: int = EXPERTS, s: float = 1.2) -> np.ndarray:
    p = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return p / p.sum()


def route_tokens(tokens: int = MOE_TOKENS, experts: int = EXPERTS, topk: int = TOPK, seed: int = 6,
                 s: float = 1.2) -> np.ndarray:
    """Per token, topk distinct experts drawn without replacement from Zipf(s)
    over the expert ranks (expert e has rank e+1).  Gumbel-top-k draws exactly
    that distribution.  Returns int32 [tokens, topk]."""
    g = np.random.Generator(np.random.PCG64(seed))
    logp = np.log(zipf_probs(experts, s))
    keys = logp[None, :] + g.gumbel(size=(tokens, experts))
    return np.argsort(-keys, axis=1)[:, :topk].astype(np.int32)


def grouped_layout(choice: np.ndarray, experts: int = EXPERTS, align: int = GROUP_ALIGN):
    """Sort routed (token, slot) rows by expert into a padded contiguous layout.

    Returns (row_token, group_offsets, group_sizes, total_rows):
      row_token[r]     token feeding padded row r, or -1 for a padding row;
      group_offsets[e] start row of expert e (multiples of align), [experts+1];
      group_sizes[e]   routed rows of expert e.
    """
    tokens, topk = choice.shape
    flat_e = choice.reshape(-1)
    flat_t = np.repeat(np.arange(tokens, dtype=np.int32), topk)
    order = np.argsort(flat_e, kind="stable")
    sizes = np.bincount(flat_e, minlength=experts).astype(np.int32)
    padded = ((sizes + align - 1) // align) * align
    offsets = np.zeros(experts + 1, np.int32)
    offsets[1:] = np.cumsum(padded)
    total = int(offsets[-1])
    row_token = np.full(total, -1, np.int32)
    pos = 0
    for e in range(experts):
        n = int(sizes[e])
        row_token[offsets[e]:offsets[e] + n] = flat_t[order[pos:pos + n]]
        pos += n
    return row_token, offsets, sizes, total


def grouped_inputs(tokens: int = MOE_TOKENS, experts: int = EXPERTS, hidden: int = HIDDEN,
                   inter: int = INTERMEDIATE):
    """Grouped MoE: token activations [tokens, hidden] N(0,1) seed 5, routing
    seed 6, padded routed activations, gate_up weights [E, inter, hidden] and
    down weights [E, hidden, hidden] ~ N(0, 0.02^2) (seeds 8 and 9)."""
    x = normal_bf16((tokens, hidden), 5)
    choice = route_tokens(tokens, experts, seed=6)
    row_token, offsets, sizes, total = grouped_layout(choice, experts)
    a = np.zeros((total, hidden), np.uint16)
    valid = row_token >= 0
    a[valid] = x[row_token[valid]]
    w_gate_up = normal_bf16((experts, inter, hidden), 8, 0.02)
    w_down = normal_bf16((experts, hidden, hidden), 9, 0.02)
    return dict(x=x, choice=choice, row_token=row_token, offsets=offsets, sizes=sizes, a=a,
                w_gate_up=w_gate_up, w_down=w_down)


def sweep_shape(nbytes: int, cols: int) -> tuple[int, int]:
    """Bandwidth sweep: rows = floor(elems / cols) rounded down to a multiple of 32."""
    elems = nbytes // 2
    rows = (elems // cols) // 32 * 32
    return rows, cols


def student_t_bf16(shape, seed: int = 7, df: float = 3.0, outlier_frac: float = 1e-3,
                   factor: float = 100.0) -> np.ndarray:
    """Student-t(df) values with outlier_frac of the positions (seeded) scaled by factor."""
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_t(df, size=shape).astype(np.float32)
    n = int(x.size * outlier_frac)
    idx = g.choice(x.size, size=n, replace=False)
    x.reshape(-1)[idx] *= np.float32(factor)
    return bf16_bits(x)


def student_t_bf16_device(rows: int, cols: int, seed: int = 7, device="cuda", df: float = 3.0,
                          outlier_frac: float = 1e-3, factor: float = 100.0):
    """Large-sweep variant drawn on the device by torch's seeded generator
    (for sizes numpy cannot draw in reasonable time).  Returns a bf16 tensor."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    # Student-t = N / sqrt(chi2_df / df); chi2_df = 2 * Gamma(df/2).
    z = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32)
    chi2 = torch.zeros_like(z)
    for _ in range(int(df)):
        u = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32)
        chi2 += u * u
        del u
    x = z / torch.sqrt(chi2 / df)
    del z, chi2
    n = int(x.numel() * outlier_frac)
    idx = torch.randint(0, x.numel(), (n,), generator=gen, device=device)
    x.view(-1)[idx] *= factor
    return x.to(torch.bfloat16)
