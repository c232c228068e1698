#!/usr/bin/env python
"""bench.py -- throughput of the MXFP4 training hot path on B200.

One step = the forward and backward MXFP4 pass of one GPT-OSS-20B expert
linear layer (gate_up: hidden 2880 -> intermediate 5760, 4096 tokens) under the
ALTO recipe ("Training an MoE LLM in MXFP4", abstract; "MXFP4" (aiwiki.ai),
"Training with MXFP4"):
  quantize X   one read: 1D row blocks (RNE) and 1D blocks along tokens with
               RHT-32 (RNE)                                [4096 x 2880]
  quantize W   2D 32x32 blocks, RNE, + transposed copy     [5760 x 2880]
  fprop        Y  = X  W^T   (4096 x 5760 x 2880)
  quantize dY  one read: 1D row blocks with stochastic rounding and 1D blocks
               along tokens with RHT-32 (same signs as X) + SR  [4096 x 5760]
  dgrad        dX = dY W     (4096 x 2880 x 5760, B = W^T copy)
  wgrad        dW = dY^T X   (5760 x 2880 x 4096)
Inputs are synthetic (seeded) with the GPT-OSS-20B shapes; the data and weights
of the pages' workloads are not available.

`value` is GEMM TFLOP/s of the whole step (3 x 2*4096*5760*2880 FLOP / step
time); per-kernel GB/s and TFLOP/s with roofline fractions are reported too.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU, weak scaling)
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MXFP4 GEMM TFLOP/s + RHT/SR quantize GB/s, % of B200 roofline"
TOKENS, HIDDEN, INTER = synth.TOKENS, synth.HIDDEN, synth.INTERMEDIATE
SR_SEED = synth.SR_SEED
WORKLOAD = ("gpt-oss-20b expert gate_up linear, MXFP4 fwd+bwd (ALTO recipe): 4096 tokens, 2880->5760; "
            "X 1D-RNE, W 2D-RNE + W^T copy, dY 1D-SR, dY^T/X^T 1D-col RHT32 (SR/RNE); fprop, dgrad, wgrad")
GEMMS = {"fprop": (TOKENS, INTER, HIDDEN), "dgrad": (TOKENS, HIDDEN, INTER), "wgrad": (INTER, HIDDEN, TOKENS)}
STEP_FLOPS = sum(2 * m * n * k for m, n, k in GEMMS.values())
# algorithmic bytes per quantized element: bf16 read + E2M1 codes + one scale per 32
Q1D_BYTES = 2 + 0.5 + 1 / 32
Q2D_T_BYTES = 2 + 0.5 + 0.5 + 1 / 32 + 1 / 32      # 2D with transposed copy, GEMM-ready scales
# dual quantizers: one bf16 read, two sets of codes and GEMM-ready scales
QDUAL_BYTES = 2 + 2 * (0.5 + 1 / 32)
QUANT_OPS = {"quant_x_dual": TOKENS * HIDDEN * QDUAL_BYTES, "quant_w_2d": INTER * HIDDEN * Q2D_T_BYTES,
             "quant_dy_dual_sr": TOKENS * INTER * QDUAL_BYTES}
KERNELS_PER_STEP = len(QUANT_OPS) + len(GEMMS)


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# ncu captures of the kernels of one bench step (one kernel per capture).  The
# figures hold only for the kernel sources they were taken from: a changed
# source gives traffic null.
NCU_TRAFFIC = {
    "gemm": {"sources": ("gemm.cu", "ptx.cuh", "common.cuh"), "sha1": "aa4d623082758f27",
             "bytes": {"fprop": 50.86e6, "dgrad": 22.83e6, "wgrad": 30.06e6}},
    "quant": {"sources": ("quantize.cu", "common.cuh"), "sha1": "018f81653675138a",
              "bytes": {"quant_x_dual": 23.62e6, "quant_w_2d": 33.23e6, "quant_dy_dual_sr": 48.29e6},
              # thread instructions per element (ncu smsp__inst_executed x 32 / elements)
              "inst_per_elem": {"quant_dy_dual_sr": 76.9}},
}


def ncu_inst_per_elem(name: str):
    """Thread instructions per element of a quantizer launch (ncu), or None if
    the kernel source changed since they were counted."""
    import hashlib
    t = NCU_TRAFFIC["quant"]
    m = hashlib.sha1()
    for f in t["sources"]:
        with open(os.path.join(ROOT, "quantize_block_scaled_rht_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    if m.hexdigest()[:16] != t["sha1"]:
        return None
    return t["inst_per_elem"].get(name)


def ncu_traffic(kind: str, names):
    """Mean DRAM bytes per launch over `names`, or None if the kernel changed."""
    import hashlib
    t = NCU_TRAFFIC[kind]
    m = hashlib.sha1()
    for f in t["sources"]:
        with open(os.path.join(ROOT, "quantize_block_scaled_rht_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    if m.hexdigest()[:16] != t["sha1"]:
        return None
    return float(np.mean([t["bytes"][n] for n in names]))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the step
# ---------------------------------------------------------------------------
class ExpertStep:
    """Device buffers and the enqueue order of one step (all on the current stream)."""

    def __init__(self, mx, torch, x_bits, w_bits, dy_bits, device, rank=0, world=1, dw_allreduce=False):
        self.mx, self.torch = mx, torch
        # data-parallel token split: this rank holds tokens [rank * T, (rank + 1) * T)
        # of a global batch of world * T; its quantizations are its slice of the
        # whole batch's (global SR indices), and dW is summed over ranks
        self.row0, self.total_rows = rank * TOKENS, world * TOKENS
        self.world, self.dw_allreduce = world, dw_allreduce
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
        self.x, self.w, self.dy = bf(x_bits), bf(w_bits), bf(dy_bits)
        T, H, I = TOKENS, HIDDEN, INTER
        u8 = lambda *s: torch.empty(s, dtype=torch.uint8, device=device)
        f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=device)
        Q = mx.Quantized
        msb = mx.mma_scales_bytes
        self.qx = Q(u8(T, H // 2), u8(msb(T, H)), T, H, mx.LAYOUT_1D_ROW, mx.SCALES_MMA)
        self.qw = Q(u8(I, H // 2), u8(msb(I, H)), I, H, mx.LAYOUT_2D, mx.SCALES_MMA, u8(H, I // 2), u8(msb(H, I)))
        self.qdy = Q(u8(T, I // 2), u8(msb(T, I)), T, I, mx.LAYOUT_1D_ROW, mx.SCALES_MMA)
        self.qdyt = Q(u8(I, T // 2), u8(msb(I, T)), I, T, mx.LAYOUT_1D_COL, mx.SCALES_MMA)
        self.qxt = Q(u8(H, T // 2), u8(msb(H, T)), H, T, mx.LAYOUT_1D_COL, mx.SCALES_MMA)
        self.y, self.dx, self.dw = f32(T, I), f32(T, H), f32(I, H)

    def ops(self):
        mx = self.mx
        if self.world > 1:
            return self.dp_ops()
        return [
            # X: row blocks (fprop) and blocks along tokens with RHT-32 (wgrad), one read
            ("quant_x_dual", lambda: mx.mxfp4_quantize_dual(self.x, 32, mx.ROUND_RNE, SR_SEED, 0, 0, mx.SCALES_MMA,
                                                            out_row=self.qx, out_col=self.qxt)),
            ("quant_w_2d", lambda: mx.mxfp4_quantize(self.w, mx.LAYOUT_2D, 0, mx.ROUND_RNE, 0, 0, mx.SCALES_MMA,
                                                     out=self.qw)),
            ("fprop", lambda: mx.mxfp4_gemm(self.qx.codes, self.qx.scales, self.qw.codes, self.qw.scales, HIDDEN,
                                            out=self.y)),
            # dY: row blocks with SR (dgrad) and blocks along tokens with RHT-32 + SR (wgrad), one read
            ("quant_dy_dual_sr", lambda: mx.mxfp4_quantize_dual(self.dy, 32, mx.ROUND_SR, SR_SEED, 0, 0,
                                                                mx.SCALES_MMA, out_row=self.qdy, out_col=self.qdyt)),
            ("dgrad", lambda: mx.mxfp4_gemm(self.qdy.codes, self.qdy.scales, self.qw.codes_t, self.qw.scales_t,
                                            INTER, out=self.dx)),
            ("wgrad", lambda: mx.mxfp4_gemm(self.qdyt.codes, self.qdyt.scales, self.qxt.codes, self.qxt.scales,
                                            TOKENS, out=self.dw)),
        ]


    def dp_ops(self):
        """The step of one data-parallel rank: the token-slice forms of the dual
        quantizers (global SR indices), wgrad before dgrad, and with
        dw_allreduce the FP32 all-reduce (sum) of dW over ranks on a side stream,
        overlapping dgrad; the step ends when both have finished."""
        mx, torch = self.mx, self.torch
        import torch.distributed as dist
        if not hasattr(self, "comm_stream"):
            self.comm_stream = torch.cuda.Stream()
            self.ev_dw, self.ev_comm = torch.cuda.Event(), torch.cuda.Event()

        def allreduce_start():
            main = torch.cuda.current_stream()
            self.ev_dw.record(main)
            self.comm_stream.wait_event(self.ev_dw)
            with torch.cuda.stream(self.comm_stream):
                dist.all_reduce(self.dw, op=dist.ReduceOp.SUM)
                self.ev_comm.record(self.comm_stream)

        def allreduce_join():
            torch.cuda.current_stream().wait_event(self.ev_comm)

        ops = [
            ("quant_x_dual", lambda: mx.mxfp4_quantize_dual_rows(self.x, self.row0, self.total_rows, 32, mx.ROUND_RNE,
                                                                 SR_SEED, mx.SCALES_MMA, out_row=self.qx,
                                                                 out_col=self.qxt)),
            ("quant_w_2d", lambda: mx.mxfp4_quantize(self.w, mx.LAYOUT_2D, 0, mx.ROUND_RNE, 0, 0, mx.SCALES_MMA,
                                                     out=self.qw)),
            ("fprop", lambda: mx.mxfp4_gemm(self.qx.codes, self.qx.scales, self.qw.codes, self.qw.scales, HIDDEN,
                                            out=self.y)),
            ("quant_dy_dual_sr", lambda: mx.mxfp4_quantize_dual_rows(self.dy, self.row0, self.total_rows, 32,
                                                                     mx.ROUND_SR, SR_SEED, mx.SCALES_MMA,
                                                                     out_row=self.qdy, out_col=self.qdyt)),
            ("wgrad", lambda: mx.mxfp4_gemm(self.qdyt.codes, self.qdyt.scales, self.qxt.codes, self.qxt.scales,
                                            TOKENS, out=self.dw)),
        ]
        if self.dw_allreduce:
            ops.append(("dw_allreduce_start", allreduce_start))
        ops.append(("dgrad", lambda: mx.mxfp4_gemm(self.qdy.codes, self.qdy.scales, self.qw.codes_t,
                                                   self.qw.scales_t, INTER, out=self.dx)))
        if self.dw_allreduce:
            ops.append(("dw_allreduce_join", allreduce_join))
        return ops


def rank_inputs(rank: int):
    """Seeded synthetic inputs; rank r draws its own tokens (weak scaling)."""
    if rank == 0:
        x, w = synth.fprop_inputs()
        dy = synth.backward_inputs()
    else:
        x = synth.activations_with_outliers(TOKENS, HIDDEN, seed=2 + 1000 * rank)
        w = synth.normal_bf16((INTER, HIDDEN), 3, 0.02)                # weights replicated
        dy = synth.normal_bf16((TOKENS, INTER), 4 + 1000 * rank, 1e-3)
    return x, w, dy


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(x, w, dy, tokens: int, hidden: int, inter: int):
    """Run the step on a sub-problem (first `tokens` tokens, first hidden/inter
    features) through the oracle; returns (seconds, GEMM FLOPs of the sample)."""
    import oracle
    xs = np.ascontiguousarray(x[:tokens, :hidden])
    ws = np.ascontiguousarray(w[:inter, :hidden])
    dys = np.ascontiguousarray(dy[:tokens, :inter])
    t0 = time.perf_counter()
    cx, sx = oracle.quantize(xs, oracle.LAYOUT_1D_ROW)
    cw, sw, cwt = oracle.quantize(ws, oracle.LAYOUT_2D, transposed_copy=True)
    oracle.gemm(cx, sx, cw, sw, hidden, 0, 1, want_abs=False)
    cdy, sdy = oracle.quantize(dys, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, SR_SEED)
    oracle.gemm(cdy, sdy, cwt, sw, inter, 0, 2, want_abs=False)
    cdyt, sdyt = oracle.quantize(dys, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, SR_SEED)
    cxt, sxt = oracle.quantize(xs, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_RNE, SR_SEED)
    oracle.gemm(cdyt, sdyt, cxt, sxt, tokens, want_abs=False)
    dt = time.perf_counter() - t0
    return dt, 3 * 2 * tokens * hidden * inter


def cpu_baseline(x, w, dy):
    import oracle
    tokens = 64
    dt, flops = oracle_sample(x, w, dy, tokens, HIDDEN, INTER)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"the step on {tokens} of {TOKENS} tokens (full 2880/5760 features, W quantized in full): "
                      f"{flops / 1e9:.2f} GFLOP in {dt:.2f} s"}


def run_reference(args, rank):
    """Reference arm: the oracle as it stands on the host cores, each step a
    bounded sample of the workload, sized so that the run ends in minutes."""
    if rank != 0:
        return 0
    import oracle
    x, w, dy = rank_inputs(0)
    # calibrate on the smallest sample, then pick the sub-problem for the budget
    budget_s = args.ref_budget_s
    n_total = args.steps + args.warmup
    ladder = [(32, 256, 512), (32, 512, 1024), (32, 1024, 2048), (64, 1440, 2880), (64, HIDDEN, INTER)]
    dt0, fl0 = oracle_sample(x, w, dy, *ladder[0])
    choice = ladder[0]
    for cand in ladder[1:]:
        est = dt0 * (cand[0] * cand[1] * cand[2]) / (ladder[0][0] * ladder[0][1] * ladder[0][2])
        if est * n_total <= budget_s:
            choice = cand
    for _ in range(args.warmup):
        oracle_sample(x, w, dy, *choice)
    t_sum, flops = 0.0, 0
    for _ in range(args.steps):
        dt, fl = oracle_sample(x, w, dy, *choice)
        t_sum += dt
        flops += fl
    value = flops / t_sum / 1e12
    sample = (f"per step the step on a {choice[0]} tokens x {choice[1]} hidden x {choice[2]} intermediate "
              f"sub-problem of the workload ({3 * 2 * choice[0] * choice[1] * choice[2] / 1e6:.1f} MFLOP)")
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000 * t_sum / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": TOKENS, "hidden": HIDDEN, "intermediate": INTER},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# rows the step does not exercise: the grouped MoE GEMM and the quantizer sweep
# ---------------------------------------------------------------------------
def _timed(torch, fn, reps):
    """Median time of `reps` launches (ms), events on the current stream."""
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ts]))


def grouped_bench(mx, torch, device, peaks, reps=10):
    """Grouped MoE GEMMs on 16384 tokens routed top-4 of 32 experts (Zipf 1.2,
    rows sorted by expert, groups padded to 128 rows), forward and backward of
    the expert layers: gate_up 2880 -> 5760 and down 2880 -> 2880 (fprop), and
    for gate_up the dgrad (dY W_e through the 2D transposed weight copies) and
    the wgrad (dW_e = dY_e^T X_e over each expert's tokens, both operands
    quantized along tokens with RHT-32).  Activations N(0,1), gradients
    N(0, 1e-3^2) and weights N(0, 0.02^2) are drawn on the device with seeded
    generators (the recipe of synth.grouped_inputs), padding rows zero, and
    quantized by the library.  Operands (A 94-190 MB, B up to 265 MB) and
    outputs (0.75-2.1 GB) exceed L2, so no flush is needed between launches.
    TFLOP/s count the routed rows, not the padding."""
    E, H, I = synth.EXPERTS, synth.HIDDEN, synth.INTERMEDIATE
    choice = synth.route_tokens(synth.MOE_TOKENS, E, seed=6)
    _, offsets, sizes, total = synth.grouped_layout(choice, E)
    valid = np.zeros(total, bool)
    for e in range(E):
        valid[offsets[e]:offsets[e] + sizes[e]] = True
    pad = torch.from_numpy(~valid).to(device)
    g = torch.Generator(device=device)
    g.manual_seed(5)
    a = torch.randn((total, H), generator=g, device=device).to(torch.bfloat16)
    a[pad] = 0
    qa = mx.mxfp4_quantize(a, mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    off_d = torch.from_numpy(offsets).to(device)
    size_d = torch.from_numpy(sizes).to(device)
    routed = int(sizes.sum())
    out = {}

    def record(name, ms, flops, shape):
        tf = flops / (ms / 1e3) / 1e12
        out[name] = {"us": ms * 1e3, "TFLOP/s": tf, "frac_fp4_peak": tf / (4 * peaks["bf16"]), "shape": shape}

    wt_codes = wt_scales = None
    for name, n_out, seed in (("gate_up", I, 8), ("down", H, 9)):
        g.manual_seed(seed)
        codes, scales, codes_t, scales_t = [], [], [], []
        for _ in range(E):
            w = (torch.randn((n_out, H), generator=g, device=device) * 0.02).to(torch.bfloat16)
            q = mx.mxfp4_quantize(w, mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA, transposed_copy=name == "gate_up")
            codes.append(q.codes)
            scales.append(q.scales)
            if name == "gate_up":
                codes_t.append(q.codes_t)
                scales_t.append(q.scales_t)
        b_codes, b_scales = torch.stack(codes), torch.cat(scales)
        if name == "gate_up":
            wt_codes, wt_scales = torch.stack(codes_t), torch.cat(scales_t)
        del codes, scales, codes_t, scales_t
        c = torch.empty((qa.codes.shape[0], n_out), dtype=torch.float32, device=device)
        ms = _timed(torch, lambda: mx.mxfp4_grouped_gemm(qa.codes, qa.scales, off_d, size_d, b_codes, b_scales,
                                                          n_out, H, out=c), reps)
        record(name, ms, 2.0 * routed * n_out * H, f"{routed} routed rows ({total} padded) x {n_out} x {H}")
        del c
        if name == "gate_up":
            # the same product with the bf16 epilogue (half the output bytes)
            c16 = torch.empty((qa.codes.shape[0], n_out), dtype=torch.bfloat16, device=device)
            ms = _timed(torch, lambda: mx.mxfp4_grouped_gemm_bf16(qa.codes, qa.scales, off_d, size_d, b_codes,
                                                                   b_scales, n_out, H, out=c16), reps)
            record("gate_up_bf16_out", ms, 2.0 * routed * n_out * H,
                   f"{routed} routed rows ({total} padded) x {n_out} x {H}, bf16 output")
            del c16
        del b_codes, b_scales

    # backward of gate_up: dgrad through W^T copies, wgrad over each expert's tokens
    g.manual_seed(4)
    dy = (torch.randn((total, I), generator=g, device=device) * 1e-3).to(torch.bfloat16)
    dy[pad] = 0
    qdy = mx.mxfp4_quantize(dy, mx.LAYOUT_1D_ROW, 0, mx.ROUND_SR, synth.SR_SEED, scale_layout=mx.SCALES_MMA)
    c = torch.empty((total, H), dtype=torch.float32, device=device)
    ms = _timed(torch, lambda: mx.mxfp4_grouped_gemm(qdy.codes, qdy.scales, off_d, size_d, wt_codes, wt_scales,
                                                      H, I, out=c), reps)
    record("gate_up_dgrad", ms, 2.0 * routed * H * I, f"{routed} routed rows ({total} padded) x {H} x {I}")
    del c, qdy, wt_codes, wt_scales
    qdyt = mx.mxfp4_quantize(dy, mx.LAYOUT_1D_COL, 32, mx.ROUND_SR, synth.SR_SEED, scale_layout=mx.SCALES_MMA)
    qxt = mx.mxfp4_quantize(a, mx.LAYOUT_1D_COL, 32, mx.ROUND_RNE, synth.SR_SEED, scale_layout=mx.SCALES_MMA)
    del dy, a
    c = torch.empty((E * I, H), dtype=torch.float32, device=device)
    ms = _timed(torch, lambda: mx.mxfp4_grouped_gemm_wgrad(qdyt.codes, qdyt.scales, qxt.codes, qxt.scales, off_d,
                                                            total, out=c), reps)
    record("gate_up_wgrad", ms, 2.0 * routed * I * H, f"{E} experts x {I} x {H}, K = {routed} routed rows")
    del c
    c16 = torch.empty((E * I, H), dtype=torch.bfloat16, device=device)
    ms = _timed(torch, lambda: mx.mxfp4_grouped_gemm_wgrad_bf16(qdyt.codes, qdyt.scales, qxt.codes, qxt.scales,
                                                                 off_d, total, out=c16), reps)
    record("gate_up_wgrad_bf16_out", ms, 2.0 * routed * I * H,
           f"{E} experts x {I} x {H}, K = {routed} routed rows, bf16 output")
    if mx.mxfp4_get_error() != mx.MXFP4_OK:
        raise RuntimeError("device-side error in the grouped GEMMs")
    del c16, qdyt, qxt, qa
    torch.cuda.empty_cache()
    return out


class L2Flush:
    """Evicts L2 between timed launches, outside their events: writes a buffer
    larger than L2, then reads a second one, so that the lines left in L2 are
    clean.  After a write alone the timed launch also pays for writing the
    flush's 126 MB of dirty lines back to HBM (the sweep's 256 MiB row
    quantizer measured 0.85 of HBM that way, 0.99 with the read)."""

    def __init__(self, torch, device, mib=256):
        self.w = torch.empty(mib << 20, dtype=torch.uint8, device=device)
        self.r = torch.zeros(mib << 20, dtype=torch.uint8, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.amax()


def _timed_flushed(torch, fn, reps, flush):
    """Median time (ms) of `reps` launches, L2 flushed before each (outside the
    events), events on the current stream."""
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ts]))


SWEEP_MIB = (64, 128, 256, 512, 1024, 2048)
SWEEP_COLS = (2880, 5760)


def sweep_bench(mx, torch, device, peaks, sizes_mib=SWEEP_MIB, widths=SWEEP_COLS, reps=5):
    """The quantizer bandwidth sweep: bf16 tensors of 64 MiB to 2 GiB with rows
    of 2880 and of 5760 elements (rows rounded down to a multiple of 32) of
    Student-t(3) values with 0.1% outliers x100 (drawn on the device, seed 7);
    every layout x RHT size x rounding, quantize and then dequantize (bf16
    out).  Algorithmic bytes per element: 2 read + 0.5 + 1/32 written (1D;
    2D: + 1/1024), and the reverse for dequantize.  L2 is flushed before every
    launch, so the tensors that fit in L2 are timed from HBM too.  Each mode
    maps to [quantize GB/s, fraction of HBM, dequantize GB/s, fraction]."""
    flush = L2Flush(torch, device)
    hbm = peaks["hbm"]
    table = {}
    worst = {}
    for cols in widths:
        for mib in sizes_mib:
            rows, _ = synth.sweep_shape(mib << 20, cols)
            x = synth.student_t_bf16_device(rows, cols, seed=7, device=device)
            n = rows * cols
            out = torch.empty_like(x)
            res = {}
            for layout, lname in ((mx.LAYOUT_1D_ROW, "row"), (mx.LAYOUT_1D_COL, "col"), (mx.LAYOUT_2D, "2d")):
                sbytes = 1 / 1024 if layout == mx.LAYOUT_2D else 1 / 32
                for rht in (0, 16, 32):
                    for rnd, rname in ((mx.ROUND_RNE, "rne"), (mx.ROUND_SR, "sr")):
                        q = mx.mxfp4_quantize(x, layout, rht, rnd, 42)
                        tq = _timed_flushed(torch, lambda: mx.mxfp4_quantize(x, layout, rht, rnd, 42, out=q), reps,
                                            flush)
                        td = _timed_flushed(torch, lambda: mx.mxfp4_dequantize(q.codes, q.scales, rows, cols, layout,
                                                                               rht, 42, out=out), reps, flush)
                        gq = n * (2 + 0.5 + sbytes) / (tq / 1e3) / 1e9
                        gd = n * (2 + 0.5 + sbytes) / (td / 1e3) / 1e9
                        key = f"{lname}_rht{rht}_{rname}"
                        res[key] = [round(gq), round(gq / hbm, 3), round(gd), round(gd / hbm, 3)]
                        w = worst.setdefault(key, [1e9, 1e9])
                        w[0], w[1] = min(w[0], gq / hbm), min(w[1], gd / hbm)
                        del q
            table[f"{mib}MiB_x{cols}"] = {"shape": f"{rows} x {cols}", "modes": res}
            del x, out
            torch.cuda.empty_cache()
    # the scale-rule variants cost no extra traffic; measured on the 1D-row and
    # 2D RNE paths at 1 GiB x 2880
    rows, cols = synth.sweep_shape(1 << 30, 2880)
    x = synth.student_t_bf16_device(rows, cols, seed=7, device=device)
    n = rows * cols
    rules = {}
    for layout, lname in ((mx.LAYOUT_1D_ROW, "row"), (mx.LAYOUT_2D, "2d")):
        sbytes = 1 / 1024 if layout == mx.LAYOUT_2D else 1 / 32
        for rule, rname in ((mx.SCALE_ROUNDUP, "roundup"), (mx.SCALE_PRESCALE_34, "prescale34")):
            q = mx.mxfp4_quantize(x, layout, 0, mx.ROUND_RNE, 42, scale_rule=rule)
            tq = _timed_flushed(torch, lambda: mx.mxfp4_quantize(x, layout, 0, mx.ROUND_RNE, 42, out=q,
                                                                 scale_rule=rule), reps, flush)
            gq = n * (2 + 0.5 + sbytes) / (tq / 1e3) / 1e9
            rules[f"{lname}_rht0_rne_{rname}"] = [round(gq), round(gq / hbm, 3)]
            del q
    if mx.mxfp4_get_error() != mx.MXFP4_OK:
        raise RuntimeError("device-side error in the sweep")
    del x, flush
    torch.cuda.empty_cache()
    return {"sizes": table, "scale_rules_1GiB_x2880": rules,
            "worst_frac_over_sizes": {k: [round(a, 3), round(b, 3)] for k, (a, b) in worst.items()},
            "columns": "mode: [quantize GB/s, fraction of HBM, dequantize GB/s, fraction of HBM]",
            "note": "SR modes are bound by the integer work of Philox4x32-10 and the exact SR decision, not HBM"}


def bf16_out_bench(mx, torch, device, peaks, reps=20):
    """The expert fprop GEMM (4096 x 5760 x 2880, activations N(0,1), weights
    N(0, 0.02^2) drawn on the device) with its FP32 output and with the fused
    epilogues (bf16 output; MXFP4 output, 1D row blocks RNE); L2 flushed
    before each launch."""
    g = torch.Generator(device=device)
    g.manual_seed(2)
    a = torch.randn((TOKENS, HIDDEN), generator=g, device=device).to(torch.bfloat16)
    w = (torch.randn((INTER, HIDDEN), generator=g, device=device) * 0.02).to(torch.bfloat16)
    qa = mx.mxfp4_quantize(a, mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qw = mx.mxfp4_quantize(w, mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA)
    c32 = torch.empty((TOKENS, INTER), dtype=torch.float32, device=device)
    c16 = torch.empty((TOKENS, INTER), dtype=torch.bfloat16, device=device)
    cq = mx.mxfp4_gemm_mxfp4(qa.codes, qa.scales, qw.codes, qw.scales, HIDDEN, scale_layout=mx.SCALES_MMA)
    flush = L2Flush(torch, device)
    res = {}
    for name, fn in (("fp32_out", lambda: mx.mxfp4_gemm(qa.codes, qa.scales, qw.codes, qw.scales, HIDDEN, out=c32)),
                     ("bf16_out", lambda: mx.mxfp4_gemm_bf16(qa.codes, qa.scales, qw.codes, qw.scales, HIDDEN,
                                                             out=c16)),
                     ("mxfp4_out", lambda: mx.mxfp4_gemm_mxfp4(qa.codes, qa.scales, qw.codes, qw.scales, HIDDEN,
                                                               scale_layout=mx.SCALES_MMA, out=cq))):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            ts.append((e0, e1))
        torch.cuda.synchronize()
        ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in ts]))
        tf = 2.0 * TOKENS * INTER * HIDDEN / (ms / 1e3) / 1e12
        res[name] = {"us": ms * 1e3, "TFLOP/s": tf, "frac_fp4_peak": tf / (4 * peaks["bf16"])}
    if mx.mxfp4_get_error() != mx.MXFP4_OK:
        raise RuntimeError("device-side error in the bf16-output measurements")
    del qa, qw, c32, c16, cq, a, w, flush
    torch.cuda.empty_cache()
    res["shape"] = f"{TOKENS} x {INTER} x {HIDDEN}"
    return res


def nvfp4_bench(mx, torch, device, peaks, reps=10):
    """NVFP4 ("Comparison with NVFP4": blocks of 16, E4M3 block scale, FP32
    tensor scale): quantize (tensor amax + blocks) of the 1 GiB sweep tensor,
    and the GEMM at the expert fprop shape 4096 x 5760 x 2880 (activations
    N(0,1), weights N(0, 0.02^2), L2 flushed before each launch)."""
    rows, cols = synth.sweep_shape(1 << 30, 2880)
    x = synth.student_t_bf16_device(rows, cols, seed=7, device=device)
    n = rows * cols
    q = mx.mxfp4_nvfp4_quantize(x)
    tq = _timed(torch, lambda: mx.mxfp4_nvfp4_quantize(x, out=q), 5)
    # bytes: the amax pass reads x once more; 2 + 2 read, 0.5 + 1/16 written
    gq = n * (2 + 0.5 + 1 / 16) / (tq / 1e3) / 1e9
    del q, x
    g = torch.Generator(device=device)
    g.manual_seed(2)
    a = torch.randn((TOKENS, HIDDEN), generator=g, device=device).to(torch.bfloat16)
    w = (torch.randn((INTER, HIDDEN), generator=g, device=device) * 0.02).to(torch.bfloat16)
    qa = mx.mxfp4_nvfp4_quantize(a, scale_layout=mx.SCALES_MMA)
    qw = mx.mxfp4_nvfp4_quantize(w, scale_layout=mx.SCALES_MMA)
    c = torch.empty((TOKENS, INTER), dtype=torch.float32, device=device)
    flush = L2Flush(torch, device)

    # time the GEMM alone: events around the launch, the flush before them
    mx.mxfp4_nvfp4_gemm(qa, qw, out=c)
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mx.mxfp4_nvfp4_gemm(qa, qw, out=c)
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in ts]))
    if mx.mxfp4_get_error() != mx.MXFP4_OK:
        raise RuntimeError("device-side error in the NVFP4 measurements")
    tf = 2.0 * TOKENS * INTER * HIDDEN / (ms / 1e3) / 1e12
    del qa, qw, c, a, w, flush
    torch.cuda.empty_cache()
    return {"quantize_1GiB": {"us": tq * 1e3, "GB/s": gq, "frac_hbm": gq / peaks["hbm"],
                              "note": "algorithmic bytes 2.5625 per element; the amax pass reads the tensor again"},
            "gemm_fprop": {"us": ms * 1e3, "TFLOP/s": tf, "frac_fp4_peak": tf / (4 * peaks["bf16"]),
                           "shape": f"{TOKENS} x {INTER} x {HIDDEN}"}}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="reference arm: host seconds the warm-up and timed samples may take together")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-mib", type=int, default=256)
    ap.add_argument("--dw-allreduce", action="store_true",
                    help="N > 1: the data-parallel training step -- the token split of a global batch with an FP32 "
                         "NCCL all-reduce (sum) of dW every step; without it the ranks run independent steps")
    ap.add_argument("--ncu-case", default=None,
                    help="profiling case for one ncu capture: run the step once to build the operands, then the named "
                         "launch of the step (fprop, dgrad, wgrad, quant_x_dual, quant_w_2d, quant_dy_dual_sr) "
                         "--steps times, and exit without timing or a JSON line")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the grouped-MoE GEMM and quantizer-sweep measurements (1-GPU runs only)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        sys.exit(run_reference(args, rank))

    import torch
    import torch.distributed as dist
    import quantize_block_scaled_rht_b200 as mx

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    mx.lib()
    peaks = load_peaks()

    x, w, dy = rank_inputs(rank)
    dp_kw = dict(rank=rank, world=world, dw_allreduce=args.dw_allreduce and world > 1)
    step = ExpertStep(mx, torch, x, w, dy, device, **dp_kw)
    ops = step.ops()
    if args.ncu_case is not None and args.ncu_case.startswith("sweep:"):
        # sweep:<row|col|2d>:<rht>:<rne|sr>:<quant|dequant>:<MiB>[:<cols>] -- one
        # quantizer-sweep launch on a tensor of that size (drawn on the device)
        _, lname, rht, rname, what, mib, *rest = args.ncu_case.split(":")
        layout = {"row": mx.LAYOUT_1D_ROW, "col": mx.LAYOUT_1D_COL, "2d": mx.LAYOUT_2D}[lname]
        rnd = {"rne": mx.ROUND_RNE, "sr": mx.ROUND_SR}[rname]
        rows, cols = synth.sweep_shape(int(mib) << 20, int(rest[0]) if rest else 2880)
        xs = synth.student_t_bf16_device(rows, cols, seed=7, device=device)
        q = mx.mxfp4_quantize(xs, layout, int(rht), rnd, 42)
        out = torch.empty_like(xs)
        fn = ((lambda: mx.mxfp4_quantize(xs, layout, int(rht), rnd, 42, out=q)) if what == "quant" else
              (lambda: mx.mxfp4_dequantize(q.codes, q.scales, rows, cols, layout, int(rht), 42, out=out)))
        for _ in range(args.steps):
            fn()
        torch.cuda.synchronize()
        if mx.mxfp4_get_error() != mx.MXFP4_OK:
            raise RuntimeError("device-side error in the profiling case")
        print(f"ncu case {args.ncu_case}: {rows} x {cols}, {args.steps} launches", flush=True)
        return
    if args.ncu_case is not None:
        named = dict(ops)
        if args.ncu_case not in named:
            ap.error(f"--ncu-case must be one of {sorted(named)}")
        for _, fn in ops:
            fn()
        torch.cuda.synchronize()
        for _ in range(args.steps):
            named[args.ncu_case]()
        torch.cuda.synchronize()
        if mx.mxfp4_get_error() != mx.MXFP4_OK:
            raise RuntimeError("device-side error in the profiling case")
        print(f"ncu case {args.ncu_case}: {args.steps} launches after one step", flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    flush = L2Flush(torch, device, args.flush_mib)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        for _, fn in ops:
            fn()
    torch.cuda.synchronize()
    if mx.mxfp4_get_error() != mx.MXFP4_OK:
        raise RuntimeError("device-side error during warm-up")

    K = args.steps
    n_ops = len(ops)
    sampler = ClockSampler(local)

    def run_steps(n, per_op):
        """n steps, L2 flushed before each; events at the step boundaries, or
        also between kernels (the breakdown pass: an event between two launches
        keeps the second from starting early, so the step time is taken
        without them)."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ops + 1 if per_op else 2)] for _ in range(n)]
        for i in range(n):
            flush()                                     # L2 flush between timed steps (outside the step)
            e = evs[i]
            e[0].record(stream)
            for j, (_, fn) in enumerate(ops):
                fn()
                if per_op:
                    e[j + 1].record(stream)
            if not per_op:
                e[1].record(stream)
        return evs

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)   # let the sampler start before the load
    t_wall = time.perf_counter()
    evs = run_steps(K, per_op=False)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    err = mx.mxfp4_get_error()
    if err != mx.MXFP4_OK:
        raise RuntimeError(f"device-side error in the timed region: {mx.status_string(err)}")
    step_ms = np.array([e[0].elapsed_time(e[1]) for e in evs])
    total_ms = float(step_ms.sum())
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / K
    value = STEP_FLOPS * world / (total_ms / K / 1e3) / 1e12

    # breakdown pass: the same steps with an event after every kernel
    KB = min(K, 300)
    evs_b = run_steps(KB, per_op=True)
    torch.cuda.synchronize()
    per_op = np.zeros((KB, n_ops))
    for i in range(KB):
        for j in range(n_ops):
            per_op[i, j] = evs_b[i][j].elapsed_time(evs_b[i][j + 1])     # ms

    # per-kernel figures (averaged over the breakdown pass)
    names = [n for n, _ in ops]
    avg_ms = per_op.mean(axis=0)
    kernels = {}
    gemm_ms = 0.0
    quant_ms, quant_bytes = 0.0, 0.0
    for j, n in enumerate(names):
        if n.startswith("dw_allreduce"):
            # the collective's issue (start) and the wait for it after dgrad (join)
            kernels[n] = {"us": avg_ms[j] * 1e3, "bytes": step.dw.numel() * 4}
            continue
        if n in GEMMS:
            m_, n_, k_ = GEMMS[n]
            tf = 2 * m_ * n_ * k_ / (avg_ms[j] / 1e3) / 1e12
            kernels[n] = {"us": avg_ms[j] * 1e3, "TFLOP/s": tf, "frac_fp4_peak": tf / (4 * peaks["bf16"])}
            gemm_ms += avg_ms[j]
        else:
            gbs = QUANT_OPS[n] / (avg_ms[j] / 1e3) / 1e9
            kernels[n] = {"us": avg_ms[j] * 1e3, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm"]}
            quant_ms += avg_ms[j]
            quant_bytes += QUANT_OPS[n]
    gemm_tf = STEP_FLOPS / (gemm_ms / 1e3) / 1e12
    fp4_peak = 4 * peaks["bf16"]
    roofline = {"bound": "tensor", "kernel": "mxfp4_gemm_kernel (fprop+dgrad+wgrad launches)",
                "achieved": gemm_tf, "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tf / fp4_peak,
                "traffic": ncu_traffic("gemm", list(GEMMS)),
                "traffic_note": "mean DRAM bytes per GEMM launch from ncu (cold caches); output lines still in "
                                "L2 when the kernel ends are not counted as writes",
                "peak_note": f"dense FP4 = 4 x {peaks['src']} bf16 burst ({peaks['bf16']} TFLOP/s), "
                             "the nominal 9 : 2.25 PFLOP/s ratio"}
    quant_gbs = quant_bytes / (quant_ms / 1e3) / 1e9
    roofline_q = {"bound": "hbm", "kernel": "mxfp4 quantize kernels (3 launches per step)", "achieved": quant_gbs,
                  "peak": peaks["hbm"], "unit": "GB/s", "frac": quant_gbs / peaks["hbm"],
                  "traffic": ncu_traffic("quant", list(QUANT_OPS)),
                  "peak_note": f"{peaks['src']} copy bandwidth"}

    # The SR dual quantizer of dY is bound by integer issue, not by HBM: its
    # thread instructions per second (ncu count per element x elements / the
    # breakdown pass's time) against the issue rate of 4 schedulers x 32 lanes
    # per SM per cycle at the SM clock sampled during the timed region.
    roofline_sr = None
    ipe = ncu_inst_per_elem("quant_dy_dual_sr")
    if ipe is not None and clocks:
        n_sms = torch.cuda.get_device_properties(device).multi_processor_count
        ach = ipe * TOKENS * INTER / (kernels["quant_dy_dual_sr"]["us"] / 1e6) / 1e12
        peak_i = n_sms * 4 * 32 * clocks["sm_mhz"] * 1e6 / 1e12
        roofline_sr = {"bound": "alu", "kernel": "quant_dual_sr_kernel (dY: row SR + column RHT-32 SR)",
                       "achieved": ach, "peak": peak_i, "unit": "T thread-instructions/s", "frac": ach / peak_i,
                       "traffic": ncu_traffic("quant", ["quant_dy_dual_sr"]),
                       "peak_note": f"issue rate {n_sms} SMs x 4 schedulers x 32 lanes x {clocks['sm_mhz']:.0f} MHz "
                                    f"(median sampled); {ipe} thread instructions per element from ncu"}

    # end to end through the public API with host buffers.  Every step copies
    # its inputs in from pinned host memory and its three results out, inside
    # the timed region.  Two device buffer sets and three streams (upload,
    # compute, download) let step i+1's upload and step i-1's download run
    # while step i computes; the host link is full duplex.  Events order the
    # reuse of each set: its inputs are overwritten only after the step that
    # read them has finished, its outputs only after their download.
    e2e = None
    if args.e2e_steps > 0:
        sets = [step, ExpertStep(mx, torch, x, w, dy, device, **dp_kw)]
        set_ops = [st.ops() for st in sets]
        hx = step.x.cpu().pin_memory()
        hw = step.w.cpu().pin_memory()
        hdy = step.dy.cpu().pin_memory()
        hout = [tuple(torch.empty(t.shape, dtype=torch.float32).pin_memory() for t in (st.y, st.dx, st.dw))
                for st in sets]
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            b = i & 1
            st = sets[b]
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(ev_done[b])
                st.x.copy_(hx, non_blocking=True)
                st.w.copy_(hw, non_blocking=True)
                st.dy.copy_(hdy, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if used[b]:
                stream.wait_event(ev_out[b])
            for _, fn in set_ops[b]:
                fn()
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                for h, d in zip(hout[b], (st.y, st.dx, st.dw)):
                    h.copy_(d, non_blocking=True)
                ev_out[b].record(s_out)
            used[b] = True

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(4, 4 + args.e2e_steps):
            e2e_step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        if world > 1:
            t = torch.tensor([e2e_ms], dtype=torch.float64, device=device)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        hy, hdx, hdw = hout[0]
        h2d = (hx.numel() + hw.numel() + hdy.numel()) * 2
        d2h = (hy.numel() + hdx.numel() + hdw.numel()) * 4
        e2e = {"value": STEP_FLOPS * world / (e2e_ms / args.e2e_steps / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.e2e_steps}

    extras = {}
    if world == 1 and not args.no_extras:
        extras["grouped_moe"] = grouped_bench(mx, torch, device, peaks)
        extras["quantizer_sweep"] = sweep_bench(mx, torch, device, peaks)
        extras["nvfp4"] = nvfp4_bench(mx, torch, device, peaks)
        extras["gemm_bf16_out"] = bf16_out_bench(mx, torch, device, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x, w, dy)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "mxfp4 e2m1/e8m0 operands, fp32 accumulate", "data": "synthetic",
                "config": {"workload": WORKLOAD, "tokens_per_gpu": TOKENS, "hidden": HIDDEN, "intermediate": INTER,
                           "parallelism": (f"dp{world} (token split of a {world * TOKENS}-token batch; FP32 NCCL "
                                           f"all-reduce of dW every step, overlapping dgrad)" if dp_kw["dw_allreduce"]
                                           else f"dp{world} (independent tokens per rank, no collective)"),
                           "l2": f"flushed between timed steps, outside the step events: a {args.flush_mib} MiB write, then a "
                                 f"{args.flush_mib} MiB read of another buffer (clean lines left in L2)"},
                "roofline": roofline, "roofline_quantize": roofline_q, "roofline_sr_dual": roofline_sr,
                "kernels": kernels,
                "quantize_GBps": quant_gbs, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": KERNELS_PER_STEP * K, "clocks": clocks, "wall_s_timed_region": t_wall,
                "breakdown": f"per-kernel figures from {KB} further steps with an event after every kernel",
                **extras}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
