"""GPU parity at the full workload sizes, in the launch configuration bench.py
times: the GPT-OSS-20B expert linear fwd+bwd step (fprop 4096x5760x2880,
dgrad 4096x2880x5760, wgrad 5760x2880x4096 with RHT-32 + SR along tokens), the
grouped MoE GEMM (16384 tokens, top-4 of 32 Zipf-routed experts), and the
quantizer bandwidth sweep (64 MiB in full, 2 GiB on sampled rows).

Quantizer outputs are compared bit for bit; GEMM outputs on sampled entries the
oracle computes one by one, within |C - C_fp64| <= 1e-5 * sum|a b|.
"""
import numpy as np
import pytest
import torch

import oracle
import quantize_block_scaled_rht_b200 as mx
import synth
from mxfp4_testutil import assert_gemm_close, dev_bf16, expand_2d, from_mma, host

pytestmark = pytest.mark.gpu


def _sample_pairs(M, N, n, seed):
    g = np.random.default_rng(seed)
    pairs = list(zip(g.integers(0, M, n), g.integers(0, N, n)))
    pairs += [(0, 0), (M - 1, N - 1), (M - 1, 0), (0, N - 1)]
    return pairs


def _check_sampled(c_gpu, ca, sa, cb, sb, K, pairs, a_mode=0, b_mode=0):
    ref, s = oracle.gemm_entries(ca, sa, cb, sb, K, pairs, a_mode, b_mode)
    got = np.array([c_gpu[m, n] for m, n in pairs], np.float64)
    assert_gemm_close(got, ref, s)


@pytest.fixture(scope="module")
def expert_step():
    """Run the bench step once (same buffers and calls as bench.ExpertStep)."""
    import bench
    x, w, dy = bench.rank_inputs(0)
    step = bench.ExpertStep(mx, torch, x, w, dy, torch.device("cuda"))
    for _, fn in step.ops():
        fn()
    torch.cuda.synchronize()
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    return x, w, dy, step


def test_expert_quantizers_bit_exact(expert_step):
    x, w, dy, st = expert_step
    T, H, I = synth.TOKENS, synth.HIDDEN, synth.INTERMEDIATE
    cx, sx = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    assert np.array_equal(host(st.qx.codes), cx)
    assert np.array_equal(from_mma(host(st.qx.scales), T, H), sx)
    cw, sw, cwt = oracle.quantize(w, oracle.LAYOUT_2D, transposed_copy=True)
    assert np.array_equal(host(st.qw.codes), cw) and np.array_equal(host(st.qw.codes_t), cwt)
    assert np.array_equal(from_mma(host(st.qw.scales), I, H), expand_2d(sw, I))
    assert np.array_equal(from_mma(host(st.qw.scales_t), H, I), expand_2d(sw.T, H))
    cdy, sdy = oracle.quantize(dy, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, synth.SR_SEED)
    assert np.array_equal(host(st.qdy.codes), cdy)
    assert np.array_equal(from_mma(host(st.qdy.scales), T, I), sdy)
    cdyt, sdyt = oracle.quantize(dy, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, synth.SR_SEED)
    assert np.array_equal(host(st.qdyt.codes), cdyt)
    assert np.array_equal(from_mma(host(st.qdyt.scales), I, T), sdyt)
    cxt, sxt = oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_RNE, synth.SR_SEED)
    assert np.array_equal(host(st.qxt.codes), cxt)
    assert np.array_equal(from_mma(host(st.qxt.scales), H, T), sxt)


def test_expert_gemms_sampled(expert_step):
    x, w, dy, st = expert_step
    T, H, I = synth.TOKENS, synth.HIDDEN, synth.INTERMEDIATE
    cx, sx = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    cw, sw, cwt = oracle.quantize(w, oracle.LAYOUT_2D, transposed_copy=True)
    cdy, sdy = oracle.quantize(dy, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, synth.SR_SEED)
    cdyt, sdyt = oracle.quantize(dy, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, synth.SR_SEED)
    cxt, sxt = oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_RNE, synth.SR_SEED)
    _check_sampled(host(st.y), cx, sx, cw, sw, H, _sample_pairs(T, I, 3000, 1), 0, 1)
    _check_sampled(host(st.dx), cdy, sdy, cwt, sw, I, _sample_pairs(T, H, 2000, 2), 0, 2)
    _check_sampled(host(st.dw), cdyt, sdyt, cxt, sxt, T, _sample_pairs(I, H, 2000, 3))


def test_expert_gemms_bf16_output(expert_step):
    """The three expert GEMMs with the bf16 epilogue, from the step's quantized
    operands: every entry is the round-to-nearest-even of the FP32 product,
    and sampled entries fall within the bf16 bound of the fp64 oracle."""
    x, w, dy, st = expert_step
    T, H, I = synth.TOKENS, synth.HIDDEN, synth.INTERMEDIATE
    cases = [(st.qx, st.qw.codes, st.qw.scales, H, st.y), (st.qdy, st.qw.codes_t, st.qw.scales_t, I, st.dx),
             (st.qdyt, st.qxt.codes, st.qxt.scales, T, st.dw)]
    for qa, b_codes, b_scales, K, c32 in cases:
        c16 = mx.mxfp4_gemm_bf16(qa.codes, qa.scales, b_codes, b_scales, K)
        torch.cuda.synchronize()
        assert torch.equal(c16.view(torch.int16), c32.to(torch.bfloat16).view(torch.int16))
    cx, sx = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    cw, sw = oracle.quantize(w, oracle.LAYOUT_2D)[:2]
    pairs = _sample_pairs(T, I, 2000, 4)
    ref, s = oracle.gemm_entries(cx, sx, cw, sw, H, pairs, 0, 1)
    c16 = host(mx.mxfp4_gemm_bf16(st.qx.codes, st.qx.scales, st.qw.codes, st.qw.scales, H).float())
    got = np.array([c16[m, n] for m, n in pairs], np.float64)
    err = np.abs(got - ref)
    bound = 1e-5 * s + 2.0 ** -8 * (np.abs(ref) + 1e-5 * s)   # FP32 bound + one bf16 rounding
    assert np.all(err <= bound)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK


@pytest.fixture(scope="module")
def moe():
    return synth.grouped_inputs()


def test_grouped_moe_gate_up_sampled(moe):
    """16384 tokens x 2880, top-4 of 32 experts (Zipf 1.2), gate_up 2880 -> 5760."""
    d = moe
    E, N, K = synth.EXPERTS, synth.INTERMEDIATE, synth.HIDDEN
    rows = d["a"].shape[0]
    qa = mx.mxfp4_quantize(dev_bf16(d["a"]), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    wq = [mx.mxfp4_quantize(dev_bf16(d["w_gate_up"][e]), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA)
          for e in range(E)]
    b_codes = torch.stack([q.codes for q in wq])
    b_scales = torch.cat([q.scales for q in wq])
    offsets = torch.from_numpy(d["offsets"]).cuda()
    sizes = torch.from_numpy(d["sizes"]).cuda()
    c = mx.mxfp4_grouped_gemm(qa.codes, qa.scales, offsets, sizes, b_codes, b_scales, N, K)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    c = host(c)
    ca, sa = oracle.quantize(d["a"], oracle.LAYOUT_1D_ROW)
    assert np.array_equal(host(qa.codes), ca)
    g = np.random.default_rng(5)
    for e in range(E):
        o, n = int(d["offsets"][e]), int(d["sizes"][e])
        if n == 0:
            continue
        cw, sw = oracle.quantize(d["w_gate_up"][e], oracle.LAYOUT_2D)
        rs = np.unique(np.concatenate([g.integers(0, n, 12), [0, n - 1]]))
        pairs = [(int(o + r), int(cc)) for r in rs for cc in g.integers(0, N, 8)]
        ref, s = oracle.gemm_entries(ca, sa, cw, sw, K, pairs, 0, 1)
        got = np.array([c[m, nn] for m, nn in pairs], np.float64)
        assert_gemm_close(got, ref, s)


def test_expert_dgrad_full_tensor(expert_step):
    """Every entry of the dgrad output (4096 x 2880, K = 5760, the longest
    reduction of the step) against the oracle's fp64 GEMM of the oracle's own
    quantization of dY (row blocks, SR) and of W (2D, transposed copy)."""
    x, w, dy, st = expert_step
    T, H, I = synth.TOKENS, synth.HIDDEN, synth.INTERMEDIATE
    _, sw, cwt = oracle.quantize(w, oracle.LAYOUT_2D, transposed_copy=True)
    cdy, sdy = oracle.quantize(dy, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, synth.SR_SEED)
    ref, s = oracle.gemm(cdy, sdy, cwt, sw, I, 0, 2)
    worst = assert_gemm_close(host(st.dx), ref, s)
    assert worst < 1e-5


def test_grouped_moe_down_sampled(moe):
    """The MoE down projection at full size: 16384 tokens routed top-4 of 32
    experts (65,536 routed rows, groups padded to 128), 2880 -> 2880 per
    expert, activations 1D row RNE, weights 2D RNE, FP32 out; every expert
    sampled (rows including its first and last, random columns)."""
    d = moe
    E, H = synth.EXPERTS, synth.HIDDEN
    qa = mx.mxfp4_quantize(dev_bf16(d["a"]), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    wq = [mx.mxfp4_quantize(dev_bf16(d["w_down"][e]), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA) for e in range(E)]
    offsets = torch.from_numpy(d["offsets"]).cuda()
    sizes = torch.from_numpy(d["sizes"]).cuda()
    c = mx.mxfp4_grouped_gemm(qa.codes, qa.scales, offsets, sizes, torch.stack([q.codes for q in wq]),
                              torch.cat([q.scales for q in wq]), H, H)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    c = host(c)
    del wq
    ca, sa = oracle.quantize(d["a"], oracle.LAYOUT_1D_ROW)
    g = np.random.default_rng(7)
    checked = 0
    for e in range(E):
        o, n = int(d["offsets"][e]), int(d["sizes"][e])
        if n == 0:
            continue
        cw, sw = oracle.quantize(d["w_down"][e], oracle.LAYOUT_2D)
        rs = np.unique(np.concatenate([g.integers(0, n, 12), [0, n - 1]]))
        pairs = [(int(o + r), int(cc)) for r in rs for cc in list(g.integers(0, H, 8)) + [0, H - 1]]
        ref, s = oracle.gemm_entries(ca, sa, cw, sw, H, pairs, 0, 1)
        got = np.array([c[m, nn] for m, nn in pairs], np.float64)
        assert_gemm_close(got, ref, s)
        checked += 1
    assert checked >= 16


def test_grouped_moe_backward_sampled(moe):
    """Backward of the gate_up expert layer on the same routing: dgrad
    dX_e = dY_e W_e through the 2D transposed weight copies, and wgrad
    dW_e = dY_e^T X_e over each expert's tokens (operands quantized along
    tokens with RHT-32; SR for dY).  Sampled entries against the oracle, which
    quantizes only the sampled rows / columns (with their stream offsets)."""
    d = moe
    E, I, H = synth.EXPERTS, synth.INTERMEDIATE, synth.HIDDEN
    offsets, sizes = d["offsets"], d["sizes"]
    total = d["a"].shape[0]
    valid = d["row_token"] >= 0
    dy = np.zeros((total, I), np.uint16)
    dy[valid] = synth.normal_bf16((int(valid.sum()), I), 12, 1e-3)
    seed = synth.SR_SEED
    qdy = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_ROW, 0, mx.ROUND_SR, seed, scale_layout=mx.SCALES_MMA)
    experts = [0, 1, 17, 31]
    codes_t, scales_t = [], []
    for e in range(E):
        q = mx.mxfp4_quantize(dev_bf16(d["w_gate_up"][e]), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA,
                              transposed_copy=True)
        codes_t.append(q.codes_t)
        scales_t.append(q.scales_t)
    off_d, size_d = torch.from_numpy(offsets).cuda(), torch.from_numpy(sizes).cuda()
    dx = host(mx.mxfp4_grouped_gemm(qdy.codes, qdy.scales, off_d, size_d, torch.stack(codes_t),
                                    torch.cat(scales_t), H, I))
    del codes_t, scales_t, qdy
    qdyt = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_COL, 32, mx.ROUND_SR, seed, scale_layout=mx.SCALES_MMA)
    qxt = mx.mxfp4_quantize(dev_bf16(d["a"]), mx.LAYOUT_1D_COL, 32, mx.ROUND_RNE, seed, scale_layout=mx.SCALES_MMA)
    dw = mx.mxfp4_grouped_gemm_wgrad(qdyt.codes, qdyt.scales, qxt.codes, qxt.scales, off_d, total)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    g = np.random.default_rng(13)
    for e in experts:
        o, n = int(offsets[e]), int(sizes[e])
        if n == 0:
            continue
        _, sw, cwt = oracle.quantize(d["w_gate_up"][e], oracle.LAYOUT_2D, transposed_copy=True)
        # dgrad: sampled rows of the expert, quantized with their stream offsets
        for r in np.unique(np.concatenate([g.integers(0, n, 4), [n - 1]])):
            row = o + int(r)
            ca, sa = oracle.quantize(dy[row:row + 1], oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, seed,
                                     elem_offset=row * I)
            cols = [int(c) for c in g.integers(0, H, 6)] + [H - 1]
            ref, s = oracle.gemm_entries(ca, sa, cwt, sw, I, [(0, c) for c in cols], 0, 2)
            assert_gemm_close(dx[row, cols].astype(np.float64), ref, s)
        # wgrad: sampled (m, n) of dW_e from single columns of dY and X over the expert's tokens
        k0, k1 = o, int(offsets[e + 1])
        for m, col in zip(g.integers(0, I, 4), g.integers(0, H, 4)):
            m, col = int(m), int(col)
            ca, sa = oracle.quantize(np.ascontiguousarray(dy[:, m:m + 1]), oracle.LAYOUT_1D_COL, 32,
                                     oracle.ROUND_SR, seed, elem_offset=m * total)
            cb, sb = oracle.quantize(np.ascontiguousarray(d["a"][:, col:col + 1]), oracle.LAYOUT_1D_COL, 32,
                                     oracle.ROUND_RNE, seed, elem_offset=col * total)
            ref, s = oracle.gemm_entries(ca[:, k0 // 2:k1 // 2], sa[:, k0 // 32:k1 // 32], cb[:, k0 // 2:k1 // 2],
                                         sb[:, k0 // 32:k1 // 32], k1 - k0, [(0, 0)])
            got = float(dw[e * I + m, col].item())
            assert_gemm_close(np.array([got]), ref, s)
    del qdyt, qxt, dw
    torch.cuda.empty_cache()


@pytest.mark.parametrize("layout", [mx.LAYOUT_1D_ROW, mx.LAYOUT_1D_COL, mx.LAYOUT_2D])
def test_sweep_64mib_all_modes(layout):
    rows, cols = synth.sweep_shape(64 << 20, 2880)
    x = synth.student_t_bf16((rows, cols), seed=7)
    xd = dev_bf16(x)
    for rht in (0, 16, 32):
        for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
            q = mx.mxfp4_quantize(xd, layout, rht, rnd, 42)
            codes, scales = oracle.quantize(x, layout, rht, rnd, 42)[:2]
            assert np.array_equal(host(q.codes), codes), (rht, rnd)
            assert np.array_equal(host(q.scales), scales), (rht, rnd)
            back = mx.mxfp4_dequantize(q.codes, q.scales, rows, cols, layout, rht, 42, out_dtype=torch.float32)
            f32, _ = oracle.dequantize(codes, scales, rows, cols, layout, rht, 42)
            assert np.array_equal(host(back).view(np.uint32), f32.view(np.uint32)), (rht, rnd)


def test_sweep_2gib_sampled_rows():
    """Largest sweep size: 2 GiB of bf16 (372,800 x 2880), drawn on the device;
    sampled row blocks are copied back and quantized by the oracle."""
    rows, cols = synth.sweep_shape(2 << 30, 2880)
    x = synth.student_t_bf16_device(rows, cols, seed=7)
    for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
        q = mx.mxfp4_quantize(x, mx.LAYOUT_1D_ROW, 32, rnd, 42)
        g = np.random.default_rng(9)
        for r0 in list(g.integers(0, rows // 32, 6) * 32) + [rows - 32]:
            xs = host(x[r0:r0 + 32])
            codes, scales = oracle.quantize(xs, oracle.LAYOUT_1D_ROW, 32, rnd, 42, elem_offset=int(r0) * cols)
            assert np.array_equal(host(q.codes[r0:r0 + 32]), codes)
            assert np.array_equal(host(q.scales[r0:r0 + 32]), scales)
        del q
    for rnd in (mx.ROUND_SR, mx.ROUND_RNE):     # RNE walks strips of 8 row tiles; the last tile holds 64 rows
        qc = mx.mxfp4_quantize(x, mx.LAYOUT_1D_COL, 32, rnd, 42)
        g = np.random.default_rng(10)
        for c0 in list(g.integers(0, cols // 8, 4) * 8) + [cols - 8]:
            xs = host(x[:, c0:c0 + 8])
            codes, scales = oracle.quantize(np.ascontiguousarray(xs), oracle.LAYOUT_1D_COL, 32, rnd, 42,
                                            elem_offset=int(c0) * rows)
            assert np.array_equal(host(qc.codes[c0:c0 + 8]), codes)
            assert np.array_equal(host(qc.scales[c0:c0 + 8]), scales)
        del qc
    del x
    torch.cuda.empty_cache()


def test_nvfp4_expert_fprop_sampled():
    """NVFP4 at the expert fprop shape: X 4096 x 2880 (with the outlier
    columns), W 5760 x 2880; quantizers bit-exact, GEMM on sampled entries."""
    x, w = synth.fprop_inputs()
    qx = mx.mxfp4_nvfp4_quantize(dev_bf16(x), scale_layout=mx.SCALES_MMA)
    qw = mx.mxfp4_nvfp4_quantize(dev_bf16(w), scale_layout=mx.SCALES_MMA)
    c = host(mx.mxfp4_nvfp4_gemm(qx, qw))
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    cx, sx, ax = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_ROW)
    cw, sw, aw = oracle.nvfp4_quantize(w, oracle.LAYOUT_1D_ROW)
    assert np.array_equal(host(qx.codes), cx) and np.array_equal(host(qw.codes), cw)
    assert float(qx.amax.item()) == ax and float(qw.amax.item()) == aw
    pairs = _sample_pairs(4096, 5760, 1500, 21)
    ref, s = oracle.nvfp4_gemm_entries(cx, sx, ax, cw, sw, aw, 2880, pairs)
    got = np.array([c[m, n] for m, n in pairs], np.float64)
    assert_gemm_close(got, ref, s)
