"""Multi-rank path on CPU: two gloo ranks quantize their shards with element
offsets from quantize_block_scaled_rht_b200.shard, gather, and must reproduce
the single-process quantization bit for bit (stochastic rounding included)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from quantize_block_scaled_rht_b200.shard import LAYOUT_1D_COL, LAYOUT_1D_ROW, LAYOUT_2D, shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, layout, out_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    rows, cols = 192, 96
    x = synth.student_t_bf16((rows, cols), seed=31)
    sh = shard(rows, cols, world, rank, layout)
    part = x[sh.start:sh.start + sh.size] if sh.axis == 0 else x[:, sh.start:sh.start + sh.size]
    codes, scales = oracle.quantize(np.ascontiguousarray(part), layout, 32, oracle.ROUND_SR, 42,
                                    sh.elem_offset)[:2]
    gathered_c = [None] * world
    gathered_s = [None] * world
    dist.all_gather_object(gathered_c, codes)
    dist.all_gather_object(gathered_s, scales)
    if rank == 0:
        np.save(os.path.join(out_dir, "codes.npy"), np.concatenate(gathered_c, axis=0))
        np.save(os.path.join(out_dir, "scales.npy"), np.concatenate(gathered_s, axis=0))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("layout", [LAYOUT_1D_ROW, LAYOUT_1D_COL, LAYOUT_2D])
def test_two_gloo_ranks_reproduce_single_process_sr(tmp_path, layout):
    import oracle
    import synth
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), layout, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    x = synth.student_t_bf16((192, 96), seed=31)
    codes, scales = oracle.quantize(x, layout, 32, oracle.ROUND_SR, 42)[:2]
    assert np.array_equal(np.load(tmp_path / "codes.npy"), codes)
    assert np.array_equal(np.load(tmp_path / "scales.npy"), scales)


def test_shard_bounds_cover_exactly():
    for world in (1, 2, 3, 8):
        for layout in (LAYOUT_1D_ROW, LAYOUT_1D_COL, LAYOUT_2D):
            rows, cols = 32 * 13, 32 * 7
            parts = [shard(rows, cols, world, r, layout) for r in range(world)]
            ext = cols if layout == LAYOUT_1D_COL else rows
            assert parts[0].start == 0 and sum(p.size for p in parts) == ext
            for a, b in zip(parts, parts[1:]):
                assert a.start + a.size == b.start and a.size % 32 == 0
    with pytest.raises(ValueError):
        shard(33, 64, 2, 0)


def _dw_worker(rank, world, port, out_dir):
    """One data-parallel rank of the expert layer's weight gradient: quantize
    this rank's token slice along tokens (X with RHT-32 + RNE, dY with RHT-32 +
    SR, both as slices of the whole batch), form the local dW = dY_r^T X_r, and
    all-reduce (sum) it across ranks."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    T, H, I = 256, 64, 96
    x = synth.student_t_bf16((T, H), seed=41)
    dy = synth.normal_bf16((T, I), 43, 1e-3)
    sh = shard(T, H, world, rank, LAYOUT_1D_ROW)          # token split on 32-row boundaries
    t0, n = sh.start, sh.size
    cx, sx = oracle.quantize(np.ascontiguousarray(x[t0:t0 + n]), LAYOUT_1D_COL, 32, oracle.ROUND_RNE, 42,
                             elem_offset=t0, sr_ld=T)
    cdy, sdy = oracle.quantize(np.ascontiguousarray(dy[t0:t0 + n]), LAYOUT_1D_COL, 32, oracle.ROUND_SR, 42,
                               elem_offset=t0, sr_ld=T)
    dw, s = oracle.gemm(cdy, sdy, cx, sx, n)                 # [I, H] over this rank's tokens, fp64
    dw_t = torch.from_numpy(np.ascontiguousarray(dw))
    s_t = torch.from_numpy(np.ascontiguousarray(s))
    dist.all_reduce(dw_t, op=dist.ReduceOp.SUM)
    dist.all_reduce(s_t, op=dist.ReduceOp.SUM)
    parts = [None] * world
    dist.all_gather_object(parts, (t0, cdy, sdy, cx, sx))
    if rank == 0:
        np.save(os.path.join(out_dir, "dw.npy"), dw_t.numpy())
        np.save(os.path.join(out_dir, "s.npy"), s_t.numpy())
        import pickle
        with open(os.path.join(out_dir, "parts.pkl"), "wb") as f:
            pickle.dump(parts, f)
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_wgrad_allreduce_matches_single_process(tmp_path):
    """Token-split weight gradient with the one exchange of data-parallel
    training, an all-reduce (sum) of dW: every rank's quantized slices equal the
    whole batch's bit for bit (global SR indices), and the summed dW equals the
    single-process dW within 1e-5 * sum |a b| ("Conversion rules": block dot
    products summed in FP32; here the oracle sums in fp64)."""
    import pickle
    import oracle
    import synth
    world = 2
    mp.start_processes(_dw_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    T, H, I = 256, 64, 96
    x = synth.student_t_bf16((T, H), seed=41)
    dy = synth.normal_bf16((T, I), 43, 1e-3)
    cx, sx = oracle.quantize(x, LAYOUT_1D_COL, 32, oracle.ROUND_RNE, 42)
    cdy, sdy = oracle.quantize(dy, LAYOUT_1D_COL, 32, oracle.ROUND_SR, 42)
    dw_ref, s_ref = oracle.gemm(cdy, sdy, cx, sx, T)
    with open(tmp_path / "parts.pkl", "rb") as f:
        parts = pickle.load(f)
    for t0, pcdy, psdy, pcx, psx in parts:
        n = pcdy.shape[1] * 2
        assert np.array_equal(pcdy, cdy[:, t0 // 2:(t0 + n) // 2]) and np.array_equal(psdy, sdy[:, t0 // 32:(t0 + n) // 32])
        assert np.array_equal(pcx, cx[:, t0 // 2:(t0 + n) // 2]) and np.array_equal(psx, sx[:, t0 // 32:(t0 + n) // 32])
    dw = np.load(tmp_path / "dw.npy")
    assert np.allclose(np.load(tmp_path / "s.npy"), s_ref, rtol=1e-12, atol=0)
    assert np.all(np.abs(dw - dw_ref) <= 1e-5 * s_ref)
    assert np.abs(dw_ref).max() > 0
