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
