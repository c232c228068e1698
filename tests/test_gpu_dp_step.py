"""GPU: the data-parallel form of the bench step (token split of a global batch,
dW all-reduced over ranks) on one GPU.

Only one GPU is available to these tests, so the multi-rank exchange itself is
covered on CPU (tests/test_multirank.py, gloo).  Here rank 1 of a 2-rank token
split runs its step through a 1-rank NCCL group: its quantized operands must be
its slice of the whole 2-rank batch's quantization (global SR indices), and the
all-reduce plumbing (side stream, events, the join before the step ends) must
leave dW equal to the rank's own wgrad, bit for bit.
"""
import os
import socket

import numpy as np
import pytest
import torch

import quantize_block_scaled_rht_b200 as mx
from mxfp4_testutil import host

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_dp_step_rank_slice_and_dw_allreduce_plumbing():
    import torch.distributed as dist
    import bench
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev)
    try:
        x0, w, dy0 = bench.rank_inputs(0)
        x1, _, dy1 = bench.rank_inputs(1)
        st = bench.ExpertStep(mx, torch, x1, w, dy1, dev, rank=1, world=2, dw_allreduce=True)
        names = [n for n, _ in st.ops()]
        assert names.index("wgrad") < names.index("dw_allreduce_start") < names.index("dgrad")
        for _, fn in st.ops():
            fn()
        torch.cuda.synchronize()
        assert mx.mxfp4_get_error() == mx.MXFP4_OK
        # the whole batch (rank 0's tokens, then rank 1's), quantized at once
        T = bench.TOKENS
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        X = torch.cat([bf(x0), bf(x1)])
        DY = torch.cat([bf(dy0), bf(dy1)])
        wr, wc = mx.mxfp4_quantize_dual(X, 32, mx.ROUND_RNE, bench.SR_SEED)
        dr, dc = mx.mxfp4_quantize_dual(DY, 32, mx.ROUND_SR, bench.SR_SEED)
        assert torch.equal(st.qx.codes, wr.codes[T:])
        assert torch.equal(st.qxt.codes, wc.codes[:, T // 2:])
        assert torch.equal(st.qdy.codes, dr.codes[T:])
        assert torch.equal(st.qdyt.codes, dc.codes[:, T // 2:])
        # a 1-rank all-reduce leaves the rank's own wgrad
        dw = mx.mxfp4_gemm(st.qdyt.codes, st.qdyt.scales, st.qxt.codes, st.qxt.scales, T)
        assert np.array_equal(host(st.dw).view(np.uint32), host(dw).view(np.uint32))
    finally:
        dist.destroy_process_group()
