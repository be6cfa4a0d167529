"""Row-sharded NVFP4 quantization, host logic on CPU: two gloo ranks each take
the abs-max of their rows, one all-reduce(MAX) gives the tensor's, and the
rank's quantization with it equals the whole tensor's quantization on those
rows. The per-rank arithmetic is the oracle here (the CPU stand-in for the
library kernels the GPU path calls)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import oracle
    from microscaling_fp4_quantization_bf16_b200 import sharded, synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = synth.workload("c3_strategy_sweep_t3", rows=64, cols=256)["x"]
        x = x.float().numpy()
        x[1:32:7] *= 30.0   # the tensor maximum lies in rank 0's rows
        x = synth.to_bf16(x)
        rows = slice(32 * rank, 32 * rank + 32)
        mine = x[rows]
        stand_in = lambda t, rot: torch.tensor([float(oracle.global_amax(synth.bits16(t), rot))])
        for rot in (0, 16):
            ga = sharded.global_amax_sharded(mine, rot, local_amax=stand_in)
            full = oracle.global_amax(synth.bits16(x), rot)
            o_part = oracle.quantize(synth.bits16(mine), "nvfp4", 16, "four_over_six", rot,
                                     global_amax=float(ga.item()))
            o_full = oracle.quantize(synth.bits16(x), "nvfp4", 16, "four_over_six", rot)
            out[(rank, rot)] = (float(ga.item()) == float(full),
                                np.array_equal(o_part["codes"], o_full["codes"][rows]),
                                np.array_equal(o_part["scales"], o_full["scales"][rows]),
                                float(o_part["global_scale"]) == float(o_full["global_scale"]))
    finally:
        dist.destroy_process_group()


def test_sharded_global_amax_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert len(out) == 4
    assert all(all(v) for v in out.values()), dict(out)


@pytest.mark.gpu
def test_sharded_single_rank_nccl_on_gpu():
    """The NCCL form on one GPU (world size 1): the all-reduce is the identity and
    the sharded quantization equals the plain one bit for bit."""
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import microscaling_fp4_quantization_bf16_b200 as fp4q
    from microscaling_fp4_quantization_bf16_b200 import sharded, synth

    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x = synth.workload("c3_strategy_sweep_t3", rows=64, cols=256)["x"].cuda()
        a = sharded.quantize_sharded(x, "nvfp4", 16, "four_over_six", rot=16)
        b = fp4q.quantize(x, "nvfp4", 16, "four_over_six", 16)
        torch.cuda.synchronize()
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
        assert torch.equal(a.global_scale, b.global_scale)
    finally:
        dist.destroy_process_group()
