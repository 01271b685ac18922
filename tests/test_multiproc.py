"""The multi-process path of bench.py on CPU: two gloo ranks, each timing its
own copy of the workload, agree on the max-over-ranks step time and the
whole-job throughput (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    step_ms = bench.max_over_ranks(local_ms, torch.device("cpu"))
    bench.barrier()
    wl = bench.synth.WORKLOADS["mid_32k_d128"]
    value = w * wl.attn_flops / (step_ms * 1e-3) / 1e12
    out[rank] = (step_ms, value)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1]
    step_ms, value = out[0]
    assert step_ms == 15.0
    assert abs(value - 2 * 4 * 40 * 32768 ** 2 * 128 / 15e-3 / 1e12) < 1e-6
