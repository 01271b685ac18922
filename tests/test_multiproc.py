"""The multi-process paths on CPU, two gloo ranks:
- bench.py: each rank times its own copy of the workload, and both agree on
  the max-over-ranks step time and the whole-job throughput (weak scaling, no
  data-path collective);
- the head split: head_range partitions the heads, and gather_heads
  assembles the per-rank output heads into the full tensor, uneven splits
  included."""
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


def test_head_range_partitions():
    import bit_fp8_attention_smooth_b200 as vc

    for H in (1, 5, 24, 40, 48):
        for world in (1, 2, 3, 8):
            ranges = [vc.head_range(r, world, H) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        vc.head_range(2, 2, 4)


def _gather_worker(rank, world, port, H, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bit_fp8_attention_smooth_b200 as vc

    h0, h1 = vc.head_range(rank, world, H)
    local = torch.arange(h0, h1, dtype=torch.float32).view(1, h1 - h0, 1, 1).expand(2, h1 - h0, 3, 4).contiguous()
    full = vc.gather_heads(local, H)
    out[rank] = full.clone()
    dist.destroy_process_group()


@pytest.mark.parametrize("H", [4, 5])
def test_gather_heads_two_gloo_ranks(H):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, H, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    expect = torch.arange(H, dtype=torch.float32).view(1, H, 1, 1).expand(2, H, 3, 4)
    for r in range(world):
        assert torch.equal(out[r], expect)
