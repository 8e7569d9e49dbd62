"""World-size-2 check of the benchmark's multi-rank host logic on CPU (gloo).

Every rank runs its own layer (independent problems, no data-path
collective); timings are combined as the max over ranks and throughput is
the bytes of all ranks over that max."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from dequant_gemv_tq4_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [1.0 + rank, 5.0 - rank, 2.5]
        out[rank] = {
            "max": bench.max_over_ranks(times, world),
            "seed": bench.rank_seed(rank),
            "k_head": inputs.llama3_8b_layer(seed=bench.rank_seed(rank), names=["k"])[0]["k"][:2, :64].float()
            .numpy().tolist(),
        }
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_timing_and_independent_layers():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0]["max"] == out[1]["max"] == [2.0, 5.0, 2.5]
    assert out[0]["seed"] != out[1]["seed"]
    assert out[0]["k_head"] != out[1]["k_head"]  # each rank has its own layer
    # whole-job throughput: bytes of all ranks over the slowest rank's time
    assert abs(bench.job_gbs(1_000_000_000, world, 2.0) - 1000.0) < 1e-9
