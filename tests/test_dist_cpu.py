"""Multi-rank host logic of bench.py on the CPU: two gloo ranks (no GPU).

The GPU path has no data-path collective (independent replicas); the process
group only carries the barrier and the max-over-ranks step time. These tests
run that logic with world_size 2 over gloo on 127.0.0.1.
"""

import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import bench
    from synthetic import MOE_CONFIGS
    w, r, _ = bench.dist_setup(backend="gloo")
    try:
        assert (w, r) == (world, rank)
        bench.barrier(w)
        step = 1.0 + rank  # the slower replica sets the job's time
        slowest = bench.max_over_ranks(step, w, device="cpu")
        inp = bench.rank_inputs(MOE_CONFIGS["moe_small_c40"], rank)
        out[rank] = {"slowest": slowest,
                     "value": bench.job_throughput(300, w, slowest),
                     "x_sum": float(inp["x"].float().sum()),
                     "w_sum": float(inp["wgu"].float().sum() + inp["wd"].float().sum())}
        bench.barrier(w)
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_replica_inputs():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0]["slowest"] == res[1]["slowest"] == 2.0
    assert res[0]["value"] == res[1]["value"] == 2 * 300 / 2.0
    assert res[0]["w_sum"] == res[1]["w_sum"]       # one model on every replica
    assert res[0]["x_sum"] != res[1]["x_sum"]       # each replica its own batch


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(8192, 1, 0.5) == 16384.0
    torch.manual_seed(0)
