"""Host logic of bench.py's multi-GPU run (one replica per rank, weak
scaling), on CPU with the gloo backend at world size 2: every rank gets its
own seeded inputs of the same shape, the timings are the maximum over the
ranks on every rank, and the whole-job throughput counts every rank's
units. (The GPU side of the run needs the library and a device per rank.)"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        mine = [1.0 + rank, 10.0 - 3.0 * rank, 0.5 * (rank + 1)]
        agg = bench.max_over_ranks(mine, world)
        w, x = bench.make_inputs("llama3.2-3b_T8k", rank)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), agg=np.array(agg), Q=x.Q[0, 0, :4], K=x.K[0, 0, :4],
                 shape=np.array(x.K.shape))
    finally:
        dist.destroy_process_group()


def test_replica_timing_and_inputs_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    z = [np.load(tmp_path / f"r{r}.npz") for r in range(world)]
    for r in range(world):
        np.testing.assert_array_equal(z[r]["agg"], [2.0, 10.0, 1.0])   # max over the ranks, on every rank
    np.testing.assert_array_equal(z[0]["shape"], z[1]["shape"])        # the same workload on every rank
    assert not np.array_equal(z[0]["K"], z[1]["K"])                    # seeded per rank
    assert not np.array_equal(z[0]["Q"], z[1]["Q"])


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1, 512, 0.1) == 512 / 1e-4
    assert bench.job_throughput(4, 512, 0.1) == 4 * 512 / 1e-4
    assert bench.max_over_ranks([0.25, 3.0], 1) == [0.25, 3.0]
