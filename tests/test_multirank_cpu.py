"""The multi-rank host logic of bench.py with two gloo ranks on CPU: the
max-over-ranks step time, per-rank inputs (weak scaling: every rank decodes
its own batch, no collective on the data path) and the reference arm that
only rank 0 runs."""
import argparse
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    from top_block_sparse_b200.inputs import WORKLOADS, make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        # the job's time is its slowest rank's
        slowest = bench.reduce_max(0.25 + rank, world, cpu)
        # every rank draws its own batch
        w = WORKLOADS["tiny_decode"].scaled(ctx_len=256, n_needles=0)
        q = make_inputs(w, seed=bench.rank_seed(rank))["Q"]
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, q.double().sum().reshape(1))
        # the reference arm runs on rank 0 only
        args = argparse.Namespace(ref_pairs=1, warmup=0, steps=1)
        line = bench.run_reference(args, w, rank, world)
        out[rank] = (slowest, [float(x) for x in sums], line is None, None if line is None else line["n_gpus"])
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 1.25                      # max of 0.25 and 1.25
    assert out[0][1] == out[1][1] and out[0][1][0] != out[0][1][1]   # distinct per-rank inputs
    assert out[0][2] is False and out[0][3] == world          # rank 0 reports for the whole job
    assert out[1][2] is True                                  # other ranks print nothing
