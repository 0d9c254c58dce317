"""bench.py's multi-rank logic on CPU: two gloo ranks, the max-over-ranks time,
distinct per-rank batches and the whole-job throughput formula."""
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from exact_attention_106_b200 import workloads as W
        mx = bench.reduce_max(10.0 * (rank + 1), torch.device("cpu"))
        w = bench.rank_workload(W.TINY, rank)
        out[rank] = (mx, w.seed_base)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 20.0          # max over ranks, seen by every rank
    assert out[0][1] != out[1][1]                  # each rank draws its own batch


def test_job_throughput_and_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5   # no process group: identity
    # 2 ranks x 10 steps x 1e12 flop in 1 s -> 20 TFLOP/s
    assert abs(bench.job_throughput(2, 1e12, 10, 1000.0) - 20.0) < 1e-9
