"""Multi-rank plumbing of bench.py on CPU: two gloo ranks.

The path has no data exchange (every rank runs its own replica of the
workload), so the multi-GPU logic is: disjoint input streams per rank, a
barrier, the slowest rank's time (max over ranks) and the whole-job
throughput.  These run here with the gloo backend, no GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from decode_attention_q4kv_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank reports a different elapsed time; all must agree on the max
        mx = bench.reduce_max(0.5 + rank, torch.device("cpu"))
        # disjoint data: the first K row of layer 0 differs between ranks
        w = W.TINY
        k, _ = W.kv_tokens(w, bench.rank_layer_id(0, rank), 4, "cpu")
        gathered = [torch.zeros_like(k) for _ in range(world)]
        dist.all_gather(gathered, k)
        dist.barrier()
        out.put((rank, mx, all(not torch.equal(gathered[0], gathered[r]) for r in range(1, world))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, disjoint in results:
        assert mx == 1.5
        assert disjoint


def test_throughput_and_single_rank_reduce():
    assert bench.job_throughput(4, 1e9, 10, 2.0) == 20.0
    assert bench.reduce_max(3.25, torch.device("cpu")) == 3.25   # no process group: identity
    assert bench.rank_layer_id(7, 0) == 7 and bench.rank_layer_id(7, 2) == 2007
