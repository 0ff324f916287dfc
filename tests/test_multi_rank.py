"""Replica (multi-rank) host logic of bench.py on CPU: two gloo ranks.

The operator's (sequence, head) chains are independent, so several GPUs run
independent replicas; the only cross-rank traffic is the timing reduction.
These tests cover that host logic without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import kda_inputs
        res = {}
        res["max"] = bench._max_over_ranks(float(rank + 1), ws)
        res["sum"] = bench._sum_over_ranks(float(rank + 1), ws)
        # rank r processed 1000 (r + 1) units in 10 (r + 1) ms
        res["thr"] = bench.replica_throughput(1000.0 * (rank + 1), 10.0 * (rank + 1), ws)
        bench._barrier(ws)
        seed = bench.replica_seed(1, rank)
        inp = kda_inputs.make_prefill([16], 2, torch.float32, torch.float32, 3.0, False, seed)
        res["seed"] = seed
        res["q_sum"] = float(inp["q"].double().sum())
        out.put((rank, res))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_draw_distinct_batches():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(ws):
        assert got[r]["max"] == 2.0
        assert got[r]["sum"] == 3.0
        # (1000 + 2000) units over the slowest rank's 20 ms
        assert got[r]["thr"] == pytest.approx(3000.0 / 0.020)
    assert got[0]["seed"] != got[1]["seed"]
    assert got[0]["q_sum"] != got[1]["q_sum"]
