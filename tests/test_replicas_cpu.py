"""Multi-GPU layout of bench.py on CPU: N independent replicas, one process per rank, a gloo process group
carrying only the barrier and the max-over-ranks of the measured time (world size 2)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    w, r, _ = bench.dist_init(None, backend="gloo")
    assert (w, r) == (ws, rank)
    bench.barrier(w)
    ms = 100.0 + 50.0 * r  # rank 1 is the slow one
    m = bench.max_over_ranks(ms, w)
    out[r] = (m, bench.replica_throughput(32 * 64, m, w))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_replicas_time_is_the_max_and_value_sums_all_ranks():
    ws = 2
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(ws, _free_port(), out), nprocs=ws, join=True)
        res = dict(out)
    for r in range(ws):
        m, v = res[r]
        assert m == 150.0                       # the slowest rank's time
        assert v == pytest.approx(32 * 64 * 2 / 0.150)  # tokens of both replicas over that time


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(10, 1000.0, 1) == 10.0
