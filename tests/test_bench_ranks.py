"""Multi-process checks of bench.py's rank plumbing on CPU (gloo, world size 2).

Every rank solves an independent problem (weak scaling, no data-path
collective); the only collectives are the barrier around the timed region
and the max over ranks of the measured time.  These run here without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    r, w, local, pg = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    dev = torch.device("cpu")
    bench.barrier(pg, dev)
    got = bench.max_over_ranks(1.5 + rank, pg, dev)
    # A rank whose workload seed differs gets a different, equal-size problem.
    import synth
    wl = synth.CONFIGS[1]
    wr = synth.Workload(**{**wl.__dict__, "key": wl.key + 100 * rank})
    q = synth.chunk_tokens(wr, 1, device="cpu", want=("q",))["q"]
    out[rank] = (got, float(q.float().sum()))
    pg.destroy_process_group()


def test_two_rank_max_and_independent_problems():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0][0] == out[1][0] == 2.5          # max over ranks, same on every rank
    assert out[0][1] != out[1][1]                  # each rank has its own inputs


def test_single_rank_needs_no_process_group():
    import bench
    os.environ.pop("WORLD_SIZE", None)
    r, w, local, pg = bench.dist_setup(1)
    assert (r, w, pg) == (0, 1, None)
    assert bench.max_over_ranks(3.0, None, torch.device("cpu")) == 3.0
