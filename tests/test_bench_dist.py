"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

Each rank of `bench.py --gpus N` runs its own independent workload (weak
scaling, no collective on the data path); torch.distributed is used only for
barriers and for taking the max of the per-rank times.  This checks that
plumbing with two CPU ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    D = bench.Dist(backend="gloo")
    try:
        D.barrier()
        local = 10.0 + 5.0 * rank          # rank 1 is the slow one
        m = D.max(local)
        out[rank] = (D.rank, D.world, m, bench.rank_seed(1, D.rank))
        D.barrier()
    finally:
        D.close()


def test_two_rank_max_and_seeds():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][2] == out[1][2] == 15.0            # every rank sees the max over ranks
    assert {out[0][0], out[1][0]} == {0, 1} and out[0][1] == 2
    assert out[0][3] != out[1][3]                     # independent workloads per rank


def test_single_rank_needs_no_process_group():
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    D = bench.Dist()
    assert D.world == 1 and D.dist is None
    assert D.max(3.5) == 3.5
    D.barrier()
    D.close()


def test_reference_arm_other_ranks_exit(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""
