"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The decode has no exchange step (replicas only), so the only cross-rank
traffic is plumbing: the encoded blob broadcast from rank 0, barriers, and
the max-over-ranks time / sum-over-ranks bytes that make up the reported
throughput.  These run here with the gloo backend; no GPU is involved.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(backend="gloo")
    blob = np.arange(1000, dtype=np.uint8) if rank == 0 else None
    got = d.broadcast_bytes(blob)
    d.barrier()
    ms, units = bench.combine(10.0 + rank, 100.0 * (rank + 1), d)
    out[rank] = (bool(np.array_equal(got, np.arange(1000, dtype=np.uint8))), ms, units, d.world, d.rank)
    d.close()


def test_two_rank_plumbing():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for rank in (0, 1):
        ok, ms, units, world, r = res[rank]
        assert ok and world == 2 and r == rank
        assert ms == 11.0          # slowest rank's time
        assert units == 300.0      # all ranks' decoded bytes


def test_reference_arm_other_ranks_do_nothing(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_single_rank_combine_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    os.environ.pop("WORLD_SIZE", None)
    d = bench.Dist()
    assert d.world == 1
    assert bench.combine(5.0, 7.0, d) == (5.0, 7.0)
