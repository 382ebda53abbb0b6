"""Multi-process host logic of a multi-GPU run, on CPU with gloo (world size 2):
rank setup from the environment, max-over-ranks timing and the whole-job
weak-scaling throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from quantized_recurrent_state_lq_b200 import dist as D
    w, r, lr, pg = D.setup(timeout_s=60)
    assert (w, r, lr) == (world, rank, rank) and pg is not None
    D.barrier(pg)
    seconds = 1.0 + rank            # the slower rank decides
    t = D.max_over_ranks(seconds, pg)
    out[rank] = (t, D.weak_scaling_value(1000.0, w, t))
    D.teardown(pg)


def test_two_rank_timing_reduction():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1] == (2.0, 1000.0)


def test_single_process_needs_no_group(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    from quantized_recurrent_state_lq_b200 import dist as D
    w, r, lr, pg = D.setup()
    assert (w, r, lr, pg) == (1, 0, 0, None)
    assert D.max_over_ranks(3.5, pg) == 3.5
    assert D.weak_scaling_value(10.0, 1, 2.0) == 5.0
