"""The several-GPU path on the CPU: two `gloo` ranks run the replica plumbing
that `bench.py` uses under torchrun (per-rank seeds, the slowest rank's time,
the whole-job rate).  The layer has no exchange step, so this reduction of
one timing scalar is the only collective of the path."""
import os
import socket
from datetime import timedelta

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_compressed_02_b200 import replicas, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, local = replicas.rank_world()
        ms = 1.5 + rank                                   # this replica's step time
        slowest = replicas.max_over_ranks(ms)
        seed = replicas.replica_seed(r)
        inp, _ = synth.prefill_inputs_device("csa_prefill", "cpu", seed=seed, S=64)
        q.put((r, w, local, slowest, seed, float(inp["q"].float().sum()), replicas.job_rate(100.0, w, slowest * 1e-3)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [x[0] for x in res] == [0, 1] and all(x[1] == 2 and x[2] == x[0] for x in res)
    # every rank sees the slowest replica's time and the same whole-job rate
    assert all(x[3] == 2.5 for x in res)
    assert all(x[6] == pytest.approx(2 * 100.0 / 2.5e-3) for x in res)
    # replicas draw different inputs
    assert res[0][4] != res[1][4] and res[0][5] != res[1][5]


def test_single_process_defaults():
    assert replicas.max_over_ranks(3.25) == 3.25
    assert replicas.replica_seed(0) == 0 and replicas.replica_seed(3, base=1) == 4
    assert replicas.job_rate(10.0, 4, 2.0) == 20.0
    with pytest.raises(ValueError):
        replicas.job_rate(1.0, 1, 0.0)
