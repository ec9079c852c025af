"""Multi-rank host logic of the replica run (2 ranks, gloo, CPU): timings combine as the
slowest rank, the job's throughput counts every rank's tokens, and ranks draw different
sequences."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_dsa_b200 import replicas, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        replicas.barrier()
        mx = replicas.max_over_ranks(local_ms)
        thr = replicas.job_throughput(200000, world, mx)
        gen = synth.StructuredIndexer("replica", 1, 64, 4, 16, r=4, base_std=1.0, noise_std=0.2, device="cpu",
                                      seed=replicas.rank_seed(1000, rank))
        k = gen.keys(0)
        gathered = [torch.zeros_like(k) for _ in range(world)]
        dist.all_gather(gathered, k)
        out[rank] = (mx, thr, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    for r in range(world):
        mx, thr, same = res[r]
        assert mx == 150.0                       # the slowest rank's time, on every rank
        assert thr == pytest.approx(2 * 200000 / 0.150)
        assert not same                          # each rank its own sequence


def test_single_process_is_identity():
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.job_throughput(10, 1, 1000.0) == pytest.approx(10.0)
    with pytest.raises(ValueError):
        replicas.job_throughput(10, 1, 0.0)
