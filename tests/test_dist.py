"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The data path has no collective (ranks process independent batches); the
ranks only agree on timing: max over ranks, whole-job rate = units of all
ranks / slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [3.0, 5.0][rank]
    m = bench.max_over_ranks(ms, world, device="cpu")
    rate = bench.whole_job_rate(4096, world, m)
    seed = bench.rank_seed("prefill4k", rank)
    t = torch.tensor([m, rate, float(seed)], dtype=torch.float64)
    gathered = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(gathered, t)
    if rank == 0:
        out.put([g.tolist() for g in gathered])
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_agree_on_max_time_and_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (m0, r0, s0), (m1, r1, s1) = res
    assert m0 == m1 == 5.0
    assert r0 == r1 == pytest.approx(2 * 4096 / 5e-3)
    assert s0 != s1  # independent batches per rank
