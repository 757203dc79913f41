"""Multi-process (world size 2, gloo, CPU) checks of the N>1 host logic.

The GEMM path has no exchange step: each rank runs independent problems.  What
the ranks share is the host logic around it: the max-over-ranks timing
reduction, rank-0-only reporting, and that per-rank work is independent
(rank r's shard of a grouped problem, computed alone, equals that slice of the
whole problem).  These run as gloo ranks on the CPU with the oracle standing in
for the per-rank GEMM.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        import bench
        import oracle
        from fp8_fine_grained_nt_b200 import inputs

        # 1. timing reduction: max over ranks
        mx = bench.max_over_ranks(10.0 + rank, world, device="cpu")

        # 2. independent shards: each rank takes a contiguous range of experts of
        # one masked problem and computes it alone; gathered, the shards equal
        # the whole problem computed at once.
        prob = inputs.make_masked(4, 24, 136, 256, seed=9, masked_m=[24, 3, 0, 17])
        per = prob.G // world
        gs = slice(rank * per, (rank + 1) * per)
        mine = oracle.gemm_masked(prob.a[gs], prob.sa[gs], prob.b[gs], prob.sb[gs],
                                  prob.masked_m[gs], per, prob.M_max, prob.N, prob.K)
        t = torch.from_numpy(np.nan_to_num(mine, nan=-1.0))
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t)
        whole = np.nan_to_num(oracle.gemm_masked(prob.a, prob.sa, prob.b, prob.sb, prob.masked_m,
                                                 prob.G, prob.M_max, prob.N, prob.K), nan=-1.0)
        same = bool(np.array_equal(torch.cat(parts).numpy(), whole))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, mx, same, None))
    except Exception as e:  # report, never hang the parent
        q.put((rank, None, False, repr(e)))


def test_two_gloo_ranks_host_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, mx, same, err in results:
        assert err is None, f"rank {rank}: {err}"
        assert mx == 11.0
        assert same


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class A:
        steps, warmup, gpus, reference_budget_s = 1, 3, 2, 0.1
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""
