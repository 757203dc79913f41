"""Multi-process (world size 2 and 3, gloo, CPU) checks of the N>1 host logic.

The GEMM path has no exchange step: each rank computes its own shard of every
workload.  What the ranks share is the host logic around it: the partition of
each workload into shards (bench.shard_problem), the max-over-ranks timing
reduction, rank-0-only reporting, and that per-rank work is independent (each
rank's shard, computed alone, equals its slice of the whole problem).  These
run as gloo ranks on the CPU with the oracle standing in for the per-rank GEMM.
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


def _shard_worker(rank, world, port, q):
    """Each rank takes bench.py's shard of a dense, a contiguous and a masked
    problem, computes it alone with the oracle, and the shards are gathered
    on every rank and put side by side."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        import bench
        import oracle
        from fp8_fine_grained_nt_b200 import inputs

        out = {}
        probs = {
            # 5 blocks of N (the last partial: 40 columns) over the ranks
            "dense": inputs.make_dense(20, 4 * 128 + 40, 256, seed=41),
            # 3 experts, one empty, segments 128-aligned
            "contiguous": inputs.make_contiguous(3, 136, 256, seed=42, counts=[130, 0, 70]),
            "masked": inputs.make_masked(5, 24, 136, 256, seed=43, masked_m=[24, 3, 0, 17, 9]),
        }
        for kind, whole in probs.items():
            mine = bench.shard_problem(whole, rank, world)
            if kind == "dense":
                d = oracle.gemm_dense(mine.a, mine.sa, mine.b, mine.sb, mine.M, mine.N, mine.K) \
                    if mine.N else np.zeros((mine.M, 0))
                ref = oracle.gemm_dense(whole.a, whole.sa, whole.b, whole.sb, whole.M, whole.N,
                                        whole.K)
                axis = 1
            elif kind == "contiguous":
                d = oracle.gemm_contiguous(mine.a, mine.sa, mine.b, mine.sb, mine.m_indices,
                                           mine.num_groups, mine.M_sum, mine.N, mine.K) \
                    if mine.num_groups else np.zeros((0, mine.N))
                ref = oracle.gemm_contiguous(whole.a, whole.sa, whole.b, whole.sb,
                                             whole.m_indices, whole.num_groups, whole.M_sum,
                                             whole.N, whole.K)
                axis = 0
            else:
                d = oracle.gemm_masked(mine.a, mine.sa, mine.b, mine.sb, mine.masked_m, mine.G,
                                       mine.M_max, mine.N, mine.K) \
                    if mine.G else np.zeros((0, mine.M_max, mine.N))
                ref = oracle.gemm_masked(whole.a, whole.sa, whole.b, whole.sb, whole.masked_m,
                                         whole.G, whole.M_max, whole.N, whole.K)
                axis = 0
            parts = [None] * world
            dist.all_gather_object(parts, (np.nan_to_num(d, nan=-7.0), mine.flops))
            got = np.concatenate([p[0] for p in parts], axis=axis)
            flops = sum(p[1] for p in parts)
            out[kind] = (bool(np.array_equal(got, np.nan_to_num(ref, nan=-7.0))),
                         flops == whole.flops)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, out, None))
    except Exception as e:  # report, never hang the parent
        import traceback
        q.put((rank, None, traceback.format_exc()))


@pytest.mark.parametrize("world", [2, 3])
def test_bench_shards_cover_the_whole_problem(world):
    """bench.py's shard partition at world size 2 and 3 (gloo, CPU): every
    rank's shard computed alone, gathered, equals the whole problem bit for
    bit (the oracle's per-element sums do not depend on the partition), and
    the shards' FLOP add up to the whole."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, out, err in results:
        assert err is None, f"rank {rank}: {err}"
        for kind, (same, flops_ok) in out.items():
            assert same, f"rank {rank}: {kind} shards differ from the whole problem"
            assert flops_ok, f"rank {rank}: {kind} shard FLOP do not add up"


def test_shard_ranges_partition():
    import bench
    for n in (0, 1, 5, 8, 17, 56):
        for world in (1, 2, 3, 4, 8):
            spans = [bench.shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1


def test_gpus_flag_must_match_world_size(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--gpus", "4"])
    assert bench.main() == 2


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class A:
        steps, warmup, gpus, reference_budget_s = 1, 3, 2, 0.1
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line(monkeypatch, capsys):
    """Rank 0 of the reference arm (the CPU oracle on a bounded sample) prints
    one JSON line with the same metric, unit, config and scaling as the
    library's arm, plus its cpu_baseline and a zero-copy e2e."""
    import json
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)

    class A:
        steps, warmup, gpus, reference_budget_s = 1, 1, 1, 0.2
    assert bench.run_reference(A()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["config"] == bench.bench_config(1) and line["scaling"] == "strong"
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
