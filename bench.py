"""Benchmark: FP8 TFLOPS and fraction of the B200 roofline, per shape and in total.

One step = one call of each measured workload through the library's C ABI,
inputs resident in HBM:
  dense 128x128x512, dense decode 64x2112x7168, dense prefill 4096x7168x2048
  and 256x7168x2048, contiguous m-grouped 8 experts x (4096, 7168), masked
  m-grouped 16 x 256 for (N, K) = (4096, 7168) and (7168, 2048).
Inputs are the seeded synthetic workloads of fp8_fine_grained_nt_b200.inputs.
`value` = total algorithmic FLOP of a step / device time of a step (CUDA events,
max over ranks).  `e2e` times the same step through the same C-ABI calls with
the inputs in pinned host memory: host-to-device copies, the GEMMs and the
device-to-host copy of every output inside the timed region.

Multi-GPU: `--gpus N` runs N ranks, one per GPU (under torchrun, or spawned
by this script through torch.distributed.run when WORLD_SIZE is unset).  Each
rank computes its own shard of every workload, with no exchange between ranks
(shard_problem: dense calls split N into 128-column blocks, the contiguous
form splits experts, the masked form splits groups); value = FLOP of the whole
workloads / max-over-ranks time, "scaling": "strong".

--impl reference times the CPU oracle (the only reference that exists for this
path) on a bounded sample of the same workloads, on rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from fp8_fine_grained_nt_b200 import inputs  # noqa: E402

METRIC = "FP8 TFLOPS and % of B200 roofline per shape (dense, contiguous, masked)"
UNIT = "TFLOP/s"
NOMINAL_FP8_TFLOPS = 4500.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
WORKLOAD_NAMES = [
    "dense_128x128x512",
    "dense_decode_64x2112x7168",
    "dense_prefill_4096x7168x2048",
    "dense_prefill_256x7168x2048",
    "contiguous_8x4096x7168",
    "masked_16x256_4096x7168",
    "masked_16x256_7168x2048",
]
WORKLOAD_DESC = ("dense 128x128x512 + decode 64x2112x7168 + prefill 4096x7168x2048 + "
                 "prefill 256x7168x2048 + contiguous 8 experts (4096,7168) + "
                 "masked 16x256 (4096,7168) + masked 16x256 (7168,2048), one call each per step")


def bench_config(world: int) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": WORKLOAD_DESC,
            "l2": "each step streams ~1.6 GB of distinct operands (> 126 MB L2); "
                  "every call's operands are evicted by the rest of the step",
            "parallelism": (f"{world} ranks, each an independent shard of every "
                            "workload (dense: blocks of N; contiguous: experts; "
                            "masked: groups)" if world > 1 else "1 GPU")}


# launch-latency-bound: reported, not a roofline target
LATENCY_BOUND = {"dense_128x128x512"}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- workloads


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Balanced contiguous share [lo, hi) of n units for `rank` of `world`."""
    return n * rank // world, n * (rank + 1) // world


def shard_problem(prob, rank: int, world: int):
    """`rank`'s independent part of a workload: no data moves between ranks,
    and the ranks' outputs, put side by side, are the whole problem's output.

    dense:       a range of 128-column blocks of N (the rows of B and sb of
                 those blocks, all of A); D's columns of those blocks.
    contiguous:  a range of experts: their 128-aligned row segments of A (and
                 sa columns, m_indices renumbered from 0), their B and sb.
    masked:      a range of groups.
    A rank whose range is empty gets a problem with no rows or columns.
    """
    if world == 1:
        return prob
    if isinstance(prob, inputs.DenseProblem):
        nb = inputs.ceil_div(prob.N, 128)
        b0, b1 = shard_range(nb, rank, world)
        c0, c1 = 128 * b0, min(prob.N, 128 * b1)
        return inputs.DenseProblem(prob.M, max(0, c1 - c0), prob.K, prob.a, prob.sa,
                                   prob.b[c0:c1].contiguous(), prob.sb[b0:b1].contiguous(),
                                   prob.seed)
    if isinstance(prob, inputs.ContiguousProblem):
        e0, e1 = shard_range(prob.num_groups, rank, world)
        padded = [inputs.ceil_div(c, inputs.M_ALIGNMENT_CONTIGUOUS) * inputs.M_ALIGNMENT_CONTIGUOUS
                  for c in prob.counts]
        offs = np.concatenate([[0], np.cumsum(padded)]).astype(np.int64)
        r0, r1 = int(offs[e0]), int(offs[e1])
        mi = prob.m_indices[r0:r1].clone()
        mi[mi >= 0] -= e0
        return inputs.ContiguousProblem(e1 - e0, r1 - r0, prob.N, prob.K,
                                        prob.a[r0:r1].contiguous(),
                                        prob.sa[:, r0:r1].contiguous(),
                                        prob.b[e0:e1].contiguous(), prob.sb[e0:e1].contiguous(),
                                        mi, list(prob.counts[e0:e1]), prob.seed)
    g0, g1 = shard_range(prob.G, rank, world)
    return inputs.MaskedProblem(g1 - g0, prob.M_max, prob.N, prob.K, prob.a[g0:g1].contiguous(),
                                prob.sa[g0:g1].contiguous(), prob.b[g0:g1].contiguous(),
                                prob.sb[g0:g1].contiguous(), prob.masked_m[g0:g1].contiguous(),
                                prob.seed)


def problem_is_empty(prob) -> bool:
    if isinstance(prob, inputs.DenseProblem):
        return prob.M == 0 or prob.N == 0
    if isinstance(prob, inputs.ContiguousProblem):
        return prob.num_groups == 0 or prob.M_sum == 0
    return prob.G == 0


class Case:
    """One workload: its device tensors and the C-ABI call that computes it."""

    def __init__(self, name: str, prob, rank: int = 0, world: int = 1):
        self.name = name
        self.kind = type(prob).__name__.replace("Problem", "").lower()
        self.whole_flops = prob.flops  # the whole workload (all ranks' shards)
        self.prob = shard_problem(prob, rank, world)
        self.empty = problem_is_empty(self.prob)
        self.flops = self.prob.flops
        self.bytes = self.prob.algorithmic_bytes
        self.host = {}
        self.dev = {}

    def to_device(self):
        if self.empty:
            return
        p = self.prob
        self.dev = {"a": p.a.cuda(), "sa": p.sa.cuda(), "b": p.b.cuda(), "sb": p.sb.cuda()}
        if self.kind == "dense":
            self.dev["d"] = torch.empty((p.M, p.N), dtype=torch.bfloat16, device="cuda")
        elif self.kind == "contiguous":
            self.dev["mi"] = p.m_indices.cuda()
            self.dev["d"] = torch.empty((p.M_sum, p.N), dtype=torch.bfloat16, device="cuda")
        else:
            self.dev["mm"] = p.masked_m.cuda()
            self.dev["d"] = torch.empty((p.G, p.M_max, p.N), dtype=torch.bfloat16, device="cuda")
            self.expected_m = max(1, int(round(float(p.masked_m.float().mean()))))

    def pin_host(self):
        if self.empty:
            return
        p = self.prob
        self.host = {"a": p.a.pin_memory(), "sa": p.sa.pin_memory(), "b": p.b.pin_memory(),
                     "sb": p.sb.pin_memory(), "d": torch.empty_like(self.dev["d"], device="cpu").pin_memory()}
        if self.kind == "contiguous":
            self.host["mi"] = p.m_indices.pin_memory()
        if self.kind == "masked":
            self.host["mm"] = p.masked_m.pin_memory()

    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for k, t in self.host.items() if k != "d")

    def d2h_bytes(self) -> int:
        if self.empty:
            return 0
        return self.host["d"].numel() * self.host["d"].element_size()

    def call(self, stream=None):
        import fp8_fine_grained_nt_b200 as fp8
        if self.empty:
            return
        d = self.dev
        if self.kind == "dense":
            fp8.gemm_fp8_fp8_bf16_nt(d["a"], d["sa"], d["b"], d["sb"], d["d"], stream=stream)
        elif self.kind == "contiguous":
            fp8.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(d["a"], d["sa"], d["b"], d["sb"], d["d"],
                                                          d["mi"], stream=stream)
        else:
            fp8.m_grouped_gemm_fp8_fp8_bf16_nt_masked(d["a"], d["sa"], d["b"], d["sb"], d["d"],
                                                      d["mm"], self.expected_m, stream=stream)

    def e2e_call(self, stream):
        if self.empty:
            return
        for k, t in self.host.items():
            if k != "d":
                self.dev[k].copy_(t, non_blocking=True)
        self.call(stream)
        self.host["d"].copy_(self.dev["d"], non_blocking=True)

    def roofline_time_s(self, peaks) -> tuple[float, str]:
        fp8_peak = 2.0 * peaks["bf16_tflops"] * 1e12
        t_tensor = self.flops / fp8_peak
        t_hbm = self.bytes / (peaks["hbm_gbs"] * 1e9)
        return (t_tensor, "tensor") if t_tensor >= t_hbm else (t_hbm, "hbm")


def make_cases(rank: int = 0, world: int = 1) -> list[Case]:
    cases = []
    for name in WORKLOAD_NAMES:
        t0 = time.time()
        cases.append(Case(name, inputs.make_workload(name), rank, world))
        log(f"generated {name} in {time.time() - t0:.1f}s")
    return cases


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        # raw samples go to BENCH_CLOCKS_DIR (kept as evidence) or a temporary file
        out_dir = os.environ.get("BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_rank{device_index}_{os.getpid()}.csv")

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- traffic


def profiled_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the library build now loaded (same source digest), else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    from fp8_fine_grained_nt_b200 import build
    if d.get("source_digest") != build.current_digest():
        return None
    ent = d.get("kernels", {}).get(kernel_tag)
    return None if ent is None else ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle


def oracle_sample(cases: list[Case], budget_s: float, seed: int = 0) -> dict:
    """Time the oracle on sampled output elements of every workload, each
    workload's share of elements proportional to its share of the step's FLOP,
    in rounds until about budget_s seconds have been spent."""
    import oracle
    rng = np.random.default_rng(seed)
    total_flops = sum(c.flops for c in cases)
    flops = 0.0
    elems = 0
    batch = 64  # elements of the largest-FLOP workload per pass, grown adaptively
    start = time.time()
    while True:
        t0 = time.time()
        for c in cases:
            n = max(1, int(round(batch * c.flops / total_flops * len(cases))))
            k = _oracle_elems(c, n, rng)
            flops += k * 2.0 * c.prob.K
            elems += k
        dt = time.time() - t0
        spent = time.time() - start
        if spent >= budget_s:
            break
        if dt < 0.5:
            batch *= 2
        elif spent + dt > budget_s * 1.2:
            batch = max(1, int(batch * (budget_s - spent) / dt))
    return {"flops": flops, "seconds": time.time() - start, "elements": elems,
            "cores": oracle.num_threads()}


def _oracle_elems(c: Case, n: int, rng) -> int:
    import oracle
    p = c.prob
    if c.kind == "dense":
        rows, cols = rng.integers(0, p.M, n), rng.integers(0, p.N, n)
        oracle.gemm_dense_sampled(p.a, p.sa, p.b, p.sb, p.M, p.N, p.K, rows, cols)
    elif c.kind == "contiguous":
        valid = np.nonzero(p.m_indices.numpy() >= 0)[0]
        rows, cols = valid[rng.integers(0, len(valid), n)], rng.integers(0, p.N, n)
        oracle.gemm_contiguous_sampled(p.a, p.sa, p.b, p.sb, p.m_indices, p.num_groups, p.M_sum,
                                       p.N, p.K, rows, cols)
    else:
        mm = p.masked_m.numpy()
        act = np.nonzero(mm > 0)[0]
        g = act[rng.integers(0, len(act), n)]
        rows = rng.integers(0, 1 << 30, n) % mm[g]
        cols = rng.integers(0, p.N, n)
        oracle.gemm_masked_sampled(p.a, p.sa, p.b, p.sb, p.masked_m, p.G, p.M_max, p.N, p.K,
                                   g, rows, cols)
    return n


# ---------------------------------------------------------------- main


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device: str = "cuda") -> float:
    """The maximum of `value` over all ranks (value itself when world == 1)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def init_dist(world: int, backend: str):
    if world > 1:
        import datetime
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=300))


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    cases = make_cases()
    budget = args.reference_budget_s
    for _ in range(args.warmup):
        oracle_sample(cases, budget / 10, seed=1)
    flops = 0.0
    secs = 0.0
    cores = 1
    elems = 0
    for s in range(args.steps):
        r = oracle_sample(cases, budget, seed=100 + s)
        flops += r["flops"]
        secs += r["seconds"]
        cores = r["cores"]
        elems += r["elements"]
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{elems} sampled output elements over all seven workloads, "
                                   f"proportional to FLOP, ~{budget:.0f}s per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# small calls timed as a batch in a CUDA graph: name -> number of distinct
# problem sets the graph cycles through
GRAPH_BATCHED = {"dense_decode_64x2112x7168": 16, "dense_128x128x512": 16,
                 "dense_prefill_256x7168x2048": 16}


def measure_graph_batched(fp8, name: str, rank: int, world: int, peaks, iters: int = 10) -> dict:
    """Per-call device time of a short call (decode-sized, or the 256-row
    prefill), measured as a batch: one CUDA graph holds `n` back-to-back
    calls, each on its own seeded problem (distinct operands, as the layers of
    a model have distinct weights; for the decode shape n x 15 MB of B exceeds
    the 126 MB L2, so every call reads its weights from HBM), replayed `iters`
    times between CUDA events.  A single
    call timed between two events on this part carries several microseconds of
    launch and event overhead (an empty kernel reads ~5 us), which dominates a
    call whose roofline time is ~2.4 us; inside a graph only the gap between
    consecutive kernels remains."""
    n = GRAPH_BATCHED[name]
    spec = dict(inputs.WORKLOADS[name])
    sets = []
    for i in range(n):
        prob = inputs.make_dense(spec["M"], spec["N"], spec["K"], seed=1000 + 17 * i + spec["seed"])
        prob = shard_problem(prob, rank, world)
        if problem_is_empty(prob):
            return {"empty_shard": True}
        sets.append((prob.a.cuda(), prob.sa.cuda(), prob.b.cuda(), prob.sb.cuda(),
                     torch.empty(prob.M, prob.N, dtype=torch.bfloat16, device="cuda")))
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for a, sa, b, sb, d in sets:
            fp8.gemm_fp8_fp8_bf16_nt(a, sa, b, sb, d, stream=stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for a, sa, b, sb, d in sets:
            fp8.gemm_fp8_fp8_bf16_nt(a, sa, b, sb, d, stream=stream)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(iters):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        e0.record(cur)
        graph.replay()
        e1.record(cur)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) / n)
    del graph
    ms = statistics.median(times)
    bytes_ = prob.algorithmic_bytes
    t_roof = max(prob.flops / (2.0 * peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9))
    return {"us_per_call": round(ms * 1e3, 3), "calls_per_graph": n,
            "gbs": round(bytes_ / (ms * 1e-3) / 1e9, 1),
            "roofline_frac": round(t_roof / (ms * 1e-3), 4)}


def measure_next_rows(fp8, peaks, iters: int = 20) -> dict:
    """The rows built beyond the fine-grained GEMM, each timed alone (CUDA
    events around every call, L2 flushed before each): the 1x128 activation
    quantiser (also back to back over four inputs larger than the L2), the
    per-tensor-scale GEMM and a skewed (Zipf-like) expert load for the
    contiguous grouped GEMM."""
    dev = "cuda"
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn) -> float:
        for _ in range(3):
            fn()
        total = 0.0
        for _ in range(iters):
            flush.max()  # reads 256 MB: evicts L2 without leaving dirty lines
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            total += e0.elapsed_time(e1)
        return total / iters * 1e-3

    out = {}
    g = torch.Generator(device=dev).manual_seed(99)
    M, K = 4096, 7168
    ld = fp8.get_tma_aligned_size(M, 4)
    q = torch.empty(M, K, dtype=torch.uint8, device=dev)
    sa = torch.empty(K // 128, ld, dtype=torch.float32, device=dev)
    for name, dt, esz in (("fp32", torch.float32, 4), ("bf16", torch.bfloat16, 2)):
        # four distinct inputs (4 x 58 or 117 MB, above the L2) for the
        # back-to-back timing below; the per-call timing uses the first
        xs = [torch.randn(M, K, generator=g, device=dev).to(dt) for _ in range(4)]
        t = timed(lambda: fp8.quantize_fp8_1x128(xs[0], q, sa))
        nbytes = esz * M * K + M * K + 4 * M * (K // 128)
        row = {"us": round(t * 1e6, 2), "gbs": round(nbytes / t / 1e9, 1), "bytes": nbytes,
               "bound": "hbm", "roofline_frac": round(nbytes / t / 1e9 / peaks["hbm_gbs"], 4)}
        # back to back: 20 calls cycling over the four inputs between one pair
        # of events (each call's input was last read three calls earlier and
        # has left the L2), so no per-call event or launch overhead is counted
        for i in range(8):
            fp8.quantize_fp8_1x128(xs[i % 4], q, sa)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(20):
            fp8.quantize_fp8_1x128(xs[i % 4], q, sa)
        e1.record(stream)
        e1.synchronize()
        tb = e0.elapsed_time(e1) * 1e-3 / 20
        row["back_to_back"] = {"us": round(tb * 1e6, 2), "gbs": round(nbytes / tb / 1e9, 1),
                               "roofline_frac": round(nbytes / tb / 1e9 / peaks["hbm_gbs"], 4)}
        out[f"quantize_1x128_{name}_{M}x{K}"] = row
        del xs
    M, N, K = 4096, 7168, 2048
    a = torch.randint(0, 0x7E, (M, K), generator=g, device=dev, dtype=torch.uint8)
    b = torch.randint(0, 0x7E, (N, K), generator=g, device=dev, dtype=torch.uint8)
    sa1 = torch.tensor([0.01], device=dev)
    sb1 = torch.tensor([0.02], device=dev)
    d = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    t = timed(lambda: fp8.gemm_fp8_fp8_bf16_nt_per_tensor(a, sa1, b, sb1, d))
    flop = 2 * M * N * K
    peak = 2.0 * peaks["bf16_tflops"]
    out[f"per_tensor_gemm_{M}x{N}x{K}"] = {
        "us": round(t * 1e6, 2), "tflops": round(flop / t / 1e12, 1), "flop": flop,
        "bound": "tensor", "roofline_frac": round(flop / t / 1e12 / peak, 4)}
    # skewed expert load: counts ~ Zipf(1.2) over 8 experts, 32768 tokens in
    # all, each segment padded to the alignment (the contiguous workload's N, K)
    from fp8_fine_grained_nt_b200 import inputs
    weights = np.array([1.0 / (e + 1) ** 1.2 for e in range(8)])
    counts = [int(round(c)) for c in 32768 * weights / weights.sum()]
    prob = inputs.make_contiguous(8, 4096, 7168, seed=7, counts=counts)
    a, sa_c, b, sb_c = (prob.a.to(dev), prob.sa.to(dev), prob.b.to(dev), prob.sb.to(dev))
    mi = prob.m_indices.to(dev)
    d = torch.empty(prob.M_sum, 4096, dtype=torch.bfloat16, device=dev)
    t = timed(lambda: fp8.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(a, sa_c, b, sb_c, d, mi))
    flop = 2 * sum(counts) * 4096 * 7168
    out["contiguous_zipf_8x4096x7168"] = {
        "us": round(t * 1e6, 2), "tflops": round(flop / t / 1e12, 1), "flop": flop,
        "counts": counts, "bound": "tensor", "roofline_frac": round(flop / t / 1e12 / peak, 4)}
    status = fp8.get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after the extra rows: {fp8.status_string(status)}")
    return out


def run_gpu(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    import fp8_fine_grained_nt_b200 as fp8
    fp8.load_library()
    peaks = measured_peaks()

    cases = make_cases(rank, world)
    for c in cases:
        c.to_device()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # warm-up (also validates the calls)
    for _ in range(args.warmup):
        for c in cases:
            c.call()
    torch.cuda.synchronize()
    status = fp8.get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {fp8.status_string(status)}")

    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in cases] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for s in range(args.steps):
        for i, c in enumerate(cases):
            ev[s][i][0].record(stream)
            c.call()
            ev[s][i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    barrier()
    elapsed_ms = start.elapsed_time(end)
    per_case_ms = [sum(ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(args.steps)) / args.steps
                   for i in range(len(cases))]
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = elapsed_ms / args.steps
    # every rank computed its shard of each workload: together, the whole step
    step_flops = sum(c.whole_flops for c in cases)
    value = step_flops / (ms_per_step * 1e-3) / 1e12

    # e2e: host buffers through the same calls
    for c in cases:
        c.pin_host()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(2):
        for c in cases:
            c.e2e_call(stream)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for c in cases:
            c.e2e_call(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_value = step_flops / (e2e_ms * 1e-3) / 1e12
    h2d = sum(c.h2d_bytes() for c in cases)
    d2h = sum(c.d2h_bytes() for c in cases)
    status = fp8.get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {fp8.status_string(status)}")

    per_shape = {}
    launches_per_step = 0
    for c, ms in zip(cases, per_case_ms):
        if c.empty:
            per_shape[c.name] = {"empty_shard": True}
            continue
        t_roof, bound = c.roofline_time_s(peaks)
        tflops = c.flops / (ms * 1e-3) / 1e12
        cfg = fp8.select_config(
            {"dense": fp8.KIND_DENSE, "contiguous": fp8.KIND_CONTIGUOUS,
             "masked": fp8.KIND_MASKED}[c.kind],
            getattr(c.prob, "M", None) or getattr(c.prob, "M_sum", None) or c.prob.M_max,
            c.prob.N, c.prob.K, getattr(c.prob, "num_groups", getattr(c.prob, "G", 1)),
            getattr(c, "expected_m", 0), 0)
        per_shape[c.name] = {
            "ms": round(ms, 5), "tflops": round(tflops, 2),
            "gbs": round(c.bytes / (ms * 1e-3) / 1e9, 1),
            "bound": bound, "roofline_frac": round(t_roof / (ms * 1e-3), 4),
            "frac_of_nominal_fp8": round(tflops / NOMINAL_FP8_TFLOPS, 4),
            "flop": c.flops, "bytes": c.bytes,
            "tile": f"{cfg['block_m']}x{cfg['block_n']}", "stages": cfg["stages"],
            "split": cfg["split"], "swap_ab": cfg["swap_ab"],
        }
        # a dense call whose last partial wave runs on the small-M kernel
        # is two launches
        if cfg["tail_tiles"]:
            per_shape[c.name]["tail_tiles"] = cfg["tail_tiles"]
        launches_per_step += 2 if cfg["tail_tiles"] else 1
        if c.name in LATENCY_BOUND:
            per_shape[c.name]["note"] = "launch-latency bound: reported, not a roofline target"

    # decode-sized calls: also timed as a batch inside a CUDA graph
    for c in cases:
        if c.name in GRAPH_BATCHED and not c.empty:
            per_shape[c.name]["graph_batched"] = measure_graph_batched(fp8, c.name, rank, world, peaks)

    # dominant kernel: the case with the largest share of step time
    dom_i = int(np.argmax(per_case_ms))
    dom = cases[dom_i]
    t_roof, bound = dom.roofline_time_s(peaks)
    dom_ms = per_case_ms[dom_i]
    if bound == "tensor":
        achieved = dom.flops / (dom_ms * 1e-3) / 1e12
        peak = 2.0 * peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = dom.bytes / (dom_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    traffic = profiled_traffic(dom.name)

    next_rows = measure_next_rows(fp8, peaks) if (rank == 0 and not args.no_next_rows) else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample(cases, args.cpu_budget_s)
        cpu = {"value": r["flops"] / r["seconds"] / 1e12, "unit": UNIT, "cores": r["cores"],
               "kind": "oracle",
               "sample": f"{r['elements']} sampled output elements over all seven workloads, "
                         f"proportional to FLOP ({r['seconds']:.1f}s)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "fp8_e4m3", "data": "synthetic",
            "config": bench_config(world),
            "per_shape": per_shape,
            "roofline": {"kernel": dom.name, "bound": bound, "achieved": round(achieved, 2),
                         "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
                         # the same against the nominal dense FP8 peak (4.5 PFLOP/s)
                         # or the nominal 8 TB/s HBM, for comparison
                         "frac_of_nominal": round(achieved / (NOMINAL_FP8_TFLOPS if bound == "tensor"
                                                              else NOMINAL_HBM_GBS), 4),
                         "traffic": traffic,
                         "peak_source": (f"{peaks['source']}: "
                                         + ("2 x bf16 burst (fp8:bf16 nominal ratio 2)"
                                            if bound == "tensor" else "hbm copy"))},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clock_info,
            "next_rows": next_rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--reference-budget-s", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip timing the quantiser and the per-tensor GEMM")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        return spawn_ranks(args)
    if world_env is not None and int(world_env) != args.gpus:
        log(f"--gpus {args.gpus} does not match WORLD_SIZE={world_env}")
        return 2
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


def spawn_ranks(args) -> int:
    """Run this script as `args.gpus` ranks on this node (torch.distributed.run,
    rendezvous on 127.0.0.1); rank 0 prints the JSON line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.run(cmd).returncode


if __name__ == "__main__":
    sys.exit(main())
