"""Build libfp8nt.so in-tree with nvcc for sm_100a (ahead of time, no JIT).

Compiles csrc/api.cu and one object per kernel shape listed in
csrc/kernels.def (csrc/instance.cu with -DFP8NT_MW / -DFP8NT_BN / -DFP8NT_PAIR / -DFP8NT_SCALAR)
and per small-M kernel listed in csrc/skinny.def (csrc/instance_skinny.cu with
-DFP8NT_SKINNY_MN), in parallel, then links them with the static CUDA runtime.  ptxas's resource
report is checked for every kernel: the kernels rebalance registers between
warpgroups with setmaxnreg, which is only safe when each kernel is launched
with exactly the per-thread register count that split assumes, and spills are
reported.

Usage: python -m fp8_fine_grained_nt_b200.build [--force] [-j N]
"""

from __future__ import annotations

import argparse
import hashlib
import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(HERE, "libfp8nt.so")
REGS_AT_LAUNCH = 168

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON_FLAGS = ARCH_FLAGS + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
                             "-Xptxas", "-v", f"-I{os.path.join(ROOT, 'include')}",
                             "--expt-relaxed-constexpr"]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def kernel_list() -> list[tuple[int, int, int, int]]:
    """(MW, BN, PAIR, SCALAR) of every kernel listed in csrc/kernels.def."""
    shapes = []
    with open(os.path.join(CSRC, "kernels.def")) as f:
        for line in f:
            m = re.match(r"\s*FP8NT_KERNEL\(\s*(\d+)\s*,\s*(\d+)\s*,\s*(\d+)\s*,\s*(\d+)\s*\)",
                         line)
            if m:
                shapes.append(tuple(int(m.group(i)) for i in range(1, 5)))
    return shapes


def skinny_list() -> list[int]:
    """MN of every small-M dense kernel listed in csrc/skinny.def."""
    mns = []
    with open(os.path.join(CSRC, "skinny.def")) as f:
        for line in f:
            m = re.match(r"\s*FP8NT_SKINNY\(\s*(\d+)\s*\)", line)
            if m:
                mns.append(int(m.group(1)))
    return mns


def kernel_shapes() -> list[tuple[int, int, int]]:
    """(MW, BN, PAIR) of every fine-grained-scale kernel."""
    return [(mw, bn, pair) for mw, bn, pair, scalar in kernel_list() if not scalar]


def scalar_kernel_shapes() -> list[int]:
    """BN of every per-tensor-scale kernel (MW = 1)."""
    return [bn for mw, bn, pair, scalar in kernel_list() if scalar]


def _sources_digest(extra: list[str]) -> str:
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(ROOT, "include", "fp8_nt.h"), "rb") as f:
        h.update(f.read())
    flags = [f for f in COMMON_FLAGS + extra if not f.startswith("-I")]
    h.update(" ".join(flags).encode())
    return h.hexdigest()


def current_digest() -> str:
    """Digest of the library sources and flags (identifies a build)."""
    return _sources_digest([])


def _compile(src: str, obj: str, defines: list[str]) -> str:
    cmd = [nvcc()] + COMMON_FLAGS + defines + ["-c", src, "-o", obj]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(obj)}:\n{proc.stdout}\n{proc.stderr}")
    return proc.stderr + proc.stdout


def _check_ptxas(report: str, what: str) -> list[str]:
    """Return warnings; raise if a GEMM kernel's launch register count is off."""
    notes = []
    current = None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current and "fp8_gemm_kernel" in current:
            regs = int(m.group(1))
            if regs != REGS_AT_LAUNCH:
                raise RuntimeError(f"{what}: kernel uses {regs} registers at launch, the "
                                   f"setmaxnreg split assumes {REGS_AT_LAUNCH}")
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and current and (int(m.group(1)) or int(m.group(2))):
            notes.append(f"{what}: {line.strip()}")
    return notes


def build(force: bool = False, jobs: int | None = None, verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    digest = _sources_digest([])
    stamp = os.path.join(BUILD_DIR, "libfp8nt.digest")
    if (not force and os.path.exists(LIB_PATH) and os.path.exists(stamp)
            and open(stamp).read() == digest):
        return LIB_PATH
    jobs = jobs or max(1, os.cpu_count() or 1)
    tasks = [(os.path.join(CSRC, "api.cu"), os.path.join(BUILD_DIR, "api.o"), [], "api"),
             (os.path.join(CSRC, "quantize.cu"), os.path.join(BUILD_DIR, "quantize.o"), [],
              "quantize"),
             (os.path.join(CSRC, "selftest.cu"), os.path.join(BUILD_DIR, "selftest.o"), [],
              "selftest")]
    for mw, bn, pair, scalar in kernel_list():
        tag = f"mw{mw}_bn{bn}_p{pair}_s{scalar}"
        tasks.append((os.path.join(CSRC, "instance.cu"), os.path.join(BUILD_DIR, f"kernel_{tag}.o"),
                      [f"-DFP8NT_MW={mw}", f"-DFP8NT_BN={bn}", f"-DFP8NT_PAIR={pair}",
                       f"-DFP8NT_SCALAR={scalar}"], tag))
    for mn in skinny_list():
        tasks.append((os.path.join(CSRC, "instance_skinny.cu"),
                      os.path.join(BUILD_DIR, f"skinny_mn{mn}.o"), [f"-DFP8NT_SKINNY_MN={mn}"],
                      f"skinny_mn{mn}"))
    notes = []
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        futures = [(t, pool.submit(_compile, t[0], t[1], t[2])) for t in tasks]
        for t, fut in futures:
            report = fut.result()
            if verbose:
                print(report)
            notes += _check_ptxas(report, t[3])
    for n in notes:
        print("warning:", n, file=sys.stderr)
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH_FLAGS + ["-shared", "-o", tmp] + [t[1] for t in tasks] + [
        "-cudart", "static"]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError(f"link failed:\n{proc.stdout}\n{proc.stderr}")
    os.replace(tmp, LIB_PATH)
    with open(stamp, "w") as f:
        f.write(digest)
    return LIB_PATH


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("-v", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, jobs=a.j, verbose=a.v))


if __name__ == "__main__":
    main()
