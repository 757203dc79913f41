"""Seeded synthetic inputs for the FP8 (E4M3) NT GEMM with fine-grained scaling.

This module prepares operands; it holds none of the GEMM's arithmetic.  Both
the CUDA path (through the tests and the benchmark) and the CPU oracle consume
the bytes and scales produced here, so neither side can influence the other's
inputs.

Recipe (stated once, used everywhere):

* Values are drawn N(0, 1) in FP32 from a ``torch.Generator`` seeded per
  workload.  Draw order is fixed: group sizes first (grouped forms), then A,
  then B.
* Quantisation follows the fine-grained scaling that DeepSeek-V3 proposed and
  that the DeepGEMM README (introduction) names: one FP32 scale per row per
  128-wide K block for the LHS ("1x128") and one per 128x128 block for the
  RHS.  A scale is a dequantisation multiplier, x ~ dec(q) * s with
  s = max(amax, 1e-4) / 448; 448 is the E4M3 maximum (hnwysp.cn DeepGEMM
  blog, section 4.1).  x / s is clamped to [-448, 448] and rounded to
  nearest-even E4M3 by torch's ``float8_e4m3fn`` cast (which does not
  saturate on its own: 500 becomes NaN).
* LHS scales are stored column-major and TMA-aligned, [ceil(K/128)][ld] with
  ld = ``tma_aligned_size(M, 4)`` (DeepGEMM README, "utility functions":
  ``get_tma_aligned_size`` / ``get_col_major_tma_aligned_tensor``).  The
  padding columns between M and ld are filled with NaN so that a kernel that
  lets them reach a stored output is caught.
* RHS scales are row-major [ceil(N/128)][ceil(K/128)] (per group for the
  grouped forms).  A partial last block (N or K not a multiple of 128) takes
  its amax over the rows it has.
* Contiguous layout (DeepGEMM README, "contiguous" grouped GEMM): per-expert
  token counts are drawn uniformly in [lo, hi], each segment is padded up to
  the 128-row M-block alignment, padding rows hold random data, and
  ``m_indices`` holds the expert of each row or -1 on padding rows.
* Masked layout (DeepGEMM README, "masked" grouped GEMM): A is [G, Mmax, K],
  ``masked_m[g]`` is drawn uniformly in [0, Mmax].
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

E4M3_MAX = 448.0
BLOCK_K = 128
BLOCK_N_SCALE = 128
AMAX_FLOOR = 1e-4
M_ALIGNMENT_CONTIGUOUS = 128


def ceil_div(a: int, b: int) -> int:
    return (a + b - 1) // b


def tma_aligned_size(x: int, element_size: int) -> int:
    """Smallest count >= x whose byte size is a multiple of 16."""
    align = 16 // element_size
    return ceil_div(x, align) * align


def _to_e4m3_bytes(scaled: torch.Tensor) -> torch.Tensor:
    clamped = scaled.clamp(-E4M3_MAX, E4M3_MAX)
    return clamped.to(torch.float8_e4m3fn).view(torch.uint8)


def quantize_lhs(x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-row, per-128-K-block quantisation of an FP32 [M, K] tensor.

    Returns (q uint8 [M, K], s float32 [M, ceil(K/128)]) with x ~ dec(q) * s.
    """
    M, K = x.shape
    nkb = ceil_div(K, BLOCK_K)
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M, nkb), dtype=torch.float32, device=x.device)
    for kb in range(nkb):
        blk = x[:, kb * BLOCK_K:(kb + 1) * BLOCK_K]
        amax = blk.abs().amax(dim=1).clamp_min(AMAX_FLOOR)
        scale = amax / E4M3_MAX
        q[:, kb * BLOCK_K:(kb + 1) * BLOCK_K] = _to_e4m3_bytes(blk / scale[:, None])
        s[:, kb] = scale
    return q, s


def quantize_rhs(x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-128x128-block quantisation of an FP32 [N, K] tensor.

    Returns (q uint8 [N, K], s float32 [ceil(N/128), ceil(K/128)]).
    """
    N, K = x.shape
    nnb, nkb = ceil_div(N, BLOCK_N_SCALE), ceil_div(K, BLOCK_K)
    q = torch.empty((N, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((nnb, nkb), dtype=torch.float32, device=x.device)
    for nb in range(nnb):
        rows = slice(nb * BLOCK_N_SCALE, (nb + 1) * BLOCK_N_SCALE)
        for kb in range(nkb):
            cols = slice(kb * BLOCK_K, (kb + 1) * BLOCK_K)
            blk = x[rows, cols]
            scale = blk.abs().amax().clamp_min(AMAX_FLOOR) / E4M3_MAX
            q[rows, cols] = _to_e4m3_bytes(blk / scale)
            s[nb, kb] = scale
    return q, s


def col_major_tma_aligned(s: torch.Tensor, pad_value: float = float("nan")) -> torch.Tensor:
    """[M, nkb] row-per-token scales -> column-major [nkb, ld] storage."""
    M, nkb = s.shape
    ld = tma_aligned_size(M, 4)
    out = torch.full((nkb, ld), pad_value, dtype=torch.float32, device=s.device)
    out[:, :M] = s.t()
    return out


# ----------------------------------------------------------------------------
# Problems


@dataclasses.dataclass
class DenseProblem:
    M: int
    N: int
    K: int
    a: torch.Tensor        # uint8 [M, K]
    sa: torch.Tensor       # float32 [nkb, ld(M)]  (column-major LHS scales)
    b: torch.Tensor        # uint8 [N, K]
    sb: torch.Tensor       # float32 [nnb, nkb]
    seed: int = 0

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def algorithmic_bytes(self) -> int:
        nkb, nnb = ceil_div(self.K, 128), ceil_div(self.N, 128)
        return (self.M * self.K + self.N * self.K + 4 * self.M * nkb
                + 4 * nnb * nkb + 2 * self.M * self.N)


@dataclasses.dataclass
class ContiguousProblem:
    num_groups: int
    M_sum: int
    N: int
    K: int
    a: torch.Tensor          # uint8 [M_sum, K]
    sa: torch.Tensor         # float32 [nkb, ld(M_sum)]
    b: torch.Tensor          # uint8 [G, N, K]
    sb: torch.Tensor         # float32 [G, nnb, nkb]
    m_indices: torch.Tensor  # int32 [M_sum], -1 on padding rows
    counts: list             # valid rows per expert
    seed: int = 0

    @property
    def valid_rows(self) -> int:
        return int(sum(self.counts))

    @property
    def flops(self) -> int:
        return 2 * self.valid_rows * self.N * self.K

    @property
    def algorithmic_bytes(self) -> int:
        nkb, nnb = ceil_div(self.K, 128), ceil_div(self.N, 128)
        active = sum(1 for c in self.counts if c > 0)
        m = self.valid_rows
        return (m * self.K + active * self.N * self.K + 4 * m * nkb
                + 4 * active * nnb * nkb + 2 * m * self.N)


@dataclasses.dataclass
class MaskedProblem:
    G: int
    M_max: int
    N: int
    K: int
    a: torch.Tensor         # uint8 [G, M_max, K]
    sa: torch.Tensor        # float32 [G, nkb, ld(M_max)]
    b: torch.Tensor         # uint8 [G, N, K]
    sb: torch.Tensor        # float32 [G, nnb, nkb]
    masked_m: torch.Tensor  # int32 [G]
    seed: int = 0

    @property
    def valid_rows(self) -> int:
        return int(self.masked_m.sum())

    @property
    def flops(self) -> int:
        return 2 * self.valid_rows * self.N * self.K

    @property
    def algorithmic_bytes(self) -> int:
        nkb, nnb = ceil_div(self.K, 128), ceil_div(self.N, 128)
        active = int((self.masked_m > 0).sum())
        m = self.valid_rows
        return (m * self.K + active * self.N * self.K + 4 * m * nkb
                + 4 * active * nnb * nkb + 2 * m * self.N)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(shape, gen) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def make_dense(M: int, N: int, K: int, seed: int = 0) -> DenseProblem:
    gen = _gen(seed)
    x = _randn((M, K), gen)
    w = _randn((N, K), gen)
    a, sa = quantize_lhs(x)
    b, sb = quantize_rhs(w)
    return DenseProblem(M, N, K, a, col_major_tma_aligned(sa), b, sb, seed)


def make_contiguous(num_groups: int, N: int, K: int, seed: int = 0,
                    count_range: tuple[int, int] = (1, 8192),
                    counts: Optional[Sequence[int]] = None) -> ContiguousProblem:
    gen = _gen(seed)
    lo, hi = count_range
    drawn = torch.randint(lo, hi + 1, (num_groups,), generator=gen).tolist()
    if counts is None:
        counts = drawn
    counts = [int(c) for c in counts]
    padded = [ceil_div(c, M_ALIGNMENT_CONTIGUOUS) * M_ALIGNMENT_CONTIGUOUS for c in counts]
    M_sum = sum(padded)
    x = _randn((M_sum, K), gen)
    a, sa = quantize_lhs(x)
    del x
    b = torch.empty((num_groups, N, K), dtype=torch.uint8)
    nnb, nkb = ceil_div(N, 128), ceil_div(K, 128)
    sb = torch.empty((num_groups, nnb, nkb), dtype=torch.float32)
    for g in range(num_groups):
        w = _randn((N, K), gen)
        b[g], sb[g] = quantize_rhs(w)
    m_indices = torch.full((M_sum,), -1, dtype=torch.int32)
    row = 0
    for g, (c, p) in enumerate(zip(counts, padded)):
        m_indices[row:row + c] = g
        row += p
    return ContiguousProblem(num_groups, M_sum, N, K, a, col_major_tma_aligned(sa), b, sb,
                             m_indices, counts, seed)


def make_masked(G: int, M_max: int, N: int, K: int, seed: int = 0,
                masked_m: Optional[Sequence[int]] = None) -> MaskedProblem:
    gen = _gen(seed)
    drawn = torch.randint(0, M_max + 1, (G,), generator=gen, dtype=torch.int64)
    mm = drawn if masked_m is None else torch.tensor(list(masked_m), dtype=torch.int64)
    nkb, nnb = ceil_div(K, 128), ceil_div(N, 128)
    ld = tma_aligned_size(M_max, 4)
    a = torch.empty((G, M_max, K), dtype=torch.uint8)
    sa = torch.empty((G, nkb, ld), dtype=torch.float32)
    for g in range(G):
        x = _randn((M_max, K), gen)
        q, s = quantize_lhs(x)
        a[g] = q
        sa[g] = col_major_tma_aligned(s)
    b = torch.empty((G, N, K), dtype=torch.uint8)
    sb = torch.empty((G, nnb, nkb), dtype=torch.float32)
    for g in range(G):
        w = _randn((N, K), gen)
        b[g], sb[g] = quantize_rhs(w)
    return MaskedProblem(G, M_max, N, K, a, sa, b, sb, mm.to(torch.int32), seed)


# ----------------------------------------------------------------------------
# The workloads measured: seeds are fixed per workload.

WORKLOADS = {
    "dense_128x128x512": dict(kind="dense", M=128, N=128, K=512, seed=0),
    "dense_decode_64x2112x7168": dict(kind="dense", M=64, N=2112, K=7168, seed=1),
    "dense_prefill_4096x7168x2048": dict(kind="dense", M=4096, N=7168, K=2048, seed=2),
    "dense_prefill_256x7168x2048": dict(kind="dense", M=256, N=7168, K=2048, seed=3),
    "contiguous_8x4096x7168": dict(kind="contiguous", G=8, N=4096, K=7168, seed=4),
    "masked_16x256_4096x7168": dict(kind="masked", G=16, M_max=256, N=4096, K=7168, seed=5),
    "masked_16x256_7168x2048": dict(kind="masked", G=16, M_max=256, N=7168, K=2048, seed=6),
}


def make_workload(name: str):
    spec = dict(WORKLOADS[name])
    kind = spec.pop("kind")
    if kind == "dense":
        return make_dense(spec["M"], spec["N"], spec["K"], spec["seed"])
    if kind == "contiguous":
        return make_contiguous(spec["G"], spec["N"], spec["K"], spec["seed"])
    return make_masked(spec["G"], spec["M_max"], spec["N"], spec["K"], spec["seed"])


def sentinel_bf16_bits() -> int:
    """Bit pattern prefilled into outputs to detect stray writes (a NaN)."""
    return 0x7FC1


def as_numpy_u8(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().numpy().view(np.uint8)
