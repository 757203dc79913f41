"""Shared test helpers: device copies of generated problems, CUDA-path calls
through the Python binding (which calls the C ABI), and the parity check."""

from __future__ import annotations

import math

import numpy as np
import torch

from fp8_fine_grained_nt_b200 import inputs

SENTINEL = inputs.sentinel_bf16_bits()


def tolerance_report(gpu: np.ndarray, ref: np.ndarray) -> dict:
    """Per-element bound |gpu - ref| <= 2^-7 |ref| + 1e-3 rms(ref), and the
    global normalised error 1 - 2<x,y> / (|x|^2 + |y|^2) < 1e-5.

    The element bound covers BF16 output rounding (at most 2^-8 relative), the
    single rounding of sa * sb in FP32 and FP32 accumulation over K blocks; the
    absolute term covers outputs near zero where rows cancel.
    """
    gpu = np.asarray(gpu, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert gpu.shape == ref.shape
    if ref.size == 0:
        return {"ok": True, "n": 0}
    rms = math.sqrt(float(np.mean(ref * ref)))
    bound = 2.0 ** -7 * np.abs(ref) + 1e-3 * rms
    diff = np.abs(gpu - ref)
    finite = np.isfinite(gpu)
    elem_ok = bool(finite.all() and (diff <= bound).all())
    denom = float(np.dot(gpu, gpu) + np.dot(ref, ref))
    glob = 0.0 if denom == 0 else 1.0 - 2.0 * float(np.dot(gpu, ref)) / denom
    worst = int(np.argmax(np.where(finite, diff / np.maximum(bound, 1e-300), np.inf)))
    return {"ok": elem_ok and glob < 1e-5, "elem_ok": elem_ok, "global": glob, "n": ref.size,
            "worst_index": worst, "worst_gpu": float(gpu[worst]), "worst_ref": float(ref[worst]),
            "max_ratio": float(np.max(np.where(finite, diff / np.maximum(bound, 1e-300), np.inf)))}


def assert_close(gpu, ref, what=""):
    rep = tolerance_report(gpu, ref)
    assert rep["ok"], f"{what}: parity failed {rep}"
    return rep


def bf16_bits_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)


def sentinel_like(shape, device="cuda") -> torch.Tensor:
    d = torch.full(shape, SENTINEL, dtype=torch.int16, device=device)
    return d.view(torch.bfloat16)


def run_dense(prob: inputs.DenseProblem, d: torch.Tensor | None = None):
    import fp8_fine_grained_nt_b200 as fp8
    a, sa, b, sb = (prob.a.cuda(), prob.sa.cuda(), prob.b.cuda(), prob.sb.cuda())
    if d is None:
        d = sentinel_like((prob.M, prob.N))
    fp8.gemm_fp8_fp8_bf16_nt(a, sa, b, sb, d)
    torch.cuda.synchronize()
    return d


def run_contiguous(prob: inputs.ContiguousProblem, d: torch.Tensor | None = None):
    import fp8_fine_grained_nt_b200 as fp8
    if d is None:
        d = sentinel_like((prob.M_sum, prob.N))
    fp8.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(prob.a.cuda(), prob.sa.cuda(), prob.b.cuda(),
                                                  prob.sb.cuda(), d, prob.m_indices.cuda())
    torch.cuda.synchronize()
    return d


def run_masked(prob: inputs.MaskedProblem, d: torch.Tensor | None = None, expected_m: int = 0):
    import fp8_fine_grained_nt_b200 as fp8
    if d is None:
        d = sentinel_like((prob.G, prob.M_max, prob.N))
    fp8.m_grouped_gemm_fp8_fp8_bf16_nt_masked(prob.a.cuda(), prob.sa.cuda(), prob.b.cuda(),
                                              prob.sb.cuda(), d, prob.masked_m.cuda(), expected_m)
    torch.cuda.synchronize()
    return d


def untouched(d: torch.Tensor) -> np.ndarray:
    """Boolean mask of elements still holding the sentinel bits."""
    return (d.view(torch.int16) == SENTINEL).cpu().numpy()
