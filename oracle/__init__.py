"""CPU oracle for the FP8 (E4M3) NT GEMM with fine-grained scaling.

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers.  The oracle is plain C
(``oracle.c``, FP64, OpenMP over output rows); this module compiles it with
gcc on first use and wraps it with ctypes.  It imports nothing from the CUDA
library and the CUDA library imports nothing from it.

Every function takes the operand bytes and scales exactly as the library's
C-ABI does (A/B as uint8 E4M3 bytes, LHS scales column-major with a leading
dimension, RHS scales per 128x128 block) and returns FP64 results; elements
that the definition does not produce (contiguous padding rows, masked-out
rows) are NaN.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP; no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OracleLib:
    """ctypes handle on one compiled copy of the oracle (normally liboracle.so)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_long
        lib.oracle_e4m3_table.argtypes = [P]
        lib.oracle_e4m3_table.restype = None
        sigs = {
            "oracle_gemm_dense": [P, P, L, P, P, I, I, I, P],
            "oracle_gemm_dense_sampled": [P, P, L, P, P, I, I, I, P, P, L, P],
            "oracle_gemm_contiguous": [P, P, L, P, P, P, I, I, I, I, P],
            "oracle_gemm_contiguous_sampled": [P, P, L, P, P, P, I, I, I, I, P, P, L, P],
            "oracle_gemm_masked": [P, P, L, P, P, P, I, I, I, I, P],
            "oracle_gemm_masked_sampled": [P, P, L, P, P, P, I, I, I, I, P, P, P, L, P],
            "oracle_quantize_1x128": [P, I, I, P, P, L],
        }
        for name, argtypes in sigs.items():
            fn = getattr(lib, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def e4m3_table(self) -> np.ndarray:
        out = np.empty(256, dtype=np.float64)
        self.lib.oracle_e4m3_table(_ptr(out))
        return out

    def gemm_dense(self, a, sa, b, sb, M: int, N: int, K: int) -> np.ndarray:
        """D[M, N] in FP64.  a: [M,K] bytes, sa: [nkb, ld] column-major, b: [N,K],
        sb: [nnb, nkb]."""
        a, b = _np(a, np.uint8), _np(b, np.uint8)
        sa, sb = _np(sa, np.float32), _np(sb, np.float32)
        out = np.empty((M, N), dtype=np.float64)
        _check(self.lib.oracle_gemm_dense(_ptr(a), _ptr(sa), sa.shape[-1], _ptr(b), _ptr(sb),
                                          M, N, K, _ptr(out)), "gemm_dense")
        return out

    def gemm_dense_sampled(self, a, sa, b, sb, M, N, K, rows, cols) -> np.ndarray:
        a, b = _np(a, np.uint8), _np(b, np.uint8)
        sa, sb = _np(sa, np.float32), _np(sb, np.float32)
        rows, cols = _np(rows, np.int32), _np(cols, np.int32)
        out = np.empty(rows.shape[0], dtype=np.float64)
        _check(self.lib.oracle_gemm_dense_sampled(
            _ptr(a), _ptr(sa), sa.shape[-1], _ptr(b), _ptr(sb), M, N, K, _ptr(rows),
            _ptr(cols), rows.shape[0], _ptr(out)), "gemm_dense_sampled")
        return out

    def gemm_contiguous(self, a, sa, b, sb, m_indices, num_groups, M_sum, N, K) -> np.ndarray:
        a, b = _np(a, np.uint8), _np(b, np.uint8)
        sa, sb = _np(sa, np.float32), _np(sb, np.float32)
        mi = _np(m_indices, np.int32)
        out = np.empty((M_sum, N), dtype=np.float64)
        _check(self.lib.oracle_gemm_contiguous(
            _ptr(a), _ptr(sa), sa.shape[-1], _ptr(b), _ptr(sb), _ptr(mi), num_groups, M_sum,
            N, K, _ptr(out)), "gemm_contiguous")
        return out

    def gemm_contiguous_sampled(self, a, sa, b, sb, m_indices, num_groups, M_sum, N, K,
                                rows, cols) -> np.ndarray:
        a, b = _np(a, np.uint8), _np(b, np.uint8)
        sa, sb = _np(sa, np.float32), _np(sb, np.float32)
        mi = _np(m_indices, np.int32)
        rows, cols = _np(rows, np.int32), _np(cols, np.int32)
        out = np.empty(rows.shape[0], dtype=np.float64)
        _check(self.lib.oracle_gemm_contiguous_sampled(
            _ptr(a), _ptr(sa), sa.shape[-1], _ptr(b), _ptr(sb), _ptr(mi), num_groups, M_sum,
            N, K, _ptr(rows), _ptr(cols), rows.shape[0], _ptr(out)), "gemm_contiguous_sampled")
        return out

    def gemm_masked(self, a, sa, b, sb, masked_m, G, M_max, N, K) -> np.ndarray:
        a, b = _np(a, np.uint8), _np(b, np.uint8)
        sa, sb = _np(sa, np.float32), _np(sb, np.float32)
        mm = _np(masked_m, np.int32)
        out = np.empty((G, M_max, N), dtype=np.float64)
        _check(self.lib.oracle_gemm_masked(
            _ptr(a), _ptr(sa), sa.shape[-1], _ptr(b), _ptr(sb), _ptr(mm), G, M_max, N, K,
            _ptr(out)), "gemm_masked")
        return out

    def quantize_1x128(self, x, M: int, K: int, ld_sa: int | None = None):
        """(q uint8 [M, K], sa float32 [K/128, ld_sa]) of an FP32 [M, K] input
        (BF16 inputs: pass their exact FP32 values).  Columns M..ld_sa-1 of sa
        are left NaN (not part of the definition)."""
        x = _np(x, np.float32)
        ld = ld_sa if ld_sa is not None else (M + 3) // 4 * 4
        q = np.empty((M, K), dtype=np.uint8)
        sa = np.full((K // 128, ld), np.nan, dtype=np.float32)
        _check(self.lib.oracle_quantize_1x128(_ptr(x), M, K, _ptr(q), _ptr(sa), ld),
               "quantize_1x128")
        return q, sa

    def gemm_masked_sampled(self, a, sa, b, sb, masked_m, G, M_max, N, K, groups, rows,
                            cols) -> np.ndarray:
        a, b = _np(a, np.uint8), _np(b, np.uint8)
        sa, sb = _np(sa, np.float32), _np(sb, np.float32)
        mm = _np(masked_m, np.int32)
        groups, rows, cols = (_np(groups, np.int32), _np(rows, np.int32),
                              _np(cols, np.int32))
        out = np.empty(rows.shape[0], dtype=np.float64)
        _check(self.lib.oracle_gemm_masked_sampled(
            _ptr(a), _ptr(sa), sa.shape[-1], _ptr(b), _ptr(sb), _ptr(mm), G, M_max, N, K,
            _ptr(groups), _ptr(rows), _ptr(cols), rows.shape[0], _ptr(out)),
            "gemm_masked_sampled")
        return out


def _np(x, dtype) -> np.ndarray:
    """Contiguous numpy array from a numpy array or a CPU torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().contiguous().numpy()
    arr = np.ascontiguousarray(x)
    if dtype is np.uint8 and arr.dtype != np.uint8:
        arr = arr.view(np.uint8)
    return arr if arr.dtype == dtype else arr.astype(dtype)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: bad arguments (code {rc})")


def default() -> OracleLib:
    """The oracle built from oracle.c (compiled on first use)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = OracleLib(build())
    return _lib


def e4m3_table():
    return default().e4m3_table()


def gemm_dense(*args, **kw):
    return default().gemm_dense(*args, **kw)


def gemm_dense_sampled(*args, **kw):
    return default().gemm_dense_sampled(*args, **kw)


def gemm_contiguous(*args, **kw):
    return default().gemm_contiguous(*args, **kw)


def gemm_contiguous_sampled(*args, **kw):
    return default().gemm_contiguous_sampled(*args, **kw)


def gemm_masked(*args, **kw):
    return default().gemm_masked(*args, **kw)


def gemm_masked_sampled(*args, **kw):
    return default().gemm_masked_sampled(*args, **kw)


def quantize_1x128(*args, **kw):
    return default().quantize_1x128(*args, **kw)


def gemm_per_tensor(a, scale_a: float, b, scale_b: float, M: int, N: int, K: int,
                    lib: OracleLib | None = None) -> np.ndarray:
    """Per-tensor scaling (one FP32 scale per operand; the tensor-wise recipe
    of the FP8-training blog page, section 4.2): the fine-grained definition
    with every LHS and RHS block scale equal, i.e.
    D = scale_a * scale_b * sum_k dec(A[m,k]) dec(B[n,k])."""
    nkb = K // 128
    sa = np.full((nkb, M), np.float32(scale_a), dtype=np.float32)
    sb = np.full(((N + 127) // 128, nkb), np.float32(scale_b), dtype=np.float32)
    return (lib or default()).gemm_dense(a, sa, b, sb, M, N, K)


def num_threads() -> int:
    """Threads OpenMP will use for the oracle (OMP_NUM_THREADS, else all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    return os.cpu_count() or 1
