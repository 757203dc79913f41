"""Python binding over the C-ABI library ``libfp8nt.so`` (declared in include/fp8_nt.h).

Argument marshalling only: each call checks dtypes, devices and shapes, passes
raw device pointers, sizes and the current CUDA stream to the library, and
raises ``Fp8NtError`` on a nonzero status.  Every step of the GEMM runs in the
library's kernels.  The library is loaded on first use; if it is missing or
fails to load, the call raises (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

__all__ = [
    "Fp8NtError",
    "library_path",
    "load_library",
    "gemm_fp8_fp8_bf16_nt",
    "gemm_fp8_fp8_bf16_nt_per_tensor",
    "quantize_fp8_1x128",
    "m_grouped_gemm_fp8_fp8_bf16_nt_contiguous",
    "m_grouped_gemm_fp8_fp8_bf16_nt_masked",
    "get_m_alignment_for_contiguous_layout",
    "get_tma_aligned_size",
    "get_col_major_tma_aligned_tensor",
    "set_num_sms",
    "get_num_sms",
    "get_device_status",
    "selftest_wait_timeout",
    "select_config",
    "force_config",
    "force_swap_ab",
    "force_tail_split",
    "status_string",
    "KIND_DENSE",
    "KIND_CONTIGUOUS",
    "KIND_MASKED",
    "KIND_DENSE_PER_TENSOR",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libfp8nt.so"
_lock = threading.Lock()
_lib = None

KIND_DENSE, KIND_CONTIGUOUS, KIND_MASKED, KIND_DENSE_PER_TENSOR = 0, 1, 2, 3


class Fp8NtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class DgConfig(ctypes.Structure):
    _fields_ = [("block_m", ctypes.c_int), ("block_n", ctypes.c_int),
                ("stages", ctypes.c_int),
                ("num_tiles", ctypes.c_int), ("grid", ctypes.c_int),
                ("smem_bytes", ctypes.c_int), ("tmem_cols", ctypes.c_int),
                ("split", ctypes.c_int), ("cta_pair", ctypes.c_int),
                ("swap_ab", ctypes.c_int), ("tail_tiles", ctypes.c_int)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load_library():
    """Load libfp8nt.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with "
                              "`python -m fp8_fine_grained_nt_b200.build`")
        lib = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.gemm_fp8_fp8_bf16_nt.argtypes = [P, P, P, P, P, I, I, I, P]
        lib.gemm_fp8_fp8_bf16_nt_per_tensor.argtypes = [P, P, P, P, P, I, I, I, P]
        lib.quantize_fp8_1x128.argtypes = [P, I, P, P, I, I, P]
        lib.dg_selftest_wait_timeout.argtypes = [I, P]
        lib.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
        lib.m_grouped_gemm_fp8_fp8_bf16_nt_masked.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
        lib.get_m_alignment_for_contiguous_layout.argtypes = []
        lib.get_tma_aligned_size.argtypes = [I, I]
        lib.set_num_sms.argtypes = [I]
        lib.get_num_sms.argtypes = []
        lib.dg_status_string.argtypes = [I]
        lib.dg_status_string.restype = ctypes.c_char_p
        lib.dg_get_device_status.argtypes = [P]
        lib.dg_select_config.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(DgConfig)]
        lib.dg_force_config.argtypes = [I, I, I, I]
        lib.dg_force_swap_ab.argtypes = [I]
        lib.dg_force_tail_split.argtypes = [I]
        _lib = lib
        return lib


def status_string(status: int) -> str:
    try:
        return load_library().dg_status_string(status).decode()
    except ImportError:
        return "unknown"


def _check(status: int, where: str):
    if status != 0:
        raise Fp8NtError(status, where)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str, dtypes, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


_FP8 = (torch.float8_e4m3fn, torch.uint8)
_F32 = (torch.float32,)


def gemm_fp8_fp8_bf16_nt(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor,
                         sb: torch.Tensor, d: torch.Tensor, stream=None) -> torch.Tensor:
    """D[M,N] (bf16) = sum_kb (A_kb B_kb^T) sa[m,kb] sb[n/128,kb].

    a: [M,K] E4M3 (or its uint8 bytes); sa: [ceil(K/128), tma_aligned(M)] fp32
    column-major LHS scales; b: [N,K] E4M3; sb: [ceil(N/128), ceil(K/128)] fp32;
    d: [M,N] bf16 output.
    """
    M, K = a.shape
    N = b.shape[0]
    args = (_dev(a, "a", _FP8, 2), _dev(sa, "sa", _F32, 2), _dev(b, "b", _FP8, 2),
            _dev(sb, "sb", _F32, 2), _dev(d, "d", (torch.bfloat16,), 2))
    if tuple(d.shape) != (M, N) or b.shape[1] != K:
        raise ValueError("shape mismatch between a, b and d")
    _check(load_library().gemm_fp8_fp8_bf16_nt(*args, M, N, K, _stream_ptr(stream)),
           "gemm_fp8_fp8_bf16_nt")
    return d


def gemm_fp8_fp8_bf16_nt_per_tensor(a: torch.Tensor, scale_a: torch.Tensor, b: torch.Tensor,
                                    scale_b: torch.Tensor, d: torch.Tensor,
                                    stream=None) -> torch.Tensor:
    """D[M,N] (bf16) = scale_a * scale_b * (A B^T), FP32 accumulation over all of K.

    a: [M,K] E4M3; b: [N,K] E4M3; scale_a, scale_b: one-element fp32 device
    tensors; d: [M,N] bf16 output.
    """
    M, K = a.shape
    N = b.shape[0]
    if scale_a.numel() != 1 or scale_b.numel() != 1:
        raise ValueError("scale_a and scale_b hold one value each")
    args = (_dev(a, "a", _FP8, 2), _dev(scale_a.reshape(1), "scale_a", _F32, 1),
            _dev(b, "b", _FP8, 2), _dev(scale_b.reshape(1), "scale_b", _F32, 1),
            _dev(d, "d", (torch.bfloat16,), 2))
    if tuple(d.shape) != (M, N) or b.shape[1] != K:
        raise ValueError("shape mismatch between a, b and d")
    _check(load_library().gemm_fp8_fp8_bf16_nt_per_tensor(*args, M, N, K, _stream_ptr(stream)),
           "gemm_fp8_fp8_bf16_nt_per_tensor")
    return d


def quantize_fp8_1x128(x: torch.Tensor, q: torch.Tensor, sa: torch.Tensor,
                       stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """1x128 quantiser: x [M,K] fp32 or bf16 -> q [M,K] E4M3 (uint8 or
    float8_e4m3fn) and sa [K/128, get_tma_aligned_size(M, 4)] fp32 column-major."""
    M, K = x.shape
    dtype = {torch.float32: 0, torch.bfloat16: 1}.get(x.dtype)
    if dtype is None:
        raise TypeError(f"x has dtype {x.dtype}, expected float32 or bfloat16")
    args = (_dev(x, "x", (torch.float32, torch.bfloat16), 2), dtype, _dev(q, "q", _FP8, 2),
            _dev(sa, "sa", _F32, 2))
    if tuple(q.shape) != (M, K) or sa.shape[0] != K // 128 or sa.shape[1] != get_tma_aligned_size(M, 4):
        raise ValueError("shape mismatch between x, q and sa")
    _check(load_library().quantize_fp8_1x128(*args, M, K, _stream_ptr(stream)),
           "quantize_fp8_1x128")
    return q, sa


def m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(a, sa, b, sb, d, m_indices, stream=None):
    """Contiguous m-grouped GEMM: row m of A uses expert m_indices[m] (-1 = padding).

    a: [M_sum,K]; sa: [ceil(K/128), M_sum] (M_sum is a multiple of the alignment);
    b: [G,N,K]; sb: [G, ceil(N/128), ceil(K/128)]; d: [M_sum,N] bf16;
    m_indices: [M_sum] int32 on the device.
    """
    M_sum, K = a.shape
    G, N = b.shape[0], b.shape[1]
    args = (_dev(a, "a", _FP8, 2), _dev(sa, "sa", _F32, 2), _dev(b, "b", _FP8, 3),
            _dev(sb, "sb", _F32, 3), _dev(d, "d", (torch.bfloat16,), 2),
            _dev(m_indices, "m_indices", (torch.int32,), 1))
    if tuple(d.shape) != (M_sum, N) or b.shape[2] != K or m_indices.shape[0] != M_sum:
        raise ValueError("shape mismatch between a, b, d and m_indices")
    _check(load_library().m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(
        *args, G, M_sum, N, K, _stream_ptr(stream)), "m_grouped_gemm_fp8_fp8_bf16_nt_contiguous")
    return d


def m_grouped_gemm_fp8_fp8_bf16_nt_masked(a, sa, b, sb, d, masked_m, expected_m: int,
                                          stream=None):
    """Masked m-grouped GEMM: group g computes its first masked_m[g] rows only.

    a: [G,M_max,K]; sa: [G, ceil(K/128), tma_aligned(M_max)]; b: [G,N,K];
    sb: [G, ceil(N/128), ceil(K/128)]; d: [G,M_max,N] bf16; masked_m: [G] int32
    on the device (never read by the host); expected_m: a host hint for the
    typical masked_m, used only to choose the tile configuration.
    """
    G, M_max, K = a.shape
    N = b.shape[1]
    args = (_dev(a, "a", _FP8, 3), _dev(sa, "sa", _F32, 3), _dev(b, "b", _FP8, 3),
            _dev(sb, "sb", _F32, 3), _dev(d, "d", (torch.bfloat16,), 3),
            _dev(masked_m, "masked_m", (torch.int32,), 1))
    if tuple(d.shape) != (G, M_max, N) or tuple(b.shape) != (G, N, K) or masked_m.shape[0] != G:
        raise ValueError("shape mismatch between a, b, d and masked_m")
    _check(load_library().m_grouped_gemm_fp8_fp8_bf16_nt_masked(
        *args, G, M_max, N, K, int(expected_m), _stream_ptr(stream)),
        "m_grouped_gemm_fp8_fp8_bf16_nt_masked")
    return d


def get_m_alignment_for_contiguous_layout() -> int:
    return load_library().get_m_alignment_for_contiguous_layout()


def get_tma_aligned_size(x: int, element_size: int) -> int:
    r = load_library().get_tma_aligned_size(int(x), int(element_size))
    if r < 0:
        raise Fp8NtError(-r, "get_tma_aligned_size")
    return r


def get_col_major_tma_aligned_tensor(s: torch.Tensor) -> torch.Tensor:
    """[..., M, nkb] per-row scales -> column-major TMA-aligned [..., nkb, ld] storage.

    A layout helper (torch copy ops, not on the GEMM path): the padding columns
    between M and ld are left as zeros.
    """
    *batch, M, nkb = s.shape
    ld = get_tma_aligned_size(M, 4)
    out = torch.zeros((*batch, nkb, ld), dtype=torch.float32, device=s.device)
    out[..., :M] = s.transpose(-1, -2).float()
    return out


def set_num_sms(n: int) -> None:
    _check(load_library().set_num_sms(int(n)), "set_num_sms")


def get_num_sms() -> int:
    return load_library().get_num_sms()


def selftest_wait_timeout(timeout_us: int = 20000, stream=None) -> None:
    """Enqueue the bounded-wait self-test: a device wait that nothing satisfies
    gives up after timeout_us and records DG_ERR_DEVICE_TIMEOUT (read it with
    get_device_status())."""
    _check(load_library().dg_selftest_wait_timeout(int(timeout_us), _stream_ptr(stream)),
           "dg_selftest_wait_timeout")


def get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side status word."""
    return load_library().dg_get_device_status(_stream_ptr(stream))


def select_config(kind: int, M: int, N: int, K: int, num_groups: int = 1,
                  expected_m: int = 0, num_sms: int = 148) -> dict:
    """The tile configuration the library would launch (host logic only, no GPU)."""
    cfg = DgConfig()
    _check(load_library().dg_select_config(kind, M, N, K, num_groups, expected_m, num_sms,
                                           ctypes.byref(cfg)), "dg_select_config")
    return cfg.as_dict()


def force_config(block_m: int = 0, block_n: int = 0, split: int = 0, cta_pair: int = 0) -> None:
    """Pin the tile shape (0, 0 = automatic), split-K factor (0 = automatic)
    and CTA-pair mode (0 = automatic, 1 = one CTA per tile, 2 = CTA pairs)
    for later calls.  For tests."""
    _check(load_library().dg_force_config(int(block_m), int(block_n), int(split),
                                          int(cta_pair)), "dg_force_config")


def force_swap_ab(mode: int = 0) -> None:
    """Small-M kernel choice for later dense calls: 0 = automatic (M <= 256
    uses it), 1 = never, 2 = wherever it applies.  For tests."""
    _check(load_library().dg_force_swap_ab(int(mode)), "dg_force_swap_ab")


def force_tail_split(mode: int = 0) -> None:
    """Split of a dense call's last partial wave onto the small-M kernel:
    0 = automatic (off), 1 = never, 2 = wherever the block layout allows it,
    3 = where the layout allows it and the cycle estimate favours it."""
    _check(load_library().dg_force_tail_split(int(mode)), "dg_force_tail_split")
