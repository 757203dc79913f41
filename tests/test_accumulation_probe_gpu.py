"""Probe of the tensor core's FP8 accumulation width on B200.

The DeepGEMM pages give imprecise FP8 tensor-core accumulation as the reason
for promoting partial sums on CUDA cores (README, introduction; launch report,
on two-level accumulation).  The kernels here promote every 128-K block, so
what matters is whether one block's partial (four tcgen05.mma of K = 32 into
TMEM) is the exact sum when that sum fits FP32.

Input: two K blocks with unit RHS scales and LHS scales +1 and -1.  Block 0
holds eight products 32 * 32 = 2^10 and one product 2^-5 * 2^-5 = 2^-10;
block 1 the same eight large products without the small one.  The exact
block-0 partial 8192 + 2^-10 needs 24 significant bits: representable in
FP32, lost by any narrower accumulator.  With exact FP32 partials the result
is D = 2^-10 in every element (exact in BF16); a narrower accumulation gives
0.  The oracle (exact FP64 sums) is the checker.  The small product is placed
in the same K = 32 MMA as the large ones (the tensor core's internal sum) or
in another one (the sum across MMAs in TMEM).
"""

import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_nt_b200 as fp8
from fp8_fine_grained_nt_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu

K = 256


def e4m3(v: float) -> int:
    return int(torch.tensor([v]).to(torch.float8_e4m3fn).view(torch.uint8).item())


def probe_problem(M: int, N: int, small_pos: int, large_pos: list[int]) -> inputs.DenseProblem:
    a = torch.zeros(M, K, dtype=torch.uint8)
    b = torch.zeros(N, K, dtype=torch.uint8)
    for blk in (0, 1):
        for p in large_pos:
            a[:, blk * 128 + p] = e4m3(32.0)
            b[:, blk * 128 + p] = e4m3(32.0)
    a[:, small_pos] = e4m3(2.0 ** -5)
    b[:, small_pos] = e4m3(2.0 ** -5)
    ld = inputs.tma_aligned_size(M, 4)
    sa = torch.full((2, ld), float("nan"))
    sa[0, :M] = 1.0
    sa[1, :M] = -1.0
    sb = torch.ones(inputs.ceil_div(N, 128), 2)
    return inputs.DenseProblem(M, N, K, a, sa, b, sb)


CASES = {
    # small product in the same K = 32 MMA as the eight large ones
    "same_mma": (3, [0, 1, 2, 4, 5, 6, 7, 8]),
    # small product in the last MMA of the block, large ones in the first
    "other_mma": (127, [0, 1, 2, 4, 5, 6, 7, 8]),
    # large products spread over all four MMAs, small one in the second
    "spread": (40, [0, 17, 33, 50, 64, 90, 100, 126]),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("M,N", [(256, 256), (64, 256)])
def test_block_partial_is_exact_fp32(case, M, N):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    small, large = CASES[case]
    prob = probe_problem(M, N, small, large)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, M, N, K)
    assert np.all(ref == 2.0 ** -10), "oracle: exact result is 2^-10"
    d = H.run_dense(prob)
    assert fp8.get_device_status() == 0
    got = H.bf16_bits_to_f64(d)
    # bit-exact: the result is exactly representable and has one rounding-free path
    assert np.array_equal(got, ref), (
        f"{case}: tensor-core block partial not exact in FP32 "
        f"(values seen: {np.unique(got)[:8]})")
