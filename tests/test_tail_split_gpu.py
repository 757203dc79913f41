"""GPU parity of the opt-in split of a dense call's last partial wave: the
tiles of that wave that form one block of D (the last M block from a 128-column
boundary on) are computed by the small-M kernel after the main kernel, which
runs whole waves only.  Every element is compared with the CPU oracle, with
the split on and off, and the rows of D past M are checked untouched.
"""

import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_nt_b200 as fp8
from fp8_fine_grained_nt_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_fine_grained_nt_b200 import build
    build.build()
    yield
    fp8.force_config(0, 0)
    fp8.force_tail_split(0)
    fp8.set_num_sms(0)


def check_status():
    st = fp8.get_device_status()
    assert st == 0, f"device status {st}: {fp8.status_string(st)}"


def run_padded(prob):
    """D as the first M rows of a larger sentinel-filled buffer."""
    big = H.sentinel_like((prob.M + 3, prob.N))
    H.run_dense(prob, big[: prob.M])
    check_status()
    assert H.untouched(big[prob.M:]).all(), "rows past M were written"
    return big[: prob.M]


# (M, N, K, block_m, block_n, SM bound, tail tiles)
CASES = [
    (320, 768, 1024, 128, 256, 8, 1),    # 9 tiles on 8 SMs: the last at column 512
    (300, 1280, 640, 128, 256, 6, 3),    # 15 on 6: three tiles of a 44-row block
    (300, 1280, 640, 128, 256, 7, 1),    # 15 on 7: one tile
    (300, 960, 640, 128, 192, 4, 3),     # BLOCK_N = 192, tail from column 384
    (600, 640, 512, 256, 128, 4, 3),     # 256-row tiles, an 88-row last block
    (200, 1024, 2048, 128, 128, 12, 4),  # 2 x 8 tiles on 12 SMs, 16 K blocks
]


@pytest.mark.parametrize("M,N,K,bm,bn,sms,tail", CASES)
def test_tail_split_all_elements(M, N, K, bm, bn, sms, tail):
    prob = inputs.make_dense(M, N, K, seed=1200 + M + N + bn + sms)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    fp8.force_config(bm, bn)
    fp8.set_num_sms(sms)
    try:
        fp8.force_tail_split(2)
        cfg = fp8.select_config(fp8.KIND_DENSE, M, N, K, num_sms=sms)
        assert cfg["tail_tiles"] == tail and cfg["swap_ab"] == 0, cfg
        d_tail = run_padded(prob)
        H.assert_close(H.bf16_bits_to_f64(d_tail), ref, f"tail split {M}x{N}x{K}")
        d_again = run_padded(prob)
        assert torch.equal(d_tail.view(torch.int16), d_again.view(torch.int16)), "not deterministic"
        fp8.force_tail_split(1)
        assert fp8.select_config(fp8.KIND_DENSE, M, N, K, num_sms=sms)["tail_tiles"] == 0
        d_whole = run_padded(prob)
        H.assert_close(H.bf16_bits_to_f64(d_whole), ref, f"no tail split {M}x{N}x{K}")
        # the main kernel's tiles are the same launch shape either way
        m_blocks = -(-M // bm)
        n_blocks = -(-N // bn)
        full = (m_blocks * n_blocks) // min(sms, m_blocks * n_blocks) * min(sms, m_blocks * n_blocks)
        row0 = (m_blocks - 1) * bm
        col0 = (full - (m_blocks - 1) * n_blocks) * bn
        a = d_tail.view(torch.int16).cpu().numpy()
        b = d_whole.view(torch.int16).cpu().numpy()
        assert np.array_equal(a[:row0], b[:row0]) and np.array_equal(a[row0:, :col0], b[row0:, :col0])
    finally:
        fp8.force_tail_split(0)
        fp8.set_num_sms(0)
        fp8.force_config(0, 0)


def test_tail_split_full_size_block():
    """Dense 4096 x 7168 x 2048 with the split by estimate: 888 tiles in six
    whole waves and the last 8 (rows 3968.., columns 5120..) on the small-M
    kernel.  The whole tail block, and the main kernel's rows and
    columns next to it, against the oracle."""
    prob = inputs.make_workload("dense_prefill_4096x7168x2048")
    fp8.force_tail_split(3)
    try:
        cfg = fp8.select_config(fp8.KIND_DENSE, prob.M, prob.N, prob.K)
        assert cfg["tail_tiles"] == 8
        d = H.run_dense(prob)
    finally:
        fp8.force_tail_split(0)
    check_status()
    got = H.bf16_bits_to_f64(d)
    r0, c0 = 3968, 5120
    rr, cc = np.meshgrid(np.arange(r0, prob.M), np.arange(c0, prob.N), indexing="ij")
    rows = np.concatenate([rr.ravel(), np.full(prob.N, r0 - 1), np.arange(r0, prob.M)])
    cols = np.concatenate([cc.ravel(), np.arange(prob.N), np.full(prob.M - r0, c0 - 1)])
    ref = oracle.gemm_dense_sampled(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K,
                                    rows, cols)
    H.assert_close(got[rows, cols], ref, "dense 4096x7168x2048 tail block")
