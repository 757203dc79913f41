"""GPU parity of the small-M dense kernel (dense calls with M <= 256: tiles of
128 columns of D by blocks of up to 128 rows, computed transposed, the K range
of a tile split over the CTAs of a cluster and combined through distributed
shared memory) against the CPU oracle, element by element, through the Python
binding and the C ABI.

Covers every built width (MN = 16, 32, 64, 128) with M at and around its
edges, every cluster size 1..8 (including more CTAs than K blocks), reuse of
the TMEM partial ring and of the operand ring (long K ranges), clusters that
walk several tiles (a lowered SM bound), ragged N, and the decode-shaped and
128x128x512 workloads at full size.
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
    fp8.force_config(0, 0)
    fp8.force_swap_ab(0)
    yield
    fp8.force_config(0, 0)
    fp8.force_swap_ab(0)
    fp8.set_num_sms(0)


def check_status():
    st = fp8.get_device_status()
    assert st == 0, f"device status {st}: {fp8.status_string(st)}"


def run_and_compare(prob, what, repeat=True):
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    cfg = fp8.select_config(fp8.KIND_DENSE, prob.M, prob.N, prob.K)
    assert cfg["swap_ab"] == 1, cfg
    d1 = H.run_dense(prob)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d1), ref, what)
    if repeat:
        d2 = H.run_dense(prob)
        check_status()
        assert torch.equal(d1.view(torch.int16), d2.view(torch.int16)), f"{what}: not deterministic"
    return d1


@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 31, 32, 33, 48, 63, 64, 65, 100, 127, 128])
def test_small_m_every_width(M):
    """All MN widths, M at and around each edge, ragged N (three full tiles
    plus 8 columns), 5 K blocks."""
    prob = inputs.make_dense(M, 392, 640, seed=500 + M)
    run_and_compare(prob, f"small-M M={M}")


@pytest.mark.parametrize("M", [129, 136, 200, 255, 256])
def test_small_m_blocks_of_rows(M):
    """M in (128, 256]: the kernel walks M in blocks of 128 rows (the last
    one partial), each block its own tile; ragged N, 9 K blocks."""
    prob = inputs.make_dense(M, 392, 128 * 9, seed=450 + M)
    run_and_compare(prob, f"small-M blocks M={M}")


@pytest.mark.parametrize("split", [1, 3, 8])
def test_small_m_blocks_of_rows_split(split):
    """Blocks of rows together with split K over a cluster."""
    prob = inputs.make_dense(200, 264, 128 * 11, seed=470 + split)
    fp8.force_config(0, 0, split)
    try:
        run_and_compare(prob, f"small-M blocks split={split}")
    finally:
        fp8.force_config(0, 0, 0)


@pytest.mark.parametrize("split", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("M", [24, 64, 128])
def test_small_m_every_split(split, M):
    """Each cluster size, 11 K blocks (not a multiple of most splits)."""
    prob = inputs.make_dense(M, 264, 128 * 11, seed=600 + 10 * split + M)
    fp8.force_config(0, 0, split)
    try:
        assert fp8.select_config(fp8.KIND_DENSE, prob.M, prob.N, prob.K)["split"] == split
        run_and_compare(prob, f"small-M M={M} split={split}")
    finally:
        fp8.force_config(0, 0, 0)


@pytest.mark.parametrize("split", [5, 8])
def test_small_m_more_ctas_than_k_blocks(split):
    """K = 3 blocks over 5 or 8 CTAs: CTAs with an empty K range add zeros."""
    prob = inputs.make_dense(40, 136, 384, seed=700 + split)
    fp8.force_config(0, 0, split)
    try:
        run_and_compare(prob, f"small-M empty K ranges split={split}")
    finally:
        fp8.force_config(0, 0, 0)


@pytest.mark.parametrize("M", [16, 32, 64, 128])
def test_small_m_ring_reuse(M):
    """56 K blocks on one CTA per tile: the TMEM partial ring (16, 16, 8 or 4
    buffers) and the operand ring both wrap many times."""
    prob = inputs.make_dense(M, 136, 7168, seed=800 + M)
    fp8.force_config(0, 0, 1)
    try:
        run_and_compare(prob, f"small-M ring reuse M={M}")
    finally:
        fp8.force_config(0, 0, 0)


@pytest.mark.parametrize("split", [1, 2, 3])
def test_small_m_clusters_walk_several_tiles(split):
    """A lowered SM bound: fewer clusters than tiles, each walking several
    tiles (the rings and barrier phases carry over between tiles)."""
    prob = inputs.make_dense(40, 128 * 20 + 8, 1024, seed=900 + split)
    fp8.force_config(0, 0, split)
    fp8.set_num_sms(6)
    try:
        cfg = fp8.select_config(fp8.KIND_DENSE, prob.M, prob.N, prob.K, num_sms=6)
        assert cfg["grid"] <= 6 and cfg["num_tiles"] == 21
        run_and_compare(prob, f"small-M persistent split={split}")
    finally:
        fp8.set_num_sms(0)
        fp8.force_config(0, 0, 0)


def test_small_m_matches_other_kernel():
    """The same call through the 128-row kernels gives results within the
    tolerance of each other (both are checked against the oracle)."""
    prob = inputs.make_dense(64, 1040, 2048, seed=950)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    d_small = H.run_dense(prob)
    check_status()
    fp8.force_swap_ab(1)
    try:
        d_wide = H.run_dense(prob)
    finally:
        fp8.force_swap_ab(0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d_small), ref, "small-M kernel")
    H.assert_close(H.bf16_bits_to_f64(d_wide), ref, "128-row kernel")


def test_small_m_no_stray_writes():
    """Only the M x N region of D changes (D is a slice of a larger buffer)."""
    prob = inputs.make_dense(50, 264, 512, seed=960)
    big = H.sentinel_like((prob.M + 5, prob.N))
    H.run_dense(prob, big[: prob.M])
    check_status()
    assert H.untouched(big[prob.M:]).all()
    assert not H.untouched(big[: prob.M]).any()


@pytest.mark.parametrize("name", ["dense_decode_64x2112x7168", "dense_128x128x512",
                                  "dense_prefill_256x7168x2048"])
def test_small_m_full_size_all_elements(name):
    """The decode-shaped and 128x128x512 workloads, in the configuration the
    benchmark launches, every element against the oracle."""
    prob = inputs.make_workload(name)
    run_and_compare(prob, name)
