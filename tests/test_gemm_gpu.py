"""GPU parity: the CUDA path (through the Python binding and the C ABI) against
the CPU oracle on the same seeded inputs.

Small cases compare every element; full-size cases (the measured workloads, in
the configuration the benchmark launches) compare sampled elements and whole
rows, and check the properties that hold at any size: rows that must stay
untouched keep their sentinel bits, and repeated calls are bit-identical.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_nt_b200 as fp8
from fp8_fine_grained_nt_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu

BUILT_SHAPES = None


def built_shapes():
    from fp8_fine_grained_nt_b200 import build
    return build.kernel_shapes()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_fine_grained_nt_b200 import build
    build.build()
    fp8.force_config(0, 0)
    yield
    fp8.force_config(0, 0)


def check_status():
    st = fp8.get_device_status()
    assert st == 0, f"device status {st}: {fp8.status_string(st)}"


# --------------------------------------------------------------------- dense


def force_shape(mw, bn, pair, split=0):
    """Pin one built kernel: (MW, BN) with one CTA per tile, or a CTA pair."""
    fp8.force_config(256 if pair else 128 * mw, bn, split, 2 if pair else 1)


@pytest.mark.parametrize("mw,bn,pair", built_shapes())
def test_dense_every_kernel_shape_ragged(mw, bn, pair):
    """Each built tile shape on a shape with ragged M, N tails and several K blocks."""
    prob = inputs.make_dense(300, 400, 512, seed=100 + bn + mw + 7 * pair)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    force_shape(mw, bn, pair)
    try:
        cfg = fp8.select_config(fp8.KIND_DENSE, prob.M, prob.N, prob.K)
        assert cfg["cta_pair"] == (2 if pair else 1)
        d = H.run_dense(prob)
    finally:
        fp8.force_config(0, 0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, f"dense mw{mw} bn{bn} pair{pair}")


@pytest.mark.parametrize("M", [1, 100, 128, 200, 256, 300, 520])
@pytest.mark.parametrize("bn", [128, 256])
def test_dense_cta_pair_row_edges(M, bn):
    """CTA pairs where the second CTA's 128 rows are partly or wholly past M,
    with 11 K blocks (a partial promotion step) and a ragged N tail."""
    prob = inputs.make_dense(M, bn * 2 + 40, 128 * 11, seed=400 + M + bn)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    force_shape(1, bn, True)
    try:
        d1 = H.run_dense(prob)
        d2 = H.run_dense(prob)
    finally:
        fp8.force_config(0, 0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d1), ref, f"pair M{M} bn{bn}")
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


def test_dense_cta_pair_more_tiles_than_pairs():
    """A pair walks several 256-row tiles (persistent loop) with the SM
    bound lowered so that every pair takes many tiles."""
    prob = inputs.make_dense(1000, 1040, 1024, seed=77)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    force_shape(1, 160, True)
    fp8.set_num_sms(8)
    try:
        d = H.run_dense(prob)
    finally:
        fp8.set_num_sms(0)
        fp8.force_config(0, 0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, "pair persistent")


@pytest.mark.parametrize("mw,bn", [(1, 16), (1, 32), (1, 48), (1, 64), (2, 32), (2, 64)])
def test_dense_grouped_promotion_partial_steps(mw, bn):
    """K = 11 blocks: promotion steps of several K blocks end with a partial step."""
    prob = inputs.make_dense(200, 136, 128 * 11, seed=200 + bn + mw)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    fp8.force_config(128 * mw, bn)
    try:
        d = H.run_dense(prob)
    finally:
        fp8.force_config(0, 0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, f"dense K=1408 mw{mw} bn{bn}")


@pytest.mark.parametrize("mw,bn,split", [(1, 16, 2), (1, 64, 4), (1, 128, 2), (1, 112, 4),
                                         (2, 32, 2), (1, 96, 4), (1, 128, 8), (1, 32, 8)])
def test_dense_split_k(mw, bn, split):
    """Split-K over a thread-block cluster: ragged M and N, K blocks not a
    multiple of the split, reduction through distributed shared memory."""
    # 11 K blocks (19 for 8 CTAs: at least two per CTA), not a multiple of the split
    prob = inputs.make_dense(100 if mw == 1 else 300, 336, 128 * (11 if split <= 4 else 19),
                             seed=300 + bn + split)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    fp8.force_config(128 * mw, bn, split)
    try:
        d1 = H.run_dense(prob)
        d2 = H.run_dense(prob)
    finally:
        fp8.force_config(0, 0, 0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d1), ref, f"split-K mw{mw} bn{bn} s{split}")
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16)), "split-K not deterministic"


@pytest.mark.parametrize("M,N,K", [(1, 8, 128), (1, 16, 128), (5, 24, 256), (128, 128, 512),
                                   (129, 136, 384), (257, 8, 128), (64, 2112, 7168)])
def test_dense_auto_config(M, N, K):
    prob = inputs.make_dense(M, N, K, seed=M * 7 + N + K)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, M, N, K)
    d = H.run_dense(prob)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, f"dense {M}x{N}x{K}")


def test_dense_exact_small_integers():
    """Unit scales and small-integer FP8 values give an exact result: bit-exact BF16."""
    M, N, K = 200, 144, 512
    one = torch.tensor([1.0]).to(torch.float8_e4m3fn).view(torch.uint8)
    vals = torch.tensor([float(i % 4 + 1) for i in range(M)]).to(torch.float8_e4m3fn)
    a = vals.view(torch.uint8)[:, None].expand(M, K).contiguous()
    b = one.expand(N, K).contiguous()
    ld = inputs.tma_aligned_size(M, 4)
    prob = inputs.DenseProblem(M, N, K, a, torch.ones(K // 128, ld), b,
                               torch.ones(math.ceil(N / 128), K // 128))
    d = H.run_dense(prob)
    got = H.bf16_bits_to_f64(d)
    expect = np.array([[512.0 * (i % 4 + 1)] * N for i in range(M)])
    assert np.array_equal(got, expect)


def test_dense_deterministic_and_no_stray_writes():
    prob = inputs.make_dense(250, 264, 1024, seed=5)
    d1 = H.run_dense(prob)
    d2 = H.run_dense(prob)
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
    # a larger buffer: only the M x N region may change
    big = H.sentinel_like((prob.M + 3, prob.N))
    H.run_dense(prob, big[: prob.M])
    assert H.untouched(big[prob.M:]).all()


# --------------------------------------------------------------------- contiguous


def test_contiguous_small_all_rows():
    prob = inputs.make_contiguous(4, 272, 384, seed=21, counts=[0, 5, 130, 257])
    ref = oracle.gemm_contiguous(prob.a, prob.sa, prob.b, prob.sb, prob.m_indices,
                                 prob.num_groups, prob.M_sum, prob.N, prob.K)
    d = H.run_contiguous(prob)
    check_status()
    valid = prob.m_indices.numpy() >= 0
    H.assert_close(H.bf16_bits_to_f64(d)[valid], ref[valid], "contiguous small")
    assert H.untouched(d)[~valid].all(), "padding rows were written"


@pytest.mark.parametrize("bn", [64, 112, 256])
def test_contiguous_forced_shapes(bn):
    prob = inputs.make_contiguous(3, 320, 256, seed=22 + bn, counts=[129, 1, 300])
    ref = oracle.gemm_contiguous(prob.a, prob.sa, prob.b, prob.sb, prob.m_indices,
                                 prob.num_groups, prob.M_sum, prob.N, prob.K)
    fp8.force_config(128, bn)
    try:
        d = H.run_contiguous(prob)
    finally:
        fp8.force_config(0, 0)
    check_status()
    valid = prob.m_indices.numpy() >= 0
    H.assert_close(H.bf16_bits_to_f64(d)[valid], ref[valid], f"contiguous bn{bn}")
    assert H.untouched(d)[~valid].all()


def test_contiguous_bad_expert_index_reported():
    prob = inputs.make_contiguous(2, 64, 128, seed=23, counts=[128, 128])
    prob.m_indices[128:256] = 7  # out of range for 2 experts
    d = H.run_contiguous(prob)
    assert fp8.get_device_status() == 7
    assert H.untouched(d)[128:].all()
    assert fp8.get_device_status() == 0  # cleared


# --------------------------------------------------------------------- masked


@pytest.mark.parametrize("expected_m", [0, 1, 100])
def test_masked_small_all_rows(expected_m):
    prob = inputs.make_masked(5, 200, 272, 384, seed=31, masked_m=[0, 200, 1, 128, 129])
    ref = oracle.gemm_masked(prob.a, prob.sa, prob.b, prob.sb, prob.masked_m, prob.G,
                             prob.M_max, prob.N, prob.K)
    d = H.run_masked(prob, expected_m=expected_m)
    check_status()
    got = H.bf16_bits_to_f64(d)
    valid = ~np.isnan(ref)
    H.assert_close(got[valid], ref[valid], "masked small")
    assert H.untouched(d)[~valid].all(), "rows at or beyond masked_m were written"


@pytest.mark.parametrize("mw,bn,pair", [(1, 64, 0), (1, 224, 0), (2, 64, 0), (2, 128, 0),
                                        (1, 128, 1), (1, 256, 1)])
def test_masked_forced_shapes(mw, bn, pair):
    prob = inputs.make_masked(4, 300, 256, 256, seed=32 + bn + pair,
                              masked_m=[300, 0, 129, 257])
    ref = oracle.gemm_masked(prob.a, prob.sa, prob.b, prob.sb, prob.masked_m, prob.G,
                             prob.M_max, prob.N, prob.K)
    force_shape(mw, bn, pair)
    try:
        d = H.run_masked(prob)
    finally:
        fp8.force_config(0, 0)
    check_status()
    valid = ~np.isnan(ref)
    H.assert_close(H.bf16_bits_to_f64(d)[valid], ref[valid], f"masked mw{mw} bn{bn}")
    assert H.untouched(d)[~valid].all()


def test_masked_all_empty_and_out_of_range():
    prob = inputs.make_masked(3, 64, 128, 128, seed=33, masked_m=[0, 0, 0])
    d = H.run_masked(prob)
    check_status()
    assert H.untouched(d).all()
    prob.masked_m[1] = 500  # beyond M_max: clamped, flagged
    d = H.run_masked(prob)
    assert fp8.get_device_status() == 7
    ref = oracle.gemm_masked(prob.a, prob.sa, prob.b, prob.sb, torch.tensor([0, 64, 0],
                             dtype=torch.int32), 3, 64, 128, 128)
    got = H.bf16_bits_to_f64(d)
    H.assert_close(got[1], ref[1], "masked clamped")


# --------------------------------------------------------------------- full size


def _sample(rng, n, hi):
    return rng.integers(0, hi, n)


@pytest.mark.parametrize("name", ["dense_128x128x512", "dense_decode_64x2112x7168",
                                  "dense_prefill_4096x7168x2048", "dense_prefill_256x7168x2048"])
def test_full_size_dense(name):
    prob = inputs.make_workload(name)
    d = H.run_dense(prob)
    check_status()
    got = H.bf16_bits_to_f64(d)
    rng = np.random.default_rng(1)
    rows = np.concatenate([_sample(rng, 3000, prob.M), np.full(prob.N, prob.M - 1)])
    cols = np.concatenate([_sample(rng, 3000, prob.N), np.arange(prob.N)])
    ref = oracle.gemm_dense_sampled(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K,
                                    rows, cols)
    H.assert_close(got[rows, cols], ref, name)
    d2 = H.run_dense(prob)
    assert torch.equal(d.view(torch.int16), d2.view(torch.int16))


def test_full_size_contiguous():
    prob = inputs.make_workload("contiguous_8x4096x7168")
    d = H.run_contiguous(prob)
    check_status()
    got = H.bf16_bits_to_f64(d)
    mi = prob.m_indices.numpy()
    valid_rows = np.nonzero(mi >= 0)[0]
    rng = np.random.default_rng(2)
    rows = valid_rows[rng.integers(0, len(valid_rows), 4000)]
    cols = _sample(rng, 4000, prob.N)
    # whole first and last row of every expert
    starts = np.nonzero(np.diff(np.concatenate([[-2], mi])) != 0)[0]
    edge_rows = []
    for s in starts:
        if mi[s] >= 0:
            e = mi[s]
            last = s + int(np.sum(mi[s:s + 9000] == e)) - 1
            edge_rows += [s, last]
    rows = np.concatenate([rows, np.repeat(edge_rows, prob.N)])
    cols = np.concatenate([cols, np.tile(np.arange(prob.N), len(edge_rows))])
    # one whole 128 x 256 output tile at an expert boundary: the last, partly
    # padded M block of the first expert whose count is not a multiple of 128,
    # every row of it (valid rows compared, padding rows must keep the sentinel)
    # over the tile's 256 columns at the end of N
    e_b = next(e for e, c in enumerate(prob.counts) if c % 128 != 0)
    seg0 = sum(-(-c // 128) * 128 for c in prob.counts[:e_b])
    blk0 = seg0 + (prob.counts[e_b] // 128) * 128
    t_rows = np.arange(blk0, blk0 + 128)
    t_valid = t_rows[mi[t_rows] >= 0]
    t_cols = np.arange(prob.N - 256, prob.N)
    rows = np.concatenate([rows, np.repeat(t_valid, 256)])
    cols = np.concatenate([cols, np.tile(t_cols, len(t_valid))])
    ref = oracle.gemm_contiguous_sampled(prob.a, prob.sa, prob.b, prob.sb, prob.m_indices,
                                         prob.num_groups, prob.M_sum, prob.N, prob.K, rows, cols)
    H.assert_close(got[rows, cols], ref, "contiguous full")
    assert H.untouched(d)[mi < 0].all(), "padding rows were written"
    assert 0 < len(t_valid) < 128 and H.untouched(d)[t_rows[mi[t_rows] < 0]][:, t_cols].all()


@pytest.mark.parametrize("name", ["masked_16x256_4096x7168", "masked_16x256_7168x2048"])
def test_full_size_masked(name):
    prob = inputs.make_workload(name)
    # the same hint (and so the same tile configuration) as the benchmark
    expected_m = max(1, int(round(float(prob.masked_m.float().mean()))))
    d = H.run_masked(prob, expected_m=expected_m)
    check_status()
    got = H.bf16_bits_to_f64(d)
    mm = prob.masked_m.numpy()
    rng = np.random.default_rng(3)
    act = np.nonzero(mm > 0)[0]
    groups = act[rng.integers(0, len(act), 4000)]
    rows = rng.integers(0, 1 << 30, 4000) % mm[groups]
    cols = _sample(rng, 4000, prob.N)
    last_g = act
    groups = np.concatenate([groups, np.repeat(last_g, prob.N)])
    rows = np.concatenate([rows, np.repeat(mm[last_g] - 1, prob.N)])
    cols = np.concatenate([cols, np.tile(np.arange(prob.N), len(last_g))])
    ref = oracle.gemm_masked_sampled(prob.a, prob.sa, prob.b, prob.sb, prob.masked_m, prob.G,
                                     prob.M_max, prob.N, prob.K, groups, rows, cols)
    H.assert_close(got[groups, rows, cols], ref, name)
    unt = H.untouched(d)
    for g in range(prob.G):
        assert unt[g, mm[g]:].all(), f"group {g}: rows beyond masked_m written"


# --------------------------------------------------------------------- per-tensor scaling


def run_per_tensor(a, scale_a, b, scale_b, M, N):
    d = H.sentinel_like((M, N))
    fp8.gemm_fp8_fp8_bf16_nt_per_tensor(a.cuda(), torch.tensor([scale_a], device="cuda"), b.cuda(),
                                        torch.tensor([scale_b], device="cuda"), d)
    torch.cuda.synchronize()
    return d


def per_tensor_problem(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    b = torch.randn(N, K, generator=g).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    return a, b


def scalar_shapes():
    from fp8_fine_grained_nt_b200 import build
    return build.scalar_kernel_shapes()


@pytest.mark.parametrize("bn", scalar_shapes())
def test_per_tensor_every_kernel_shape(bn):
    """Whole-K accumulation in TMEM, ragged M and N, several K blocks."""
    M, N, K = 300, 400, 1280
    a, b = per_tensor_problem(M, N, K, 500 + bn)
    ref = oracle.gemm_per_tensor(a, 0.02, b, 0.5, M, N, K)
    fp8.force_config(128, bn)
    try:
        d = run_per_tensor(a, 0.02, b, 0.5, M, N)
    finally:
        fp8.force_config(0, 0)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, f"per-tensor bn{bn}")


@pytest.mark.parametrize("M,N,K", [(1, 8, 128), (129, 136, 7168), (512, 2112, 7168)])
def test_per_tensor_auto_config(M, N, K):
    a, b = per_tensor_problem(M, N, K, M + N + K)
    ref = oracle.gemm_per_tensor(a, 0.125, b, 0.25, M, N, K)
    d = run_per_tensor(a, 0.125, b, 0.25, M, N)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, f"per-tensor {M}x{N}x{K}")


def test_per_tensor_full_size_sampled():
    """4096 x 7168 x 2048 in the configuration the benchmark launches: sampled
    rows against the oracle, and bit-identical repeats."""
    M, N, K = 4096, 7168, 2048
    a, b = per_tensor_problem(M, N, K, 77)
    d1 = run_per_tensor(a, 0.01, b, 0.03, M, N)
    d2 = run_per_tensor(a, 0.01, b, 0.03, M, N)
    check_status()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
    rows = np.random.default_rng(3).choice(M, 24, replace=False)
    ref = oracle.gemm_per_tensor(a[rows].contiguous(), 0.01, b, 0.03, len(rows), N, K)
    H.assert_close(H.bf16_bits_to_f64(d1)[rows], ref, "per-tensor full size")


# --------------------------------------------------------------------- quantiser (1x128)


def run_quantize(x: torch.Tensor):
    M, K = x.shape
    ld = inputs.tma_aligned_size(M, 4)
    q = torch.full((M, K), 0xAA, dtype=torch.uint8, device="cuda")
    sa = torch.full((K // 128, ld), float("nan"), dtype=torch.float32, device="cuda")
    fp8.quantize_fp8_1x128(x.cuda(), q, sa)
    torch.cuda.synchronize()
    check_status()
    return q.cpu().numpy(), sa.cpu().numpy()


def assert_quant_equal(x32: np.ndarray, q, sa, what):
    M, K = x32.shape
    q_ref, sa_ref = oracle.quantize_1x128(x32, M, K, ld_sa=sa.shape[1])
    assert np.array_equal(q, q_ref), f"{what}: {int((q != q_ref).sum())} codes differ"
    assert np.array_equal(sa[:, :M], sa_ref[:, :M]), f"{what}: scales differ"
    assert np.isnan(sa[:, M:]).all(), f"{what}: padding columns written"


@pytest.mark.parametrize("M,K", [(1, 128), (31, 256), (300, 1280), (64, 7168)])
def test_quantize_fp32_bit_exact(M, K):
    g = torch.Generator().manual_seed(M * 131 + K)
    x = torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g) * 3)
    q, sa = run_quantize(x)
    assert_quant_equal(x.numpy(), q, sa, f"fp32 {M}x{K}")


def test_quantize_bf16_bit_exact():
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(257, 1024, generator=g) * 5).to(torch.bfloat16)
    q, sa = run_quantize(x)
    assert_quant_equal(x.float().numpy(), q, sa, "bf16")


def test_quantize_edge_values():
    """Zero blocks (amax floor), -0, huge and tiny magnitudes, exact maxima."""
    x = torch.zeros(40, 512)
    x[1, :128] = -0.0
    x[2, 128:256] = 1e30
    x[2, 130] = -3e30
    x[3, 256:384] = 1e-30
    x[4, :] = torch.linspace(-448, 448, 512)
    x[5, 384:] = torch.tensor([1.0625, 1.1875, -1.0625] * 42 + [448.0, -448.0])
    q, sa = run_quantize(x)
    assert_quant_equal(x.numpy(), q, sa, "edges")


def test_quantize_full_size_then_gemm():
    """4096 x 7168 activations quantised on the device match the oracle
    bit for bit, and feed the GEMM directly."""
    M, K, N = 4096, 7168, 256
    g = torch.Generator().manual_seed(21)
    x = torch.randn(M, K, generator=g)
    q, sa = run_quantize(x)
    assert_quant_equal(x.numpy(), q, sa, "full size")
    prob = inputs.make_dense(M, N, K, seed=22)
    d = H.sentinel_like((M, N))
    fp8.gemm_fp8_fp8_bf16_nt(torch.from_numpy(q).cuda(), torch.from_numpy(sa).cuda(), prob.b.cuda(),
                             prob.sb.cuda(), d)
    torch.cuda.synchronize()
    rows = np.arange(0, M, 97)
    ref = oracle.gemm_dense(q[rows], sa[:, rows].copy(), prob.b, prob.sb, len(rows), N, K)
    H.assert_close(H.bf16_bits_to_f64(d)[rows], ref, "quantised then GEMM")


# --------------------------------------------------------------------- many experts


def test_contiguous_many_experts():
    """64 experts with counts from 0 to 300 (many empty or single-block
    segments), every row compared."""
    G = 64
    counts = [int(c) for c in np.random.default_rng(64).integers(0, 301, G)]
    counts[5] = 0
    counts[6] = 1
    prob = inputs.make_contiguous(G, 256, 256, seed=64, counts=counts)
    ref = oracle.gemm_contiguous(prob.a, prob.sa, prob.b, prob.sb, prob.m_indices,
                                 prob.num_groups, prob.M_sum, prob.N, prob.K)
    d = H.run_contiguous(prob)
    check_status()
    valid = prob.m_indices.numpy() >= 0
    H.assert_close(H.bf16_bits_to_f64(d)[valid], ref[valid], "contiguous 64 experts")
    assert H.untouched(d)[~valid].all()


def test_masked_many_groups():
    """256 groups of up to 64 rows (the device enumerates the tiles of every
    group from masked_m), rows past masked_m untouched."""
    G = 256
    mm = [int(c) for c in np.random.default_rng(256).integers(0, 65, G)]
    prob = inputs.make_masked(G, 64, 128, 256, seed=256, masked_m=mm)
    ref = oracle.gemm_masked(prob.a, prob.sa, prob.b, prob.sb, prob.masked_m, prob.G,
                             prob.M_max, prob.N, prob.K)
    d = H.run_masked(prob)
    check_status()
    valid = ~np.isnan(ref)
    H.assert_close(H.bf16_bits_to_f64(d)[valid], ref[valid], "masked 256 groups")
    assert H.untouched(d)[~valid].all()


def test_contiguous_skewed_experts():
    """A Zipf-like expert load (most tokens on a few experts, some experts
    empty), every row compared."""
    counts = [1500, 700, 260, 90, 31, 7, 1, 0]
    prob = inputs.make_contiguous(8, 384, 512, seed=99, counts=counts)
    ref = oracle.gemm_contiguous(prob.a, prob.sa, prob.b, prob.sb, prob.m_indices,
                                 prob.num_groups, prob.M_sum, prob.N, prob.K)
    d = H.run_contiguous(prob)
    check_status()
    valid = prob.m_indices.numpy() >= 0
    H.assert_close(H.bf16_bits_to_f64(d)[valid], ref[valid], "contiguous skewed")
    assert H.untouched(d)[~valid].all()


# --------------------------------------------------------------------- failure detection


def test_bounded_wait_reports_timeout_and_context_survives():
    """A device wait that nothing satisfies gives up after its limit and is
    reported through the status word; no fault, and later calls still work."""
    assert fp8.get_device_status() == 0
    fp8.selftest_wait_timeout(20000)  # 20 ms
    assert fp8.get_device_status() == 6, "expected DG_ERR_DEVICE_TIMEOUT"
    assert fp8.get_device_status() == 0, "status word not cleared"
    prob = inputs.make_dense(130, 200, 384, seed=8)
    ref = oracle.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    d = H.run_dense(prob)
    check_status()
    H.assert_close(H.bf16_bits_to_f64(d), ref, "after the timeout self-test")
