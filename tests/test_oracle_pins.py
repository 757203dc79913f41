"""Pins for the CPU oracle: checks against facts that do not come from the oracle.

Each pin is a function of an oracle handle so that the mutation test at the
bottom can run the same pins against deliberately broken copies of oracle.c
(mistakes are planted in the oracle, on the CPU) and show that every planted
mistake fails at least one pin.
"""

import math
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_nt_b200 import inputs
from tests.conftest import read_golden

E4M3 = torch.float8_e4m3fn


def torch_decode(u8) -> np.ndarray:
    """Decode E4M3 bytes with torch's float8 type (independent of the oracle)."""
    t = torch.as_tensor(np.ascontiguousarray(u8)).view(E4M3)
    return t.to(torch.float64).numpy()


def encode(values) -> np.ndarray:
    """E4M3 bytes for exactly representable values, via torch's encoder."""
    t = torch.tensor(values, dtype=torch.float32).to(E4M3)
    back = t.to(torch.float32)
    assert torch.equal(back, torch.tensor(values, dtype=torch.float32)), "not representable"
    return t.view(torch.uint8).numpy()


def random_finite_bytes(rng, shape) -> np.ndarray:
    b = rng.integers(0, 256, size=shape, dtype=np.uint8)
    nan = (b & 0x7F) == 0x7F
    b[nan] ^= 0x01  # 0x7F -> 0x7E (448), 0xFF -> 0xFE (-448)
    return b


def col_major(sa_rows: np.ndarray, pad=np.nan) -> np.ndarray:
    M, nkb = sa_rows.shape
    ld = inputs.tma_aligned_size(M, 4)
    out = np.full((nkb, ld), pad, dtype=np.float32)
    out[:, :M] = sa_rows.T
    return out


def dense_reference_by_matmul(a, sa_rows, b, sb, K):
    """Independent route: expand the scales to per-k factors and use float64 matmul."""
    A = torch_decode(a)
    B = torch_decode(b)
    nkb = math.ceil(K / 128)
    out = np.zeros((A.shape[0], B.shape[0]))
    for kb in range(nkb):
        ks = slice(kb * 128, min(K, (kb + 1) * 128))
        part = A[:, ks] @ B[:, ks].T
        col_scale = np.repeat(sb[:, kb].astype(np.float64), 128)[: B.shape[0]]
        out += part * sa_rows[:, kb].astype(np.float64)[:, None] * col_scale[None, :]
    return out


# ---------------------------------------------------------------------------
# Pins, each a function of an oracle handle; each returns None or raises.


def pin_decode_table_matches_torch(lib):
    table = lib.e4m3_table()
    ref = torch_decode(np.arange(256, dtype=np.uint8))
    nan_t, nan_r = np.isnan(table), np.isnan(ref)
    assert np.array_equal(nan_t, nan_r)
    assert set(np.nonzero(nan_t)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(table[~nan_t], ref[~nan_r])


def pin_decode_golden_range(lib):
    table = lib.e4m3_table()
    for byte, value in read_golden("e4m3_range.txt"):
        assert table[int(byte, 16)] == float(value)
    finite = table[~np.isnan(table)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert not np.isinf(table).any()
    # smallest subnormal and smallest normal, from the bit layout's closed form
    assert table[0x01] == 2.0 ** -9 and table[0x08] == 2.0 ** -6


def pin_small_integer_exact(lib):
    """A row i = (i mod 4) + 1, B = 1, unit scales, K = 512: D = 512 ((i mod 4) + 1)."""
    M, N, K = 8, 16, 512
    a = np.stack([np.repeat(encode([float(i % 4 + 1)]), K) for i in range(M)])
    b = np.repeat(encode([1.0]), N * K).reshape(N, K)
    sa = col_major(np.ones((M, K // 128), np.float32))
    sb = np.ones((1, K // 128), np.float32)
    D = lib.gemm_dense(a, sa, b, sb, M, N, K)
    expect = np.array([[512.0 * (i % 4 + 1)] * N for i in range(M)])
    assert np.array_equal(D, expect)


def pin_scale_indexing_closed_form(lib):
    """A = B = 1, sa[m,kb] = (m+1)(kb+1), sb[nb,kb] = (nb+1) 2^kb:
    D[m,n] = 128 (m+1)(n//128 + 1) sum_kb (kb+1) 2^kb."""
    M, N, K = 3, 300, 512
    nkb, nnb = K // 128, math.ceil(N / 128)
    a = np.repeat(encode([1.0]), M * K).reshape(M, K)
    b = np.repeat(encode([1.0]), N * K).reshape(N, K)
    sa_rows = np.array([[(m + 1) * (kb + 1) for kb in range(nkb)] for m in range(M)], np.float32)
    sb = np.array([[(nb + 1) * 2.0 ** kb for kb in range(nkb)] for nb in range(nnb)], np.float32)
    D = lib.gemm_dense(a, col_major(sa_rows), b, sb, M, N, K)
    s = sum((kb + 1) * 2 ** kb for kb in range(nkb))
    expect = np.array([[128.0 * (m + 1) * (n // 128 + 1) * s for n in range(N)]
                       for m in range(M)])
    assert np.array_equal(D, expect)


def pin_sign_and_per_k_products(lib):
    """Alternating-sign operands: D[m,n] = sum_k a_k b_k with a closed form."""
    K = 256
    av = [(-1.0) ** k * (1 + (k % 3)) for k in range(K)]       # +-1, +-2, +-3
    bv = [0.5 if k < 128 else -4.0 for k in range(K)]
    a = encode(av).reshape(1, K)
    b = encode(bv).reshape(1, K)
    sa = col_major(np.array([[1.0, 0.25]], np.float32))
    sb = np.array([[2.0, 8.0]], np.float32)
    D = lib.gemm_dense(a, sa, b, sb, 1, 1, K)
    p0 = sum(av[k] * bv[k] for k in range(128))
    p1 = sum(av[k] * bv[k] for k in range(128, 256))
    assert D[0, 0] == p0 * 1.0 * 2.0 + p1 * 0.25 * 8.0


def pin_brute_force_tiny(lib):
    """Direct per-k sum with per-k scale lookup on tiny random shapes."""
    rng = np.random.default_rng(1234)
    for (M, N, K) in [(1, 1, 128), (3, 5, 256), (8, 8, 384), (2, 136, 256), (5, 3, 128)]:
        a = random_finite_bytes(rng, (M, K))
        b = random_finite_bytes(rng, (N, K))
        nkb, nnb = K // 128, math.ceil(N / 128)
        sa_rows = rng.uniform(1e-3, 2.0, (M, nkb)).astype(np.float32)
        sb = rng.uniform(1e-3, 2.0, (nnb, nkb)).astype(np.float32)
        D = lib.gemm_dense(a, col_major(sa_rows), b, sb, M, N, K)
        A, B = torch_decode(a), torch_decode(b)
        for m in range(M):
            for n in range(N):
                terms = [A[m, k] * B[n, k] * float(sa_rows[m, k // 128]) * float(sb[n // 128, k // 128])
                         for k in range(K)]
                ref = math.fsum(terms)
                assert abs(D[m, n] - ref) <= 1e-12 * max(1.0, abs(ref)), (M, N, K, m, n)


def pin_unit_scales_equal_library_matmul(lib):
    rng = np.random.default_rng(7)
    M, N, K = 37, 70, 640
    a = random_finite_bytes(rng, (M, K))
    b = random_finite_bytes(rng, (N, K))
    sa = col_major(np.ones((M, K // 128), np.float32))
    sb = np.ones((1, K // 128), np.float32)
    D = lib.gemm_dense(a, sa, b, sb, M, N, K)
    ref = torch_decode(a) @ torch_decode(b).T  # every partial sum is exact in FP64
    assert np.array_equal(D, ref)


def pin_scaled_matches_expanded_matmul(lib):
    prob = inputs.make_dense(70, 260, 384, seed=11)
    sa_rows = prob.sa[:, :prob.M].T.numpy()
    D = lib.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    ref = dense_reference_by_matmul(prob.a.numpy(), sa_rows, prob.b.numpy(), prob.sb.numpy(),
                                    prob.K)
    assert np.allclose(D, ref, rtol=1e-13, atol=1e-12)


def pin_linearity_in_scale_block(lib):
    """Doubling sa[m,kb] adds sa[m,kb] * sb[n//128,kb] * partial_kb[m,n] to row m only."""
    prob = inputs.make_dense(6, 200, 512, seed=12)
    base = lib.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    m, kb = 4, 2
    sa2 = prob.sa.clone()
    sa2[kb, m] *= 2
    moved = lib.gemm_dense(prob.a, sa2, prob.b, prob.sb, prob.M, prob.N, prob.K)
    A, B = torch_decode(prob.a.numpy()), torch_decode(prob.b.numpy())
    ks = slice(kb * 128, (kb + 1) * 128)
    partial = A[m, ks] @ B[:, ks].T
    col_scale = np.repeat(prob.sb[:, kb].numpy().astype(np.float64), 128)[:prob.N]
    delta = float(prob.sa[kb, m]) * col_scale * partial
    assert np.allclose(moved[m] - base[m], delta, rtol=1e-12, atol=1e-9)
    others = [i for i in range(prob.M) if i != m]
    assert np.array_equal(moved[others], base[others])
    # and in sb: doubling sb[nb,kb] only moves columns of block nb
    sb2 = prob.sb.clone()
    sb2[1, kb] *= 2
    moved_b = lib.gemm_dense(prob.a, prob.sa, prob.b, sb2, prob.M, prob.N, prob.K)
    assert np.array_equal(moved_b[:, :128], base[:, :128])
    assert not np.array_equal(moved_b[:, 128:], base[:, 128:])


def pin_contiguous_closed_form(lib):
    """A = 1, expert e's B = e + 1, unit scales: D[m, n] = K (e + 1); padding rows NaN."""
    G, N, K = 3, 48, 256
    counts = [5, 0, 130]
    padded = [math.ceil(c / 128) * 128 for c in counts]
    M_sum = sum(padded)
    a = np.repeat(encode([1.0]), M_sum * K).reshape(M_sum, K)
    b = np.stack([np.repeat(encode([float(e + 1)]), N * K).reshape(N, K) for e in range(G)])
    mi = np.full(M_sum, -1, np.int32)
    row = 0
    for e, (c, p) in enumerate(zip(counts, padded)):
        mi[row:row + c] = e
        row += p
    sa = col_major(np.ones((M_sum, K // 128), np.float32))
    sb = np.ones((G, 1, K // 128), np.float32)
    D = lib.gemm_contiguous(a, sa, b, sb, mi, G, M_sum, N, K)
    for m in range(M_sum):
        if mi[m] < 0:
            assert np.isnan(D[m]).all()
        else:
            assert np.array_equal(D[m], np.full(N, float(K * (mi[m] + 1))))


def pin_contiguous_equals_per_expert_dense(lib):
    prob = inputs.make_contiguous(3, 136, 256, seed=13, counts=[100, 1, 257])
    D = lib.gemm_contiguous(prob.a, prob.sa, prob.b, prob.sb, prob.m_indices, prob.num_groups,
                            prob.M_sum, prob.N, prob.K)
    row = 0
    for e, c in enumerate(prob.counts):
        rows = slice(row, row + c)
        sa_e = prob.sa[:, rows].contiguous()
        ref = lib.gemm_dense(prob.a[rows], sa_e, prob.b[e], prob.sb[e], c, prob.N, prob.K)
        assert np.array_equal(D[rows], ref)
        row += math.ceil(c / 128) * 128


def pin_masked_closed_form_and_untouched(lib):
    """A = 1, group g's B = g + 1: D[g, m, n] = K (g + 1) for m < masked_m[g]; NaN beyond."""
    G, Mmax, N, K = 4, 10, 16, 128
    masked_m = np.array([0, 10, 3, 7], np.int32)
    a = np.repeat(encode([1.0]), G * Mmax * K).reshape(G, Mmax, K)
    b = np.stack([np.repeat(encode([float(g + 1)]), N * K).reshape(N, K) for g in range(G)])
    ld = inputs.tma_aligned_size(Mmax, 4)
    sa = np.ones((G, 1, ld), np.float32)
    sb = np.ones((G, 1, 1), np.float32)
    D = lib.gemm_masked(a, sa, b, sb, masked_m, G, Mmax, N, K)
    for g in range(G):
        assert np.array_equal(D[g, :masked_m[g]], np.full((masked_m[g], N), float(K * (g + 1))))
        assert np.isnan(D[g, masked_m[g]:]).all()


def pin_masked_equals_per_group_dense(lib):
    prob = inputs.make_masked(3, 40, 136, 256, seed=14, masked_m=[40, 0, 17])
    D = lib.gemm_masked(prob.a, prob.sa, prob.b, prob.sb, prob.masked_m, prob.G, prob.M_max,
                        prob.N, prob.K)
    for g in range(prob.G):
        mm = int(prob.masked_m[g])
        ref = lib.gemm_dense(prob.a[g], prob.sa[g], prob.b[g], prob.sb[g], prob.M_max, prob.N,
                             prob.K)
        assert np.array_equal(D[g, :mm], ref[:mm])


def pin_sampled_equal_full(lib):
    prob = inputs.make_dense(50, 300, 256, seed=15)
    full = lib.gemm_dense(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, prob.M, 200)
    cols = rng.integers(0, prob.N, 200)
    samp = lib.gemm_dense_sampled(prob.a, prob.sa, prob.b, prob.sb, prob.M, prob.N, prob.K,
                                  rows, cols)
    assert np.array_equal(samp, full[rows, cols])
    cprob = inputs.make_contiguous(2, 136, 256, seed=16, counts=[3, 140])
    cfull = lib.gemm_contiguous(cprob.a, cprob.sa, cprob.b, cprob.sb, cprob.m_indices, 2,
                                cprob.M_sum, cprob.N, cprob.K)
    rows = rng.integers(0, cprob.M_sum, 200)
    cols = rng.integers(0, cprob.N, 200)
    csamp = lib.gemm_contiguous_sampled(cprob.a, cprob.sa, cprob.b, cprob.sb, cprob.m_indices,
                                        2, cprob.M_sum, cprob.N, cprob.K, rows, cols)
    assert np.array_equal(np.isnan(csamp), np.isnan(cfull[rows, cols]))
    ok = ~np.isnan(csamp)
    assert np.array_equal(csamp[ok], cfull[rows, cols][ok])
    mprob = inputs.make_masked(3, 20, 136, 128, seed=17, masked_m=[20, 5, 0])
    mfull = lib.gemm_masked(mprob.a, mprob.sa, mprob.b, mprob.sb, mprob.masked_m, 3, 20,
                            mprob.N, mprob.K)
    groups = rng.integers(0, 3, 200)
    rows = rng.integers(0, 20, 200)
    cols = rng.integers(0, mprob.N, 200)
    msamp = lib.gemm_masked_sampled(mprob.a, mprob.sa, mprob.b, mprob.sb, mprob.masked_m, 3,
                                    20, mprob.N, mprob.K, groups, rows, cols)
    ref = mfull[groups, rows, cols]
    assert np.array_equal(np.isnan(msamp), np.isnan(ref))
    assert np.array_equal(msamp[~np.isnan(ref)], ref[~np.isnan(ref)])


def pin_per_tensor_equals_scaled_library_matmul(lib):
    """Per-tensor scaling is the special case of equal block scales: it must
    equal scale_a * scale_b * (decoded A) @ (decoded B)^T, the partials being
    exact in FP64 (any order)."""
    rng = np.random.default_rng(11)
    M, N, K = 37, 45, 640
    a = random_finite_bytes(rng, (M, K))
    b = random_finite_bytes(rng, (N, K))
    sa_, sb_ = 0.0078125 * 3, 1.0 / 448.0
    got = oracle.gemm_per_tensor(a, sa_, b, sb_, M, N, K, lib=lib)
    ref = (torch_decode(a) @ torch_decode(b).T) * (np.float64(np.float32(sa_)) * np.float64(np.float32(sb_)))
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-9 * np.abs(ref).max())


def pin_quantize_exact_blocks(lib):
    """Blocks whose amax is 448 * 2^j hold values dec(code) * 2^j: the scale
    must be exactly 2^j and every code must come back unchanged; a zero
    block gets the amax floor (1e-4 / 448 in FP32) and zero codes; the block
    maximum lands on +-448."""
    rng = np.random.default_rng(5)
    M, K = 6, 384
    codes = random_finite_bytes(rng, (M, K))
    codes[codes == 0x80] = 0x00              # -0 encodes as +0 after scaling
    x = np.empty((M, K), dtype=np.float32)
    exps = [-3, 0, 5]
    for kb in range(K // 128):
        blk = codes[:, kb * 128:(kb + 1) * 128]
        blk[:, 7] = 0x7E                     # each row's amax is exactly 448
        x[:, kb * 128:(kb + 1) * 128] = torch_decode(blk) * 2.0 ** exps[kb]
    x[5, 128:256] = 0.0
    q, sa = lib.quantize_1x128(x, M, K)
    expect_q = codes.copy()
    expect_q[5, 128:256] = 0
    assert np.array_equal(q, expect_q)
    for kb in range(K // 128):
        want = np.full(M, np.float32(2.0 ** exps[kb]), dtype=np.float32)
        if kb == 1:
            want[5] = np.float32(np.float32(1e-4) / np.float32(448.0))
        assert np.array_equal(sa[kb, :M], want), kb


def pin_quantize_ties_to_even(lib):
    """With a unit scale (amax 448), values halfway between two E4M3 values
    go to the even mantissa: 1.0625 -> 1.0 (0x38), 1.1875 -> 1.25 (0x3A),
    -1.0625 -> -1.0 (0xB8); 0.0009765625 (half of the smallest subnormal)
    -> 0."""
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, :5] = [448.0, 1.0625, 1.1875, -1.0625, 0.0009765625]
    q, sa = lib.quantize_1x128(x, 1, 128)
    assert sa[0, 0] == 1.0
    assert q[0, :5].tolist() == [0x7E, 0x38, 0x3A, 0xB8, 0x00]


def pin_quantize_unit_scale_equals_library_cast(lib):
    """With a unit scale the quantiser is a plain round-to-nearest-even cast,
    which torch's float8_e4m3fn conversion (a library routine) performs."""
    rng = np.random.default_rng(9)
    x = rng.uniform(-448, 448, size=(4, 256)).astype(np.float32)
    x[:, 0] = 448.0
    x[:, 128] = -448.0
    q, sa = lib.quantize_1x128(x, 4, 256)
    assert np.all(sa[:, :4] == 1.0)
    ref = torch.from_numpy(x).to(E4M3).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def pin_quantize_round_trip_bound(lib):
    """For N(0,1) data: dec(q) * s is within half an E4M3 step of x (relative
    2^-4 for normal values, absolute 2^-10 * s below), signs agree, and the
    scale is amax / 448 to within one FP32 rounding."""
    rng = np.random.default_rng(13)
    M, K = 33, 512
    x = rng.standard_normal((M, K)).astype(np.float32)
    q, sa = lib.quantize_1x128(x, M, K)
    s = np.repeat(sa[:, :M].T, 128, axis=1).astype(np.float64)
    back = torch_decode(q) * s
    err = np.abs(back - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert np.all((np.sign(back) == np.sign(x)) | (back == 0))
    amax = np.abs(x.reshape(M, K // 128, 128)).max(axis=2)
    assert np.allclose(sa[:, :M].T, amax / 448.0, rtol=2.0 ** -23, atol=0)


PINS = [
    pin_decode_table_matches_torch,
    pin_decode_golden_range,
    pin_small_integer_exact,
    pin_scale_indexing_closed_form,
    pin_sign_and_per_k_products,
    pin_brute_force_tiny,
    pin_unit_scales_equal_library_matmul,
    pin_scaled_matches_expanded_matmul,
    pin_linearity_in_scale_block,
    pin_contiguous_closed_form,
    pin_contiguous_equals_per_expert_dense,
    pin_masked_closed_form_and_untouched,
    pin_masked_equals_per_group_dense,
    pin_sampled_equal_full,
    pin_per_tensor_equals_scaled_library_matmul,
    pin_quantize_exact_blocks,
    pin_quantize_ties_to_even,
    pin_quantize_unit_scale_equals_library_cast,
    pin_quantize_round_trip_bound,
]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_oracle_rejects_bad_arguments(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.gemm_masked(np.zeros((1, 4, 128), np.uint8), np.ones((1, 1, 4), np.float32),
                               np.zeros((1, 8, 128), np.uint8), np.ones((1, 1, 1), np.float32),
                               np.array([5], np.int32), 1, 4, 8, 128)
    with pytest.raises(ValueError):
        oracle_lib.gemm_contiguous(np.zeros((128, 128), np.uint8), np.ones((1, 128), np.float32),
                                   np.zeros((1, 8, 128), np.uint8), np.ones((1, 1, 1), np.float32),
                                   np.full(128, 3, np.int32), 1, 128, 8, 128)


# ---------------------------------------------------------------------------
# Mutation check: each plausible mistake planted in a copy of oracle.c must
# fail at least one pin.

MUTANTS = {
    "mantissa_sign": ("8.0 + mantissa", "8.0 - mantissa"),
    "exponent_bias": ("exponent - 10", "exponent - 9"),
    "subnormal_scale": ("ldexp((double)mantissa, -9)", "ldexp((double)mantissa, -10)"),
    "sign_dropped": ("return sign ? -magnitude : magnitude;", "return magnitude;"),
    "nan_code": ("exponent == 15 && mantissa == 7", "exponent == 15 && mantissa == 6"),
    "sb_not_per_kb": ("(double)sb_row[kb]", "(double)sb_row[0]"),
    "sa_row_major": ("sa_col[(long)kb * ld_sa]", "sa_col[kb]"),
    "sb_block_index": ("(long)(n / ORACLE_BLOCK) * nkb, K);\n    return 0;\n}\n\n/* Dense, at",
                       "(long)(n % ORACLE_BLOCK) * nkb, K);\n    return 0;\n}\n\n/* Dense, at"),
    "block_partial_not_reset": ("double partial = 0.0;\n", "static double partial = 0.0;\n"),
    "dropped_last_k": ("for (int k = k0; k < k1; ++k)", "for (int k = k0; k < k1 - 1; ++k)"),
    "transposed_operand_b": ("dec[b_row[k]]", "dec[a_row[k]]"),
    "contiguous_expert_offset": ("const uint8_t *Be = B + (long)e * N * K;",
                                 "const uint8_t *Be = B;"),
    "masked_sa_group_offset": ("const float *sag = sa + (long)g * nkb * ld_sa;",
                               "const float *sag = sa;"),
    "masked_row_bound": ("if (m >= masked_m[g]) {\n                for",
                         "if (m > masked_m[g]) {\n                for"),
    "quant_ties_away": ("(err == best_err && (code & 1) == 0 && (best & 1) == 1)",
                        "(err == best_err && fabs(d) > fabs(dec[best]))"),
    "quant_no_floor": ("if (amax < floor_amax)\n                amax = floor_amax;",
                       "if (amax < 0.0f)\n                amax = floor_amax;"),
    "quant_amax_signed": ("float a = fabsf(xb[k]);", "float a = xb[k];"),
    "quant_scale_row_major": ("sa[(long)kb * ld_sa + m] = s;", "sa[(long)m * nkb + kb] = s;"),
    "quant_scale_448_off": ("const float e4m3_max = 448.0f;", "const float e4m3_max = 440.0f;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-w",
                           "-o", str(so_path), str(c_path), "-lm"])
    lib = oracle.OracleLib(str(so_path))
    failures = []
    for pin in PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"
