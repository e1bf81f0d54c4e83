"""Pins of the affine (asymmetric) 4-bit oracle and of the bias + ReLU
epilogue against what the pages and the mathematics fix: a worked example,
exact rational arithmetic of every rounding in the page's order, zero coded
exactly, the round-trip bound, exhaustive bytes, the per-group algebra of
the matmul and hand-computed bounds.  None of these tests touches the GPU."""

from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact_fp import rn16, rn32


def _exact_affine_group(ws):
    """(s, z, [q]) of one group by exact rational arithmetic, following the
    inference-engine page's step 2 with the stated fp32/fp16 roundings."""
    vals = [Fraction(float(v)) for v in ws]
    mn, mx = min(vals), max(vals)
    d = rn32(mx - mn)
    s = rn16(rn32(d / 15))
    if s == 0:
        return 0.0, 0, [0] * len(vals)
    z = int(min(15, max(0, round(rn32(-mn / s)))))
    q = [int(min(15, max(0, round(rn32(rn32(v / s) + z))))) for v in vals]
    return float(s), z, q


def test_worked_example():
    """w = [-1, 0, 2, 14], group 4: min -1, max 14, scale 15/15 = 1, zero point
    round(1/1) = 1, codes round(w + 1) = [0, 1, 3, 15]; element 2j in the low
    nibble gives bytes 0x10, 0xF3; (q - z) s = w exactly."""
    w = np.array([[-1.0, 0.0, 2.0, 14.0]], dtype=np.float32)
    packed, scales, zeros, K = oracle.quantize_uint4_affine(w, 4)
    assert K == 4 and float(scales[0, 0]) == 1.0 and int(zeros[0, 0]) == 1
    assert packed.tolist() == [[0x10, 0xF3]]
    assert oracle.unpack_uint4(packed, 4).tolist() == [[0, 1, 3, 15]]
    assert np.array_equal(oracle.dequantize_uint4_affine(packed, scales, zeros, 4, 4), w)


@pytest.mark.parametrize("seed", range(4))
def test_codes_match_exact_arithmetic(seed):
    """Scales, zero points and codes equal the exact-rational evaluation of
    the page's formulas on random groups, including groups of one sign and
    values placed on half-integer quotients."""
    rng = np.random.default_rng(seed)
    N, group = 24, 8
    w = rng.normal(size=(N, 4 * group)).astype(np.float32)
    w[::3] = np.abs(w[::3])                       # all-positive groups: z clips to 0
    w[1::5] = -np.abs(w[1::5])                    # all-negative groups: z clips to 15
    # Half-integer quotients: group values k/2 with range 15 -> scale 1.
    w[2, :group] = np.array([-2.0, 13.0, 0.5, 1.5, 2.5, -1.5, 7.5, 12.5], dtype=np.float32)
    packed, scales, zeros, K = oracle.quantize_uint4_affine(w, group)
    q = oracle.unpack_uint4(packed, K)
    for n in range(N):
        for g in range(4):
            s, z, qs = _exact_affine_group(w[n, g * group:(g + 1) * group])
            assert float(scales[n, g]) == s, (n, g)
            assert int(zeros[n, g]) == z, (n, g)
            assert q[n, g * group:(g + 1) * group].tolist() == qs, (n, g)
    # Row 2, group 0: s = 1, z = 2, and the ties round half to even.
    assert float(scales[2, 0]) == 1.0 and int(zeros[2, 0]) == 2
    assert q[2, :8].tolist() == [0, 15, 2, 4, 4, 0, 10, 14]


def test_zero_is_coded_exactly_when_the_group_spans_it():
    """The LM page: the zero point aligns 0.0 with an exact integer, so zero
    is represented without error: every w == 0 in a group with min <= 0 <= max
    dequantizes to exactly 0."""
    rng = np.random.default_rng(7)
    w = rng.normal(size=(64, 256)).astype(np.float32)
    w[rng.random(w.shape) < 0.2] = 0.0
    packed, scales, zeros, K = oracle.quantize_uint4_affine(w, 32)
    w_hat = oracle.dequantize_uint4_affine(packed, scales, zeros, K, 32)
    assert (w == 0).sum() > 1000
    assert (w_hat[w == 0] == 0.0).all()


def test_round_trip_error_bound():
    """For groups with min <= 0 <= max: |w_hat - w| <= s (1/2 + 15 * 2^-11),
    the half step plus the fp16 rounding of the scale at the top code."""
    rng = np.random.default_rng(3)
    w = (rng.standard_t(3, size=(128, 1000)) * 0.02).astype(np.float32)
    for group in (32, 64, 128, 100):
        packed, scales, zeros, K = oracle.quantize_uint4_affine(w, group)
        w_hat = oracle.dequantize_uint4_affine(packed, scales, zeros, K, group)
        s = np.repeat(scales.astype(np.float64), group, axis=1)[:, :K]
        mn, mx = oracle.group_minmax(w, group)
        spans = np.repeat((mn <= 0) & (mx >= 0), group, axis=1)[:, :K]
        err = np.abs(w_hat - w.astype(np.float64))
        assert (err[spans] <= s[spans] * (0.5 + 15 * 2.0 ** -11) + 1e-12).all()


def test_constant_and_zero_groups_get_scale_zero():
    w = np.zeros((3, 12), dtype=np.float32)
    w[1, :4] = 0.25                                # constant non-zero group
    w[2, 4:8] = [1.0, 1.0, 1.0, 2.0]
    packed, scales, zeros, K = oracle.quantize_uint4_affine(w, 4)
    assert float(scales[0, 0]) == 0.0 and float(scales[1, 0]) == 0.0
    assert int(zeros[1, 0]) == 0 and (oracle.unpack_uint4(packed, K)[1, :4] == 0).all()
    w_hat = oracle.dequantize_uint4_affine(packed, scales, zeros, K, 4)
    assert (w_hat[:2] == 0.0).all()
    s = float(scales[2, 1])                        # fp16(1/15), z = clip(rint(-1/s)) = 0
    assert s == float(np.float16(np.float32(1.0) / np.float32(15.0))) and int(zeros[2, 1]) == 0


def test_partial_last_group_and_odd_k():
    rng = np.random.default_rng(5)
    w = rng.normal(size=(4, 37)).astype(np.float32)
    packed, scales, zeros, K = oracle.quantize_uint4_affine(w, 16)
    assert packed.shape == (4, 19) and scales.shape == (4, 3) and zeros.shape == (4, 3)
    assert (packed[:, -1] >> 4 == 0).all()          # the pad nibble
    s, z, qs = _exact_affine_group(w[0, 32:37])
    assert float(scales[0, 2]) == s and int(zeros[0, 2]) == z
    assert oracle.unpack_uint4(packed, K)[0, 32:].tolist() == qs


def test_unpack_exhaustive_and_pack_identity():
    b = np.arange(256, dtype=np.uint8)[None, :]
    u = oracle.unpack_uint4(b, 512)
    assert u[0, 0::2].tolist() == [v & 15 for v in range(256)]
    assert u[0, 1::2].tolist() == [v >> 4 for v in range(256)]
    assert np.array_equal(oracle.pack_unsigned(u), b)


def test_matmul_ref_equals_the_per_group_form():
    """x @ ((q - z) s)^T equals the page's per-group order, s (x.q - z sum x),
    in fp64 on a small case with several groups and a partial last group."""
    rng = np.random.default_rng(11)
    w = rng.normal(size=(9, 70)).astype(np.float32)
    x = rng.normal(size=(5, 70))
    packed, scales, zeros, K = oracle.quantize_uint4_affine(w, 16)
    a = oracle.uint4_affine_matmul_ref(x, packed, scales, zeros, K, 16)
    b = oracle.uint4_affine_matmul_groupwise(x, packed, scales, zeros, K, 16)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    assert (zeros > 0).any()


def test_matmul_row_sums_and_one_hot():
    """Codes z + 1 everywhere with scale 1: y is the row sum of x; a one-hot
    x selects a column of w_hat exactly."""
    K, group = 32, 16
    zeros = np.array([[3, 9], [0, 14]], dtype=np.uint8)
    q = np.repeat(zeros + 1, group, axis=1)
    packed = oracle.pack_unsigned(q)
    scales = np.ones((2, 2), dtype=np.float16)
    x = np.arange(2 * K, dtype=np.float64).reshape(2, K) - 20
    y = oracle.uint4_affine_matmul_ref(x, packed, scales, zeros, K, group)
    assert np.array_equal(y, np.repeat(x.sum(1)[:, None], 2, 1))
    w_hat = oracle.dequantize_uint4_affine(packed, scales, zeros, K, group)
    e = np.zeros((1, K))
    e[0, 20] = 1.0
    assert np.array_equal(oracle.uint4_affine_matmul_ref(e, packed, scales, zeros, K, group)[0],
                          w_hat[:, 20])


def test_error_bound_by_hand():
    """Codes [0, 15, 7, 3] with z = 7, s = 0.5: w_hat = [-3.5, 4, 0, -2];
    x = [2, -1, 5, 3]: sum |x||w_hat| = 7 + 4 + 0 + 6 = 17 (x.w_hat = -17)."""
    packed = oracle.pack_unsigned(np.array([[0, 15, 7, 3]], dtype=np.uint8))
    b = oracle.matmul_error_bound_affine(np.array([[2.0, -1.0, 5.0, 3.0]]), packed,
                                         np.array([[0.5]], np.float16),
                                         np.array([[7]], np.uint8), 4, 4, 1.0)
    assert b[0, 0] == 17.0


def test_linear_epilogue_by_hand():
    """The engine page's layer: x @ W_dq^T + bias, then ReLU."""
    y = np.array([[-1.0, 2.0, 0.25], [3.0, -4.0, 0.0]])
    b = np.array([0.5, -3.0, -0.25])
    assert oracle.linear_epilogue_ref(y, b, relu=False).tolist() == [[-0.5, -1.0, 0.0], [3.5, -7.0, -0.25]]
    assert oracle.linear_epilogue_ref(y, b, relu=True).tolist() == [[0.0, 0.0, 0.0], [3.5, 0.0, 0.0]]
    assert oracle.linear_epilogue_ref(y, None, relu=True).tolist() == [[0.0, 2.0, 0.25], [3.0, 0.0, 0.0]]
    tol = oracle.epilogue_error_bound(np.zeros((2, 3)), y, b)
    assert np.array_equal(tol, 2.0 ** -24 * np.abs(y + b[None, :]))
