"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each check is chosen so that a plausible slip in the oracle (a swapped nibble
order, offset-binary instead of two's complement, a reciprocal instead of a
division, round-half-away instead of half-even, a dropped partial group, a
transposed operand, a missing scale) fails at least one of them.  None of
these tests touches the GPU library.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from workloads import tiny_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


from exact_fp import FP16, FP32, round_to_format  # noqa: E402


def exact_scale(m: float) -> float:
    """fp16(fp32(m / 7)) by exact rational arithmetic."""
    t = round_to_format(Fraction(float(m)) / 7, FP32)
    s = round_to_format(t, FP16)
    return float("inf") if abs(s) > 10**300 else float(s)


def exact_code(w: float, s: float) -> int:
    """clip(rint(fp32(w / s)), -8, 7), 0 when s == 0, by exact arithmetic."""
    if s == 0.0:
        return 0
    if s == float("inf"):
        return 0
    t = round_to_format(Fraction(float(w)) / Fraction(float(s)), FP32)
    return int(min(7, max(-8, round(t))))


# ---------------------------------------------------------------------------
# The drill page's visible tests, verbatim in behaviour.
# ---------------------------------------------------------------------------
def test_drill_nibble_layout_is_even_low_odd_high():
    g = _load("drill_visible_examples.json")["nibble_layout"]
    w = np.array(g["w"], dtype=np.float32)
    packed, scale, K = oracle.quantize_int4(w, g["group"])
    assert K == 4
    assert scale.dtype == np.float16 and scale.shape == (1, 1)
    assert float(scale[0, 0]) == g["scale"]
    assert [int(b) for b in packed[0]] == [int(h, 16) for h in g["packed_hex"]]
    # The page on offset-binary packing (+8, first value low) would give
    # different bytes; the drill's bytes rule it out.
    offset_binary = [((1 + 8) | ((-1 + 8) << 4)), ((7 + 8) | ((-7 + 8) << 4))]
    assert offset_binary == [0x79, 0x1F]
    assert [int(b) for b in packed[0]] != offset_binary


def test_drill_round_trip_error_stays_within_half_a_step():
    rng = np.random.default_rng(0)
    w = rng.normal(size=(8, 256)).astype(np.float32)
    packed, scale, K = oracle.quantize_int4(w, 128)
    q = np.asarray(oracle.unpack_int4(packed, K), dtype=np.float32)
    s = np.repeat(np.asarray(scale, np.float32), 128, axis=1)[:, :K]
    err = np.abs(q * s - w)
    assert (err <= s * 0.5 + 1e-3 * s + 1e-6).all()


def test_pure_python_page_roundtrip_thresholds():
    """Pure-Python quantizer page, 'Running and Testing It': 512x512 N(0,1),
    block 64.  Its max-error bound (< 0.5) holds.  Its printed MSE bound
    (< 0.01) is not met by its own scheme at block 64 (about 0.0115), so the
    MSE is pinned instead to the uniform-quantizer closed form: rounding
    error spread evenly over one step s has mean square s^2 / 12."""
    w = np.random.default_rng(1234).normal(size=(512, 512)).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 64)
    w_hat = oracle.dequantize_int4(packed, scales, K, 64)
    diff = w.astype(np.float64) - w_hat
    assert np.max(np.abs(diff)) < 0.5
    s = np.repeat(scales.astype(np.float64), 64, axis=1)
    assert (np.abs(diff) <= 0.5 * s * (1 + 2.0 ** -10)).all()
    predicted = np.mean(s ** 2) / 12
    assert abs(np.mean(diff ** 2) - predicted) < 0.05 * predicted


# ---------------------------------------------------------------------------
# Unpack and sign extension: exhaustive over all 256 byte values.
# ---------------------------------------------------------------------------
def test_unpack_exhaustive_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    got = oracle.unpack_int4(b.reshape(1, 256), 512)[0]
    # Independent route: an arithmetic right shift of the nibble placed in the
    # top of an int8 sign-extends it.
    lo = ((b << 4).astype(np.uint8).view(np.int8) >> 4).astype(np.int8)
    hi = (b.view(np.int8) >> 4).astype(np.int8)
    assert np.array_equal(got[0::2], lo)
    assert np.array_equal(got[1::2], hi)
    assert got.min() == -8 and got.max() == 7


@pytest.mark.parametrize("byte, pair", [(0x88, (-8, -8)), (0x80, (0, -8)), (0x08, (-8, 0)),
                                        (0xF1, (1, -1)), (0x97, (7, -7)), (0x00, (0, 0)),
                                        (0x7F, (-1, 7))])
def test_unpack_named_bytes(byte, pair):
    got = oracle.unpack_int4(np.array([[byte]], dtype=np.uint8), 2)[0]
    assert tuple(int(v) for v in got) == pair


@pytest.mark.parametrize("K", [1, 2, 3, 255, 256])
def test_pack_unpack_is_identity_on_all_bytes(K):
    rng = np.random.default_rng(K)
    Kp = oracle.packed_cols(K)
    packed = rng.integers(0, 256, size=(17, Kp), dtype=np.uint8)
    if K % 2:                                   # the pad nibble is zero
        packed[:, -1] &= 0x0F
    q = oracle.unpack_int4(packed, K)
    assert q.shape == (17, K) and q.dtype == np.int8
    assert np.array_equal(oracle.pack_nibbles(q), packed)


# ---------------------------------------------------------------------------
# Scales and codes against exact rational arithmetic.
# ---------------------------------------------------------------------------
def _special_groups():
    # Each row is one group of 8; the comments give the point of each row.
    t = 2.0 ** -24
    return np.array([
        [7.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -3.5],        # s = 1: half-even ties
        [0.0] * 8,                                             # zero group -> s = 0
        [7 * 2.0 ** -25, 0, 0, 0, 0, 0, 0, 0],                 # m/7 is the tie 2^-25 -> s = 0
        [7 * 1.49 * t, -7 * 1.49 * t, 0.5 * t, 0, 0, 0, 0, 0],  # subnormal s = 2^-24, clamps to 7/-8
        [1e-5, -3e-6, 2e-6, 0, 0, 0, 0, 0],                    # subnormal scale region
        [-0.0, 0.0, -0.0, 0, 0, 0, 0, 0],                      # signed zeros
        [3.0, -3.0, 1.0, 2.0, -1.5, 0.75, 0.2, -0.1],          # s = fp16(3/7): inexact
        [458000.0, -1.0, 1.0, 0, 0, 0, 0, 0],                  # large but finite scale
    ], dtype=np.float32)


def test_scales_and_codes_match_exact_arithmetic_special_cases():
    w = _special_groups()
    packed, scales, K = oracle.quantize_int4(w, 8)
    q = oracle.unpack_int4(packed, K)
    for n in range(w.shape[0]):
        m = float(np.max(np.abs(w[n])))
        s = exact_scale(m)
        assert float(scales[n, 0]) == s, (n, float(scales[n, 0]), s)
        for k in range(8):
            assert int(q[n, k]) == exact_code(float(w[n, k]), s), (n, k)
    assert [int(v) for v in q[0]] == [7, 2, 4, -2, 0, 0, 2, -4]
    assert float(scales[1, 0]) == 0.0 and not packed[1].any()
    assert float(scales[2, 0]) == 0.0
    assert float(scales[3, 0]) == 2.0 ** -24 and list(q[3, :3]) == [7, -8, 0]


def test_scales_and_codes_match_exact_arithmetic_random():
    rng = np.random.default_rng(7)
    mags = 10.0 ** rng.uniform(-7, 4, size=(64, 1))
    w = (rng.standard_t(3, size=(64, 16)) * mags).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 16)
    q = oracle.unpack_int4(packed, K)
    for n in range(64):
        s = exact_scale(float(np.max(np.abs(w[n]))))
        assert float(scales[n, 0]) == s
        for k in range(16):
            assert int(q[n, k]) == exact_code(float(w[n, k]), s)


def test_division_is_not_a_reciprocal_multiply():
    """w / s and w * (1/s) differ in the last fp32 bit for some inputs, and
    that bit can decide a half-even tie; the oracle must follow the division."""
    rng = np.random.default_rng(11)
    s = np.float32(rng.uniform(0.01, 1.0, size=20000)).astype(np.float16).astype(np.float32)
    w = (s * rng.uniform(-7.4, 7.4, size=20000)).astype(np.float32)
    div = (w / s).astype(np.float32)
    rec = (w * (np.float32(1.0) / s)).astype(np.float32)
    assert (div != rec).any()          # the two routes really differ somewhere
    W = w.reshape(-1, 1).repeat(2, axis=1)
    W[:, 1] = 0
    # Put each w in a group whose absmax is 7*s so that the stored scale is s.
    for i in range(0, 2000):
        grp = np.array([[w[i], 7 * s[i]]], dtype=np.float32)
        packed, scales, K = oracle.quantize_int4(grp, 2)
        if float(scales[0, 0]) != float(s[i]):
            continue
        got = int(oracle.unpack_int4(packed, 2)[0, 0])
        assert got == exact_code(float(w[i]), float(s[i]))


def test_partial_last_group_and_odd_K():
    case = tiny_case()
    w, group = case["w"], case["group"]
    packed, scales, K = oracle.quantize_int4(w, group)
    assert K == 259 and packed.shape == (16, 130) and scales.shape == (16, 3)
    # The last group holds only columns 256..258.
    for n in range(16):
        assert float(scales[n, 2]) == exact_scale(float(np.abs(w[n, 256:259]).max()))
        assert float(scales[n, 0]) == exact_scale(float(np.abs(w[n, 0:128]).max()))
    # The pad nibble (high nibble of the last byte) is zero.
    assert not (packed[:, -1] >> 4).any()
    # Row 3, columns 128..255 is the all-zero group.
    assert float(scales[3, 1]) == 0.0
    assert not packed[3, 64:128].any()


def test_idempotent_requantization():
    """quantize(dequantize(quantize(w))) == quantize(w) when no scale is zero
    or subnormal: 7*s is exact, so the recomputed scale is s and q*s/s = q."""
    rng = np.random.default_rng(5)
    w = (rng.normal(size=(32, 200)) * 0.02).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 64)
    assert (scales.astype(np.float32) >= 2.0 ** -14).all()
    w_hat = oracle.dequantize_int4(packed, scales, K, 64).astype(np.float32)
    p2, s2, _ = oracle.quantize_int4(w_hat, 64)
    assert np.array_equal(p2, packed)
    assert np.array_equal(s2.view(np.uint16), scales.view(np.uint16))


def test_fp16_and_fp32_inputs_agree():
    rng = np.random.default_rng(9)
    w16 = rng.normal(size=(8, 96)).astype(np.float16)
    a = oracle.quantize_int4(w16, 32)
    b = oracle.quantize_int4(w16.astype(np.float32), 32)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_scale_overflow_gives_zero_codes():
    """absmax >= 7 * 65520 rounds the fp16 scale to +inf; w / inf = 0."""
    w = np.array([[7 * 65520.0, 1.0, -5.0, 0.0]], dtype=np.float32)
    packed, scales, K = oracle.quantize_int4(w, 4)
    assert np.isinf(scales[0, 0])
    assert not packed.any()


# ---------------------------------------------------------------------------
# Storage size: the closed form, and the language-model page's table.
# ---------------------------------------------------------------------------
def test_storage_size_closed_form():
    st = oracle.storage_bytes(16, 259, 128)
    assert st == {"packed": 16 * 130, "scales": 2 * 16 * 3, "total": 2080 + 96}
    case = tiny_case()
    packed, scales, K = oracle.quantize_int4(case["w"], 128)
    assert packed.nbytes == st["packed"] and scales.nbytes == st["scales"]


def test_storage_size_reproduces_lm_quantization_table():
    t = _load("lm_quantization_sizes.json")
    shapes = [tuple(s) for s in t["quantized_linears_per_block"]] * t["blocks"]
    n_weights = sum(a * b for a, b in shapes)
    fp32 = 4 * n_weights
    assert round(fp32 / 1e6, 2) == t["fp32_mb"]
    assert round(n_weights / 1e6, 2) == t["int8_mb"]
    for g, key, ov, comp in ((64, "int4_g64_mb", "scale_overhead_g64_mb", "compression_g64"),
                             (32, "int4_g32_mb", "scale_overhead_g32_mb", "compression_g32")):
        # The page's numbers use 4-byte scales; groups run along each row.
        st = [oracle.storage_bytes(out, inp, g, scale_bytes=4) for (inp, out) in shapes]
        total = sum(s["total"] for s in st)
        scales = sum(s["scales"] for s in st)
        assert round(total / 1e6, 2) == t[key]
        assert round(scales / 1e6, 2) == t[ov]
        assert round(fp32 / total, 2) == t[comp]
        # With the drill page's fp16 scales the same model is smaller.
        st16 = sum(oracle.storage_bytes(out, inp, g)["total"] for (inp, out) in shapes)
        assert st16 < total


# ---------------------------------------------------------------------------
# The matmul.
# ---------------------------------------------------------------------------
def test_matmul_ref_equals_groupwise_loop_tiny():
    case = tiny_case()
    packed, scales, K = oracle.quantize_int4(case["w"], 128)
    y1 = oracle.int4_matmul_ref(case["x"], packed, scales, K, 128)
    y2 = oracle.int4_matmul_groupwise(case["x"], packed, scales, K, 128)
    assert y1.shape == (4, 16)
    np.testing.assert_allclose(y1, y2, rtol=1e-13, atol=1e-13)


def test_matmul_against_direct_double_sum():
    """Brute force with Python floats over the exact dequantized weights."""
    rng = np.random.default_rng(3)
    w = rng.normal(size=(5, 37)).astype(np.float32)
    x = rng.normal(size=(3, 37)).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 8)
    q = oracle.unpack_int4(packed, K)
    y = oracle.int4_matmul_ref(x, packed, scales, K, 8)
    for m in range(3):
        for n in range(5):
            acc = Fraction(0)
            for k in range(37):
                acc += Fraction(float(x[m, k])) * int(q[n, k]) * Fraction(float(scales[n, k // 8]))
            assert abs(float(acc) - y[m, n]) <= 1e-12 * max(1.0, abs(float(acc)))


def test_matmul_hand_made_bytes_row_sums():
    """All bytes 0x11 (q = 1) with scale 1: y is the row sums of x."""
    rng = np.random.default_rng(4)
    x = rng.normal(size=(6, 50)).astype(np.float32)
    packed = np.full((9, 25), 0x11, dtype=np.uint8)
    scales = np.ones((9, 4), dtype=np.float16)
    y = oracle.int4_matmul_ref(x, packed, scales, 50, 16)
    np.testing.assert_allclose(y, np.repeat(x.astype(np.float64).sum(1, keepdims=True), 9, 1),
                               rtol=1e-13, atol=1e-13)


def test_matmul_one_hot_x_selects_a_column():
    case = tiny_case()
    packed, scales, K = oracle.quantize_int4(case["w"], 128)
    w_hat = oracle.dequantize_int4(packed, scales, K, 128)
    for k in (0, 127, 128, 255, 256, 258):
        x = np.zeros((1, K), dtype=np.float32)
        x[0, k] = 1.0
        y = oracle.int4_matmul_ref(x, packed, scales, K, 128)
        assert np.array_equal(y[0], w_hat[:, k])
        # Which scale multiplies column k: the one of group k // 128.
        q = oracle.unpack_int4(packed, K)[:, k].astype(np.float64)
        assert np.array_equal(y[0], q * scales[:, k // 128].astype(np.float64))


def test_matmul_group_equal_K_is_one_scale_per_row():
    rng = np.random.default_rng(6)
    w = rng.normal(size=(7, 64)).astype(np.float32)
    x = rng.normal(size=(2, 64)).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 64)
    assert scales.shape == (7, 1)
    q = oracle.unpack_int4(packed, K).astype(np.float64)
    y = oracle.int4_matmul_ref(x, packed, scales, K, 64)
    expect = (x.astype(np.float64) @ q.T) * scales[:, 0].astype(np.float64)[None, :]
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-14)


def test_matmul_is_linear_in_x_and_not_transposed():
    rng = np.random.default_rng(8)
    w = rng.normal(size=(6, 40)).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 16)
    a = rng.normal(size=(3, 40))
    b = rng.normal(size=(3, 40))
    ya = oracle.int4_matmul_ref(a, packed, scales, K, 16)
    yb = oracle.int4_matmul_ref(b, packed, scales, K, 16)
    yab = oracle.int4_matmul_ref(2 * a - 3 * b, packed, scales, K, 16)
    np.testing.assert_allclose(yab, 2 * ya - 3 * yb, rtol=1e-12, atol=1e-12)
    assert ya.shape == (3, 6)


def test_matmul_close_to_unquantized_product():
    """The dequantized product approximates x @ w.T within the half-step error."""
    rng = np.random.default_rng(10)
    w = rng.normal(size=(16, 256)).astype(np.float32)
    x = rng.normal(size=(4, 256)).astype(np.float32)
    packed, scales, K = oracle.quantize_int4(w, 128)
    y = oracle.int4_matmul_ref(x, packed, scales, K, 128)
    s = np.repeat(scales.astype(np.float64), 128, axis=1)
    bound = np.abs(x.astype(np.float64)) @ (0.5 * s + 1e-6).T
    assert (np.abs(y - x.astype(np.float64) @ w.astype(np.float64).T) <= bound).all()


def test_error_bound_is_zero_only_where_it_must_be():
    case = tiny_case()
    packed, scales, K = oracle.quantize_int4(case["w"], 128)
    x = np.zeros((1, K), dtype=np.float32)
    x[0, 130] = 1.0                    # inside row 3's all-zero group
    b = oracle.matmul_error_bound(x, packed, scales, K, 128, 4e-3)
    w_hat = oracle.dequantize_int4(packed, scales, K, 128)
    assert b[0, 3] == 0.0
    assert np.array_equal(b[0] == 0.0, w_hat[:, 130] == 0.0)


def test_error_bound_by_hand_mixed_signs():
    """sum_k |x||w_hat| worked by hand on hand-made bytes with mixed signs.

    Row 0: q = [-8, 5, 3, -2] with scale 0.5 (bytes 0x58, 0xE3), so w_hat =
    [-4, 2.5, 1.5, -1].  x = [-2, 3, -1, 4]:
      sum |x||w_hat| = 8 + 7.5 + 1.5 + 4 = 21
    whereas x.w_hat = 10, |x|.w_hat = -3 and x.|w_hat| = 2, so a dropped
    abs() on either side (or both) gives another number.  Row 1 holds the same
    bytes with two groups of two, scales 0.5 and 2: w_hat = [-4, 2.5, 6, -4],
    sum = 8 + 7.5 + 6 + 16 = 37.5 (one scale for the whole row gives 21 or
    84).  The second batch row is -x: the bound is even in x."""
    packed = np.array([[0x58, 0xE3]], dtype=np.uint8)
    x = np.array([[-2.0, 3.0, -1.0, 4.0], [2.0, -3.0, 1.0, -4.0]], dtype=np.float32)
    for c in (4e-3, 1e-5, 1.0):
        b4 = oracle.matmul_error_bound(x, packed, np.array([[0.5]], np.float16), 4, 4, c)
        assert b4.shape == (2, 1)
        assert b4[0, 0] == c * 21.0 and b4[1, 0] == c * 21.0
        b2 = oracle.matmul_error_bound(x, packed, np.array([[0.5, 2.0]], np.float16), 4, 2, c)
        assert b2[0, 0] == c * 37.5 and b2[1, 0] == c * 37.5


def test_error_bound_uses_the_dequantized_weights_not_w():
    """The bound is over w_hat = q s, not over the weights before rounding.

    w = [1, 0.3, -0.55, 0.9] in one group of 4: s = fp16(1/7) = 0.1428...,
    codes rint(w/s) = [7, 2, -4, 6] (0.3/s = 2.1005, 0.55/s = 3.8509, 0.9/s =
    6.3015), so sum |x||w_hat| with x = [1, 10, 100, 1000] is
    s (7 + 20 + 400 + 6000) = 6427 s = 917.9, against sum |x||w| = 959.  The
    codes and s are taken here from the drill's definition by exact
    arithmetic."""
    w = np.array([[1.0, 0.3, -0.55, 0.9]], dtype=np.float32)
    x = np.array([[1.0, 10.0, 100.0, 1000.0]], dtype=np.float32)
    packed, scales, K = oracle.quantize_int4(w, 4)
    s = exact_scale(1.0)
    q = [exact_code(float(v), s) for v in w[0]]
    assert q == [7, 2, -4, 6]
    want = Fraction(s) * sum(abs(Fraction(float(a))) * abs(qq) for a, qq in zip(x[0], q))
    assert want == Fraction(s) * 6427
    b = oracle.matmul_error_bound(x, packed, scales, K, 4, 1.0)
    assert Fraction(float(b[0, 0])) == want          # exact: every term is exact in fp64
    unquantized = float(np.abs(x[0].astype(np.float64)) @ np.abs(w[0].astype(np.float64)))
    assert abs(float(b[0, 0]) - unquantized) > 1.0


def test_tiny_case_golden():
    """Regression against the committed expected values of the tiny case
    (written by tests/golden/make_golden.py, which calls only the oracle)."""
    g = _load("tiny_case_expected.json")
    case = tiny_case()
    packed, scales, K = oracle.quantize_int4(case["w"], case["group"])
    assert packed.tobytes().hex() == g["packed_hex"]
    assert scales.view(np.uint16).tolist() == g["scales_fp16_bits"]
    y = oracle.int4_matmul_ref(case["x"], packed, scales, K, case["group"])
    np.testing.assert_allclose(y, np.array(g["y"]), rtol=0, atol=1e-12)
