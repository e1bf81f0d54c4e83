"""Properties of the integer form of x that the integer decode kernel relies
on, checked in exact integer / float arithmetic on the CPU (NumPy).

For a 128-k block with largest magnitude in [2^e, 2^(e+1)), each x becomes
v = rint(x * 2^(29 - e)), split into four signed base-256 digits.  The
kernel's results are compared with the oracle in the GPU tests; these tests
check the representation itself:
  * the digits (bytes of v + 0x808080, the low three flipped back by 128)
    are balanced and reconstruct v exactly;
  * v * 2^(e - 29) equals x for every bf16 x within 2^22 of the block's
    largest magnitude, and differs by at most 2^(e - 30) otherwise;
  * the block sums the MMA forms, sum (16 q) d_i over 128 k, and the two
    combinations P01 = S0 + 2^8 S1 and P23 = S2 + 2^8 S3, fit int32.
"""

import numpy as np
import pytest


def _bf16(a):
    """Round float32 values to bf16 (RNE) and return them as float64."""
    b = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _digits(v):
    """Balanced base-256 digits of int32 values v: d0..d2 in [-128, 127], d3 top."""
    u = (v.astype(np.int64) + 0x808080) & 0xFFFFFFFF
    u = u ^ 0x808080
    d = [((u >> (8 * i)) & 0xFF).astype(np.int64) for i in range(4)]
    return [np.where(x >= 128, x - 256, x) for x in d]


def test_digits_are_balanced_and_exact_over_the_whole_range():
    rng = np.random.default_rng(0)
    v = np.concatenate([np.arange(-(1 << 16), 1 << 16),
                        rng.integers(-(1 << 30) + 1, 1 << 30, 2_000_000),
                        [-(1 << 30) + 1, (1 << 30) - 1, 0, 127, 128, -128, -129, 0x7F7F7F, -0x808080]])
    d = _digits(v)
    back = d[0] + 256 * d[1] + 65536 * d[2] + (1 << 24) * d[3]
    assert np.array_equal(back, v)
    for x in d[:3]:
        assert x.min() >= -128 and x.max() <= 127
    assert d[3].min() >= -64 and d[3].max() <= 64


def _block_form(x):
    """v and e of one block as the kernel forms them (float64 is exact here)."""
    amax = np.abs(x).max()
    e = max(int(np.floor(np.log2(amax))), -93)
    v = np.rint(x * 2.0 ** (29 - e))     # rint: half to even, like the kernel
    return v.astype(np.int64), e


@pytest.mark.parametrize("seed", range(6))
def test_bf16_x_within_2_22_of_the_block_maximum_is_exact(seed):
    rng = np.random.default_rng(seed)
    for _ in range(200):
        top = rng.integers(-60, 60)
        spread = rng.integers(0, 30)
        mag = 2.0 ** (top - rng.uniform(0, spread, 128))
        x = _bf16(mag * rng.choice([-1.0, 1.0], 128))
        v, e = _block_form(x)
        assert np.abs(v).max() < (1 << 30)
        err = np.abs(v * 2.0 ** (e - 29) - x)
        amax = np.abs(x).max()
        near = np.abs(x) >= amax * 2.0 ** -22
        assert (err[near] == 0).all()
        assert (err <= 2.0 ** (e - 30)).all()


def test_fp16_x_within_2_19_is_exact():
    rng = np.random.default_rng(7)
    for _ in range(300):
        x = (rng.standard_normal(128) * 2.0 ** rng.uniform(-20, 12, 128)).astype(np.float16)
        x = x[np.isfinite(x)].astype(np.float64)
        if not np.any(x):
            continue
        v, e = _block_form(x)
        amax = np.abs(x).max()
        near = np.abs(x) >= amax * 2.0 ** -19
        assert (v[near] * 2.0 ** (e - 29) == x[near]).all()


def test_block_sums_and_their_combinations_fit_int32():
    # Worst case: every weight code -8 (16q = -128) against every digit at
    # its extreme, over the 128 k of a block.
    for d in (-128, 127):
        s = 128 * (-128) * d
        assert abs(s) <= 1 << 21
    lo = 128 * 128 * 128  # |S_i| <= 2^21
    assert lo + 256 * lo < 2**31 - 1  # P01, P23
    # And a random block against the identity sum_k x q = 2^(e-33) (P01 + 2^16 P23).
    rng = np.random.default_rng(3)
    q = rng.integers(-8, 8, 128)
    x = _bf16(rng.standard_normal(128) * 3.0)
    v, e = _block_form(x)
    d = _digits(v)
    S = [int(np.dot(16 * q, di)) for di in d]
    P01, P23 = S[0] + 256 * S[1], S[2] + 256 * S[3]
    assert max(abs(P01), abs(P23)) < 2**30
    assert (P01 + 65536 * P23) * 2.0 ** (e - 33) == float(np.dot(q, v)) * 2.0 ** (e - 29)
