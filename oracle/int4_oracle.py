"""CPU oracle for symmetric group-wise INT4 weight quantization and the
weight-only dequantizing matmul.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain, obviously correct
statement of what the GPU library computes. Only the test suite, the smoke
check and the CPU-baseline leg of the benchmark may import it; the product
path (the CUDA library and its Python binding) never does, and shares no code
with it.

Sources (web pages, cited by title and section):

* "Implement INT4 group quantization, nibble packing and a dequantizing
  matmul" (inferenceinterviews.com drill), problem statement: the three
  functions ``quantize_int4``, ``unpack_int4`` and ``int4_matmul``, their
  argument order, the [N, ceil(K/2)] uint8 and [N, G] fp16 layouts, the
  two's-complement nibble with element 2j in the low nibble of byte j, the
  zero pad nibble for odd K, scale 0 for an all-zero group, and the matmul
  computed one group at a time (integer weights times x, then the group's
  scale on each output column).  Its visible tests fix the byte layout of the
  [1, -1, 7, -7] example and the half-step round-trip bound.
* "Building a pure-Python INT4 transformer weight quantizer with block-wise
  per-channel scaling", sections 3-5: per-row blocks along K, scale =
  max|block| / 7, q = round(w / s) clipped to [-8, 7], w_hat = q * s.
* "Quantizing a Language Model From Scratch", sections "Symmetric
  quantization" and "Groupwise scales for INT4": the symmetric scale
  |x|max / q_max with q_max = 7 for INT4, one scale per contiguous group.

Readings taken where the pages are silent (each is also listed with the
design notes):

* Precision of the scale: fp32 ``absmax / 7`` correctly rounded, then rounded
  to fp16 by round-to-nearest-even (two defined roundings).
* The divisor of ``w``: the stored fp16 scale widened to fp32; the division is
  an IEEE fp32 division; ``round`` is round-half-to-even (NumPy's ``rint``,
  the rounding the pages' own NumPy code uses).
* A scale of 0 (an all-zero group, or ``absmax / 7`` underflowing fp16) gives
  q = 0 for the whole group.
* The matmul reference is exact-as-possible fp64 over the dequantized weights;
  any summation order is correct within the stated error bound.

Parity pins: every function here is pinned by ``tests/test_oracle.py``
against values the pages print, closed forms, exhaustive enumeration or exact
rational arithmetic.  No function is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "group_count",
    "packed_cols",
    "quantize_int4",
    "scales_from_absmax",
    "group_absmax",
    "quantize_codes",
    "pack_nibbles",
    "unpack_int4",
    "dequantize_int4",
    "int4_matmul_ref",
    "int4_matmul_groupwise",
    "matmul_error_bound",
    "storage_bytes",
]


def group_count(K: int, group: int) -> int:
    """G = ceil(K / group): groups per row; the last one may be partial.

    Drill page, problem statement ("G = ceil(K / group)").
    """
    if K < 0 or group < 1:
        raise ValueError("K must be >= 0 and group >= 1")
    return -(-K // group)


def packed_cols(K: int) -> int:
    """ceil(K / 2): bytes per packed row (drill page, problem statement)."""
    return -(-K // 2)


def _as_f32_matrix(w) -> np.ndarray:
    w = np.asarray(w)
    if w.ndim != 2:
        raise ValueError("w must be a 2-D [N, K] array")
    if w.dtype not in (np.float32, np.float16):
        raise TypeError("w must be float32 (bf16 inputs are passed widened to float32) or float16")
    # Widening fp16 -> fp32 is exact; bf16 values arrive already widened.
    return w.astype(np.float32)


def group_absmax(w32: np.ndarray, group: int) -> np.ndarray:
    """m[n, g] = max over the real elements of group g of row n of |w|.

    Pure-Python quantizer page, section 3 (max of |block| per block of a row);
    a partial last group takes the max over its real elements, the same as
    padding with zeros, which cannot change a max of absolute values.
    """
    N, K = w32.shape
    G = group_count(K, group)
    padded = np.zeros((N, G * group), dtype=np.float32)
    padded[:, :K] = np.abs(w32)
    return padded.reshape(N, G, group).max(axis=2)


def scales_from_absmax(m: np.ndarray) -> np.ndarray:
    """s = fp16_RNE(fp32(m / 7)).

    Drill page: "scale = absmax of the group / 7", stored as float16; the
    division is done in fp32 (IEEE, correctly rounded) and the result rounded
    to fp16 by round-to-nearest-even (NumPy's fp32 -> fp16 cast).
    """
    q32 = (m.astype(np.float32) / np.float32(7.0)).astype(np.float32)
    with np.errstate(over="ignore"):          # absmax >= 7 * 65520 -> +inf
        return q32.astype(np.float16)


def quantize_codes(w32: np.ndarray, scales16: np.ndarray, group: int) -> np.ndarray:
    """q = clip(rint(w / float32(s)), -8, 7) as int8; q = 0 where s == 0.

    Drill page, problem statement ("q = round(w / scale) clipped to [-8, 7]",
    "a group of zeros gets scale 0"); pure-Python quantizer page, section 4
    (divide by the expanded scale, round, clip).
    """
    N, K = w32.shape
    sf = np.repeat(scales16.astype(np.float32), group, axis=1)[:, :K]
    zero = sf == 0
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (w32 / np.where(zero, np.float32(1.0), sf)).astype(np.float32)
    q = np.clip(np.rint(t), -8, 7)
    q[zero] = 0
    return q.astype(np.int8)


def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, element 2j in the low nibble of byte j.

    Drill page, problem statement; an odd K pads one zero nibble (the high
    nibble of the row's last byte).
    """
    N, K = q.shape
    Kp = packed_cols(K)
    qq = np.zeros((N, 2 * Kp), dtype=np.int16)
    qq[:, :K] = q
    nib = (qq & 0xF).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def quantize_int4(w, group: int = 128):
    """quantize_int4(w, group) -> (packed uint8 [N, ceil(K/2)], scales fp16 [N, G], K).

    The drill page's first function, composed of the steps above in the
    pages' order: block partition, scale, quantize, pack.
    """
    if group < 1:
        raise ValueError("group must be >= 1")
    w32 = _as_f32_matrix(w)
    K = w32.shape[1]
    m = group_absmax(w32, group)
    s16 = scales_from_absmax(m)
    q = quantize_codes(w32, s16, group)
    return pack_nibbles(q), s16, K


def unpack_int4(packed, K: int) -> np.ndarray:
    """unpack_int4(packed, K) -> int8 [N, K], sign-extended.

    Drill page, problem statement. Each nibble v in 0..15 stands for v - 16
    when v >= 8 (two's complement); low nibble first, then high nibble.
    """
    p = np.asarray(packed, dtype=np.uint8)
    if p.ndim != 2 or p.shape[1] != packed_cols(K):
        raise ValueError("packed must be [N, ceil(K/2)]")
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.int16)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out[:, :K].astype(np.int8)


def dequantize_int4(packed, scales, K: int, group: int) -> np.ndarray:
    """w_hat[n, k] = q[n, k] * float(s[n, k // group]) in fp64.

    Pure-Python quantizer page, section 5 (w_hat = q * s); every product is
    exact in fp64 (|q| <= 8, s has an 11-bit significand).
    """
    q = unpack_int4(packed, K).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    if s.shape != (q.shape[0], group_count(K, group)):
        raise ValueError("scales must be [N, ceil(K/group)]")
    return q * np.repeat(s, group, axis=1)[:, :K]


def _as_f64_activations(x) -> np.ndarray:
    x = np.asarray(x)
    if x.ndim != 2:
        raise ValueError("x must be a 2-D [M, K] array")
    return x.astype(np.float64)


def int4_matmul_ref(x, packed, scales, K: int, group: int = 128) -> np.ndarray:
    """y = x @ dequantize(W).T in fp64 (brute force over the full dequantization).

    Drill page, problem statement ("y = x @ dequantize(W).T"); its hidden
    suite compares the matmul "against a full dequantization".  x is taken
    exactly as stored (fp32, fp16 or bf16 widened to fp32).
    """
    xd = _as_f64_activations(x)
    if xd.shape[1] != K:
        raise ValueError("x must be [M, K]")
    return xd @ dequantize_int4(packed, scales, K, group).T


def int4_matmul_groupwise(x, packed, scales, K: int, group: int = 128) -> np.ndarray:
    """The drill page's matmul order written out literally, in fp64.

    For each group g: multiply x by the group's integer weights (a partial sum
    per output), then apply the group's scale to each output column and add.
    Used on small cases to check the algebra of ``int4_matmul_ref``.
    """
    xd = _as_f64_activations(x)
    q = unpack_int4(packed, K).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    M = xd.shape[0]
    N = q.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    for g in range(group_count(K, group)):
        k0, k1 = g * group, min((g + 1) * group, K)
        partial = np.zeros((M, N), dtype=np.float64)
        for k in range(k0, k1):
            partial += np.outer(xd[:, k], q[:, k])
        y += partial * s[:, g][None, :]
    return y


def matmul_error_bound(x, packed, scales, K: int, group: int, c: float) -> np.ndarray:
    """Per-element tolerance c * sum_k |x[m, k]| * |w_hat[n, k]| (fp64).

    The bound the matmul must meet: c = 1e-5 for fp32 activations and
    c = 4e-3 for bf16/fp16 activations with fp32 accumulation.
    """
    xd = np.abs(_as_f64_activations(x))
    return c * (xd @ np.abs(dequantize_int4(packed, scales, K, group)).T)


def storage_bytes(N: int, K: int, group: int, scale_bytes: int = 2) -> dict:
    """Closed-form storage of one quantized [N, K] matrix.

    Drill page (its hidden suite names "the storage size"): packed bytes
    N * ceil(K/2) plus scale bytes scale_bytes * N * G (fp16: 2 bytes).
    """
    G = group_count(K, group)
    packed = N * packed_cols(K)
    sc = scale_bytes * N * G
    return {"packed": packed, "scales": sc, "total": packed + sc}
