"""CPU oracle for the asymmetric (affine) 4-bit variant, and for the matmul's
bias + ReLU epilogue.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the plain, slow
statement of what the GPU library computes.  Only the test suite, the smoke
check and the CPU-baseline leg of the benchmark may use it; the product path
never imports it and shares no code with it.

Sources (web pages, cited by title and section):

* "Build a Blockwise INT4 Inference Engine", step 2 (blockwise quantization
  with per-group scales and zero-points): scale = (max - min) / 15, zero point
  = clip(round(-min / scale), 0, 15), q = clip(round(w / scale + zero_point),
  0, 15); step 3 (the fused kernel dequantizes (q - zp) * scale and applies
  ReLU to A @ dequantize(Q)); step 4 (the runtime layer computes x @ W_dq^T +
  bias, then ReLU).
* "Quantizing a Language Model From Scratch", sections on the quantization
  and dequantization formulas: affine quantization maps [x_min, x_max] onto
  [q_min, q_max] with S = (x_max - x_min) / 15 for INT4, and x' = S (x_q - Z).

Readings taken where the pages are silent or differ (each is also listed with
the design notes):

* Groups run along K within each row, as in the symmetric scheme's layout
  ([N, G] scales), not over the flattened matrix as in the engine page.
* Layout: element 2j in the low nibble of byte j (the drill's order; the
  engine page puts the even element in the high nibble); the nibble holds the
  unsigned code 0..15.  Scales are fp16 [N, G]; zero points uint8 [N, G].
* Precision, in the pages' order of operations: d = fp32(max - min) (IEEE
  subtraction), s = fp16_RNE(fp32(d / 15)); z = clip(rint(fp32(-min / s)), 0,
  15); q = clip(rint(fp32(fp32(w / s) + z)), 0, 15), with s read back as fp32
  and every division an IEEE fp32 division; rint rounds half to even.
* The engine page floors the scale at 1e-8 to avoid dividing by zero; in
  fp16 that floor is 0, so a zero scale (a constant group, or a range that
  underflows fp16) codes the whole group as q = 0, z = 0, which dequantizes
  to 0 -- the symmetric scheme's rule for an all-zero group.
* Precondition: finite w with (max - min) / 15 below 65520 per group.

Parity pins: ``tests/test_oracle_affine.py`` (exact rational arithmetic, the
engine page's properties, a worked example, exhaustive bytes).
"""

from __future__ import annotations

import numpy as np

from .int4_oracle import group_count, packed_cols

__all__ = [
    "group_minmax",
    "affine_scales",
    "affine_zero_points",
    "affine_codes",
    "pack_unsigned",
    "quantize_uint4_affine",
    "unpack_uint4",
    "dequantize_uint4_affine",
    "uint4_affine_matmul_ref",
    "uint4_affine_matmul_groupwise",
    "matmul_error_bound_affine",
    "linear_epilogue_ref",
    "epilogue_error_bound",
]


def _as_f32_matrix(w) -> np.ndarray:
    w = np.asarray(w)
    if w.ndim != 2:
        raise ValueError("w must be a 2-D [N, K] array")
    if w.dtype not in (np.float32, np.float16):
        raise TypeError("w must be float32 (bf16 inputs are passed widened to float32) or float16")
    return w.astype(np.float32)


def group_minmax(w32: np.ndarray, group: int):
    """(min, max) over the real elements of each (row, group), exact.

    A partial last group takes its real elements only (padding with the
    group's own first value, which cannot change either extreme)."""
    N, K = w32.shape
    G = group_count(K, group)
    padded = np.empty((N, G * group), dtype=np.float32)
    padded[:, :K] = w32
    if G * group > K:
        padded[:, K:] = w32[:, (G - 1) * group][:, None]
    blocks = padded.reshape(N, G, group)
    return blocks.min(axis=2), blocks.max(axis=2)


def affine_scales(mn: np.ndarray, mx: np.ndarray) -> np.ndarray:
    """s = fp16_RNE(fp32(fp32(max - min) / 15)): the engine page's step 2
    (scale maps [min, max] onto [0, 15]), stored as fp16."""
    d = (mx.astype(np.float32) - mn.astype(np.float32)).astype(np.float32)
    q32 = (d / np.float32(15.0)).astype(np.float32)
    with np.errstate(over="ignore"):
        return q32.astype(np.float16)


def affine_zero_points(mn: np.ndarray, s16: np.ndarray) -> np.ndarray:
    """z = clip(rint(fp32(-min / s)), 0, 15), 0 where s == 0 (engine page,
    step 2: "zero_point = clip(round(-min / scale), 0, 15)")."""
    sf = s16.astype(np.float32)
    zero = sf == 0
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (-mn.astype(np.float32) / np.where(zero, np.float32(1.0), sf)).astype(np.float32)
    z = np.clip(np.rint(t), 0, 15)
    z[zero] = 0
    return z.astype(np.uint8)


def affine_codes(w32: np.ndarray, s16: np.ndarray, z: np.ndarray, group: int) -> np.ndarray:
    """q = clip(rint(fp32(fp32(w / s) + z)), 0, 15), 0 where s == 0 (engine
    page, step 2: "q = round(group / scale + zero_point)", clipped)."""
    N, K = w32.shape
    sf = np.repeat(s16.astype(np.float32), group, axis=1)[:, :K]
    zf = np.repeat(z.astype(np.float32), group, axis=1)[:, :K]
    zero = sf == 0
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (w32 / np.where(zero, np.float32(1.0), sf)).astype(np.float32)
    u = (t + zf).astype(np.float32)
    q = np.clip(np.rint(u), 0, 15)
    q[zero] = 0
    return q.astype(np.uint8)


def pack_unsigned(q: np.ndarray) -> np.ndarray:
    """Unsigned nibbles, element 2j in the low nibble of byte j; an odd K
    pads one zero nibble."""
    N, K = q.shape
    qq = np.zeros((N, 2 * packed_cols(K)), dtype=np.uint8)
    qq[:, :K] = q
    return (qq[:, 0::2] | (qq[:, 1::2] << 4)).astype(np.uint8)


def quantize_uint4_affine(w, group: int = 128):
    """-> (packed uint8 [N, ceil(K/2)], scales fp16 [N, G], zeros uint8 [N, G], K).

    The engine page's step 2 in its order: group min and max, scale, zero
    point, codes; then the nibble packing."""
    if group < 1:
        raise ValueError("group must be >= 1")
    w32 = _as_f32_matrix(w)
    K = w32.shape[1]
    mn, mx = group_minmax(w32, group)
    s16 = affine_scales(mn, mx)
    z = affine_zero_points(mn, s16)
    q = affine_codes(w32, s16, z, group)
    return pack_unsigned(q), s16, z, K


def unpack_uint4(packed, K: int) -> np.ndarray:
    """Unsigned codes uint8 [N, K]: low nibble first, then high nibble."""
    p = np.asarray(packed, dtype=np.uint8)
    if p.ndim != 2 or p.shape[1] != packed_cols(K):
        raise ValueError("packed must be [N, ceil(K/2)]")
    out = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out[:, :K]


def dequantize_uint4_affine(packed, scales, zeros, K: int, group: int) -> np.ndarray:
    """w_hat = (q - z) * s in fp64 (engine page, step 3: "(q - zp) * scale";
    LM page: x' = S (x_q - Z)); every product is exact in fp64."""
    q = unpack_uint4(packed, K).astype(np.float64)
    G = group_count(K, group)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    z = np.asarray(zeros, dtype=np.uint8).astype(np.float64)
    if s.shape != (q.shape[0], G) or z.shape != (q.shape[0], G):
        raise ValueError("scales and zeros must be [N, ceil(K/group)]")
    return (q - np.repeat(z, group, axis=1)[:, :K]) * np.repeat(s, group, axis=1)[:, :K]


def uint4_affine_matmul_ref(x, packed, scales, zeros, K: int, group: int) -> np.ndarray:
    """y = x @ w_hat^T in fp64 over the full dequantization."""
    xd = np.asarray(x).astype(np.float64)
    if xd.ndim != 2 or xd.shape[1] != K:
        raise ValueError("x must be [M, K]")
    return xd @ dequantize_uint4_affine(packed, scales, zeros, K, group).T


def uint4_affine_matmul_groupwise(x, packed, scales, zeros, K: int, group: int) -> np.ndarray:
    """The same product one group at a time, in fp64: per group, x times the
    integer codes, minus the zero point times the group's sum of x, then the
    scale -- the one extra per-group term the affine scheme adds."""
    xd = np.asarray(x).astype(np.float64)
    q = unpack_uint4(packed, K).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    z = np.asarray(zeros, dtype=np.uint8).astype(np.float64)
    y = np.zeros((xd.shape[0], q.shape[0]))
    for g in range(group_count(K, group)):
        k0, k1 = g * group, min((g + 1) * group, K)
        xq = xd[:, k0:k1] @ q[:, k0:k1].T
        xs = xd[:, k0:k1].sum(axis=1)
        y += (xq - xs[:, None] * z[None, :, g]) * s[None, :, g]
    return y


def matmul_error_bound_affine(x, packed, scales, zeros, K: int, group: int, c: float):
    """Per-element tolerance c * sum_k |x[m, k]| |w_hat[n, k]| (fp64)."""
    xd = np.abs(np.asarray(x).astype(np.float64))
    return c * (xd @ np.abs(dequantize_uint4_affine(packed, scales, zeros, K, group)).T)


def linear_epilogue_ref(y, bias=None, relu: bool = False) -> np.ndarray:
    """relu(y + b) in fp64: the engine page's step 4 layer (x @ W_dq^T +
    bias, then np.maximum(., 0)) and step 3 kernel (ReLU of A @ dequantize(Q))."""
    out = np.asarray(y, dtype=np.float64)
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)[None, :]
    if relu:
        out = np.maximum(out, 0.0)
    return out


def epilogue_error_bound(matmul_bound, y_ref, bias=None) -> np.ndarray:
    """Tolerance after the epilogue: the matmul's bound carries over (ReLU is
    1-Lipschitz) plus one fp32 rounding of the sum y + b."""
    s = np.asarray(y_ref, dtype=np.float64)
    if bias is not None:
        s = s + np.asarray(bias, dtype=np.float64)[None, :]
    return matmul_bound * (1 + 2.0 ** -23) + 2.0 ** -24 * np.abs(s)
