"""GPU parity: the CUDA library against the CPU oracle, through the C ABI.

Packed bytes, fp16 scale bits and unpacked int8 must be bit-exact; the matmul
must meet |y - y_ref| <= c * sum|x||w_hat| with c = 1e-5 (fp32 x) or 4e-3
(bf16/fp16 x).  Every kernel path is exercised on the shapes it accepts,
including ragged tails, odd K, partial last groups, all-zero groups, -8
codes and the degenerate sizes.
"""

import numpy as np
import pytest
import torch

import dequant_gemm_int4_b200 as q4
import oracle
from gpu_util import (TOL_F32, TOL_HALF, assert_matmul_close, assert_quantize_exact,
                      oracle_quantize, to_np)
from workloads import (DISTILGPT2_LINEARS, LLAMA7B_DECODE_LINEARS, make_activations,
                       make_weights, tiny_case)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    q4.lib()
    yield
    torch.cuda.synchronize()
    assert q4.device_status() == q4.OK


def _tol(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_HALF


# ---------------------------------------------------------------------------
# quantize_int4
# ---------------------------------------------------------------------------
def test_quantize_tiny_case_matches_golden_and_oracle():
    case = tiny_case()
    w = torch.from_numpy(case["w"]).to(DEV)
    packed, scales, K = q4.quantize_int4(w, case["group"])
    assert K == 259 and tuple(packed.shape) == (16, 130) and tuple(scales.shape) == (16, 3)
    assert_quantize_exact(w, packed, scales, case["group"])
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_case_expected.json")))
    assert packed.cpu().numpy().tobytes().hex() == g["packed_hex"]
    assert scales.cpu().view(torch.int16).numpy().view(np.uint16).tolist() == g["scales_fp16_bits"]


def test_quantize_drill_byte_layout():
    w = torch.tensor([[1.0, -1.0, 7.0, -7.0]], device=DEV)
    packed, scales, K = q4.quantize_int4(w, 4)
    assert float(scales[0, 0]) == 1.0
    assert packed.cpu().tolist() == [[0xF1, 0x97]]
    # The same row on the fast path (K multiple of 8, group 8).
    w8 = torch.tensor([[1.0, -1.0, 7.0, -7.0, 0.0, 0.0, 0.0, 0.0]], device=DEV)
    packed8, scales8, _ = q4.quantize_int4(w8, 8)
    assert packed8.cpu().tolist() == [[0xF1, 0x97, 0x00, 0x00]]


def _special_rows():
    t = 2.0 ** -24
    rows = [
        [7.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -3.5],
        [0.0] * 8,
        [7 * 2.0 ** -25, 0, 0, 0, 0, 0, 0, 0],
        [7 * 1.49 * t, -7 * 1.49 * t, 0.5 * t, 0, 0, 0, 0, 0],
        [1e-5, -3e-6, 2e-6, 0, 0, 0, 0, 0],
        [-0.0, 0.0, -0.0, 0, 0, 0, 0, 0],
        [3.0, -3.0, 1.0, 2.0, -1.5, 0.75, 0.2, -0.1],
        [458000.0, -1.0, 1.0, 0, 0, 0, 0, 0],
        [7 * 65520.0, 1.0, -5.0, 0, 0, 0, 0, 0],   # scale overflows to +inf
    ]
    return torch.tensor(rows, dtype=torch.float32)


@pytest.mark.parametrize("K_pad", [0, 1])
def test_quantize_special_values(K_pad):
    w = _special_rows()
    if K_pad:  # odd K forces the general kernels
        w = torch.cat([w, torch.zeros(w.shape[0], 1)], dim=1)
    w = w.to(DEV)
    packed, scales, K = q4.quantize_int4(w, 8)
    assert_quantize_exact(w, packed, scales, 8)


@pytest.mark.parametrize("group", [8, 16, 32])
def test_quantize_half_integer_quotients(group):
    """Weights placed exactly on and next to half-integer multiples of the
    scale: every fast path must agree with the IEEE division on every tie."""
    rng = np.random.default_rng(21 + group)
    s = (rng.uniform(0.01, 2.0, size=(4096, 1))).astype(np.float16).astype(np.float32)
    half = rng.integers(-7, 7, size=(4096, group - 1)) + 0.5     # -6.5 .. 6.5
    w = (half * s).astype(np.float32)
    nudge = rng.integers(-2, 3, size=w.shape).astype(np.int32)
    w = (w.view(np.int32) + nudge).view(np.float32)
    w = np.concatenate([w, 7 * s], axis=1)          # absmax = 7 s -> scale s
    wt = torch.from_numpy(w.astype(np.float32)).to(DEV)
    for dtype in (torch.float32, torch.float16, torch.bfloat16):
        wd = wt.to(dtype)
        packed, scales, K = q4.quantize_int4(wd, group)
        assert_quantize_exact(wd, packed, scales, group)


def _every_16bit_weight_under_anchors(dtype, n_anchors, seed):
    """Groups of 16: an anchor a (the group's absmax, so the scale is
    fp16(a / 7)) followed by 15 weights taken from every finite value of the
    16-bit type with |v| <= |a|, both signs.  Anchors span the normal fp16
    scale range with random significands."""
    rng = np.random.default_rng(seed)
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if dtype == torch.bfloat16:
        vals = (allbits.astype(np.uint32) << 16).view(np.float32)
    else:
        vals = allbits.view(np.float16).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    rows = []
    for _ in range(n_anchors):
        e = rng.integers(-14, 13)
        a = np.float32(7.0 * (1.0 + rng.random()) * 2.0 ** e)
        a = np.float32(torch.tensor(a).to(dtype).float().item())   # representable anchor
        v = vals[np.abs(vals) <= a]
        v = rng.permutation(v)
        pad = (-len(v)) % 15
        v = np.concatenate([v, np.zeros(pad, np.float32)]).reshape(-1, 15)
        rows.append(np.concatenate([np.full((len(v), 1), a, np.float32), v], axis=1))
    g = np.concatenate(rows, axis=0)                      # [groups, 16]
    g = np.concatenate([g, np.zeros(((-len(g)) % 16, 16), np.float32)])
    w = g.reshape(-1, 256)                                # 16 groups per row
    return torch.from_numpy(w).to(DEV).to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_every_16bit_weight(dtype):
    """Every finite bf16 / fp16 weight value, under scales from all normal
    fp16 binades, quantized by the 16-bit fast path (no tie check): codes and
    scales bit-exact against the oracle's IEEE division and rint."""
    w = _every_16bit_weight_under_anchors(dtype, n_anchors=24, seed=5 if dtype == torch.bfloat16 else 6)
    packed, scales, K = q4.quantize_int4(w, 16)
    assert_quantize_exact(w, packed, scales, 16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N, K, group", [
    (1, 8, 8), (3, 256, 32), (17, 1024, 128), (5, 1000, 64), (64, 4096, 256),
    (7, 264, 128),            # partial last group on the fast path
    (9, 259, 128), (4, 33, 32), (6, 1, 4), (2, 3, 2), (11, 515, 96), (8, 300, 300),
    (3, 100, 1000),           # one partial group larger than K
])
def test_quantize_shapes(dtype, N, K, group):
    w = make_weights(N, K, seed=N * 1000 + K, device=DEV, dtype=dtype, dist="student_t3",
                     zero_group_frac=0.1, group=group)
    packed, scales, Kout = q4.quantize_int4(w, group)
    assert Kout == K
    assert_quantize_exact(w, packed, scales, group)


@pytest.mark.parametrize("layer", DISTILGPT2_LINEARS, ids=lambda l: l.name)
def test_quantize_distilgpt2_full(layer):
    w = make_weights(layer.N, layer.K, seed=2, device=DEV, dtype=torch.float32, std=0.02)
    packed, scales, _ = q4.quantize_int4(w, layer.group)
    assert_quantize_exact(w, packed, scales, layer.group)


@pytest.mark.parametrize("N, K", [(28672, 8192), (8192, 28673)])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_quantize_bulk_full_size_every_row(N, K, group):
    """The bulk-quantize workloads at full size: every row bit-exact (compared
    on the host in chunks of rows), and unpack of every row."""
    w = make_weights(N, K, seed=5, device=DEV, dtype=torch.bfloat16, dist="student_t3",
                     zero_group_frac=0.01, group=group)
    packed, scales, _ = q4.quantize_int4(w, group)
    q = q4.unpack_int4(packed, K)
    torch.cuda.synchronize()
    for r0 in range(0, N, 4096):
        rows = np.arange(r0, min(r0 + 4096, N))
        assert_quantize_exact(w, packed, scales, group, rows=rows)
        idx = torch.as_tensor(rows, device=DEV)
        q_ref = oracle.unpack_int4(packed.index_select(0, idx).cpu().numpy(), K)
        assert np.array_equal(q.index_select(0, idx).cpu().numpy(), q_ref)


@pytest.mark.parametrize("exponents", [(0,), (-124, -125, -126), ("subnormal",), (15, 16)])
def test_scale_division_exhaustive_over_mantissas(exponents):
    """fp16(fp32(m / 7)) on every fp32 mantissa of the given binades (and on
    every subnormal): the kernel's division by the constant 7 must equal the
    IEEE division the oracle uses, bit for bit.  Group 1 makes every element
    its own group, so each one yields a scale."""
    mant = np.arange(1 << 23, dtype=np.uint32)
    parts = []
    for e in exponents:
        if e == "subnormal":
            parts.append(mant.view(np.float32))
        else:
            parts.append(((np.uint32(e + 127) << 23) | mant).view(np.float32))
    m = np.concatenate(parts).reshape(1, -1)
    w = torch.from_numpy(m).to(DEV)
    packed, scales, K = q4.quantize_int4(w, 1)
    got = scales.cpu().view(torch.int16).numpy().view(np.uint16)[0]
    p_ref, s_ref, _ = oracle.quantize_int4(m, 1)
    want = s_ref.view(np.uint16)[0]
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} scales differ, first m = {m[0, bad[0]]!r}"
    assert np.array_equal(packed.cpu().numpy(), p_ref)


def test_quantize_unaligned_pointers_take_the_general_path():
    base = make_weights(8, 1025, seed=3, device=DEV, dtype=torch.bfloat16).reshape(-1)
    w = base[1:1 + 8 * 1024].view(8, 1024)     # 2-byte aligned only
    assert w.data_ptr() % 16 != 0
    packed, scales, _ = q4.quantize_int4(w, 128)
    assert_quantize_exact(w, packed, scales, 128)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("K", [1024, 1031, 28673])
@pytest.mark.parametrize("woff, poff", [(0, 0), (1, 3), (3, 1), (5, 2)])
def test_quantize_any_alignment_through_the_abi(dtype, K, woff, poff):
    """Weights and packed output at odd element / byte offsets (rows at any
    alignment): bit-exact against the oracle, and nothing outside the output
    range is written."""
    import ctypes
    N, group = 37, 64
    wbuf = make_weights(N * K + woff, 1, seed=K + woff, device=DEV, dtype=dtype,
                        dist="student_t3").reshape(-1)
    w = wbuf[woff:woff + N * K].view(N, K)
    Kp = (K + 1) // 2
    pbuf = torch.full((N * Kp + poff + 8,), 0xA5, dtype=torch.uint8, device=DEV)
    scales = torch.empty((N, -(-K // group)), dtype=torch.float16, device=DEV)
    code = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}[dtype]
    rc = q4.lib().int4_quantize(ctypes.c_void_p(w.data_ptr()), code, N, K, group,
                                ctypes.c_void_p(pbuf.data_ptr() + poff),
                                ctypes.c_void_p(scales.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    pb = pbuf.cpu().numpy()
    assert (pb[:poff] == 0xA5).all() and (pb[poff + N * Kp:] == 0xA5).all()
    packed = torch.from_numpy(pb[poff:poff + N * Kp].reshape(N, Kp).copy()).to(DEV)
    assert_quantize_exact(w, packed, scales, group)


@pytest.mark.parametrize("K", [2, 7, 1000, 1001, 28673])
@pytest.mark.parametrize("poff, ooff", [(0, 0), (1, 0), (0, 3), (5, 7)])
def test_unpack_any_alignment_through_the_abi(K, poff, ooff):
    import ctypes
    N = 23
    Kp = (K + 1) // 2
    g = torch.Generator(device=DEV)
    g.manual_seed(K * 31 + poff)
    pbuf = torch.randint(0, 256, (N * Kp + poff,), generator=g, device=DEV,
                         dtype=torch.int32).to(torch.uint8)
    packed = pbuf[poff:].view(N, Kp)
    obuf = torch.full((N * K + ooff + 16,), 0x5A, dtype=torch.uint8, device=DEV)
    rc = q4.lib().int4_unpack(ctypes.c_void_p(packed.data_ptr()), K, N,
                              ctypes.c_void_p(obuf.data_ptr() + ooff),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    ob = obuf.cpu().numpy()
    assert (ob[:ooff] == 0x5A).all() and (ob[ooff + N * K:] == 0x5A).all()
    got = ob[ooff:ooff + N * K].view(np.int8).reshape(N, K)
    assert np.array_equal(got, oracle.unpack_int4(packed.cpu().numpy(), K))


def test_quantize_is_deterministic():
    w = make_weights(512, 2048, seed=4, device=DEV, dtype=torch.bfloat16, dist="student_t3")
    a = q4.quantize_int4(w, 64)
    b = q4.quantize_int4(w, 64)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))


# ---------------------------------------------------------------------------
# unpack_int4
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N, K", [(1, 2), (1, 1), (3, 5), (16, 259), (7, 512), (33, 1000),
                                  (5, 31), (1000, 34)])
def test_unpack_random_bytes(N, K):
    g = torch.Generator(device=DEV)
    g.manual_seed(N * 7 + K)
    Kp = (K + 1) // 2
    packed = torch.randint(0, 256, (N, Kp), generator=g, device=DEV, dtype=torch.int32).to(torch.uint8)
    if K % 2:
        packed[:, -1] &= 0x0F
    q = q4.unpack_int4(packed, K)
    assert q.dtype == torch.int8 and tuple(q.shape) == (N, K)
    assert np.array_equal(q.cpu().numpy(), oracle.unpack_int4(packed.cpu().numpy(), K))


def test_unpack_full_size_odd_k_every_row():
    """The bulk-quantize workload's odd-K matrix [8192, 28673]: every output
    byte against the oracle, compared in row chunks on the host."""
    N, K = 8192, 28673
    Kp = (K + 1) // 2
    g = torch.Generator(device=DEV)
    g.manual_seed(28673)
    packed = torch.randint(0, 256, (N, Kp), generator=g, device=DEV, dtype=torch.int32).to(torch.uint8)
    q = q4.unpack_int4(packed, K)
    for r0 in range(0, N, 1024):
        got = q[r0:r0 + 1024].cpu().numpy()
        want = oracle.unpack_int4(packed[r0:r0 + 1024].cpu().numpy(), K)
        assert np.array_equal(got, want), r0


def test_unpack_all_256_bytes_and_minus_eight():
    packed = torch.arange(256, device=DEV, dtype=torch.int32).to(torch.uint8).view(1, 256)
    q = q4.unpack_int4(packed, 512).cpu().numpy()[0]
    assert np.array_equal(q, oracle.unpack_int4(packed.cpu().numpy(), 512)[0])
    assert q[2 * 0x88] == -8 and q[2 * 0x88 + 1] == -8
    assert q[2 * 0x80] == 0 and q[2 * 0x80 + 1] == -8


def test_unpack_unaligned_pointer():
    buf = torch.randint(0, 256, (8 * 64 + 1,), device=DEV, dtype=torch.int32).to(torch.uint8)
    packed = buf[1:].view(8, 64)
    q = q4.unpack_int4(packed, 128)
    assert np.array_equal(q.cpu().numpy(), oracle.unpack_int4(packed.cpu().numpy(), 128))


# ---------------------------------------------------------------------------
# int4_matmul
# ---------------------------------------------------------------------------
def _quantized(N, K, group, seed, std=0.02, dist="normal", zero_group_frac=0.0):
    w = make_weights(N, K, seed=seed, device=DEV, dtype=torch.float32, std=std, dist=dist,
                     zero_group_frac=zero_group_frac, group=group)
    return q4.quantize_int4(w, group)


def test_matmul_tiny_case_fp32():
    case = tiny_case()
    w = torch.from_numpy(case["w"]).to(DEV)
    x = torch.from_numpy(case["x"]).to(DEV)
    packed, scales, K = q4.quantize_int4(w, 128)
    y = q4.int4_matmul(x, packed, scales, K, 128)
    assert tuple(y.shape) == (4, 16) and y.dtype == torch.float32
    assert_matmul_close(y, x, packed, scales, K, 128, TOL_F32)
    assert q4.matmul_select(torch.float32, K, 128, 4, 16) == q4.PATH_SIMT


@pytest.mark.parametrize("path", [q4.PATH_SIMT, q4.PATH_DECODE])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M, N, K, group", [
    (1, 128, 128, 128), (1, 4096, 4096, 128), (4, 11008, 4096, 128), (16, 4096, 11008, 128),
    (3, 300, 4096, 64), (9, 200, 1024, 32), (1, 2304, 768, 32), (1, 768, 3072, 64),
    (16, 77, 8224, 128), (5, 1000, 2048, 256), (2, 64, 96, 32), (7, 129, 160, 32),
    (12, 33, 640, 64), (1, 1, 32, 32),
    (4, 18000, 4096, 128),   # too tall for resident tiles: the integer kernel
    (1, 2048, 32768, 128),   # rows too long for resident tiles: the small-matrix kernel
    (9, 1500, 40960, 256),
    (16, 11000, 4096, 128),  # resident tiles, 4 warps per tile, ragged last tile
    (5, 1001, 2048, 512),
])
def test_matmul_paths(path, dtype, M, N, K, group):
    packed, scales, _ = _quantized(N, K, group, seed=M + N + K)
    x = make_activations(M, K, seed=M * 31 + K, device=DEV, dtype=dtype)
    y = q4.int4_matmul(x, packed, scales, K, group, path=path)
    torch.cuda.synchronize()
    cols = None
    if N > 2048:
        cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(N).integers(0, N, 1500)]))
    assert_matmul_close(y, x, packed, scales, K, group, _tol(dtype), cols=cols)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M, N, K, group", [(4, 16, 259, 128), (33, 70, 1000, 96), (2, 5, 3, 2),
                                            (20, 64, 512, 4), (1, 3, 1, 1), (64, 257, 4096, 128)])
def test_matmul_simt_general_shapes(dtype, M, N, K, group):
    packed, scales, _ = _quantized(N, K, group, seed=K, dist="student_t3", zero_group_frac=0.05)
    x = make_activations(M, K, seed=M + K, device=DEV, dtype=dtype)
    y = q4.int4_matmul(x, packed, scales, K, group)
    assert_matmul_close(y, x, packed, scales, K, group, _tol(dtype))


@pytest.mark.parametrize("path", [q4.PATH_SIMT, q4.PATH_DECODE])
def test_matmul_one_hot_x_is_exact(path):
    N, K, group = 96, 512, 128
    packed, scales, _ = _quantized(N, K, group, seed=9, dist="student_t3", zero_group_frac=0.2)
    w_hat = oracle.dequantize_int4(packed.cpu().numpy(), scales.cpu().numpy(), K, group)
    ks = [0, 1, 127, 128, 300, 511]
    x = torch.zeros(len(ks), K, device=DEV, dtype=torch.bfloat16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = q4.int4_matmul(x, packed, scales, K, group, path=path).cpu().numpy().astype(np.float64)
    for i, k in enumerate(ks):
        assert np.array_equal(y[i], w_hat[:, k]), (path, k)


@pytest.mark.parametrize("path", [q4.PATH_SIMT, q4.PATH_DECODE])
def test_matmul_hand_made_bytes_row_sums(path):
    N, K, group = 40, 256, 64
    packed = torch.full((N, K // 2), 0x11, dtype=torch.uint8, device=DEV)
    scales = torch.ones((N, K // group), dtype=torch.float16, device=DEV)
    x = make_activations(3, K, seed=12, device=DEV, dtype=torch.bfloat16)
    y = q4.int4_matmul(x, packed, scales, K, group, path=path)
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF)
    # All bytes 0x88 (every weight -8) with scale 1: y = -8 * row sums.
    packed.fill_(0x88)
    y = q4.int4_matmul(x, packed, scales, K, group, path=path)
    expect = -8.0 * to_np(x).astype(np.float64).sum(1)
    np.testing.assert_allclose(y.cpu().numpy(), np.repeat(expect[:, None], N, 1), rtol=1e-5, atol=1e-4)


def test_matmul_decode_is_deterministic_and_matches_simt():
    packed, scales, _ = _quantized(4096, 4096, 128, seed=1)
    x = make_activations(4, 4096, seed=2, device=DEV, dtype=torch.bfloat16)
    a = q4.int4_matmul(x, packed, scales, 4096, 128, path=q4.PATH_DECODE)
    b = q4.int4_matmul(x, packed, scales, 4096, 128, path=q4.PATH_DECODE)
    c = q4.int4_matmul(x, packed, scales, 4096, 128, path=q4.PATH_SIMT)
    assert torch.equal(a, b)
    rel = ((a - c).abs().max() / c.abs().max()).item()
    assert rel < 1e-4


@pytest.mark.parametrize("M, N, K, group", [
    (1, 128, 8192, 128),     # one row tile over up to 64 CTAs: every run is a partial tile
    (3, 256, 16384, 64),     # two tiles, many runs inside each
    (16, 64, 4096, 32),      # 64-row tiles, one tile
    (8, 1000, 12288, 128),   # ragged last tile, runs cross tile boundaries
    (2, 37, 4096, 256),      # a single short tile, group spanning two blocks
    (5, 6000, 1024, 128),    # many tiles, runs of whole tiles plus boundary pieces
    (4, 20000, 2048, 128),   # the integer kernel with digit records, split runs
    (1, 30001, 1024, 256),   # the integer kernel, x converted in the CTA, ragged
    (3, 40000, 1024, 64),    # the 16-bit kernel, group 64, split runs
    (16, 30001, 1024, 32),   # the 16-bit kernel, group 32, 64-row tiles, ragged
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_matmul_decode_split_tiles(M, N, K, group, dtype):
    """Decode work split into equal runs of (row tile, K block) units, with the
    partial tiles summed afterwards: shapes whose runs start and end inside
    tiles, many runs per tile, and ragged tiles."""
    packed, scales, _ = _quantized(N, K, group, seed=N + K, dist="student_t3", zero_group_frac=0.02)
    x = make_activations(M, K, seed=M + K, device=DEV, dtype=dtype)
    a = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_DECODE)
    b = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_DECODE)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert_matmul_close(a, x, packed, scales, K, group, _tol(dtype))


@pytest.mark.parametrize("M", [1, 5])   # x converted in the matmul; x digits from their own kernel
def test_decode_sees_weights_rewritten_just_before(M):
    """The decode kernels launch as programmatic dependents of the preceding
    kernel and ask L2 to prefetch their first weight tiles before waiting for
    it: a quantize that rewrites the same buffers right before each call,
    with no synchronization, must still be what the matmul reads."""
    N, K, group = 20000, 4096, 128
    ws = [make_weights(N, K, seed=s, device=DEV, dtype=torch.bfloat16) for s in (21, 22)]
    packed, scales, _ = q4.quantize_int4(ws[0], group)
    x = make_activations(M, K, seed=9, device=DEV, dtype=torch.bfloat16)
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(M).integers(0, N, 400)]))
    ys = []
    for i in range(4):
        q4.quantize_int4(ws[(i + 1) % 2], group, packed=packed, scales=scales)
        ys.append((q4.int4_matmul(x, packed, scales, K, group), (i + 1) % 2))
    torch.cuda.synchronize()
    for y, j in ys[-2:]:
        p_j, s_j, _ = q4.quantize_int4(ws[j], group)
        assert_matmul_close(y, x, p_j, s_j, K, group, TOL_HALF, cols=cols)
    assert not torch.equal(ys[-1][0], ys[-2][0])


def _wide_range_x(M, K, dtype, seed, outlier=2.0 ** 12, tiny=2.0 ** -14):
    """N(0, 1) activations with outlier columns (x outlier) and tiny ones (x tiny)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g)
    x[:, torch.randint(0, K, (max(K // 64, 1),), generator=g)] *= outlier
    x[:, torch.randint(0, K, (max(K // 16, 1),), generator=g)] *= tiny
    return x.to(dtype).to(DEV)


# Decode kernels by matrix height: N = 512 keeps its packed tiles resident
# in shared memory (bf16 expansion); N = 20000 takes the integer tensor-core
# kernel (x as digits: converted in the CTA at M <= 2, by the digits kernel
# above).
DECODE_KERNEL_N = [512, 20000]


def _cols(N, seed):
    if N <= 2048:
        return None
    return np.unique(np.concatenate([[0, N - 1], np.random.default_rng(seed).integers(0, N, 600)]))


@pytest.mark.parametrize("N", DECODE_KERNEL_N)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16])
def test_matmul_decode_x_dynamic_range(N, dtype, M):
    """The integer decode kernel represents each 128-k block of a batch row as
    integers relative to the block's largest |x|: blocks holding outlier
    features 2^12 above the typical value, and values 2^14 below it, must
    still meet the bound (on both decode kernels)."""
    K, group = 2048, 128
    packed, scales, _ = _quantized(N, K, group, seed=7, dist="student_t3", zero_group_frac=0.05)
    x = _wide_range_x(M, K, dtype, seed=M)
    y = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_DECODE)
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, cols=_cols(N, M))


@pytest.mark.parametrize("N", DECODE_KERNEL_N)
@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("scale", [2.0 ** -90, 2.0 ** -60, 2.0 ** 60, 2.0 ** 100])
def test_matmul_decode_extreme_magnitudes_bf16(N, M, scale):
    """bf16 activations far from 1 in both directions (whole rows scaled)."""
    K, group = 1024, 256
    packed, scales, _ = _quantized(N, K, group, seed=11)
    x = (make_activations(M, K, seed=5, device=DEV, dtype=torch.float32) * scale).to(torch.bfloat16)
    y = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_DECODE)
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, cols=_cols(N, M))


@pytest.mark.parametrize("M, N, K, group", [
    (1, 20000, 8224, 128),   # last 128-k block holds 32 k; 65 blocks (odd): a stage past the end
    (2, 9000, 8352, 256),    # groups of two blocks, the last one partial
    (3, 8000, 4128, 128),    # digits kernel, ragged last block
    (16, 8000, 1056, 384),   # groups of three blocks, 9 blocks in all
    (1, 7200, 384, 128),     # three blocks: a run of one and a half stages
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_matmul_decode_integer_kernel_ragged_k(M, N, K, group, dtype):
    """The integer decode kernel on K that is not a multiple of 128 or of the
    256-k stage, and on groups spanning several 128-k blocks."""
    assert q4.matmul_select(dtype, K, group, M, N) == q4.PATH_DECODE
    packed, scales, _ = _quantized(N, K, group, seed=K + M, dist="student_t3", zero_group_frac=0.02)
    x = make_activations(M, K, seed=K, device=DEV, dtype=dtype)
    y = q4.int4_matmul(x, packed, scales, K, group)
    a = q4.int4_matmul(x, packed, scales, K, group)
    torch.cuda.synchronize()
    assert torch.equal(y, a)
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, cols=_cols(N, K))


@pytest.mark.parametrize("N", [300, 20000])   # the small-matrix and the streaming kernel
def test_matmul_decode_nonfinite_x_poisons_only_its_row(N):
    K, group = 1024, 128
    packed, scales, _ = _quantized(N, K, group, seed=4)
    x = make_activations(3, K, seed=6, device=DEV, dtype=torch.bfloat16)
    x[1, 200] = float("inf")
    y = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_DECODE)
    assert not torch.isfinite(y[1]).any()
    assert_matmul_close(y[[0, 2]], x[[0, 2]], packed, scales, K, group, TOL_HALF)


@pytest.mark.parametrize("layer", LLAMA7B_DECODE_LINEARS, ids=lambda l: l.name)
@pytest.mark.parametrize("M", [1, 4, 16])
def test_matmul_llama7b_decode_full_size(layer, M):
    packed, scales, _ = _quantized(layer.N, layer.K, layer.group, seed=3)
    x = make_activations(M, layer.K, seed=3 + M, device=DEV, dtype=torch.bfloat16)
    assert q4.matmul_select(torch.bfloat16, layer.K, layer.group, M, layer.N) == q4.PATH_DECODE
    y = q4.int4_matmul(x, packed, scales, layer.K, layer.group)
    assert_matmul_close(y, x, packed, scales, layer.K, layer.group, TOL_HALF)


@pytest.mark.parametrize("layer", DISTILGPT2_LINEARS, ids=lambda l: l.name)
@pytest.mark.parametrize("M", [1, 1024])
def test_matmul_distilgpt2(layer, M):
    packed, scales, _ = _quantized(layer.N, layer.K, layer.group, seed=2)
    x = make_activations(M, layer.K, seed=2 + M, device=DEV, dtype=torch.float16)
    y = q4.int4_matmul(x, packed, scales, layer.K, layer.group)
    assert_matmul_close(y, x, packed, scales, layer.K, layer.group, TOL_HALF)   # every output


def test_matmul_zero_group_contributes_nothing():
    case = tiny_case()
    w = torch.from_numpy(case["w"]).to(DEV)
    packed, scales, K = q4.quantize_int4(w, 128)
    x = torch.zeros(1, K, device=DEV)
    x[0, 128:256] = 1.0                         # only row 3's zero group is hit
    y = q4.int4_matmul(x, packed, scales, K, 128)
    assert float(y[0, 3]) == 0.0


# ---------------------------------------------------------------------------
# Failure path: a bounded device-side wait gives up and reports it.
# ---------------------------------------------------------------------------
def test_bounded_wait_reports_timeout_and_context_survives():
    assert q4.device_status() == q4.OK
    q4.selftest_wait_timeout(2000)
    assert q4.device_status() == q4.ERR_TIMEOUT
    assert q4.device_status() == q4.OK          # cleared by the read
    packed, scales, _ = _quantized(64, 256, 64, seed=1)
    x = make_activations(2, 256, seed=1, device=DEV, dtype=torch.bfloat16)
    y = q4.int4_matmul(x, packed, scales, 256, 64)
    assert_matmul_close(y, x, packed, scales, 256, 64, TOL_HALF)


@pytest.mark.parametrize("N, Ma, Mb", [
    (1000, 3, 5),   # the small-matrix kernel
    (9000, 3, 5),   # the integer kernel, x digits in per-stream records
    (9000, 1, 2),   # the integer kernel, x converted in the CTA
])
def test_decode_split_scratch_on_concurrent_streams(N, Ma, Mb):
    """Split-tile decode on two streams at once: each stream has its own
    partial slots, arrival counters and x digit records, so both results
    match the oracle bound and equal a serial run bit for bit."""
    K, group = 12288, 128
    packed, scales, _ = _quantized(N, K, group, seed=77, dist="student_t3", zero_group_frac=0.02)
    xa = make_activations(Ma, K, seed=1, device=DEV, dtype=torch.bfloat16)
    xb = make_activations(Mb, K, seed=2, device=DEV, dtype=torch.bfloat16)
    ref_a = q4.int4_matmul(xa, packed, scales, K, group, path=q4.PATH_DECODE)
    ref_b = q4.int4_matmul(xb, packed, scales, K, group, path=q4.PATH_DECODE)
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    outs_a, outs_b = [], []
    for _ in range(8):
        with torch.cuda.stream(sa):
            outs_a.append(q4.int4_matmul(xa, packed, scales, K, group, path=q4.PATH_DECODE))
        with torch.cuda.stream(sb):
            outs_b.append(q4.int4_matmul(xb, packed, scales, K, group, path=q4.PATH_DECODE))
    torch.cuda.synchronize()
    assert q4.device_status() == q4.OK
    for o in outs_a:
        assert torch.equal(o, ref_a)
    for o in outs_b:
        assert torch.equal(o, ref_b)
    assert_matmul_close(ref_a, xa, packed, scales, K, group, TOL_HALF, cols=_cols(N, 5))
    assert_matmul_close(ref_b, xb, packed, scales, K, group, TOL_HALF, cols=_cols(N, 6))


@pytest.mark.parametrize("M", [1, 5])
def test_decode_split_scratch_grows_between_shapes(M):
    """A small split first, then a larger one on the same stream: the stream's
    scratch (and, at M = 5, its x digit records) grows and the counters stay
    consistent for both."""
    for N, K in [(128, 4096), (9000, 2048), (28672, 8192), (300, 8192), (9000, 4096)]:
        packed, scales, _ = _quantized(N, K, 128, seed=N, dist="normal")
        x = make_activations(M, K, seed=3, device=DEV, dtype=torch.bfloat16)
        y1 = q4.int4_matmul(x, packed, scales, K, 128, path=q4.PATH_DECODE)
        y2 = q4.int4_matmul(x, packed, scales, K, 128, path=q4.PATH_DECODE)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)
        cols = np.unique(np.random.default_rng(N).integers(0, N, 256))
        assert_matmul_close(y1, x, packed, scales, K, 128, TOL_HALF, cols=cols)
    assert q4.device_status() == q4.OK


# ---------------------------------------------------------------------------
# int4_dequantize: w_hat = q * s rounded once to the output type
# ---------------------------------------------------------------------------
def _oracle_w_hat_as(packed, scales, K, group, dtype):
    """The oracle's exact w_hat (fp64; every value is exact in fp32), rounded to
    nearest even into `dtype` by the library-independent casts of NumPy and
    PyTorch on the CPU."""
    w64 = oracle.dequantize_int4(packed.cpu().numpy(), scales.cpu().numpy(), K, group)
    w32 = w64.astype(np.float32)
    assert np.array_equal(w32.astype(np.float64), w64)
    return torch.from_numpy(w32).to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("N, K, group", [
    (16, 259, 128), (64, 4096, 128), (33, 1024, 32), (7, 96, 48), (5, 1001, 7), (300, 768, 64),
    (2, 16, 16), (1, 1, 1),
])
def test_dequantize_bit_exact(dtype, N, K, group):
    packed, scales, _ = _quantized(N, K, group, seed=N * K, dist="student_t3", zero_group_frac=0.05)
    w_hat = q4.dequantize_int4(packed, scales, K, group, dtype=dtype)
    assert w_hat.dtype == dtype and tuple(w_hat.shape) == (N, K)
    ref = _oracle_w_hat_as(packed, scales, K, group, dtype)
    got = w_hat.cpu()
    assert torch.equal(got.view(torch.int16 if dtype != torch.float32 else torch.int32),
                       ref.view(torch.int16 if dtype != torch.float32 else torch.int32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_dequantize_every_code_and_extreme_scales(dtype):
    """All 256 bytes (every code pair, -8 included) under scales spanning the
    fp16 range: subnormal scales, 1, and 65504 (where -8 * s overflows fp16
    to -inf), on the fast and the general kernel."""
    sc = [2.0 ** -24, 2.0 ** -14 * 1.5, 0.1, 1.0, 3.0, 1024.0, 65504.0, 0.0]
    for K, group in [(512, 64), (510, 51)]:       # flat kernel; general kernel
        N = len(sc)
        packed = (torch.arange(N * ((K + 1) // 2)) % 256).to(torch.uint8).view(N, -1).to(DEV)
        G = -(-K // group)
        scales = torch.tensor(sc, dtype=torch.float16)[:, None].repeat(1, G).to(DEV)
        w_hat = q4.dequantize_int4(packed, scales, K, group, dtype=dtype).cpu()
        ref = _oracle_w_hat_as(packed, scales, K, group, dtype)
        itype = torch.int16 if dtype != torch.float32 else torch.int32
        assert torch.equal(w_hat.view(itype), ref.view(itype))
        if dtype == torch.float16:
            assert bool(torch.isinf(w_hat[6]).any())
