"""GPU parity of the asymmetric (affine) variant and of the matmul's fused
bias + ReLU epilogue, through the C ABI, against the CPU oracle.

Affine quantize and dequantize are bit-exact; the matmul meets
|y - y_ref| <= c sum_k |x||w_hat| with w_hat = (q - z) s, on every kernel
path; with the epilogue the bound carries over plus one fp32 rounding of
y + bias (ReLU is 1-Lipschitz)."""

import numpy as np
import pytest
import torch

import dequant_gemm_int4_b200 as q4
import oracle
from gpu_util import TOL_F32, TOL_HALF, to_np
from workloads import make_activations, make_weights

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


def _special_affine_weights(N, K, group, seed, dtype):
    """Heavy-tailed weights with constant, all-zero, all-positive and
    all-negative groups mixed in."""
    w = make_weights(N, K, seed=seed, device="cpu", dtype=torch.float32, dist="student_t3")
    G = -(-K // group)
    g = torch.Generator().manual_seed(seed)
    kind = torch.randint(0, 10, (N, G), generator=g)
    for n in range(N):
        for gi in range(G):
            sl = slice(gi * group, min((gi + 1) * group, K))
            k = int(kind[n, gi])
            if k == 0:
                w[n, sl] = 0.0
            elif k == 1:
                w[n, sl] = 0.0123
            elif k == 2:
                w[n, sl] = w[n, sl].abs() + 0.001
            elif k == 3:
                w[n, sl] = -w[n, sl].abs() - 0.001
    return w.to(dtype).to(DEV)


def _oracle_affine(w, group):
    wn = to_np(w)
    if wn.dtype == np.float16:
        wn = wn.astype(np.float32)
    return oracle.quantize_uint4_affine(wn, group)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N, K, group", [
    (16, 1024, 128), (40, 4096, 64), (33, 768, 32), (8, 512, 8), (5, 2048, 256), (7, 256, 16),
    (9, 259, 128), (6, 1001, 100), (3, 96, 48), (2, 5, 2), (1, 1, 1),
    # 16 weights per lane: a partial last group (K % group = 16) and a
    # partial last window; group 512 (32 lanes per group)
    (10, 1040, 128), (4, 4112, 512), (3, 1552, 64),
])
def test_quantize_affine_bit_exact(dtype, N, K, group):
    w = _special_affine_weights(N, K, group, seed=N * K + group, dtype=dtype)
    packed, scales, zeros, K2 = q4.quantize_int4_affine(w, group)
    assert K2 == K
    p_ref, s_ref, z_ref, _ = _oracle_affine(w, group)
    assert np.array_equal(scales.cpu().view(torch.int16).numpy().view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(zeros.cpu().numpy(), z_ref)
    assert np.array_equal(packed.cpu().numpy(), p_ref)


@pytest.mark.parametrize("group", [32, 128])
def test_quantize_affine_full_size_sampled_rows(group):
    """W [28672, 8192] bf16 (the bench's matrix): 512 rows spread over the
    matrix, bit-exact against the oracle on those rows (quantization is per
    row)."""
    N, K = 28672, 8192
    w = make_weights(N, K, seed=11, device=DEV, dtype=torch.bfloat16, dist="student_t3",
                     zero_group_frac=0.01, group=group)
    packed, scales, zeros, _ = q4.quantize_int4_affine(w, group)
    rows = np.linspace(0, N - 1, 512).astype(np.int64)
    idx = torch.as_tensor(rows, device=DEV)
    p_ref, s_ref, z_ref, _ = _oracle_affine(w.index_select(0, idx), group)
    assert np.array_equal(scales.index_select(0, idx).cpu().view(torch.int16).numpy().view(np.uint16),
                          s_ref.view(np.uint16))
    assert np.array_equal(zeros.index_select(0, idx).cpu().numpy(), z_ref)
    assert np.array_equal(packed.index_select(0, idx).cpu().numpy(), p_ref)


def _tie_weights(N, K, group, seed):
    """fp32 weights whose quotients w / s + z fall on, and one ulp either side
    of, the half-integers k + 1/2 that rint rounds to even: each group gets
    its extremes first, then values (k + 1/2 - z) s for its own scale s and
    zero point z, kept inside the extremes."""
    rng = np.random.default_rng(seed)
    w = np.zeros((N, K), dtype=np.float32)
    for n in range(N):
        for g0 in range(0, K, group):
            g1 = min(g0 + group, K)
            a = np.float32(rng.uniform(0.01, 1.0))    # -min
            b = np.float32(rng.uniform(0.01, 1.0))    # max
            s = np.float32(np.float16(np.float32(b + a) / np.float32(15)))
            z = float(np.clip(np.rint(np.float32(a / s)), 0, 15))
            vals = [np.float32(-a), np.float32(b)]
            for j in range(g1 - g0 - 2):
                t = np.float32((rng.integers(0, 15) + 0.5 - z) * float(s))
                t = [t, np.nextafter(t, np.float32(np.inf)), np.nextafter(t, np.float32(-np.inf))][j % 3]
                vals.append(np.float32(min(max(t, -a), b)))
            w[n, g0:g1] = np.array(vals[: g1 - g0], dtype=np.float32)
    return torch.from_numpy(w).to(DEV)


@pytest.mark.parametrize("exponents", [(0,), (-23, -25), ("subnormal",), (19,)])
def test_affine_scale_division_exhaustive_over_mantissas(exponents):
    """fp16(fp32(d / 15)) on every fp32 mantissa of the given binades (and on
    every subnormal): groups of two weights {0, d} have the range d, and the
    kernel's division by the constant 15 must equal the IEEE division the
    oracle uses, bit for bit.  The binades cover the fp16 subnormal and
    overflow boundaries of the scale."""
    mant = np.arange(1 << 23, dtype=np.uint32)
    parts = []
    for e in exponents:
        if e == "subnormal":
            parts.append(mant.view(np.float32))
        else:
            parts.append(((np.uint32(e + 127) << 23) | mant).view(np.float32))
    d = np.concatenate(parts)
    w = np.zeros((1, 2 * d.size), dtype=np.float32)
    w[0, 1::2] = d
    wt = torch.from_numpy(w).to(DEV)
    packed, scales, zeros, _ = q4.quantize_int4_affine(wt, 2)
    p_ref, s_ref, z_ref, _ = oracle.quantize_uint4_affine(w, 2)
    got = scales.cpu().view(torch.int16).numpy().view(np.uint16)[0]
    bad = np.flatnonzero(got != s_ref.view(np.uint16)[0])
    assert bad.size == 0, f"{bad.size} scales differ, first d = {d[bad[0]]!r}"
    assert np.array_equal(zeros.cpu().numpy(), z_ref)
    assert np.array_equal(packed.cpu().numpy(), p_ref)


@pytest.mark.parametrize("N, K, group", [(24, 4096, 128), (16, 1024, 32), (9, 1000, 100)])
def test_quantize_affine_ties_bit_exact(N, K, group):
    """Quotients on and next to the rounding ties: the codes must be those of
    the IEEE division, bit for bit."""
    w = _tie_weights(N, K, group, seed=N + K + group)
    packed, scales, zeros, _ = q4.quantize_int4_affine(w, group)
    p_ref, s_ref, z_ref, _ = _oracle_affine(w, group)
    assert np.array_equal(scales.cpu().view(torch.int16).numpy().view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(zeros.cpu().numpy(), z_ref)
    assert np.array_equal(packed.cpu().numpy(), p_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("N, K, group", [(64, 4096, 128), (33, 1000, 40), (16, 512, 32)])
def test_dequantize_affine_bit_exact(dtype, N, K, group):
    w = _special_affine_weights(N, K, group, seed=K, dtype=torch.float32)
    packed, scales, zeros, _ = q4.quantize_int4_affine(w, group)
    w_hat = q4.dequantize_int4(packed, scales, K, group, dtype=dtype, zeros=zeros).cpu()
    ref64 = oracle.dequantize_uint4_affine(packed.cpu().numpy(), scales.cpu().numpy(),
                                           zeros.cpu().numpy(), K, group)
    ref32 = ref64.astype(np.float32)
    assert np.array_equal(ref32.astype(np.float64), ref64)
    ref = torch.from_numpy(ref32).to(dtype)
    itype = torch.int16 if dtype != torch.float32 else torch.int32
    assert torch.equal(w_hat.view(itype), ref.view(itype))


def _check(y, x, packed, scales, zeros, K, group, c, bias=None, relu=False, cols=None):
    xn = to_np(x).astype(np.float64)
    pn, sn = packed.cpu().numpy(), scales.cpu().numpy()
    zn = None if zeros is None else zeros.cpu().numpy()
    if cols is not None:
        pn, sn = pn[cols], sn[cols]
        zn = None if zn is None else zn[cols]
        y = y[:, torch.as_tensor(cols, device=y.device)]
    if zn is None:
        yr = oracle.int4_matmul_ref(xn, pn, sn, K, group)
        bound = oracle.matmul_error_bound(xn, pn, sn, K, group, c)
    else:
        yr = oracle.uint4_affine_matmul_ref(xn, pn, sn, zn, K, group)
        bound = oracle.matmul_error_bound_affine(xn, pn, sn, zn, K, group, c)
    b = None
    if bias is not None:
        b = bias.cpu().numpy().astype(np.float64)
        if cols is not None:
            b = b[cols]
    ref = oracle.linear_epilogue_ref(yr, b, relu)
    tol = oracle.epilogue_error_bound(bound, yr, b)
    yn = y.cpu().numpy().astype(np.float64)
    err = np.abs(yn - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), f"error {err[worst]:.3e} > {tol[worst]:.3e} at {worst}"
    if relu:
        assert (yn >= 0).all()


# Shapes per kernel path: (M, N, K, group, path, workspace)
PATHS = [
    (1, 28672, 4096, 128, q4.PATH_DECODE, None),     # integer kernel, x converted in the CTA
    (2, 18000, 4096, 256, q4.PATH_DECODE, None),
    (5, 18000, 4096, 128, q4.PATH_DECODE, None),     # integer kernel, x digit records
    (16, 9000, 2048, 128, q4.PATH_DECODE, None),
    (4, 18000, 4096, 128, q4.PATH_DECODE, False),    # no workspace: the 16-bit kernel
    (3, 9000, 2048, 64, q4.PATH_DECODE, None),       # resident tiles, group 64
    (12, 5000, 2048, 32, q4.PATH_DECODE, None),      # resident tiles, group 32
    (3, 30000, 2048, 64, q4.PATH_DECODE, None),      # 16-bit kernel, group 64
    (12, 30000, 2048, 32, q4.PATH_DECODE, None),     # 16-bit kernel, group 32
    (4, 2048, 4096, 128, q4.PATH_DECODE, None),      # resident-tile kernel
    (16, 4096, 11008, 128, q4.PATH_DECODE, None),    # resident-tile kernel, two n-tiles
    (3, 2048, 32768, 128, q4.PATH_DECODE, None),     # small-matrix kernel (rows too long)
    (256, 512, 1024, 128, q4.PATH_PREFILL, None),    # tensor-core kernel, K split (4 tiles)
    (300, 384, 2048, 64, q4.PATH_PREFILL, None),
    (300, 384, 2048, 64, q4.PATH_PREFILL, False),    # tensor-core kernel, whole K
    (1024, 768, 3072, 32, q4.PATH_PREFILL, None),    # groups of 32, K split
    (16, 3000, 2048, 64, q4.PATH_PREFILL, None),     # tensor-core kernel at M <= 32
    (5, 1000, 1024, 128, q4.PATH_PREFILL, False),    # the same, whole K
    (7, 100, 259, 128, q4.PATH_SIMT, None),          # CUDA-core kernel (odd K)
]


@pytest.mark.parametrize("M, N, K, group, path, ws", PATHS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_matmul_affine_every_path(M, N, K, group, path, ws, dtype):
    w = make_weights(N, K, seed=N + M, device=DEV, dtype=torch.float32, dist="student_t3",
                     zero_group_frac=0.02, group=group) + 0.004      # off-centre: z != 8
    packed, scales, zeros, _ = q4.quantize_int4_affine(w, group)
    assert int(zeros.max()) > 8 or int(zeros.min()) < 7
    x = make_activations(M, K, seed=K + M, device=DEV, dtype=dtype)
    y = q4.int4_matmul(x, packed, scales, K, group, zeros=zeros, path=path, workspace=ws)
    cols = None if N <= 2048 else np.unique(np.random.default_rng(N).integers(0, N, 600))
    _check(y, x, packed, scales, zeros, K, group, _tol(dtype), cols=cols)


@pytest.mark.parametrize("M, N, K, group, path, ws", PATHS)
@pytest.mark.parametrize("affine", [False, True])
def test_matmul_bias_relu_every_path(M, N, K, group, path, ws, affine):
    w = make_weights(N, K, seed=N * 3 + M, device=DEV, dtype=torch.float32)
    if affine:
        packed, scales, zeros, _ = q4.quantize_int4_affine(w, group)
    else:
        (packed, scales, _), zeros = q4.quantize_int4(w, group), None
    x = make_activations(M, K, seed=M, device=DEV, dtype=torch.bfloat16)
    bias = torch.randn(N, generator=torch.Generator().manual_seed(N)).mul_(0.5).to(DEV)
    cols = None if N <= 2048 else np.unique(np.random.default_rng(M).integers(0, N, 500))
    for b, relu in ((bias, False), (None, True), (bias, True)):
        y = q4.int4_matmul(x, packed, scales, K, group, zeros=zeros, bias=b, relu=relu, path=path,
                           workspace=ws)
        _check(y, x, packed, scales, zeros, K, group, TOL_HALF, bias=b, relu=relu, cols=cols)
        if relu:
            assert float((y == 0).float().mean()) > 0.2      # about half the outputs clip


def test_matmul_relu_keeps_nan():
    """ReLU after the bias keeps NaN (as max(v, 0) in IEEE arithmetic does)."""
    N, K, group = 512, 1024, 128
    packed, scales, _ = q4.quantize_int4(make_weights(N, K, seed=1, device=DEV), group)
    x = make_activations(2, K, seed=2, device=DEV, dtype=torch.bfloat16)
    x[1, 10] = float("nan")
    y = q4.int4_matmul(x, packed, scales, K, group, relu=True)
    assert torch.isnan(y[1]).all() and not torch.isnan(y[0]).any()


def test_affine_decode_bound_with_large_x_on_zero_weights():
    """The affine counterpart of the adversarial decode case: every weight of a
    group codes to its zero point (w_hat = 0) except one, and the block's
    largest |x| sits on a zero weight."""
    N, K, group = 8192, 2048, 128
    w = torch.zeros(N, K)
    rows = torch.arange(N)
    pos = 1 + rows % (group - 1)
    for g0 in range(0, K, group):
        w[rows, g0 + pos] = 7.0
        w[rows, g0] = -8.0 * (1 + (rows % 3).float()) / 16   # makes z > 0; its own w_hat != 0
    packed, scales, zeros, _ = q4.quantize_int4_affine(w.to(DEV), group)
    w_hat = oracle.dequantize_uint4_affine(packed.cpu().numpy(), scales.cpu().numpy(),
                                           zeros.cpu().numpy(), K, group)
    assert (w_hat[:, 1:group] != 0).sum(axis=1).max() == 1
    for M in (1, 4):
        x = torch.full((M, K), 2.0 ** -23 * (1 + 2.0 ** -7), dtype=torch.float64)
        x[:, 2::group] = 1.0                                  # the largest value, on a zero weight
        x = x.to(torch.bfloat16).to(DEV)
        y = q4.int4_matmul(x, packed, scales, K, group, zeros=zeros)
        _check(y, x, packed, scales, zeros, K, group, TOL_HALF)


# ---------------------------------------------------------------------------
# Int4Linear: the nn.Module drop-in
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("scheme", ["symmetric", "affine"])
@pytest.mark.parametrize("relu", [False, True])
def test_int4_linear_from_linear(scheme, relu):
    torch.manual_seed(0)
    lin = torch.nn.Linear(768, 2304).to(DEV)
    layer = q4.Int4Linear.from_linear(lin, group=64, scheme=scheme, relu=relu)
    x = torch.randn(3, 5, 768, device=DEV, dtype=torch.bfloat16)
    y = layer(x)
    assert y.shape == (3, 5, 2304) and y.dtype == torch.bfloat16
    y32 = q4.int4_matmul(x.reshape(15, 768), layer.packed, layer.scales, 768, 64, zeros=layer.zeros,
                         bias=layer.bias, relu=relu)
    assert torch.equal(y.reshape(15, 2304), y32.to(torch.bfloat16))
    _check(y32, x.reshape(15, 768), layer.packed, layer.scales, layer.zeros, 768, 64, TOL_HALF,
           bias=layer.bias, relu=relu)


def test_int4_linear_two_layer_model_and_state_dict():
    """The inference engine page's end-to-end shape (256 -> 128 with ReLU ->
    10) with both layers quantized, each checked against the oracle on the
    input it received; the buffers round-trip through state_dict."""
    torch.manual_seed(42)
    l1, l2 = torch.nn.Linear(256, 128).to(DEV), torch.nn.Linear(128, 10).to(DEV)
    q1 = q4.Int4Linear.from_linear(l1, group=128, scheme="affine", relu=True, out_dtype=torch.float32)
    q2 = q4.Int4Linear.from_linear(l2, group=128, scheme="affine", out_dtype=torch.float32)
    x = torch.randn(4, 256, device=DEV)
    h = q1(x)
    y = q2(h)
    _check(h, x, q1.packed, q1.scales, q1.zeros, 256, 128, TOL_F32, bias=q1.bias, relu=True)
    _check(y, h, q2.packed, q2.scales, q2.zeros, 128, 128, TOL_F32, bias=q2.bias)
    q3 = q4.Int4Linear(128, 10, group=128, scheme="affine")
    q3.load_state_dict(q2.state_dict())
    assert torch.equal(q3(h).float(), y)
    assert set(q2.state_dict()) == {"packed", "scales", "zeros", "bias"}


def test_sharded_layer_one_rank_uses_the_library():
    """Without a process group the sharded layer is one rank holding every
    row: the library's fused matmul, bias and ReLU, no collective."""
    from dequant_gemm_int4_b200.sharded import ShardedInt4Linear, shard_quantized
    N, K, group = 3000, 1024, 64
    w = make_weights(N, K, seed=9, device=DEV, dtype=torch.float32)
    packed, scales, zeros, _ = q4.quantize_int4_affine(w, group)
    bias = torch.randn(N, generator=torch.Generator().manual_seed(1)).to(DEV)
    p, s, z, b = shard_quantized(packed, scales, zeros, bias, 1, 0)
    layer = ShardedInt4Linear(p, s, z, b, in_features=K, out_features=N, group=group, relu=True)
    x = make_activations(4, K, seed=4, device=DEV, dtype=torch.bfloat16)
    y = layer(x)
    assert torch.equal(y, q4.int4_matmul(x, packed, scales, K, group, zeros=zeros, bias=bias,
                                         relu=True))
    _check(y, x, packed, scales, zeros, K, group, TOL_HALF, bias=bias, relu=True)
