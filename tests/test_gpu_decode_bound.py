"""The decode matmul on activations built to break a block-scaled integer
form of x, and the matmul's workspace contract, through the C ABI.

The integer decode kernel writes each 128-k block of a batch row as integers
times one power of two, which is exact only where every value of the block is
an integer multiple of 2^-29 times the block's largest power of two.  Blocks
where that fails are computed with the 16-bit products instead.  The cases
here put the large values of each block on zero weights and the small,
inexact ones on the only non-zero weight of the group, so that any rounding
of the small values shows up against sum |x||w_hat| undiluted.
"""

import ctypes

import numpy as np
import pytest
import torch

import dequant_gemm_int4_b200 as q4
import oracle
from gpu_util import TOL_HALF, assert_matmul_close, to_np
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


# Per dtype: a large value and a small one whose block-scaled integer form
# (29 bits below the large value's exponent) lands exactly half-way between
# two integers, so rounding it loses 2^-30 of the block maximum: for bf16
# 2^-23 (1 + 2^-7) under 1.0 (relative error 2^-7), for fp16 2^-9 (1 + 2^-6)
# under 2^15 (relative error 2^-6); both above the 4e-3 tolerance.
ADVERSARIAL = {torch.bfloat16: (1.0, 2.0 ** -23 * (1 + 2.0 ** -7)),
               torch.float16: (2.0 ** 15, 2.0 ** -9 * (1 + 2.0 ** -6))}


def _weights_off_the_block_start(N, K, group):
    """Row n: 7 at column 1 + (n mod (group - 1)) of every group, zero
    elsewhere (column 0 of each group is always zero); quantizes to scale 1."""
    w = torch.zeros(N, K)
    rows = torch.arange(N)
    pos = 1 + rows % (group - 1)
    for g0 in range(0, K, group):
        cols = g0 + pos
        ok = cols < K
        w[rows[ok], cols[ok]] = 7.0
    return q4.quantize_int4(w.to(DEV), group)


def _adversarial_x(M, K, dtype):
    big, tiny = ADVERSARIAL[dtype]
    x = torch.full((M, K), tiny, dtype=torch.float64)
    x[:, ::128] = big                       # the block's largest value, on a zero weight
    # Rows at other scales (powers of two, within fp16's normal range).
    x *= (2.0 ** -(torch.arange(M, dtype=torch.float64) % 4))[:, None]
    return x.to(dtype).to(DEV)


def _block_integer_form(x64, K):
    """x rounded to integers times 2^(e-29) per 128-k block (e: the exponent
    of the block's largest |x|), the representation the integer kernel uses
    where it is exact."""
    out = x64.copy()
    for b0 in range(0, K, 128):
        blk = out[:, b0:b0 + 128]
        m = np.abs(blk).max(axis=1)
        e = np.floor(np.log2(np.where(m > 0, m, 1.0)))
        step = 2.0 ** (e - 29)
        out[:, b0:b0 + 128] = np.rint(blk / step[:, None]) * step[:, None]
    return out


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M", [1, 2, 4, 16])
@pytest.mark.parametrize("mode", ["workspace", "no_workspace", "noalloc"])
@pytest.mark.parametrize("N", [8192, 20000])   # M > 2: resident tiles, then the integer kernel
def test_decode_bound_with_large_x_on_zero_weights(dtype, M, mode, N):
    K, group = 2048, 128
    assert q4.matmul_select(dtype, K, group, M, N) == q4.PATH_DECODE
    packed, scales, _ = _weights_off_the_block_start(N, K, group)
    x = _adversarial_x(M, K, dtype)
    xn = to_np(x).astype(np.float64)
    pn, sn = packed.cpu().numpy(), scales.cpu().numpy()
    # The case is adversarial: x rounded to its block-scaled integer form
    # breaks the bound on every output.
    ref = oracle.int4_matmul_ref(xn, pn, sn, K, group)
    bound = oracle.matmul_error_bound(xn, pn, sn, K, group, TOL_HALF)
    rounded = oracle.int4_matmul_ref(_block_integer_form(xn, K), pn, sn, K, group)
    assert (np.abs(rounded - ref) > bound).all()
    if mode == "noalloc":
        y = torch.empty((M, N), dtype=torch.float32, device=DEV)
        q4.int4_matmul_decode_noalloc(x, packed, scales, K, group, y)
    else:
        y = q4.int4_matmul(x, packed, scales, K, group,
                           workspace=None if mode == "workspace" else False)
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF)


@pytest.mark.parametrize("M", [1, 2, 5, 16])
@pytest.mark.parametrize("N", [9000, 20000])   # M > 2: resident tiles, then the integer kernel
def test_decode_blocks_flagged_in_some_rows_only(M, N):
    """Only some batch rows of some blocks are wide; every row of such a block
    takes the 16-bit products, the other blocks stay on the integer form, and
    the whole output meets the bound."""
    K, group = 4096, 256
    packed, scales, _ = q4.quantize_int4(
        make_weights(N, K, seed=31, device=DEV, dtype=torch.float32, dist="student_t3",
                     zero_group_frac=0.02, group=group), group)
    g = torch.Generator().manual_seed(M)
    x = torch.randn(M, K, generator=g, dtype=torch.float64)
    for m in range(0, M, 2):                # even rows: a few blocks hold a tiny value
        blocks = torch.randint(0, K // 128, (3,), generator=g)
        for b in blocks.tolist():
            x[m, b * 128 + 5] = 2.0 ** -40 * (1 + 2.0 ** -7)
    x = x.to(torch.bfloat16).to(DEV)
    y = q4.int4_matmul(x, packed, scales, K, group)
    cols = np.unique(np.random.default_rng(M).integers(0, N, 700))
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, cols=cols)


@pytest.mark.parametrize("N", [11008, 18000])
def test_decode_silu_like_activations(N):
    """Activations shaped like a gated MLP's (x sigmoid(x) of wide normals):
    values down to about 1e-12 next to values near 20 in the same block, on
    the resident-tile kernel (N = 11008) and the integer one (N = 18000)."""
    K, group, M = 4096, 128, 4
    packed, scales, _ = q4.quantize_int4(
        make_weights(N, K, seed=5, device=DEV, dtype=torch.float32), group)
    z = make_activations(M, K, seed=8, device=DEV, dtype=torch.float32) * 8.0
    x = (z * torch.sigmoid(z)).to(torch.bfloat16)
    cols = np.unique(np.random.default_rng(1).integers(0, N, 800))
    for ws in (None, False):
        y = q4.int4_matmul(x, packed, scales, K, group, workspace=ws)
        assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, cols=cols)


# ---------------------------------------------------------------------------
# Workspace contract of int4_matmul_ws
# ---------------------------------------------------------------------------
def _call_ws(x, packed, scales, K, group, y, ws, nbytes):
    L = q4.lib()
    return L.int4_matmul_ws(x.data_ptr(), 1, packed.data_ptr(), scales.data_ptr(), K, group,
                            x.shape[0], packed.shape[0], y.data_ptr(),
                            None if ws is None else ws.data_ptr(), nbytes,
                            torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M, N, K, group", [
    (1, 28672, 8192, 128),    # split tiles, x converted in the matmul
    (4, 18000, 4096, 128),    # split tiles and x digit records
    (16, 20000, 4096, 128),
    (3, 30000, 2048, 64),     # the 16-bit kernel, split
])
def test_workspace_size_is_enforced_and_sufficient(M, N, K, group):
    need = q4.matmul_workspace_size(torch.bfloat16, K, group, M, N)
    assert need > 0
    packed, scales, _ = q4.quantize_int4(
        make_weights(N, K, seed=N, device=DEV, dtype=torch.float32), group)
    x = make_activations(M, K, seed=M, device=DEV, dtype=torch.bfloat16)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    y = torch.full((M, N), 7.0, dtype=torch.float32, device=DEV)
    L = q4.lib()
    # One byte short, or no workspace given a size: refused before launching.
    assert _call_ws(x, packed, scales, K, group, y, ws, need - 1) == q4.ERR_ARG
    assert b"workspace" in L.int4_last_error()
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
    # Exactly the size: two calls in a row, same bits, counters left zero.
    for _ in range(2):
        assert _call_ws(x, packed, scales, K, group, y, ws, need) == q4.OK
        y2 = torch.empty_like(y)
        assert _call_ws(x, packed, scales, K, group, y2, ws, need) == q4.OK
        torch.cuda.synchronize()
        assert torch.equal(y, y2)
    assert int(ws[:4096].view(torch.int32).abs().sum()) == 0      # the counter region
    cols = np.unique(np.random.default_rng(N).integers(0, N, 600))
    assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, cols=cols)


@pytest.mark.parametrize("M, N, K, group", [
    (1, 28672, 8192, 128), (2, 18000, 4096, 128), (4, 18000, 4096, 128), (16, 20000, 4096, 128),
    (8, 9000, 2048, 64), (12, 5000, 2048, 32), (1, 4096, 4096, 128), (4, 11008, 4096, 128),
    (8, 30000, 2048, 64), (2, 30000, 2048, 32),
])
def test_matmul_without_workspace(M, N, K, group):
    """int4_matmul (no workspace): runs of whole row tiles, and at M > 2 the
    16-bit kernel; it meets the bound and agrees with the workspace schedule
    up to summation order."""
    packed, scales, _ = q4.quantize_int4(
        make_weights(N, K, seed=K + M, device=DEV, dtype=torch.float32, dist="student_t3",
                     zero_group_frac=0.02, group=group), group)
    x = make_activations(M, K, seed=N, device=DEV, dtype=torch.bfloat16)
    y0 = torch.empty((M, N), dtype=torch.float32, device=DEV)
    L = q4.lib()
    rc = L.int4_matmul(x.data_ptr(), 1, packed.data_ptr(), scales.data_ptr(), K, group, M, N,
                       y0.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == q4.OK
    y1 = q4.int4_matmul(x, packed, scales, K, group)                 # with a workspace
    torch.cuda.synchronize()
    cols = np.unique(np.random.default_rng(M).integers(0, N, 600))
    assert_matmul_close(y0, x, packed, scales, K, group, TOL_HALF, cols=cols)
    assert_matmul_close(y1, x, packed, scales, K, group, TOL_HALF, cols=cols)
    assert float((y0 - y1).abs().max()) <= 1e-3 * float(y1.abs().max())


def test_workspace_shared_by_shapes_on_one_stream():
    """One zero-filled workspace, large enough for every call, serves calls of
    different shapes (different CTA counts and regions) back to back."""
    shapes = [(1, 28672, 8192, 128), (16, 20000, 4096, 128), (4, 18000, 4096, 128),
              (2, 9000, 12288, 128), (3, 9000, 2048, 64), (1, 4096, 4096, 128)]
    need = max(q4.matmul_workspace_size(torch.bfloat16, K, g, M, N) for M, N, K, g in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    cases = []
    for M, N, K, g in shapes:
        packed, scales, _ = q4.quantize_int4(
            make_weights(N, K, seed=N + M, device=DEV, dtype=torch.float32), g)
        x = make_activations(M, K, seed=K, device=DEV, dtype=torch.bfloat16)
        cases.append((x, packed, scales, K, g))
    outs = [[q4.int4_matmul(x, p, s, K, g, workspace=ws) for (x, p, s, K, g) in cases]
            for _ in range(3)]
    torch.cuda.synchronize()
    for r in range(1, 3):
        for a, b in zip(outs[0], outs[r]):
            assert torch.equal(a, b)
    for (x, p, s, K, g), y in zip(cases, outs[0]):
        cols = np.unique(np.random.default_rng(K).integers(0, p.shape[0], 300))
        assert_matmul_close(y, x, p, s, K, g, TOL_HALF, cols=cols)
