"""GPU parity of the tcgen05 tensor-core matmul (the prefill path) against
the CPU oracle: |y - y_ref| <= 4e-3 * sum|x||w_hat| for bf16/fp16 x, on
shapes with ragged M, N and K tails, partial last groups, zero groups,
groups of 32 (two per pipeline stage) and of 96 (spanning stages), more
tiles than SMs, and the full-size prefill workloads (whole rows and columns
of y)."""

import numpy as np
import pytest
import torch

import dequant_gemm_int4_b200 as q4
import oracle
from gpu_util import TOL_HALF, assert_matmul_close, assert_matmul_lines
from workloads import PREFILL_LINEARS, make_activations, make_weights

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    q4.lib()
    assert q4.device_status() == q4.OK
    yield
    assert q4.device_status() == q4.OK


def _quantized(N, K, group, seed, dist="normal", zero_group_frac=0.0):
    w = make_weights(N, K, seed=seed, device=DEV, dtype=torch.float32, std=0.02, dist=dist,
                     zero_group_frac=zero_group_frac, group=group)
    return q4.quantize_int4(w, group)


def _run(M, N, K, group, dtype, seed=0, dist="normal", zero_group_frac=0.0, rows=None, cols=None):
    packed, scales, _ = _quantized(N, K, group, seed + 1, dist, zero_group_frac)
    x = make_activations(M, K, seed=seed + 2, device=DEV, dtype=dtype)
    y = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_PREFILL)
    assert q4.device_status() == q4.OK, "a bounded wait in the tensor-core kernel timed out"
    return assert_matmul_close(y, x, packed, scales, K, group, TOL_HALF, rows=rows, cols=cols)


def test_prefill_smallest_tile():
    _run(256, 128, 64, 64, torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M, N, K, group", [
    (256, 128, 128, 128), (256, 128, 1024, 128), (512, 256, 512, 64), (300, 200, 256, 128),
    (17, 130, 192, 64), (1000, 77, 4096, 128), (256, 128, 96, 64), (256, 128, 8224, 128),
    (513, 385, 640, 128), (64, 1000, 2048, 256), (257, 129, 3072, 3072),
    (300, 200, 96, 32), (500, 300, 1056, 32), (192, 128, 2016, 96), (1024, 2304, 768, 32),
    (2048, 2048, 512, 64), (4000, 1000, 256, 32),   # more tiles than SMs: several per CTA
])
def test_prefill_shapes(dtype, M, N, K, group):
    _run(M, N, K, group, dtype, seed=M + N + K)


def test_prefill_heavy_tailed_with_zero_groups():
    _run(384, 256, 2048, 64, torch.bfloat16, dist="student_t3", zero_group_frac=0.05)


def test_prefill_one_hot_x_is_exact():
    N, K, group = 256, 512, 128
    packed, scales, _ = _quantized(N, K, group, 9, "student_t3", 0.2)
    w_hat = oracle.dequantize_int4(packed.cpu().numpy(), scales.cpu().numpy(), K, group)
    ks = [0, 1, 63, 64, 127, 128, 300, 511]
    x = torch.zeros(256, K, device=DEV, dtype=torch.bfloat16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_PREFILL).cpu().numpy()
    for i, k in enumerate(ks):
        assert np.array_equal(y[i].astype(np.float64), w_hat[:, k]), k
    assert not y[len(ks):].any()


def test_prefill_matches_decode_and_simt():
    packed, scales, _ = _quantized(1024, 4096, 128, 3)
    x = make_activations(64, 4096, seed=4, device=DEV, dtype=torch.bfloat16)
    a = q4.int4_matmul(x, packed, scales, 4096, 128, path=q4.PATH_PREFILL)
    b = q4.int4_matmul(x, packed, scales, 4096, 128, path=q4.PATH_SIMT)
    c = q4.int4_matmul(x[:16], packed, scales, 4096, 128, path=q4.PATH_DECODE)
    scale = b.abs().max().item()
    assert (a - b).abs().max().item() < 1e-4 * scale
    assert (a[:16] - c).abs().max().item() < 1e-4 * scale
    d = q4.int4_matmul(x, packed, scales, 4096, 128, path=q4.PATH_PREFILL)
    assert torch.equal(a, d)                    # deterministic


def test_prefill_is_the_automatic_choice_for_large_m():
    assert q4.matmul_select(torch.bfloat16, 8192, 128, 2048, 8192) == q4.PATH_PREFILL
    assert q4.matmul_select(torch.float16, 768, 64, 1024, 2304) == q4.PATH_PREFILL
    assert q4.matmul_select(torch.float16, 768, 32, 1024, 2304) == q4.PATH_PREFILL


def test_prefill_group_32_one_hot_is_exact():
    """Group 32: two groups per 64-k stage, each with its own accumulator."""
    N, K, group = 256, 256, 32
    packed, scales, _ = _quantized(N, K, group, 5, "student_t3", 0.2)
    w_hat = oracle.dequantize_int4(packed.cpu().numpy(), scales.cpu().numpy(), K, group)
    ks = [0, 31, 32, 33, 63, 64, 95, 96, 200, 255]
    x = torch.zeros(192, K, device=DEV, dtype=torch.float16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_PREFILL).cpu().numpy()
    for i, k in enumerate(ks):
        assert np.array_equal(y[i].astype(np.float64), w_hat[:, k]), k


@pytest.mark.parametrize("layer", PREFILL_LINEARS, ids=lambda l: l.name)
@pytest.mark.parametrize("M", [2048, 8192])
def test_prefill_full_size_whole_rows_and_columns(layer, M):
    """The full-size prefill workloads: every output of 16 random activation
    rows (first and last included) and of 16 random weight rows."""
    rng = np.random.default_rng(M + layer.N)
    rows = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 14)]))
    cols = np.unique(np.concatenate([[0, layer.N - 1], rng.integers(0, layer.N, 14)]))
    packed, scales, _ = _quantized(layer.N, layer.K, layer.group, 5)
    x = make_activations(M, layer.K, seed=6, device=DEV, dtype=torch.bfloat16)
    assert q4.matmul_select(torch.bfloat16, layer.K, layer.group, M, layer.N) == q4.PATH_PREFILL
    y = q4.int4_matmul(x, packed, scales, layer.K, layer.group)
    assert q4.device_status() == q4.OK
    assert_matmul_lines(y, x, packed, scales, layer.K, layer.group, TOL_HALF, rows, cols)


@pytest.mark.parametrize("M, N, K, group, dtype", [
    (64, 4096, 4096, 128, torch.bfloat16),     # 32 tiles: K split in pieces
    (1024, 768, 3072, 32, torch.float16),      # distilgpt2 mlp c_proj shape, groups of 32
    (100, 1000, 2016, 96, torch.bfloat16),     # group 96: pieces of 3 stages, ragged M and N
    (256, 11008, 4096, 128, torch.bfloat16),   # 86 tiles: the estimate keeps it whole
    (768, 8192, 4096, 128, torch.bfloat16),    # 192 tiles: one whole wave, the other 44 in 3 pieces
    (700, 9000, 2048, 64, torch.float16),      # ragged tail tiles, groups of 64
])
def test_prefill_split_k_matches_oracle_and_unsplit(M, N, K, group, dtype):
    """With fewer tiles than SMs the binding's workspace lets the kernel cut
    K into pieces of whole groups, added in piece order by a second kernel:
    the same bound as the unsplit call, and the same bits on every call."""
    packed, scales, _ = _quantized(N, K, group, 13, "student_t3", 0.05)
    x = make_activations(M, K, seed=14, device=DEV, dtype=dtype)
    need = q4.matmul_workspace_size(dtype, K, group, M, N)
    y_split = q4.int4_matmul(x, packed, scales, K, group)
    y_plain = q4.int4_matmul(x, packed, scales, K, group, workspace=False)
    assert q4.device_status() == q4.OK
    cols = None if N <= 2048 else np.unique(np.random.default_rng(N).integers(0, N, 400))
    assert_matmul_close(y_split, x, packed, scales, K, group, TOL_HALF, cols=cols)
    assert_matmul_close(y_plain, x, packed, scales, K, group, TOL_HALF, cols=cols)
    assert torch.equal(y_split, q4.int4_matmul(x, packed, scales, K, group))   # deterministic
    if need == 0:
        assert torch.equal(y_split, y_plain)


@pytest.mark.parametrize("M, N, K, group, dtype", [
    (1, 4096, 4096, 128, torch.bfloat16),
    (5, 11008, 4096, 128, torch.float16),
    (16, 4096, 11008, 128, torch.bfloat16),
    (16, 768, 3072, 32, torch.float16),        # groups of 32: two per stage
    (32, 2304, 768, 64, torch.bfloat16),
    (9, 1000, 2016, 96, torch.bfloat16),       # ragged N, groups spanning stages
    (16, 300, 96, 32, torch.float16),          # K of one and a half stages
    (24, 28672, 1024, 128, torch.bfloat16),    # more tiles than SMs
])
def test_prefill_small_m(M, N, K, group, dtype):
    """M <= 32 forced onto the tensor-core kernel (one activation tile, rows
    past M zero-filled by the copies): with a workspace the tiles of a
    partial wave may be cut into K pieces, added in piece order; without one
    they run whole.  Both meet the bound and repeat bit for bit."""
    packed, scales, _ = _quantized(N, K, group, 21, "student_t3", 0.05)
    x = make_activations(M, K, seed=22, device=DEV, dtype=dtype)
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device=DEV)
    y_split = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_PREFILL, workspace=ws)
    y_plain = q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_PREFILL, workspace=False)
    assert q4.device_status() == q4.OK
    cols = None if N <= 2048 else np.unique(np.random.default_rng(N).integers(0, N, 500))
    assert_matmul_close(y_split, x, packed, scales, K, group, TOL_HALF, cols=cols)
    assert_matmul_close(y_plain, x, packed, scales, K, group, TOL_HALF, cols=cols)
    assert torch.equal(y_split, q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_PREFILL,
                                               workspace=ws))


def test_prefill_split_workspace_query():
    """32 tiles on a device of 148 SMs: every tile is split.  7168 tiles: 48
    whole waves, and the 64 tiles of the partial last wave cut in two (one
    128 x 256 slot of fp32 sums per piece).  148 tiles: one whole wave, no
    split."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert q4.matmul_workspace_size(torch.bfloat16, 4096, 128, 64, 4096) > 0
    need = q4.matmul_workspace_size(torch.bfloat16, 8192, 128, 8192, 28672)
    tail = 7168 % sms
    assert need == 0 or (need - 4096) % (128 * 256 * 4) == 0
    if sms == 148:
        assert need == 4096 + tail * 2 * 128 * 256 * 4
    assert q4.matmul_workspace_size(torch.bfloat16, 8192, 128, 256, 128 * sms) == 0


def test_split_prefill_leaves_decode_counters_alone():
    """One workspace serves both kernels: the split's partial sums lie past
    the arrival counters a decode call expects to find zero."""
    K, group = 4096, 128
    packed, scales, _ = _quantized(11008, K, group, 15)
    need = max(q4.matmul_workspace_size(torch.bfloat16, K, group, 4, 11008),
               q4.matmul_workspace_size(torch.bfloat16, K, group, 64, 4096))
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    xd = make_activations(4, K, seed=16, device=DEV, dtype=torch.bfloat16)
    y0 = q4.int4_matmul(xd, packed, scales, K, group, workspace=ws)
    pk2, sc2, _ = _quantized(4096, K, group, 17)
    xp = make_activations(64, K, seed=18, device=DEV, dtype=torch.bfloat16)
    yp = q4.int4_matmul(xp, pk2, sc2, K, group, workspace=ws)
    assert_matmul_close(yp, xp, pk2, sc2, K, group, TOL_HALF)
    y1 = q4.int4_matmul(xd, packed, scales, K, group, workspace=ws)
    assert q4.device_status() == q4.OK
    assert torch.equal(y0, y1)
