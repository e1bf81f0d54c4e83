"""The allocation-free decode entry point against the regular one.

Collected last (file name), so it also runs after every other GPU test has
used the regular path on the same device."""

import numpy as np
import pytest
import torch

import dequant_gemm_int4_b200 as q4
from gpu_util import TOL_HALF, assert_matmul_close
from workloads import make_activations, make_weights

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("M, N, K, group, dtype", [
    (1, 28672, 8192, 128, torch.bfloat16),   # partial tiles at most run ends
    (4, 4096, 4096, 128, torch.bfloat16),    # resident tiles: no scratch at all
    (1, 2048, 32768, 128, torch.bfloat16),   # the small-matrix kernel: no scratch at all
    (4, 18000, 4096, 128, torch.bfloat16),   # x digits (two n-tiles) and split tiles
    (8, 28672, 4096, 128, torch.bfloat16),   # x digits (four n-tiles), 64-row tiles
    (16, 20000, 4096, 128, torch.bfloat16),  # x digits in the static array
    (2, 18000, 4096, 256, torch.float16),    # x converted inside the matmul
    (16, 1000, 12288, 64, torch.float16),    # 64-row tiles, ragged last tile
    (3, 37, 4096, 32, torch.bfloat16),       # a single short tile
    (16, 30000, 2048, 64, torch.float16),    # the 16-bit kernel, split tiles
])
def test_noalloc_matches_regular_entry(M, N, K, group, dtype):
    w = make_weights(N, K, seed=N + K, device=DEV, dtype=torch.float32, dist="student_t3",
                     zero_group_frac=0.01, group=group)
    packed, scales, _ = q4.quantize_int4(w, group)
    del w
    x = make_activations(M, K, seed=M + 3, device=DEV, dtype=dtype)
    ref = [q4.int4_matmul(x, packed, scales, K, group, path=q4.PATH_DECODE) for _ in range(2)]
    outs = [torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV) for _ in range(2)]
    for o in outs:                         # two calls in a row
        q4.int4_matmul_decode_noalloc(x, packed, scales, K, group, o)
    torch.cuda.synchronize()
    assert q4.device_status() == q4.OK
    for r, o in zip(ref, outs):
        assert torch.equal(r, o)           # same kernels, same split, same bits
    cols = np.unique(np.random.default_rng(N).integers(0, N, 512))
    assert_matmul_close(outs[1], x, packed, scales, K, group, TOL_HALF, cols=cols)


def test_noalloc_rejects_shapes_the_decode_kernel_cannot_run():
    K, group, N = 4096, 128, 256
    w = make_weights(N, K, seed=1, device=DEV, dtype=torch.float32)
    packed, scales, _ = q4.quantize_int4(w, group)
    x = make_activations(17, K, seed=1, device=DEV, dtype=torch.bfloat16)   # M > 16
    out = torch.empty((17, N), dtype=torch.float32, device=DEV)
    with pytest.raises(q4.Int4Error) as ei:
        q4.int4_matmul_decode_noalloc(x, packed, scales, K, group, out)
    assert ei.value.code == q4.ERR_UNSUPPORTED


def test_noalloc_rejects_x_digits_beyond_the_static_array():
    """At M = 16 the x digit records of K = 65536 (513 blocks of 8320 bytes)
    exceed the 4 MiB the array keeps for them: the call is refused on the
    host before anything launches."""
    M, N, K, group = 16, 7200, 65536, 128
    packed = torch.zeros((N, K // 2), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((N, K // group), dtype=torch.float16, device=DEV)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=DEV)
    out = torch.full((M, N), 7.0, dtype=torch.float32, device=DEV)
    with pytest.raises(q4.Int4Error) as ei:
        q4.int4_matmul_decode_noalloc(x, packed, scales, K, group, out)
    assert ei.value.code == q4.ERR_ARG
    assert "scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())        # nothing ran
