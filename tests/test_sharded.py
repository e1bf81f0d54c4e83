"""The weight-row-sharded layer's host logic on CPU: the row partition, the
per-row independence that lets each rank hold the slices of a whole-matrix
quantization, and the forward pass on two and three gloo ranks with the
oracle standing in for the local matmul (the library needs a GPU; the
sharding and the gather are what is under test here)."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from dequant_gemm_int4_b200.sharded import shard_quantized, shard_rows

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N", [0, 1, 7, 8, 4096, 11008, 28673])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_rows_is_a_balanced_partition(N, world):
    spans = [shard_rows(N, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_quantization_is_per_row():
    """Quantizing a slice of rows gives the rows of the whole quantization,
    for both schemes: the shards are the whole matrix's bytes."""
    rng = np.random.default_rng(3)
    w = rng.standard_t(3, size=(37, 300)).astype(np.float32) * 0.02
    full = oracle.quantize_int4(w, 64)
    fa = oracle.quantize_uint4_affine(w, 64)
    for world in (2, 3):
        for r in range(world):
            a, b = shard_rows(37, world, r)
            part = oracle.quantize_int4(w[a:b], 64)
            assert np.array_equal(part[0], full[0][a:b]) and np.array_equal(part[1], full[1][a:b])
            pa = oracle.quantize_uint4_affine(w[a:b], 64)
            for i in range(3):
                assert np.array_equal(pa[i], fa[i][a:b])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_matmul(x, packed, scales, K, group, zeros, bias, relu):
    xn = x.numpy().astype(np.float64)
    if zeros is None:
        y = oracle.int4_matmul_ref(xn, packed.numpy(), scales.numpy(), K, group)
    else:
        y = oracle.uint4_affine_matmul_ref(xn, packed.numpy(), scales.numpy(), zeros.numpy(), K,
                                           group)
    y = oracle.linear_epilogue_ref(y, None if bias is None else bias.numpy(), relu)
    return torch.from_numpy(y.astype(np.float32))


def _worker(rank, world, port, scheme, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from dequant_gemm_int4_b200.sharded import ShardedInt4Linear, shard_quantized

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N, K, group = 29, 96, 32
        rng = np.random.default_rng(11)                    # same draw on every rank
        w = rng.normal(size=(N, K)).astype(np.float32)
        bias = rng.normal(size=N).astype(np.float32)
        x = rng.normal(size=(2, 3, K)).astype(np.float32)
        if scheme == "affine":
            packed, scales, zeros, _ = oracle.quantize_uint4_affine(w, group)
        else:
            (packed, scales, _), zeros = oracle.quantize_int4(w, group), None
        t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
        p, s, z, b = shard_quantized(t(packed), t(scales), t(zeros), t(bias), world, rank)
        layer = ShardedInt4Linear(p, s, z, b, in_features=K, out_features=N, group=group,
                                  relu=True, matmul=_oracle_matmul)
        y = layer(torch.from_numpy(x))
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("scheme", ["symmetric", "affine"])
def test_sharded_forward_on_gloo_ranks(world, scheme):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, scheme, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = dict(q.get(timeout=5) for _ in range(world))
    # The whole layer, unsharded, in one process.
    N, K, group = 29, 96, 32
    rng = np.random.default_rng(11)
    w = rng.normal(size=(N, K)).astype(np.float32)
    bias = rng.normal(size=N).astype(np.float32)
    x = rng.normal(size=(2, 3, K)).astype(np.float32)
    if scheme == "affine":
        packed, scales, zeros, _ = oracle.quantize_uint4_affine(w, group)
        y = oracle.uint4_affine_matmul_ref(x.reshape(6, K), packed, scales, zeros, K, group)
    else:
        packed, scales, _ = oracle.quantize_int4(w, group)
        y = oracle.int4_matmul_ref(x.reshape(6, K), packed, scales, K, group)
    want = oracle.linear_epilogue_ref(y, bias, True).astype(np.float32).reshape(2, 3, N)
    for r in range(world):
        assert got[r].shape == (2, 3, N)
        assert np.array_equal(got[r], want), r


def test_shard_quantized_slices_match_shard_rows():
    packed = torch.arange(10 * 4, dtype=torch.uint8).view(10, 4)
    scales = torch.arange(10 * 2, dtype=torch.float16).view(10, 2)
    bias = torch.arange(10, dtype=torch.float32)
    p, s, z, b = shard_quantized(packed, scales, None, bias, 3, 1)
    assert z is None and torch.equal(p, packed[4:7]) and torch.equal(s, scales[4:7])
    assert torch.equal(b, bias[4:7])
