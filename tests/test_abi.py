"""Host-side tests of the C-ABI library: it builds, loads, exports every
symbol the header declares, and rejects bad arguments before launching
anything.  No test here needs a GPU."""

import ctypes
import os
import re

import pytest

import dequant_gemm_int4_b200 as q4
from dequant_gemm_int4_b200 import build as q4build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "int4.h")


@pytest.fixture(scope="module")
def L():
    q4build.build()
    return q4.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(int4_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_page_functions():
    names = declared_functions()
    for n in ("int4_quantize", "int4_unpack", "int4_matmul", "int4_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert isinstance(getattr(L, name), ctypes._CFuncPtr)


def test_version(L):
    assert L.int4_version() == 10000


def test_quantize_rejects_bad_arguments_without_launching(L):
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert L.int4_quantize(fake, 7, 4, 4, 4, fake, fake, None) == q4.ERR_DTYPE
    assert L.int4_quantize(fake, 0, -1, 4, 4, fake, fake, None) == q4.ERR_ARG
    assert L.int4_quantize(fake, 0, 4, 0, 4, fake, fake, None) == q4.ERR_ARG
    assert L.int4_quantize(fake, 0, 4, 4, 0, fake, fake, None) == q4.ERR_ARG
    assert L.int4_quantize(None, 0, 4, 4, 4, fake, fake, None) == q4.ERR_ARG
    assert L.int4_quantize(fake, 0, 4, 4, 4, fake, None, None) == q4.ERR_ARG
    assert L.int4_quantize(ctypes.c_void_p(258), 0, 4, 4, 4, fake, fake, None) == q4.ERR_ALIGN
    assert L.int4_quantize(fake, 0, 4, 4, 4, fake, ctypes.c_void_p(257), None) == q4.ERR_ALIGN
    assert L.int4_quantize(fake, 0, 1 << 40, 1 << 30, 4, fake, fake, None) == q4.ERR_ARG
    assert b"w_dtype" in L.int4_last_error() or True
    # Empty problem: nothing to do, success, nothing launched.
    assert L.int4_quantize(None, 0, 0, 4, 4, None, None, None) == q4.OK


def test_unpack_rejects_bad_arguments(L):
    fake = ctypes.c_void_p(256)
    assert L.int4_unpack(fake, 0, 4, fake, None) == q4.ERR_ARG
    assert L.int4_unpack(fake, 4, -2, fake, None) == q4.ERR_ARG
    assert L.int4_unpack(None, 4, 4, fake, None) == q4.ERR_ARG
    assert L.int4_unpack(fake, 4, 4, None, None) == q4.ERR_ARG
    assert L.int4_unpack(None, 4, 0, None, None) == q4.OK


def test_matmul_rejects_bad_arguments(L):
    fake = ctypes.c_void_p(256)
    args = dict(x=fake, t=1, p=fake, s=fake, K=64, g=32, M=2, N=3, y=fake)

    def call(**kw):
        a = dict(args, **kw)
        return L.int4_matmul(a["x"], a["t"], a["p"], a["s"], a["K"], a["g"], a["M"], a["N"],
                             a["y"], None)

    assert call(t=9) == q4.ERR_DTYPE
    assert call(K=0) == q4.ERR_ARG
    assert call(g=0) == q4.ERR_ARG
    assert call(M=-1) == q4.ERR_ARG
    assert call(x=None) == q4.ERR_ARG
    assert call(s=None) == q4.ERR_ARG
    assert call(x=ctypes.c_void_p(257)) == q4.ERR_ALIGN
    assert call(y=ctypes.c_void_p(258)) == q4.ERR_ALIGN
    assert call(M=0) == q4.OK
    assert call(N=0) == q4.OK
    msg = L.int4_last_error()
    assert isinstance(msg, bytes)
    rc = L.int4_matmul_path(fake, 1, fake, fake, 64, 32, 2, 3, fake, 42, None, 0, None)
    assert rc == q4.ERR_ARG


def test_matmul_ws_rejects_bad_workspaces_before_launching(L):
    """The workspace entry checks its workspace on the host: a null workspace
    with a non-zero size, and one that is not 256-byte aligned."""
    fake = ctypes.c_void_p(256)
    f = L.int4_matmul_ws
    assert f(fake, 1, fake, fake, 4096, 128, 1, 8192, fake, None, 4096, None) == q4.ERR_ARG
    assert b"workspace" in L.int4_last_error()
    assert f(fake, 1, fake, fake, 4096, 128, 1, 8192, fake, ctypes.c_void_p(256 + 16), 4096,
             None) == q4.ERR_ALIGN
    assert b"256" in L.int4_last_error()
    # Argument checks come first, as for int4_matmul.
    assert f(None, 1, fake, fake, 4096, 128, 1, 8192, fake, fake, 4096, None) == q4.ERR_ARG
    assert f(fake, 5, fake, fake, 4096, 128, 1, 8192, fake, fake, 4096, None) == q4.ERR_DTYPE
    assert f(fake, 1, fake, fake, 4096, 128, 0, 8192, fake, None, 0, None) == q4.OK   # no work


def test_workspace_size_rejects_bad_arguments(L):
    out = ctypes.c_size_t(123)
    q = L.int4_matmul_workspace_size
    assert q(1, 4096, 128, 1, 8192, None) == q4.ERR_ARG
    assert q(7, 4096, 128, 1, 8192, ctypes.byref(out)) == q4.ERR_DTYPE
    assert q(1, 0, 128, 1, 8192, ctypes.byref(out)) == q4.ERR_ARG
    assert q(1, 4096, 0, 1, 8192, ctypes.byref(out)) == q4.ERR_ARG
    assert q(1, 4096, 128, -1, 8192, ctypes.byref(out)) == q4.ERR_ARG
    assert q(1, 1 << 40, 128, 1 << 30, 8192, ctypes.byref(out)) == q4.ERR_ARG
    # Paths that use no scratch need no workspace, and need no GPU to say so.
    for args in [(0, 4096, 128, 1, 8192),        # fp32 x: the CUDA-core kernel
                 (1, 4096, 128, 8192, 8192),     # the tensor-core kernel with tiles to spare
                 (1, 4100, 128, 1, 8192),        # K % 32 != 0
                 (1, 4096, 128, 0, 8192)]:       # empty
        out.value = 123
        assert q(*args, ctypes.byref(out)) == q4.OK
        assert out.value == 0
    # The tensor-core kernel with fewer tiles (64) than SMs splits K into
    # pieces whose fp32 sums live in the workspace, past 4 KB of counters,
    # one 128-row tile slot each (148 SMs assumed without a device).
    out.value = 0
    assert q(1, 4096, 128, 64, 8192, ctypes.byref(out)) == q4.OK
    assert out.value > 4096 and (out.value - 4096) % (128 * 128 * 4) == 0


def test_noalloc_rejects_what_the_decode_kernels_cannot_run(L):
    """The allocation-free entry validates and refuses on the host, before any
    CUDA call: shapes outside the decode kernels, and bad arguments."""
    fake = ctypes.c_void_p(256)
    f = L.int4_matmul_decode_noalloc
    assert f(fake, 1, fake, fake, 4096, 128, 17, 64, fake, None) == q4.ERR_UNSUPPORTED  # M > 16
    assert b"decode" in L.int4_last_error()
    assert f(fake, 0, fake, fake, 4096, 128, 2, 64, fake, None) == q4.ERR_UNSUPPORTED   # fp32 x
    assert f(fake, 1, fake, fake, 4112, 128, 2, 64, fake, None) == q4.ERR_UNSUPPORTED   # K % 32
    assert f(fake, 1, fake, fake, 4096, 96, 2, 64, fake, None) == q4.ERR_UNSUPPORTED    # group 96
    assert f(ctypes.c_void_p(264), 1, fake, fake, 4096, 128, 2, 64, fake, None) == q4.ERR_UNSUPPORTED
    assert f(None, 1, fake, fake, 4096, 128, 2, 64, fake, None) == q4.ERR_ARG
    assert f(fake, 1, fake, fake, 4096, 128, 2, 64, None, None) == q4.ERR_ARG
    assert f(fake, 9, fake, fake, 4096, 128, 2, 64, fake, None) == q4.ERR_DTYPE
    assert f(fake, 1, fake, fake, 4096, 128, 0, 64, fake, None) == q4.OK                # no work


def test_error_message_is_set(L):
    fake = ctypes.c_void_p(256)
    assert L.int4_unpack(fake, 0, 4, fake, None) == q4.ERR_ARG
    assert b"int4_unpack" in L.int4_last_error()


@pytest.mark.parametrize("dt, K, group, M, N, want", [
    (0, 259, 128, 4, 16, q4.PATH_SIMT),        # fp32 x: the CUDA-core kernel
    (1, 4096, 128, 1, 4096, q4.PATH_DECODE),    # bf16 decode
    (2, 768, 32, 1, 2304, q4.PATH_DECODE),      # fp16 decode, group 32
    (1, 4096, 64, 16, 11008, q4.PATH_DECODE),
    (1, 259, 128, 4, 16, q4.PATH_SIMT),         # odd K
    (1, 4096, 4, 1, 64, q4.PATH_SIMT),          # group 4
    (1, 4096, 96, 1, 64, q4.PATH_SIMT),         # group not 32/64/128k
])
def test_kernel_selection(L, dt, K, group, M, N, want):
    assert L.int4_matmul_select(dt, K, group, M, N) == want


def test_python_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(TypeError):
        q4.quantize_int4(torch.zeros(4, 8), 4)
    with pytest.raises(TypeError):
        q4.unpack_int4(torch.zeros(4, 4, dtype=torch.uint8), 8)


@pytest.mark.parametrize("fn", ["int4_matmul", "int4_matmul_decode_noalloc"])
def test_matmul_bindings_check_operand_shapes_before_anything_runs(fn):
    """Both matmul wrappers refuse wrong-shaped or wrong-typed operands before
    reaching the library (the C side sees only pointers), and refuse CPU
    tensors of the right shapes: there is no CPU path."""
    import torch
    K, group, N, M = 256, 128, 8, 2
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    packed = torch.zeros(N, K // 2, dtype=torch.uint8)
    scales = torch.zeros(N, 2, dtype=torch.float16)
    out = torch.zeros(M, N)
    f = getattr(q4, fn)

    def call(**kw):
        a = dict(dict(x=x, packed=packed, scales=scales, out=out), **kw)
        if fn == "int4_matmul":
            return f(a["x"], a["packed"], a["scales"], K, group, out=a["out"])
        return f(a["x"], a["packed"], a["scales"], K, group, a["out"])

    for bad in (torch.zeros(N, 1, dtype=torch.float16), torch.zeros(N - 1, 2, dtype=torch.float16),
                torch.zeros(N, 2, dtype=torch.float32), torch.zeros(N * 2, dtype=torch.float16)):
        with pytest.raises(ValueError, match="scales"):
            call(scales=bad)
    for bad in (torch.zeros(N, K // 2 - 1, dtype=torch.uint8), torch.zeros(N, K // 2, dtype=torch.int8),
                torch.zeros(N * K // 2, dtype=torch.uint8)):
        with pytest.raises(ValueError, match="packed"):
            call(packed=bad)
    with pytest.raises(ValueError, match="x must"):
        call(x=torch.zeros(M, K + 2, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out"):
        call(out=torch.zeros(M, N + 1))
    with pytest.raises(TypeError, match="CUDA"):
        call()
