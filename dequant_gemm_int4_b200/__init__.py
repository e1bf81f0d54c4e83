"""B200 (sm_100a) INT4 weight-only quantization and dequantizing matmul.

Thin Python binding over the C-ABI library ``libint4.so`` (declared in
``include/int4.h``).  It only marshals arguments: it allocates the output
tensors with PyTorch on the input's CUDA device, passes raw device pointers
and the current CUDA stream, and raises on a non-zero status.  Every step of
the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and a missing library is an error.

The three functions keep the names, argument order and layouts of the page
"Implement INT4 group quantization, nibble packing and a dequantizing
matmul" (problem statement):

* ``quantize_int4(w, group=128) -> (packed, scales, K)``
* ``unpack_int4(packed, K) -> int8 [N, K]``
* ``int4_matmul(x, packed, scales, K, group=128) -> float32 [M, N]``
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "quantize_int4", "unpack_int4", "dequantize_int4", "int4_matmul", "int4_matmul_decode_noalloc",
    "quantize_int4_affine", "EPI_RELU",
    "matmul_workspace_size", "matmul_select", "device_status",
    "selftest_wait_timeout", "lib", "library_path", "Int4Error",
    "PATH_AUTO", "PATH_SIMT", "PATH_DECODE", "PATH_PREFILL",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libint4.so")

OK, ERR_ARG, ERR_DTYPE, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = range(7)
DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2
PATH_AUTO, PATH_SIMT, PATH_DECODE, PATH_PREFILL = 0, 1, 2, 3
EPI_RELU = 1

_DTYPE_CODE = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}

_lock = threading.Lock()
_lib = None


class Int4Error(RuntimeError):
    """A non-zero status from the INT4 library."""

    def __init__(self, code: int, message: str):
        super().__init__(f"INT4 library error {code}: {message}")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libint4.so once and declare its C signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m dequant_gemm_int4_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, u32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32
        L.int4_quantize.argtypes = [vp, i32, i64, i64, i32, vp, vp, vp]
        L.int4_unpack.argtypes = [vp, i64, i64, vp, vp]
        L.int4_dequantize.argtypes = [vp, vp, i64, i32, i64, vp, i32, vp]
        L.int4_quantize_affine.argtypes = [vp, i32, i64, i64, i32, vp, vp, vp, vp]
        L.int4_dequantize_affine.argtypes = [vp, vp, vp, i64, i32, i64, vp, i32, vp]
        sz = ctypes.c_size_t
        L.int4_matmul.argtypes = [vp, i32, vp, vp, i64, i32, i64, i64, vp, vp]
        L.int4_matmul_ws.argtypes = [vp, i32, vp, vp, i64, i32, i64, i64, vp, vp, sz, vp]
        L.int4_matmul_path.argtypes = [vp, i32, vp, vp, i64, i32, i64, i64, vp, i32, vp, sz, vp]
        L.int4_matmul_ex.argtypes = [vp, i32, vp, vp, vp, i64, i32, i64, i64, vp, i32, vp, i32, vp,
                                     sz, vp]
        L.int4_matmul_workspace_size.argtypes = [i32, i64, i32, i64, i64, ctypes.POINTER(sz)]
        L.int4_matmul_select.argtypes = [i32, i64, i32, i64, i64]
        L.int4_matmul_decode_noalloc.argtypes = [vp, i32, vp, vp, i64, i32, i64, i64, vp, vp]
        L.int4_device_status.argtypes = [vp]
        L.int4_selftest_wait_timeout.argtypes = [u32, vp]
        L.int4_last_error.restype = ctypes.c_char_p
        L.int4_last_error.argtypes = []
        L.int4_version.argtypes = []
        for name in ("int4_quantize", "int4_unpack", "int4_dequantize", "int4_matmul",
                     "int4_matmul_path", "int4_matmul_ex", "int4_quantize_affine",
                     "int4_dequantize_affine",
                     "int4_matmul_ws", "int4_matmul_workspace_size", "int4_matmul_decode_noalloc",
                     "int4_matmul_select", "int4_device_status", "int4_selftest_wait_timeout",
                     "int4_version"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
        return L


def _check(rc: int) -> None:
    if rc != OK:
        msg = lib().int4_last_error()
        raise Int4Error(rc, msg.decode() if msg else "")


# The current CUDA stream of a device as a raw handle: torch's own accessor
# when it has one (no Stream object is built), else the public API.
_raw_stream_fn = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _raw_stream(device_index: int) -> int:
    if _raw_stream_fn is not None:
        return _raw_stream_fn(device_index)
    return torch.cuda.current_stream(device_index).cuda_stream


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(_raw_stream(t.get_device()))


def _need_cuda(name: str, t: torch.Tensor) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major, no padding)")


def quantize_int4(w: torch.Tensor, group: int = 128, *, packed: torch.Tensor | None = None,
                  scales: torch.Tensor | None = None):
    """Quantize w [N, K] (fp32/bf16/fp16) -> (packed uint8 [N, ceil(K/2)], scales fp16 [N, G], K).

    `packed` and `scales`, if given, are written in place (same shapes and dtypes)."""
    _need_cuda("w", w)
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    if w.dtype not in _DTYPE_CODE:
        raise TypeError("w must be float32, bfloat16 or float16")
    N, K = w.shape
    G = -(-K // group) if group >= 1 else 0
    if packed is None:
        packed = torch.empty((N, (K + 1) // 2), dtype=torch.uint8, device=w.device)
    elif (packed.dtype != torch.uint8 or tuple(packed.shape) != (N, (K + 1) // 2)
          or not packed.is_contiguous() or packed.device != w.device):
        raise ValueError("packed must be contiguous uint8 [N, ceil(K/2)] on w's device")
    if scales is None:
        scales = torch.empty((N, max(G, 0)), dtype=torch.float16, device=w.device)
    elif (scales.dtype != torch.float16 or tuple(scales.shape) != (N, max(G, 0))
          or not scales.is_contiguous() or scales.device != w.device):
        raise ValueError("scales must be contiguous float16 [N, ceil(K/group)] on w's device")
    with torch.cuda.device(w.device):
        _check(lib().int4_quantize(w.data_ptr(), _DTYPE_CODE[w.dtype], N, K, int(group),
                                   packed.data_ptr(), scales.data_ptr(), _stream(w)))
    return packed, scales, K


def unpack_int4(packed: torch.Tensor, K: int) -> torch.Tensor:
    """Unpack packed [N, ceil(K/2)] -> sign-extended int8 [N, K]."""
    _need_cuda("packed", packed)
    if packed.dtype != torch.uint8 or packed.dim() != 2 or packed.shape[1] != (K + 1) // 2:
        raise ValueError("packed must be uint8 [N, ceil(K/2)]")
    N = packed.shape[0]
    out = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    with torch.cuda.device(packed.device):
        _check(lib().int4_unpack(packed.data_ptr(), K, N, out.data_ptr(), _stream(packed)))
    return out


def dequantize_int4(packed: torch.Tensor, scales: torch.Tensor, K: int, group: int = 128,
                    dtype: torch.dtype = torch.bfloat16, *,
                    zeros: torch.Tensor | None = None) -> torch.Tensor:
    """w_hat = q * s (or (q - z) * s with the affine scheme's `zeros`) as a
    dense [N, K] tensor of `dtype`, rounded to nearest even."""
    _need_cuda("packed", packed)
    _need_cuda("scales", scales)
    if packed.dtype != torch.uint8 or packed.dim() != 2 or packed.shape[1] != (K + 1) // 2:
        raise ValueError("packed must be uint8 [N, ceil(K/2)]")
    N = packed.shape[0]
    if group < 1 or scales.dtype != torch.float16 or tuple(scales.shape) != (N, -(-K // group)):
        raise ValueError("scales must be float16 [N, ceil(K/group)]")
    if dtype not in _DTYPE_CODE:
        raise TypeError("dtype must be float32, bfloat16 or float16")
    if scales.device != packed.device:
        raise ValueError("scales must be on packed's device")
    if zeros is not None:
        _need_cuda("zeros", zeros)
        if zeros.dtype != torch.uint8 or zeros.shape != scales.shape or zeros.device != packed.device:
            raise ValueError("zeros must be uint8 [N, ceil(K/group)] on packed's device")
    out = torch.empty((N, K), dtype=dtype, device=packed.device)
    with torch.cuda.device(packed.device):
        if zeros is None:
            _check(lib().int4_dequantize(packed.data_ptr(), scales.data_ptr(), K, int(group), N,
                                         out.data_ptr(), _DTYPE_CODE[dtype], _stream(packed)))
        else:
            _check(lib().int4_dequantize_affine(packed.data_ptr(), scales.data_ptr(),
                                                zeros.data_ptr(), K, int(group), N, out.data_ptr(),
                                                _DTYPE_CODE[dtype], _stream(packed)))
    return out


def quantize_int4_affine(w: torch.Tensor, group: int = 128):
    """The asymmetric variant: w [N, K] -> (packed uint8 [N, ceil(K/2)] of
    unsigned codes, scales fp16 [N, G], zeros uint8 [N, G], K)."""
    _need_cuda("w", w)
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    if w.dtype not in _DTYPE_CODE:
        raise TypeError("w must be float32, bfloat16 or float16")
    N, K = w.shape
    G = -(-K // group) if group >= 1 else 0
    packed = torch.empty((N, (K + 1) // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((N, max(G, 0)), dtype=torch.float16, device=w.device)
    zeros = torch.empty((N, max(G, 0)), dtype=torch.uint8, device=w.device)
    with torch.cuda.device(w.device):
        _check(lib().int4_quantize_affine(w.data_ptr(), _DTYPE_CODE[w.dtype], N, K, int(group),
                                          packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
                                          _stream(w)))
    return packed, scales, zeros, K


def _matmul_operands(x, packed, scales, K: int, group: int, out=None):
    """Checks the matmul's operands (shapes and dtypes first, then that every
    tensor is a contiguous CUDA tensor on x's device) and returns (M, N)."""
    for name, t in (("x", x), ("packed", packed), ("scales", scales)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError("x must be [M, K]")
    if x.dtype not in _DTYPE_CODE:
        raise TypeError("x must be float32, bfloat16 or float16")
    if group < 1:
        raise ValueError("group must be >= 1")
    if packed.dim() != 2:
        raise ValueError("packed must be uint8 [N, ceil(K/2)]")
    M, N = x.shape[0], packed.shape[0]
    if packed.dtype != torch.uint8 or tuple(packed.shape) != (N, (K + 1) // 2):
        raise ValueError("packed must be uint8 [N, ceil(K/2)]")
    if scales.dtype != torch.float16 or tuple(scales.shape) != (N, -(-K // group)):
        raise ValueError("scales must be float16 [N, ceil(K/group)]")
    if out is not None and (not isinstance(out, torch.Tensor) or out.dtype != torch.float32
                            or tuple(out.shape) != (M, N)):
        raise ValueError("out must be float32 [M, N]")
    dev = None
    for name, t in (("x", x), ("packed", packed), ("scales", scales), ("out", out)):
        if t is None:
            continue
        _need_cuda(name, t)
        d = t.get_device()
        if dev is None:
            dev = d
        elif d != dev:
            raise ValueError(f"{name} must be on x's device")
    return M, N


def matmul_workspace_size(x_dtype: torch.dtype, K: int, group: int, M: int, N: int,
                          device=None) -> int:
    """Bytes of workspace the matmul needs for this problem on `device` (0: none)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    key = (dev.index if dev.index is not None else torch.cuda.current_device(),
           x_dtype, int(K), int(group), int(M), int(N))
    n = _ws_size_cache.get(key)
    if n is None:
        out = ctypes.c_size_t(0)
        with torch.cuda.device(key[0]):
            _check(lib().int4_matmul_workspace_size(_DTYPE_CODE[x_dtype], K, int(group), M, N,
                                                    ctypes.byref(out)))
        n = _ws_size_cache[key] = int(out.value)
    return n


# Workspaces the binding keeps for the matmul, one per (device, stream):
# allocated zero-filled with torch on the stream that uses them (the kernels
# leave them zeroed after every call), grown when a call needs more.
_ws_size_cache: dict = {}
_ws_cache: dict = {}


def _workspace_for(x: torch.Tensor, nbytes: int, stream: int | None = None) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    dev = x.get_device()
    key = (dev, _raw_stream(dev) if stream is None else stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        # torch.zeros runs on the current stream, before the call that uses it.
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=x.device)
        _ws_cache[key] = ws
    return ws


def int4_matmul(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, K: int,
                group: int = 128, *, zeros: torch.Tensor | None = None,
                bias: torch.Tensor | None = None, relu: bool = False, path: int = PATH_AUTO,
                out: torch.Tensor | None = None, workspace: torch.Tensor | bool | None = None):
    """y = x @ dequantize(W).T as float32 [M, N]; x is [M, K] fp32/bf16/fp16.

    `zeros` (uint8 [N, G]): the affine scheme's zero points (codes from
    quantize_int4_affine); `bias` (float32 [N]) and `relu` apply to each
    output before it is stored.  `workspace`: None uses a zero-filled
    workspace the binding keeps per device and stream; a uint8 CUDA tensor
    (zero-filled before its first use, at least matmul_workspace_size bytes)
    is used as given; False runs the schedule that needs no workspace (the C
    entry int4_matmul)."""
    M, N = _matmul_operands(x, packed, scales, K, group, out)
    dev = x.get_device()
    if zeros is not None:
        _need_cuda("zeros", zeros)
        if zeros.dtype != torch.uint8 or zeros.shape != scales.shape or zeros.get_device() != dev:
            raise ValueError("zeros must be uint8 [N, ceil(K/group)] on x's device")
    if bias is not None:
        _need_cuda("bias", bias)
        if bias.dtype != torch.float32 or tuple(bias.shape) != (N,) or bias.get_device() != dev:
            raise ValueError("bias must be float32 [N] on x's device")
    if out is None:
        out = x.new_empty((M, N), dtype=torch.float32)
    L = _lib if _lib is not None else lib()
    same_dev = dev == torch.cuda.current_device()
    with (_nullctx() if same_dev else torch.cuda.device(dev)):
        stream = _raw_stream(dev)
        if workspace is False:
            ws_ptr, ws_bytes = None, 0
        elif workspace is None:
            key = (dev, x.dtype, int(K), int(group), int(M), int(N))
            nb = _ws_size_cache.get(key)
            if nb is None:
                nb = matmul_workspace_size(x.dtype, K, group, M, N, x.device)
            ws = _workspace_for(x, nb, stream)
            ws_ptr, ws_bytes = (ws.data_ptr(), ws.numel()) if ws is not None else (None, 0)
        else:
            _need_cuda("workspace", workspace)
            if workspace.dtype != torch.uint8 or workspace.device != x.device:
                raise ValueError("workspace must be a uint8 tensor on x's device")
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        if zeros is None and bias is None and not relu:
            _check(L.int4_matmul_path(x.data_ptr(), _DTYPE_CODE[x.dtype], packed.data_ptr(),
                                      scales.data_ptr(), K, int(group), M, N, out.data_ptr(),
                                      int(path), ws_ptr, ws_bytes, stream))
        else:
            _check(L.int4_matmul_ex(x.data_ptr(), _DTYPE_CODE[x.dtype], packed.data_ptr(),
                                    scales.data_ptr(), None if zeros is None else zeros.data_ptr(),
                                    K, int(group), M, N, None if bias is None else bias.data_ptr(),
                                    EPI_RELU if relu else 0, out.data_ptr(), int(path), ws_ptr,
                                    ws_bytes, stream))
    return out


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def int4_matmul_decode_noalloc(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                               K: int, group: int, out: torch.Tensor) -> torch.Tensor:
    """The decode matmul into a caller-provided `out` [M, N] float32, with no
    device allocation in the call (the library's fixed scratch holds the
    partial tiles).  Calls that may overlap in time race on that scratch."""
    if out is None:
        raise ValueError("out must be float32 [M, N]")
    M, N = _matmul_operands(x, packed, scales, K, group, out)
    with torch.cuda.device(x.device):
        _check(lib().int4_matmul_decode_noalloc(x.data_ptr(), _DTYPE_CODE[x.dtype],
                                                packed.data_ptr(), scales.data_ptr(), K,
                                                int(group), M, N, out.data_ptr(), _stream(x)))
    return out


def matmul_select(x_dtype: torch.dtype, K: int, group: int, M: int, N: int) -> int:
    """The kernel path int4_matmul takes for this problem (PATH_SIMT/DECODE/PREFILL)."""
    rc = lib().int4_matmul_select(_DTYPE_CODE[x_dtype], K, group, M, N)
    if rc < 0:
        _check(-rc)
    return rc


def device_status(device=None) -> int:
    """Synchronize the current stream and read/clear the device status word.

    Returns OK (0) or ERR_TIMEOUT (5); raises on a CUDA error."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        rc = lib().int4_device_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    if rc not in (OK, ERR_TIMEOUT):
        _check(rc)
    if rc == ERR_TIMEOUT:
        # A CTA that gave up may have left an arrival counted in a workspace:
        # start over with zero-filled ones on this device.
        idx = dev.index if dev.index is not None else torch.cuda.current_device()
        for key in [k for k in _ws_cache if k[0] == idx]:
            del _ws_cache[key]
    return rc


def selftest_wait_timeout(spins: int, device=None) -> None:
    """Launch the bounded-wait self-test kernel (its wait can never be satisfied)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib().int4_selftest_wait_timeout(
            int(spins), ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))


from .module import Int4Linear  # noqa: E402  (uses the functions above)

__all__.append("Int4Linear")
