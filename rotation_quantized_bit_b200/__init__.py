"""Python binding of the B200 ConvRot W4A4 quantized Linear (``libconvrot_b200.so``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/convrot.h``.  PyTorch supplies
device memory and streams.  There is no fallback: if the shared library is
missing or the device is not an sm_100 GPU, the calls raise.

The functions carry the C names:

    convrot_pack_weight(W)                  -> (Wq, s_w)
    convrot_rotate_quant(x)                 -> (xq, s_a)
    w4a4_gemm(xq, s_a, Wq, s_w, bias)       -> y   (bf16)
    w4a4_gemm_s32(xq, Wq, K)                -> acc (int32)
    w4a4_gemm_f32(xq, s_a, Wq, s_w, bias)   -> y32 (fp32)
    convrot_w4a4_linear(x, Wq, s_w, bias)   -> y   (bf16)
    convrot_w4a4_linear_f32(x, Wq, s_w, bias) -> y32 (fp32)

Tensors are torch CUDA tensors: bf16 as ``torch.bfloat16``, packed codes as
``torch.uint8`` [rows, K/2], scales ``torch.float32``.  Outputs may be passed
in (``out=``) or are allocated with torch; the workspace likewise.
"""
from __future__ import annotations

import ctypes
import functools
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libconvrot_b200.so")

STATUS = {
    0: "CONVROT_OK", 1: "CONVROT_ERR_NULL", 2: "CONVROT_ERR_SHAPE", 3: "CONVROT_ERR_ALIGN",
    4: "CONVROT_ERR_DEVICE", 5: "CONVROT_ERR_WORKSPACE", 6: "CONVROT_ERR_CUDA", 7: "CONVROT_ERR_TIMEOUT",
}

# Every symbol include/convrot.h declares (the tests check the export list).
EXPORTS = [
    "convrot_status_string", "convrot_pack_weight", "convrot_rotate_quant", "convrot_gemm_workspace_size",
    "w4a4_gemm", "w4a4_gemm_s32", "w4a4_gemm_f32", "convrot_w4a4_workspace_size", "convrot_w4a4_linear",
    "convrot_w4a4_linear_f32", "convrot_w4a4_linear_noalloc", "convrot_w4a4_quantize", "convrot_w4a4_gemm_quantized", "convrot_device_error",
    "convrot_dispatch_counts", "convrot_last_error", "convrot_selftest_timeout", "convrot_version",
    "convrot_measure_mma_i8",
    "w8a8_workspace_size", "w8a8_quantize", "w8a8_pack_weight", "w8a8_gemm", "w8a8_gemm_f32", "w8a8_gemm_s32",
    "w8a8_linear", "w8a8_linear_f32",
    "convrot_rotate_quant_g", "convrot_pack_weight_g", "convrot_w4a4_linear_g", "convrot_w4a4_linear_g_f32",
    "convrot_w4a4_quantize_g",
    "asym_w4a8_workspace_size", "asym_w4a8_gemm", "asym_w4a8_gemm_f32", "asym_w4a8_gemm_s32", "asym_w4a8_linear",
    "asym_w4a8_linear_f32",
]

# int8 formats (include/convrot.h, w8a8_format_t)
W8A8_INT8_TENSORWISE = 0
W8A8_CONVROT_INT8_ROW = 1


class ConvRotError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg}")
        self.code = code
        self.status = STATUS.get(code, str(code))


_lib = None


def load_library():
    """Load libconvrot_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m rotation_quantized_bit_b200.build` "
            "(nvcc, sm_100a). There is no CPU or fallback path.")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.convrot_status_string.argtypes = [I]
    lib.convrot_status_string.restype = ctypes.c_char_p
    lib.convrot_version.restype = ctypes.c_char_p
    lib.convrot_last_error.restype = ctypes.c_char_p
    lib.convrot_pack_weight.argtypes = [P, I, I, P, P, P]
    lib.convrot_rotate_quant.argtypes = [P, I, I, P, P, P]
    lib.convrot_gemm_workspace_size.argtypes = [I, I, I]
    lib.convrot_gemm_workspace_size.restype = Z
    lib.convrot_w4a4_workspace_size.argtypes = [I, I, I]
    lib.convrot_w4a4_workspace_size.restype = Z
    lib.w4a4_gemm.argtypes = [P, P, P, P, P, I, I, I, P, P, Z, P]
    lib.w4a4_gemm_s32.argtypes = [P, P, I, I, I, P, P, Z, P]
    lib.w4a4_gemm_f32.argtypes = [P, P, P, P, P, I, I, I, P, P, Z, P]
    lib.convrot_w4a4_linear.argtypes = [P, P, P, P, I, I, I, P, P, Z, P]
    lib.convrot_w4a4_linear_f32.argtypes = [P, P, P, P, I, I, I, P, P, Z, P]
    lib.convrot_w4a4_linear_noalloc.argtypes = [P, P, P, P, I, I, I, P, P]
    lib.convrot_w4a4_quantize.argtypes = [P, I, I, P, Z, P]
    lib.convrot_w4a4_gemm_quantized.argtypes = [P, P, P, I, I, I, P, P, Z, P]
    lib.convrot_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.convrot_selftest_timeout.argtypes = [ctypes.c_uint, P]
    lib.convrot_dispatch_counts.argtypes = [ctypes.POINTER(ctypes.c_uint64), I]
    lib.convrot_dispatch_counts.restype = None
    lib.convrot_measure_mma_i8.argtypes = [I, I, I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
    lib.convrot_rotate_quant_g.argtypes = [P, I, I, I, P, P, P]
    lib.convrot_w4a4_quantize_g.argtypes = [P, I, I, I, P, Z, P]
    lib.convrot_pack_weight_g.argtypes = [P, I, I, I, P, P, P]
    lib.convrot_w4a4_linear_g.argtypes = [P, P, P, P, I, I, I, I, P, P, Z, P]
    lib.convrot_w4a4_linear_g_f32.argtypes = [P, P, P, P, I, I, I, I, P, P, Z, P]
    lib.w8a8_workspace_size.argtypes = [I, I, I, I]
    lib.w8a8_workspace_size.restype = Z
    lib.w8a8_quantize.argtypes = [P, I, I, I, P, P, P, Z, P]
    lib.w8a8_pack_weight.argtypes = [P, I, I, I, P, P, P, Z, P]
    lib.w8a8_gemm.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
    lib.w8a8_gemm_f32.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
    lib.w8a8_gemm_s32.argtypes = [P, P, I, I, I, P, P]
    lib.w8a8_linear.argtypes = [P, P, P, P, I, I, I, I, P, P, Z, P]
    lib.w8a8_linear_f32.argtypes = [P, P, P, P, I, I, I, I, P, P, Z, P]
    lib.asym_w4a8_workspace_size.argtypes = [I, I, I]
    lib.asym_w4a8_workspace_size.restype = Z
    lib.asym_w4a8_gemm.argtypes = [P, P, P, P, P, P, P, I, I, I, P, P]
    lib.asym_w4a8_gemm_f32.argtypes = [P, P, P, P, P, P, P, I, I, I, P, P]
    lib.asym_w4a8_gemm_s32.argtypes = [P, P, P, P, I, I, I, P, P]
    lib.asym_w4a8_linear.argtypes = [P, P, P, P, P, P, I, I, I, P, P, Z, P]
    lib.asym_w4a8_linear_f32.argtypes = [P, P, P, P, P, P, I, I, I, P, P, Z, P]
    for name in lib_status_fns():
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def lib_status_fns():
    return ["convrot_pack_weight", "convrot_rotate_quant", "w4a4_gemm", "w4a4_gemm_s32", "w4a4_gemm_f32",
            "convrot_w4a4_linear", "convrot_w4a4_linear_f32", "convrot_w4a4_linear_noalloc", "convrot_w4a4_quantize",
            "convrot_w4a4_gemm_quantized", "convrot_device_error", "convrot_selftest_timeout",
            "convrot_measure_mma_i8", "w8a8_quantize", "w8a8_pack_weight", "w8a8_gemm", "w8a8_gemm_f32",
            "w8a8_gemm_s32", "w8a8_linear", "w8a8_linear_f32", "convrot_rotate_quant_g", "convrot_pack_weight_g",
            "convrot_w4a4_linear_g", "convrot_w4a4_linear_g_f32", "convrot_w4a4_quantize_g", "asym_w4a8_gemm",
            "asym_w4a8_gemm_f32", "asym_w4a8_gemm_s32", "asym_w4a8_linear", "asym_w4a8_linear_f32"]


def _check(fn: str, rc: int):
    if rc != 0:
        lib = load_library()
        msg = lib.convrot_status_string(rc).decode()
        last = lib.convrot_last_error().decode()
        raise ConvRotError(fn, rc, msg + (f" [{last}]" if last and rc == 6 else ""))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _one_device(fn):
    """Run a call with the device of its tensor arguments current.  Every
    tensor argument must be a CUDA tensor and all must be on one device
    (ValueError otherwise), and so must an explicit ``stream``; the default
    stream is then that device's current stream, and the library's device
    checks and launches refer to the same device."""
    @functools.wraps(fn)
    def wrapped(*args, **kwargs):
        dev = None
        for a in (*args, *kwargs.values()):
            if not isinstance(a, torch.Tensor):
                continue
            if not a.is_cuda:
                raise ValueError(f"{fn.__name__}: every tensor must be a CUDA tensor, got one on {a.device}")
            if dev is None:
                dev = a.device
            elif a.device != dev:
                raise ValueError(f"{fn.__name__}: tensors on {dev} and {a.device}; all must be on one device")
        if dev is None:
            return fn(*args, **kwargs)
        for a in (*args, *kwargs.values()):
            if isinstance(a, torch.cuda.Stream) and a.device != dev:
                raise ValueError(f"{fn.__name__}: stream on {a.device}, tensors on {dev}")
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return wrapped


def convrot_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(load_library().convrot_gemm_workspace_size(M, N, K))


def convrot_w4a4_workspace_size(M: int, N: int, K: int) -> int:
    return int(load_library().convrot_w4a4_workspace_size(M, N, K))


def _workspace(ws, nbytes, device):
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _need(ws, "workspace", torch.uint8)
    return ws


@_one_device
def convrot_rotate_quant(x, xq=None, s_a=None, stream=None):
    lib = load_library()
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    xq = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device) if xq is None else xq
    s_a = torch.empty((M,), dtype=torch.float32, device=x.device) if s_a is None else s_a
    _need(xq, "xq", torch.uint8, (M, K // 2))
    _need(s_a, "s_a", torch.float32, (M,))
    _check("convrot_rotate_quant", lib.convrot_rotate_quant(_ptr(x), M, K, _ptr(xq), _ptr(s_a), _stream(stream)))
    return xq, s_a


@_one_device
def convrot_pack_weight(W, Wq=None, s_w=None, stream=None):
    lib = load_library()
    N, K = W.shape
    _need(W, "W", torch.bfloat16)
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device) if Wq is None else Wq
    s_w = torch.empty((N,), dtype=torch.float32, device=W.device) if s_w is None else s_w
    _need(Wq, "Wq", torch.uint8, (N, K // 2))
    _need(s_w, "s_w", torch.float32, (N,))
    _check("convrot_pack_weight", lib.convrot_pack_weight(_ptr(W), N, K, _ptr(Wq), _ptr(s_w), _stream(stream)))
    return Wq, s_w


def _gemm(fn_name, out_dtype, xq, s_a, Wq, s_w, bias, out, workspace, stream):
    lib = load_library()
    M, K = xq.shape[0], xq.shape[1] * 2
    N = Wq.shape[0]
    _need(xq, "xq", torch.uint8)
    _need(Wq, "Wq", torch.uint8, (N, K // 2))
    _need(s_a, "s_a", torch.float32, (M,))
    _need(s_w, "s_w", torch.float32, (N,))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=xq.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    ws = _workspace(workspace, convrot_gemm_workspace_size(M, N, K), xq.device)
    fn = getattr(lib, fn_name)
    if fn_name == "w4a4_gemm_s32":
        rc = fn(_ptr(xq), _ptr(Wq), M, N, K, _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    else:
        rc = fn(_ptr(xq), _ptr(s_a), _ptr(Wq), _ptr(s_w), _ptr(bias), M, N, K, _ptr(out), _ptr(ws), ws.numel(),
                _stream(stream))
    _check(fn_name, rc)
    return out


@_one_device
def w4a4_gemm(xq, s_a, Wq, s_w, bias=None, out=None, workspace=None, stream=None):
    return _gemm("w4a4_gemm", torch.bfloat16, xq, s_a, Wq, s_w, bias, out, workspace, stream)


@_one_device
def w4a4_gemm_f32(xq, s_a, Wq, s_w, bias=None, out=None, workspace=None, stream=None):
    return _gemm("w4a4_gemm_f32", torch.float32, xq, s_a, Wq, s_w, bias, out, workspace, stream)


@_one_device
def w4a4_gemm_s32(xq, Wq, out=None, workspace=None, stream=None):
    return _gemm("w4a4_gemm_s32", torch.int32, xq, None, Wq, None, None, out, workspace, stream)


def _linear(fn_name, out_dtype, x, Wq, s_w, bias, out, workspace, stream):
    lib = load_library()
    M, K = x.shape
    N = Wq.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(Wq, "Wq", torch.uint8, (N, K // 2))
    _need(s_w, "s_w", torch.float32, (N,))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=x.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    ws = _workspace(workspace, convrot_w4a4_workspace_size(M, N, K), x.device)
    rc = getattr(lib, fn_name)(_ptr(x), _ptr(Wq), _ptr(s_w), _ptr(bias), M, N, K, _ptr(out), _ptr(ws), ws.numel(),
                               _stream(stream))
    _check(fn_name, rc)
    return out


@_one_device
def convrot_w4a4_linear(x, Wq, s_w, bias=None, out=None, workspace=None, stream=None):
    return _linear("convrot_w4a4_linear", torch.bfloat16, x, Wq, s_w, bias, out, workspace, stream)


@_one_device
def convrot_w4a4_linear_f32(x, Wq, s_w, bias=None, out=None, workspace=None, stream=None):
    return _linear("convrot_w4a4_linear_f32", torch.float32, x, Wq, s_w, bias, out, workspace, stream)


@_one_device
def convrot_w4a4_linear_noalloc(x, Wq, s_w, bias=None, out=None, stream=None):
    """The fused Linear using the library's own static scratch instead of a
    workspace (for callers that cannot allocate device memory; see
    include/convrot.h).  ``out`` is the caller's; nothing else is allocated by
    the library.  Shapes needing more than 32 MiB of scratch raise."""
    M, K = x.shape
    N = Wq.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(Wq, "Wq", torch.uint8, (N, K // 2))
    _need(s_w, "s_w", torch.float32, (N,))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", torch.bfloat16, (M, N))
    rc = load_library().convrot_w4a4_linear_noalloc(_ptr(x), _ptr(Wq), _ptr(s_w), _ptr(bias), M, N, K, _ptr(out),
                                                    _stream(stream))
    if rc != 0:
        lib = load_library()
        raise ConvRotError("convrot_w4a4_linear_noalloc", rc,
                           lib.convrot_status_string(rc).decode() + f" [{lib.convrot_last_error().decode()}]")
    return out


@_one_device
def convrot_w4a4_quantize(x, workspace, stream=None):
    """First launch of the fused Linear: x -> activation codes + scales in ``workspace``."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    _need(workspace, "workspace", torch.uint8)
    _check("convrot_w4a4_quantize", load_library().convrot_w4a4_quantize(
        _ptr(x), M, K, _ptr(workspace), workspace.numel(), _stream(stream)))
    return workspace


@_one_device
def convrot_w4a4_gemm_quantized(workspace, M, Wq, s_w, bias=None, out=None, stream=None):
    """Second launch of the fused Linear: ``workspace`` (from convrot_w4a4_quantize) x Wq -> y."""
    N, K = Wq.shape[0], Wq.shape[1] * 2
    _need(Wq, "Wq", torch.uint8)
    _need(s_w, "s_w", torch.float32, (N,))
    _need(bias, "bias", torch.bfloat16, (N,))
    _need(workspace, "workspace", torch.uint8)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=Wq.device) if out is None else out
    _need(out, "out", torch.bfloat16, (M, N))
    _check("convrot_w4a4_gemm_quantized", load_library().convrot_w4a4_gemm_quantized(
        _ptr(Wq), _ptr(s_w), _ptr(bias), M, N, K, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def convrot_device_error(stream=None) -> int:
    """Synchronize, read and clear the device error word; raise on a timeout."""
    lib = load_library()
    code = ctypes.c_uint32(0)
    rc = lib.convrot_device_error(_stream(stream), ctypes.byref(code))
    if rc not in (0, 7):
        _check("convrot_device_error", rc)
    return int(code.value)


def convrot_selftest_timeout(limit_us: int = 20000, stream=None):
    """Run the bounded-wait failure path once (see include/convrot.h)."""
    _check("convrot_selftest_timeout", load_library().convrot_selftest_timeout(int(limit_us), _stream(stream)))


def convrot_dispatch_counts():
    lib = load_library()
    arr = (ctypes.c_uint64 * 6)()
    lib.convrot_dispatch_counts(arr, 6)
    return {"rotate_quant": arr[0], "unpack_codes": arr[1], "tc_gemm": arr[2], "tc_gemm_splitk": arr[3],
            "small_rotate_quant": arr[4], "small_gemm": arr[5]}


def convrot_measure_mma_i8(N: int = 256, a_in_tmem: bool = False, iters: int = 4096):
    """Dense int8 tensor-core rate of this GPU (see include/convrot.h):
    returns (TOPS, SM cycles per 128 x N x 32 MMA).  Blocks the host."""
    tops, cyc = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _check("convrot_measure_mma_i8", load_library().convrot_measure_mma_i8(
        int(N), 1 if a_in_tmem else 0, int(iters), ctypes.byref(tops), ctypes.byref(cyc)))
    return float(tops.value), float(cyc.value)


# ---- rotation group-size variants (256, 64, 16)

@_one_device
def convrot_rotate_quant_g(x, group, xq=None, s_a=None, stream=None):
    """convrot_rotate_quant with rotation group ``group`` (256, 64 or 16)."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    xq = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device) if xq is None else xq
    s_a = torch.empty((M,), dtype=torch.float32, device=x.device) if s_a is None else s_a
    _need(xq, "xq", torch.uint8, (M, K // 2))
    _need(s_a, "s_a", torch.float32, (M,))
    _check("convrot_rotate_quant_g", load_library().convrot_rotate_quant_g(_ptr(x), M, K, int(group), _ptr(xq),
                                                                           _ptr(s_a), _stream(stream)))
    return xq, s_a


@_one_device
def convrot_pack_weight_g(W, group, Wq=None, s_w=None, stream=None):
    """convrot_pack_weight with rotation group ``group`` (256, 64 or 16)."""
    N, K = W.shape
    _need(W, "W", torch.bfloat16)
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device) if Wq is None else Wq
    s_w = torch.empty((N,), dtype=torch.float32, device=W.device) if s_w is None else s_w
    _need(Wq, "Wq", torch.uint8, (N, K // 2))
    _need(s_w, "s_w", torch.float32, (N,))
    _check("convrot_pack_weight_g", load_library().convrot_pack_weight_g(_ptr(W), N, K, int(group), _ptr(Wq),
                                                                         _ptr(s_w), _stream(stream)))
    return Wq, s_w


@_one_device
def convrot_w4a4_quantize_g(x, workspace, group, stream=None):
    """convrot_w4a4_quantize with rotation group ``group`` (256, 64 or 16)."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    _need(workspace, "workspace", torch.uint8)
    _check("convrot_w4a4_quantize_g", load_library().convrot_w4a4_quantize_g(
        _ptr(x), M, K, int(group), _ptr(workspace), workspace.numel(), _stream(stream)))
    return workspace


def _linear_g(fn_name, out_dtype, x, Wq, s_w, bias, group, out, workspace, stream):
    M, K = x.shape
    N = Wq.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(Wq, "Wq", torch.uint8, (N, K // 2))
    _need(s_w, "s_w", torch.float32, (N,))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=x.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    ws = _workspace(workspace, convrot_w4a4_workspace_size(M, N, K), x.device)
    _check(fn_name, getattr(load_library(), fn_name)(_ptr(x), _ptr(Wq), _ptr(s_w), _ptr(bias), M, N, K, int(group),
                                                     _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


@_one_device
def convrot_w4a4_linear_g(x, Wq, s_w, bias=None, group=256, out=None, workspace=None, stream=None):
    return _linear_g("convrot_w4a4_linear_g", torch.bfloat16, x, Wq, s_w, bias, group, out, workspace, stream)


@_one_device
def convrot_w4a4_linear_g_f32(x, Wq, s_w, bias=None, group=256, out=None, workspace=None, stream=None):
    return _linear_g("convrot_w4a4_linear_g_f32", torch.float32, x, Wq, s_w, bias, group, out, workspace, stream)


# ---- int8 W8A8 formats (int8_tensorwise, ConvRot INT8 row-scaled)

def w8a8_workspace_size(M: int, N: int, K: int, fmt: int) -> int:
    return int(load_library().w8a8_workspace_size(M, N, K, int(fmt)))


def _n_scales(rows, fmt):
    return rows if fmt == W8A8_CONVROT_INT8_ROW else 1


@_one_device
def w8a8_quantize(x, fmt, x8=None, s_x=None, workspace=None, stream=None):
    """x [M, K] bf16 -> (int8 codes [M, K], scales fp32 [M] row-scaled / [1] tensorwise)."""
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    x8 = torch.empty((M, K), dtype=torch.int8, device=x.device) if x8 is None else x8
    s_x = torch.empty((_n_scales(M, fmt),), dtype=torch.float32, device=x.device) if s_x is None else s_x
    _need(x8, "x8", torch.int8, (M, K))
    _need(s_x, "s_x", torch.float32, (_n_scales(M, fmt),))
    ws = _workspace(workspace, w8a8_workspace_size(M, 8, K, fmt), x.device)
    _check("w8a8_quantize", load_library().w8a8_quantize(_ptr(x), M, K, int(fmt), _ptr(x8), _ptr(s_x), _ptr(ws),
                                                         ws.numel(), _stream(stream)))
    return x8, s_x


@_one_device
def w8a8_pack_weight(W, fmt, Wq8=None, s_w=None, workspace=None, stream=None):
    """W [N, K] bf16 -> (int8 codes [N, K], scales fp32 [N] row-scaled / [1] tensorwise)."""
    N, K = W.shape
    _need(W, "W", torch.bfloat16)
    Wq8 = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq8 is None else Wq8
    s_w = torch.empty((_n_scales(N, fmt),), dtype=torch.float32, device=W.device) if s_w is None else s_w
    _need(Wq8, "Wq8", torch.int8, (N, K))
    _need(s_w, "s_w", torch.float32, (_n_scales(N, fmt),))
    ws = _workspace(workspace, w8a8_workspace_size(N, 8, K, fmt), W.device)
    _check("w8a8_pack_weight", load_library().w8a8_pack_weight(_ptr(W), N, K, int(fmt), _ptr(Wq8), _ptr(s_w),
                                                               _ptr(ws), ws.numel(), _stream(stream)))
    return Wq8, s_w


def _gemm8(fn_name, out_dtype, x8, s_x, Wq8, s_w, bias, fmt, out, stream):
    M, K = x8.shape
    N = Wq8.shape[0]
    _need(x8, "x8", torch.int8)
    _need(Wq8, "Wq8", torch.int8, (N, K))
    _need(s_x, "s_x", torch.float32, (_n_scales(M, fmt),))
    _need(s_w, "s_w", torch.float32, (_n_scales(N, fmt),))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=x8.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    _check(fn_name, getattr(load_library(), fn_name)(_ptr(x8), _ptr(s_x), _ptr(Wq8), _ptr(s_w), _ptr(bias), M, N, K,
                                                     int(fmt), _ptr(out), _stream(stream)))
    return out


@_one_device
def w8a8_gemm(x8, s_x, Wq8, s_w, bias=None, fmt=W8A8_INT8_TENSORWISE, out=None, stream=None):
    return _gemm8("w8a8_gemm", torch.bfloat16, x8, s_x, Wq8, s_w, bias, fmt, out, stream)


@_one_device
def w8a8_gemm_f32(x8, s_x, Wq8, s_w, bias=None, fmt=W8A8_INT8_TENSORWISE, out=None, stream=None):
    return _gemm8("w8a8_gemm_f32", torch.float32, x8, s_x, Wq8, s_w, bias, fmt, out, stream)


@_one_device
def w8a8_gemm_s32(x8, Wq8, out=None, stream=None):
    M, K = x8.shape
    N = Wq8.shape[0]
    _need(x8, "x8", torch.int8)
    _need(Wq8, "Wq8", torch.int8, (N, K))
    out = torch.empty((M, N), dtype=torch.int32, device=x8.device) if out is None else out
    _need(out, "out", torch.int32, (M, N))
    _check("w8a8_gemm_s32", load_library().w8a8_gemm_s32(_ptr(x8), _ptr(Wq8), M, N, K, _ptr(out), _stream(stream)))
    return out


def _linear8(fn_name, out_dtype, x, Wq8, s_w, bias, fmt, out, workspace, stream):
    M, K = x.shape
    N = Wq8.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(Wq8, "Wq8", torch.int8, (N, K))
    _need(s_w, "s_w", torch.float32, (_n_scales(N, fmt),))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=x.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    ws = _workspace(workspace, w8a8_workspace_size(M, N, K, fmt), x.device)
    _check(fn_name, getattr(load_library(), fn_name)(_ptr(x), _ptr(Wq8), _ptr(s_w), _ptr(bias), M, N, K, int(fmt),
                                                     _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


@_one_device
def w8a8_linear(x, Wq8, s_w, bias=None, fmt=W8A8_INT8_TENSORWISE, out=None, workspace=None, stream=None):
    return _linear8("w8a8_linear", torch.bfloat16, x, Wq8, s_w, bias, fmt, out, workspace, stream)


@_one_device
def w8a8_linear_f32(x, Wq8, s_w, bias=None, fmt=W8A8_INT8_TENSORWISE, out=None, workspace=None, stream=None):
    return _linear8("w8a8_linear_f32", torch.float32, x, Wq8, s_w, bias, fmt, out, workspace, stream)


# ---- asymmetric W4A8: idx [N, K/2] uint8, s_rel [N, K/16] uint8 (e4m3 bytes),
# codebook [16] fp32, s_channel [N] fp32; activations from
# w8a8_quantize(x, W8A8_CONVROT_INT8_ROW)

def asym_w4a8_workspace_size(M: int, N: int, K: int) -> int:
    return int(load_library().asym_w4a8_workspace_size(M, N, K))


def _need_asym(idx, s_rel, codebook, s_channel, K):
    N = idx.shape[0]
    _need(idx, "idx", torch.uint8, (N, K // 2))
    _need(s_rel, "s_rel", torch.uint8, (N, K // 16))
    _need(codebook, "codebook", torch.float32, (16,))
    _need(s_channel, "s_channel", torch.float32, (N,))
    return N


def _gemm_asym(fn_name, out_dtype, x8, s_a, idx, s_rel, codebook, s_channel, bias, out, stream):
    M, K = x8.shape
    _need(x8, "x8", torch.int8)
    N = _need_asym(idx, s_rel, codebook, s_channel, K)
    _need(s_a, "s_a", torch.float32, (M,))
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=x8.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    _check(fn_name, getattr(load_library(), fn_name)(_ptr(x8), _ptr(s_a), _ptr(idx), _ptr(s_rel), _ptr(codebook),
                                                     _ptr(s_channel), _ptr(bias), M, N, K, _ptr(out),
                                                     _stream(stream)))
    return out


@_one_device
def asym_w4a8_gemm(x8, s_a, idx, s_rel, codebook, s_channel, bias=None, out=None, stream=None):
    return _gemm_asym("asym_w4a8_gemm", torch.bfloat16, x8, s_a, idx, s_rel, codebook, s_channel, bias, out, stream)


@_one_device
def asym_w4a8_gemm_f32(x8, s_a, idx, s_rel, codebook, s_channel, bias=None, out=None, stream=None):
    return _gemm_asym("asym_w4a8_gemm_f32", torch.float32, x8, s_a, idx, s_rel, codebook, s_channel, bias, out,
                      stream)


@_one_device
def asym_w4a8_gemm_s32(x8, idx, s_rel, codebook, out=None, stream=None):
    M, K = x8.shape
    _need(x8, "x8", torch.int8)
    N = idx.shape[0]
    _need(idx, "idx", torch.uint8, (N, K // 2))
    _need(s_rel, "s_rel", torch.uint8, (N, K // 16))
    _need(codebook, "codebook", torch.float32, (16,))
    out = torch.empty((M, N), dtype=torch.int32, device=x8.device) if out is None else out
    _need(out, "out", torch.int32, (M, N))
    _check("asym_w4a8_gemm_s32", load_library().asym_w4a8_gemm_s32(_ptr(x8), _ptr(idx), _ptr(s_rel), _ptr(codebook),
                                                                   M, N, K, _ptr(out), _stream(stream)))
    return out


def _linear_asym(fn_name, out_dtype, x, idx, s_rel, codebook, s_channel, bias, out, workspace, stream):
    M, K = x.shape
    _need(x, "x", torch.bfloat16)
    N = _need_asym(idx, s_rel, codebook, s_channel, K)
    _need(bias, "bias", torch.bfloat16, (N,))
    out = torch.empty((M, N), dtype=out_dtype, device=x.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    ws = _workspace(workspace, asym_w4a8_workspace_size(M, N, K), x.device)
    _check(fn_name, getattr(load_library(), fn_name)(_ptr(x), _ptr(idx), _ptr(s_rel), _ptr(codebook), _ptr(s_channel),
                                                     _ptr(bias), M, N, K, _ptr(out), _ptr(ws), ws.numel(),
                                                     _stream(stream)))
    return out


@_one_device
def asym_w4a8_linear(x, idx, s_rel, codebook, s_channel, bias=None, out=None, workspace=None, stream=None):
    return _linear_asym("asym_w4a8_linear", torch.bfloat16, x, idx, s_rel, codebook, s_channel, bias, out, workspace,
                        stream)


@_one_device
def asym_w4a8_linear_f32(x, idx, s_rel, codebook, s_channel, bias=None, out=None, workspace=None, stream=None):
    return _linear_asym("asym_w4a8_linear_f32", torch.float32, x, idx, s_rel, codebook, s_channel, bias, out,
                        workspace, stream)


def convrot_version() -> str:
    return load_library().convrot_version().decode()
