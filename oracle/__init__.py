"""CPU oracle for the ConvRot W4A4 quantized Linear -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it; the two share no code.

The arithmetic lives in ``convrot_oracle.c`` (plain C, fp32 rotation with no
FMA contraction, int64 GEMM).  This module only builds that file with gcc and
marshals numpy arrays into it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "convrot_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libconvrot_oracle.so")
_lib = None

# -ffp-contract=off: every a*b+c stays two rounded ops; no -ffast-math, so
# IEEE semantics (rint = round half to even, true division) hold.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libconvrot_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_rotate_rows_f32.argtypes = [P, I, I, I]
        lib.oracle_rotate_quant_ex.argtypes = [P, I, I, I, P, P, P, P]
        lib.oracle_rotate_quant.argtypes = [P, I, I, P, P]
        lib.oracle_pack_weight.argtypes = [P, I, I, P, P]
        lib.oracle_gemm_s64_rows.argtypes = [P, P, I, I, I, I, I, P]
        lib.oracle_epilogue.argtypes = [P, P, P, P, I, I, P, P]
        lib.oracle_linear_rows.argtypes = [P, P, P, P, I, I, I, I, I, P, P]
        lib.oracle_pack_codes.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_unpack_codes.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_quant8.argtypes = [P, I, I, I, I, P, P]
        lib.oracle_gemm8_s64_rows.argtypes = [P, P, I, I, I, I, I, P]
        lib.oracle_linear8_rows.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P]
        lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        lib.oracle_asym_decode.argtypes = [P, P, P, I, I, P]
        lib.oracle_asym_linear_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, P]
        lib.oracle_lloyd_max16.argtypes = [P, ctypes.c_int64, I, P]
        lib.oracle_asym_convert.argtypes = [P, I, I, I, P, P, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def rotate_rows_f32(x, group: int = 256):
    """Block-diagonal ConvRot rotation of fp32 rows (a copy is returned)."""
    a = np.array(x, dtype=np.float32, copy=True, order="C")
    M, K = a.shape
    _check(_load().oracle_rotate_rows_f32(_ptr(a), M, K, group), "rotate_rows_f32")
    return a


def rotate_quant_ex(x_bits, group: int = 256):
    """bf16 bits [M, K] -> (codes int8 [M,K], packed uint8 [M,K/2], s fp32 [M], rotated fp32 [M,K])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    packed = np.empty((M, K // 2), np.uint8)
    s = np.empty((M,), np.float32)
    rot = np.empty((M, K), np.float32)
    _check(_load().oracle_rotate_quant_ex(_ptr(x), M, K, group, _ptr(codes), _ptr(packed), _ptr(s), _ptr(rot)),
           "rotate_quant_ex")
    return codes, packed, s, rot


def rotate_quant(x_bits):
    """bf16 bits [M, K] -> (packed codes uint8 [M, K/2], s_a fp32 [M])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    xq = np.empty((M, K // 2), np.uint8)
    s = np.empty((M,), np.float32)
    _check(_load().oracle_rotate_quant(_ptr(x), M, K, _ptr(xq), _ptr(s)), "rotate_quant")
    return xq, s


def pack_weight(w_bits):
    """bf16 bits [N, K] -> (packed codes uint8 [N, K/2], s_w fp32 [N])."""
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    wq = np.empty((N, K // 2), np.uint8)
    s = np.empty((N,), np.float32)
    _check(_load().oracle_pack_weight(_ptr(w), N, K, _ptr(wq), _ptr(s)), "pack_weight")
    return wq, s


def gemm_s64(xq, wq, K: int, rows=None):
    """int64 acc[m, n] = sum_k q_a[m,k] q_w[n,k]; ``rows=(m0, m1)`` limits the rows."""
    xq = _c(xq, np.uint8)
    wq = _c(wq, np.uint8)
    M, N = xq.shape[0], wq.shape[0]
    m0, m1 = rows if rows is not None else (0, M)
    acc = np.empty((m1 - m0, N), np.int64)
    _check(_load().oracle_gemm_s64_rows(_ptr(xq), _ptr(wq), M, N, K, m0, m1, _ptr(acc)), "gemm_s64")
    return acc


def epilogue(acc, s_a, s_w, bias_bits=None):
    """Rank-one rescale + bias: returns (y32 fp32 [M,N], y bf16 bits [M,N])."""
    acc = _c(acc, np.int64)
    M, N = acc.shape
    s_a = _c(s_a, np.float32)
    s_w = _c(s_w, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y32 = np.empty((M, N), np.float32)
    y16 = np.empty((M, N), np.uint16)
    _check(_load().oracle_epilogue(_ptr(acc), _ptr(s_a), _ptr(s_w), _ptr(b), M, N, _ptr(y32), _ptr(y16)),
           "epilogue")
    return y32, y16


def linear(x_bits, wq, s_w, bias_bits, K: int, rows=None):
    """Whole Linear: returns (y32 fp32, y bf16 bits) for rows ``rows=(m0, m1)`` (default all)."""
    x = _c(x_bits, np.uint16)
    wq = _c(wq, np.uint8)
    s_w = _c(s_w, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    M, N = x.shape[0], wq.shape[0]
    m0, m1 = rows if rows is not None else (0, M)
    y32 = np.empty((m1 - m0, N), np.float32)
    y16 = np.empty((m1 - m0, N), np.uint16)
    _check(_load().oracle_linear_rows(_ptr(x), _ptr(wq), _ptr(s_w), _ptr(b), M, N, K, m0, m1, _ptr(y32), _ptr(y16)),
           "linear")
    return y32, y16


# ---- int8 formats: int8_tensorwise (group 0, one scale per tensor) and
# ConvRot INT8 row-scaled (group 256, one scale per row)

TENSORWISE = (0, False)
CONVROT_ROW = (256, True)


def quant8(x_bits, group: int = 0, per_row: bool = False):
    """bf16 bits [M, K] -> (int8 codes [M, K], scales fp32: [M] per row, [1] per tensor)."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    s = np.empty((M if per_row else 1,), np.float32)
    _check(_load().oracle_quant8(_ptr(x), M, K, group, 1 if per_row else 0, _ptr(codes), _ptr(s)), "quant8")
    return codes, s


def gemm8_s64(x8, w8, rows=None):
    """int64 acc[m, n] = sum_k x8[m,k] w8[n,k]; ``rows=(m0, m1)`` limits the rows."""
    x8 = _c(x8, np.int8)
    w8 = _c(w8, np.int8)
    M, K = x8.shape
    N = w8.shape[0]
    m0, m1 = rows if rows is not None else (0, M)
    acc = np.empty((m1 - m0, N), np.int64)
    _check(_load().oracle_gemm8_s64_rows(_ptr(x8), _ptr(w8), M, N, K, m0, m1, _ptr(acc)), "gemm8_s64")
    return acc


def linear8(x_bits, w8, s_w, bias_bits, group: int = 0, per_row: bool = False, rows=None):
    """The int8 Linear: returns (y32 fp32, y bf16 bits) for rows ``rows=(m0, m1)``."""
    x = _c(x_bits, np.uint16)
    w8 = _c(w8, np.int8)
    s_w = _c(s_w, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    M, K = x.shape
    N = w8.shape[0]
    m0, m1 = rows if rows is not None else (0, M)
    y32 = np.empty((m1 - m0, N), np.float32)
    y16 = np.empty((m1 - m0, N), np.uint16)
    _check(_load().oracle_linear8_rows(_ptr(x), _ptr(w8), _ptr(s_w), _ptr(b), M, N, K, group, 1 if per_row else 0,
                                       m0, m1, _ptr(y32), _ptr(y16)), "linear8")
    return y32, y16


def pack_codes(q):
    q = _c(q, np.int8).reshape(-1)
    out = np.empty((q.size // 2,), np.uint8)
    _load().oracle_pack_codes(_ptr(q), q.size, _ptr(out))
    return out


def unpack_codes(b):
    b = _c(b, np.uint8).reshape(-1)
    out = np.empty((b.size * 2,), np.int8)
    _load().oracle_unpack_codes(_ptr(b), b.size * 2, _ptr(out))
    return out


def f32_to_bf16(v: float) -> int:
    return int(_load().oracle_f32_to_bf16(float(v)))


def bf16_to_f32(h: int) -> float:
    return float(_load().oracle_bf16_to_f32(int(h)))


# ---- asymmetric W4A8 (asym_w4a8_int8): 4-bit codebook indices, an e4m3 scale
# per 16 weights along K, one scale per output channel, a 16-level codebook per
# tensor, the ConvRot INT8 row-scaled activations

def e4m3_to_f32(b):
    """e4m3fn bytes -> fp32 values (any shape)."""
    lib = _load()
    table = np.array([lib.oracle_e4m3_to_f32(i) for i in range(256)], np.float32)
    return table[np.asarray(b, np.uint8)]


def f32_to_e4m3(v):
    """fp32 values -> e4m3fn bytes, round to nearest even, saturating at 448."""
    lib = _load()
    a = np.asarray(v, np.float32)
    return np.array([lib.oracle_f32_to_e4m3(float(t)) for t in a.reshape(-1)], np.uint8).reshape(a.shape)


def asym_decode(idx, s_rel, codebook):
    """idx u8 [N, K/2], s_rel u8 [N, K/16], codebook fp32 [16] -> int8 weights [N, K]."""
    idx = _c(idx, np.uint8)
    s_rel = _c(s_rel, np.uint8)
    cb = _c(codebook, np.float32)
    N, K = idx.shape[0], 2 * idx.shape[1]
    w8 = np.empty((N, K), np.int8)
    _check(_load().oracle_asym_decode(_ptr(idx), _ptr(s_rel), _ptr(cb), N, K, _ptr(w8)), "asym_decode")
    return w8


def asym_linear(x_bits, idx, s_rel, codebook, s_channel, bias_bits, rows=None):
    """The asymmetric W4A8 Linear: returns (y32 fp32, y bf16 bits) for rows ``rows=(m0, m1)``."""
    x = _c(x_bits, np.uint16)
    idx = _c(idx, np.uint8)
    s_rel = _c(s_rel, np.uint8)
    cb = _c(codebook, np.float32)
    sc = _c(s_channel, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    M, K = x.shape
    N = idx.shape[0]
    m0, m1 = rows if rows is not None else (0, M)
    y32 = np.empty((m1 - m0, N), np.float32)
    y16 = np.empty((m1 - m0, N), np.uint16)
    _check(_load().oracle_asym_linear_rows(_ptr(x), _ptr(idx), _ptr(s_rel), _ptr(cb), _ptr(sc), _ptr(b), M, N, K,
                                           m0, m1, _ptr(y32), _ptr(y16)), "asym_linear")
    return y32, y16


def lloyd_max16(u, iters: int = 100):
    """16 Lloyd-Max levels (float64) of the values ``u``."""
    u = _c(u, np.float32).reshape(-1)
    lv = np.empty(16, np.float64)
    _check(_load().oracle_lloyd_max16(_ptr(u), u.size, iters, _ptr(lv)), "lloyd_max16")
    return lv


def asym_convert(w_bits, iters: int = 100):
    """bf16 bits W [N, K] -> (idx u8 [N, K/2], s_rel u8 [N, K/16], s_channel fp32 [N], codebook fp32 [16])."""
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    idx = np.empty((N, K // 2), np.uint8)
    s_rel = np.empty((N, K // 16), np.uint8)
    sc = np.empty((N,), np.float32)
    cb = np.empty((16,), np.float32)
    _check(_load().oracle_asym_convert(_ptr(w), N, K, iters, _ptr(idx), _ptr(s_rel), _ptr(sc), _ptr(cb)),
           "asym_convert")
    return idx, s_rel, sc, cb
