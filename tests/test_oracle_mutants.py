"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins catch each one: a dropped term, a wrong sign, a wrong stride or
index, a wrong rounding rule, a swapped nibble order, a transposed operand.

Each mutant is the oracle source with one textual edit, compiled to its own
shared library in a temporary directory; the shipped oracle is untouched.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
import synthetic

SRC = os.path.join(os.path.dirname(oracle.__file__), "convrot_oracle.c")

H4 = np.array([[1, 1, 1, -1], [1, 1, -1, 1], [1, -1, 1, 1], [-1, 1, 1, 1]], dtype=np.int64)
H256 = np.kron(np.kron(H4, H4), np.kron(H4, H4))

MUTANTS = {
    "butterfly_sign": ("v[i + 3 * st] = r - q;", "v[i + 3 * st] = q - r;"),
    "butterfly_pairing": ("float t = c - d;", "float t = d - c;"),
    "stage_stride": ("int st = 1 << (2 * s);", "int st = 1 << s;"),
    "scale_exponent": ("float scale = ldexpf(1.0f, -S);", "float scale = ldexpf(1.0f, -S - 1);"),
    "round_half_away": ("float r = rintf(row[k] / s);", "float r = roundf(row[k] / s);"),
    "scale_divisor": ("float s = amax / 7.0f;", "float s = amax / 8.0f;"),
    "multiply_by_reciprocal": ("float r = rintf(row[k] / s);", "float r = rintf(row[k] * (1.0f / s));"),
    "nibble_order": ("(((uint8_t)q[2 * i + 1] & 0x0Fu) << 4)", "(((uint8_t)q[2 * i + 1] & 0x0Fu) << 0) | (0)"),
    "dropped_k_term": ("for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)wr[k];",
                       "for (int k = 1; k < K; ++k) s += (int64_t)a[k] * (int64_t)wr[k];"),
    "transposed_scale": ("v = v * s_w[n];", "v = v * s_w[m % N];"),
    "amax_first_group_only": ("for (int k = 0; k < K; ++k) {\n      float a = fabsf(row[k]);",
                              "for (int k = 0; k < group; ++k) {\n      float a = fabsf(row[k]);"),
}


class Lib:
    def __init__(self, path):
        lib = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.oracle_rotate_rows_f32.argtypes = [P, I, I, I]
        lib.oracle_rotate_quant_ex.argtypes = [P, I, I, I, P, P, P, P]
        lib.oracle_gemm_s64_rows.argtypes = [P, P, I, I, I, I, I, P]
        lib.oracle_epilogue.argtypes = [P, P, P, P, I, I, P, P]
        self.lib = lib

    @staticmethod
    def p(a):
        return a.ctypes.data_as(ctypes.c_void_p)

    def rotate(self, x):
        a = np.array(x, np.float32, copy=True)
        self.lib.oracle_rotate_rows_f32(self.p(a), a.shape[0], a.shape[1], 256)
        return a

    def rq(self, xb):
        M, K = xb.shape
        xb = np.ascontiguousarray(xb, np.uint16)
        codes, packed = np.empty((M, K), np.int8), np.empty((M, K // 2), np.uint8)
        s, rot = np.empty(M, np.float32), np.empty((M, K), np.float32)
        self.lib.oracle_rotate_quant_ex(self.p(xb), M, K, 256, self.p(codes), self.p(packed), self.p(s), self.p(rot))
        return codes, packed, s, rot

    def gemm(self, xq, wq, K):
        acc = np.empty((xq.shape[0], wq.shape[0]), np.int64)
        self.lib.oracle_gemm_s64_rows(self.p(xq), self.p(wq), xq.shape[0], wq.shape[0], K, 0, xq.shape[0], self.p(acc))
        return acc

    def epi(self, acc, s_a, s_w):
        M, N = acc.shape
        y32, y16 = np.empty((M, N), np.float32), np.empty((M, N), np.uint16)
        self.lib.oracle_epilogue(self.p(acc), self.p(s_a), self.p(s_w), None, M, N, self.p(y32), self.p(y16))
        return y32


def pins_hold(lib: Lib) -> bool:
    """A compact re-run of the pins in test_oracle_pins.py against ``lib``."""
    ok = True
    # Kronecker basis pin
    ok &= np.array_equal(lib.rotate(16.0 * np.eye(256, dtype=np.float32)), H256.T.astype(np.float32))
    # constant vector is a fixed point
    ones = synthetic.to_bf16_bits(np.full((1, 512), 3.0))
    ok &= np.array_equal(lib.rq(ones)[3], np.full((1, 512), 3.0, np.float32))
    # hand-derived ties (s_a = 1, +-2.5 -> +-2, +-3.5 -> +-4)
    x = np.zeros((2, 512))
    x[:, 0] = 112.0
    x[0, 256], x[1, 256] = 40.0, 56.0
    codes, packed, s, _ = lib.rq(synthetic.to_bf16_bits(x))
    ok &= bool(np.all(s == 1.0))
    ok &= np.array_equal(codes[0, 256:], 2 * H256[:, 0]) and np.array_equal(codes[1, 256:], 4 * H256[:, 0])
    # division, not multiplication by the reciprocal (golden/division_ties.txt)
    x = np.zeros((2, 512))
    x[0, 0], x[0, 256], x[1, 0], x[1, 256] = 1.421875, 1.3203125, 2.0625, 1.03125
    codes = lib.rq(synthetic.to_bf16_bits(x))[0]
    ok &= np.array_equal(codes[0, 256:], 6 * H256[:, 0]) and np.array_equal(codes[1, 256:], 4 * H256[:, 0])
    # independent numpy re-derivation of scale and codes on heavy-tailed data
    xb = synthetic.activations("qwen3_4b", 8, 1024)
    codes, packed, s, rot = lib.rq(xb)
    ok &= np.array_equal(s, (np.abs(rot).max(1) / np.float32(7)).astype(np.float32))
    ok &= np.array_equal(codes.astype(np.int64), np.clip(np.rint(rot / s[:, None]), -8, 7).astype(np.int64))
    # packing
    lo = (packed & 0xF).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    ok &= np.array_equal(codes[:, 0::2].astype(np.int64) % 16, lo) and np.array_equal(codes[:, 1::2].astype(np.int64) % 16, hi)
    # brute-force GEMM
    rng = np.random.default_rng(4)
    xq = rng.integers(0, 256, size=(8, 128), dtype=np.uint8)
    wq = rng.integers(0, 256, size=(8, 128), dtype=np.uint8)

    def dec(p):
        l, h = (p & 0xF).astype(np.int64), (p >> 4).astype(np.int64)
        l, h = np.where(l >= 8, l - 16, l), np.where(h >= 8, h - 16, h)
        o = np.empty((p.shape[0], p.shape[1] * 2), np.int64)
        o[:, 0::2], o[:, 1::2] = l, h
        return o

    ok &= np.array_equal(lib.gemm(xq, wq, 256), dec(xq) @ dec(wq).T)
    # epilogue against the float32 sequence
    acc = rng.integers(-1000, 1000, size=(5, 7)).astype(np.int64)
    s_a = (rng.random(5) + 0.5).astype(np.float32)
    s_w = (rng.random(7) + 0.5).astype(np.float32)
    ok &= np.array_equal(lib.epi(acc, s_a, s_w), (acc.astype(np.float32) * s_a[:, None]) * s_w[None, :])
    return bool(ok)


def _build(tmp_path, name, src_text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), "-lm"])
    return str(so)


def test_unmutated_copy_passes(tmp_path):
    with open(SRC) as f:
        assert pins_hold(Lib(_build(tmp_path, "orig", f.read())))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    with open(SRC) as f:
        text = f.read()
    old, new = MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    assert not pins_hold(Lib(_build(tmp_path, name, text.replace(old, new))))
