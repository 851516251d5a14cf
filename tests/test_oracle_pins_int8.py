"""Pins for the CPU oracle's int8 formats (the W8A8 layers the pages mix with
W4A4): "int8_tensorwise" (one scale per tensor, no rotation; "Qwen-Image-Edit-
2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)", intro) and
"ConvRot INT8 (row-scaled)" (group-256 rotation, one scale per row;
"rockerBOO/qwen3-4b-nvfp4-convrot", file table).  Each test checks the oracle
against something other than itself: hand-derived ties, an independent numpy
re-derivation of the quantizer (on top of the rotation pinned in
test_oracle_pins.py), brute-force integer products, invariances.  Mutants of
the int8 code are planted on the CPU at the end.  No test here needs a GPU.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
import synthetic

H4 = np.array([[1, 1, 1, -1], [1, 1, -1, 1], [1, -1, 1, 1], [-1, 1, 1, 1]], dtype=np.int64)
H256 = np.kron(np.kron(H4, H4), np.kron(H4, H4))


# Rows [A, B] (one scale per tensor, s = A / 127) where B / s sits at a
# half-integer: rint of the true quotient and rint of B * fl(1 / s) differ, so
# a reciprocal-based quantizer gets them wrong.  Found by a float32 search
# over bf16 values (B = A / 2, quotient 63.5 up to the rounding of s).
DIVISION_TIES = [(2.734375, 1.3671875), (4.75, 2.375), (6.5, 3.25), (9.375, 4.6875), (13.3125, 6.65625),
                 (15.0625, 7.53125), (18.5, 9.25), (22.875, 11.4375)]


def bits(a):
    return synthetic.to_bf16_bits(np.asarray(a, dtype=np.float64))


def widen(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- quantizer

def test_division_not_reciprocal_multiplication():
    f = np.float32
    for A, B in DIVISION_TIES:
        c, s = oracle.quant8(bits([[A, B]]), 0, False)
        s_ref = f(A) / f(127)
        assert s[0] == s_ref
        assert int(c[0, 1]) == int(np.rint(f(B) / s_ref))
        assert np.rint(f(B) / s_ref) != np.rint(f(B) * (f(1) / s_ref))


def test_tensorwise_hand_ties():
    # amax 127 -> s = 1 exactly; half-integers round to even, the clamp is symmetric
    vals = [127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 126.5, -127.0, 0.0]
    codes, s = oracle.quant8(bits([vals]), 0, False)
    assert s.tolist() == [1.0]
    assert codes[0].tolist() == [127, 2, 4, -2, 0, 0, 2, 126, -127, 0]


def test_convrot_row_hand_ties():
    # 2032 e_0 rotates to +-127 on group 0 (s = 1); 40 e_0 / 56 e_0 on group 1
    # rotate to +-2.5 / +-3.5 -> +-2 / +-4 (round half to even)
    x = np.zeros((2, 512))
    x[:, 0] = 2032.0
    x[0, 256], x[1, 256] = 40.0, 56.0
    codes, s = oracle.quant8(bits(x), 256, True)
    assert s.tolist() == [1.0, 1.0]
    assert np.array_equal(codes[:, :256], 127 * np.tile(H256[:, 0], (2, 1)))
    assert np.array_equal(codes[0, 256:], 2 * H256[:, 0])
    assert np.array_equal(codes[1, 256:], 4 * H256[:, 0])


@pytest.mark.parametrize("workload,M,K", [("qwen3_4b", 9, 512), ("dit6b", 5, 768), ("small", 32, 512)])
def test_tensorwise_against_numpy_rederivation(workload, M, K):
    xb = synthetic.activations(workload, M, K)
    x = widen(xb)
    s = np.float32(np.abs(x).max()) / np.float32(127)
    ref = np.clip(np.rint(x / s), -127, 127).astype(np.int64)
    codes, sc = oracle.quant8(xb, 0, False)
    assert sc.view(np.uint32)[0] == np.float32(s).view(np.uint32)
    assert np.array_equal(codes.astype(np.int64), ref)


@pytest.mark.parametrize("workload,M,K", [("qwen3_4b", 9, 512), ("dit6b", 5, 768)])
def test_convrot_row_against_numpy_rederivation(workload, M, K):
    xb = synthetic.activations(workload, M, K)
    rot = oracle.rotate_rows_f32(widen(xb), 256)  # the rotation pinned in test_oracle_pins.py
    s = (np.abs(rot).max(1) / np.float32(127)).astype(np.float32)
    ref = np.clip(np.rint(rot / s[:, None]), -127, 127).astype(np.int64)
    codes, sc = oracle.quant8(xb, 256, True)
    assert np.array_equal(sc.view(np.uint32), s.view(np.uint32))
    assert np.array_equal(codes.astype(np.int64), ref)


@pytest.mark.parametrize("group,per_row", [(0, False), (256, True), (0, True), (256, False)])
def test_symmetric_range_and_amax_element(group, per_row):
    xb = synthetic.activations("qwen3_4b", 6, 512)
    codes, _ = oracle.quant8(xb, group, per_row)
    assert codes.min() >= -127 and codes.max() <= 127
    a = np.abs(codes.astype(np.int64))
    if per_row:
        assert np.all(a.max(1) == 127)
    else:
        assert a.max() == 127


@pytest.mark.parametrize("k", [-3, 2])
@pytest.mark.parametrize("group,per_row", [(0, False), (256, True)])
def test_power_of_two_invariance(k, group, per_row):
    xb = synthetic.activations("qwen3_4b", 4, 512)
    c1, s1 = oracle.quant8(xb, group, per_row)
    c2, s2 = oracle.quant8(bits(widen(xb).astype(np.float64) * 2.0 ** k), group, per_row)
    assert np.array_equal(c1, c2)
    assert np.array_equal(s2, (s1 * np.float32(2.0 ** k)).astype(np.float32))


def test_tensorwise_scale_ignores_row_order_and_row_scale_does_not_mix_rows():
    xb = synthetic.activations("qwen3_4b", 7, 512)
    perm = np.array([3, 0, 6, 1, 5, 2, 4])
    c, s = oracle.quant8(xb, 0, False)
    cp, sp = oracle.quant8(xb[perm], 0, False)
    assert np.array_equal(s, sp) and np.array_equal(c[perm], cp)
    c, s = oracle.quant8(xb, 256, True)
    cp, sp = oracle.quant8(xb[perm], 256, True)
    assert np.array_equal(s[perm], sp) and np.array_equal(c[perm], cp)


def test_clamp_is_symmetric_where_rounding_reaches_128():
    # The smallest bf16 subnormal 2^-133 on channel 0 rotates to +-2^-137 on
    # every channel of group 0; s = RN(2^-137 / 127) = 2^-144 (a subnormal:
    # 32.25 units of 2^-149 round to 32), so x' / s = +-128 exactly and the
    # clamp to [-127, 127] decides the codes.
    x = np.zeros((1, 256), np.uint16)
    x[0, 0] = 0x0001
    c, s = oracle.quant8(x, 256, True)
    assert float(s[0]) == 2.0 ** -144
    assert np.array_equal(c[0].astype(np.int64), 127 * H256[:, 0])


def test_zero_tensor_and_zero_rows():
    z = np.zeros((3, 256), np.uint16)
    c, s = oracle.quant8(z, 0, False)
    assert s.tolist() == [0.0] and not c.any()
    x = np.zeros((2, 512))
    x[1, 3] = 5.0
    c, s = oracle.quant8(bits(x), 256, True)
    assert s[0] == 0.0 and not c[0].any() and s[1] > 0


# ---------------------------------------------------------------- GEMM

def test_gemm8_brute_force_8x256x8():
    rng = np.random.default_rng(8)
    a = rng.integers(-127, 128, size=(8, 256)).astype(np.int8)
    w = rng.integers(-127, 128, size=(8, 256)).astype(np.int8)
    acc = oracle.gemm8_s64(a, w)
    assert np.array_equal(acc, a.astype(np.int64) @ w.astype(np.int64).T)
    ref64 = np.array([[sum(float(a[i, k]) * float(w[j, k]) for k in range(256)) for j in range(8)] for i in range(8)])
    assert np.array_equal(acc.astype(np.float64), ref64)


def test_gemm8_extremes_and_rows():
    K = 1024
    a = np.full((3, K), 127, np.int8)
    w = np.full((2, K), -127, np.int8)
    assert np.all(oracle.gemm8_s64(a, w) == -127 * 127 * K)
    rng = np.random.default_rng(2)
    a = rng.integers(-127, 128, size=(6, K)).astype(np.int8)
    full = oracle.gemm8_s64(a, w)
    assert np.array_equal(oracle.gemm8_s64(a, w, rows=(2, 5)), full[2:5])


# ---------------------------------------------------------------- the Linear

@pytest.mark.parametrize("group,per_row", [(0, False), (256, True)])
def test_linear8_composes_its_steps(group, per_row):
    M, K, N = 6, 512, 24
    xb = synthetic.activations("qwen3_4b", M, K)
    wb, bb = synthetic.weights("qwen3_4b", N, K)
    w8, sw = oracle.quant8(wb, group, per_row)
    y32, y16 = oracle.linear8(xb, w8, sw, bb, group, per_row)
    x8, sx = oracle.quant8(xb, group, per_row)
    acc = x8.astype(np.int64) @ w8.astype(np.int64).T
    sa = sx if per_row else np.full(M, sx[0], np.float32)
    swv = sw if per_row else np.full(N, sw[0], np.float32)
    ref = (acc.astype(np.float32) * sa[:, None]) * swv[None, :] + widen(bb)[None, :]
    assert np.array_equal(y32.view(np.uint32), ref.astype(np.float32).view(np.uint32))
    # rows of a per-tensor linear still use the whole tensor's scale
    y32r, _ = oracle.linear8(xb, w8, sw, bb, group, per_row, rows=(2, 5))
    assert np.array_equal(y32r.view(np.uint32), y32[2:5].view(np.uint32))


def test_linear8_error_and_rotation_helps_on_outliers():
    M, K, N = 16, 1024, 64
    xb = synthetic.activations("qwen3_4b", M, K)  # t(4) with outlier channels x30
    wb, bb = synthetic.weights("qwen3_4b", N, K)
    ref = widen(xb).astype(np.float64) @ widen(wb).astype(np.float64).T + widen(bb)[None, :]
    errs = {}
    for group, per_row in [(0, False), (256, True)]:
        w8, sw = oracle.quant8(wb, group, per_row)
        if group:
            # the ConvRot weights are rotated: the product is x R (W R)^T = x W^T
            pass
        y32, _ = oracle.linear8(xb, w8, sw, bb, group, per_row)
        errs[(group, per_row)] = np.linalg.norm(y32 - ref) / np.linalg.norm(ref)
    assert errs[(256, True)] < errs[(0, False)]
    assert errs[(256, True)] < 0.05


# ---------------------------------------------------------------- mutants

SRC = os.path.join(os.path.dirname(oracle.__file__), "convrot_oracle.c")

MUTANTS8 = {
    "q8_divisor_128": ("float s = amax / 127.0f;", "float s = amax / 128.0f;"),
    "q8_clamp_128": ("if (qv < -127.0f) qv = -127.0f;", "if (qv < -128.0f) qv = -128.0f;"),
    "q8_round_half_away": ("float qv = rintf(row[k] / s);", "float qv = roundf(row[k] / s);"),
    "q8_reciprocal": ("float qv = rintf(row[k] / s);", "float qv = rintf(row[k] * (1.0f / s));"),
    "q8_tensor_amax_first_row": ("for (size_t i = 0; i < (size_t)M * (size_t)K; ++i) {\n      float a = fabsf(v[i]);",
                                 "for (size_t i = 0; i < (size_t)K; ++i) {\n      float a = fabsf(v[i]);"),
    "q8_no_rotation": ("for (int g = 0; g < K / group; ++g) rotate_group(v + (size_t)m * K + (size_t)g * group, S);",
                       "for (int g = 0; g < K / group - 1; ++g) rotate_group(v + (size_t)m * K + (size_t)g * group, S);"),
    "gemm8_dropped_term": ("for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)w[k];",
                           "for (int k = 0; k < K - 1; ++k) s += (int64_t)a[k] * (int64_t)w[k];"),
}


class Lib8:
    def __init__(self, path):
        lib = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.oracle_quant8.argtypes = [P, I, I, I, I, P, P]
        lib.oracle_gemm8_s64_rows.argtypes = [P, P, I, I, I, I, I, P]
        lib.oracle_rotate_rows_f32.argtypes = [P, I, I, I]
        self.lib = lib

    @staticmethod
    def p(a):
        return a.ctypes.data_as(ctypes.c_void_p)

    def q8(self, xb, group, per_row):
        xb = np.ascontiguousarray(xb, np.uint16)
        M, K = xb.shape
        c, s = np.empty((M, K), np.int8), np.empty(M if per_row else 1, np.float32)
        self.lib.oracle_quant8(self.p(xb), M, K, group, int(per_row), self.p(c), self.p(s))
        return c, s

    def gemm8(self, a, w):
        acc = np.empty((a.shape[0], w.shape[0]), np.int64)
        self.lib.oracle_gemm8_s64_rows(self.p(a), self.p(w), a.shape[0], w.shape[0], a.shape[1], 0, a.shape[0],
                                       self.p(acc))
        return acc


def pins8_hold(lib: Lib8) -> bool:
    """A compact re-run of the int8 pins above against ``lib``."""
    ok = True
    c, s = lib.q8(bits([[127.0, 2.5, 3.5, -2.5, -127.0, 1.5]]), 0, False)
    ok &= s.tolist() == [1.0] and c[0].tolist() == [127, 2, 4, -2, -127, 2]
    x = np.zeros((2, 512))
    x[:, 0] = 2032.0
    x[0, 256], x[1, 256] = 40.0, 56.0
    c, s = lib.q8(bits(x), 256, True)
    ok &= s.tolist() == [1.0, 1.0] and np.array_equal(c[0, 256:], 2 * H256[:, 0])
    ok &= np.array_equal(c[:, :256], 127 * np.tile(H256[:, 0], (2, 1)))
    for group, per_row in [(0, False), (256, True)]:
        xb = synthetic.activations("qwen3_4b", 9, 512)
        v = widen(xb)
        if group:
            v = oracle.rotate_rows_f32(v, 256)
        s_ref = (np.abs(v).max(1) if per_row else np.array([np.abs(v).max()])).astype(np.float32) / np.float32(127)
        ref = np.clip(np.rint(v / (s_ref[:, None] if per_row else s_ref[0])), -127, 127).astype(np.int64)
        c, s = lib.q8(xb, group, per_row)
        ok &= np.array_equal(s.view(np.uint32), s_ref.astype(np.float32).view(np.uint32))
        ok &= np.array_equal(c.astype(np.int64), ref)
    # ties that separate division from reciprocal multiplication
    for A, B in DIVISION_TIES:
        c, s = lib.q8(bits([[A, B]]), 0, False)
        ok &= int(c[0, 1]) == int(np.rint(np.float32(B) / (np.float32(A) / np.float32(127))))
    rng = np.random.default_rng(8)
    a = rng.integers(-127, 128, size=(8, 256)).astype(np.int8)
    w = rng.integers(-127, 128, size=(8, 256)).astype(np.int8)
    ok &= np.array_equal(lib.gemm8(a, w), a.astype(np.int64) @ w.astype(np.int64).T)
    # symmetric clamp where rounding reaches 128 (subnormal scale)
    xs = np.zeros((1, 256), np.uint16)
    xs[0, 0] = 0x0001
    c, s = lib.q8(xs, 256, True)
    ok &= np.array_equal(c[0].astype(np.int64), 127 * H256[:, 0])
    # a tensor whose amax sits in the last row, with -127 reached
    xb = bits(np.vstack([np.full((1, 256), 0.5), np.linspace(-3.0, 3.0, 256)[None, :]]))
    c, s = lib.q8(xb, 0, False)
    ok &= float(s[0]) == float(np.float32(3.0) / np.float32(127)) and int(c.min()) == -127
    return bool(ok)


def _build(tmp_path, name, src_text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), "-lm"])
    return str(so)


def test_int8_unmutated_copy_passes(tmp_path):
    with open(SRC) as f:
        assert pins8_hold(Lib8(_build(tmp_path, "orig8", f.read())))


@pytest.mark.parametrize("name", sorted(MUTANTS8))
def test_int8_mutant_is_caught(tmp_path, name):
    with open(SRC) as f:
        text = f.read()
    old, new = MUTANTS8[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    assert not pins8_hold(Lib8(_build(tmp_path, name, text.replace(old, new))))
