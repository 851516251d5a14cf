"""Pins for the CPU oracle: each test checks it against something other than itself.

The pins come from what the pages and the mathematics fix:
  * the rotation is the group-256 regular Hadamard ("Qwen-Image-Edit-2511 --
    INT4 tensorwise W4A4 (+ConvRot...)", intro): compared against an explicit
    Kronecker product built here with numpy, orthogonality H H^T = 256 I,
    symmetry, row sums of 16, exact inverse, norm preservation, and the
    outlier-spreading property ("JoaoZaokk/Z-Image-Turbo-W4A4-ConvRot", "Where
    Z-Image sits": one outlier ends up shared over all N channels of its group);
  * the quantizer (amax/7, round half to even, clamp, two codes per byte):
    hand-derived ties in ``golden/quant_ties.txt``, an independent numpy
    re-derivation, power-of-two invariance;
  * the GEMM: brute force against numpy int64 / float64 on 8x256x8;
  * the epilogue: identity scales reduce it to the accumulator;
  * bf16 rounding: torch's own float -> bfloat16 conversion.
No test here needs a GPU.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

H4 = np.array([[1, 1, 1, -1], [1, 1, -1, 1], [1, -1, 1, 1], [-1, 1, 1, 1]], dtype=np.int64)


def kron_hadamard(order: int) -> np.ndarray:
    """Unscaled regular Hadamard of order 4^s as an explicit Kronecker power."""
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < order:
        h = np.kron(h, H4)
    return h


H256 = kron_hadamard(256)


def bits(a):
    return synthetic.to_bf16_bits(a)


# ---------------------------------------------------------------- rotation


def test_rotation_of_basis_vectors_is_the_kronecker_matrix():
    eye16 = 16.0 * np.eye(256, dtype=np.float32)
    r = oracle.rotate_rows_f32(eye16)  # row j = 16 e_j rotated = column j of H
    assert np.array_equal(r, H256.T.astype(np.float32))
    # the bf16 entry point widens and runs the same rotation
    _, _, _, rot = oracle.rotate_quant_ex(bits(eye16))
    assert np.array_equal(rot, H256.T.astype(np.float32))


@pytest.mark.parametrize("group", [16, 64, 256])
def test_rotation_group_variants_match_kronecker(group):
    K = 512
    x = np.zeros((group, K), np.float32)
    for j in range(group):
        x[j, 256 + j] = float(np.sqrt(group))  # inside the second 256-block
    r = oracle.rotate_rows_f32(x, group=group)
    h = kron_hadamard(group).astype(np.float32)
    for j in range(group):
        g0 = (256 + j) // group * group
        out = r[j]
        assert np.array_equal(out[g0:g0 + group], h[:, j])
        out2 = out.copy()
        out2[g0:g0 + group] = 0
        assert not out2.any()


def test_hadamard_matrix_properties():
    eye = np.eye(256, dtype=np.float32) * 16.0
    H = oracle.rotate_rows_f32(eye).astype(np.int64)  # built by the oracle
    assert np.array_equal(H, H.T)  # symmetric
    assert np.array_equal(H @ H.T, 256 * np.eye(256, dtype=np.int64))  # orthogonal
    assert np.all(H.sum(axis=1) == 16)  # regular: all row sums equal 16
    assert np.all(np.abs(H) == 1)


@pytest.mark.parametrize("c", [1.0, -3.0, 0.015625, 12.5, 1e-3])
def test_constant_vector_is_a_fixed_point(c):
    x = np.full((3, 512), c, dtype=np.float64)
    xb = bits(x)
    _, _, _, rot = oracle.rotate_quant_ex(xb)
    assert np.array_equal(rot, synthetic.bf16_bits_to_f32(xb))


def test_exact_inverse_on_small_integers():
    rng = np.random.default_rng(1)
    x = rng.integers(-16, 17, size=(64, 768)).astype(np.float32)
    once = oracle.rotate_rows_f32(x)
    twice = oracle.rotate_rows_f32(once)
    assert np.array_equal(twice, x)  # all intermediates are exact multiples of 1/16


def test_inverse_and_norm_on_random_inputs():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((32, 1024)).astype(np.float32) * 3
    r = oracle.rotate_rows_f32(x)
    rr = oracle.rotate_rows_f32(r)
    assert np.max(np.abs(rr - x)) <= 1e-5 * np.max(np.abs(x))
    for g in range(4):
        n0 = np.linalg.norm(x[:, 256 * g:256 * (g + 1)].astype(np.float64), axis=1)
        n1 = np.linalg.norm(r[:, 256 * g:256 * (g + 1)].astype(np.float64), axis=1)
        assert np.allclose(n0, n1, rtol=2e-6, atol=0)


def test_rotation_against_float64_matmul():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((16, 512)).astype(np.float32)
    x[:, 7] *= 40
    r = oracle.rotate_rows_f32(x).astype(np.float64)
    ref = np.concatenate([x[:, :256].astype(np.float64) @ H256 / 16.0,
                          x[:, 256:].astype(np.float64) @ H256 / 16.0], axis=1)
    # 8 rounded fp32 adds along each output's path; each bounded by u * sum|x|
    u = 2.0 ** -24
    bound = 8 * u * np.concatenate([np.repeat(np.abs(x[:, :256]).sum(1, keepdims=True), 256, 1),
                                    np.repeat(np.abs(x[:, 256:]).sum(1, keepdims=True), 256, 1)], 1) / 16
    assert np.all(np.abs(r - ref) <= bound + 1e-30)


@pytest.mark.parametrize("j,A", [(0, 112.0), (37, -3.0), (255, 0.125), (128, 1024.0)])
def test_outlier_spreads_evenly_over_the_group(j, A):
    x = np.zeros((1, 256), np.float64)
    x[0, j] = A
    _, _, _, rot = oracle.rotate_quant_ex(bits(x))
    assert np.array_equal(rot[0], (A / 16.0) * H256[:, j].astype(np.float32))


# ---------------------------------------------------------------- quantizer


def _tie_rows():
    rows = []
    with open(os.path.join(GOLDEN, "quant_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            j0, j1, v1, rot_abs, code_abs = line.split()
            rows.append((int(j0), int(j1), float(v1), float(rot_abs), int(code_abs)))
    return rows


def test_hand_derived_ties():
    rows = _tie_rows()
    x = np.zeros((len(rows) + 1, 512), np.float64)  # the last row stays all-zero
    for i, (j0, j1, v1, _, _) in enumerate(rows):
        x[i, j0] = 112.0
        x[i, 256 + j1] = v1
    codes, packed, s, rot = oracle.rotate_quant_ex(bits(x))
    for i, (j0, j1, v1, rot_abs, code_abs) in enumerate(rows):
        assert s[i] == np.float32(1.0)
        assert np.array_equal(codes[i, :256], 7 * H256[:, j0])
        assert np.array_equal(np.abs(rot[i, 256:]), np.full(256, rot_abs, np.float32))
        assert np.array_equal(codes[i, 256:], code_abs * H256[:, j1])
    assert s[-1] == 0.0 and not codes[-1].any() and not packed[-1].any()


def _np_rint_half_even_codes(rot, s):
    q = np.zeros_like(rot, dtype=np.int64)
    nz = s != 0
    quot = rot[nz] / s[nz][:, None]  # float32 / float32: one IEEE division
    q[nz] = np.clip(np.rint(quot), -8, 7).astype(np.int64)  # numpy rint rounds half to even
    return q


@pytest.mark.parametrize("workload", ["small", "qwen3_4b", "dit6b"])
def test_quantizer_against_numpy_rederivation(workload):
    x = synthetic.activations(workload, 24, 1024)
    codes, packed, s, rot = oracle.rotate_quant_ex(x)
    amax = np.max(np.abs(rot), axis=1)
    assert np.array_equal(s, (amax / np.float32(7.0)).astype(np.float32))
    assert np.array_equal(codes.astype(np.int64), _np_rint_half_even_codes(rot, s))
    # the amax element maps to +-7 and every code lies in [-7, 7]
    assert codes.min() >= -7 and codes.max() <= 7
    for i in range(codes.shape[0]):
        k = int(np.argmax(np.abs(rot[i])))
        assert abs(int(codes[i, k])) == 7


@pytest.mark.parametrize("k", [-3, -1, 1, 4])
def test_power_of_two_invariance(k):
    x = synthetic.activations("qwen3_4b", 16, 512)
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    c0, _, s0, _ = oracle.rotate_quant_ex(x)
    c1, _, s1, _ = oracle.rotate_quant_ex(bits(xf * 2.0 ** k))
    assert np.array_equal(c0, c1)
    assert np.array_equal(s1, (s0 * np.float32(2.0 ** k)).astype(np.float32))


def test_weight_packing_is_the_same_math_per_output_channel():
    w, _ = synthetic.weights("small", 64, 512)
    wq, s_w = oracle.pack_weight(w)
    xq, s_a = oracle.rotate_quant(w)
    assert np.array_equal(wq, xq) and np.array_equal(s_w, s_a)
    assert wq.nbytes == 64 * 512 // 2  # exactly 0.5 byte per weight ("2/byte")


def test_division_not_reciprocal_multiplication():
    rows = []
    with open(os.path.join(GOLDEN, "division_ties.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                A, B, quot, code, rcode = line.split()
                rows.append((float(A), float(B), float(quot), int(code), int(rcode)))
    x = np.zeros((len(rows), 512))
    for i, (A, B, _, _, _) in enumerate(rows):
        x[i, 0], x[i, 256] = A, B
    codes, _, s, rot = oracle.rotate_quant_ex(bits(x))
    for i, (A, B, quot, code, rcode) in enumerate(rows):
        b16 = np.float32(B) * np.float32(0.0625)
        assert s[i] == np.float32(np.float32(A) * np.float32(0.0625)) / np.float32(7.0)
        assert np.float32(b16 / s[i]) == np.float32(quot)  # numpy's IEEE float32 division
        assert np.rint(np.float32(b16 * (np.float32(1.0) / s[i]))) == rcode  # what a reciprocal would give
        assert np.array_equal(codes[i, 256:], code * H256[:, 0])


# ---------------------------------------------------------------- packing


def test_packing_golden_table():
    with open(os.path.join(GOLDEN, "packing.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    q = np.array([[int(a), int(b)] for a, b, _ in rows], np.int8).reshape(-1)
    want = np.array([int(h, 16) for _, _, h in rows], np.uint8)
    assert np.array_equal(oracle.pack_codes(q), want)
    assert np.array_equal(oracle.unpack_codes(want), q)


def test_packing_round_trip_all_bytes_and_pairs():
    allb = np.arange(256, dtype=np.uint8)
    assert np.array_equal(oracle.pack_codes(oracle.unpack_codes(allb)), allb)
    q0, q1 = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8), indexing="ij")
    q = np.stack([q0.ravel(), q1.ravel()], 1).astype(np.int8).reshape(-1)
    b = oracle.pack_codes(q)
    assert np.array_equal(b.astype(np.int64), (q0.ravel() % 16) + 16 * (q1.ravel() % 16))


# ---------------------------------------------------------------- GEMM


def _decode(packed):
    lo = (packed & 0xF).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def test_gemm_brute_force_8x256x8():
    rng = np.random.default_rng(4)
    xq = rng.integers(0, 256, size=(8, 128), dtype=np.uint8)
    wq = rng.integers(0, 256, size=(8, 128), dtype=np.uint8)
    acc = oracle.gemm_s64(xq, wq, 256)
    a, w = _decode(xq), _decode(wq)
    assert np.array_equal(acc, a @ w.T)
    f = np.array([[sum(float(a[i, k]) * float(w[j, k]) for k in range(256)) for j in range(8)] for i in range(8)])
    assert np.array_equal(acc.astype(np.float64), f)


def test_gemm_extremes():
    K = 3840
    sevens = np.full((2, K // 2), 0x77, np.uint8)
    assert np.all(oracle.gemm_s64(sevens, sevens, K) == 49 * K)
    minus8 = np.full((2, K // 2), 0x88, np.uint8)
    assert np.all(oracle.gemm_s64(minus8, minus8, K) == 64 * K)
    assert np.all(oracle.gemm_s64(minus8, sevens, K) == -56 * K)


def test_gemm_row_subset_matches_full():
    rng = np.random.default_rng(5)
    xq = rng.integers(0, 256, size=(20, 256), dtype=np.uint8)
    wq = rng.integers(0, 256, size=(12, 256), dtype=np.uint8)
    full = oracle.gemm_s64(xq, wq, 512)
    assert np.array_equal(oracle.gemm_s64(xq, wq, 512, rows=(5, 17)), full[5:17])


# ---------------------------------------------------------------- epilogue


def test_epilogue_identity_scales_give_the_accumulator():
    rng = np.random.default_rng(6)
    acc = rng.integers(-(1 << 20), 1 << 20, size=(9, 33)).astype(np.int64)
    y32, _ = oracle.epilogue(acc, np.ones(9, np.float32), np.ones(33, np.float32), None)
    assert np.array_equal(y32, acc.astype(np.float32))


def test_epilogue_matches_float32_sequence_and_bf16_rounding():
    rng = np.random.default_rng(7)
    acc = rng.integers(-200000, 200000, size=(17, 40)).astype(np.int64)
    s_a = rng.random(17).astype(np.float32) + np.float32(0.01)
    s_w = (rng.random(40).astype(np.float32) * np.float32(0.003)).astype(np.float32)
    b = synthetic.bias(11, 40)
    y32, y16 = oracle.epilogue(acc, s_a, s_w, b)
    want = (acc.astype(np.float32) * s_a[:, None]) * s_w[None, :] + synthetic.bf16_bits_to_f32(b)[None, :]
    assert np.array_equal(y32, want.astype(np.float32))
    tb = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y16, tb)


def test_bf16_rounding_against_torch():
    vals = np.array([1.0, 1.00390625, 1.01171875, -1.00390625, 3.0e38, -0.0, 1e-40, 65504.0,
                     1.0 + 2.0 ** -8 + 2.0 ** -20, 0.1, np.inf, -np.inf], np.float32)
    rng = np.random.default_rng(8)
    vals = np.concatenate([vals, (rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000)).astype(np.float32)])
    mine = np.array([oracle.f32_to_bf16(float(v)) for v in vals], np.uint16)
    tb = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, tb)


# ---------------------------------------------------------------- the whole Linear


def test_linear_composes_its_steps():
    x = synthetic.activations("small", 32, 512)
    w, b = synthetic.weights("small", 256, 512)
    wq, s_w = oracle.pack_weight(w)
    y32, y16 = oracle.linear(x, wq, s_w, b, 512)
    xq, s_a = oracle.rotate_quant(x)
    acc = oracle.gemm_s64(xq, wq, 512)
    e32, e16 = oracle.epilogue(acc, s_a, s_w, b)
    assert np.array_equal(y32, e32) and np.array_equal(y16, e16)
    r32, r16 = oracle.linear(x, wq, s_w, b, 512, rows=(3, 29))
    assert np.array_equal(r32, y32[3:29]) and np.array_equal(r16, y16[3:29])


def _rel_err(y, ref):
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def test_linear_error_band_and_rotation_helps_on_outliers():
    # The per-layer W4A4 error on the pages' models sits near 0.12, well above
    # the bf16 floor of ~0.002 ("JoaoZaokk/Z-Image-Turbo-W4A4-ConvRot", "The
    # files"); here a synthetic band, and the rotation must beat plain per-row
    # INT4 on inputs with outlier channels.
    x = synthetic.activations("small", 32, 512)
    w, b = synthetic.weights("small", 256, 512)
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    wf = synthetic.bf16_bits_to_f32(w).astype(np.float64)
    ref = xf @ wf.T + synthetic.bf16_bits_to_f32(b)[None, :]
    wq, s_w = oracle.pack_weight(w)
    y32, _ = oracle.linear(x, wq, s_w, b, 512)
    e_rot = _rel_err(y32.astype(np.float64), ref)

    def plain_int4(a):
        s = np.abs(a).max(1, keepdims=True) / 7.0
        return np.clip(np.rint(a / s), -8, 7) * s

    e_plain = _rel_err(plain_int4(xf) @ plain_int4(wf).T + synthetic.bf16_bits_to_f32(b)[None, :], ref)
    assert 0.01 < e_rot < 0.5
    assert e_rot < e_plain


def test_larger_rotation_group_gives_lower_error():
    # "JoaoZaokk/Z-Image-Turbo-W4A4-ConvRot", "Where Z-Image sits": the error
    # falls as the rotation group grows (cg 256 < 64 < 16 in error).
    x = synthetic.activations("qwen3_4b", 64, 2560)
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    errs = []
    for g in (256, 64, 16):
        codes, _, s, _ = oracle.rotate_quant_ex(x, group=g)
        deq = codes.astype(np.float32) * s[:, None]
        back = oracle.rotate_rows_f32(deq, group=g).astype(np.float64)  # the rotation is its own inverse
        errs.append(_rel_err(back, xf))
    assert errs[0] < errs[1] < errs[2]


def test_shape_errors():
    with pytest.raises(ValueError):
        oracle.rotate_quant(np.zeros((2, 300), np.uint16))
    with pytest.raises(ValueError):
        oracle.rotate_quant_ex(np.zeros((2, 512), np.uint16), group=32)
