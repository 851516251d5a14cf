"""GPU parity of the int8 W8A8 formats (int8_tensorwise; ConvRot INT8
row-scaled) through the C ABI, against the CPU oracle on the same seeded
inputs.

Bar: codes and scales (raw fp32 bits) and the int32 accumulators bit-exact;
the fp32 output bit-identical to the oracle's operation order (which is
within 1e-5 * max|y|); the bf16 output within one bf16 ulp.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.gpu_util import dev, dev_bf16, f32_bits, host, host_bits

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
FORMATS = {"tensorwise": (0, 0, False), "convrot_row": (1, 256, True)}  # name: (ABI format, group, per_row)


@pytest.fixture(scope="module")
def rq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import rotation_quantized_bit_b200 as rq
    rq.load_library()
    return rq


def bf16_ulp_diff(a_bits, b_bits):
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(key(a_bits) - key(b_bits))


def check_f32(y, ref):
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    assert float(np.max(np.abs(y.astype(np.float64) - ref.astype(np.float64)))) <= F32_TOL * scale
    assert np.array_equal(f32_bits(y), f32_bits(ref))


def special_rows(K=512):
    """Zero row, half-integer ties (s = 1 after the row's 127), division ties,
    a subnormal-scale row whose quotients reach 128, huge and tiny values."""
    rows = [np.zeros(K)]
    for v in (2.5, 3.5, 126.5, -0.5):
        r = np.zeros(K); r[0] = 127.0; r[1] = v; rows.append(r)
    for A, B in ((2.734375, 1.3671875), (4.75, 2.375), (18.5, 9.25)):
        r = np.zeros(K); r[0] = A; r[300] = B; rows.append(r)
    r = np.zeros(K); r[7] = 1.0e37; r[8] = -8.0e36; rows.append(r)
    r = np.zeros(K); r[::3] = 1e-30; rows.append(r)
    bits = synthetic.to_bf16_bits(np.stack(rows))
    sub = np.zeros((1, K), np.uint16)
    sub[0, 0] = 0x0001  # 2^-133: rotates to +-2^-137, scale 2^-144 (ConvRot)
    return np.vstack([bits, sub])


QUANT_CASES = [("qwen3_4b", 1, 256), ("qwen3_4b", 77, 2560), ("edit20b", 300, 3072), ("dit6b", 5, 12288),
               ("small", 32, 512), ("qwen3_4b", 129, 9728)]


@pytest.mark.parametrize("fmt", sorted(FORMATS))
@pytest.mark.parametrize("workload,M,K", QUANT_CASES)
def test_quantize_bit_exact(rq, fmt, workload, M, K):
    f, group, per_row = FORMATS[fmt]
    x = synthetic.activations(workload, M, K)
    c_ref, s_ref = oracle.quant8(x, group, per_row)
    c, s = rq.w8a8_quantize(dev_bf16(x), f)
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(c), c_ref)


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_quantize_special_rows(rq, fmt):
    f, group, per_row = FORMATS[fmt]
    x = special_rows()
    if not per_row:  # one scale for the tensor: check the rows one at a time
        for i in range(x.shape[0]):
            c_ref, s_ref = oracle.quant8(x[i:i + 1], group, per_row)
            c, s = rq.w8a8_quantize(dev_bf16(x[i:i + 1]), f)
            assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref)), i
            assert np.array_equal(host(c), c_ref), i
    c_ref, s_ref = oracle.quant8(x, group, per_row)
    c, s = rq.w8a8_quantize(dev_bf16(x), f)
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(c), c_ref)


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_pack_weight_bit_exact(rq, fmt):
    f, group, per_row = FORMATS[fmt]
    w, _ = synthetic.weights("edit20b", 264, 3072)
    c_ref, s_ref = oracle.quant8(w, group, per_row)
    c, s = rq.w8a8_pack_weight(dev_bf16(w), f)
    assert np.array_equal(host(c), c_ref)
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))


GEMM8_CASES = [(8, 256, 256), (77, 264, 768), (1, 128, 2560), (300, 1000, 512), (193, 136, 256),
               (3, 8, 12288), (16, 1032, 9728), (64, 136, 32768), (1000, 1280, 1024), (777, 2056, 768)]


@pytest.mark.parametrize("M,N,K", GEMM8_CASES)
def test_gemm8_s32_bit_exact(rq, M, N, K):
    rng = np.random.default_rng(M * 31 + N + K)
    a = rng.integers(-128, 128, size=(M, K)).astype(np.int8)  # every byte, -128 included
    w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    ref = oracle.gemm8_s64(a, w)
    acc = rq.w8a8_gemm_s32(dev(a), dev(w))
    assert np.array_equal(host(acc).astype(np.int64), ref)


def test_gemm8_extremes(rq):
    K = 12288
    a = np.full((24, K), 127, np.int8)
    w = np.full((136, K), -127, np.int8)
    assert np.all(host(rq.w8a8_gemm_s32(dev(a), dev(w))) == -127 * 127 * K)
    a = np.full((5, K), -128, np.int8)
    w = np.full((8, K), -128, np.int8)
    assert np.all(host(rq.w8a8_gemm_s32(dev(a), dev(w))) == 128 * 128 * K)


LINEAR8_CASES = [("small", 32, 512, 256), ("qwen3_4b", 77, 2560, 264), ("qwen3_4b", 1, 2560, 1024),
                 ("edit20b", 250, 3072, 384), ("edit20b", 16, 3072, 3072), ("qwen3_4b", 8, 9728, 2560),
                 ("dit6b", 600, 3840, 1024)]


@pytest.mark.parametrize("fmt", sorted(FORMATS))
@pytest.mark.parametrize("workload,M,K,N", LINEAR8_CASES)
def test_linear8_matches_oracle(rq, fmt, workload, M, K, N):
    f, group, per_row = FORMATS[fmt]
    x = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    w8, s_w = oracle.quant8(w, group, per_row)
    y32_ref, y16_ref = oracle.linear8(x, w8, s_w, b, group, per_row)
    dx, dw, dsw, db = dev_bf16(x), dev(w8), dev(s_w), dev_bf16(b)
    check_f32(host(rq.w8a8_linear_f32(dx, dw, dsw, db, f)), y32_ref)
    y16 = host_bits(rq.w8a8_linear(dx, dw, dsw, db, f))
    assert bf16_ulp_diff(y16, y16_ref).max() <= 1
    # the GEMM alone on the oracle's codes, and without bias
    x8, s_x = oracle.quant8(x, group, per_row)
    check_f32(host(rq.w8a8_gemm_f32(dev(x8), dev(s_x), dw, dsw, db, f)), y32_ref)
    y32n, _ = oracle.linear8(x, w8, s_w, None, group, per_row)
    check_f32(host(rq.w8a8_gemm_f32(dev(x8), dev(s_x), dw, dsw, None, f)), y32n)


# The shapes the int8 layers take in the pages' models: the 20B edit DiT's
# value/output projections (int8_tensorwise) and the Qwen3-4B attention
# projections (ConvRot INT8 row-scaled), at the benchmark's token counts.
FULL8 = [("tensorwise", "edit20b", 8704, 3072, 3072), ("convrot_row", "qwen3_4b", 1220, 2560, 4096),
         ("convrot_row", "qwen3_4b", 76, 2560, 1024)]


@pytest.mark.parametrize("fmt,workload,M,K,N", FULL8)
def test_full_size_linear8_sampled_rows(rq, fmt, workload, M, K, N):
    f, group, per_row = FORMATS[fmt]
    x = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    dw, dsw = rq.w8a8_pack_weight(dev_bf16(w), f)
    w8, s_w = host(dw), host(dsw)
    wrows = sorted(set(range(4)) | set(range(N - 4, N)))
    if per_row:
        c_ref, s_ref = oracle.quant8(w[wrows], group, per_row)
        assert np.array_equal(w8[wrows], c_ref) and np.array_equal(f32_bits(s_w[wrows]), f32_bits(s_ref))
    y32 = host(rq.w8a8_linear_f32(dev_bf16(x), dw, dsw, dev_bf16(b), f))
    for r0, r1 in ((0, min(M, 8)), (M // 2 - 4, M // 2 + 4), (max(0, M - 8), M)):
        ref32, _ = oracle.linear8(x, w8, s_w, b, group, per_row, rows=(r0, r1))
        check_f32(y32[r0:r1], ref32)


def test_int8_errors_raise_before_launch(rq):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.ConvRotError):
        rq.w8a8_quantize(x, 5)
    assert rq.w8a8_workspace_size(4, 8, 256, 7) == 0
    assert rq.w8a8_workspace_size(4, 8, 300, 0) == 0
    w8 = torch.zeros((8, 256), dtype=torch.int8, device="cuda")
    with pytest.raises(rq.ConvRotError):
        rq.w8a8_gemm_s32(torch.zeros((4, 300), dtype=torch.int8, device="cuda"),
                         torch.zeros((8, 300), dtype=torch.int8, device="cuda"))
    assert rq.convrot_device_error() == 0
    del w8
