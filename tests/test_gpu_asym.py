"""GPU parity of the asymmetric W4A8 format (4-bit codebook indices, an e4m3
scale per 16 weights, a per-channel scale, a 16-level codebook; ConvRot INT8
row-scaled activations) through the C ABI, against the CPU oracle on the same
seeded inputs.

Bar: the int32 accumulators bit-exact (so every decoded int8 weight is
right); the fp32 output bit-identical to the oracle's operation order (within
1e-5 * max|y|); the bf16 output within one bf16 ulp.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.gpu_util import dev, dev_bf16, f32_bits, host, host_bits

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5


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


def random_format(seed, N, K, every_byte=False):
    """idx / s_rel / codebook with every index and (optionally) every scale
    byte -- zeros, negatives, subnormals, 448, NaN -- and levels that tie at
    .5 or saturate."""
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    if every_byte:
        s_rel = rng.integers(0, 256, size=(N, K // 16)).astype(np.uint8)
    else:
        s_rel = rng.integers(0x40, 0x71, size=(N, K // 16)).astype(np.uint8)
    cb = np.sort(rng.uniform(-1.0, 1.0, 16)).astype(np.float32)
    if every_byte:
        cb[0], cb[7], cb[8], cb[15] = -1e30, 0.5, 0.25, 3.0
    s_channel = rng.uniform(1e-5, 3e-4, N).astype(np.float32)
    return idx, s_rel, cb, s_channel


# (M, N, K): one unit, ragged token and channel tails, split-K (small M),
# whole-tile schedules (large M), K up to the 20B DiT's MLP down projection.
GEMM_CASES = [(8, 256, 256), (77, 264, 768), (1, 128, 2560), (300, 1000, 512), (193, 136, 256),
              (3, 8, 12288), (16, 1032, 9728), (1000, 1280, 1024), (777, 2056, 768), (129, 384, 3072)]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_asym_gemm_s32_bit_exact(rq, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    a = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    idx, s_rel, cb, _ = random_format(M + N + K, N, K, every_byte=True)
    ref = oracle.gemm8_s64(a, oracle.asym_decode(idx, s_rel, cb))
    acc = rq.asym_w4a8_gemm_s32(dev(a), dev(idx), dev(s_rel), dev(cb))
    assert np.array_equal(host(acc).astype(np.int64), ref)


def test_asym_gemm_extremes(rq):
    """Every weight at +-127 (saturated decode) against +-127 activations:
    |acc| = 127^2 K, the largest the format reaches."""
    K = 12288
    cb = np.full(16, -1.0, np.float32)
    cb[8:] = 1.0
    idx = np.full((136, K // 2), 0x88, np.uint8)  # index 8 everywhere: level +1
    s_rel = np.full((136, K // 16), 0x7E, np.uint8)  # 448
    a = np.full((24, K), -127, np.int8)
    acc = host(rq.asym_w4a8_gemm_s32(dev(a), dev(idx), dev(s_rel), dev(cb)))
    assert np.all(acc == -127 * 127 * K)
    idx[:, :] = 0x00  # level -1 -> -127
    acc = host(rq.asym_w4a8_gemm_s32(dev(np.full((5, K), 127, np.int8)), dev(idx), dev(s_rel), dev(cb)))
    assert np.all(acc == -127 * 127 * K)


LINEAR_CASES = [("small", 32, 512, 256), ("qwen3_4b", 77, 2560, 264), ("qwen3_4b", 1, 2560, 1024),
                ("edit20b", 250, 3072, 384), ("qwen3_4b", 8, 9728, 256), ("dit6b", 600, 3840, 512)]


@pytest.mark.parametrize("workload,M,K,N", LINEAR_CASES)
def test_asym_linear_matches_oracle_on_converted_weights(rq, workload, M, K, N):
    x = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    idx, s_rel, s_channel, cb = oracle.asym_convert(w, iters=30)
    y32_ref, y16_ref = oracle.asym_linear(x, idx, s_rel, cb, s_channel, b)
    dx, di, ds, dc, dsc, db = dev_bf16(x), dev(idx), dev(s_rel), dev(cb), dev(s_channel), dev_bf16(b)
    check_f32(host(rq.asym_w4a8_linear_f32(dx, di, ds, dc, dsc, db)), y32_ref)
    y16 = host_bits(rq.asym_w4a8_linear(dx, di, ds, dc, dsc, db))
    assert bf16_ulp_diff(y16, y16_ref).max() <= 1
    # the GEMM alone on the oracle's activation codes, with and without bias
    x8, s_a = oracle.quant8(x, *oracle.CONVROT_ROW)
    check_f32(host(rq.asym_w4a8_gemm_f32(dev(x8), dev(s_a), di, ds, dc, dsc, db)), y32_ref)
    y32n, _ = oracle.asym_linear(x, idx, s_rel, cb, s_channel, None)
    check_f32(host(rq.asym_w4a8_gemm_f32(dev(x8), dev(s_a), di, ds, dc, dsc, None)), y32n)


# The shapes of the pages' W4A8 text encoder (Qwen3-VL-4B decoder Linears) at
# the benchmark's token counts, with random-format weights: sampled rows.
FULL = [("qwen3_4b", 1220, 2560, 9728), ("qwen3_4b", 76, 9728, 2560), ("qwen3_4b", 16, 2560, 9728)]


@pytest.mark.parametrize("workload,M,K,N", FULL)
def test_full_size_asym_linear_sampled_rows(rq, workload, M, K, N):
    x = synthetic.activations(workload, M, K)
    _, b = synthetic.weights(workload, N, K)
    idx, s_rel, cb, s_channel = synthetic.asym_format(workload, N, K)
    y32 = host(rq.asym_w4a8_linear_f32(dev_bf16(x), dev(idx), dev(s_rel), dev(cb), dev(s_channel), dev_bf16(b)))
    for r0, r1 in ((0, min(M, 8)), (M // 2 - 4, M // 2 + 4), (max(0, M - 8), M)):
        ref32, _ = oracle.asym_linear(x, idx, s_rel, cb, s_channel, b, rows=(r0, r1))
        check_f32(y32[r0:r1], ref32)


def test_asym_errors_raise_before_launch(rq):
    x8 = torch.zeros((4, 256), dtype=torch.int8, device="cuda")
    idx = torch.zeros((8, 128), dtype=torch.uint8, device="cuda")
    s_rel = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    cb = torch.zeros(16, dtype=torch.float32, device="cuda")
    lib = rq.load_library()
    acc = torch.empty((4, 8), dtype=torch.int32, device="cuda")
    stream = rq._stream(None)
    # a null codebook, K not a multiple of 256, N not a multiple of 8
    assert lib.asym_w4a8_gemm_s32(rq._ptr(x8), rq._ptr(idx), rq._ptr(s_rel), None, 4, 8, 256, rq._ptr(acc),
                                  stream) == 1
    assert lib.asym_w4a8_gemm_s32(rq._ptr(x8), rq._ptr(idx), rq._ptr(s_rel), rq._ptr(cb), 4, 8, 128, rq._ptr(acc),
                                  stream) == 2
    assert lib.asym_w4a8_gemm_s32(rq._ptr(x8), rq._ptr(idx), rq._ptr(s_rel), rq._ptr(cb), 4, 12, 256, rq._ptr(acc),
                                  stream) == 2
    assert rq.asym_w4a8_workspace_size(4, 8, 300) == 0
    with pytest.raises(rq.ConvRotError):
        rq.asym_w4a8_linear(torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda"), idx, s_rel, cb,
                            torch.zeros(8, dtype=torch.float32, device="cuda"), workspace=torch.empty(
                                16, dtype=torch.uint8, device="cuda"))
    assert rq.convrot_device_error() == 0
