"""GPU parity of the small-M path (M <= 16 tokens): the one-CTA-per-token
prologue and the bandwidth-bound GEMM, through the C ABI, against the CPU
oracle on the same seeded inputs.

Same bar as the other parity files: codes and scales (raw bits) and the
int32 accumulators bit-exact, the fp32 output bit-equal to the oracle's
operation order (within 1e-5 * max|y| is the contract), bf16 within one ulp.
The shapes cover one K block, ragged output tiles (N % 128 != 0), the
largest K, tiles whose K range is split over many CTAs, and more CTAs than
units; repeated calls on one workspace check that the GEMM leaves its
arrival counters at zero.
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


def _ulps(a, b):
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(key(a) - key(b))


def _r256(v):
    return (v + 255) // 256 * 256


def _ws_codes(ws, M, K):
    """Packed codes [M, K/2] and scales [M] from a quantized small-M workspace
    (codes region of M*K bytes, then the scales, each on a 256-byte boundary)."""
    w = host(ws)
    codes = w[: M * K // 2].reshape(M, K // 2)
    off = _r256(M * K)
    scales = w[off: off + 4 * M].view(np.float32)
    return codes, scales


@pytest.mark.parametrize("group", [256, 64, 16])
@pytest.mark.parametrize("M,K", [(1, 256), (2, 2560), (7, 3072), (8, 9728), (9, 12288), (16, 2560), (3, 32768),
                                 (16, 16384)])
def test_small_prologue_codes_bit_exact(rq, M, K, group):
    x = synthetic.activations("qwen3_4b", M, K, seed_extra=K + group)
    _, xq_ref, s_ref, _ = oracle.rotate_quant_ex(x, group)
    ws = torch.zeros(rq.convrot_w4a4_workspace_size(M, 256, K), dtype=torch.uint8, device="cuda")
    rq.convrot_w4a4_quantize_g(dev_bf16(x), ws, group)
    codes, scales = _ws_codes(ws, M, K)
    assert np.array_equal(f32_bits(scales), f32_bits(s_ref))
    assert np.array_equal(codes, xq_ref)


def test_small_prologue_special_rows(rq):
    # Zero row (s = 0), half-integer ties, division-vs-reciprocal ties, tiny
    # and huge values: the same rows as the large-M prologue's test, 16 at a time.
    from tests.test_gpu_parity import special_rows
    x = special_rows()
    for r0 in range(0, x.shape[0], 16):
        xs = x[r0:r0 + 16]
        M, K = xs.shape
        xq_ref, s_ref = oracle.rotate_quant(xs)
        ws = torch.zeros(rq.convrot_w4a4_workspace_size(M, 256, K), dtype=torch.uint8, device="cuda")
        rq.convrot_w4a4_quantize(dev_bf16(xs), ws)
        codes, scales = _ws_codes(ws, M, K)
        assert np.array_equal(f32_bits(scales), f32_bits(s_ref))
        assert np.array_equal(codes, xq_ref)


SMALL_GEMM = [(1, 8, 256), (3, 136, 512), (8, 256, 1024), (16, 264, 768), (9, 128, 2560), (16, 1032, 512),
              (5, 384, 256), (12, 520, 1280), (1, 2560, 32768), (16, 19456, 512), (16, 9728, 2560),
              (8, 2560, 9728), (4, 12288, 3072), (16, 3072, 12288), (2, 24, 7936)]


def _codes(seed, rows, K):
    rng = np.random.default_rng(seed)
    return rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)  # every nibble, -8 included


@pytest.mark.parametrize("M,N,K", SMALL_GEMM)
def test_small_gemm_s32_bit_exact(rq, M, N, K):
    xq = _codes(M * 31 + K, M, K)
    wq = _codes(N * 17 + K, N, K)
    ref = oracle.gemm_s64(xq, wq, K)
    before = rq.convrot_dispatch_counts()["small_gemm"]
    acc = rq.w4a4_gemm_s32(dev(xq), dev(wq))
    assert rq.convrot_dispatch_counts()["small_gemm"] == before + 1
    assert np.array_equal(host(acc).astype(np.int64), ref)


def test_small_gemm_extremes(rq):
    # -8 x -8 everywhere: 64 K per output, the largest accumulator magnitude.
    K = 32768
    for a, b, want in ((0x88, 0x88, 64 * K), (0x77, 0x88, -56 * K), (0x77, 0x77, 49 * K)):
        xq = np.full((16, K // 2), a, np.uint8)
        wq = np.full((136, K // 2), b, np.uint8)
        assert np.all(host(rq.w4a4_gemm_s32(dev(xq), dev(wq))) == want)


@pytest.mark.parametrize("M,N,K", [(1, 264, 512), (8, 1032, 2560), (16, 2560, 9728), (13, 12288, 3072)])
def test_small_gemm_f32_and_bf16(rq, M, N, K):
    x = synthetic.activations("qwen3_4b", M, K)
    w, b = synthetic.weights("qwen3_4b", N, K)
    xq, s_a = oracle.rotate_quant(x)
    wq, s_w = oracle.pack_weight(w)
    acc = oracle.gemm_s64(xq, wq, K)
    y32_ref, y16_ref = oracle.epilogue(acc, s_a, s_w, b)
    args = (dev(xq), dev(s_a), dev(wq), dev(s_w), dev_bf16(b))
    y32 = host(rq.w4a4_gemm_f32(*args))
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))
    y16 = host_bits(rq.w4a4_gemm(*args))
    assert _ulps(y16, y16_ref).max() <= 1
    y32n = host(rq.w4a4_gemm_f32(dev(xq), dev(s_a), dev(wq), dev(s_w), None))
    assert np.array_equal(f32_bits(y32n), f32_bits(oracle.epilogue(acc, s_a, s_w, None)[0]))


@pytest.mark.parametrize("workload,M,K,N", [("small", 1, 512, 256), ("qwen3_4b", 16, 2560, 9728),
                                            ("qwen3_4b", 8, 9728, 2560), ("edit20b", 5, 12288, 3072),
                                            ("edit20b", 16, 3072, 12288), ("dit6b", 11, 3840, 1032)])
def test_small_linear_matches_oracle(rq, workload, M, K, N):
    x = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    wq, s_w = oracle.pack_weight(w)
    y32_ref, y16_ref = oracle.linear(x, wq, s_w, b, K)
    dx, dwq, dsw, db = dev_bf16(x), dev(wq), dev(s_w), dev_bf16(b)
    before = rq.convrot_dispatch_counts()
    y32 = host(rq.convrot_w4a4_linear_f32(dx, dwq, dsw, db))
    after = rq.convrot_dispatch_counts()
    assert after["small_rotate_quant"] == before["small_rotate_quant"] + 1
    assert after["small_gemm"] == before["small_gemm"] + 1
    scale = float(np.max(np.abs(y32_ref)))
    assert float(np.max(np.abs(y32.astype(np.float64) - y32_ref))) <= F32_TOL * scale
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))
    y16 = host_bits(rq.convrot_w4a4_linear(dx, dwq, dsw, db))
    assert _ulps(y16, y16_ref).max() <= 1


@pytest.mark.parametrize("group", [64, 16])
def test_small_linear_groups(rq, group):
    M, K, N = 6, 3072, 1032
    x = synthetic.activations("edit20b", M, K)
    w, b = synthetic.weights("edit20b", N, K)
    _, wq, s_w, _ = oracle.rotate_quant_ex(w, group)
    _, xq, s_a, _ = oracle.rotate_quant_ex(x, group)
    y32_ref = oracle.epilogue(oracle.gemm_s64(xq, wq, K), s_a, s_w, b)[0]
    y32 = host(rq.convrot_w4a4_linear_g_f32(dev_bf16(x), dev(wq), dev(s_w), dev_bf16(b), group=group))
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))


def test_small_quantize_once_gemm_many_and_repeat(rq):
    # One quantization, several GEMMs on the same workspace one after another
    # (the counters each GEMM leaves behind must be zero for the next), and
    # the same GEMM again: identical bits every time.
    M, K = 16, 2560
    x = synthetic.activations("qwen3_4b", M, K)
    xq_ref, s_a = oracle.rotate_quant(x)
    shapes = [9728, 1024, 1032, 4096, 9728]
    ws = torch.empty(max(rq.convrot_w4a4_workspace_size(M, N, K) for N in shapes), dtype=torch.uint8, device="cuda")
    ws.fill_(0xA5)  # the GEMM must not depend on the workspace's previous contents
    rq.convrot_w4a4_quantize(dev_bf16(x), ws)
    first = None
    for N in shapes:
        w, b = synthetic.weights("qwen3_4b", N, K)
        wq, s_w = oracle.pack_weight(w)
        y16_ref = oracle.epilogue(oracle.gemm_s64(xq_ref, wq, K), s_a, s_w, b)[1]
        y16 = host_bits(rq.convrot_w4a4_gemm_quantized(ws, M, dev(wq), dev(s_w), dev_bf16(b)))
        assert _ulps(y16, y16_ref).max() <= 1, N
        if first is None:
            first = y16
        elif N == shapes[0]:
            assert np.array_equal(y16, first)
    assert rq.convrot_device_error() == 0


def test_pack_then_linear_on_one_stream(rq):
    # Weight packing, then the Linear right after it on the same stream: the
    # GEMM streams weights before it waits for its predecessor, so the
    # packing kernel must not let it start early.
    M, K, N = 4, 9728, 2560
    x = synthetic.activations("qwen3_4b", M, K)
    w, b = synthetic.weights("qwen3_4b", N, K)
    wq_ref, sw_ref = oracle.pack_weight(w)
    y16_ref = oracle.linear(x, wq_ref, sw_ref, b, K)[1]
    dx, dw, db = dev_bf16(x), dev_bf16(w), dev_bf16(b)
    for _ in range(3):
        wq = torch.full((N, K // 2), 0x88, dtype=torch.uint8, device="cuda")
        s_w = torch.zeros((N,), dtype=torch.float32, device="cuda")
        rq.convrot_pack_weight(dw, Wq=wq, s_w=s_w)
        y16 = host_bits(rq.convrot_w4a4_linear(dx, wq, s_w, db))
        assert _ulps(y16, y16_ref).max() <= 1


def test_m17_takes_the_tensor_core_path(rq):
    before = rq.convrot_dispatch_counts()
    x = dev_bf16(synthetic.activations("small", 17, 512))
    w, b = synthetic.weights("small", 256, 512)
    wq, s_w = rq.convrot_pack_weight(dev_bf16(w))
    rq.convrot_w4a4_linear(x, wq, s_w, dev_bf16(b))
    after = rq.convrot_dispatch_counts()
    assert after["small_gemm"] == before["small_gemm"]
    assert after["tc_gemm"] + after["tc_gemm_splitk"] == before["tc_gemm"] + before["tc_gemm_splitk"] + 1
