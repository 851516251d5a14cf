"""GPU parity of the rotation group-size variants (256, 64, 16; the
convrot_groupsize ablation of "JoaoZaokk/Z-Image-Turbo-W4A4-ConvRot", "Where
Z-Image sits") through the C ABI, against the CPU oracle, whose group-64 and
group-16 rotations are pinned against their Kronecker matrices.

Bar: codes and scales bit-exact; the fp32 output bit-identical to the
oracle's composition (rotate/quantize -> int64 GEMM -> rank-one epilogue);
bf16 within one ulp.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.gpu_util import dev, dev_bf16, f32_bits, host, host_bits

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("group", [64, 16, 256])
@pytest.mark.parametrize("workload,M,K", [("qwen3_4b", 1, 256), ("qwen3_4b", 77, 2560), ("dit6b", 300, 3840),
                                          ("edit20b", 5, 12288), ("small", 32, 512)])
def test_rotate_quant_groups_bit_exact(rq, group, workload, M, K):
    x = synthetic.activations(workload, M, K)
    _, packed_ref, s_ref, _ = oracle.rotate_quant_ex(x, group)
    xq, s = rq.convrot_rotate_quant_g(dev_bf16(x), group)
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(xq), packed_ref)


@pytest.mark.parametrize("group", [64, 16])
def test_pack_weight_groups_bit_exact(rq, group):
    w, _ = synthetic.weights("qwen3_4b", 136, 2560)
    _, packed_ref, s_ref, _ = oracle.rotate_quant_ex(w, group)
    wq, s = rq.convrot_pack_weight_g(dev_bf16(w), group)
    assert np.array_equal(host(wq), packed_ref)
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))


@pytest.mark.parametrize("group", [64, 16])
@pytest.mark.parametrize("workload,M,K,N", [("small", 32, 512, 256), ("qwen3_4b", 77, 2560, 264),
                                            ("dit6b", 600, 3840, 1024), ("qwen3_4b", 8, 9728, 2560)])
def test_linear_groups_match_oracle(rq, group, workload, M, K, N):
    x = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    _, wq, s_w, _ = oracle.rotate_quant_ex(w, group)
    _, xq, s_a, _ = oracle.rotate_quant_ex(x, group)
    acc = oracle.gemm_s64(xq, wq, K)
    y32_ref, y16_ref = oracle.epilogue(acc, s_a, s_w, b)
    dx, dwq, dsw, db = dev_bf16(x), dev(wq), dev(s_w), dev_bf16(b)
    y32 = host(rq.convrot_w4a4_linear_g_f32(dx, dwq, dsw, db, group))
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))
    y16 = host_bits(rq.convrot_w4a4_linear_g(dx, dwq, dsw, db, group))
    assert bf16_ulp_diff(y16, y16_ref).max() <= 1


def test_group_256_is_the_default_path(rq):
    x = synthetic.activations("qwen3_4b", 77, 2560)
    w, b = synthetic.weights("qwen3_4b", 264, 2560)
    dx, db = dev_bf16(x), dev_bf16(b)
    dwq, dsw = rq.convrot_pack_weight(dev_bf16(w))
    a = host_bits(rq.convrot_w4a4_linear(dx, dwq, dsw, db))
    g = host_bits(rq.convrot_w4a4_linear_g(dx, dwq, dsw, db, 256))
    assert np.array_equal(a, g)


def test_bad_group_is_rejected(rq):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    for g in (0, 4, 32, 128, 512):
        with pytest.raises(rq.ConvRotError):
            rq.convrot_rotate_quant_g(x, g)
    assert rq.convrot_device_error() == 0
