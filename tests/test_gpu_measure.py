"""The library's dense int8 tensor-core rate measurement (the denominator the
GEMM's roofline fraction is compared with): it runs, reports a plausible rate
and leaves no device error."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import rotation_quantized_bit_b200 as rq
    rq.load_library()
    return rq


@pytest.mark.parametrize("N,a_in_tmem", [(256, False), (256, True), (16, True)])
def test_measure_mma_i8(rq, N, a_in_tmem):
    tops, cycles = rq.convrot_measure_mma_i8(N, a_in_tmem, 256)
    # 148 SMs x 8192 int8 MACs/clk x 2 x <= 2.1 GHz bounds the rate from above;
    # an MMA takes at least N / 2 cycles of one SM's tensor core.
    assert 0 < tops < 148 * 8192 * 2 * 2.1e9 / 1e12
    assert cycles >= N / 2 * 0.95
    assert rq.convrot_device_error() == 0


def test_measure_mma_i8_rejects_bad_shapes(rq):
    with pytest.raises(rq.ConvRotError):
        rq.convrot_measure_mma_i8(24, False, 16)
    with pytest.raises(rq.ConvRotError):
        rq.convrot_measure_mma_i8(512, False, 16)
