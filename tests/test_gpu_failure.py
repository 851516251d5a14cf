"""Failure detection on the GPU without faulting it: a bounded wait that can
never complete (a barrier nothing arrives at) gives up after a short limit,
the kernel returns, the host reads CONVROT_ERR_TIMEOUT, and the context keeps
working (a following linear still matches the oracle bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.gpu_util import dev_bf16, f32_bits, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import rotation_quantized_bit_b200 as rq
    rq.load_library()
    return rq


def test_bounded_wait_times_out_and_reports(rq):
    assert rq.convrot_device_error() == 0          # clean start
    rq.convrot_selftest_timeout(20000)              # 20 ms limit
    assert rq.convrot_device_error() == 1           # bit 0: a bounded wait expired (and the word is cleared)
    assert rq.convrot_device_error() == 0


def test_context_usable_after_timeout(rq):
    rq.convrot_selftest_timeout(5000)
    assert rq.convrot_device_error() == 1
    x = synthetic.activations("small", 32, 512)
    w, b = synthetic.weights("small", 256, 512)
    wq, s_w = oracle.pack_weight(w)
    ref32, _ = oracle.linear(x, wq, s_w, b, 512)
    y32 = host(rq.convrot_w4a4_linear_f32(dev_bf16(x), torch.from_numpy(wq).cuda(), torch.from_numpy(s_w).cuda(),
                                          dev_bf16(b)))
    assert np.array_equal(f32_bits(y32), f32_bits(ref32))
    assert rq.convrot_device_error() == 0


def test_limit_argument_is_checked(rq):
    with pytest.raises(rq.ConvRotError):
        rq.convrot_selftest_timeout(0)
