"""Out-of-bounds writes, without a sanitizer: every output and workspace of
the C ABI is handed to the library as the middle of a larger buffer whose
4 KB guard bands before and after hold a byte pattern; after the call (and a
device synchronisation) the bands must be untouched.  Ragged shapes (token
and channel tails, one token, split-K and whole-tile schedules) and every
weight format.  Runs last: a failure here must not hide the parity tests.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests.gpu_util import dev, dev_bf16

pytestmark = pytest.mark.gpu

GUARD = 4096      # bytes on each side (a multiple of 16: the view stays 16-byte aligned)
PATTERN = 0xA5


@pytest.fixture(scope="module")
def rq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import rotation_quantized_bit_b200 as rq
    rq.load_library()
    return rq


class Guarded:
    """A device buffer of `nbytes` (viewed as `dtype`, `shape`) between two guard bands."""

    def __init__(self, shape, dtype):
        itemsize = torch.tensor([], dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        self.nbytes = n * itemsize
        self.raw = torch.full((GUARD + self.nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.view = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(*shape)
        assert self.view.data_ptr() % 16 == 0 and self.view.is_contiguous()

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[GUARD + self.nbytes:].cpu().numpy()
        return bool(np.all(head == PATTERN) and np.all(tail == PATTERN))


SHAPES = [(1, 256, 8), (77, 768, 264), (16, 2560, 1032), (193, 512, 136), (1220, 2560, 1024)]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_w4a4_outputs_and_workspaces_stay_in_bounds(rq, M, K, N):
    x = dev_bf16(synthetic.activations("qwen3_4b", M, K))
    w, b = synthetic.weights("qwen3_4b", N, K)
    wd, bd = dev_bf16(w), dev_bf16(b)
    wq, sw = Guarded((N, K // 2), torch.uint8), Guarded((N,), torch.float32)
    rq.convrot_pack_weight(wd, Wq=wq.view, s_w=sw.view)
    assert wq.intact() and sw.intact()
    xq, sa = Guarded((M, K // 2), torch.uint8), Guarded((M,), torch.float32)
    rq.convrot_rotate_quant(x, xq=xq.view, s_a=sa.view)
    assert xq.intact() and sa.intact()
    ws = Guarded((rq.convrot_w4a4_workspace_size(M, N, K),), torch.uint8)
    y = Guarded((M, N), torch.bfloat16)
    rq.convrot_w4a4_linear(x, wq.view, sw.view, bd, out=y.view, workspace=ws.view)
    assert y.intact() and ws.intact()
    y32 = Guarded((M, N), torch.float32)
    rq.convrot_w4a4_linear_f32(x, wq.view, sw.view, bd, out=y32.view, workspace=ws.view)
    assert y32.intact() and ws.intact()
    acc = Guarded((M, N), torch.int32)
    gws = Guarded((rq.convrot_gemm_workspace_size(M, N, K),), torch.uint8)
    rq.w4a4_gemm_s32(xq.view, wq.view, out=acc.view, workspace=gws.view)
    assert acc.intact() and gws.intact()
    assert rq.convrot_device_error() == 0


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (77, 768, 264), (300, 3072, 136)])
def test_int8_outputs_and_workspaces_stay_in_bounds(rq, fmt, M, K, N):
    x = dev_bf16(synthetic.activations("qwen3_4b", M, K))
    w, b = synthetic.weights("qwen3_4b", N, K)
    nsc = M if fmt == 1 else 1
    x8, sx = Guarded((M, K), torch.int8), Guarded((nsc,), torch.float32)
    wsq = Guarded((rq.w8a8_workspace_size(M, 8, K, fmt),), torch.uint8)
    rq.w8a8_quantize(x, fmt, x8=x8.view, s_x=sx.view, workspace=wsq.view)
    assert x8.intact() and sx.intact() and wsq.intact()
    w8, s_w = rq.w8a8_pack_weight(dev_bf16(w), fmt)
    ws = Guarded((rq.w8a8_workspace_size(M, N, K, fmt),), torch.uint8)
    y = Guarded((M, N), torch.bfloat16)
    rq.w8a8_linear(x, w8, s_w, dev_bf16(b), fmt, out=y.view, workspace=ws.view)
    assert y.intact() and ws.intact()
    assert rq.convrot_device_error() == 0


@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (77, 768, 264), (1220, 2560, 1024)])
def test_asym_outputs_and_workspaces_stay_in_bounds(rq, M, K, N):
    x = dev_bf16(synthetic.activations("qwen3_4b", M, K))
    idx, s_rel, cb, sch = synthetic.asym_format("qwen3_4b", N, K)
    di, ds, dc, dsc = dev(idx), dev(s_rel), dev(cb), dev(sch)
    ws = Guarded((rq.asym_w4a8_workspace_size(M, N, K),), torch.uint8)
    y = Guarded((M, N), torch.bfloat16)
    rq.asym_w4a8_linear(x, di, ds, dc, dsc, None, out=y.view, workspace=ws.view)
    assert y.intact() and ws.intact()
    acc = Guarded((M, N), torch.int32)
    x8, sa = rq.w8a8_quantize(x, rq.W8A8_CONVROT_INT8_ROW)
    rq.asym_w4a8_gemm_s32(x8, di, ds, dc, out=acc.view)
    assert acc.intact()
    assert rq.convrot_device_error() == 0
