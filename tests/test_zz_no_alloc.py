"""The no-allocation variant of the fused Linear, convrot_w4a4_linear_noalloc.

It exists for callers that cannot allocate device memory (code inside a host
framework that owns all device allocations, fixed-budget deployments,
plugin or foreign-language callers without a CUDA allocator binding): it
takes no workspace and uses a static scratch array inside the library.

These tests call it through the C ABI, on two calls in a row (the scratch
keeps the previous call's contents), and require its output to be the same
bits as the existing entry point's, convrot_w4a4_linear with a caller-supplied
workspace (both run the same kernels on the same inputs), and to match the
CPU oracle within the bf16 bar of the other GPU tests.  This file is named
so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import rotation_quantized_bit_b200 as rq
    return rq.load_library()


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _ulps(a, b):
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(key(a) - key(b))


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _prepare(lib, workload, M, K, N):
    xb = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    x, W, bias = _bf16(xb), _bf16(w), _bf16(b)
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s_w = torch.empty((N,), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.convrot_pack_weight(_p(W), N, K, _p(Wq), _p(s_w), stream) == 0
    # The oracle's result on the oracle's own packing of W (sampled rows).
    wq_ref, sw_ref = oracle.pack_weight(w)
    rows = (0, min(M, 8))
    ref16 = oracle.linear(xb, wq_ref, sw_ref, b, K, rows=rows)[1]
    return x, Wq, s_w, bias, stream, (rows, ref16)


def _reference(lib, x, Wq, s_w, bias, M, K, N, stream):
    ws_bytes = lib.convrot_w4a4_workspace_size(M, N, K)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert lib.convrot_w4a4_linear(_p(x), _p(Wq), _p(s_w), _p(bias), M, N, K, _p(y), _p(ws), ws_bytes, stream) == 0
    return y


def _check(y, y_ref, oracle_rows):
    # The same kernels on the same inputs: identical bits.
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    (r0, r1), ref16 = oracle_rows
    assert _ulps(_bits(y)[r0:r1], ref16).max() <= 1  # the bf16 bar of the other GPU tests


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    # Two calls in a row with different shapes: the second one runs on
    # scratch that still holds the first call's codes.  The second shape is
    # a small-M one (its GEMM splits K and keeps counters in the scratch).
    for workload, M, K, N in (("qwen3_4b", 1220, 2560, 1024), ("qwen3_4b", 8, 9728, 1024),
                              ("qwen3_4b", 76, 9728, 2560)):
        x, Wq, s_w, bias, stream, ref = _prepare(lib, workload, M, K, N)
        y_ref = _reference(lib, x, Wq, s_w, bias, M, K, N, stream)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = lib.convrot_w4a4_linear_noalloc(_p(x), _p(Wq), _p(s_w), _p(bias), M, N, K, _p(y), stream)
        assert rc == 0, lib.convrot_last_error().decode()
        torch.cuda.synchronize()
        _check(y, y_ref, ref)


def test_noalloc_repeated_call_same_shape(lib):
    for M, K, N in ((64, 3072, 12288), (16, 3072, 12288)):
        x, Wq, s_w, bias, stream, ref = _prepare(lib, "edit20b", M, K, N)
        y_ref = _reference(lib, x, Wq, s_w, bias, M, K, N, stream)
        for _ in range(2):
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            assert lib.convrot_w4a4_linear_noalloc(_p(x), _p(Wq), _p(s_w), _p(bias), M, N, K, _p(y), stream) == 0
            torch.cuda.synchronize()
            _check(y, y_ref, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    # 8704 x 12288 activation codes need ~102 MiB, above the 32 MiB scratch:
    # rejected before any launch, with a message saying why.
    fake = ctypes.c_void_p(0x10000)
    rc = lib.convrot_w4a4_linear_noalloc(fake, fake, fake, None, 8704, 3072, 12288, fake, None)
    assert rc == 5  # CONVROT_ERR_WORKSPACE
    assert b"limit" in lib.convrot_last_error()
