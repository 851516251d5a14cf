"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/convrot.h declares, and rejects bad arguments before it
touches a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from rotation_quantized_bit_b200 import build
    build.build()
    import rotation_quantized_bit_b200 as rq
    return rq.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "convrot.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_0-9]+)\s*\(", text)) - {"if", "sizeof"})


def test_header_declares_the_public_names():
    names = declared_functions()
    for need in ["convrot_pack_weight", "convrot_rotate_quant", "w4a4_gemm", "convrot_w4a4_linear"]:
        assert need in names


def test_every_declared_symbol_is_exported(lib):
    import rotation_quantized_bit_b200 as rq
    names = declared_functions()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/convrot.h but not exported"
    assert sorted(rq.EXPORTS) == names


def test_status_strings(lib):
    for code in range(8):
        s = lib.convrot_status_string(code).decode()
        assert s.startswith("CONVROT_")
    assert b"UNKNOWN" in lib.convrot_status_string(99)


def test_workspace_sizes(lib):
    assert lib.convrot_w4a4_workspace_size(32, 256, 512) >= 32 * 512 + 32 * 4
    assert lib.convrot_gemm_workspace_size(1220, 9728, 2560) >= 1220 * 2560
    assert lib.convrot_w4a4_workspace_size(32, 256, 300) == 0  # bad K
    assert lib.convrot_w4a4_workspace_size(0, 256, 512) == 0
    assert lib.convrot_w4a4_workspace_size(32, 250, 512) == 0  # N % 8 != 0


def _r256(v):
    return (v + 255) // 256 * 256


def _small_scratch(M, N, K):
    # The small-M GEMM takes one CTA per 16-channel slab; it splits K into
    # parts only where a slab's K range would not fit its shared memory (96
    # blocks of 128) or there are fewer slabs than SMs (148), at least 4
    # blocks per part, at most 64 parts.  Split slabs need one counter per
    # slab and one int32 partial slab (8 or 16 tokens x 16 channels) per part.
    tiles, nb = (N + 15) // 16, K // 128
    parts = max((nb + 95) // 96, (148 + tiles - 1) // tiles)
    parts = max(1, min(parts, max(nb // 4, 1), 64))
    if parts == 1:
        return 256
    return _r256(4 * tiles) + _r256(tiles * parts * (8 if M <= 8 else 16) * 16 * 4)


def test_workspace_layout(lib):
    # Codes (one byte each) then the per-token scales, each rounded to 256;
    # for M <= 16 the small-M GEMM's scratch follows.
    for M, N, K in ((4224, 3840, 3840), (76, 2560, 9728), (77, 264, 768), (17, 256, 512)):
        assert lib.convrot_gemm_workspace_size(M, N, K) == _r256(M * K)
        assert lib.convrot_w4a4_workspace_size(M, N, K) == _r256(M * K) + _r256(4 * M)
    for M, N, K in ((1, 9728, 2560), (8, 256, 512), (9, 2560, 9728), (16, 12288, 3072), (16, 2560, 32768),
                    (3, 1024, 2560)):
        assert lib.convrot_gemm_workspace_size(M, N, K) == _small_scratch(M, N, K)
        assert lib.convrot_w4a4_workspace_size(M, N, K) == _r256(M * K) + _r256(4 * M) + _small_scratch(M, N, K)


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
FAKE_ODD = ctypes.c_void_p(0x10001)  # misaligned


@pytest.mark.parametrize("M,N,K,code", [
    (0, 256, 512, 2), (32, 0, 512, 2), (32, 12, 512, 2), (32, 256, 500, 2), (32, 256, 128, 2),
    (32, 256, 65536, 2),
])
def test_shape_errors_are_synchronous(lib, M, N, K, code):
    rc = lib.convrot_w4a4_linear(FAKE, FAKE, FAKE, None, M, N, K, FAKE, FAKE, 1 << 30, None)
    assert rc == code


def test_null_alignment_and_workspace_errors(lib):
    assert lib.convrot_w4a4_linear(None, FAKE, FAKE, None, 32, 256, 512, FAKE, FAKE, 1 << 30, None) == 1
    assert lib.convrot_w4a4_linear(FAKE_ODD, FAKE, FAKE, None, 32, 256, 512, FAKE, FAKE, 1 << 30, None) == 3
    assert lib.convrot_w4a4_linear(FAKE, FAKE, FAKE, None, 32, 256, 512, FAKE, FAKE, 16, None) == 5
    assert lib.convrot_w4a4_linear(FAKE, FAKE, FAKE, None, 32, 256, 512, FAKE, None, 1 << 30, None) == 5
    assert lib.convrot_rotate_quant(FAKE, 4, 512, None, FAKE, None) == 1
    assert lib.w4a4_gemm_s32(FAKE, FAKE, 4, 256, 512, FAKE_ODD, FAKE, 1 << 30, None) == 3
    assert lib.w4a4_gemm(FAKE, None, FAKE, FAKE, None, 4, 256, 512, FAKE, FAKE, 1 << 30, None) == 1


def test_dispatch_counters_without_a_gpu(lib):
    import torch
    arr = (ctypes.c_uint64 * 8)(*([7] * 8))
    lib.convrot_dispatch_counts(arr, 8)
    assert list(arr[6:]) == [7, 7]  # six kinds are counted; the rest of the array is left alone
    if not torch.cuda.is_available():
        assert list(arr[:6]) == [0] * 6  # argument errors never reach a launch


def test_version(lib):
    assert b"sm_100a" in lib.convrot_version()


def test_int8_workspace_sizes(lib):
    # codes M*K, scales (M floats), 256 bytes of reduction scratch, each 256-aligned
    assert lib.w8a8_workspace_size(76, 1024, 2560, 0) == _r256(76 * 2560) + _r256(76 * 4) + 256
    assert lib.w8a8_workspace_size(76, 1024, 2560, 1) == _r256(76 * 2560) + _r256(76 * 4) + 256
    assert lib.w8a8_workspace_size(76, 1024, 2560, 2) == 0      # unknown format
    assert lib.w8a8_workspace_size(76, 1024, 300, 0) == 0       # K % 256
    assert lib.w8a8_workspace_size(76, 1020, 2560, 0) == 0      # N % 8


def test_int8_and_group_arguments_rejected_before_any_device_call(lib):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 16)
    good = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    null = P(0)
    # NULL pointers
    assert lib.w8a8_quantize(null, 4, 256, 0, good, good, good, 4096, null) == 1
    assert lib.w8a8_gemm(null, good, good, good, null, 4, 8, 256, 0, good, null) == 1
    assert lib.convrot_rotate_quant_g(null, 4, 256, 64, good, good, null) == 1
    # bad format / group / shape
    assert lib.w8a8_quantize(good, 4, 256, 9, good, good, good, 4096, null) == 2
    assert lib.w8a8_gemm(good, good, good, good, null, 4, 8, 256, 5, good, null) == 2
    assert lib.w8a8_gemm_s32(good, good, 4, 8, 300, good, null) == 2
    assert lib.convrot_rotate_quant_g(good, 4, 256, 32, good, good, null) == 2
    assert lib.convrot_w4a4_quantize_g(good, 4, 256, 128, good, 4096, null) == 2
    # misaligned pointer
    bad = P(good.value + 4)
    assert lib.w8a8_gemm_s32(bad, good, 4, 8, 256, good, null) == 3
    # a too small workspace for the fused int8 linear
    assert lib.w8a8_linear(good, good, good, null, 4, 8, 256, 0, good, good, 16, null) == 5


def test_asym_workspace_sizes(lib):
    # the asymmetric W4A8 activations are the ConvRot INT8 row-scaled codes and scales
    assert lib.asym_w4a8_workspace_size(76, 1024, 2560) == _r256(76 * 2560) + _r256(76 * 4) + 256
    assert lib.asym_w4a8_workspace_size(1, 8, 256) == _r256(256) + _r256(4) + 256
    assert lib.asym_w4a8_workspace_size(76, 1024, 300) == 0   # K % 256
    assert lib.asym_w4a8_workspace_size(76, 1020, 2560) == 0  # N % 8
    assert lib.asym_w4a8_workspace_size(0, 8, 256) == 0       # M >= 1


def test_asym_arguments_rejected_before_any_device_call(lib):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 16)
    good = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    null = P(0)
    # NULL operands: activations, indices, group scales, codebook; scales except for the s32 sink
    assert lib.asym_w4a8_gemm(null, good, good, good, good, good, null, 4, 8, 256, good, null) == 1
    assert lib.asym_w4a8_gemm(good, good, good, null, good, good, null, 4, 8, 256, good, null) == 1
    assert lib.asym_w4a8_gemm(good, good, good, good, null, good, null, 4, 8, 256, good, null) == 1
    assert lib.asym_w4a8_gemm_f32(good, null, good, good, good, good, null, 4, 8, 256, good, null) == 1
    assert lib.asym_w4a8_gemm_f32(good, good, good, good, good, null, null, 4, 8, 256, good, null) == 1
    assert lib.asym_w4a8_gemm_s32(good, good, good, null, 4, 8, 256, good, null) == 1
    assert lib.asym_w4a8_linear(good, good, good, good, null, null, 4, 8, 256, good, good, 4096, null) == 1
    # shapes: K % 256, N % 8, M >= 1
    assert lib.asym_w4a8_gemm_s32(good, good, good, good, 4, 8, 128, good, null) == 2
    assert lib.asym_w4a8_gemm_s32(good, good, good, good, 4, 12, 256, good, null) == 2
    assert lib.asym_w4a8_gemm_s32(good, good, good, good, 0, 8, 256, good, null) == 2
    assert lib.asym_w4a8_linear_f32(good, good, good, good, good, null, 4, 8, 300, good, good, 4096, null) == 2
    # misaligned codebook / group scales
    bad = P(good.value + 4)
    assert lib.asym_w4a8_gemm_s32(good, good, good, bad, 4, 8, 256, good, null) == 3
    assert lib.asym_w4a8_gemm_s32(good, good, bad, good, 4, 8, 256, good, null) == 3
    # a too small workspace for the fused linear
    assert lib.asym_w4a8_linear(good, good, good, good, good, null, 4, 8, 256, good, good, 16, null) == 5


def test_binding_takes_cuda_tensors_on_one_device():
    # Host tensors are refused by the binding itself, before any library call
    # (no CPU path); tensors on several devices are refused the same way.
    import torch
    import rotation_quantized_bit_b200 as rq
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    wq = torch.zeros(8, 128, dtype=torch.uint8)
    s = torch.zeros(8)
    for call in (lambda: rq.convrot_w4a4_linear(x, wq, s), lambda: rq.convrot_rotate_quant(x),
                 lambda: rq.convrot_pack_weight(x), lambda: rq.w4a4_gemm_s32(wq, wq),
                 lambda: rq.convrot_w4a4_linear_noalloc(x, wq, s), lambda: rq.w8a8_quantize(x, rq.W8A8_INT8_TENSORWISE),
                 lambda: rq.convrot_w4a4_linear_g(x, wq, s, group=64)):
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
    meta = torch.zeros(8, 128, dtype=torch.uint8, device="meta")
    with pytest.raises(ValueError):
        rq.w4a4_gemm_s32(meta, meta)
