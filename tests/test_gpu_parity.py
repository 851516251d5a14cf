"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on the same seeded inputs.

Bar (stated by the method's contract):
  * codes (packed bytes), scales (raw fp32 bits) and the int32 accumulators:
    bit-exact;
  * fp32 output: |y - y_oracle| <= 1e-5 * max|y_oracle|;
  * bf16 output: within one bf16 ulp of the oracle's bf16.
Small cases span several tiles and ragged tails; the full workload shapes
(the ones the benchmark times, through the same entry point and launch
configuration) are checked on sampled rows that include the first tile, a
middle tile and the M tail.
"""
import functools

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
    """|a - b| in units of bf16 ulps, via the monotone integer mapping."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(key(a_bits) - key(b_bits))


def check_f32(y, ref):
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    err = float(np.max(np.abs(y.astype(np.float64) - ref.astype(np.float64))))
    assert err <= F32_TOL * scale, f"max err {err} > {F32_TOL} * {scale}"


# ------------------------------------------------------------- rotate / quant

RQ_CASES = [("small", 32, 512), ("qwen3_4b", 77, 2560), ("qwen3_4b", 1, 256), ("dit6b", 300, 3840),
            ("edit20b", 5, 12288), ("qwen3_4b", 129, 9728), ("dit6b", 64, 10240)]


@pytest.mark.parametrize("workload,M,K", RQ_CASES)
def test_rotate_quant_bit_exact(rq, workload, M, K):
    x = synthetic.activations(workload, M, K)
    xq_ref, s_ref = oracle.rotate_quant(x)
    xq, s = rq.convrot_rotate_quant(dev_bf16(x))
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(xq), xq_ref)


def special_rows(K=512):
    rows = []
    z = np.zeros(K)
    rows.append(z.copy())                                    # all zero -> s = 0, codes 0
    for v1 in (8, 24, 40, 56, 72, 88, 104):                  # exact half-integer ties
        r = z.copy(); r[0] = 112.0; r[256] = v1; rows.append(r)
    for A, B in ((1.421875, 1.3203125), (1.53125, 1.421875), (2.0625, 1.03125),
                 (2.546875, 1.2734375), (2.609375, 1.3046875)):  # division vs reciprocal ties
        r = z.copy(); r[0] = A; r[256] = B; rows.append(r)
    r = z.copy(); r[:] = 3.0; rows.append(r)                 # constant vector
    r = z.copy(); r[5] = -1e-38; r[300] = 3e-39; rows.append(r)  # subnormal scale
    r = z.copy(); r[7] = 1.0e37; r[8] = -8.0e36; rows.append(r)  # huge values, partial sums stay finite
    r = z.copy(); r[::3] = 1e-30; rows.append(r)             # tiny values
    return synthetic.to_bf16_bits(np.stack(rows))


def near_tie_rows(n_rows=384, K=512, seed=11):
    """Rows whose quotients x'/s_a sit at or next to a half-integer, kept only
    where a quotient formed as x' * fl(1/s_a) would round to another code than
    the division: the cases a reciprocal-based quantizer gets wrong.

    Each row holds A at channel 0 (group 0 rotates to +-A/16, the row amax)
    and B at channel 256 (group 1 rotates to +-B/16).  Two families:
      * exact ties: A = 7 m 2^e, B = (k + 1/2) m 2^e, so fl(A/16)/7 is exact
        and B/16 divided by it is exactly k + 1/2;
      * near ties: A = c B with c = 14 / (2k + 1), so the quotient is
        (k + 1/2)(1 + d) with d the rounding of s_a = fl(fl(A/16) / 7).
    The filter runs in numpy fp32 (IEEE division and multiplication)."""
    rng = np.random.default_rng(seed)
    f = np.float32
    cand = []
    for _ in range(40000):
        if len(cand) >= 2 * n_rows:
            break
        k = int(rng.integers(0, 7))
        e = float(2.0 ** int(rng.integers(-20, 20)))
        if rng.random() < 0.5:
            m = int(rng.integers(1, 37))
            A, B = 7 * m * e, (k + 0.5) * m * e
        else:
            B = float(synthetic.bf16_bits_to_f32(synthetic.to_bf16_bits(np.array([rng.uniform(0.5, 1.0) * e])))[0])
            A = 14.0 / (2 * k + 1) * B
        bits = synthetic.to_bf16_bits(np.array([A, B]))
        Af, Bf = synthetic.bf16_bits_to_f32(bits).astype(np.float32)
        if Af != np.float32(A) or Bf != np.float32(B) or abs(Af) <= abs(Bf):
            continue
        s = f(f(Af / f(16)) / f(7))
        x = f(Bf / f(16))
        if np.rint(f(x / s)) != np.rint(f(x * f(f(1) / s))):
            cand.append((float(Af), float(Bf)))
    cand = sorted(set(cand))[:n_rows]
    rows = np.zeros((len(cand), K))
    for i, (A, B) in enumerate(cand):
        rows[i, 0] = A
        rows[i, 256] = -B if i % 2 else B
    return synthetic.to_bf16_bits(rows)


def test_rotate_quant_near_ties(rq):
    x = near_tie_rows()
    assert x.shape[0] >= 32, "the search found too few rows that separate division from reciprocal"
    xq_ref, s_ref = oracle.rotate_quant(x)
    xq, s = rq.convrot_rotate_quant(dev_bf16(x))
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(xq), xq_ref)


@pytest.mark.parametrize("M", [1, 7, 77, 300, 1220])
@pytest.mark.parametrize("K", [256, 512, 2560, 3072, 3840, 9728, 12288, 32768])
def test_rotate_quant_shape_grid(rq, M, K):
    if M * K > 1220 * 12288:
        pytest.skip("keeps the CPU oracle within seconds")
    x = synthetic.activations("qwen3_4b", M, K, seed_extra=K)
    xq_ref, s_ref = oracle.rotate_quant(x)
    xq, s = rq.convrot_rotate_quant(dev_bf16(x))
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(xq), xq_ref)


def test_rotate_quant_special_rows(rq):
    x = special_rows()
    xq_ref, s_ref = oracle.rotate_quant(x)
    xq, s = rq.convrot_rotate_quant(dev_bf16(x))
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))
    assert np.array_equal(host(xq), xq_ref)


@pytest.mark.parametrize("workload,N,K", [("small", 256, 512), ("qwen3_4b", 1024, 2560), ("dit6b", 136, 3840)])
def test_pack_weight_bit_exact(rq, workload, N, K):
    w, _ = synthetic.weights(workload, N, K)
    wq_ref, s_ref = oracle.pack_weight(w)
    wq, s = rq.convrot_pack_weight(dev_bf16(w))
    assert np.array_equal(host(wq), wq_ref)
    assert np.array_equal(f32_bits(host(s)), f32_bits(s_ref))


# ------------------------------------------------------------- GEMM sinks

GEMM_CASES = [(8, 256, 256), (32, 256, 512), (77, 264, 768), (1, 128, 2560), (16, 2560, 2560),
              (200, 384, 1024), (300, 1000, 512), (193, 136, 256), (600, 4096, 512),
              # split-K clusters: one tile split 8 ways; ragged N; the largest
              # small-M tile; uneven K shares; whole small-M tiles
              (3, 8, 12288), (16, 1032, 9728), (128, 2056, 768), (64, 136, 32768), (40, 3072, 1280),
              (16, 19456, 512),
              # persistent large-M path: several tiles per SM, ragged M and N tails
              (1000, 1280, 1024), (777, 2056, 768), (2100, 1024, 256)]


def random_codes(seed, rows, K):
    rng = np.random.default_rng(seed)
    return rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)  # every nibble, -8 included


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_gemm_s32_bit_exact(rq, M, N, K):
    xq = random_codes(M * 7 + K, M, K)
    wq = random_codes(N * 13 + K, N, K)
    ref = oracle.gemm_s64(xq, wq, K)
    acc = rq.w4a4_gemm_s32(dev(xq), dev(wq))
    assert np.array_equal(host(acc).astype(np.int64), ref)


def test_gemm_s32_extremes(rq):
    K = 3840
    for a, b, want in ((0x77, 0x77, 49 * K), (0x88, 0x88, 64 * K), (0x88, 0x77, -56 * K)):
        xq = np.full((24, K // 2), a, np.uint8)
        wq = np.full((136, K // 2), b, np.uint8)
        assert np.all(host(rq.w4a4_gemm_s32(dev(xq), dev(wq))) == want)


@pytest.mark.parametrize("M,N,K", [(32, 256, 512), (77, 264, 768), (193, 136, 256), (600, 4096, 512)])
def test_gemm_f32_and_bf16(rq, M, N, K):
    x = synthetic.activations("qwen3_4b", M, K)
    w, b = synthetic.weights("qwen3_4b", N, K)
    xq, s_a = oracle.rotate_quant(x)
    wq, s_w = oracle.pack_weight(w)
    acc = oracle.gemm_s64(xq, wq, K)
    y32_ref, y16_ref = oracle.epilogue(acc, s_a, s_w, b)
    args = (dev(xq), dev(s_a), dev(wq), dev(s_w), dev_bf16(b))
    y32 = host(rq.w4a4_gemm_f32(*args))
    check_f32(y32, y32_ref)
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))  # same op order as the oracle -> identical bits
    y16 = host_bits(rq.w4a4_gemm(*args))
    assert bf16_ulp_diff(y16, y16_ref).max() <= 1
    # no bias
    y32n = host(rq.w4a4_gemm_f32(dev(xq), dev(s_a), dev(wq), dev(s_w), None))
    check_f32(y32n, oracle.epilogue(acc, s_a, s_w, None)[0])


# ------------------------------------------------------------- fused Linear

LINEAR_CASES = [("small", 32, 512, 256), ("qwen3_4b", 77, 2560, 264), ("qwen3_4b", 1, 2560, 1024),
                ("dit6b", 250, 3840, 384), ("edit20b", 16, 3072, 12288), ("qwen3_4b", 8, 9728, 2560),
                ("dit6b", 600, 3840, 1024), ("qwen3_4b", 1220, 2560, 1024)]


@pytest.mark.parametrize("workload,M,K,N", LINEAR_CASES)
def test_linear_matches_oracle(rq, workload, M, K, N):
    x = synthetic.activations(workload, M, K)
    w, b = synthetic.weights(workload, N, K)
    wq, s_w = oracle.pack_weight(w)
    y32_ref, y16_ref = oracle.linear(x, wq, s_w, b, K)
    dx, dwq, dsw, db = dev_bf16(x), dev(wq), dev(s_w), dev_bf16(b)
    y32 = host(rq.convrot_w4a4_linear_f32(dx, dwq, dsw, db))
    check_f32(y32, y32_ref)
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))
    y16 = host_bits(rq.convrot_w4a4_linear(dx, dwq, dsw, db))
    assert bf16_ulp_diff(y16, y16_ref).max() <= 1


def test_quantize_once_gemm_many(rq):
    # Projections sharing one input: one quantization, several GEMMs on the
    # same workspace, which they only read.
    M, K = 76, 2560
    x = synthetic.activations("qwen3_4b", M, K)
    xq_ref, s_a = oracle.rotate_quant(x)
    shapes = [4096, 1024, 1032, 9728]
    ws = torch.empty(max(rq.convrot_w4a4_workspace_size(M, N, K) for N in shapes), dtype=torch.uint8,
                     device="cuda")
    rq.convrot_w4a4_quantize(dev_bf16(x), ws)
    for N in shapes:
        w, b = synthetic.weights("qwen3_4b", N, K)
        wq, s_w = oracle.pack_weight(w)
        y16_ref = oracle.epilogue(oracle.gemm_s64(xq_ref, wq, K), s_a, s_w, b)[1]
        y16 = host_bits(rq.convrot_w4a4_gemm_quantized(ws, M, dev(wq), dev(s_w), dev_bf16(b)))
        assert bf16_ulp_diff(y16, y16_ref).max() <= 1, N


def test_linear_special_rows(rq):
    # Ties, division-vs-reciprocal cases, zero / subnormal / huge rows through
    # the fused path (its prologue writes byte codes for the GEMM operand).
    x = special_rows()
    M, K, N = x.shape[0], x.shape[1], 264
    w, b = synthetic.weights("qwen3_4b", N, K)
    wq, s_w = oracle.pack_weight(w)
    y32_ref, _ = oracle.linear(x, wq, s_w, b, K)
    y32 = host(rq.convrot_w4a4_linear_f32(dev_bf16(x), dev(wq), dev(s_w), dev_bf16(b)))
    assert np.array_equal(f32_bits(y32), f32_bits(y32_ref))


def sample_rows(M, BT_guess=192):
    rows = set(range(min(M, 8)))
    rows |= set(range(max(0, M - 8), M))
    mid = M // 2
    rows |= set(range(max(0, mid - 4), min(M, mid + 4)))
    return sorted(rows)


FULL = [s for wl in ("qwen3_4b", "dit6b", "edit20b", "small_m") for s in synthetic.workload_shapes(wl)]


@functools.lru_cache(maxsize=2)
def _full_x(wl, M, K):
    return synthetic.activations(wl, M, K)


@functools.lru_cache(maxsize=2)
def _full_w(wl, N, K):
    """The weights and bias of a full-size linear, and the oracle's packing of
    the whole weight matrix (its codes and scales are the reference)."""
    w, b = synthetic.weights(wl, N, K)
    wq_ref, sw_ref = oracle.pack_weight(w)
    return w, b, wq_ref, sw_ref


@pytest.mark.parametrize("shape", FULL, ids=lambda s: f"{s.name}-M{s.M}-K{s.K}-N{s.N}")
def test_full_size_linear_sampled_rows(rq, shape):
    wl = next(w for w in ("qwen3_4b", "dit6b", "edit20b", "small_m")
              if shape in synthetic.workload_shapes(w))
    M, K, N = shape.M, shape.K, shape.N
    x = _full_x(wl, M, K)
    w, b, wq_ref, sw_ref = _full_w(wl, N, K)
    # The weights prepared on the GPU are the oracle's, every code and scale.
    dwq, dsw = rq.convrot_pack_weight(dev_bf16(w))
    assert np.array_equal(host(dwq), wq_ref)
    assert np.array_equal(f32_bits(host(dsw)), f32_bits(sw_ref))
    y32 = host(rq.convrot_w4a4_linear_f32(dev_bf16(x), dwq, dsw, dev_bf16(b)))
    y16 = host_bits(rq.convrot_w4a4_linear(dev_bf16(x), dwq, dsw, dev_bf16(b)))
    # The reference Linear uses the oracle's own codes and scales only.
    for r0, r1 in _runs(sample_rows(M)):
        ref32, ref16 = oracle.linear(x, wq_ref, sw_ref, b, K, rows=(r0, r1))
        check_f32(y32[r0:r1], ref32)
        assert np.array_equal(f32_bits(y32[r0:r1]), f32_bits(ref32))
        assert bf16_ulp_diff(y16[r0:r1], ref16).max() <= 1


def _runs(rows):
    out, start, prev = [], rows[0], rows[0]
    for r in rows[1:]:
        if r != prev + 1:
            out.append((start, prev + 1))
            start = r
        prev = r
    out.append((start, prev + 1))
    return out


# ------------------------------------------------------------- boundary behaviour


def test_errors_raise_before_launch(rq):
    x = torch.zeros((4, 300), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.ConvRotError) as e:
        rq.convrot_rotate_quant(x)
    assert e.value.status == "CONVROT_ERR_SHAPE"
    buf = torch.zeros(4 * 512 * 2 + 16, dtype=torch.uint8, device="cuda")
    lib = rq.load_library()
    import ctypes
    rc = lib.convrot_rotate_quant(ctypes.c_void_p(buf.data_ptr() + 2), 4, 512, ctypes.c_void_p(buf.data_ptr()),
                                  ctypes.c_void_p(buf.data_ptr()), None)
    assert rq.STATUS[rc] == "CONVROT_ERR_ALIGN"


def test_dispatch_counts_and_no_device_error(rq):
    before = rq.convrot_dispatch_counts()
    x = dev_bf16(synthetic.activations("small", 32, 512))
    w, b = synthetic.weights("small", 256, 512)
    wq, s_w = rq.convrot_pack_weight(dev_bf16(w))
    rq.convrot_w4a4_linear(x, wq, s_w, dev_bf16(b))
    after = rq.convrot_dispatch_counts()
    assert after["rotate_quant"] == before["rotate_quant"] + 2
    assert after["tc_gemm"] + after["tc_gemm_splitk"] == before["tc_gemm"] + before["tc_gemm_splitk"] + 1
    assert rq.convrot_device_error() == 0
