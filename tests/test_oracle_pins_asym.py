"""Pins for the CPU oracle's asymmetric W4A8 format ("asym_w4a8_int8":
"Nicolaslas/Rebels_w4a8s", "What's inside a file" -- 4-bit codebook indices two
per byte, an fp8 scale per 16 weights, one scale per output channel, a 16-level
Lloyd-Max codebook per tensor under the group-256 ConvRot rotation; int8
tensor cores do the math).  Each test checks the oracle against something
other than itself: torch's e4m3 conversions (a library routine), hand-derived
decodes (ties, saturation, nibble and group order), the reduction to the
ConvRot INT8 row-scaled Linear pinned in test_oracle_pins_int8.py, the
optimality conditions of a Lloyd-Max quantizer, and the pages' ~7 % weight
error as a plausibility band.  Mutants of the asym code are planted on the
CPU at the end.  No test here needs a GPU.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import synthetic

E4M3_ONE = 0x38  # 1.0
E4M3_MAX = 0x7E  # 448
E4M3_NAN = 0x7F


def torch_e4m3_decode(b):
    t = torch.from_numpy(np.ascontiguousarray(b, np.uint8)).view(torch.float8_e4m3fn)
    return t.float().numpy()


def torch_e4m3_encode(v):
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pack_idx(i):
    i = np.asarray(i, np.uint8)
    return (i[..., 0::2] | (i[..., 1::2] << 4)).astype(np.uint8)


# ---------------------------------------------------------------- e4m3

def test_e4m3_decode_matches_torch_on_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    mine, ref = oracle.e4m3_to_f32(b), torch_e4m3_decode(b)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.isnan(mine).sum() == 2  # 0x7F and 0xFF
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok].view(np.uint32), ref[ok].view(np.uint32))  # signed zeros included
    assert float(mine[E4M3_MAX]) == 448.0 and float(mine[1]) == 2.0 ** -9


def test_e4m3_encode_round_to_nearest_even_matches_torch():
    rng = np.random.default_rng(3)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = torch_e4m3_decode(codes)
    # every finite code round-trips; midpoints of neighbours go to the even code
    assert np.array_equal(oracle.f32_to_e4m3(vals), codes)
    pos = np.sort(np.unique(vals[vals > 0]))
    mids = ((pos[:-1].astype(np.float64) + pos[1:]) / 2).astype(np.float32)
    sweep = np.concatenate([mids, -mids, rng.uniform(-447.0, 447.0, 3000).astype(np.float32),
                            rng.uniform(-0.02, 0.02, 1000).astype(np.float32)])
    assert np.array_equal(oracle.f32_to_e4m3(sweep), torch_e4m3_encode(sweep))
    # saturation above the largest finite value (reading; the converter never reaches it)
    assert oracle.f32_to_e4m3(np.array([500.0, -1e9], np.float32)).tolist() == [E4M3_MAX, 0x80 | E4M3_MAX]


# ---------------------------------------------------------------- decode

def test_decode_integer_codebook_and_nibble_order():
    cb = np.arange(-8, 8, dtype=np.float32)            # level i = i - 8
    idx = np.tile(np.arange(16, dtype=np.uint8), 2)[None, :]  # k -> index k % 16
    w8 = oracle.asym_decode(pack_idx(idx), np.full((1, 2), E4M3_ONE, np.uint8), cb)
    assert w8[0].tolist() == [i - 8 for i in range(16)] * 2
    # one byte 0x10 holds index 0 at even k and index 1 at odd k
    w8 = oracle.asym_decode(np.full((1, 8), 0x10, np.uint8), np.full((1, 1), E4M3_ONE, np.uint8), cb)
    assert w8[0].tolist() == [-8, -7] * 8


def test_decode_ties_saturation_signs_and_nan():
    cb = np.array([0.5, 1.5, 2.5, -0.5, -2.5, 1.0, -1.0, 0.0, 7.0, 126.5, 127.49, -3.5, 0.25, 0.75, 3.0, 5.0],
                  np.float32)
    idx = pack_idx(np.arange(16)[None, :])
    dec = lambda sb: oracle.asym_decode(idx, np.array([[sb]], np.uint8), cb)[0].tolist()
    assert dec(E4M3_ONE) == [0, 2, 2, 0, -2, 1, -1, 0, 7, 126, 127, -4, 0, 1, 3, 5]
    # 448: every product beyond +-127 clamps to +-127 (never -128)
    assert dec(E4M3_MAX) == [127, 127, 127, -127, -127, 127, -127, 0, 127, 127, 127, -127, 112, 127, 127, 127]
    assert dec(0xB8) == [0, -2, -2, 0, 2, -1, 1, 0, -7, -126, -127, 4, 0, -1, -3, -5]  # s_rel = -1
    assert dec(0x00) == [0] * 16 and dec(0x80) == [0] * 16
    assert dec(E4M3_NAN) == [0] * 16  # NaN products decode to 0 (reading)
    assert dec(0x01) == [0] * 8 + [0, 0, 0, 0, 0, 0, 0, 0]  # 2^-9: every |product| < 0.5


def test_decode_uses_the_group_of_sixteen():
    K = 256
    cb = np.full(16, 1.0, np.float32)
    cb[3] = -2.0
    s_rel = torch_e4m3_encode(np.arange(1, 17, dtype=np.float32))[None, :]  # group g scale g + 1 (exact)
    idx = np.zeros((1, K), np.uint8)
    idx[0, 5::16] = 3
    w8 = oracle.asym_decode(pack_idx(idx), s_rel, cb)[0]
    g = np.arange(K) // 16
    expect = np.where(np.arange(K) % 16 == 5, -2 * (g + 1), g + 1)
    assert w8.tolist() == expect.tolist()


@pytest.mark.parametrize("bias", [True, False])
def test_asym_linear_reduces_to_the_int8_row_linear(bias):
    """With integer levels and s_rel = 1 the decoded weights are the levels, so
    the asym Linear is the ConvRot INT8 row-scaled Linear on those weights."""
    M, N, K = 9, 24, 512
    rng = np.random.default_rng(11)
    x = synthetic.activations("qwen3_4b", M, K)
    cb = np.array(sorted(rng.choice(np.arange(-127, 128), 16, replace=False)), np.float32)
    idx = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    sc = (rng.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)
    bb = synthetic.to_bf16_bits(rng.normal(0, 0.01, N)) if bias else None
    y32, y16 = oracle.asym_linear(x, pack_idx(idx), np.full((N, K // 16), E4M3_ONE, np.uint8), cb, sc, bb)
    r32, r16 = oracle.linear8(x, cb[idx].astype(np.int8), sc, bb, *oracle.CONVROT_ROW)
    assert np.array_equal(y32.view(np.uint32), r32.view(np.uint32)) and np.array_equal(y16, r16)
    # a row window gives the same rows
    w32, _ = oracle.asym_linear(x, pack_idx(idx), np.full((N, K // 16), E4M3_ONE, np.uint8), cb, sc, bb, rows=(3, 8))
    assert np.array_equal(w32, y32[3:8])


# ---------------------------------------------------------------- Lloyd-Max

def cells(u, levels):
    return np.argmin(np.abs(u[:, None].astype(np.float64) - levels[None, :]), axis=1)


def test_lloyd_recovers_sixteen_clusters():
    rng = np.random.default_rng(5)
    centres = np.linspace(-0.9, 0.9, 16) + rng.uniform(-0.02, 0.02, 16)
    pts = np.concatenate([c + rng.uniform(-0.01, 0.01, 200) for c in centres]).astype(np.float32)
    lv = oracle.lloyd_max16(pts)
    for j in range(16):
        assert lv[j] == pytest.approx(pts[200 * j:200 * (j + 1)].astype(np.float64).mean(), abs=1e-12)


def test_lloyd_fixed_point_conditions_and_monotone_distortion():
    u = (synthetic.student_t4(17, 20000) * 0.3).clip(-1.2, 1.2).astype(np.float32)
    lv = oracle.lloyd_max16(u, 200)
    assert np.all(np.diff(lv) > 0)
    c = cells(u, lv)
    for j in range(16):  # centroid condition: each level is the mean of its nearest-neighbour cell
        assert lv[j] == pytest.approx(u[c == j].astype(np.float64).mean(), abs=1e-12)
    dist = []
    for it in range(1, 12):
        l = oracle.lloyd_max16(u, it)
        dist.append(np.mean((u - l[cells(u, l)]) ** 2))
    assert all(b <= a + 1e-15 for a, b in zip(dist, dist[1:]))
    assert dist[-1] < dist[0]


def test_lloyd_uniform_data_keeps_the_uniform_quantizer():
    # for u uniform on [-1, 1] the optimal 16-level quantizer has levels at the
    # centres of 16 equal cells (closed form); the start is that point
    u = ((np.arange(32000) + 0.5) / 16000.0 - 1.0).astype(np.float32)
    lv = oracle.lloyd_max16(u, 50)
    assert np.allclose(lv, -1.0 + (2 * np.arange(16) + 1) / 16.0, atol=1e-7)


# ---------------------------------------------------------------- converter

def test_convert_follows_its_steps_and_error_band():
    N, K = 64, 512
    W, _ = synthetic.weights("qwen3_4b", N, K)
    idx, s_rel, sc, cb = oracle.asym_convert(W)
    wr = oracle.rotate_rows_f32(synthetic.bf16_bits_to_f32(W), 256)  # pinned in test_oracle_pins.py
    sc_ref = np.abs(wr).max(1) / np.float32(127)
    assert np.array_equal(sc.view(np.uint32), sc_ref.astype(np.float32).view(np.uint32))
    ga = np.abs(wr).reshape(N, K // 16, 16).max(2)
    assert np.array_equal(s_rel, torch_e4m3_encode(ga / sc_ref[:, None]))
    d = (sc_ref[:, None] * torch_e4m3_decode(s_rel)).astype(np.float32)
    u = (wr.reshape(N, K // 16, 16) / d[:, :, None]).reshape(N, K)
    ii = np.stack([idx & 15, idx >> 4], -1).reshape(N, K)
    assert np.array_equal(ii, cells(u.reshape(-1), cb.astype(np.float64)).reshape(N, K))
    assert np.all(np.diff(cb) > 0)
    # the pages report ~7 % relative L2 weight error for this format (a
    # plausibility band around the printed value, not an exact pin)
    deq = sc[:, None].astype(np.float64) * oracle.asym_decode(idx, s_rel, cb)
    rel = np.linalg.norm(deq - wr) / np.linalg.norm(wr)
    assert abs(rel - read_layout()["weight_rel_l2_printed"]) < 0.03


# ---------------------------------------------------------------- mutants

SRC = os.path.join(os.path.dirname(oracle.__file__), "convrot_oracle.c")

MUTANTS_ASYM = {
    "asym_nibble_swap": ("int i = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);",
                         "int i = (k % 2 == 0) ? (byte >> 4) : (byte & 0xF);"),
    "asym_group_swap": ("s_rel[(size_t)n * (K / 16) + k / 16]);", "s_rel[(size_t)n * (K / 16) + ((k / 16) ^ 1)]);"),
    "asym_round_half_away": ("return (int8_t)rintf(p);", "return (int8_t)roundf(p);"),
    "asym_clamp_128": ("if (p < -127.0f) return -127;", "if (p < -128.0f) return -128;"),
    "e4m3_exponent_bias": ("ldexp(8.0 + (double)m, e - 10)", "ldexp(8.0 + (double)m, e - 11)"),
    "e4m3_subnormal_scale": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "e4m3_ties_to_odd": ("if (d < bd || (d == bd && (c & 1) == 0)) {", "if (d < bd || (d == bd && (c & 1) == 1)) {"),
    "lloyd_biased_mean": ("levels[j] = sum[j] / (double)cnt[j];", "levels[j] = sum[j] / (double)(cnt[j] + 1);"),
    "convert_channel_128": ("float sc = amax / 127.0f;", "float sc = amax / 128.0f;"),
}


class LibAsym:
    def __init__(self, path):
        lib = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        lib.oracle_asym_decode.argtypes = [P, P, P, I, I, P]
        lib.oracle_lloyd_max16.argtypes = [P, ctypes.c_int64, I, P]
        lib.oracle_asym_convert.argtypes = [P, I, I, I, P, P, P, P]
        self.lib = lib

    @staticmethod
    def p(a):
        return a.ctypes.data_as(ctypes.c_void_p)

    def decode(self, idx, s_rel, cb):
        idx, s_rel, cb = (np.ascontiguousarray(a) for a in (idx, s_rel, np.asarray(cb, np.float32)))
        w8 = np.empty((idx.shape[0], 2 * idx.shape[1]), np.int8)
        self.lib.oracle_asym_decode(self.p(idx), self.p(s_rel), self.p(cb), idx.shape[0], 2 * idx.shape[1], self.p(w8))
        return w8

    def lloyd(self, u, iters):
        u = np.ascontiguousarray(u, np.float32)
        lv = np.empty(16, np.float64)
        self.lib.oracle_lloyd_max16(self.p(u), u.size, iters, self.p(lv))
        return lv

    def convert(self, W):
        W = np.ascontiguousarray(W, np.uint16)
        N, K = W.shape
        idx, s_rel = np.empty((N, K // 2), np.uint8), np.empty((N, K // 16), np.uint8)
        sc, cb = np.empty(N, np.float32), np.empty(16, np.float32)
        self.lib.oracle_asym_convert(self.p(W), N, K, 100, self.p(idx), self.p(s_rel), self.p(sc), self.p(cb))
        return idx, s_rel, sc, cb


def pins_asym_hold(lib: LibAsym) -> bool:
    """A compact re-run of the pins above against ``lib``."""
    ok = True
    b = np.arange(256, dtype=np.uint8)
    mine = np.array([lib.lib.oracle_e4m3_to_f32(int(i)) for i in b], np.float32)
    ref = torch_e4m3_decode(b)
    fin = ~np.isnan(ref)
    ok &= np.array_equal(np.isnan(mine), ~fin) and np.array_equal(mine[fin], ref[fin])
    pos = np.sort(np.unique(ref[fin & (ref > 0)]))
    mids = ((pos[:-1].astype(np.float64) + pos[1:]) / 2).astype(np.float32)
    ok &= [lib.lib.oracle_f32_to_e4m3(float(v)) for v in mids] == torch_e4m3_encode(mids).tolist()
    cb = np.array([0.5, 1.5, 2.5, -0.5, -2.5, 1.0, -1.0, 0.0, 7.0, 126.5, 127.49, -3.5, 0.25, 0.75, 3.0, 5.0],
                  np.float32)
    idx = pack_idx(np.arange(16)[None, :])
    ok &= lib.decode(idx, np.array([[E4M3_ONE]], np.uint8), cb)[0].tolist() == \
        [0, 2, 2, 0, -2, 1, -1, 0, 7, 126, 127, -4, 0, 1, 3, 5]
    ok &= lib.decode(idx, np.array([[E4M3_MAX]], np.uint8), cb)[0].tolist() == \
        [127, 127, 127, -127, -127, 127, -127, 0, 127, 127, 127, -127, 112, 127, 127, 127]
    cbg = np.full(16, 1.0, np.float32)
    cbg[3] = -2.0
    s_rel = torch_e4m3_encode(np.arange(1, 17, dtype=np.float32))[None, :]
    ii = np.zeros((1, 256), np.uint8)
    ii[0, 5::16] = 3
    g = np.arange(256) // 16
    ok &= lib.decode(pack_idx(ii), s_rel, cbg)[0].tolist() == np.where(np.arange(256) % 16 == 5, -2 * (g + 1),
                                                                        g + 1).tolist()
    rng = np.random.default_rng(5)
    centres = np.linspace(-0.9, 0.9, 16) + rng.uniform(-0.02, 0.02, 16)
    pts = np.concatenate([c + rng.uniform(-0.01, 0.01, 200) for c in centres]).astype(np.float32)
    lv = lib.lloyd(pts, 100)
    ok &= bool(np.allclose(lv, pts.reshape(16, 200).astype(np.float64).mean(1), atol=1e-12, rtol=0))
    W, _ = synthetic.weights("qwen3_4b", 16, 256)
    idx, s_rel, sc, cb = lib.convert(W)
    wr = oracle.rotate_rows_f32(synthetic.bf16_bits_to_f32(W), 256)
    ok &= np.array_equal(sc, (np.abs(wr).max(1) / np.float32(127)).astype(np.float32))
    return bool(ok)


def _build(tmp_path, name, src_text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), "-lm"])
    return str(so)


def test_asym_unmutated_copy_passes(tmp_path):
    with open(SRC) as f:
        assert pins_asym_hold(LibAsym(_build(tmp_path, "orig_asym", f.read())))


@pytest.mark.parametrize("name", sorted(MUTANTS_ASYM))
def test_asym_mutant_is_caught(tmp_path, name):
    with open(SRC) as f:
        text = f.read()
    old, new = MUTANTS_ASYM[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    assert not pins_asym_hold(LibAsym(_build(tmp_path, name, text.replace(old, new))))


# ---------------------------------------------------------------- the pages' printed layout

def read_layout():
    path = os.path.join(os.path.dirname(__file__), "golden", "asym_w4a8_layout.txt")
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    return vals


def test_layout_matches_the_pages_printed_storage():
    """The oracle's tensors for a Qwen3-VL-4B gate projection (2560 -> 9728)
    have the shapes the pages list, and their bytes per weight round to the
    printed ~0.56 (4-bit codes + one fp8 scale per 16 + per-channel scale +
    codebook)."""
    lay = read_layout()
    N, K = 64, 512
    W, _ = synthetic.weights("qwen3_4b", N, K)
    idx, s_rel, sc, cb = oracle.asym_convert(W, iters=20)
    assert idx.shape == (N, K // int(lay["codes_per_byte"])) and idx.dtype == np.uint8
    assert s_rel.shape == (N, K // int(lay["scale_group"])) and s_rel.itemsize == int(lay["scale_bytes"])
    assert cb.shape == (int(lay["codebook_levels"]),) and sc.shape == (N,)
    assert K % int(lay["convrot_group"]) == 0
    Nq, Kq = 9728, 2560
    per_elem = (Nq * Kq / lay["codes_per_byte"] + Nq * Kq / lay["scale_group"] * lay["scale_bytes"] + 4 * Nq
                + 4 * lay["codebook_levels"]) / (Nq * Kq)
    assert round(per_elem, 2) == lay["bytes_per_elem_printed"]
