"""Seeded synthetic inputs for the ConvRot W4A4 Linear workloads.

This module only draws random numbers; it holds none of the method's
arithmetic.  Both the CPU oracle (through the tests) and the CUDA path (through
the tests, the smoke check and the benchmark) take their inputs from here, so
both sides see the same bf16 bits.

Generator (all vectorised numpy, deterministic across machines):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state_i = seed + (i+1) * 0x9E3779B97F4A7C15,
    then the published 64-bit finaliser.
  * uniform doubles in [0, 1): top 53 bits * 2^-53.
  * standard normal: Box-Muller, z = sqrt(-2 ln(1-u1)) cos(2 pi u2).
  * Student-t(nu=4): Z / sqrt(V / 4), V = -2 ln((1-u1)(1-u2)) (chi-square, 4 dof).
  * Laplace(0, 1): -sgn(u) ln(1 - 2|u|), u = uniform - 1/2.
  * lognormal(0, 1): exp(N(0, 1)).
  * outlier channels: a partial Fisher-Yates shuffle of range(K).
  * bf16: float64 -> float32 (round to nearest even) -> bf16 (round to nearest
    even on the top 16 bits).

Workloads (shapes and distributions of the pages' text-encoder and DiT
linears; the real weights and activations are not available, these stand in):
  * ``small``   : x[32, 512] ~ N(0,1) with 5 outlier channels x20; W[256, 512]
                  ~ N(0, 0.02); bias ~ N(0, 0.01).
  * ``qwen3_4b``: Qwen3-4B text-encoder decoder-layer linears, hidden 2560,
                  M in {76, 1220}; x ~ 0.5 * Student-t(4) with round(1% K)
                  outlier channels x30.
  * ``dit6b``   : 6B-class DiT block at 1024x1024 (4096 image + 128 text
                  tokens), hidden 3840; x ~ Laplace(0,1) * per-channel
                  lognormal(0,1) scales.
  * ``edit20b`` : 20B-class image-edit DiT, 8192 + 512 tokens, hidden 3072;
                  activations as ``qwen3_4b``.
  * ``small_m`` : M in {1, 8, 16, 64, 128} over four (K, N) shapes;
                  activations as ``qwen3_4b``.
Weights are N(0, 0.02) and biases N(0, 0.01) everywhere.
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, n: int) -> np.ndarray:
    """The first ``n`` outputs of SplitMix64 started at ``seed`` (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(1, n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _C1
        z = (z ^ (z >> np.uint64(27))) * _C2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(seed: int, n: int) -> np.ndarray:
    """Uniform doubles in [0, 1)."""
    return (splitmix64(seed, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, n: int) -> np.ndarray:
    u = uniform(seed, 2 * n)
    u1, u2 = u[:n], u[n:]
    return np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)


def student_t4(seed: int, n: int) -> np.ndarray:
    z = normal(seed, n)
    u = uniform(seed ^ 0x5EED5EED5EED5EED, 2 * n)
    v = -2.0 * (np.log1p(-u[:n]) + np.log1p(-u[n:]))
    return z / np.sqrt(v / 4.0)


def laplace(seed: int, n: int) -> np.ndarray:
    u = uniform(seed, n) - 0.5
    return -np.sign(u) * np.log1p(-2.0 * np.abs(u))


def lognormal(seed: int, n: int) -> np.ndarray:
    return np.exp(normal(seed, n))


def choose_channels(seed: int, K: int, count: int) -> np.ndarray:
    """``count`` distinct channels of range(K) by a partial Fisher-Yates shuffle."""
    perm = np.arange(K, dtype=np.int64)
    r = splitmix64(seed, count)
    for i in range(count):
        j = i + int(r[i] % np.uint64(K - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:count])


def to_bf16_bits(a) -> np.ndarray:
    """float -> bf16 bits (uint16), round to nearest even (via float32)."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    with np.errstate(over="ignore"):
        r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    r = np.where(nan, (u >> np.uint32(16)) | np.uint32(0x40), r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def derive_seed(base: int, role: str, *dims: int) -> int:
    """A fixed 64-bit hash of (role, dims) xor the workload's base seed."""
    h = hashlib.sha256(f"{role}:{':'.join(str(d) for d in dims)}".encode()).digest()
    return int.from_bytes(h[:8], "little") ^ (base & 0xFFFFFFFFFFFFFFFF)


# ---- activation / weight recipes ---------------------------------------------

def act_normal_outliers(seed: int, M: int, K: int, n_out: int = 5, factor: float = 20.0) -> np.ndarray:
    x = normal(seed, M * K).reshape(M, K)
    ch = choose_channels(seed ^ 0xC4A77E15, K, n_out)
    x[:, ch] *= factor
    return to_bf16_bits(x)


def act_t4_outliers(seed: int, M: int, K: int, frac: float = 0.01, factor: float = 30.0) -> np.ndarray:
    x = 0.5 * student_t4(seed, M * K).reshape(M, K)
    n_out = int(round(frac * K))
    if n_out:
        ch = choose_channels(seed ^ 0xC4A77E15, K, n_out)
        x[:, ch] *= factor
    return to_bf16_bits(x)


def act_laplace_lognormal(seed: int, M: int, K: int) -> np.ndarray:
    x = laplace(seed, M * K).reshape(M, K)
    scale = lognormal(seed ^ 0x10915CA1E, K)
    return to_bf16_bits(x * scale[None, :])


def weight(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    return to_bf16_bits(std * normal(seed, N * K).reshape(N, K))


def bias(seed: int, N: int, std: float = 0.01) -> np.ndarray:
    return to_bf16_bits(std * normal(seed, N))


@dataclasses.dataclass(frozen=True)
class LinearShape:
    name: str
    M: int
    K: int
    N: int
    # The activation tensor the linear reads: linears of one layer that read
    # the same tensor (q/k/v; gate/up) share it, and one rotate + quantize
    # of it serves all of them.
    input: str = ""
    # Weight/activation format: "w4a4" (ConvRot W4A4), "int8_tensorwise" or
    # "convrot_int8" (the int8 W8A8 formats the pages mix with W4A4), or
    # "asym_w4a8" (4-bit codebook weights, ConvRot INT8 row-scaled activations).
    fmt: str = "w4a4"

    @property
    def source(self) -> str:
        return self.input or self.name


_ACT = {
    "small": act_normal_outliers,
    "qwen3_4b": act_t4_outliers,
    "dit6b": act_laplace_lognormal,
    "edit20b": act_t4_outliers,
    "small_m": act_t4_outliers,
    "edit20b_int8": act_t4_outliers,
    "qwen3_4b_mixed": act_t4_outliers,
    "qwen3_4b_w4a8": act_t4_outliers,
    "small_m_w4a8": act_t4_outliers,
}
_BASE_SEED = {"small": 0, "qwen3_4b": 1, "dit6b": 2, "edit20b": 3, "small_m": 4, "edit20b_int8": 3,
              "qwen3_4b_mixed": 1, "qwen3_4b_w4a8": 1, "small_m_w4a8": 4}


def workload_shapes(workload: str) -> list[LinearShape]:
    """The (name, M, K, N) linears of a workload."""
    if workload == "small":
        return [LinearShape("linear", 32, 512, 256)]
    if workload == "qwen3_4b":
        lin = [("q_proj", 2560, 4096, "attn_in"), ("k_proj", 2560, 1024, "attn_in"), ("v_proj", 2560, 1024, "attn_in"),
               ("o_proj", 2560, 2560, "attn_out"), ("gate_proj", 2560, 9728, "mlp_in"),
               ("up_proj", 2560, 9728, "mlp_in"), ("down_proj", 9728, 2560, "mlp_act")]
        return [LinearShape(f"{n}@{M}", M, K, N, f"{src}@{M}") for M in (76, 1220) for (n, K, N, src) in lin]
    if workload == "dit6b":
        M = 4096 + 128
        lin = [("qkv", 3840, 3 * 3840, "attn_in"), ("out", 3840, 3840, "attn_out"),
               ("ffn_up", 3840, 10240, "mlp_in"), ("ffn_down", 10240, 3840, "mlp_act")]
        return [LinearShape(n, M, K, N, src) for (n, K, N, src) in lin]
    if workload == "edit20b":
        M = 8192 + 512
        lin = [("to_q", 3072, 3072, "attn_in"), ("to_k", 3072, 3072, "attn_in"), ("to_v", 3072, 3072, "attn_in"),
               ("to_out", 3072, 3072, "attn_out"), ("mlp_up", 3072, 12288, "mlp_in"),
               ("mlp_down", 12288, 3072, "mlp_act")]
        return [LinearShape(n, M, K, N, src) for (n, K, N, src) in lin]
    if workload == "edit20b_int8":
        # the value / output projections of the 20B edit DiT in stock int8_tensorwise
        M = 8192 + 512
        return [LinearShape("to_v", M, 3072, 3072, "attn_in", "int8_tensorwise"),
                LinearShape("to_out", M, 3072, 3072, "attn_out", "int8_tensorwise")]
    if workload == "qwen3_4b_mixed":
        # the Qwen3-4B layer with its attention projections in ConvRot INT8
        # (row-scaled) and its MLP in W4A4
        out = []
        for s in workload_shapes("qwen3_4b"):
            fmt = "convrot_int8" if s.name.split("@")[0] in ("q_proj", "k_proj", "v_proj", "o_proj") else "w4a4"
            out.append(dataclasses.replace(s, fmt=fmt))
        return out
    if workload == "qwen3_4b_w4a8":
        # the Qwen3-VL-4B text encoder's decoder Linears in the asymmetric W4A8 format
        return [dataclasses.replace(s, fmt="asym_w4a8") for s in workload_shapes("qwen3_4b")]
    if workload == "small_m_w4a8":
        return [dataclasses.replace(s, fmt="asym_w4a8") for s in workload_shapes("small_m")]
    if workload == "small_m":
        kn = [(2560, 9728), (9728, 2560), (3072, 12288), (12288, 3072)]
        return [LinearShape(f"k{K}_n{N}@{M}", M, K, N) for M in (1, 8, 16, 64, 128) for (K, N) in kn]
    raise KeyError(f"unknown workload {workload!r}")


def activations(workload: str, M: int, K: int, seed_extra: int = 0) -> np.ndarray:
    """bf16 bits [M, K] drawn with the workload's activation recipe."""
    seed = derive_seed(_BASE_SEED[workload] ^ seed_extra, "x", M, K)
    return _ACT[workload](seed, M, K)


def source_seed(source: str) -> int:
    """seed_extra of a named activation tensor (a fixed hash of its name)."""
    h = 0
    for ch in source.encode():
        h = (h * 131 + ch) & 0xFFFFFFFF
    return h


def weights(workload: str, N: int, K: int, seed_extra: int = 0):
    """(W bf16 bits [N, K], bias bf16 bits [N])."""
    base = _BASE_SEED[workload] ^ seed_extra
    return weight(derive_seed(base, "w", N, K), N, K), bias(derive_seed(base, "b", N, K), N)


def asym_format(workload: str, N: int, K: int, seed_extra: int = 0):
    """Random tensors in the asymmetric W4A8 storage layout, for timing and
    for parity at sizes the offline converter is too slow for:
    (idx uint8 [N, K/2] uniform bytes, s_rel uint8 [N, K/16] e4m3 bytes drawn
    uniformly from 0x50..0x70 (the values 8 .. 128), codebook fp32 [16]:
    16 sorted N(0, 0.4) draws clipped to [-1, 1], s_channel fp32 [N]:
    (|N(0, 1)| + 0.5) * 1e-4).  Plain random draws; no quantizer runs here."""
    base = derive_seed(_BASE_SEED[workload] ^ seed_extra, "asym", N, K)
    idx = (splitmix64(base, N * K // 2) & np.uint64(0xFF)).astype(np.uint8).reshape(N, K // 2)
    s_rel = (0x50 + (splitmix64(base ^ 0x5E1, N * K // 16) % np.uint64(0x21))).astype(np.uint8).reshape(N, K // 16)
    codebook = np.sort(np.clip(0.4 * normal(base ^ 0xC0DE, 16), -1.0, 1.0)).astype(np.float32)
    s_channel = ((np.abs(normal(base ^ 0x5C, N)) + 0.5) * 1e-4).astype(np.float32)
    return idx, s_rel, codebook, s_channel
