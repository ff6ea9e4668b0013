"""Seeded synthetic inputs for BitLinear workloads.

This module only draws random numbers and rounds them to the storage type of
the inputs (fp32 or bf16).  It holds none of the BitLinear arithmetic
(no absmean, no absmax, no quantisation, no product), so both the CPU oracle
and the CUDA path can take their inputs from it without sharing any of the
method's code.

Recipe (one stream per tensor):
  * splitmix64 over the counter i = 0, 1, 2, ... of a per-tensor base state
    derived from (seed, tensor_id); uniform u = ((r >> 11) + 0.5) * 2^-53,
    which lies strictly inside (0, 1).
  * Normal: Box-Muller in float64, z = sqrt(-2 ln u1) * cos(2 pi u2), with
    u1 / u2 taken from the even / odd counters; then times sigma, rounded to
    fp32, then (for bf16 tensors) rounded to bf16 half-to-even.
  * Student-t with nu = 4: Z / sqrt(V / 4) with V = -2 ln(u3 * u4), which is
    chi-squared with 4 degrees of freedom.
  * Outlier channels: round(p * K) channel indices picked by a seeded
    Fisher-Yates partial shuffle; the same channels for every token; the
    channel value is multiplied by the outlier factor in fp32 before the bf16
    rounding.
  * RMSNorm gain: uniform in [0.5, 1.5), rounded to the activation dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _base_state(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([(seed * 0x100000001B3 + tensor_id * 0x9E3779B1 + 0x632BE59BD9B4E019)
                      & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
        return _mix64(s)[0]


def uniform(seed: int, tensor_id: int, n: int, start: int = 0) -> np.ndarray:
    """n uniforms in (0, 1) from counters start .. start+n-1 of the stream."""
    base = _base_state(seed, tensor_id)
    out = np.empty(n, dtype=np.float64)
    with np.errstate(over="ignore"):
        for c0 in range(0, n, _CHUNK):
            c1 = min(n, c0 + _CHUNK)
            ctr = np.arange(start + c0 + 1, start + c1 + 1, dtype=np.uint64)
            r = _mix64(base + ctr * _GOLDEN)
            out[c0:c1] = ((r >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    return out


def normal(seed: int, tensor_id: int, n: int) -> np.ndarray:
    """n standard normals (float64) by Box-Muller on consecutive uniform pairs."""
    out = np.empty(n, dtype=np.float64)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        u = uniform(seed, tensor_id, 2 * (c1 - c0), start=2 * c0)
        out[c0:c1] = np.sqrt(-2.0 * np.log(u[0::2])) * np.cos(2.0 * math.pi * u[1::2])
    return out


def student_t4(seed: int, tensor_id: int, n: int) -> np.ndarray:
    """n Student-t (nu = 4) draws, float64: Z / sqrt(V / 4), V ~ chi2(4)."""
    z = normal(seed, tensor_id, n)
    out = np.empty(n, dtype=np.float64)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        u = uniform(seed, tensor_id + 0x7777, 2 * (c1 - c0), start=2 * c0)
        v = -2.0 * np.log(u[0::2] * u[1::2])
        out[c0:c1] = z[c0:c1] / np.sqrt(v / 4.0)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (half to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x32: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 array rounded to the storage dtype ('f32' or 'bf16'), returned as fp32 values."""
    if dtype == "f32":
        return np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(x32))
    raise ValueError(dtype)


def outlier_channels(seed: int, tensor_id: int, K: int, frac: float) -> np.ndarray:
    """round(frac * K) distinct channel indices from a seeded Fisher-Yates partial shuffle."""
    c = int(round(frac * K))
    perm = np.arange(K, dtype=np.int64)
    u = uniform(seed, tensor_id + 0x5151, c)
    for i in range(c):
        j = i + int(u[i] * (K - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:c])


def weights(N: int, K: int, sigma: float, seed: int, tensor_id: int) -> np.ndarray:
    """Latent fp32 weight matrix N x K (row n = output feature n), entries N(0, sigma^2)."""
    w = (normal(seed, tensor_id, N * K) * sigma).astype(np.float32)
    return w.reshape(N, K)


def activations(M: int, K: int, seed: int, tensor_id: int, dist: str = "normal",
                outlier_frac: float = 0.0, outlier_scale: float = 1.0,
                dtype: str = "bf16") -> np.ndarray:
    """Activation matrix M x K as fp32 values already rounded to `dtype`."""
    if dist == "normal":
        v = normal(seed, tensor_id, M * K)
    elif dist == "student_t4":
        v = student_t4(seed, tensor_id, M * K)
    else:
        raise ValueError(dist)
    x = v.astype(np.float32).reshape(M, K)
    if outlier_frac > 0.0:
        ch = outlier_channels(seed, tensor_id, K, outlier_frac)
        x[:, ch] = x[:, ch] * np.float32(outlier_scale)
    return round_to(x, dtype)


def gain(K: int, seed: int, tensor_id: int, dtype: str = "bf16") -> np.ndarray:
    """RMSNorm gain vector, uniform in [0.5, 1.5), rounded to `dtype`."""
    g = (uniform(seed, tensor_id, K) + 0.5).astype(np.float32)
    return round_to(g, dtype)


# ---------------------------------------------------------------------------
# Named workloads.  Each linear is (M, K, N) with its input recipe; shapes and
# distributions follow the BitNet b1.58 block sizes the benchmarks use.
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    M: int
    K: int
    N: int
    w_sigma: float
    x_dist: str = "normal"
    x_dtype: str = "bf16"
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    norm: bool = False
    y_dtype: str = "bf16"
    w_id: int = 1
    x_id: int = 2
    g_id: int = 3

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K

    def make_w(self, seed: int = 0) -> np.ndarray:
        return weights(self.N, self.K, self.w_sigma, seed, self.w_id)

    def make_x(self, seed: int = 0) -> np.ndarray:
        return activations(self.M, self.K, seed, self.x_id, self.x_dist,
                           self.outlier_frac, self.outlier_scale, self.x_dtype)

    def make_gain(self, seed: int = 0) -> Optional[np.ndarray]:
        return gain(self.K, seed, self.g_id, self.x_dtype) if self.norm else None


def _block25(M: int) -> list:
    # 2.5B-class block: hidden 2560, Q|K|V 2560 -> 2560+640+640, O 2560 -> 2560,
    # up|gate 2560 -> 2x6912, down 6912 -> 2560; every input RMS-normalised.
    return [
        Linear("qkv", M, 2560, 3840, 0.02, norm=True, w_id=11, x_id=12, g_id=13),
        Linear("o", M, 2560, 2560, 0.02, norm=True, w_id=21, x_id=22, g_id=23),
        Linear("upgate", M, 2560, 13824, 0.02, norm=True, w_id=31, x_id=32, g_id=33),
        Linear("down", M, 6912, 2560, 0.02, norm=True, w_id=41, x_id=42, g_id=43),
    ]


WORKLOADS = {
    # single BitLinear, fp32 everywhere, the small correctness case
    "bitlinear_m4_k256_n256": [
        Linear("l", 4, 256, 256, 0.02, x_dtype="f32", y_dtype="f32")],
    # decode GEMV, 1% outlier channels x20
    "decode_m1_2p5b_ffn": [
        Linear("up", 1, 2560, 6912, 0.02, outlier_frac=0.01, outlier_scale=20.0, w_id=51, x_id=52),
        Linear("down", 1, 6912, 2560, 0.02, outlier_frac=0.01, outlier_scale=20.0, w_id=61, x_id=62)],
    # batched decode M=64 through one 2.5B-class block
    "decode_m64_2p5b_block": _block25(64),
    # prefill GEMM, Student-t activations
    "prefill_m4096_2p5b_ffn": [
        Linear("up", 4096, 2560, 6912, 0.02, x_dist="student_t4", w_id=71, x_id=72),
        Linear("down", 4096, 6912, 2560, 0.02, x_dist="student_t4", w_id=81, x_id=82)],
    # 27B-class FFN shapes at M = 1, 16, 2048; 0.5% outlier channels x30
    **{f"ffn27b_m{m}": [
        Linear("up", m, 5376, 21504, 0.01, outlier_frac=0.005, outlier_scale=30.0, w_id=91, x_id=92),
        Linear("down", m, 21504, 5376, 0.01, outlier_frac=0.005, outlier_scale=30.0, w_id=101, x_id=102)]
       for m in (1, 16, 2048)},
}


@dataclasses.dataclass(frozen=True)
class FfnBlock:
    """Feed-forward block of three BitLinears: up and gate (D -> F), squared-ReLU
    gating, down (F -> D), with an RMSNorm gain on each BitLinear input."""
    name: str
    M: int
    D: int
    F: int
    w_sigma: float
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    ids: tuple = (1, 2, 3, 4, 5, 6)  # up, gate, down, x, gain_in, gain_sub

    def make_w(self, which: str, seed: int = 0) -> np.ndarray:
        i = {"up": 0, "gate": 1, "down": 2}[which]
        N, K = (self.D, self.F) if which == "down" else (self.F, self.D)
        return weights(N, K, self.w_sigma, seed, self.ids[i])

    def make_x(self, seed: int = 0) -> np.ndarray:
        return activations(self.M, self.D, seed, self.ids[3], "normal", self.outlier_frac, self.outlier_scale, "bf16")

    def make_gains(self, seed: int = 0):
        return gain(self.D, seed, self.ids[4], "bf16"), gain(self.F, seed, self.ids[5], "bf16")

    @property
    def weight_bytes(self) -> int:
        return 3 * self.F * self.D // 4


FFN_BLOCKS = {
    # the 2.5B-class FFN (up/gate 2560 -> 6912, down 6912 -> 2560) at decode, 1% outlier channels x20
    "ffn_block_m1_2p5b": FfnBlock("ffn_block_m1_2p5b", 1, 2560, 6912, 0.02, 0.01, 20.0, (51, 55, 61, 52, 53, 63)),
    # the 27B-class FFN (up/gate 5376 -> 21504, down 21504 -> 5376), 0.5% outlier channels x30
    "ffn_block_m1_27b": FfnBlock("ffn_block_m1_27b", 1, 5376, 21504, 0.01, 0.005, 30.0, (91, 95, 101, 92, 93, 103)),
}
