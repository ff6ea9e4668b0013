"""CPU oracle for the BitLinear forward -- TEST INFRASTRUCTURE ONLY.

Loads the plain single-threaded C++ oracle (bitnet_oracle.cpp, built into
liboracle.so beside this file) and wraps it for numpy arrays.  Only the
tests, the smoke check and the CPU-baseline leg of the benchmark use it; the
CUDA library never imports or links it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitnet_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_CXXFLAGS = ["-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with g++ (IEEE fp32, no contraction) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *_CXXFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        L.oracle_absmean_gamma.argtypes = [P, I64, I64]
        L.oracle_absmean_gamma.restype = F
        L.oracle_ternarize.argtypes = [P, I64, I64, F, P, P]
        L.oracle_ternarize.restype = ctypes.c_int
        L.oracle_pack_codes.argtypes = [P, I64, I64, P]
        L.oracle_pack_codes.restype = None
        L.oracle_unpack_codes.argtypes = [P, I64, I64, P]
        L.oracle_unpack_codes.restype = I64
        L.oracle_pack_weights.argtypes = [P, I64, I64, F, P, P]
        L.oracle_pack_weights.restype = ctypes.c_int
        L.oracle_rmsnorm_row.argtypes = [P, P, I64, F, P]
        L.oracle_rmsnorm_row.restype = None
        L.oracle_quant_act.argtypes = [P, I64, I64, P, F, P, P, P]
        L.oracle_quant_act.restype = None
        L.oracle_dot.argtypes = [P, P, I64, F, F, P, P]
        L.oracle_dot.restype = ctypes.c_int
        L.oracle_bitlinear.argtypes = [P, F, I64, I64, P, P, I64, P, P]
        L.oracle_bitlinear.restype = ctypes.c_int
        L.oracle_bitlinear_sampled.argtypes = [P, F, I64, I64, P, P, I64, P, P, I64, P, P]
        L.oracle_bitlinear_sampled.restype = ctypes.c_int
        L.oracle_f32_to_bf16.argtypes = [P, I64, P]
        L.oracle_f32_to_bf16.restype = None
        L.oracle_relu2_gate.argtypes = [P, P, I64, P]
        L.oracle_relu2_gate.restype = None
        L.oracle_b3_padded_k.argtypes = [I64]
        L.oracle_b3_padded_k.restype = I64
        L.oracle_pack_codes_b3.argtypes = [P, I64, I64, P]
        L.oracle_pack_codes_b3.restype = None
        L.oracle_unpack_codes_b3.argtypes = [P, I64, I64, P]
        L.oracle_unpack_codes_b3.restype = I64
        L.oracle_bitlinear_b3.argtypes = [P, F, I64, I64, P, P, I64, P, P]
        L.oracle_bitlinear_b3.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def absmean_gamma(W: np.ndarray) -> np.float32:
    W = _f32(W)
    N, K = W.shape
    return np.float32(lib().oracle_absmean_gamma(_p(W), N, K))


def ternarize(W: np.ndarray, eps: float):
    """Returns (q int8 N x K, gamma float32).  Raises on non-finite W."""
    W = _f32(W)
    N, K = W.shape
    q = np.empty((N, K), dtype=np.int8)
    g = np.zeros(1, dtype=np.float32)
    st = lib().oracle_ternarize(_p(W), N, K, eps, _p(q), _p(g))
    if st != 0:
        raise ValueError(f"oracle_ternarize status {st}")
    return q, g[0]


def pack_codes(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.empty((N, K // 4), dtype=np.uint8)
    lib().oracle_pack_codes(_p(q), N, K, _p(out))
    return out


def unpack_codes(packed: np.ndarray, K: int):
    """Returns (q int8 N x K, number of illegal code-3 fields)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    q = np.empty((N, K), dtype=np.int8)
    bad = lib().oracle_unpack_codes(_p(packed), N, K, _p(q))
    return q, int(bad)


def pack_weights(W: np.ndarray, eps: float):
    """Returns (packed uint8 N x K/4, gamma float32), or raises on non-finite W."""
    W = _f32(W)
    N, K = W.shape
    out = np.empty((N, K // 4), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    st = lib().oracle_pack_weights(_p(W), N, K, eps, _p(out), _p(g))
    if st != 0:
        raise ValueError(f"oracle_pack_weights status {st}")
    return out, g[0]


def rmsnorm_row(v: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    v = _f32(v)
    g = _f32(g)
    h = np.empty_like(v)
    lib().oracle_rmsnorm_row(_p(v), _p(g), v.shape[0], eps, _p(h))
    return h


def quant_act(x: np.ndarray, gain=None, rms_eps: float = 1e-5):
    """x: M x K fp32 values.  Returns (x_q int8 M x K, a float32 M, rowsum int32 M)."""
    x = _f32(x)
    M, K = x.shape
    xq = np.empty((M, K), dtype=np.int8)
    a = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.int32)
    gp = None
    if gain is not None:
        gain = _f32(gain)
        gp = _p(gain)
    lib().oracle_quant_act(_p(x), M, K, gp, rms_eps, _p(xq), _p(a), _p(rs))
    return xq, a, rs


def bitlinear(packed: np.ndarray, gamma, K: int, xq: np.ndarray, a: np.ndarray):
    """Returns (acc int32 M x N, y float32 M x N)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    a = _f32(a)
    N = packed.shape[0]
    M = xq.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    y = np.empty((M, N), dtype=np.float32)
    st = lib().oracle_bitlinear(_p(packed), np.float32(gamma), N, K, _p(xq), _p(a), M, _p(acc), _p(y))
    if st != 0:
        raise ValueError(f"oracle_bitlinear status {st}")
    return acc, y


def bitlinear_sampled(packed: np.ndarray, gamma, K: int, xq: np.ndarray, a: np.ndarray,
                      ms: np.ndarray, ns: np.ndarray):
    """The product at positions (ms[i], ns[i]) only.  Returns (acc int32, y float32)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    a = _f32(a)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    N = packed.shape[0]
    M = xq.shape[0]
    acc = np.empty(ms.shape[0], dtype=np.int32)
    y = np.empty(ms.shape[0], dtype=np.float32)
    st = lib().oracle_bitlinear_sampled(_p(packed), np.float32(gamma), N, K, _p(xq), _p(a), M,
                                        _p(ms), _p(ns), ms.shape[0], _p(acc), _p(y))
    if st != 0:
        raise ValueError(f"oracle_bitlinear_sampled status {st}")
    return acc, y


def f32_to_bf16(y: np.ndarray) -> np.ndarray:
    y = _f32(y)
    out = np.empty(y.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16(_p(y), y.size, _p(out))
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the fp32 values they stand for (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def relu2_gate(u: np.ndarray, g: np.ndarray) -> np.ndarray:
    """RN32(RN32(r*r)*u) with r = max(g, +0): the squared-ReLU gate of the FFN."""
    u = _f32(u)
    g = _f32(g)
    assert u.shape == g.shape
    out = np.empty_like(u)
    lib().oracle_relu2_gate(_p(u), _p(g), u.size, _p(out))
    return out


def bitlinear_forward(x: np.ndarray, packed: np.ndarray, gamma, gain=None, rms_eps: float = 1e-5):
    """One BitLinear on fp32 token rows x (M x K): optional RMSNorm, absmax int8
    quantisation, exact ternary product, dequant.  Returns (acc int32, y fp32)."""
    x = _f32(x)
    xq, a, _ = quant_act(x, gain, rms_eps)
    return bitlinear(packed, gamma, x.shape[1], xq, a)


def ffn(x: np.ndarray, up, gate, down, gain_in=None, eps_in: float = 1e-5, gain_sub=None, eps_sub: float = 1e-5):
    """Feed-forward block of BitNet b1.58 built from BitLinears.

    up, gate: (packed F x D/4, gamma); down: (packed D x F/4, gamma).  x: M x D
    fp32 values (bf16 values in the block).  Steps: u = BitLinear_up(x) and
    g = BitLinear_gate(x), both normalising x with gain_in; h = bf16 of the
    squared-ReLU gate relu2_gate(u, g) (the down projection's input, stored
    as bf16 like every activation of the block); y = BitLinear_down(h),
    normalising h with gain_sub (the sub-layer norm).
    Returns (h bf16 bits M x F, acc_down int32 M x D, y fp32 M x D)."""
    _, u = bitlinear_forward(x, up[0], up[1], gain_in, eps_in)
    _, g = bitlinear_forward(x, gate[0], gate[1], gain_in, eps_in)
    h_bits = f32_to_bf16(relu2_gate(u, g))
    acc, y = bitlinear_forward(bf16_to_f32(h_bits), down[0], down[1], gain_sub, eps_sub)
    return h_bits, acc, y


def b3_padded_k(K: int) -> int:
    return int(lib().oracle_b3_padded_k(K))


def pack_codes_b3(q: np.ndarray) -> np.ndarray:
    """Base-3 packing of ternary codes (N x K int8) -> N x b3_padded_k(K)/5 bytes."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.empty((N, b3_padded_k(K) // 5), dtype=np.uint8)
    lib().oracle_pack_codes_b3(_p(q), N, K, _p(out))
    return out


def unpack_codes_b3(packed: np.ndarray, K: int):
    """Returns (q int8 N x K, number of invalid bytes or non-zero padded codes)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    q = np.empty((N, K), dtype=np.int8)
    bad = lib().oracle_unpack_codes_b3(_p(packed), N, K, _p(q))
    return q, int(bad)


def pack_weights_b3(W: np.ndarray, eps: float):
    """Absmean ternarisation + base-3 packing.  Returns (packed, gamma)."""
    q, g = ternarize(W, eps)
    return pack_codes_b3(q), g


def bitlinear_b3(packed: np.ndarray, gamma, K: int, xq: np.ndarray, a: np.ndarray):
    """The BitLinear product against base-3 packed weights.  Returns (acc int32, y fp32)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    a = _f32(a)
    N = packed.shape[0]
    M = xq.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    y = np.empty((M, N), dtype=np.float32)
    st = lib().oracle_bitlinear_b3(_p(packed), np.float32(gamma), N, K, _p(xq), _p(a), M, _p(acc), _p(y))
    if st != 0:
        raise ValueError(f"oracle_bitlinear_b3 status {st}")
    return acc, y


# ----------------------------------------------------------------------------
# Straight-through estimator (STE) backward of the BitLinear.
#
# Training keeps full-precision latent weights and lets the forward use the
# rounded ones (Habr repost on juhe.plus, section "А откуда взялась сама
# идея?": the precise values accumulate the small updates, the computation
# uses the coarse ones); the rounding step has a zero derivative almost
# everywhere, so the backward pass treats it as absent and passes the
# gradient straight through (same page, section "Когда - три лучше двух":
# forward with the real rounding, backward as if it were not there).  The forward used W_hat = gamma * q and x_hat[m] = a[m] *
# x_q[m] (y = x_hat W_hat^T), so with the quantisers treated as identities:
#   dX[m, k] = sum_n dY[m, n] * gamma * q[n, k]     (gradient at the quantiser input)
#   dW[n, k] = sum_m dY[m, n] * a[m] * x_q[m, k]    (gradient reaching the latent W)
# Reading of the precision: dY is bf16 (bf16 training); dX = RN32(gamma * S)
# with S the exact sum; the weight-gradient product takes bf16 operands, so
# its left operand is dYs = bf16_RNE(RN32(dY * a[m])) and dW = RN32(exact sum
# of dYs * x_q).  The sums use numpy's fp64 matmul as a primitive: every
# product and partial sum here is exact in fp64 for |dY| below 2^60.


def ste_backward_input(dY: np.ndarray, packed: np.ndarray, gamma, K: int) -> np.ndarray:
    """dX = RN32(gamma * (dY @ q)), dY: M x N fp32 values (bf16 values in use)."""
    q, bad = unpack_codes(packed, K)
    if bad:
        raise ValueError("packed weights hold an illegal code")
    S = np.asarray(dY, np.float64) @ q.astype(np.float64)
    return (np.float32(gamma).astype(np.float64) * S).astype(np.float32)


def ste_scale_grad(dY: np.ndarray, a: np.ndarray) -> np.ndarray:
    """dYs = bf16_RNE(RN32(dY[m, n] * a[m])) as bf16 bit patterns."""
    dY = _f32(dY)
    a = _f32(a)
    return f32_to_bf16((dY * a[:, None]).astype(np.float32))


def ste_backward_weight(dY: np.ndarray, xq: np.ndarray, a: np.ndarray) -> np.ndarray:
    """dW = RN32(sum_m dYs[m, n] * x_q[m, k]) with dYs = ste_scale_grad(dY, a); N x K fp32."""
    dYs = bf16_to_f32(ste_scale_grad(dY, a)).astype(np.float64)
    return (dYs.T @ np.asarray(xq, np.float64)).astype(np.float32)


def ste_backward_weight_exact(dY: np.ndarray, xq: np.ndarray, a: np.ndarray) -> np.ndarray:
    """The same sum without the bf16 rounding of the left operand, in fp64."""
    x_hat = np.asarray(xq, np.float64) * np.asarray(a, np.float64)[:, None]
    return np.asarray(dY, np.float64).T @ x_hat
