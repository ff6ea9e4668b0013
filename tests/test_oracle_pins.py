"""Pins for the CPU oracle, checked against things other than the oracle itself.

Each test ties one oracle function to a closed form, a library routine
(math.fsum, numpy integer matmul, torch's bf16 cast), an exact invariant,
brute force on tiny inputs, or a hand-worked fixture under tests/golden/.
The definitions come from the BitNet b1.58 pages: absmean ternarisation
(inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów", "Trenowany od zera"),
8-bit activations and the four BitLinear steps (comrad404.com review,
"Метод: как устроен BitNet b1.58") and the add/subtract form of the ternary
product (Habr repost on juhe.plus, "Когда - три лучше двух").
"""
import math
import os

import numpy as np
import pytest

from bitlinear_absmean_ternary_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, vals = line.split(":", 1)
            out[key.strip()] = vals.split()
    return out


def _ulp32(x):
    x = np.abs(np.float32(x))
    return np.float32(np.nextafter(x, np.float32(np.inf)) - x)


# ----------------------------------------------------------------------------
# gamma = mean |W|
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,sigma,seed", [(256, 256, 0.02, 0), (48, 640, 0.01, 3), (7, 64, 1.0, 5),
                                            (300, 2560, 0.02, 1)])
def test_gamma_matches_exact_mean(orc, N, K, sigma, seed):
    W = synth.weights(N, K, sigma, seed, 1)
    g = orc.absmean_gamma(W)
    exact = np.float32(math.fsum(np.abs(W.astype(np.float64)).ravel()) / (N * K))
    assert abs(np.float64(g) - np.float64(exact)) <= _ulp32(exact), (g, exact)


def test_gamma_exact_when_mean_representable(orc):
    rng = np.random.default_rng(7)
    N, K = 4, 64
    mag = rng.choice(np.array([0.5, 1.0], dtype=np.float32), size=(N, K))
    sgn = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=(N, K))
    W = mag * sgn
    expect = np.float32(float(mag.astype(np.float64).sum()) / (N * K))
    assert float(expect) * N * K == float(mag.astype(np.float64).sum())  # the mean is exact
    assert orc.absmean_gamma(W) == expect


def test_gamma_ignores_sign_and_position(orc):
    W = synth.weights(64, 128, 0.02, 2, 1)
    g = orc.absmean_gamma(W)
    g_neg = orc.absmean_gamma(-W)
    assert g == g_neg
    # a permuted or transposed matrix has the same mean up to summation order
    rng = np.random.default_rng(0)
    Wp = np.ascontiguousarray(W[rng.permutation(64)][:, rng.permutation(128)])
    Wt = np.ascontiguousarray(W.T)
    for other in (Wp, Wt):
        assert abs(np.float64(g) - np.float64(orc.absmean_gamma(other))) <= _ulp32(g)


# ----------------------------------------------------------------------------
# ternary codes
# ----------------------------------------------------------------------------

def test_power_of_two_magnitudes_give_sign_codes(orc):
    # W = +-2^j everywhere: gamma = 2^j exactly and q = sign(W).
    rng = np.random.default_rng(11)
    for j in (-7, 0, 3):
        W = (rng.choice([-1.0, 1.0], size=(32, 128)) * 2.0 ** j).astype(np.float32)
        q, g = orc.ternarize(W, 1e-5)
        assert g == np.float32(2.0 ** j)
        np.testing.assert_array_equal(q, np.sign(W).astype(np.int8))


def test_codes_agree_with_fp64_rounding_away_from_ties(orc):
    W = synth.weights(128, 512, 0.02, 4, 1)
    eps = 1e-5
    q, g = orc.ternarize(W, eps)
    assert set(np.unique(q)).issubset({-1, 0, 1})
    d = np.float64(np.float32(g) + np.float32(eps))
    t = W.astype(np.float64) / d
    ref = np.clip(np.round(t), -1, 1).astype(np.int8)
    near_tie = np.abs(np.abs(t) - 0.5) < 1e-6
    assert np.array_equal(q[~near_tie], ref[~near_tie])
    # about 0.5 * gamma is the threshold: a third or so of N(0, s^2) entries are zero
    frac0 = float(np.mean(q == 0))
    assert 0.25 < frac0 < 0.45


def test_weight_ties_round_half_even(orc):
    gold = _golden("round_half_even_ties.txt")
    w = np.array([float(v) for v in gold["weights_w"]], dtype=np.float32)
    q_expect = np.array([int(v) for v in gold["weights_q"]], dtype=np.int8)
    # Pad the row to K = 64 with small fillers so that gamma < 1, then choose
    # eps = 1 - gamma, which makes gamma + eps exactly 1.
    row = np.full(64, 0.125, dtype=np.float32)
    row[: w.size] = w
    W = row[None, :]
    g = orc.absmean_gamma(W)
    assert g < 1
    eps = np.float32(1.0) - g
    assert np.float32(g + eps) == np.float32(1.0)
    q, _ = orc.ternarize(W, float(eps))
    np.testing.assert_array_equal(q[0, : w.size], q_expect)
    assert np.all(q[0, w.size:] == 0)


def test_nonfinite_weight_rejected(orc):
    W = synth.weights(4, 64, 0.02, 0, 1)
    W[2, 5] = np.inf
    with pytest.raises(ValueError):
        orc.ternarize(W, 1e-5)
    W[2, 5] = np.nan
    with pytest.raises(ValueError):
        orc.pack_weights(W, 1e-5)


# ----------------------------------------------------------------------------
# 2-bit storage
# ----------------------------------------------------------------------------

def test_pack_layout_golden(orc):
    gold = _golden("pack_layout_k16.txt")
    q = np.array([[int(v) for v in gold["codes"]]], dtype=np.int8)
    expect = np.array([[int(v) for v in gold["bytes"]]], dtype=np.uint8)
    np.testing.assert_array_equal(orc.pack_codes(q), expect)
    back, bad = orc.unpack_codes(expect, 16)
    assert bad == 0
    np.testing.assert_array_equal(back, q)


def test_pack_word_shift_mask_gives_four_consecutive_weights(orc):
    # (word >> 2j) & 0x03030303 holds codes of weights 4j..4j+3, byte b = weight 4j+b.
    rng = np.random.default_rng(3)
    q = rng.integers(-1, 2, size=(8, 256)).astype(np.int8)
    packed = orc.pack_codes(q)
    words = packed.view("<u4")
    for j in range(4):
        part = ((words >> np.uint32(2 * j)) & np.uint32(0x03030303)).astype("<u4")
        got = part.view(np.uint8).reshape(8, 256 // 16, 4).astype(np.int16) - 1
        expect = q.reshape(8, 256 // 16, 16)[:, :, 4 * j: 4 * j + 4]
        np.testing.assert_array_equal(got, expect)


def test_pack_roundtrip_and_no_illegal_code(orc):
    W = synth.weights(96, 320 // 64 * 64, 0.02, 9, 1)
    packed, g = orc.pack_weights(W, 1e-5)
    q, g2 = orc.ternarize(W, 1e-5)
    assert g == g2
    fields = np.stack([(packed >> (2 * j)) & 3 for j in range(4)])
    assert not np.any(fields == 3)
    back, bad = orc.unpack_codes(packed, W.shape[1])
    assert bad == 0
    np.testing.assert_array_equal(back, q)
    assert packed.nbytes * 4 == W.size


def test_unpack_counts_illegal_code(orc):
    packed = np.full((1, 4), 0x55, dtype=np.uint8)  # all codes 1 (q = 0)
    packed[0, 2] = 0x57  # one field holds code 3
    q, bad = orc.unpack_codes(packed, 16)
    assert bad == 1
    assert np.all(q == 0)


# ----------------------------------------------------------------------------
# activation quantisation
# ----------------------------------------------------------------------------

def test_act_ties_round_half_even(orc):
    gold = _golden("round_half_even_ties.txt")
    xv = np.array([float(v) for v in gold["act_x"]], dtype=np.float32)
    expect = np.array([int(v) for v in gold["act_q"]], dtype=np.int8)
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, : xv.size] = xv
    xq, a, rs = orc.quant_act(x)
    np.testing.assert_array_equal(xq[0, : xv.size], expect)
    assert a[0] == np.float32(1.0)
    assert rs[0] == int(expect.astype(np.int64).sum())


def test_one_hot_token(orc):
    x = np.zeros((3, 128), dtype=np.float32)
    x[0, 17] = 3.25
    x[1, 0] = -0.001
    x[2, 127] = 1e30
    xq, a, rs = orc.quant_act(x)
    for m, (k, v) in enumerate([(17, 3.25), (0, -0.001), (127, 1e30)]):
        expect = np.zeros(128, dtype=np.int8)
        expect[k] = 127 if v > 0 else -127
        np.testing.assert_array_equal(xq[m], expect)
        assert a[m] == np.float32(abs(np.float32(v))) / np.float32(127.0)


def test_zero_token(orc):
    x = np.zeros((2, 64), dtype=np.float32)
    x[1, 3] = 1.0
    xq, a, rs = orc.quant_act(x)
    assert np.all(xq[0] == 0) and a[0] == 0 and rs[0] == 0
    g = synth.gain(64, 0, 3, "bf16")
    xq, a, rs = orc.quant_act(x, g, 1e-5)
    assert np.all(xq[0] == 0) and a[0] == 0 and rs[0] == 0


@pytest.mark.parametrize("k", [-5, -1, 3, 8])
def test_act_quant_invariant_to_power_of_two_scaling(orc, k):
    x = synth.activations(6, 512, 1, 2, "normal", 0.01, 20.0, "bf16")
    xs = (x * np.float32(2.0 ** k)).astype(np.float32)
    xq, a, rs = orc.quant_act(x)
    xq2, a2, rs2 = orc.quant_act(xs)
    np.testing.assert_array_equal(xq, xq2)
    np.testing.assert_array_equal(a2, (a * np.float32(2.0 ** k)).astype(np.float32))
    np.testing.assert_array_equal(rs, rs2)
    # with RMSNorm, scaling x by 2^k and eps by 4^k leaves everything unchanged
    g = synth.gain(512, 1, 3, "bf16")
    eps = 1e-5
    xq, a, _ = orc.quant_act(x, g, eps)
    xq2, a2, _ = orc.quant_act(xs, g, eps * 4.0 ** k)
    np.testing.assert_array_equal(xq, xq2)
    np.testing.assert_array_equal(a, a2)


def test_act_quant_matches_fp64_away_from_ties(orc):
    x = synth.activations(16, 1024, 5, 2, "student_t4", 0.0, 1.0, "bf16")
    xq, a, rs = orc.quant_act(x)
    x64 = x.astype(np.float64)
    amax = np.abs(x64).max(axis=1, keepdims=True)
    t = x64 * (127.0 / amax)
    ref = np.clip(np.round(t), -127, 127)
    near = np.abs(np.abs(t - np.floor(t)) - 0.5) < 1e-4
    assert np.array_equal(xq[~near], ref[~near].astype(np.int8))
    assert np.all(np.abs(xq.astype(np.int64) - ref) <= 1)
    assert np.all(np.abs(xq).max(axis=1) == 127)
    np.testing.assert_array_equal(rs, xq.astype(np.int64).sum(axis=1))
    # dequantised activations are within half a step of the input
    a64 = a.astype(np.float64)[:, None]
    assert np.all(np.abs(xq * a64 - x64) <= 0.5 * a64 * (1 + 1e-6))
    np.testing.assert_allclose(a.astype(np.float64) * 127.0, amax[:, 0], rtol=2 ** -23)


@pytest.mark.parametrize("eps", [1e-5, 0.5])
def test_rmsnorm_matches_fp64(orc, eps):
    K = 2560
    v = synth.activations(1, K, 3, 2, "normal", 0.01, 20.0, "bf16")[0]
    g = synth.gain(K, 3, 3, "bf16")
    h = orc.rmsnorm_row(v, g, eps)
    v64 = v.astype(np.float64)
    ref = v64 / np.sqrt(np.mean(v64 * v64) + np.float64(np.float32(eps))) * g.astype(np.float64)
    np.testing.assert_allclose(h, ref, rtol=2 ** -19, atol=0)
    # doubling the gain doubles the output exactly
    h2 = orc.rmsnorm_row(v, (g * 2).astype(np.float32), eps)
    np.testing.assert_array_equal(h2, h * 2)


def test_rmsnorm_constant_token_closed_form(orc):
    # |v| = c everywhere: mean square c^2, so h = g * sign(v) / sqrt(1 + eps/c^2)
    K = 512
    rng = np.random.default_rng(2)
    v = (rng.choice([-1.0, 1.0], size=K) * 4.0).astype(np.float32)
    g = np.ones(K, dtype=np.float32)
    h = orc.rmsnorm_row(v, g, 16e-6)
    np.testing.assert_allclose(h, np.sign(v) / np.sqrt(1 + 1e-6), rtol=2 ** -21)
    xq, a, _ = orc.quant_act(v[None, :], g, 16e-6)
    np.testing.assert_array_equal(xq[0], (np.sign(v) * 127).astype(np.int8))


# ----------------------------------------------------------------------------
# the ternary product and the dequant epilogue
# ----------------------------------------------------------------------------

def test_dot_brute_force_exhaustive_small_k(orc):
    import ctypes
    import itertools
    L = orc.lib()
    rng = np.random.default_rng(0)
    for K in (1, 2, 5, 7):
        xs = [rng.integers(-127, 128, size=K).astype(np.int8) for _ in range(4)]
        xs.append(np.full(K, 127, dtype=np.int8))
        xs.append(np.full(K, -127, dtype=np.int8))
        for qt in itertools.product((-1, 0, 1), repeat=K):
            q = np.array(qt, dtype=np.int8)
            for x in xs:
                acc = ctypes.c_int32()
                y = ctypes.c_float()
                st = L.oracle_dot(q.ctypes.data, x.ctypes.data, K, 1.0, 1.0,
                                  ctypes.byref(acc), ctypes.byref(y))
                assert st == 0
                assert acc.value == int(np.dot(q.astype(np.int64), x.astype(np.int64)))
                assert y.value == float(acc.value)


@pytest.mark.parametrize("M,N,K", [(4, 256, 256), (3, 40, 192), (9, 7, 64)])
def test_bitlinear_acc_matches_integer_matmul(orc, M, N, K):
    rng = np.random.default_rng(M * N + K)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    a = rng.uniform(0.001, 0.1, size=M).astype(np.float32)
    gamma = np.float32(0.0173)
    acc, y = orc.bitlinear(orc.pack_codes(q), gamma, K, xq, a)
    ref = xq.astype(np.int64) @ q.astype(np.int64).T  # M x N
    np.testing.assert_array_equal(acc, ref)
    exact = ref.astype(np.float64) * np.float64(gamma) * a.astype(np.float64)[:, None]
    # two fp32 roundings: within one fp32 ulp of the exact value
    ulp = np.abs(np.spacing(np.abs(exact).astype(np.float32))).astype(np.float64)
    assert np.all(np.abs(y.astype(np.float64) - exact) <= 2 * ulp)
    # the left-to-right order acc*gamma*max|x|/127 agrees within one ulp too
    amax = (a * np.float32(127.0)).astype(np.float32)
    ltr = ((acc.astype(np.float32) * gamma) * amax[:, None]).astype(np.float32) / np.float32(127.0)
    assert np.all(np.abs(ltr.astype(np.float64) - y.astype(np.float64)) <= 3 * ulp + 1e-45)


def test_sampled_matches_full(orc):
    rng = np.random.default_rng(5)
    M, N, K = 5, 33, 128
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    a = rng.uniform(0.001, 0.1, size=M).astype(np.float32)
    p = orc.pack_codes(q)
    acc, y = orc.bitlinear(p, 0.02, K, xq, a)
    ms = rng.integers(0, M, size=50)
    ns = rng.integers(0, N, size=50)
    acc_s, y_s = orc.bitlinear_sampled(p, 0.02, K, xq, a, ms, ns)
    np.testing.assert_array_equal(acc_s, acc[ms, ns])
    np.testing.assert_array_equal(y_s, y[ms, ns])


def test_zero_weight_row_and_zero_token_give_zero(orc):
    W = synth.weights(16, 128, 0.02, 1, 1)
    W[5] = 0.0
    x = synth.activations(3, 128, 1, 2, "normal", 0.0, 1.0, "f32")
    x[1] = 0.0
    packed, g = orc.pack_weights(W, 1e-5)
    xq, a, _ = orc.quant_act(x)
    acc, y = orc.bitlinear(packed, g, 128, xq, a)
    assert np.all(y[:, 5] == 0) and np.all(acc[:, 5] == 0)
    assert np.all(y[1] == 0)


@pytest.mark.parametrize("i,j", [(0, 0), (3, -6), (-2, 4)])
def test_closed_form_reconstruction_matches_dense_product(orc, i, j):
    # W = 2^j * T with T in {-1, +1}; x = 2^i * Q / 127 with max|Q| = 127.
    # Then q = T, gamma = 2^j, x_q = Q, and y equals the dense product W x.
    rng = np.random.default_rng(17)
    N, K, M = 24, 192, 5
    T = rng.choice([-1, 1], size=(N, K)).astype(np.int8)
    Q = rng.integers(-126, 127, size=(M, K))
    Q[:, 7] = 127
    W = (T.astype(np.float64) * 2.0 ** j).astype(np.float32)
    x = (Q * (2.0 ** i / 127.0)).astype(np.float32)
    packed, g = orc.pack_weights(W, 1e-6)
    assert g == np.float32(2.0 ** j)
    xq, a, _ = orc.quant_act(x)
    np.testing.assert_array_equal(xq, Q.astype(np.int8))
    acc, y = orc.bitlinear(packed, g, K, xq, a)
    dense = x.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(y, dense, rtol=1e-6, atol=1e-6 * np.abs(dense).max())


def test_full_chain_close_to_dense_float_product(orc):
    # The whole BitLinear chain approximates the dense product of the
    # dequantised operands exactly up to fp32 rounding.
    W = synth.weights(64, 256, 0.02, 0, 1)
    x = synth.activations(4, 256, 0, 2, "normal", 0.0, 1.0, "f32")
    packed, g = orc.pack_weights(W, 1e-5)
    q, _ = orc.unpack_codes(packed, 256)
    xq, a, _ = orc.quant_act(x)
    _, y = orc.bitlinear(packed, g, 256, xq, a)
    ref = (xq.astype(np.float64) * a.astype(np.float64)[:, None]) @ (q.astype(np.float64) * np.float64(g)).T
    np.testing.assert_allclose(y, ref, rtol=2 ** -21, atol=1e-9)


def test_bf16_rounding_matches_torch(orc):
    import torch
    rng = np.random.default_rng(1)
    y = rng.standard_normal(4096).astype(np.float32) * 10
    ties = (np.arange(1, 65, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    y = np.concatenate([y, (ties + np.uint32(0x3F800000)).view(np.float32), np.array([0.0, -0.0], np.float32)])
    got = orc.f32_to_bf16(y)
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)
