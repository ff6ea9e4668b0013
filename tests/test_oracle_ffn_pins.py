"""Pins for the oracle's feed-forward pieces: the squared-ReLU gate and the
FFN built from BitLinears (up, gate, squared-ReLU gating, down).

The FFN of BitNet b1.58 uses a squared ReLU and a sub-layer norm
(inferownia.pl, "BitNet b1.58: era 1-bitowych LLM-ów", "Zrób to sam";
kripta.biz 2B4T news: ReLU^2 in the FFN layers), and every linear of it is a
BitLinear (comrad404.com review, "Метод: как устроен BitNet b1.58").  The
tests tie the oracle to closed forms, integer arithmetic, an fp64 dense
reference and torch's bf16 cast, never to the oracle itself.
"""
import numpy as np
import pytest
import torch

from bitlinear_absmean_ternary_b200 import synth


def _bf16(v: float) -> float:
    return float(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).float())


# ----------------------------------------------------------------------------
# the squared-ReLU gate
# ----------------------------------------------------------------------------

def test_relu2_gate_nonpositive_gate_gives_zero_with_sign_of_up(orc):
    g = np.array([-3.0, -0.0, 0.0, -1e-30, -np.inf], dtype=np.float32)
    for uval in (2.0, -2.0, 0.0):
        u = np.full(g.shape, uval, dtype=np.float32)
        out = orc.relu2_gate(u, g)
        assert np.all(out == 0.0)
        # r = +0, so the zero carries the sign of u
        assert np.all(np.signbit(out) == np.signbit(np.float32(uval)))


@pytest.mark.parametrize("j", [-12, -3, 0, 5, 10])
def test_relu2_gate_powers_of_two_are_exact(orc, j):
    i = np.arange(-20, 21)
    u = np.concatenate([2.0 ** i, -(2.0 ** i)]).astype(np.float32)
    g = np.full(u.shape, 2.0 ** j, dtype=np.float32)
    out = orc.relu2_gate(u, g)
    np.testing.assert_array_equal(out, (u.astype(np.float64) * 4.0 ** j).astype(np.float32))


def test_relu2_gate_small_integers_are_exact(orc):
    gg, uu = np.meshgrid(np.arange(-40, 41), np.arange(-100, 101))
    g = gg.astype(np.float32).ravel()
    u = uu.astype(np.float32).ravel()
    out = orc.relu2_gate(u, g)
    expect = np.where(gg > 0, gg * gg * uu, 0).ravel()  # |g^2 u| < 2^24: exact in fp32
    np.testing.assert_array_equal(out, expect.astype(np.float32))


def test_relu2_gate_within_two_roundings_of_fp64(orc):
    rng = np.random.default_rng(5)
    u = rng.standard_normal(20000).astype(np.float32)
    g = (rng.standard_normal(20000) * 3).astype(np.float32)
    out = orc.relu2_gate(u, g).astype(np.float64)
    r = np.maximum(g.astype(np.float64), 0.0)
    exact = r * r * u.astype(np.float64)
    # two correctly rounded fp32 operations: relative error <= 2^-24 (2 + 2^-24)
    assert np.all(np.abs(out - exact) <= np.abs(exact) * 2.0 ** -23 * (1 + 2.0 ** -20))


def test_relu2_gate_applies_the_activation_to_the_gate_only(orc):
    u = np.array([-2.0, 3.0], dtype=np.float32)
    g = np.array([3.0, -2.0], dtype=np.float32)
    np.testing.assert_array_equal(orc.relu2_gate(u, g), np.array([-18.0, 0.0], dtype=np.float32))
    np.testing.assert_array_equal(orc.relu2_gate(g, u), np.array([0.0, -18.0], dtype=np.float32))


# ----------------------------------------------------------------------------
# the FFN composition
# ----------------------------------------------------------------------------

def _pm1(rng, shape):
    return rng.choice([-1, 1], size=shape).astype(np.int64)


def test_ffn_one_hot_tokens_closed_form(orc):
    """W = 2^j T (T in {-1,+1}) gives gamma = 2^j and q = T exactly.  Token m
    is 127 * 2^i_m on channel k_m and zero elsewhere, so x_q = 127 e_k and
    a = 2^i exactly; then u_f = 127 Tu[f,k] 2^(i+ju) and g_f = 127 Tg[f,k]
    2^(i+jg) are exact, h_f = Tu[f,k] [Tg[f,k] > 0] B with B = bf16(127^3
    2^(3i+2jg+ju)), the down input quantises to 127 * sign, and y_d =
    B 2^jd S_d with the integer S_d = sum_f Td[d,f] Tu[f,k] [Tg[f,k] > 0]."""
    rng = np.random.default_rng(23)
    D, F = 128, 192
    ju, jg, jd = -5, -6, -4
    Tu, Tg, Td = _pm1(rng, (F, D)), _pm1(rng, (F, D)), _pm1(rng, (D, F))
    up = orc.pack_weights((Tu * 2.0 ** ju).astype(np.float32), 1e-6)
    gate = orc.pack_weights((Tg * 2.0 ** jg).astype(np.float32), 1e-6)
    down = orc.pack_weights((Td * 2.0 ** jd).astype(np.float32), 1e-6)
    assert (up[1], gate[1], down[1]) == (np.float32(2.0 ** ju), np.float32(2.0 ** jg), np.float32(2.0 ** jd))
    ks, iexp = [3, 77, 127], [0, -2, 3]
    x = np.zeros((3, D), dtype=np.float32)
    for m, (k, i) in enumerate(zip(ks, iexp)):
        x[m, k] = 127.0 * 2.0 ** i
    h_bits, acc, y = orc.ffn(x, up, gate, down)
    h = orc.bf16_to_f32(h_bits)
    for m, (k, i) in enumerate(zip(ks, iexp)):
        B = _bf16(127.0 ** 3 * 2.0 ** (3 * i + 2 * jg + ju))
        assert B == 2048000.0 * 2.0 ** (3 * i + 2 * jg + ju)  # 127^3 = 2048383 rounds down to 8 bits
        sel = Tu[:, k] * (Tg[:, k] > 0)
        np.testing.assert_array_equal(h[m], (sel * B).astype(np.float32))
        S = Td @ sel  # integer
        np.testing.assert_array_equal(acc[m], 127 * S)
        expect = B * 2.0 ** jd * S.astype(np.float64)
        np.testing.assert_allclose(y[m], expect, rtol=2.0 ** -23, atol=0)


def test_ffn_zero_gate_matrix_or_zero_token_gives_zero(orc):
    rng = np.random.default_rng(4)
    D, F = 64, 128
    up = orc.pack_weights(rng.standard_normal((F, D)).astype(np.float32) * 0.02, 1e-5)
    gate0 = orc.pack_weights(np.zeros((F, D), dtype=np.float32), 1e-5)
    down = orc.pack_weights(rng.standard_normal((D, F)).astype(np.float32) * 0.02, 1e-5)
    x = rng.standard_normal((2, D)).astype(np.float32)
    h_bits, acc, y = orc.ffn(x, up, gate0, down)
    assert np.all(orc.bf16_to_f32(h_bits) == 0.0)
    assert np.all(acc == 0) and np.all(y == 0.0)
    gate = orc.pack_weights(rng.standard_normal((F, D)).astype(np.float32) * 0.02, 1e-5)
    h_bits, acc, y = orc.ffn(np.zeros((1, D), dtype=np.float32), up, gate, down)
    assert np.all(orc.bf16_to_f32(h_bits) == 0.0) and np.all(y == 0.0)


def _dense_ffn(x, Wu, Wg, Wd, gain_in, gain_sub, eps, eps_w=1e-5, swap=False, square=True):
    """fp64 dense reference of the FFN on the absmean-ternarised weights
    (numpy only): RMSNorm, the three products, squared-ReLU gating."""
    def tern(W):
        W = W.astype(np.float64)
        gam = np.float32(np.abs(W).mean())
        q = np.clip(np.rint(W / np.float64(np.float32(gam + np.float32(eps_w)))), -1, 1)
        return float(gam) * q

    def norm(v, gain):
        v = v.astype(np.float64)
        if gain is None:
            return v
        return v / np.sqrt((v * v).mean(axis=1, keepdims=True) + eps) * gain.astype(np.float64)

    xn = norm(x, gain_in)
    u = xn @ tern(Wu).T
    g = xn @ tern(Wg).T
    if swap:
        u, g = g, u
    r = np.maximum(g, 0.0)
    h = (r * r if square else r) * u
    return norm(h, gain_sub) @ tern(Wd).T


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_ffn_close_to_dense_fp64_reference(orc):
    """The quantised FFN stays near the fp64 dense FFN on the same ternary
    weights (8-bit activations on both BitLinear inputs, bf16 h), while the
    plausible composition mistakes (activation on the up branch, ReLU without
    the square, a missing norm gain) land far away."""
    D, F, M = 256, 512, 4
    Wu = synth.weights(F, D, 0.02, 0, 11)
    Wg = synth.weights(F, D, 0.02, 0, 12)
    Wd = synth.weights(D, F, 0.02, 0, 13)
    x = synth.activations(M, D, 0, 14, "normal", 0.0, 1.0, "bf16")
    gain_in = synth.gain(D, 0, 15, "bf16")
    gain_sub = synth.gain(F, 0, 16, "bf16")
    eps = 1e-5
    up, gate, down = orc.pack_weights(Wu, 1e-5), orc.pack_weights(Wg, 1e-5), orc.pack_weights(Wd, 1e-5)
    _, _, y = orc.ffn(x, up, gate, down, gain_in, eps, gain_sub, eps)
    ref = _dense_ffn(x, Wu, Wg, Wd, gain_in, gain_sub, eps)
    err = _rel(y, ref)
    assert err < 0.05, err  # about 0.022 on this draw
    # each mistake is 0.36 or more away on the same inputs
    assert _rel(_dense_ffn(x, Wu, Wg, Wd, gain_in, gain_sub, eps, swap=True), ref) > 0.25
    assert _rel(_dense_ffn(x, Wu, Wg, Wd, gain_in, gain_sub, eps, square=False), ref) > 0.25
    assert _rel(_dense_ffn(x, Wu, Wg, Wd, gain_in, None, eps), ref) > 0.25
    assert _rel(_dense_ffn(x, Wu, Wg, Wd, None, gain_sub, eps), ref) > 0.25
