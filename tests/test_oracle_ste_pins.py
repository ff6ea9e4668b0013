"""Pins for the oracle's straight-through-estimator backward of the BitLinear
(Habr repost on juhe.plus: latent precise weights with the coarse ones used
in the computation, section "А откуда взялась сама идея?"; the gradient
passed through the rounding as if it were absent, section "Когда - три лучше
двух").  Tied to PyTorch autograd on an fp64 forward written with the STE
trick (an independent route to the same gradients), and to closed forms."""
import numpy as np
import pytest
import torch

from bitlinear_absmean_ternary_b200 import synth


def _autograd(W, x, x_deq, dY, eps_w=1e-5):
    """fp64 STE forward y = x_hat W_hat^T with x_hat = x + (x_deq - x).detach()
    and W_hat = W + (gamma T(W) - W).detach(); returns autograd's dX, dW for dY.
    x_deq is the forward's dequantised activation a[m] * x_q[m] (the absmax
    quantiser itself is pinned elsewhere); the weight quantiser is recomputed
    here in fp64."""
    W = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    x = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    with torch.no_grad():
        gam = float(np.float32(np.abs(W.detach().numpy().astype(np.float64)).mean()))
        d = float(np.float32(np.float32(gam) + np.float32(eps_w)))
        w_t = gam * torch.clamp(torch.round(W / d), -1, 1)
    W_hat = W + (w_t - W).detach()
    x_hat = x + (torch.tensor(x_deq, dtype=torch.float64) - x).detach()
    y = x_hat @ W_hat.T
    y.backward(torch.tensor(dY, dtype=torch.float64))
    return x.grad.numpy(), W.grad.numpy()


@pytest.mark.parametrize("M,N,K", [(5, 64, 128), (16, 96, 256), (3, 200, 64)])
def test_ste_backward_matches_autograd(orc, M, N, K):
    W = synth.weights(N, K, 0.02, M, 1)
    x = synth.activations(M, K, M, 2, "normal", 0.0, 1.0, "f32")
    dY = synth.activations(M, N, M, 3, "normal", 0.0, 1.0, "bf16")
    packed, g = orc.pack_weights(W, 1e-5)
    xq, a, _ = orc.quant_act(x)
    gx, gw = _autograd(W, x, xq.astype(np.float64) * a.astype(np.float64)[:, None], dY)
    dX = orc.ste_backward_input(dY, packed, g, K)
    # dX: one rounding to fp32 of the exact sum
    np.testing.assert_allclose(dX, gx, rtol=2 ** -23, atol=1e-30)
    # dW without operand rounding equals autograd's exactly up to fp64 rounding
    dWe = orc.ste_backward_weight_exact(dY, xq, a)
    np.testing.assert_allclose(dWe, gw, rtol=1e-12, atol=1e-12 * np.abs(gw).max())
    # with the bf16 rounding of dY * a: within 2^-8 of each term's size
    dW = orc.ste_backward_weight(dY, xq, a)
    bound = 2.0 ** -8 * (np.abs(dY).T.astype(np.float64) @ np.abs(xq * a[:, None]).astype(np.float64))
    assert np.all(np.abs(dW - gw) <= bound + 1e-30)


def test_ste_one_hot_gradient_closed_form(orc):
    N, K, M = 48, 128, 4
    rng = np.random.default_rng(9)
    T = rng.choice([-1, 0, 1], size=(N, K)).astype(np.int8)
    packed = orc.pack_codes(T)
    gamma = np.float32(0.0371)
    dY = np.zeros((M, N), np.float32)
    dY[2, 17] = 1.0
    dX = orc.ste_backward_input(dY, packed, gamma, K)
    expect = np.zeros((M, K), np.float32)
    expect[2] = gamma * T[17].astype(np.float32)
    np.testing.assert_array_equal(dX, expect)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    a = np.array([0.5, 0.25, 2.0 ** -7, 1.0], np.float32)  # powers of two: dY * a exact in bf16
    dW = orc.ste_backward_weight(dY, xq, a)
    expectw = np.zeros((N, K), np.float32)
    expectw[17] = np.float32(2.0 ** -7) * xq[2].astype(np.float32)
    np.testing.assert_array_equal(dW, expectw)


def test_ste_scale_grad_rounds_to_bf16(orc):
    dY = np.array([[1.0, -3.0, 0.1]], np.float32)
    a = np.array([1.0 / 3.0], np.float32)
    bits = orc.ste_scale_grad(dY, a)
    expect = torch.tensor(dY * a[:, None]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, expect)
