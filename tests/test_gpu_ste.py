"""GPU parity of the straight-through-estimator backward GEMMs against the
oracle.  Both sides compute the same products from the same bf16 / int8 /
ternary operands; the GPU accumulates in fp32 in the tensor core's order, the
oracle sums exactly in fp64.  The tolerance follows from that: an fp32
accumulation of up to 4096 partial sums (one rounding per 16-term MMA step
of at most 2^-24 relative to the running sum) stays within 2^-12 of the sum
of the terms' magnitudes; a wrong operand, index or transpose is off by the
size of the terms themselves."""
import numpy as np
import pytest

import bitlinear_absmean_ternary_b200 as bl
from bitlinear_absmean_ternary_b200 import synth

pytestmark = pytest.mark.gpu

EPS_W = 1e-5
TOL = 2.0 ** -12


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bl.lib()
    return torch.device("cuda:0")


def _bf16_dev(x32, dev):
    import torch
    bits = synth.f32_to_bf16_bits(x32).view(np.int16)
    return torch.from_numpy(bits.copy()).to(dev).view(torch.bfloat16)


STE_CASES = [(64, 64, 64), (128, 256, 256), (300, 1000, 640), (512, 6912, 2560), (77, 2560, 6912)]


@pytest.mark.parametrize("M,N,K", STE_CASES)
def test_ste_backward_input_parity(dev, orc, M, N, K):
    import torch
    W = synth.weights(N, K, 0.02, M, 1)
    dY = synth.activations(M, N, M, 5, "normal", 0.01, 10.0, "bf16")
    P, G = bl.bitnet_pack_weights(torch.from_numpy(W).to(dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    ref = orc.ste_backward_input(dY, p_ref, g_ref, K)
    q, _ = orc.unpack_codes(p_ref, K)
    mag = np.float64(g_ref) * (np.abs(dY).astype(np.float64) @ np.abs(q).astype(np.float64))
    dYd = _bf16_dev(dY, dev)
    dX = bl.bitnet_ste_backward_input(P, G, dYd, out_dtype=torch.float32)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
    got = dX.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= TOL * mag + 1e-30), float((err / (mag + 1e-30)).max())
    # bf16 output: the RNE of the same fp32 value
    dXb = bl.bitnet_ste_backward_input(P, G, dYd, out_dtype=torch.bfloat16)
    assert torch.equal(dXb, dX.to(torch.bfloat16))


@pytest.mark.parametrize("M,N,K", STE_CASES)
def test_ste_backward_weight_parity(dev, orc, M, N, K):
    import torch
    x = synth.activations(M, K, M, 6, "normal", 0.01, 20.0, "bf16")
    dY = synth.activations(M, N, M, 7, "normal", 0.0, 1.0, "bf16")
    xq_r, a_r, _ = orc.quant_act(x)
    xq = torch.from_numpy(xq_r).to(dev)
    a = torch.from_numpy(a_r).to(dev)
    ref = orc.ste_backward_weight(dY, xq_r, a_r)
    dys = orc.bf16_to_f32(orc.ste_scale_grad(dY, a_r)).astype(np.float64)
    mag = np.abs(dys).T @ np.abs(xq_r).astype(np.float64)
    dYd = _bf16_dev(dY, dev)
    dW = bl.bitnet_ste_backward_weight(dYd, xq, a, out_dtype=torch.float32)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
    got = dW.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= TOL * mag + 1e-30), float((err / (mag + 1e-30)).max())
    dWb = bl.bitnet_ste_backward_weight(dYd, xq, a, out_dtype=torch.bfloat16)
    assert torch.equal(dWb, dW.to(torch.bfloat16))


def test_ste_one_hot_gradient_is_exact(dev, orc):
    """A one-hot dY makes every sum a single term: dX row = gamma * q row and
    dW row = bf16(a) * x_q row, exactly."""
    import torch
    M, N, K = 96, 256, 384
    W = synth.weights(N, K, 0.02, 0, 8)
    P, G = bl.bitnet_pack_weights(torch.from_numpy(W).to(dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    dY = np.zeros((M, N), np.float32)
    dY[41, 200] = 1.0
    dX = bl.bitnet_ste_backward_input(P, G, _bf16_dev(dY, dev)).cpu().numpy()
    np.testing.assert_array_equal(dX, orc.ste_backward_input(dY, p_ref, g_ref, K))
    x = synth.activations(M, K, 0, 9, "normal", 0.0, 1.0, "bf16")
    xq_r, a_r, _ = orc.quant_act(x)
    dW = bl.bitnet_ste_backward_weight(_bf16_dev(dY, dev), torch.from_numpy(xq_r).to(dev),
                                       torch.from_numpy(a_r).to(dev)).cpu().numpy()
    np.testing.assert_array_equal(dW, orc.ste_backward_weight(dY, xq_r, a_r))
