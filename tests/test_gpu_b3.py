"""GPU parity of the base-3 storage (five ternary codes per byte): the pack
kernel's bytes against the oracle's, and the fused decode BitLinear on base-3
rows against the oracle's product and against the 2-bit fused kernel on the
same matrix (identical results: the codes, activations and arithmetic are the
same, only the storage differs)."""
import numpy as np
import pytest

import bitlinear_absmean_ternary_b200 as bl
from bitlinear_absmean_ternary_b200 import synth

pytestmark = pytest.mark.gpu

EPS_W = 1e-5
EPS_RMS = 1e-5


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bl.lib()
    return torch.device("cuda:0")


def _x_dev(x32, dtype, dev):
    import torch
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(x32).view(np.int16)
        return torch.from_numpy(bits.copy()).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(dev)


@pytest.mark.parametrize("N,K", [(256, 256), (6912, 2560), (2560, 6912), (7, 64), (129, 192), (5376, 21504)])
def test_pack_b3_parity(dev, orc, N, K):
    import torch
    W = synth.weights(N, K, 0.02, 3, 1)
    P, G = bl.bitnet_pack_weights_b3(torch.from_numpy(W).to(dev), EPS_W)
    p_ref, g_ref = orc.pack_weights_b3(W, EPS_W)
    assert G.item() == g_ref
    np.testing.assert_array_equal(P.cpu().numpy(), p_ref)


B3_CASES = [
    # M, N, K, x dtype, norm, y dtype
    (1, 6912, 2560, "bf16", True, "bf16"),
    (1, 2560, 6912, "bf16", False, "f32"),
    (1, 5376, 21504, "bf16", False, "bf16"),   # 3 chunks of 90 groups... per row, padded K = 21520
    (4, 256, 256, "f32", False, "f32"),
    (8, 300, 2688, "bf16", True, "i32"),
    (3, 129, 64, "f32", True, "bf16"),        # K < 80: one padded group
    (2, 1000, 4096, "bf16", False, "bf16"),
    (3, 77, 6912, "bf16", True, "f32"),      # 3 x 6960 padded bytes of x_q
    (1, 3000, 16384, "bf16", True, "bf16"),  # the norm's row read in three passes
]


@pytest.mark.parametrize("M,N,K,dt,norm,yt", B3_CASES)
def test_b3_gemv_parity(dev, orc, M, N, K, dt, norm, yt):
    import torch
    W = synth.weights(N, K, 0.02, M + N, 1)
    x = synth.activations(M, K, M + K, 2, "normal", 0.01, 20.0, dt)
    x[0, :3] = 0.0
    g = synth.gain(K, 1, 3, dt) if norm else None
    Wd = torch.from_numpy(W).to(dev)
    P3, G3 = bl.bitnet_pack_weights_b3(Wd, EPS_W)
    P2, G2 = bl.bitnet_pack_weights(Wd, EPS_W)
    p_ref, g_ref = orc.pack_weights_b3(W, EPS_W)
    xq_r, a_r, _ = orc.quant_act(x, g, EPS_RMS)
    acc_r, y_r = orc.bitlinear_b3(p_ref, g_ref, K, xq_r, a_r)
    out = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32}[yt]
    xd = _x_dev(x, dt, dev)
    gd = None if g is None else _x_dev(g, dt, dev)
    y = bl.bitnet_bitlinear_gemv_b3(xd, P3, G3, gd, EPS_RMS, out_dtype=out)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
    if yt == "i32":
        np.testing.assert_array_equal(y.cpu().numpy(), acc_r)
    elif yt == "f32":
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), y_r.view(np.uint32))
    else:
        np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), orc.f32_to_bf16(y_r))
    # the same as the 2-bit fused kernel on the same matrix
    assert torch.equal(y, bl.bitnet_bitlinear_gemv(xd, P2, G2, gd, EPS_RMS, out_dtype=out))
