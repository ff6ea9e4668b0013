"""GPU parity of the one-launch decode FFN (bitnet_bitlinear_ffn_gemv) against
the CPU oracle's FFN: up and gate BitLinears, squared-ReLU gating to bf16 h,
down BitLinear.  h, the int32 accumulators of the down projection and the
dequantised outputs must match the oracle bit for bit."""
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


def _bf16_dev(x32, dev):
    import torch
    bits = synth.f32_to_bf16_bits(x32).view(np.int16)
    return torch.from_numpy(bits.copy()).to(dev).view(torch.bfloat16)


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _make(orc, dev, M, D, F, norm_in, norm_sub, seed):
    import torch
    Wu = synth.weights(F, D, 0.02, seed, 1)
    Wg = synth.weights(F, D, 0.02, seed, 2)
    Wd = synth.weights(D, F, 0.02, seed, 3)
    x = synth.activations(M, D, seed, 4, "normal", 0.01, 20.0, "bf16")
    gi = synth.gain(D, seed, 5, "bf16") if norm_in else None
    gs = synth.gain(F, seed, 6, "bf16") if norm_sub else None
    dv = {}
    ref = {}
    for name, W in (("up", Wu), ("gate", Wg), ("down", Wd)):
        P, G = bl.bitnet_pack_weights(torch.from_numpy(W).to(dev), EPS_W)
        p_ref, g_ref = orc.pack_weights(W, EPS_W)
        assert G.item() == g_ref and np.array_equal(P.cpu().numpy(), p_ref)
        dv[name] = (P, G)
        ref[name] = (p_ref, g_ref)
        del W
    return x, gi, gs, dv, ref


FFN_CASES = [
    # M, D, F, norm in, norm sub, y dtype
    (1, 2560, 6912, True, True, "bf16"),
    (1, 2560, 6912, False, False, "f32"),
    (2, 256, 512, True, False, "f32"),
    (4, 320, 640, False, True, "i32"),      # ragged: 4-5 features and 2-3 down rows per CTA
    (8, 64, 128, True, True, "bf16"),       # most CTAs own 0 or 1 feature
    (3, 1024, 4096, True, True, "f32"),
    (5, 2560, 6912, True, True, "bf16"),
    (1, 5376, 21504, True, True, "bf16"),   # 27B-class FFN, one token: the gated one-token GEMV, then the down GEMV
    (1, 5376, 21504, False, True, "f32"),   # the same without the input norm
    (1, 3072, 12288, True, False, "i32"),   # gated one-token GEMV: 84 features per CTA, a ragged last slot
    (2, 5376, 21504, True, True, "i32"),    # 27B-class FFN, two tokens: the one-launch kernel's rings
]


@pytest.mark.parametrize("M,D,F,norm_in,norm_sub,yt", FFN_CASES)
def test_ffn_parity(dev, orc, M, D, F, norm_in, norm_sub, yt):
    import torch
    x, gi, gs, dv, ref = _make(orc, dev, M, D, F, norm_in, norm_sub, seed=M + D)
    h_r, acc_r, y_r = orc.ffn(x, ref["up"], ref["gate"], ref["down"], gi, EPS_RMS, gs, EPS_RMS)
    out = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32}[yt]
    h, y = bl.bitnet_bitlinear_ffn_gemv(_bf16_dev(x, dev), *dv["up"], *dv["gate"], *dv["down"],
                                        None if gi is None else _bf16_dev(gi, dev), EPS_RMS,
                                        None if gs is None else _bf16_dev(gs, dev), EPS_RMS, out_dtype=out)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
    np.testing.assert_array_equal(_bits(h), h_r)
    if yt == "i32":
        np.testing.assert_array_equal(y.cpu().numpy(), acc_r)
    elif yt == "f32":
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), y_r.view(np.uint32))
    else:
        np.testing.assert_array_equal(_bits(y), orc.f32_to_bf16(y_r))


def test_ffn_matches_the_separate_bitlinear_calls(dev, orc):
    """Same result as fused decode BitLinears for up and gate (fp32 out), the
    gating, and a fused decode BitLinear for down on h."""
    import torch
    M, D, F = 2, 2560, 6912
    x, gi, gs, dv, _ = _make(orc, dev, M, D, F, True, True, seed=9)
    xd, gid, gsd = _bf16_dev(x, dev), _bf16_dev(gi, dev), _bf16_dev(gs, dev)
    h, y = bl.bitnet_bitlinear_ffn_gemv(xd, *dv["up"], *dv["gate"], *dv["down"], gid, EPS_RMS, gsd, EPS_RMS,
                                        out_dtype=torch.float32)
    u = bl.bitnet_bitlinear_gemv(xd, *dv["up"], gid, EPS_RMS, out_dtype=torch.float32)
    g = bl.bitnet_bitlinear_gemv(xd, *dv["gate"], gid, EPS_RMS, out_dtype=torch.float32)
    h2_bits = orc.f32_to_bf16(orc.relu2_gate(u.cpu().numpy(), g.cpu().numpy()))
    np.testing.assert_array_equal(_bits(h), h2_bits)
    y2 = bl.bitnet_bitlinear_gemv(h, *dv["down"], gsd, EPS_RMS, out_dtype=torch.float32)
    assert torch.equal(y, y2)


def test_ffn_shared_sync_words_repeat_and_graph_capture(dev, orc):
    """Back-to-back launches on one stream share the barrier words; results
    repeat bit for bit, eagerly and replayed from a CUDA graph, and the
    arrival counter has grown by one barrier of all CTAs per launch."""
    import torch
    M, D, F = 1, 2560, 6912
    x, gi, gs, dv, _ = _make(orc, dev, M, D, F, True, True, seed=3)
    xd, gid, gsd = _bf16_dev(x, dev), _bf16_dev(gi, dev), _bf16_dev(gs, dev)
    sync = torch.zeros(bl.BITNET_FFN_SYNC_BYTES, dtype=torch.uint8, device=dev)
    args = (xd, *dv["up"], *dv["gate"], *dv["down"], gid, EPS_RMS, gsd, EPS_RMS)
    h0, y0 = bl.bitnet_bitlinear_ffn_gemv(*args, sync=sync)
    hs = [torch.empty_like(h0) for _ in range(4)]
    ys = [torch.empty_like(y0) for _ in range(4)]
    for h, y in zip(hs, ys):
        bl.bitnet_bitlinear_ffn_gemv(*args, h=h, y=y, sync=sync)
    for h, y in zip(hs, ys):
        assert torch.equal(h, h0) and torch.equal(y, y0)
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for h, y in zip(hs, ys):
            bl.bitnet_bitlinear_ffn_gemv(*args, h=h, y=y, sync=sync)
    for h, y in zip(hs, ys):
        h.zero_()
        y.zero_()
    with torch.cuda.stream(stream):
        graph.replay()
        graph.replay()
    torch.cuda.synchronize(dev)
    for h, y in zip(hs, ys):
        assert torch.equal(h, h0) and torch.equal(y, y0)
    count = int(sync[:8].view(torch.int64).item())
    G = torch.cuda.get_device_properties(dev).multi_processor_count
    assert count == 13 * G  # 1 + 4 eager launches and 2 replays of 4, one barrier of G arrivals each
    assert bl.bitnet_get_device_status() == bl.BITNET_OK


def test_ffn_barrier_timeout_is_reported_and_context_survives(dev, orc):
    """Failure detection without a fault: start the barrier's arrival counter at
    1 instead of 0.  The CTA that arrives last then computes a target one
    barrier further on that no arrival will reach, gives up after the bounded
    wait (about 2 s), flags the device error word and returns; the host reads
    BITNET_ERR_TIMEOUT and the context stays usable: after re-zeroing the
    counter the next call is correct again."""
    import torch
    M, D, F = 1, 256, 512
    x, gi, gs, dv, ref = _make(orc, dev, M, D, F, True, True, seed=21)
    h_r, _, y_r = orc.ffn(x, ref["up"], ref["gate"], ref["down"], gi, EPS_RMS, gs, EPS_RMS)
    args = (_bf16_dev(x, dev), *dv["up"], *dv["gate"], *dv["down"], _bf16_dev(gi, dev), EPS_RMS,
            _bf16_dev(gs, dev), EPS_RMS)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
    sync = torch.zeros(bl.BITNET_FFN_SYNC_BYTES, dtype=torch.uint8, device=dev)
    sync[0] = 1  # arrival counter = 1: not a multiple of the CTA count
    bl.bitnet_bitlinear_ffn_gemv(*args, sync=sync, out_dtype=torch.float32)
    assert bl.bitnet_get_device_status() == bl.BITNET_ERR_TIMEOUT
    assert bl.bitnet_get_device_status() == bl.BITNET_OK  # the status was read and cleared
    sync.zero_()
    h, y = bl.bitnet_bitlinear_ffn_gemv(*args, sync=sync, out_dtype=torch.float32)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
    np.testing.assert_array_equal(_bits(h), h_r)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), y_r.view(np.uint32))
