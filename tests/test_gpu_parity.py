"""GPU parity: every step of the CUDA path against the CPU oracle, element by
element, on the same seeded inputs.

Integer results (packed weight bytes, int8 activations, int32 accumulators)
and the fp32 scales must match bit for bit.  Dequantised outputs must lie
within 1 ulp (fp32) or 1 bf16 ulp of the oracle; both sides run the same
sequence of correctly rounded fp32 operations, so in practice they match
exactly, and the tests also report that.
"""
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


def _t(a, dev, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return t if dtype is None else t.to(dtype)


def _x_dev(x32, dtype, dev):
    """fp32 values already rounded to dtype -> device tensor of that dtype (exact)."""
    import torch
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(x32).view(np.int16)
        return torch.from_numpy(bits.copy()).to(dev).view(torch.bfloat16)
    return _t(x32.astype(np.float32), dev)


def ulp_diff_f32(a, b):
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    ai = np.where(ai < 0, -(ai & 0x7FFFFFFF), ai)
    bi = np.where(bi < 0, -(bi & 0x7FFFFFFF), bi)
    return np.abs(ai - bi)


def ulp_diff_bf16(a_bits, b_bits):
    ai = np.asarray(a_bits, np.uint16).astype(np.int64)
    bi = np.asarray(b_bits, np.uint16).astype(np.int64)
    ai = np.where(ai >= 0x8000, -(ai & 0x7FFF), ai)
    bi = np.where(bi >= 0x8000, -(bi & 0x7FFF), bi)
    return np.abs(ai - bi)


# --------------------------------------------------------------------------- pack

PACK_SHAPES = [(256, 256, 0.02), (6912, 2560, 0.02), (2560, 6912, 0.02), (1, 64, 0.02), (7, 192, 1.0),
               (300, 640, 0.01), (13824, 2560, 0.02), (129, 2048, 3.0)]


@pytest.mark.parametrize("N,K,sigma", PACK_SHAPES)
def test_pack_parity(dev, orc, N, K, sigma):
    W = synth.weights(N, K, sigma, 7, 1)
    p_gpu, g_gpu = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    assert g_gpu.cpu().numpy()[0] == g_ref
    np.testing.assert_array_equal(p_gpu.cpu().numpy(), p_ref)


def test_pack_parity_27b_shape(dev, orc):
    W = synth.weights(21504, 5376, 0.01, 0, 91)
    p_gpu, g_gpu = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    assert g_gpu.cpu().numpy()[0] == g_ref
    assert np.array_equal(p_gpu.cpu().numpy(), p_ref)


def test_pack_edge_cases(dev, orc):
    # all-zero matrix: gamma 0, every code 0 (byte 0x55)
    p, g = bl.bitnet_pack_weights(_t(np.zeros((5, 128), np.float32), dev), EPS_W)
    assert g.item() == 0.0 and np.all(p.cpu().numpy() == 0x55)
    # +-2^j: gamma exact, codes = sign
    rng = np.random.default_rng(1)
    W = (rng.choice([-1.0, 1.0], size=(64, 256)) * 0.25).astype(np.float32)
    p, g = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    assert g.item() == 0.25
    q, bad = orc.unpack_codes(p.cpu().numpy(), 256)
    assert bad == 0 and np.array_equal(q, np.sign(W).astype(np.int8))
    # exact ties, with the divisor made exactly 1 (eps = 1 - gamma)
    row = np.full(64, 0.125, np.float32)
    row[:6] = [0.5, -0.5, 1.5, -1.5, 2.5, 0.75]
    g_ref = orc.absmean_gamma(row[None])
    eps = float(np.float32(1.0) - g_ref)
    p, g = bl.bitnet_pack_weights(_t(row[None], dev), eps)
    p_ref, _ = orc.pack_weights(row[None], eps)
    np.testing.assert_array_equal(p.cpu().numpy(), p_ref)
    # non-finite input is reported
    W = synth.weights(8, 64, 0.02, 0, 1)
    W[3, 9] = np.nan
    with pytest.raises(bl.BitnetError) as e:
        bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    assert e.value.status == bl.BITNET_ERR_NONFINITE


# --------------------------------------------------------------------------- quant

QUANT_CASES = [
    # M, K, dist, outlier frac, outlier scale, dtype, norm
    (4, 256, "normal", 0.0, 1.0, "f32", False),
    (1, 2560, "normal", 0.01, 20.0, "bf16", False),
    (1, 6912, "normal", 0.01, 20.0, "bf16", False),
    (64, 2560, "normal", 0.0, 1.0, "bf16", True),
    (64, 6912, "normal", 0.0, 1.0, "bf16", True),
    (4096, 2560, "student_t4", 0.0, 1.0, "bf16", False),
    (16, 21504, "normal", 0.005, 30.0, "bf16", False),
    (2048, 5376, "normal", 0.005, 30.0, "bf16", False),
    (3, 64, "normal", 0.0, 1.0, "bf16", True),
    (5, 1344, "student_t4", 0.0, 1.0, "f32", True),
    (2, 32768, "normal", 0.0, 1.0, "bf16", True),
    (2, 16384, "normal", 0.0, 1.0, "f32", False),
    # from 512 bf16 rows with K <= 6144 a warp quantises each row (quant_rows_kernel)
    (512, 2560, "normal", 0.01, 20.0, "bf16", True),
    (1024, 2624, "student_t4", 0.0, 1.0, "bf16", True),   # 328 chunks: lanes own 10 or 11
    (600, 6144, "normal", 0.01, 20.0, "bf16", True),     # 24 chunks per lane, the most a warp holds
    (513, 6080, "normal", 0.0, 1.0, "bf16", False),      # 760 chunks: lanes own 23 or 24
    (600, 6912, "normal", 0.01, 20.0, "bf16", True),     # K above 6144: a CTA per row again
    (520, 6208, "normal", 0.0, 1.0, "bf16", True),       # the first K past the warp kernel's registers
    (600, 21504, "normal", 0.005, 30.0, "bf16", True),   # the 27B down projection's input
    (513, 32768, "student_t4", 0.0, 1.0, "bf16", False),  # the longest bf16 row
    (777, 64, "normal", 0.0, 1.0, "bf16", True),         # 8 chunks: 24 lanes own none
    (640, 1344, "student_t4", 0.0, 1.0, "bf16", False),
    (2048, 5376, "normal", 0.005, 30.0, "bf16", True),
    (4096, 6912, "student_t4", 0.0, 1.0, "bf16", False),  # the prefill down projection's input
    (511, 2560, "normal", 0.0, 1.0, "bf16", True),       # one row below the warp kernel's threshold
    (1024, 1344, "normal", 0.0, 1.0, "f32", True),       # fp32 input: a CTA per row at any M
    # rows past the norm path's register budget, read in three passes
    (3, 8192, "normal", 0.01, 20.0, "f32", True),        # a row per SM: 1024 threads per row
    (200, 12288, "normal", 0.01, 20.0, "f32", True),     # more rows than SMs: 256 threads per row
    (300, 12288, "normal", 0.005, 30.0, "bf16", True),   # bf16, 6 chunks per lane
    (1, 21504, "normal", 0.005, 30.0, "bf16", True),     # one token, the 27B FFN's sub-norm input
    # more than two long rows per SM: persistent CTAs stream the rows through shared memory
    (297, 8192, "normal", 0.0, 1.0, "bf16", False),      # the first M and bf16 K that take it (256 threads)
    (350, 4096, "normal", 0.01, 20.0, "f32", False),     # the first f32 K that takes it
    (297, 12352, "normal", 0.0, 1.0, "bf16", False),     # the first bf16 K past 24 KB rows (512 threads)
    (400, 8192, "normal", 0.01, 20.0, "f32", True),      # f32 rows with the gain (one CTA per SM)
    (400, 16384, "normal", 0.0, 1.0, "f32", False),      # 64-KB f32 rows
]


@pytest.mark.parametrize("M,K,dist,of,osc,dt,norm", QUANT_CASES)
def test_quant_parity(dev, orc, M, K, dist, of, osc, dt, norm):
    x = synth.activations(M, K, 3, 2, dist, of, osc, dt)
    g = synth.gain(K, 3, 3, dt) if norm else None
    xq, a, rs = bl.bitnet_quant_act(_x_dev(x, dt, dev), None if g is None else _x_dev(g, dt, dev), EPS_RMS,
                                    want_rowsum=True)
    xq_r, a_r, rs_r = orc.quant_act(x, g, EPS_RMS)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_r)
    np.testing.assert_array_equal(a.cpu().numpy(), a_r)
    np.testing.assert_array_equal(rs.cpu().numpy(), rs_r)


def test_quant_edge_tokens(dev, orc):
    K = 128
    x = synth.activations(6, K, 1, 2, "normal", 0.0, 1.0, "f32")
    x[0] = 0.0                                   # zero token
    x[1] = 0.0
    x[1, 77] = -3.0                              # one-hot
    x[2, :10] = [127, 0.5, 1.5, 2.5, -2.5, -0.5, 126.5, 3.5, -3.5, 0.25]
    x[2, 10:] = 0.0                              # exact ties
    x[3] *= np.float32(2.0 ** 40)                # huge
    x[4] *= np.float32(2.0 ** -60)               # tiny
    for norm in (False, True):
        g = synth.gain(K, 1, 3, "f32") if norm else None
        xq, a, rs = bl.bitnet_quant_act(_t(x, dev), None if g is None else _t(g, dev), EPS_RMS, want_rowsum=True)
        xq_r, a_r, rs_r = orc.quant_act(x, g, EPS_RMS)
        np.testing.assert_array_equal(xq.cpu().numpy(), xq_r)
        np.testing.assert_array_equal(a.cpu().numpy(), a_r)
        np.testing.assert_array_equal(rs.cpu().numpy(), rs_r)
    # the quantisation without rowsum output gives the same codes
    xq2, a2, rs2 = bl.bitnet_quant_act(_t(x, dev))
    assert rs2 is None
    np.testing.assert_array_equal(xq2.cpu().numpy(), orc.quant_act(x)[0])


def test_quant_edge_tokens_many_rows(dev, orc):
    """The same edge rows among 640 bf16 tokens, where one warp quantises each
    row (rows streamed through shared memory for K = 21504): zero, one-hot, exact ties after
    scaling, huge, tiny and a row whose maximum sits in its last chunk (held
    by lane 31 for K = 2560 and 6144)."""
    import torch
    for K in (128, 2560, 6144, 21504):
        x = synth.activations(640, K, 5, 2, "normal", 0.0, 1.0, "bf16")
        x[0] = 0.0
        x[1] = 0.0
        x[1, K - 1] = -3.0
        x[2, :10] = [127, 0.5, 1.5, 2.5, -2.5, -0.5, 126.5, 3.5, -3.5, 0.25]
        x[2, 10:] = 0.0
        x[3] *= np.float32(2.0 ** 40)
        x[4] *= np.float32(2.0 ** -60)
        x[5, K - 8:] = 100.0
        x = orc.bf16_to_f32(orc.f32_to_bf16(x))
        for norm in (False, True):
            g = synth.gain(K, 5, 3, "bf16") if norm else None
            xq, a, rs = bl.bitnet_quant_act(_x_dev(x, "bf16", dev), None if g is None else _x_dev(g, "bf16", dev),
                                            EPS_RMS, want_rowsum=True)
            xq_r, a_r, rs_r = orc.quant_act(x, g, EPS_RMS)
            np.testing.assert_array_equal(xq.cpu().numpy(), xq_r)
            np.testing.assert_array_equal(a.cpu().numpy(), a_r)
            np.testing.assert_array_equal(rs.cpu().numpy(), rs_r)
        # the first 511 rows alone (below the warp-per-row threshold): same codes and scales
        xq5, a5, _ = bl.bitnet_quant_act(_x_dev(x[:511], "bf16", dev), _x_dev(g, "bf16", dev), EPS_RMS)
        assert torch.equal(xq5, xq[:511]) and torch.equal(a5, a[:511])


# --------------------------------------------------------------------------- linear

def _ref_linear(orc, packed, gamma, K, xq, a):
    acc, y = orc.bitlinear(packed, gamma, K, xq, a)
    return acc, y


def _check_linear(dev, orc, fn, M, N, K, seed=0, zero_row=None, zero_tok=None, sample=None):
    import torch
    rng = np.random.default_rng(seed)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    if zero_row is not None:
        q[zero_row] = 0
    packed = orc.pack_codes(q)
    x = synth.activations(M, K, seed, 5, "student_t4", 0.0, 1.0, "f32")
    if zero_tok is not None:
        x[zero_tok] = 0.0
    xq, a, rs = orc.quant_act(x)
    gamma = np.float32(0.0173)
    P, G = _t(packed, dev), _t(np.array([gamma], np.float32), dev)
    XQ, A, RS = _t(xq, dev), _t(a, dev), _t(rs, dev)
    if sample is None:
        acc_r, y_r = orc.bitlinear(packed, gamma, K, xq, a)
    else:
        ms = np.concatenate([rng.integers(0, M, sample), np.arange(M), np.full(N if N < 64 else 64, M - 1)])
        ns = np.concatenate([rng.integers(0, N, sample), np.full(M, N - 1), np.arange(N if N < 64 else 64)])
        acc_r, y_r = orc.bitlinear_sampled(packed, gamma, K, xq, a, ms, ns)
    for rowsum in (None, RS):
        acc_g = fn(P, G, XQ, A, rowsum, out_dtype=torch.int32).cpu().numpy()
        y32 = fn(P, G, XQ, A, rowsum, out_dtype=torch.float32).cpu().numpy()
        yb = fn(P, G, XQ, A, rowsum, out_dtype=torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)
        if sample is not None:
            acc_g, y32, yb = acc_g[ms, ns], y32[ms, ns], yb[ms, ns]
        np.testing.assert_array_equal(acc_g, acc_r)
        d32 = ulp_diff_f32(y32, y_r)
        assert d32.max() <= 1, f"fp32 output off by {d32.max()} ulp"
        db = ulp_diff_bf16(yb, orc.f32_to_bf16(y_r))
        assert db.max() <= 1, f"bf16 output off by {db.max()} ulp"
        assert d32.max() == 0 and db.max() == 0, "expected bit-exact outputs"


GEMV_CASES = [(1, 256, 256), (4, 256, 256), (8, 6912, 2560), (1, 2560, 6912), (3, 129, 192), (5, 1, 64),
              (2, 37, 4160), (7, 300, 640), (1, 1000, 21504), (6, 77, 8192),
              # 27B-class shapes: the deep-ring launch plan (long chunks, several slots per warp)
              (1, 21504, 5376), (3, 21504, 5376), (2, 5376, 21504), (1, 5373, 21504),
              # one token, large shares (whole-row slots): ragged rows and slots, 2/8/16 column
              # segments per row, and the first K past the register budget (the item kernel again)
              (1, 10007, 8192), (1, 3001, 32768), (1, 600, 65536), (1, 700, 65600)]


@pytest.mark.parametrize("M,N,K", GEMV_CASES)
def test_gemv_parity(dev, orc, M, N, K):
    _check_linear(dev, orc, bl.bitnet_linear_gemv, M, N, K, seed=M + N + K, zero_row=min(3, N - 1), zero_tok=0)


GEMM_CASES = [(4, 256, 256), (16, 256, 256), (1, 128, 128), (17, 129, 192), (64, 3840, 2560), (33, 200, 64),
              (100, 300, 640), (129, 257, 1088), (256, 512, 1024), (300, 1000, 2048), (64, 2560, 6912)]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_gemm_parity(dev, orc, M, N, K):
    _check_linear(dev, orc, bl.bitnet_linear_gemm, M, N, K, seed=M * 7 + N + K, zero_row=min(5, N - 1),
                  zero_tok=min(2, M - 1))


@pytest.mark.parametrize("M,N,K", [(4096, 6912, 2560), (2048, 5376, 21504), (16, 21504, 5376)])
def test_gemm_parity_large_sampled(dev, orc, M, N, K):
    _check_linear(dev, orc, bl.bitnet_linear_gemm, M, N, K, seed=1, sample=3000)


def test_gemv_and_gemm_agree(dev, orc):
    import torch
    rng = np.random.default_rng(9)
    N, K = 640, 2560
    P = _t(orc.pack_codes(rng.integers(-1, 2, size=(N, K)).astype(np.int8)), dev)
    G = _t(np.array([0.02], np.float32), dev)
    for M in range(1, 9):
        x = synth.activations(M, K, M, 5, "normal", 0.0, 1.0, "bf16")
        xq, a, rs = bl.bitnet_quant_act(_x_dev(x, "bf16", dev), want_rowsum=True)
        y1 = bl.bitnet_linear_gemv(P, G, xq, a, rs, out_dtype=torch.float32)
        y2 = bl.bitnet_linear_gemm(P, G, xq, a, None, out_dtype=torch.float32)
        assert torch.equal(y1, y2)


# --------------------------------------------------------------------------- fused decode BitLinear

FUSED_CASES = [
    # M, N, K, x dtype, norm, y dtype
    (1, 6912, 2560, "bf16", False, "bf16"),
    (1, 2560, 6912, "bf16", True, "f32"),
    (1, 5376, 21504, "bf16", False, "bf16"),
    (4, 256, 256, "f32", False, "f32"),
    (8, 300, 2688, "bf16", True, "i32"),
    (3, 129, 64, "f32", True, "bf16"),
    (2, 1000, 4096, "bf16", False, "bf16"),
    (1, 21504, 5376, "bf16", False, "bf16"),   # 27B up: deep-ring plan, one token (masked fields)
    (2, 5376, 10752, "bf16", True, "f32"),     # deep-ring plan with two tokens
    (1, 21501, 5376, "bf16", True, "i32"),     # ragged last group of the last CTA
    (1, 9000, 12288, "f32", True, "bf16"),     # one token, whole-row slots, f32 input with the norm
    (1, 6144, 16384, "bf16", True, "bf16"),    # one token, the norm's row read in three passes
    (2, 700, 10752, "f32", True, "bf16"),      # item GEMV, two f32 tokens, the same
]


@pytest.mark.parametrize("M,N,K,dt,norm,yt", FUSED_CASES)
def test_fused_bitlinear_gemv_parity(dev, orc, M, N, K, dt, norm, yt):
    import torch
    W = synth.weights(N, K, 0.02, M + N, 1)
    x = synth.activations(M, K, M + K, 2, "normal", 0.01, 20.0, dt)
    x[0, :3] = 0.0
    g = synth.gain(K, 1, 3, dt) if norm else None
    P, G = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    xq_r, a_r, _ = orc.quant_act(x, g, EPS_RMS)
    acc_r, y_r = orc.bitlinear(p_ref, g_ref, K, xq_r, a_r)
    out = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32}[yt]
    xd = _x_dev(x, dt, dev)
    gd = None if g is None else _x_dev(g, dt, dev)
    y = bl.bitnet_bitlinear_gemv(xd, P, G, gd, EPS_RMS, out_dtype=out)
    if yt == "i32":
        np.testing.assert_array_equal(y.cpu().numpy(), acc_r)
    elif yt == "f32":
        assert ulp_diff_f32(y.cpu().numpy(), y_r).max() == 0
    else:
        yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert ulp_diff_bf16(yb, orc.f32_to_bf16(y_r)).max() == 0
    # identical to the two-call path
    xq, a, rs = bl.bitnet_quant_act(xd, gd, EPS_RMS, want_rowsum=True)
    assert torch.equal(y, bl.bitnet_linear_gemv(P, G, xq, a, rs, out_dtype=out))


@pytest.mark.parametrize("M,N,K,dt,norm,yt", [(1, 21504, 5376, "bf16", False, "bf16"),
                                                (2, 1000, 4096, "f32", True, "f32"),
                                                (1, 300, 2688, "bf16", True, "i32")])
def test_fused_bitlinear_gemv_host_buffers(dev, orc, M, N, K, dt, norm, yt):
    """The host-buffer form: pinned x in, pinned y out, on a side stream,
    several calls in flight before one synchronisation; every y_host equals
    the device path's output and the oracle's."""
    import torch
    W = synth.weights(N, K, 0.02, M + N, 1)
    P, G = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    g = synth.gain(K, 1, 3, dt) if norm else None
    gd = None if g is None else _x_dev(g, dt, dev)
    out = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32}[yt]
    xs = [synth.activations(M, K, M + K + i, 2, "normal", 0.01, 20.0, dt) for i in range(3)]
    x_host = [_x_dev(x, dt, dev).cpu().pin_memory() for x in xs]
    y_host = [torch.empty((M, N), dtype=out).pin_memory() for _ in xs]
    x_dev = [torch.empty_like(h, device=dev) for h in x_host]
    y_dev = [torch.empty((M, N), dtype=out, device=dev) for _ in xs]
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        for i in range(len(xs)):
            bl.bitnet_bitlinear_gemv_host(x_host[i], x_dev[i], P, G, y_dev[i], y_host[i], gd, EPS_RMS)
    s.synchronize()
    for i, x in enumerate(xs):
        xq_r, a_r, _ = orc.quant_act(x, g, EPS_RMS)
        acc_r, y_r = orc.bitlinear(p_ref, g_ref, K, xq_r, a_r)
        assert torch.equal(y_host[i], y_dev[i].cpu())
        if yt == "i32":
            np.testing.assert_array_equal(y_host[i].numpy(), acc_r)
        elif yt == "f32":
            assert ulp_diff_f32(y_host[i].numpy(), y_r).max() == 0
        else:
            yb = y_host[i].view(torch.int16).numpy().view(np.uint16)
            assert ulp_diff_bf16(yb, orc.f32_to_bf16(y_r)).max() == 0


# --------------------------------------------------------------------------- whole workloads

_PACKED = {}


def _packed_weights(lin, dev, orc):
    """(device pack, oracle pack) of a workload's weights, checked once per weight spec."""
    key = (lin.N, lin.K, lin.w_sigma, lin.w_id)
    if key not in _PACKED:
        if len(_PACKED) >= 2:
            _PACKED.clear()
        W = lin.make_w(0)
        P, G = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
        p_ref, g_ref = orc.pack_weights(W, EPS_W)
        assert G.item() == g_ref
        assert np.array_equal(P.cpu().numpy(), p_ref)
        _PACKED[key] = (P, G, p_ref, g_ref)
    return _PACKED[key]


@pytest.mark.parametrize("workload", list(synth.WORKLOADS))
def test_workload_end_to_end(dev, orc, workload):
    """pack -> quant -> product on each named workload at full size, in the
    launch configuration the benchmark uses; outputs checked on samples."""
    import torch
    for lin in synth.WORKLOADS[workload]:
        x = lin.make_x(0)
        g = lin.make_gain(0)
        P, G, p_ref, g_ref = _packed_weights(lin, dev, orc)
        xq, a, rs = bl.bitnet_quant_act(_x_dev(x, lin.x_dtype, dev),
                                        None if g is None else _x_dev(g, lin.x_dtype, dev), EPS_RMS,
                                        want_rowsum=True)
        xq_r, a_r, rs_r = orc.quant_act(x, g, EPS_RMS)
        assert np.array_equal(xq.cpu().numpy(), xq_r)
        assert np.array_equal(a.cpu().numpy(), a_r)
        out = torch.float32 if lin.y_dtype == "f32" else torch.bfloat16
        fns = [bl.bitnet_linear_gemv, bl.bitnet_linear_gemm] if lin.M <= 8 else [bl.bitnet_linear_gemm]
        rng = np.random.default_rng(0)
        ms = rng.integers(0, lin.M, 2000)
        ns = rng.integers(0, lin.N, 2000)
        acc_r, y_r = orc.bitlinear_sampled(p_ref, g_ref, lin.K, xq_r, a_r, ms, ns)
        for fn in fns:
            acc = fn(P, G, xq, a, rs, out_dtype=torch.int32).cpu().numpy()[ms, ns]
            np.testing.assert_array_equal(acc, acc_r)
            y = fn(P, G, xq, a, rs, out_dtype=out)
            if out == torch.float32:
                assert ulp_diff_f32(y.cpu().numpy()[ms, ns], y_r).max() == 0
            else:
                yb = y.view(torch.int16).cpu().numpy().view(np.uint16)[ms, ns]
                assert ulp_diff_bf16(yb, orc.f32_to_bf16(y_r)).max() == 0


def test_repeatable_and_status_clean(dev, orc):
    import torch
    lin = synth.WORKLOADS["decode_m64_2p5b_block"][3]
    P, G = bl.bitnet_pack_weights(_t(lin.make_w(0), dev), EPS_W)
    x = _x_dev(lin.make_x(0), "bf16", dev)
    g = _x_dev(lin.make_gain(0), "bf16", dev)
    outs = []
    for _ in range(3):
        xq, a, rs = bl.bitnet_quant_act(x, g, EPS_RMS, want_rowsum=True)
        y = bl.bitnet_linear_gemm(P, G, xq, a, rs, out_dtype=torch.float32)
        outs.append((xq.clone(), a.clone(), rs.clone(), y))
    for o in outs[1:]:
        for u, v in zip(outs[0], o):
            assert torch.equal(u, v)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK


def test_gemv_after_a_kernel_that_writes_the_weights(dev, orc):
    """The decode kernels request their first weight tiles before waiting on
    the previous kernel (programmatic dependent launch).  A torch kernel that
    writes W_packed just before them on the same stream (here a copy from a
    second buffer) does not signal early completion, so the kernels still see
    the new weights: checked against the oracle for both decode entry points."""
    import torch
    N, K = 21504, 5376
    rng = np.random.default_rng(3)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = orc.pack_codes(q)
    x = synth.activations(1, K, 4, 2, "normal", 0.01, 20.0, "bf16")
    xq_r, a_r, _ = orc.quant_act(x)
    gamma = np.float32(0.0125)
    _, y_r = orc.bitlinear(packed, gamma, K, xq_r, a_r)
    src = _t(packed, dev)
    G = _t(np.array([gamma], np.float32), dev)
    xd = _x_dev(x, "bf16", dev)
    xq, a, rs = bl.bitnet_quant_act(xd, want_rowsum=True)
    for trial in range(3):
        P = torch.zeros_like(src)
        torch.cuda.synchronize()
        P.copy_(src)                      # writes W_packed on the current stream ...
        y1 = bl.bitnet_bitlinear_gemv(xd, P, G, out_dtype=torch.float32)   # ... read right after
        P2 = torch.zeros_like(src)
        P2.copy_(src)
        y2 = bl.bitnet_linear_gemv(P2, G, xq, a, rs, out_dtype=torch.float32)
        assert ulp_diff_f32(y1.cpu().numpy(), y_r).max() == 0
        assert ulp_diff_f32(y2.cpu().numpy(), y_r).max() == 0


# --------------------------------------------------------------------------- stream-K GEMM (M <= 64)

SK_CASES = [(1, 128, 64), (16, 21504, 5376), (16, 5376, 21504), (64, 3840, 2560), (64, 2560, 6912),
            (5, 300, 320), (33, 1000, 2624), (17, 777, 5376), (64, 13824, 2560), (2, 129, 21504)]


@pytest.mark.parametrize("M,N,K", SK_CASES)
def test_gemm_stream_k_matches_tiles_and_oracle(dev, orc, M, N, K):
    """Stream-K (equal work per SM, partial tiles added through the workspace;
    forced at every size) against the persistent-tile path, the automatic
    choice and the oracle, with one workspace reused by every call (the calls
    must leave its flags and accumulation slots zero)."""
    import torch
    rng = np.random.default_rng(M + N + K)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = orc.pack_codes(q)
    x = synth.activations(M, K, 11, 5, "student_t4", 0.0, 1.0, "f32")
    xq, a, rs = orc.quant_act(x)
    gamma = np.float32(0.0211)
    P, G = _t(packed, dev), _t(np.array([gamma], np.float32), dev)
    XQ, A, RS = _t(xq, dev), _t(a, dev), _t(rs, dev)
    ws = torch.zeros(bl.bitnet_linear_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    ms = rng.integers(0, M, 4000)
    ns = rng.integers(0, N, 4000)
    acc_r, y_r = orc.bitlinear_sampled(packed, gamma, K, xq, a, ms, ns)
    for rowsum in (RS, None):
        for out in (torch.int32, torch.float32, torch.bfloat16):
            y_sk = bl.bitnet_linear_gemm_stream_k(P, G, XQ, A, rowsum, out_dtype=out, workspace=ws)
            y_t = bl.bitnet_linear_gemm(P, G, XQ, A, rowsum, out_dtype=out, stream_k=False)
            y_auto = bl.bitnet_linear_gemm(P, G, XQ, A, rowsum, out_dtype=out, workspace=ws)
            assert torch.equal(y_sk, y_t) and torch.equal(y_sk, y_auto)
            if out == torch.int32:
                np.testing.assert_array_equal(y_sk.cpu().numpy()[ms, ns], acc_r)
            elif out == torch.float32:
                assert ulp_diff_f32(y_sk.cpu().numpy()[ms, ns], y_r).max() == 0
            else:
                yb = y_sk.view(torch.int16).cpu().numpy().view(np.uint16)[ms, ns]
                assert ulp_diff_bf16(yb, orc.f32_to_bf16(y_r)).max() == 0
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    assert int(ws[:4 * sms].view(torch.int32).abs().sum()) == 0, "flags left raised"
    assert int(ws.view(torch.int32).abs().sum()) == 0, "accumulation slots left non-zero"
    assert bl.bitnet_get_device_status() == bl.BITNET_OK


def test_gemm_stream_k_in_a_cuda_graph(dev, orc):
    """Several stream-K calls sharing one workspace inside a CUDA graph, the
    graph replayed three times: every replay exact, flags zero at the end."""
    import torch
    M, N, K = 16, 6912, 2560
    rng = np.random.default_rng(5)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = orc.pack_codes(q)
    x = synth.activations(M, K, 2, 5, "normal", 0.01, 20.0, "bf16")
    xq, a, rs = orc.quant_act(x)
    gamma = np.float32(0.0187)
    acc_r, _ = orc.bitlinear(packed, gamma, K, xq, a)
    P, G = _t(packed, dev), _t(np.array([gamma], np.float32), dev)
    XQ, A, RS = _t(xq, dev), _t(a, dev), _t(rs, dev)
    ws = torch.zeros(bl.bitnet_linear_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    ys = [torch.empty((M, N), dtype=torch.int32, device=dev) for _ in range(3)]
    s = torch.cuda.Stream(dev)
    bl.bitnet_linear_gemm_stream_k(P, G, XQ, A, RS, y=ys[0], workspace=ws)  # first call outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for y in ys:
            bl.bitnet_linear_gemm_stream_k(P, G, XQ, A, RS, y=y, workspace=ws)
    for _ in range(3):
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        for y in ys:
            np.testing.assert_array_equal(y.cpu().numpy(), acc_r)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    assert int(ws[:4 * sms].view(torch.int32).abs().sum()) == 0
    assert bl.bitnet_get_device_status() == bl.BITNET_OK


# --------------------------------------------------------------------------- FFN up|gate with the squared-ReLU gate

UPGATE_CASES = [(64, 6912, 2560, False), (5, 200, 320, True), (16, 21504, 5376, False), (33, 777, 1344, True),
                (2048, 6912, 2560, False)]


@pytest.mark.parametrize("M,F,K,signed", UPGATE_CASES)
def test_upgate_gemm_matches_oracle_ffn_gate(dev, orc, M, F, K, signed):
    """h = bf16(relu(g)^2 u) from one tensor-core product of the up and gate
    weights, against the oracle's BitLinears and squared-ReLU gate (bit-exact;
    sampled at M = 2048)."""
    import torch
    W_up = synth.weights(F, K, 0.02, 3, 31)
    W_gate = synth.weights(F, K, 0.02, 3, 32)
    x = synth.activations(M, K, 3, 33, "normal", 0.01, 20.0, "bf16")
    g_in = synth.gain(K, 3, 34, "bf16")
    pu, gu = orc.pack_weights(W_up, EPS_W)
    pg, gg = orc.pack_weights(W_gate, EPS_W)
    xq_r, a_r, _ = orc.quant_act(x, g_in, EPS_RMS)
    Pu, Gu = bl.bitnet_pack_weights(_t(W_up, dev), EPS_W)
    Pg, Gg = bl.bitnet_pack_weights(_t(W_gate, dev), EPS_W)
    xq, a, rs = bl.bitnet_quant_act(_x_dev(x, "bf16", dev), _x_dev(g_in, "bf16", dev), EPS_RMS, want_rowsum=True)
    assert np.array_equal(xq.cpu().numpy(), xq_r)
    ws = torch.zeros(bl.bitnet_linear_upgate_workspace_bytes(M, F, K), dtype=torch.uint8, device=dev)
    h = bl.bitnet_linear_upgate_gemm(Pu, Gu, Pg, Gg, xq, a, None if signed else rs, workspace=ws)
    hb = h.view(torch.int16).cpu().numpy().view(np.uint16)
    if M * F <= 64 * 21504:
        _, u = orc.bitlinear(pu, gu, K, xq_r, a_r)
        _, g = orc.bitlinear(pg, gg, K, xq_r, a_r)
        np.testing.assert_array_equal(hb, orc.f32_to_bf16(orc.relu2_gate(u, g)))
    else:
        rng = np.random.default_rng(0)
        ms, ns = rng.integers(0, M, 4000), rng.integers(0, F, 4000)
        _, u = orc.bitlinear_sampled(pu, gu, K, xq_r, a_r, ms, ns)
        _, g = orc.bitlinear_sampled(pg, gg, K, xq_r, a_r, ms, ns)
        np.testing.assert_array_equal(hb[ms, ns], orc.f32_to_bf16(orc.relu2_gate(u, g)))
    # the same h from the two separate products and the oracle's gate on their outputs
    u_d = bl.bitnet_linear_gemm(Pu, Gu, xq, a, rs, out_dtype=torch.float32)
    g_d = bl.bitnet_linear_gemm(Pg, Gg, xq, a, rs, out_dtype=torch.float32)
    ref = orc.f32_to_bf16(orc.relu2_gate(u_d.cpu().numpy(), g_d.cpu().numpy()))
    np.testing.assert_array_equal(hb, ref)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    assert int(ws[:4 * sms].view(torch.int32).abs().sum()) == 0
    assert bl.bitnet_get_device_status() == bl.BITNET_OK


# --------------------------------------------------------------------------- fused quantisation + stream-K (M <= 64)

FQ_CASES = [
    # M, N, K, x dtype, norm, y dtype
    (64, 3840, 2560, "bf16", True, "bf16"),      # the 2.5B block's Q|K|V at M = 64
    (64, 2560, 6912, "bf16", True, "f32"),       # its down projection
    (16, 21504, 5376, "bf16", False, "bf16"),    # 27B up at M = 16
    (16, 5376, 21504, "bf16", False, "i32"),     # 27B down at M = 16 (16 chunks per thread)
    (5, 300, 320, "f32", True, "f32"),
    (33, 777, 1344, "f32", False, "bf16"),
    (1, 128, 64, "bf16", True, "f32"),           # one unit: a grid of one CTA quantises every row
    (9, 129, 8192, "f32", True, "i32"),
    (16, 2048, 21504, "bf16", True, "f32"),      # the norm's rows read in three passes inside the product
]


@pytest.mark.parametrize("M,N,K,dt,norm,yt", FQ_CASES)
def test_fused_bitlinear_gemm_parity(dev, orc, M, N, K, dt, norm, yt):
    """Quantisation inside the stream-K product (one launch, grid barrier in the
    workspace) against the oracle and against the two-call path."""
    import torch
    W = synth.weights(N, K, 0.02, M + N, 1)
    x = synth.activations(M, K, M + K, 2, "normal", 0.01, 20.0, dt)
    x[0, :3] = 0.0
    if M > 2:
        x[2] = 0.0                                   # an all-zero token
    g = synth.gain(K, 1, 3, dt) if norm else None
    P, G = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
    p_ref, g_ref = orc.pack_weights(W, EPS_W)
    xq_r, a_r, _ = orc.quant_act(x, g, EPS_RMS)
    out = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32}[yt]
    xd = _x_dev(x, dt, dev)
    gd = None if g is None else _x_dev(g, dt, dev)
    ws = torch.zeros(bl.bitnet_bitlinear_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    y = bl.bitnet_bitlinear_gemm_stream_k(xd, P, G, gd, EPS_RMS, out_dtype=out, workspace=ws)
    if M * N * K <= 64 * 3840 * 2560:
        acc_r, y_r = orc.bitlinear(p_ref, g_ref, K, xq_r, a_r)
        got = y.cpu().numpy() if yt != "bf16" else None
    else:
        rng = np.random.default_rng(1)
        ms, ns = rng.integers(0, M, 4000), rng.integers(0, N, 4000)
        acc_r, y_r = orc.bitlinear_sampled(p_ref, g_ref, K, xq_r, a_r, ms, ns)
        got = y.cpu().numpy()[ms, ns] if yt != "bf16" else None
    if yt == "i32":
        np.testing.assert_array_equal(got, acc_r)
    elif yt == "f32":
        assert ulp_diff_f32(got, y_r).max() == 0
    else:
        yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
        if M * N * K > 64 * 3840 * 2560:
            yb = yb[ms, ns]
        assert ulp_diff_bf16(yb, orc.f32_to_bf16(y_r)).max() == 0
    # identical to the two-call path, and again with the same workspace (barrier words reused)
    xq, a, rs = bl.bitnet_quant_act(xd, gd, EPS_RMS, want_rowsum=True)
    y2 = bl.bitnet_linear_gemm(P, G, xq, a, rs, out_dtype=out)
    assert torch.equal(y, y2)
    y3 = bl.bitnet_bitlinear_gemm(xd, P, G, gd, EPS_RMS, out_dtype=out, workspace=ws)  # the automatic choice
    assert torch.equal(y, y3)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK


def test_fused_bitlinear_gemm_shares_a_workspace_across_shapes_and_graph_replays(dev, orc):
    """One workspace for launches of different grid sizes (the barrier's arrival
    count returns to zero after each), captured in a CUDA graph and replayed."""
    import torch
    shapes = [(16, 21504, 5376), (3, 128, 64), (64, 2560, 2560), (16, 21504, 5376)]
    ws_bytes = max(bl.bitnet_bitlinear_gemm_workspace_bytes(*s) for s in shapes)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    cases = []
    for i, (M, N, K) in enumerate(shapes):
        W = synth.weights(N, K, 0.02, i, 7)
        x = synth.activations(M, K, i, 8, "normal", 0.0, 1.0, "bf16")
        g = synth.gain(K, i, 9, "bf16")
        P, G = bl.bitnet_pack_weights(_t(W, dev), EPS_W)
        xd, gd = _x_dev(x, "bf16", dev), _x_dev(g, "bf16", dev)
        xq, a, rs = bl.bitnet_quant_act(xd, gd, EPS_RMS, want_rowsum=True)
        ref = bl.bitnet_linear_gemm(P, G, xq, a, rs, out_dtype=torch.int32)
        cases.append((xd, gd, P, G, ref, torch.empty_like(ref)))
    for xd, gd, P, G, ref, y in cases:
        bl.bitnet_bitlinear_gemm_stream_k(xd, P, G, gd, EPS_RMS, y=y, workspace=ws)
        assert torch.equal(y, ref)
    s = torch.cuda.Stream(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for xd, gd, P, G, ref, y in cases:
            bl.bitnet_bitlinear_gemm_stream_k(xd, P, G, gd, EPS_RMS, y=y, workspace=ws)
    for _ in range(3):
        for *_, y in cases:
            y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for xd, gd, P, G, ref, y in cases:
            assert torch.equal(y, ref)
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
