"""The C ABI library: it loads on a machine without a GPU, exports every
entry point include/bitnet.h declares, and rejects bad arguments on the
host before touching CUDA (every call below fails validation, so nothing is
launched and no CUDA call is made)."""
import ctypes

import pytest

import bitlinear_absmean_ternary_b200 as bl
from bitlinear_absmean_ternary_b200 import build as blbuild


@pytest.fixture(scope="module")
def L():
    blbuild.build()
    return bl.lib()


def test_every_declared_symbol_is_exported(L):
    names = bl.declared_functions()
    assert set(names) >= {"bitnet_pack_weights", "bitnet_quant_act", "bitnet_linear_gemv", "bitnet_linear_gemm",
                          "bitnet_pack_workspace_bytes", "bitnet_get_device_status", "bitnet_status_string"}
    for n in names:
        assert hasattr(L, n), n


def test_every_declared_entry_point_has_a_same_named_binding(L):
    names = bl.declared_functions()
    assert {"bitnet_b3_row_bytes", "bitnet_pack_weights_b3", "bitnet_bitlinear_gemv_b3", "bitnet_bitlinear_ffn_gemv",
            "bitnet_ste_backward_input", "bitnet_ste_backward_weight"} <= set(names)
    for n in names:
        assert callable(getattr(bl, n, None)), n


def test_status_strings(L):
    for code in range(6):
        s = bl.status_string(code)
        assert s and s != "unknown status"
    assert bl.status_string(99) == "unknown status"


def test_workspace_bytes(L):
    assert bl.bitnet_pack_workspace_bytes(0, 64) == 0
    for N in (1, 7, 2560, 21504):
        b = bl.bitnet_pack_workspace_bytes(N, 2560)
        assert b >= 8 * N + 8 and b % 256 == 0


FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced: validation fails first
MIS = FAKE + 4   # misaligned for 16-byte rules


def pack(L, W=FAKE, N=4, K=64, eps=1e-5, out=FAKE, g=FAKE, ws=FAKE, wsb=1 << 20):
    return L.bitnet_pack_weights(W, N, K, eps, out, g, ws, wsb, None)


def test_pack_rejects_bad_arguments(L):
    assert pack(L, W=None) == bl.BITNET_ERR_INVALID_ARG
    assert pack(L, out=None) == bl.BITNET_ERR_INVALID_ARG
    assert pack(L, W=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert pack(L, eps=0.0) == bl.BITNET_ERR_INVALID_ARG
    assert pack(L, eps=-1.0) == bl.BITNET_ERR_INVALID_ARG
    assert pack(L, eps=float("nan")) == bl.BITNET_ERR_INVALID_ARG
    assert pack(L, K=100) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert pack(L, K=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert pack(L, N=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert pack(L, wsb=16) == bl.BITNET_ERR_INVALID_ARG


def quant(L, x=FAKE, dt=bl.BITNET_BF16, M=2, K=64, g=None, eps=1e-5, xq=FAKE, a=FAKE, rs=None):
    return L.bitnet_quant_act(x, dt, M, K, g, eps, xq, a, rs, None)


def test_quant_rejects_bad_arguments(L):
    assert quant(L, x=None) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, a=None) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, x=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, dt=bl.BITNET_I32) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, dt=7) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, g=FAKE, eps=0.0) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, rs=FAKE + 2) == bl.BITNET_ERR_INVALID_ARG
    assert quant(L, K=96) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert quant(L, M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert quant(L, K=32768 + 64) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert quant(L, dt=bl.BITNET_F32, K=16384 + 64) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("name", ["bitnet_linear_gemv", "bitnet_linear_gemm"])
def test_linear_rejects_bad_arguments(L, name):
    fn = getattr(L, name)

    def call(W=FAKE, g=FAKE, N=8, K=64, xq=FAKE, a=FAKE, rs=None, M=1, y=FAKE, yd=bl.BITNET_BF16, ws=None, wsb=0):
        if name == "bitnet_linear_gemm":
            return fn(W, g, N, K, xq, a, rs, M, y, yd, ws, wsb, None)
        return fn(W, g, N, K, xq, a, rs, M, y, yd, None)

    assert call(W=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(g=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(y=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(W=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert call(y=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert call(g=FAKE + 1) == bl.BITNET_ERR_INVALID_ARG
    assert call(yd=5) == bl.BITNET_ERR_INVALID_ARG
    assert call(K=32) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(K=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(N=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(N=1 << 31) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    if name == "bitnet_linear_gemv":
        assert call(M=9) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    else:
        need = bl.bitnet_linear_gemm_workspace_bytes(16, 8, 64)
        assert call(ws=MIS, wsb=need) == bl.BITNET_ERR_INVALID_ARG      # misaligned workspace
        assert call(M=16, ws=FAKE, wsb=need - 16) == bl.BITNET_ERR_INVALID_ARG  # workspace too small


def test_gemm_workspace_bytes(L):
    # one flag per SM (rounded to 256 bytes) and one int32 slot of 128 rows x 64 tokens per SM, the same
    # for every M <= 64 (calls of different token counts share one workspace)
    sms = [bl.bitnet_linear_gemm_workspace_bytes(m, 256, 256) for m in (1, 16, 17, 32, 33, 64)]
    assert len(set(sms)) == 1
    assert sms[0] > 0 and sms[0] % 256 == 0
    assert bl.bitnet_linear_gemm_workspace_bytes(65, 256, 256) == 0
    assert bl.bitnet_linear_gemm_workspace_bytes(0, 256, 256) == 0
    assert bl.bitnet_linear_gemm_workspace_bytes(8, 256, 100) == 0
    assert sms[0] >= 64 * 128 * 4


def test_upgate_rejects_bad_arguments(L):
    need = bl.bitnet_linear_upgate_workspace_bytes(64, 128, 256)
    assert need == bl.bitnet_linear_gemm_workspace_bytes(64, 128, 256) and need > 0
    assert bl.bitnet_linear_upgate_workspace_bytes(2048, 128, 256) == need      # token tiles of 64 at any M
    assert bl.bitnet_linear_upgate_workspace_bytes(4, 128, 100) == 0

    def call(Wu=FAKE, gu=FAKE, Wg=FAKE, gg=FAKE, F=128, K=256, xq=FAKE, a=FAKE, rs=None, M=4, h=FAKE, ws=FAKE,
             wsb=1 << 24):
        return L.bitnet_linear_upgate_gemm(Wu, gu, Wg, gg, F, K, xq, a, rs, M, h, ws, wsb, None)

    for kw in ({"Wu": None}, {"gg": None}, {"xq": None}, {"h": None}, {"ws": None}):
        assert call(**kw) == bl.BITNET_ERR_INVALID_ARG, kw
    for kw in ({"Wg": MIS}, {"h": MIS}, {"ws": MIS}, {"gu": FAKE + 2}, {"rs": FAKE + 1}):
        assert call(**kw) == bl.BITNET_ERR_INVALID_ARG, kw
    assert call(wsb=16) == bl.BITNET_ERR_INVALID_ARG
    assert call(K=96) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(F=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_fused_gemm_rejects_bad_arguments(L):
    need = bl.bitnet_bitlinear_gemm_workspace_bytes(16, 256, 512)
    assert need > bl.bitnet_linear_gemm_workspace_bytes(16, 256, 512)   # + barrier, scales, x_q
    assert bl.bitnet_bitlinear_gemm_workspace_bytes(65, 256, 512) == 0
    assert bl.bitnet_bitlinear_gemm_workspace_bytes(4, 256, 100) == 0

    def call(x=FAKE, dt=bl.BITNET_BF16, g=None, eps=1e-5, W=FAKE, gam=FAKE, N=256, K=512, M=16, y=FAKE,
             yd=bl.BITNET_BF16, ws=FAKE, wsb=1 << 30):
        return L.bitnet_bitlinear_gemm(x, dt, g, eps, W, gam, N, K, M, y, yd, ws, wsb, None)

    for kw in ({"x": None}, {"W": None}, {"gam": None}, {"y": None}, {"ws": None}):
        assert call(**kw) == bl.BITNET_ERR_INVALID_ARG, kw
    for kw in ({"x": MIS}, {"W": MIS}, {"ws": MIS}, {"g": MIS}, {"gam": FAKE + 2}):
        assert call(**kw) == bl.BITNET_ERR_INVALID_ARG, kw
    assert call(dt=bl.BITNET_I32) == bl.BITNET_ERR_INVALID_ARG
    assert call(yd=7) == bl.BITNET_ERR_INVALID_ARG
    assert call(g=FAKE, eps=0.0) == bl.BITNET_ERR_INVALID_ARG
    assert call(wsb=need - 16) == bl.BITNET_ERR_INVALID_ARG
    assert call(M=65) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(K=96) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(dt=bl.BITNET_F32, K=16384 + 64) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_fused_rejects_bad_arguments(L):
    def call(x=FAKE, dt=bl.BITNET_BF16, g=None, eps=1e-5, W=FAKE, gam=FAKE, N=8, K=64, M=1, y=FAKE,
             yd=bl.BITNET_BF16):
        return L.bitnet_bitlinear_gemv(x, dt, g, eps, W, gam, N, K, M, y, yd, None)

    assert call(x=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(W=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert call(dt=bl.BITNET_I32) == bl.BITNET_ERR_INVALID_ARG
    assert call(yd=9) == bl.BITNET_ERR_INVALID_ARG
    assert call(g=FAKE, eps=0.0) == bl.BITNET_ERR_INVALID_ARG
    assert call(M=9) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=2, K=21504) == bl.BITNET_ERR_UNSUPPORTED_SHAPE  # quantised rows must fit in shared memory
    assert call(K=100) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(N=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_fused_host_rejects_bad_arguments_before_any_copy(L):
    def call(xh=FAKE, x=FAKE, dt=bl.BITNET_BF16, g=None, eps=1e-5, W=FAKE, gam=FAKE, N=8, K=64, M=1, y=FAKE,
             yh=FAKE, yd=bl.BITNET_BF16):
        return L.bitnet_bitlinear_gemv_host(xh, x, dt, g, eps, W, gam, N, K, M, y, yh, yd, None)

    assert call(xh=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(yh=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(x=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(x=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert call(yd=9) == bl.BITNET_ERR_INVALID_ARG
    assert call(g=FAKE, eps=float("nan")) == bl.BITNET_ERR_INVALID_ARG
    assert call(M=9) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=2, K=21504) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_ffn_rejects_bad_arguments(L):
    def call(x=FAKE, dt=bl.BITNET_BF16, M=1, D=64, F=128, gi=None, ei=1e-5, Wu=FAKE, gu=FAKE, Wg=FAKE, gg=FAKE,
             gs=None, es=1e-5, Wd=FAKE, gd=FAKE, h=FAKE, y=FAKE, yd=bl.BITNET_BF16, sync=FAKE):
        return L.bitnet_bitlinear_ffn_gemv(x, dt, M, D, F, gi, ei, Wu, gu, Wg, gg, gs, es, Wd, gd, h, y, yd, sync,
                                           None)

    for kw in ({"x": None}, {"Wu": None}, {"gg": None}, {"Wd": None}, {"h": None}, {"y": None}, {"sync": None}):
        assert call(**kw) == bl.BITNET_ERR_INVALID_ARG, kw
    for kw in ({"x": MIS}, {"Wg": MIS}, {"h": MIS}, {"gi": MIS}, {"sync": FAKE + 4}, {"gd": FAKE + 2}):
        assert call(**kw) == bl.BITNET_ERR_INVALID_ARG, kw
    assert call(dt=bl.BITNET_F32) == bl.BITNET_ERR_INVALID_ARG  # bf16 activations only
    assert call(yd=7) == bl.BITNET_ERR_INVALID_ARG
    assert call(gi=FAKE, ei=0.0) == bl.BITNET_ERR_INVALID_ARG
    assert call(gs=FAKE, es=float("inf")) == bl.BITNET_ERR_INVALID_ARG
    assert call(M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=9) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(D=96) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(F=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(F=24576 + 64) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    # the quantised rows of h (8 x 24576 bytes) do not fit beside a 2-slot ring
    assert call(M=8, F=24576) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_b3_rejects_bad_arguments(L):
    assert bl.bitnet_b3_row_bytes(2560) == 512 and bl.bitnet_b3_row_bytes(6912) == 1392
    assert bl.bitnet_b3_row_bytes(64) == 16 and bl.bitnet_b3_row_bytes(100) == 0
    assert L.bitnet_pack_weights_b3(None, 4, 64, 1e-5, FAKE, FAKE, FAKE, 1 << 20, None) == bl.BITNET_ERR_INVALID_ARG
    assert L.bitnet_pack_weights_b3(FAKE, 4, 64, 0.0, FAKE, FAKE, FAKE, 1 << 20, None) == bl.BITNET_ERR_INVALID_ARG
    assert L.bitnet_pack_weights_b3(FAKE, 4, 96, 1e-5, FAKE, FAKE, FAKE, 1 << 20, None) == \
        bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_pack_weights_b3(FAKE, 4, 64, 1e-5, FAKE, FAKE, FAKE, 8, None) == bl.BITNET_ERR_INVALID_ARG

    def call(x=FAKE, dt=bl.BITNET_BF16, g=None, eps=1e-5, W=FAKE, gam=FAKE, N=8, K=64, M=1, y=FAKE,
             yd=bl.BITNET_BF16):
        return L.bitnet_bitlinear_gemv_b3(x, dt, g, eps, W, gam, N, K, M, y, yd, None)

    assert call(x=None) == bl.BITNET_ERR_INVALID_ARG
    assert call(W=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert call(dt=bl.BITNET_I32) == bl.BITNET_ERR_INVALID_ARG
    assert call(g=FAKE, eps=-1.0) == bl.BITNET_ERR_INVALID_ARG
    assert call(M=9) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(K=100) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert call(M=2, K=21504) == bl.BITNET_ERR_UNSUPPORTED_SHAPE  # 2 x 21520 padded rows > 24000
    assert call(dt=bl.BITNET_F32, K=8192 + 64) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_ste_rejects_bad_arguments(L):
    assert bl.bitnet_ste_weight_workspace_bytes(100, 16, 64) == (16 + 64) * 128 * 2
    assert bl.bitnet_ste_weight_workspace_bytes(0, 16, 64) == 0
    assert bl.bitnet_ste_input_workspace_bytes(100, 64) == 64 * 128 * 2
    assert bl.bitnet_ste_input_workspace_bytes(100, 96) == 0

    def dx(W=FAKE, g=FAKE, N=64, K=64, dY=FAKE, M=8, out=FAKE, od=bl.BITNET_F32, ws=FAKE, wsb=1 << 20):
        return L.bitnet_ste_backward_input(W, g, N, K, dY, M, out, od, ws, wsb, None)

    assert dx(W=None) == bl.BITNET_ERR_INVALID_ARG
    assert dx(ws=None) == bl.BITNET_ERR_INVALID_ARG
    assert dx(dY=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert dx(od=bl.BITNET_I32) == bl.BITNET_ERR_INVALID_ARG
    assert dx(wsb=64) == bl.BITNET_ERR_INVALID_ARG
    assert dx(N=60) == bl.BITNET_ERR_UNSUPPORTED_SHAPE   # dY rows must be 16-byte multiples
    assert dx(K=96) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert dx(M=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE

    def dw(dY=FAKE, xq=FAKE, a=FAKE, M=8, N=64, K=64, out=FAKE, od=bl.BITNET_F32, ws=FAKE, wsb=1 << 20):
        return L.bitnet_ste_backward_weight(dY, xq, a, M, N, K, out, od, ws, wsb, None)

    assert dw(a=None) == bl.BITNET_ERR_INVALID_ARG
    assert dw(xq=MIS) == bl.BITNET_ERR_INVALID_ARG
    assert dw(od=9) == bl.BITNET_ERR_INVALID_ARG
    assert dw(wsb=16) == bl.BITNET_ERR_INVALID_ARG
    assert dw(N=12) == bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert dw(K=0) == bl.BITNET_ERR_UNSUPPORTED_SHAPE


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(bl, "_lib", None)
    monkeypatch.setattr(bl, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        bl.lib()
