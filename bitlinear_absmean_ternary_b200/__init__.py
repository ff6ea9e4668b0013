"""BitNet b1.58 BitLinear forward (W1.58A8) on NVIDIA B200 (sm_100a).

Python binding of the C ABI in include/bitnet.h.  Every function has the
name of the C entry point it calls and does argument marshalling only
(PyTorch tensors -> device pointers, sizes, the current CUDA stream); all of
the computation runs in the library's CUDA kernels.  There is no CPU path:
if libbitnet_b200.so is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "bitnet.h")

BITNET_OK = 0
BITNET_ERR_INVALID_ARG = 1
BITNET_ERR_UNSUPPORTED_SHAPE = 2
BITNET_ERR_NONFINITE = 3
BITNET_ERR_CUDA = 4
BITNET_ERR_TIMEOUT = 5

BITNET_F32 = 0
BITNET_BF16 = 1
BITNET_I32 = 2

BITNET_FFN_SYNC_BYTES = 64

_lib = None


class BitnetError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: status {status} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """The loaded CUDA library.  Raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m bitlinear_absmean_ternary_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, F, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
        L.bitnet_pack_workspace_bytes.argtypes = [I64, I64]
        L.bitnet_pack_workspace_bytes.restype = ctypes.c_size_t
        L.bitnet_pack_weights.argtypes = [P, I64, I64, F, P, P, P, ctypes.c_size_t, P]
        L.bitnet_pack_weights.restype = I
        L.bitnet_quant_act.argtypes = [P, I, I64, I64, P, F, P, P, P, P]
        L.bitnet_quant_act.restype = I
        L.bitnet_linear_gemv.argtypes = [P, P, I64, I64, P, P, P, I64, P, I, P]
        L.bitnet_linear_gemv.restype = I
        L.bitnet_linear_gemm.argtypes = [P, P, I64, I64, P, P, P, I64, P, I, P, ctypes.c_size_t, P]
        L.bitnet_linear_gemm.restype = I
        L.bitnet_linear_gemm_stream_k.argtypes = [P, P, I64, I64, P, P, P, I64, P, I, P, ctypes.c_size_t, P]
        L.bitnet_linear_gemm_stream_k.restype = I
        L.bitnet_linear_gemm_workspace_bytes.argtypes = [I64, I64, I64]
        L.bitnet_linear_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.bitnet_bitlinear_gemm_workspace_bytes.argtypes = [I64, I64, I64]
        L.bitnet_bitlinear_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.bitnet_bitlinear_gemm.argtypes = [P, I, P, F, P, P, I64, I64, I64, P, I, P, ctypes.c_size_t, P]
        L.bitnet_bitlinear_gemm.restype = I
        L.bitnet_bitlinear_gemm_stream_k.argtypes = [P, I, P, F, P, P, I64, I64, I64, P, I, P, ctypes.c_size_t, P]
        L.bitnet_bitlinear_gemm_stream_k.restype = I
        L.bitnet_linear_upgate_workspace_bytes.argtypes = [I64, I64, I64]
        L.bitnet_linear_upgate_workspace_bytes.restype = ctypes.c_size_t
        L.bitnet_linear_upgate_gemm.argtypes = [P, P, P, P, I64, I64, P, P, P, I64, P, P, ctypes.c_size_t, P]
        L.bitnet_linear_upgate_gemm.restype = I
        L.bitnet_bitlinear_gemv.argtypes = [P, I, P, F, P, P, I64, I64, I64, P, I, P]
        L.bitnet_bitlinear_gemv.restype = I
        L.bitnet_bitlinear_gemv_host.argtypes = [P, P, I, P, F, P, P, I64, I64, I64, P, P, I, P]
        L.bitnet_bitlinear_gemv_host.restype = I
        L.bitnet_bitlinear_ffn_gemv.argtypes = [P, I, I64, I64, I64, P, F, P, P, P, P, P, F, P, P, P, P, I, P, P]
        L.bitnet_bitlinear_ffn_gemv.restype = I
        L.bitnet_pack_weights_noalloc.argtypes = [P, I64, I64, F, P, P, P]
        L.bitnet_pack_weights_noalloc.restype = I
        L.bitnet_b3_row_bytes.argtypes = [I64]
        L.bitnet_b3_row_bytes.restype = ctypes.c_size_t
        L.bitnet_pack_weights_b3.argtypes = [P, I64, I64, F, P, P, P, ctypes.c_size_t, P]
        L.bitnet_pack_weights_b3.restype = I
        L.bitnet_bitlinear_gemv_b3.argtypes = [P, I, P, F, P, P, I64, I64, I64, P, I, P]
        L.bitnet_bitlinear_gemv_b3.restype = I
        L.bitnet_ste_input_workspace_bytes.argtypes = [I64, I64]
        L.bitnet_ste_input_workspace_bytes.restype = ctypes.c_size_t
        L.bitnet_ste_backward_input.argtypes = [P, P, I64, I64, P, I64, P, I, P, ctypes.c_size_t, P]
        L.bitnet_ste_backward_input.restype = I
        L.bitnet_ste_weight_workspace_bytes.argtypes = [I64, I64, I64]
        L.bitnet_ste_weight_workspace_bytes.restype = ctypes.c_size_t
        L.bitnet_ste_backward_weight.argtypes = [P, P, P, I64, I64, I64, P, I, P, ctypes.c_size_t, P]
        L.bitnet_ste_backward_weight.restype = I
        L.bitnet_get_device_status.argtypes = [P]
        L.bitnet_get_device_status.restype = I
        L.bitnet_status_string.argtypes = [I]
        L.bitnet_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def declared_functions() -> list:
    """Names of the entry points include/bitnet.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    try:
        return lib().bitnet_status_string(int(status)).decode()
    except Exception:  # the library itself is unavailable
        return "unknown"


def bitnet_status_string(status: int) -> str:
    """Text of a bitnet_status code."""
    return status_string(status)


def _check(fn: str, status: int) -> None:
    if status != BITNET_OK:
        raise BitnetError(fn, status)


# ----------------------------------------------------------------- marshalling

_torch_mod = None


def _torch():
    global _torch_mod
    if _torch_mod is None:
        import torch
        _torch_mod = torch
    return _torch_mod


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    """The current CUDA stream of `device` as a raw handle (the stream a torch user is launching on)."""
    torch = _torch()
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    idx = device if isinstance(device, int) else getattr(device, "index", None)
    if raw is not None and idx is not None:
        return raw(idx)  # no Stream object built per call
    return torch.cuda.current_stream(device).cuda_stream


def _dtype_code(dtype) -> int:
    torch = _torch()
    if dtype == torch.float32:
        return BITNET_F32
    if dtype == torch.bfloat16:
        return BITNET_BF16
    if dtype == torch.int32:
        return BITNET_I32
    raise ValueError(f"unsupported dtype {dtype}")


def _need_cuda(*ts) -> None:
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensor must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensor must be contiguous")


def bitnet_pack_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitnet_pack_workspace_bytes(N, K))


def bitnet_pack_weights(W, eps: float = 1e-5, W_packed=None, gamma=None, workspace=None):
    """Absmean ternarisation + 2-bit packing of fp32 W (N x K) on the GPU.

    Returns (W_packed uint8 N x K/4, gamma float32 [1]).  Synchronises.
    """
    torch = _torch()
    _need_cuda(W)
    N, K = W.shape
    if W_packed is None:
        W_packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    nbytes = bitnet_pack_workspace_bytes(N, K)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _need_cuda(W_packed, gamma, workspace)
    st = lib().bitnet_pack_weights(_ptr(W), N, K, eps, _ptr(W_packed), _ptr(gamma), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(W.device))
    _check("bitnet_pack_weights", st)
    return W_packed, gamma


def bitnet_pack_weights_noalloc(W, eps: float = 1e-5, W_packed=None, gamma=None):
    """As bitnet_pack_weights, with the library's own fixed scratch instead of a
    caller workspace (at most BITNET_PACK_NOALLOC_MAX_ROWS rows; concurrent calls
    must not overlap).  Returns (W_packed, gamma).  Synchronises."""
    torch = _torch()
    _need_cuda(W)
    N, K = W.shape
    if W_packed is None:
        W_packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    _need_cuda(W_packed, gamma)
    st = lib().bitnet_pack_weights_noalloc(_ptr(W), N, K, eps, _ptr(W_packed), _ptr(gamma), _stream(W.device))
    _check("bitnet_pack_weights_noalloc", st)
    return W_packed, gamma


def bitnet_quant_act(x, rms_gain=None, rms_eps: float = 1e-5, x_q=None, a_scale=None, x_rowsum=None,
                     want_rowsum: bool = False):
    """Fused RMSNorm (when rms_gain is given) + per-token absmax int8 quant.

    x: M x K float32 or bfloat16 on the GPU.  Returns (x_q int8, a_scale
    float32 [M], x_rowsum int32 [M] or None).  Asynchronous.
    """
    torch = _torch()
    _need_cuda(x, rms_gain)
    M, K = x.shape
    if x_q is None:
        x_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if a_scale is None:
        a_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    if x_rowsum is None and want_rowsum:
        x_rowsum = torch.empty(M, dtype=torch.int32, device=x.device)
    _need_cuda(x_q, a_scale, x_rowsum)
    st = lib().bitnet_quant_act(_ptr(x), _dtype_code(x.dtype), M, K, _ptr(rms_gain), rms_eps, _ptr(x_q),
                                _ptr(a_scale), _ptr(x_rowsum), _stream(x.device))
    _check("bitnet_quant_act", st)
    return x_q, a_scale, x_rowsum


def _linear_args(W_packed, gamma, x_q, a_scale, x_rowsum, y, out_dtype):
    torch = _torch()
    _need_cuda(W_packed, gamma, x_q, a_scale, x_rowsum, y)
    N = W_packed.shape[0]
    K = W_packed.shape[1] * 4
    M = x_q.shape[0]
    if x_q.shape[1] != K:
        raise ValueError("x_q and W_packed disagree on K")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=x_q.device)
    return M, N, K, y


def bitnet_linear_gemv(W_packed, gamma, x_q, a_scale, x_rowsum=None, y=None, out_dtype=None):
    """W1.58A8 product for M <= 8 tokens (CUDA cores).  Returns y (M x N)."""
    M, N, K, y = _linear_args(W_packed, gamma, x_q, a_scale, x_rowsum, y, out_dtype)
    st = lib().bitnet_linear_gemv(_ptr(W_packed), _ptr(gamma), N, K, _ptr(x_q), _ptr(a_scale), _ptr(x_rowsum), M,
                                  _ptr(y), _dtype_code(y.dtype), _stream(x_q.device))
    _check("bitnet_linear_gemv", st)
    return y


def bitnet_linear_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    """Workspace bytes of bitnet_linear_gemm on the current device (0 when none is used)."""
    return int(lib().bitnet_linear_gemm_workspace_bytes(M, N, K))


def bitnet_linear_gemm(W_packed, gamma, x_q, a_scale, x_rowsum=None, y=None, out_dtype=None, workspace=None,
                       stream_k=None):
    """W1.58A8 product for any M (tcgen05 tensor cores).  Returns y (M x N).

    workspace: a zeroed uint8 device tensor of bitnet_linear_gemm_workspace_bytes
    bytes, reused across calls on one stream (the calls leave it zeroed), or None
    to allocate a zeroed one for this call when M <= 64.  stream_k: None lets the
    library choose (stream-K from 12 units of work per SM when a workspace is
    given), True forces stream-K (bitnet_linear_gemm_stream_k), False passes no
    workspace (the persistent-tile path).  The results are the same."""
    torch = _torch()
    M, N, K, y = _linear_args(W_packed, gamma, x_q, a_scale, x_rowsum, y, out_dtype)
    if stream_k is False:
        workspace = None
    elif workspace is None:
        nbytes = bitnet_linear_gemm_workspace_bytes(M, N, K)
        if nbytes:
            workspace = torch.zeros(nbytes, dtype=torch.uint8, device=x_q.device)
    _need_cuda(workspace)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = lib().bitnet_linear_gemm_stream_k if stream_k else lib().bitnet_linear_gemm
    st = fn(_ptr(W_packed), _ptr(gamma), N, K, _ptr(x_q), _ptr(a_scale), _ptr(x_rowsum), M, _ptr(y),
            _dtype_code(y.dtype), _ptr(workspace), wsb, _stream(x_q.device))
    _check("bitnet_linear_gemm_stream_k" if stream_k else "bitnet_linear_gemm", st)
    return y


def bitnet_linear_gemm_stream_k(W_packed, gamma, x_q, a_scale, x_rowsum=None, y=None, out_dtype=None,
                                workspace=None):
    """bitnet_linear_gemm with the stream-K product forced (M <= 64)."""
    return bitnet_linear_gemm(W_packed, gamma, x_q, a_scale, x_rowsum, y, out_dtype, workspace, stream_k=True)


def bitnet_linear_upgate_workspace_bytes(M: int, F: int, K: int) -> int:
    """Workspace bytes of bitnet_linear_upgate_gemm on the current device."""
    return int(lib().bitnet_linear_upgate_workspace_bytes(M, F, K))


def bitnet_linear_upgate_gemm(W_up, gamma_up, W_gate, gamma_gate, x_q, a_scale, x_rowsum=None, h=None,
                              workspace=None):
    """FFN up and gate products with the squared-ReLU gate fused in the epilogue:
    h = bf16(relu(g)^2 * u), M x F.  workspace: zeroed uint8 device tensor of
    bitnet_linear_upgate_workspace_bytes bytes, reused across calls (allocated
    zeroed for this call when None).  Returns h."""
    torch = _torch()
    _need_cuda(W_up, gamma_up, W_gate, gamma_gate, x_q, a_scale, x_rowsum, h, workspace)
    F = W_up.shape[0]
    K = W_up.shape[1] * 4
    M = x_q.shape[0]
    if tuple(W_gate.shape) != tuple(W_up.shape) or x_q.shape[1] != K:
        raise ValueError("W_up, W_gate (F x K/4) and x_q (M x K) disagree")
    if h is None:
        h = torch.empty((M, F), dtype=torch.bfloat16, device=x_q.device)
    if workspace is None:
        workspace = torch.zeros(bitnet_linear_upgate_workspace_bytes(M, F, K), dtype=torch.uint8,
                                device=x_q.device)
    st = lib().bitnet_linear_upgate_gemm(_ptr(W_up), _ptr(gamma_up), _ptr(W_gate), _ptr(gamma_gate), F, K,
                                         _ptr(x_q), _ptr(a_scale), _ptr(x_rowsum), M, _ptr(h), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(x_q.device))
    _check("bitnet_linear_upgate_gemm", st)
    return h


def bitnet_bitlinear_gemv(x, W_packed, gamma, rms_gain=None, rms_eps: float = 1e-5, y=None, out_dtype=None):
    """Fused decode BitLinear (M <= 8): quantisation (with RMSNorm when
    rms_gain is given) and the ternary product in one kernel.  Returns y."""
    torch = _torch()
    _need_cuda(x, rms_gain, W_packed, gamma, y)
    M, K = x.shape
    N = W_packed.shape[0]
    if W_packed.shape[1] * 4 != K:
        raise ValueError("x and W_packed disagree on K")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=x.device)
    st = lib().bitnet_bitlinear_gemv(_ptr(x), _dtype_code(x.dtype), _ptr(rms_gain), rms_eps, _ptr(W_packed),
                                     _ptr(gamma), N, K, M, _ptr(y), _dtype_code(y.dtype), _stream(x.device))
    _check("bitnet_bitlinear_gemv", st)
    return y


def bitnet_bitlinear_gemv_host(x_host, x, W_packed, gamma, y, y_host, rms_gain=None, rms_eps: float = 1e-5):
    """bitnet_bitlinear_gemv with the tokens and the result in host memory:
    copies x_host (M x K, pinned CPU tensor) into the device tensor x, runs the
    fused kernel into y and copies y back into y_host (pinned CPU tensor), all
    on the current stream.  Synchronise the stream before reading y_host."""
    _need_cuda(x, rms_gain, W_packed, gamma, y)
    for t in (x_host, y_host):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("x_host and y_host must be contiguous host tensors")
    if x_host.shape != x.shape or x_host.dtype != x.dtype or y_host.shape != y.shape or y_host.dtype != y.dtype:
        raise ValueError("host and device buffers disagree in shape or dtype")
    M, K = x.shape
    N = W_packed.shape[0]
    if W_packed.shape[1] * 4 != K or tuple(y.shape) != (M, N):
        raise ValueError("x, W_packed and y disagree on the shape")
    st = lib().bitnet_bitlinear_gemv_host(_ptr(x_host), _ptr(x), _dtype_code(x.dtype), _ptr(rms_gain), rms_eps,
                                          _ptr(W_packed), _ptr(gamma), N, K, M, _ptr(y), _ptr(y_host),
                                          _dtype_code(y.dtype), _stream(x.device))
    _check("bitnet_bitlinear_gemv_host", st)
    return y_host


def bitnet_bitlinear_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    """Workspace bytes of bitnet_bitlinear_gemm on the current device (0 outside M = 1..64)."""
    return int(lib().bitnet_bitlinear_gemm_workspace_bytes(M, N, K))


def bitnet_bitlinear_gemm(x, W_packed, gamma, rms_gain=None, rms_eps: float = 1e-5, y=None, out_dtype=None,
                          workspace=None, stream_k=None):
    """BitLinear for 1 <= M <= 64 tokens: quantisation (with RMSNorm when
    rms_gain is given) into the workspace, then the tensor-core product
    (stream-K or tiles), two launches; stream_k=True takes the one-launch kernel
    (quantisation inside the stream-K product).  workspace: zeroed uint8 device
    tensor of bitnet_bitlinear_gemm_workspace_bytes bytes, reused across calls on
    one stream (allocated zeroed for this call when None).  Returns y (M x N)."""
    torch = _torch()
    _need_cuda(x, rms_gain, W_packed, gamma, y, workspace)
    M, K = x.shape
    N = W_packed.shape[0]
    if W_packed.shape[1] * 4 != K:
        raise ValueError("x and W_packed disagree on K")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.zeros(max(1, bitnet_bitlinear_gemm_workspace_bytes(M, N, K)), dtype=torch.uint8,
                                device=x.device)
    fn = lib().bitnet_bitlinear_gemm_stream_k if stream_k else lib().bitnet_bitlinear_gemm
    st = fn(_ptr(x), _dtype_code(x.dtype), _ptr(rms_gain), rms_eps, _ptr(W_packed), _ptr(gamma), N, K, M, _ptr(y),
            _dtype_code(y.dtype), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(x.device))
    _check("bitnet_bitlinear_gemm_stream_k" if stream_k else "bitnet_bitlinear_gemm", st)
    return y


def bitnet_bitlinear_gemm_stream_k(x, W_packed, gamma, rms_gain=None, rms_eps: float = 1e-5, y=None,
                                   out_dtype=None, workspace=None):
    """bitnet_bitlinear_gemm as one launch (quantisation inside the stream-K product)."""
    return bitnet_bitlinear_gemm(x, W_packed, gamma, rms_gain, rms_eps, y, out_dtype, workspace, stream_k=True)


def bitnet_bitlinear_ffn_gemv(x, W_up, gamma_up, W_gate, gamma_gate, W_down, gamma_down, rms_gain_in=None,
                              rms_eps_in: float = 1e-5, rms_gain_sub=None, rms_eps_sub: float = 1e-5, h=None, y=None,
                              out_dtype=None, sync=None):
    """Decode FFN block (M <= 8) in one launch: u, g = BitLinear_up/gate(x),
    h = bf16 squared-ReLU gate, y = BitLinear_down(h).  x: M x D bf16.
    sync: BITNET_FFN_SYNC_BYTES zeroed device bytes reused across calls on one
    stream (allocated per call when None).  Returns (h, y)."""
    torch = _torch()
    _need_cuda(x, W_up, gamma_up, W_gate, gamma_gate, W_down, gamma_down, rms_gain_in, rms_gain_sub, h, y, sync)
    M, D = x.shape
    F = W_up.shape[0]
    if tuple(W_up.shape) != (F, D // 4) or tuple(W_gate.shape) != (F, D // 4) or tuple(W_down.shape) != (D, F // 4):
        raise ValueError("W_up/W_gate must be F x D/4 and W_down D x F/4 packed bytes")
    if h is None:
        h = torch.empty((M, F), dtype=torch.bfloat16, device=x.device)
    if y is None:
        y = torch.empty((M, D), dtype=out_dtype or torch.bfloat16, device=x.device)
    if sync is None:
        sync = torch.zeros(BITNET_FFN_SYNC_BYTES, dtype=torch.uint8, device=x.device)
    st = lib().bitnet_bitlinear_ffn_gemv(_ptr(x), _dtype_code(x.dtype), M, D, F, _ptr(rms_gain_in), rms_eps_in,
                                         _ptr(W_up), _ptr(gamma_up), _ptr(W_gate), _ptr(gamma_gate),
                                         _ptr(rms_gain_sub), rms_eps_sub, _ptr(W_down), _ptr(gamma_down), _ptr(h),
                                         _ptr(y), _dtype_code(y.dtype), _ptr(sync), _stream(x.device))
    _check("bitnet_bitlinear_ffn_gemv", st)
    return h, y


def bitnet_b3_row_bytes(K: int) -> int:
    return int(lib().bitnet_b3_row_bytes(K))


def bitnet_pack_weights_b3(W, eps: float = 1e-5, W_b3=None, gamma=None, workspace=None):
    """Absmean ternarisation + base-3 packing (5 codes per byte) of fp32 W (N x K).
    Returns (W_b3 uint8 N x bitnet_b3_row_bytes(K), gamma float32 [1]).  Synchronises."""
    torch = _torch()
    _need_cuda(W)
    N, K = W.shape
    rb = bitnet_b3_row_bytes(K)
    if rb == 0:
        raise ValueError("K must be a positive multiple of 64")
    if W_b3 is None:
        W_b3 = torch.empty((N, rb), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    nbytes = bitnet_pack_workspace_bytes(N, K)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _need_cuda(W_b3, gamma, workspace)
    st = lib().bitnet_pack_weights_b3(_ptr(W), N, K, eps, _ptr(W_b3), _ptr(gamma), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(W.device))
    _check("bitnet_pack_weights_b3", st)
    return W_b3, gamma


def bitnet_bitlinear_gemv_b3(x, W_b3, gamma, rms_gain=None, rms_eps: float = 1e-5, y=None, out_dtype=None):
    """Fused decode BitLinear (M <= 8) on base-3 packed weights.  Returns y (M x N)."""
    torch = _torch()
    _need_cuda(x, rms_gain, W_b3, gamma, y)
    M, K = x.shape
    N = W_b3.shape[0]
    if W_b3.shape[1] != bitnet_b3_row_bytes(K):
        raise ValueError("x and W_b3 disagree on K")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=x.device)
    st = lib().bitnet_bitlinear_gemv_b3(_ptr(x), _dtype_code(x.dtype), _ptr(rms_gain), rms_eps, _ptr(W_b3),
                                        _ptr(gamma), N, K, M, _ptr(y), _dtype_code(y.dtype), _stream(x.device))
    _check("bitnet_bitlinear_gemv_b3", st)
    return y


def bitnet_ste_input_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitnet_ste_input_workspace_bytes(N, K))


def bitnet_ste_backward_input(W_packed, gamma, dY, dX=None, out_dtype=None, workspace=None):
    """STE input gradient dX = gamma * dY q (M x K), dY: M x N bf16."""
    torch = _torch()
    _need_cuda(W_packed, gamma, dY, dX, workspace)
    M, N = dY.shape
    K = W_packed.shape[1] * 4
    if W_packed.shape[0] != N:
        raise ValueError("dY and W_packed disagree on N")
    if dX is None:
        dX = torch.empty((M, K), dtype=out_dtype or torch.float32, device=dY.device)
    if workspace is None:
        workspace = torch.empty(bitnet_ste_input_workspace_bytes(N, K), dtype=torch.uint8, device=dY.device)
    st = lib().bitnet_ste_backward_input(_ptr(W_packed), _ptr(gamma), N, K, _ptr(dY), M, _ptr(dX),
                                         _dtype_code(dX.dtype), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(dY.device))
    _check("bitnet_ste_backward_input", st)
    return dX


def bitnet_ste_weight_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bitnet_ste_weight_workspace_bytes(M, N, K))


def bitnet_ste_backward_weight(dY, x_q, a_scale, dW=None, out_dtype=None, workspace=None):
    """STE weight gradient dW = bf16(dY * a)^T x_q (N x K), dY: M x N bf16."""
    torch = _torch()
    _need_cuda(dY, x_q, a_scale, dW, workspace)
    M, N = dY.shape
    K = x_q.shape[1]
    if x_q.shape[0] != M:
        raise ValueError("dY and x_q disagree on M")
    if dW is None:
        dW = torch.empty((N, K), dtype=out_dtype or torch.float32, device=dY.device)
    if workspace is None:
        workspace = torch.empty(bitnet_ste_weight_workspace_bytes(M, N, K), dtype=torch.uint8, device=dY.device)
    st = lib().bitnet_ste_backward_weight(_ptr(dY), _ptr(x_q), _ptr(a_scale), M, N, K, _ptr(dW),
                                          _dtype_code(dW.dtype), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(dY.device))
    _check("bitnet_ste_backward_weight", st)
    return dW


def bitnet_get_device_status(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device error status."""
    torch = _torch()
    dev = device if device is not None else torch.cuda.current_device()
    return int(lib().bitnet_get_device_status(_stream(dev)))


def bitlinear(x, W_packed, gamma, rms_gain=None, rms_eps: float = 1e-5, out_dtype=None):
    """One BitLinear forward: quantise x (fused RMSNorm when rms_gain is given),
    then the ternary product with dequant.  Uses the fused decode kernel for
    M <= 8 when the quantised rows fit its shared memory, the fused stream-K
    kernel for M <= 64, else the quantisation and the tensor-core product."""
    M, K = x.shape
    if M <= 8 and M * K <= 21504:
        return bitnet_bitlinear_gemv(x, W_packed, gamma, rms_gain, rms_eps, out_dtype=out_dtype)
    if M <= 64 and K <= (32768 if x.dtype == _torch().bfloat16 else 16384):
        return bitnet_bitlinear_gemm(x, W_packed, gamma, rms_gain, rms_eps, out_dtype=out_dtype)
    x_q, a, rs = bitnet_quant_act(x, rms_gain, rms_eps, want_rowsum=True)
    if x.shape[0] <= 8:
        return bitnet_linear_gemv(W_packed, gamma, x_q, a, rs, out_dtype=out_dtype)
    return bitnet_linear_gemm(W_packed, gamma, x_q, a, rs, out_dtype=out_dtype)
