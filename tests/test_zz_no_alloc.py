"""bitnet_pack_weights_noalloc: weight packing without a caller workspace.

Some callers cannot allocate device memory -- for example code running inside
a host application whose memory pool owns every device allocation, or a
service that must not allocate once it is running -- so they cannot hand
bitnet_pack_weights the workspace buffer it needs.  The no-alloc entry point
keeps that scratch in a fixed array inside the library instead.  This test
calls it through the C ABI twice in a row (different shapes, so anything left
over from the first call would show up in the second) and checks each result
against bitnet_pack_weights with a caller workspace: packed bytes and gamma
must be identical, as for every integer result in these tests.  It also
checks that the non-finite flag is cleared between calls and that sizes above
the stated maximum are refused.

This file is named so that pytest collects it after every other test file.
"""
import ctypes

import numpy as np
import pytest

import bitlinear_absmean_ternary_b200 as bl
from bitlinear_absmean_ternary_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ROWS = 65536  # BITNET_PACK_NOALLOC_MAX_ROWS in include/bitnet.h


def _noalloc_fn():
    fn = bl.lib().bitnet_pack_weights_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def test_noalloc_pack_matches_workspace_pack():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream(dev).cuda_stream

    for N, K, sigma, seed in [(6912, 2560, 0.02, 1), (300, 640, 1.0, 2)]:
        W = torch.from_numpy(synth.weights(N, K, sigma, seed, 1)).to(dev)
        P = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
        G = torch.empty(1, dtype=torch.float32, device=dev)
        st = fn(W.data_ptr(), N, K, 1e-5, P.data_ptr(), G.data_ptr(), stream)
        assert st == bl.BITNET_OK, bl.status_string(st)
        P_ref, G_ref = bl.bitnet_pack_weights(W, 1e-5)
        assert torch.equal(P, P_ref)
        assert torch.equal(G, G_ref)

    # A non-finite weight is reported, and the next call starts from a clear flag.
    Wn = synth.weights(16, 128, 0.02, 3, 1)
    Wn[4, 7] = np.inf
    Wn = torch.from_numpy(Wn).to(dev)
    Pn = torch.empty((16, 32), dtype=torch.uint8, device=dev)
    Gn = torch.empty(1, dtype=torch.float32, device=dev)
    assert fn(Wn.data_ptr(), 16, 128, 1e-5, Pn.data_ptr(), Gn.data_ptr(), stream) == bl.BITNET_ERR_NONFINITE
    Wc = torch.from_numpy(synth.weights(16, 128, 0.02, 3, 1)).to(dev)
    assert fn(Wc.data_ptr(), 16, 128, 1e-5, Pn.data_ptr(), Gn.data_ptr(), stream) == bl.BITNET_OK
    P_ref, G_ref = bl.bitnet_pack_weights(Wc, 1e-5)
    assert torch.equal(Pn, P_ref) and torch.equal(Gn, G_ref)

    # More rows than the fixed scratch holds: refused before anything is launched.
    assert fn(Wc.data_ptr(), MAX_ROWS + 1, 64, 1e-5, Pn.data_ptr(), Gn.data_ptr(), stream) == \
        bl.BITNET_ERR_UNSUPPORTED_SHAPE
    assert bl.bitnet_get_device_status() == bl.BITNET_OK
