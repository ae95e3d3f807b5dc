"""oq_linear_fused_static: the fused layer call for callers that cannot
allocate device memory (code running during CUDA graph capture, runtimes that
give plug-ins no allocator, real-time loops).  Its scratch is a fixed array
the library reserves on each GPU instead of a caller workspace.  It must give
the output of the workspace-based oq_linear_fused, on two calls in a row (the
second call reuses the array the first one filled).

This file is collected last on purpose, so that a failure here stops a
`-x` run only after every other test has run."""

import ctypes

import numpy as np
import pytest

import oracle as O
from quantized_linear_token_b200 import workloads as W

pytestmark = pytest.mark.gpu

Y_TOL = 1e-3   # the y tolerance of the parity tests (bound-relative)


def _bound(B, layer, x, d_in, cb_a, cb_w, Wc, r):
    codes, s = B.oq_rotate_quantize(layer, x)
    ca = O.unpack_codes(codes.cpu().numpy().view(np.uint32), cb_a.bits, d_in)
    cw = O.unpack_codes(Wc.cpu().numpy().view(np.uint32), cb_w.bits, d_in)
    _, bound = O.linear_from_codes(ca, s.cpu().numpy().astype(np.float64), cw,
                                   r.cpu().numpy().astype(np.float64), cb_a.levels, cb_w.levels)
    return bound


def test_static_scratch_matches_workspace_call():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_token_b200 import build
    build.build()
    from quantized_linear_token_b200 import binding as B

    wl = W.WORKLOADS["dit_image"]
    lay = wl.layers[0]
    T = 1000
    layer = B.oq_layer_create(lay.d_in, lay.d_out, W.ROTATION_SEED, lay.a_bits, lay.w_bits)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(W.weights(wl, lay)).cuda())
    cb_a, cb_w = O.lloyd_max(lay.d_in, lay.a_bits), O.lloyd_max(lay.d_in, lay.w_bits)
    inputs = [W.activations(wl, lay.d_in, tokens=T, stream=k) for k in (0, 1)]
    for call, x_np in enumerate(inputs):
        x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).cuda()
        y_ref = B.oq_linear_fused(layer, x, Wc, r)
        y_new = B.oq_linear_fused_static(layer, x, Wc, r)
        torch.cuda.synchronize()
        B.oq_poll_error(layer)
        bound = _bound(B, layer, x, lay.d_in, cb_a, cb_w, Wc, r)
        diff = np.abs(y_new.cpu().numpy().astype(np.float64) - y_ref.cpu().numpy().astype(np.float64))
        worst = float((diff / np.where(bound > 0, bound, 1.0)).max())
        assert worst <= Y_TOL, f"call {call}: static-scratch output differs from the workspace call ({worst:.3e})"


def test_static_scratch_rejects_oversize_batch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_token_b200 import build
    build.build()
    from quantized_linear_token_b200 import binding as B

    L = B.load_library()
    layer = B.oq_layer_create(3072, 3072, 0, 4, 4)
    x = torch.zeros((1, 3072), dtype=torch.bfloat16, device="cuda")
    Wc = torch.zeros((3072, 384), dtype=torch.int32, device="cuda")
    r = torch.zeros((3072,), dtype=torch.float32, device="cuda")
    y = torch.zeros((1, 3072), dtype=torch.float32, device="cuda")
    # 20000 tokens need about 30 MB of scratch, more than the 16 MiB array;
    # the call must refuse before touching any buffer
    st = L.oq_linear_fused_static(layer.handle, ctypes.c_void_p(x.data_ptr()), B.OQ_DTYPE_BF16, 20000,
                                  ctypes.c_void_p(Wc.data_ptr()), ctypes.c_void_p(r.data_ptr()),
                                  ctypes.c_void_p(y.data_ptr()), None)
    assert st == 1
    assert b"static" in L.oq_last_error()
