"""oq_linear_fused_static: the fused layer call for callers that cannot
allocate device memory (inference runtimes that give plug-ins no allocator,
deployments whose device memory is fixed at start-up, real-time loops where an
allocation is not allowed).  Its scratch is a fixed array the library reserves
on each GPU instead of a caller workspace.  The array serves as the fused
call's least workspace, so the call must give exactly the output of the
workspace-based oq_linear_fused given that least workspace, on two calls in a
row (the second call reuses the array the first one filled), and stay within
the parity tests' y tolerance of the oracle.

This file is collected last on purpose, so that a failure here stops a
`-x` run only after every other test has run."""

import ctypes

import numpy as np
import pytest

import oracle as O
from quantized_linear_token_b200 import workloads as W

pytestmark = pytest.mark.gpu

Y_TOL = 1e-3   # the y tolerance of the parity tests (bound-relative)


def _oracle_terms(B, layer, x, d_in, cb_a, cb_w, Wc, r):
    # the oracle's contraction of the fused route's own codes: the fp16 A
    # operand mapped back to codes (every value must be a codebook level)
    a16, s = B.oq_rotate_quantize_levels(layer, x)
    lv = (layer.a_scale * np.asarray(cb_a.levels, dtype=np.float64)).astype(np.float16).view(np.uint16)
    a = a16.cpu().numpy().view(np.uint16)
    order = np.argsort(lv)
    pos = np.minimum(np.searchsorted(lv[order], a), len(lv) - 1)
    assert np.all(lv[order][pos] == a)
    ca = order[pos]
    cw = O.unpack_codes(Wc.cpu().numpy().view(np.uint32), cb_w.bits, d_in)
    return O.linear_from_codes(ca, s.cpu().numpy().astype(np.float64), cw,
                               r.cpu().numpy().astype(np.float64), cb_a.levels, cb_w.levels)


def test_static_scratch_matches_workspace_call():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_token_b200 import build
    build.build()
    from quantized_linear_token_b200 import binding as B

    wl = W.WORKLOADS["dit_image"]
    lay = wl.layers[0]
    layer = B.oq_layer_create(lay.d_in, lay.d_out, W.ROTATION_SEED, lay.a_bits, lay.w_bits)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(W.weights(wl, lay)).cuda())
    cb_a, cb_w = O.lloyd_max(lay.d_in, lay.a_bits), O.lloyd_max(lay.d_in, lay.w_bits)
    # a batch on the CTA-pair contraction, then one on the small-batch kernel
    for call, T in enumerate((1000, 128)):
        x_np = W.activations(wl, lay.d_in, tokens=T, stream=call)
        x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).cuda()
        # below W16_MIN_T tokens the workspace the fused call asks for is its
        # least one (no decoded weights)
        assert T < B.W16_MIN_T
        ws = torch.empty((B.oq_linear_fused_workspace_size(layer, T),), dtype=torch.uint8, device="cuda")
        y_ref = B.oq_linear_fused(layer, x, Wc, r, workspace=ws)
        y_new = B.oq_linear_fused_static(layer, x, Wc, r)
        torch.cuda.synchronize()
        B.oq_poll_error(layer)
        np.testing.assert_array_equal(y_new.cpu().numpy(), y_ref.cpu().numpy(),
                                      err_msg=f"call {call}: static-scratch output differs from the workspace call")
        y_or, bound = _oracle_terms(B, layer, x, lay.d_in, cb_a, cb_w, Wc, r)
        worst = float((np.abs(y_new.cpu().numpy().astype(np.float64) - y_or) / np.where(bound > 0, bound, 1.0)).max())
        assert worst <= Y_TOL, f"call {call}: {worst:.3e} from the oracle"


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
    # 20000 tokens need 2 * 3072 + 4 bytes each (the fp16 A operand and the
    # norm), about 123 MB, more than the 16 MiB array; the call must refuse
    # before touching any buffer
    st = L.oq_linear_fused_static(layer.handle, ctypes.c_void_p(x.data_ptr()), B.OQ_DTYPE_BF16, 20000,
                                  ctypes.c_void_p(Wc.data_ptr()), ctypes.c_void_p(r.data_ptr()),
                                  ctypes.c_void_p(y.data_ptr()), None)
    assert st == 1
    assert b"static" in L.oq_last_error()
