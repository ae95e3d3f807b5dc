"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs (bounds in tests/parity.py).  Needs a B200."""

import math

import numpy as np
import pytest

import oracle as O
from quantized_linear_token_b200 import workloads as W

from parity import check_codes, check_linear, to_numpy_u32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_token_b200 import build
    build.build()
    from quantized_linear_token_b200 import binding as B
    B.load_library()
    return torch, B


def _x_tensor(torch, x_np):
    if x_np.dtype == np.uint16:
        return torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).cuda(), O.bf16_bits_to_f64(x_np)
    return torch.from_numpy(x_np).cuda(), x_np.astype(np.float64)


def _check_fused_operands(env, layer, x_t, Wc, r, x64, perm, h, signs, cb_a, cb_w, a_bits, d_in, Wc_np, r_np,
                          y_rows, label):
    """The fused call checked on its own operands: the A operand in its
    workspace holds fp16 codebook levels whose codes and norms meet the
    oracle's bounds, y meets the oracle on those codes, and y is the
    decoded-weight contraction of those operands bit for bit."""
    torch, B = env
    yf, a16, s = fused_with_operands(env, layer, x_t, Wc, r)
    lv = (layer.a_scale * np.asarray(cb_a.levels, dtype=np.float64)).astype(np.float16).view(np.uint16)
    c16 = levels_to_codes(a16, lv, label + " fused levels")
    words = O.pack_codes(c16, a_bits)
    check_codes(words, x64, perm, h, cb_a, a_bits, signs, s, label + " fused x")
    check_linear(yf.cpu().numpy(), words, s, Wc_np, r_np, cb_a, cb_w, d_in, label + " fused y", rows=y_rows)
    a16_t = torch.from_numpy(a16.view(np.int16)).view(torch.float16).cuda()
    y_dec = B.oq_linear_decoded(layer, a16_t, torch.from_numpy(s).cuda(), B.oq_weight_levels(layer, Wc), r)
    torch.cuda.synchronize()
    assert torch.equal(yf.view(torch.int32), y_dec.view(torch.int32)), label + ": fused y is not its operands'"
    return yf.cpu().numpy()


def _run_layer(env, d_in, d_out, a_bits, w_bits, x_np, Wm, flags=0, seed=0, w_rows=None, y_rows=None,
               label=""):
    torch, B = env
    layer = B.oq_layer_create(d_in, d_out, seed, a_bits, w_bits, flags)
    gauss = bool(flags & B.OQ_FLAG_GAUSSIAN_MARGINAL)
    cb_a, cb_w = O.lloyd_max(d_in, a_bits, gauss), O.lloyd_max(d_in, w_bits, gauss)
    h = O.hadamard_block_size(d_in)
    perm = O.rpbh_permutation(d_in, seed)
    signs = O.rademacher_signs(d_in, seed) if flags & B.OQ_FLAG_SIGNS else None
    np.testing.assert_array_equal(layer.perm().astype(np.int64), perm)

    x_t, x64 = _x_tensor(torch, x_np)
    W_t = torch.from_numpy(Wm).cuda()
    Wc, r = B.oq_weight_prepare(layer, W_t)
    codes, s = B.oq_rotate_quantize(layer, x_t)
    y = B.oq_linear(layer, codes, s, Wc, r)
    yf = B.oq_linear_fused(layer, x_t, Wc, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)

    # weight rows (sampled for large layers)
    wr = np.arange(d_out) if w_rows is None else w_rows
    Wc_np, r_np = to_numpy_u32(Wc), r.cpu().numpy()
    check_codes(Wc_np[wr], Wm[wr].astype(np.float64), perm, h, cb_w, w_bits, signs, r_np[wr], label + " W")
    # activations, all rows
    codes_np, s_np = to_numpy_u32(codes), s.cpu().numpy()
    _, _, st = check_codes(codes_np, x64, perm, h, cb_a, a_bits, signs, s_np, label + " x")
    # contraction on the GPU's own codes
    y_np, yf_np = y.cpu().numpy(), yf.cpu().numpy()
    lin = check_linear(y_np, codes_np, s_np, Wc_np, r_np, cb_a, cb_w, d_in, label + " y", rows=y_rows)
    if x_np.dtype == np.uint16 and d_out % 256 == 0:
        # fp16-level route: its rotate-quantize kernel may be the tensor-core
        # FWHT one (h = 1024), whose fp32 rounding differs from the code
        # route's, so its codes are checked against the oracle on their own;
        # the fused call runs that route and gives its y bit for bit
        y2 = _check_level_stages(env, layer, x_t, Wc, r, x64, perm, h, signs, cb_a, a_bits, d_in,
                                 Wc_np, r_np, cb_w, y_rows, label)
        if fused_kernel_cc(d_in, d_out, x_np.shape[0], flags):
            # the fused kernel's own transform: checked on its own operands
            _check_fused_operands(env, layer, x_t, Wc, r, x64, perm, h, signs, cb_a, cb_w, a_bits, d_in, Wc_np,
                                  r_np, y_rows, label)
        else:
            np.testing.assert_array_equal(yf_np, y2)
    else:
        # the fused call computes the code route's codes, so the same y
        _same_y(yf_np, y_np, codes_np, s_np, Wc_np, r_np, cb_a, cb_w, d_in, T_small=False,
                label=label + " fused", rows=y_rows)
    return st, lin


SKINNY_MAX_T = 256   # batches up to this size take the small-batch kernel on the fp16-level route
W16_MIN_T = 1024     # from this many tokens the fused call decodes the weights once


def fused_with_operands(env, layer, x_t, Wc, r, y_dtype=None):
    """The fused call with its own workspace, which on the fp16-level route
    starts with the call's A operand (fp16 levels [T, d_in], rounded up to 256
    bytes) and its norms [T] (the layout the header gives).  Returns (y, a16
    bits as uint16 [T, d_in], s)."""
    torch, B = env
    T, d = x_t.shape
    ws = torch.empty((B.oq_linear_fused_workspace_size(layer, T),), dtype=torch.uint8, device=x_t.device)
    y = B.oq_linear_fused(layer, x_t, Wc, r, workspace=ws, y_dtype=y_dtype)
    torch.cuda.synchronize()
    a_bytes = (T * d * 2 + 255) // 256 * 256
    a16 = ws[:T * d * 2].cpu().numpy().view(np.uint16).reshape(T, d)
    s = ws[a_bytes:a_bytes + 4 * T].cpu().numpy().view(np.float32).copy()
    return y, a16, s


def fused_kernel_cc(d_in, d_out, T, flags, x_bf16=True):
    """Whether the fused call runs the fused kernel with the block transform
    on the CUDA cores (h = 1024), whose rounding differs from the stand-alone
    rotate-quantize kernel's."""
    h = d_in & -d_in
    return (x_bf16 and d_out % 256 == 0 and d_out <= d_in and T >= W16_MIN_T and h == 1024 and d_in // h <= 8
            and not flags & 1)


def _same_y(y_new, y_ref, codes_np, s_np, Wc_np, r_np, cb_a, cb_w, d_in, T_small, label, rows=None):
    if not T_small:
        np.testing.assert_array_equal(y_new, y_ref)
        return
    check_linear(y_new, codes_np, s_np, Wc_np, r_np, cb_a, cb_w, d_in, label, rows=rows)
    _, bound = O.linear_from_codes(O.unpack_codes(codes_np, cb_a.bits, d_in), s_np.astype(np.float64),
                                   O.unpack_codes(Wc_np, cb_w.bits, d_in), r_np.astype(np.float64),
                                   cb_a.levels, cb_w.levels)
    diff = np.abs(y_new.astype(np.float64) - y_ref.astype(np.float64))
    assert float((diff / np.where(bound > 0, bound, 1.0)).max()) <= 1e-5, label


def levels_to_codes(a16_bits: np.ndarray, levels_f16: np.ndarray, label: str) -> np.ndarray:
    """Codes of an fp16 level operand: every value must be one of the
    codebook's fp16 levels (which are distinct)."""
    order = np.argsort(levels_f16)
    pos = np.searchsorted(levels_f16[order], a16_bits)
    pos = np.minimum(pos, len(order) - 1)
    ok = levels_f16[order][pos] == a16_bits
    assert ok.all(), f"{label}: {int((~ok).sum())} values that are no codebook level"
    return order[pos].astype(np.int64)


def _check_level_stages(env, layer, x_t, Wc, r, x64, perm, h, signs, cb_a, a_bits, d_in, Wc_np, r_np, cb_w,
                        y_rows, label):
    """The fused call's fp16 route as two calls: the A operand holds exactly
    the fp16 value of a_scale times the level of a code, those codes and the
    norms match the oracle (same bounds as the code route), and the
    contraction of the operand matches the oracle on those codes.  Returns
    the route's y."""
    torch, B = env
    a16, s2 = B.oq_rotate_quantize_levels(layer, x_t)
    y2 = B.oq_linear_levels(layer, a16, s2, Wc, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    lv = (layer.a_scale * np.asarray(cb_a.levels, dtype=np.float64)).astype(np.float16).view(np.uint16)
    c16 = levels_to_codes(a16.cpu().numpy().view(np.uint16), lv, label + " levels")
    words16, s2_np = O.pack_codes(c16, a_bits), s2.cpu().numpy()
    check_codes(words16, x64, perm, h, cb_a, a_bits, signs, s2_np, label + " levels x")
    y2_np = y2.cpu().numpy()
    check_linear(y2_np, words16, s2_np, Wc_np, r_np, cb_a, cb_w, d_in, label + " levels y", rows=y_rows)
    # the split-K small-batch path adds its splits in a fixed order: repeat
    # calls give the same bits
    y3 = B.oq_linear_levels(layer, a16, s2, Wc, r)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y3.cpu().numpy(), y2_np)
    _check_decoded(env, layer, a16, s2, Wc, r, words16, s2_np, y2_np, d_in, Wc_np, r_np, cb_a, cb_w, y_rows, label)
    return y2_np


def _check_decoded(env, layer, a16, s, Wc, r, codes_np, s_np, y_np, d_in, Wc_np, r_np, cb_a, cb_w, y_rows, label):
    """The decode-then-contract route: the weights' fp16 levels hold exactly
    fp16(w_scale C_w[code]), and the contraction of the two fp16 operands gives
    the y of oq_linear_levels on the same A operand (the same MMAs in the same
    order on CTA pairs; to fp32 summation order against the small-batch
    kernel)."""
    torch, B = env
    w16 = B.oq_weight_levels(layer, Wc)
    y4 = B.oq_linear_decoded(layer, a16, s, w16, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    c = O.unpack_codes(Wc_np, cb_w.bits, d_in)
    want = (layer.w_scale * np.asarray(cb_w.levels, dtype=np.float64))[c].astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(w16.cpu().numpy().view(np.uint16), want)
    _same_y(y4.cpu().numpy(), y_np, codes_np, s_np, Wc_np, r_np, cb_a, cb_w, d_in,
            T_small=codes_np.shape[0] <= SKINNY_MAX_T, label=label + " decoded", rows=y_rows)


CASES = [
    # key,        d_in,  d_out, a, w, T,   recipe source
    ("pr1", 256, 256, 4, 4, 64),
    ("dit_image", 3072, 3072, 4, 4, 300),
    ("dit_mlp_up", 3072, 12288, 4, 2, 200),
    ("dit_mlp_down", 12288, 3072, 4, 2, 130),
    ("video_w4a4", 5120, 5120, 4, 4, 150),
    ("video_w3a3", 5120, 5120, 3, 3, 150),
    ("stress_w2a4", 13824, 5120, 4, 2, 129),
    ("stress_w3a3", 13824, 5120, 3, 3, 129),
    ("stress_w4a4", 13824, 5120, 4, 4, 129),
    ("stress_w4a8", 13824, 5120, 8, 4, 129),
]


def _inputs(key, d_in, d_out, T):
    if key == "pr1":
        wl = W.WORKLOADS["pr1"]
        return W.activations(wl, d_in, T), W.weights(wl, wl.layers[0])
    if key.startswith("dit_image"):
        wl = W.WORKLOADS["dit_image"]
        return W.activations(wl, d_in, T), W.weights(wl, wl.layers[0])
    if key.startswith("dit_mlp"):
        wl = W.WORKLOADS["dit_mlp"]
        lay = wl.layers[0] if key.endswith("up") else wl.layers[1]
        return W.activations(wl, d_in, T, gelu=key.endswith("down"), stream=int(key.endswith("down"))), \
            W.weights(wl, lay)
    if key.startswith("video"):
        wl = W.WORKLOADS["video_dit"]
        lay = wl.layers[0] if key.endswith("w4a4") else wl.layers[1]
        return W.activations(wl, d_in, T), W.weights(wl, lay)
    wl = W.WORKLOADS["stress"]
    lay = [l for l in wl.layers if key.endswith(l.name)][0]
    return W.activations(wl, d_in, T), W.weights(wl, lay)


@pytest.mark.parametrize("key,d_in,d_out,a_bits,w_bits,T", CASES, ids=[c[0] for c in CASES])
def test_workload_parity(env, key, d_in, d_out, a_bits, w_bits, T):
    x_np, Wm = _inputs(key, d_in, d_out, T)
    rng = np.random.default_rng(7)
    w_rows = None if d_out <= 1024 else np.unique(np.concatenate(
        [np.arange(64), np.arange(d_out - 64, d_out), rng.choice(d_out, 128, replace=False)]))
    st, lin = _run_layer(env, d_in, d_out, a_bits, w_bits, x_np, Wm, w_rows=w_rows, label=key)
    print(key, st, lin)


EDGE = [
    # d_in, d_out, a, w, T, flags
    (32, 16, 4, 4, 1, 0),          # h = 32, one block, one token
    (96, 48, 2, 2, 37, 0),         # h = 32, k = 3, single-pass kernel, ragged everything
    (192, 80, 3, 3, 129, 0),       # h = 64, k = 3, ragged N (80)
    (128, 128, 8, 4, 5, 0),        # h = 128, 8-bit activations
    (640, 272, 4, 3, 257, 1),      # h = 128, k = 5, Rademacher signs
    (1024, 256, 4, 4, 130, 2),     # Gaussian-marginal codebook
    (3072, 512, 4, 4, 96, 3),      # image-DiT width, signed RPBH and Gaussian marginal together
    (2048, 128, 4, 2, 70, 0),      # h = 2048 (64 per thread, two passes)
    (6144, 512, 3, 4, 33, 0),      # h = 2048, k = 3
    (1024, 256, 4, 4, 1, 0),       # h = 1024 tensor-core FWHT: one block, one token
    (7168, 256, 3, 3, 37, 0),      # h = 1024 tensor-core FWHT: seven blocks (warps) per row
    (5120, 768, 2, 2, 300, 0),     # h = 1024 tensor-core FWHT: 2-bit codebook
    (512, 256, 3, 3, 17, 0),       # h = 512 tensor-core FWHT (H_16 x H_32): one block
    (1536, 256, 4, 4, 130, 2),     # h = 512 tensor-core FWHT: three blocks, Gaussian-marginal codebook
]


@pytest.mark.parametrize("d_in,d_out,a_bits,w_bits,T,flags", EDGE)
def test_edge_shapes(env, d_in, d_out, a_bits, w_bits, T, flags):
    x_np = W.custom_activations(T, d_in, seed=d_in + T, outliers=min(4, d_in // 8))
    Wm = W.custom_weights(d_out, d_in, seed=d_out)
    _run_layer(env, d_in, d_out, a_bits, w_bits, x_np, Wm, flags=flags, seed=3, label=f"edge{d_in}x{d_out}")


@pytest.mark.parametrize("T", [1, 16, 64, 200, 256, 257])
def test_small_batch_sweep(env, T):
    # the small-T end of the workload sweep (d 13824 -> 5120, W4A4): up to 24
    # tokens take the GEMV kernel, up to 256 the split-K small-batch kernel,
    # 257 the CTA pair
    x_np, Wm = _inputs("stress_w4a4", 13824, 5120, T)
    rng = np.random.default_rng(11)
    w_rows = np.unique(np.concatenate([np.arange(32), rng.choice(5120, 64, replace=False)]))
    _run_layer(env, 13824, 5120, 4, 4, x_np, Wm, w_rows=w_rows, label=f"small{T}")


GEMV = [
    # d_in, d_out, a, w, T: batches of up to 24 tokens take the GEMV kernel
    # (weights streamed once, warp MMAs over one to three tiles of 8 tokens, K
    # split over a CTA's warps): every weight width, a K that is not a
    # multiple of the 128-position chunk, 8-bit activations, every tile count
    # with ragged last tiles, the largest batch it takes, and the stress layer
    # at batch 1, 8, 16 and 24 (25 tokens: the small-batch kernel)
    (96, 256, 4, 2, 3),
    (3072, 512, 4, 4, 1),
    (3072, 512, 3, 3, 8),
    (5120, 256, 4, 2, 2),
    (13824, 512, 8, 4, 5),
    (13824, 5120, 4, 4, 1),
    (13824, 5120, 4, 2, 8),
    (5120, 5120, 3, 3, 7),
    (96, 256, 4, 3, 9),
    (3072, 512, 4, 4, 16),
    (5120, 256, 4, 2, 21),
    (3072, 768, 3, 3, 24),
    (13824, 512, 8, 4, 23),
    (13824, 5120, 4, 4, 16),
    (13824, 5120, 4, 4, 24),
    (13824, 5120, 4, 4, 25),
]


@pytest.mark.parametrize("d_in,d_out,a_bits,w_bits,T", GEMV)
def test_gemv_batches(env, d_in, d_out, a_bits, w_bits, T):
    x_np = W.custom_activations(T, d_in, seed=d_in + 11 * T)
    Wm = W.custom_weights(d_out, d_in, seed=d_out + 13)
    _run_layer(env, d_in, d_out, a_bits, w_bits, x_np, Wm, label=f"gemv {d_in}x{d_out} T={T}")


@pytest.mark.parametrize("T", [1, 8, 24])
def test_gemv_repeats_bit_for_bit(env, T):
    # repeated calls, on the level stages and through the fused call, give
    # one y bit for bit
    torch, B = env
    d_in, d_out = 13824, 5120
    x_np, Wm = _inputs("stress_w4a4", d_in, d_out, T)
    layer = B.oq_layer_create(d_in, d_out, 0, 4, 4)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).cuda())
    x_t, _ = _x_tensor(torch, x_np)
    a16, s = B.oq_rotate_quantize_levels(layer, x_t)
    ys = [B.oq_linear_levels(layer, a16, s, Wc, r) for _ in range(3)]
    ys += [B.oq_linear_fused(layer, x_t, Wc, r) for _ in range(3)]
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int32), ys[0].view(torch.int32))


@pytest.mark.parametrize("T,d_in,d_out,w_bf16", [(2, 3072, 18432, False), (7, 1024, 256, True),
                                                   (300, 512, 384, False)])
def test_int4_weight_only_layer(env, T, d_in, d_out, w_bf16):
    # the AdaLN exception path (INT4 weight-only RTN; modulation width 6 x 3072
    # at batch 2, a bf16-weight case, and more than 256 tokens): codes and
    # scales bit-exact against the oracle (both decide in fp32), y against the
    # oracle's fp64 contraction of the same codes
    torch, B = env
    layer = B.oq_layer_create(d_in, d_out, 0, 16, 4, B.OQ_FLAG_WEIGHT_ONLY_INT4)
    Wm = W.custom_weights(d_out, d_in, seed=d_out + 1)
    if w_bf16:
        Wm = W.bf16_bits_to_f32(W.f32_to_bf16_bits(Wm))
        W_t = torch.from_numpy(Wm).cuda().to(torch.bfloat16)
    else:
        W_t = torch.from_numpy(Wm).cuda()
    Wc, r = B.oq_weight_prepare(layer, W_t)
    x_np = W.custom_activations(T, d_in, seed=T + 3)
    x_t, x64 = _x_tensor(torch, x_np)
    y = B.oq_linear_fused(layer, x_t, Wc, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    codes_or, scale_or = O.int4_rtn_weight_prepare(Wm)
    np.testing.assert_array_equal(r.cpu().numpy().view(np.uint32), scale_or.view(np.uint32))
    np.testing.assert_array_equal(O.unpack_codes(to_numpy_u32(Wc), 4, d_in), codes_or)
    y_or, bound = O.int4_rtn_linear(x64, codes_or, scale_or)
    rel = np.abs(y.cpu().numpy().astype(np.float64) - y_or) / np.where(bound > 0, bound, 1.0)
    assert float(rel.max()) <= 1e-3
    for call in (lambda: B.oq_rotate_quantize(layer, x_t), lambda: B.oq_linear(layer, Wc, r, Wc, r)):
        with pytest.raises(B.OrbitQuantError):
            call()


def _e4m3(v: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value (4 significant bits, exponent bias 7, ties to even)
    of positive or negative finite numbers inside e4m3's normal range."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(np.abs(v))                 # |v| = m 2^e, m in [0.5, 1)
    q = np.rint(m * 16.0)                      # 4 significant bits, ties to even
    return np.sign(v) * np.ldexp(q / 16.0, e)


def _fp8_levels(levels: np.ndarray) -> np.ndarray:
    """The FP8 mode's decoded levels, worked out from its definition: the
    codebook is scaled by the alpha in [8, 16) / c_max (4096 equal steps, the
    first of equally good ones) whose positive levels round to e4m3 with the
    smallest largest relative error; each level decodes to e4m3(alpha c) and
    the epilogue divides by alpha."""
    levels = np.asarray(levels, dtype=np.float64)
    pos = levels[len(levels) // 2:]
    base = 8.0 / levels[-1]
    alphas = base * (1.0 + np.arange(4096) / 4096.0)
    v = alphas[:, None] * pos[None, :]
    worst = np.max(np.abs(_e4m3(v) - v) / v, axis=1)
    alpha = alphas[int(np.argmin(worst))]
    return _e4m3(alpha * levels) / alpha


def test_fp8_contraction_mode(env):
    # the lower-precision contraction variant (a separate mode): the same codes
    # and norms as the default mode, y from e4m3 levels on kind::f8f6f4 MMAs.
    # y must equal the oracle's contraction of the same codes on the e4m3
    # levels within the default mode's 1e-3 bound; its distance from the
    # exact-level contraction (the e4m3 rounding of the levels, a few 1e-2 of
    # the bound) is reported
    torch, B = env
    d_in, d_out, T = 3072, 512, 300
    x_np, Wm = _inputs("dit_image", d_in, d_out, T)
    Wm = np.ascontiguousarray(Wm[:d_out])
    x_t, x64 = _x_tensor(torch, x_np)
    W_t = torch.from_numpy(Wm).cuda()
    ref = B.oq_layer_create(d_in, d_out, 0, 4, 4)
    f8 = B.oq_layer_create(d_in, d_out, 0, 4, 4, B.OQ_FLAG_FP8_CONTRACTION)
    Wc, r = B.oq_weight_prepare(ref, W_t)
    Wc8, r8 = B.oq_weight_prepare(f8, W_t)
    codes, s = B.oq_rotate_quantize(ref, x_t)
    codes8, s8 = B.oq_rotate_quantize(f8, x_t)
    y8 = B.oq_linear(f8, codes8, s8, Wc8, r8)
    y8f = B.oq_linear_fused(f8, x_t, Wc8, r8)
    torch.cuda.synchronize()
    B.oq_poll_error(f8)
    np.testing.assert_array_equal(to_numpy_u32(codes8), to_numpy_u32(codes))
    np.testing.assert_array_equal(to_numpy_u32(Wc8), to_numpy_u32(Wc))
    np.testing.assert_array_equal(y8f.cpu().numpy(), y8.cpu().numpy())
    cb = O.lloyd_max(d_in, 4)
    ca = O.unpack_codes(to_numpy_u32(codes), 4, d_in)
    cw = O.unpack_codes(to_numpy_u32(Wc), 4, d_in)
    s64, r64 = s.cpu().numpy().astype(np.float64), r.cpu().numpy().astype(np.float64)
    lv8 = _fp8_levels(cb.levels)
    y_or8, bound8 = O.linear_from_codes(ca, s64, cw, r64, lv8, lv8)
    y8n = y8.cpu().numpy().astype(np.float64)
    rel8 = np.abs(y8n - y_or8) / np.where(bound8 > 0, bound8, 1.0)
    assert float(rel8.max()) <= 1e-3, f"fp8 mode: {float(rel8.max()):.3e} from the e4m3-level oracle"
    y_or, bound = O.linear_from_codes(ca, s64, cw, r64, cb.levels, cb.levels)
    rel = np.abs(y8n - y_or) / np.where(bound > 0, bound, 1.0)
    yn = np.linalg.norm(y8n - y_or) / np.linalg.norm(y_or)
    print(f"fp8 mode: {float(rel8.max()):.2e} from the e4m3-level oracle; from the exact levels: "
          f"max bound-relative {rel.max():.4f}, relative l2 {yn:.4f}")
    assert float(rel.max()) < 0.05 and yn < 0.05
    with pytest.raises(B.OrbitQuantError):
        B.oq_rotate_quantize_levels(f8, x_t)


DECODED = [
    # d_in, d_out, a, w, T: ragged M and K tails, every weight width, T past
    # the fused call's switch to the decoded-weight route
    (96, 256, 4, 2, 1100),       # K = 96: a half K block of 64
    (640, 512, 3, 3, 1024),
    (3072, 768, 4, 4, 1300),
    (13824, 256, 8, 4, 1030),
]


@pytest.mark.parametrize("d_in,d_out,a_bits,w_bits,T", DECODED)
def test_decoded_weight_route(env, d_in, d_out, a_bits, w_bits, T):
    # the fused call from 1024 tokens on with its full workspace (weights
    # decoded once, both operands by TMA) against the stage calls, the codes
    # route and the oracle; with the least workspace it keeps decoding weights
    # inside the contraction
    torch, B = env
    x_np = W.custom_activations(T, d_in, seed=d_in + T)
    Wm = W.custom_weights(d_out, d_in, seed=d_out + 3)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(T - 8, T),
                                     np.random.default_rng(T).choice(T, 48, replace=False)]))
    _run_layer(env, d_in, d_out, a_bits, w_bits, x_np, Wm, w_rows=np.arange(0, d_out, 5), y_rows=rows,
               label=f"decoded {d_in}x{d_out} T={T}")
    layer = B.oq_layer_create(d_in, d_out, 0, a_bits, w_bits, 0)
    x_t, _ = _x_tensor(torch, x_np)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).cuda())
    full = B.oq_linear_fused_workspace_size(layer, T)
    assert full >= d_out * d_in * 2 + T * d_in * 2
    y_full = B.oq_linear_fused(layer, x_t, Wc, r)
    a16, s = B.oq_rotate_quantize_levels(layer, x_t)
    w16 = B.oq_weight_levels(layer, Wc)
    y_stage = B.oq_linear_decoded(layer, a16, s, w16, r)
    # the same route after its weight decode: where the block size allows, the
    # kernel that rotates, quantizes and contracts in one launch
    y_fd = B.oq_linear_fused_decoded(layer, x_t, w16, r)
    # the least workspace: the fp16 A operand (rounded up to 256 bytes) and the norms
    least = (T * d_in * 2 + 255) // 256 * 256 + T * 4
    ws = torch.empty((least,), dtype=torch.uint8, device="cuda")
    y_least = B.oq_linear_fused(layer, x_t, Wc, r, workspace=ws)
    y_lv = B.oq_linear_levels(layer, a16, s, Wc, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    np.testing.assert_array_equal(y_fd.cpu().numpy(), y_full.cpu().numpy())
    np.testing.assert_array_equal(y_least.cpu().numpy(), y_lv.cpu().numpy())
    if not fused_kernel_cc(d_in, d_out, T, 0):
        np.testing.assert_array_equal(y_full.cpu().numpy(), y_stage.cpu().numpy())
        np.testing.assert_array_equal(y_full.cpu().numpy(), y_lv.cpu().numpy())
    with pytest.raises(B.OrbitQuantError):
        B.oq_linear_fused(layer, x_t, Wc, r, workspace=ws[:least - 256])


HOST_IO = [
    # d_in, d_out, a, w, T, x dtype: several chunks with a ragged last one on
    # the decoded-weight route; one chunk below the decode threshold; a batch
    # of the small-batch kernel; fp32 x (packed-code route) over three chunks;
    # d_out not a multiple of 256 (code route, one-SM contraction)
    (3072, 768, 4, 4, 2600, "bf16"),
    (640, 512, 3, 3, 700, "bf16"),
    (1024, 256, 4, 2, 37, "bf16"),
    (256, 256, 4, 4, 2100, "f32"),
    (512, 384, 4, 4, 1500, "bf16"),
]


@pytest.mark.parametrize("d_in,d_out,a_bits,w_bits,T,xdt", HOST_IO)
def test_host_buffer_pipeline(env, d_in, d_out, a_bits, w_bits, T, xdt):
    # x and y in pinned host memory, copies overlapped with the computation
    # chunk by chunk: y equals the device-buffer fused call's y bit for bit
    torch, B = env
    x_np = W.custom_activations(T, d_in, seed=d_in + 7 * T)
    if xdt == "f32":
        x_np = W.bf16_bits_to_f32(x_np)
    Wm = W.custom_weights(d_out, d_in, seed=d_out + 11)
    layer = B.oq_layer_create(d_in, d_out, 0, a_bits, w_bits, 0)
    x_t, _ = _x_tensor(torch, x_np)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).cuda())
    y_dev = B.oq_linear_fused(layer, x_t, Wc, r)
    x_host = x_t.cpu().pin_memory()
    ys = []
    for _ in range(2):                  # a second call reuses the layer's copy streams
        y_host = torch.full((T, d_out), float("nan"), dtype=torch.float32).pin_memory()
        B.oq_linear_fused_host(layer, x_host, Wc, r, y_host)
        torch.cuda.current_stream().synchronize()
        ys.append(y_host.numpy().copy())
    B.oq_poll_error(layer)
    ref = y_dev.cpu().numpy()
    for y in ys:
        np.testing.assert_array_equal(y, ref)
    need = B.oq_linear_fused_host_workspace_size(layer, B.OQ_DTYPE_BF16 if xdt == "bf16" else B.OQ_DTYPE_F32, T)
    small = torch.empty((need - 256,), dtype=torch.uint8, device="cuda")
    with pytest.raises(B.OrbitQuantError):
        B.oq_linear_fused_host(layer, x_host, Wc, r, workspace=small)
    with pytest.raises(ValueError):
        B.oq_linear_fused_host(layer, x_t, Wc, r)


@pytest.mark.parametrize("d_in,d_out", [(256, 128), (1024, 256)])
def test_degenerate_tokens(env, d_in, d_out):
    # a zero token (s = 0, every code L/2 - 1, y = 0) and tokens with very
    # small and very large norms; d_in = 1024 takes the tensor-core FWHT on the
    # fp16-level route
    torch, B = env
    T = 6
    x = W.bf16_bits_to_f32(W.custom_activations(T, d_in, seed=5))
    x[1] = 0.0
    x[2] *= 1e-12
    x[3] *= 1e12
    x[4] = 0.0
    x[4, 17] = -3.0                      # one-hot token
    x_np = W.f32_to_bf16_bits(x)
    Wm = W.custom_weights(d_out, d_in, seed=9)
    _run_layer(env, d_in, d_out, 4, 4, x_np, Wm, label=f"degenerate {d_in}")
    layer = B.oq_layer_create(d_in, d_out, 0, 4, 4, 0)
    xt = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).cuda()
    codes, s = B.oq_rotate_quantize(layer, xt)
    c = O.unpack_codes(to_numpy_u32(codes), 4, d_in)
    assert float(s[1]) == 0.0 and np.all(c[1] == 7)
    if d_out % 256 == 0:
        a16, s2 = B.oq_rotate_quantize_levels(layer, xt)
        mid = np.float16(layer.a_scale * O.lloyd_max(d_in, 4).levels[7]).view(np.uint16)
        assert float(s2[1]) == 0.0 and np.all(a16[1].cpu().numpy().view(np.uint16) == mid)


def test_bounded_wait_timeout(env):
    # the failure path every kernel shares: a bounded wait that runs out (an
    # mbarrier nobody arrives on, 2 ms bound) sets the layer's error word and
    # returns, the kernel ends, oq_poll_error reports OQ_ERR_TIMEOUT once and
    # clears the word, and the context and the layer keep working
    torch, B = env
    x_np, Wm = _inputs("pr1", 256, 256, 64)
    layer = B.oq_layer_create(256, 256, 0, 4, 4, 0)
    B.oq_poll_error(layer)
    B.oq_check_wait_timeout(layer, 2000)
    with pytest.raises(B.OrbitQuantError) as err:
        B.oq_poll_error(layer)
    assert err.value.status == 4
    B.oq_poll_error(layer)                      # cleared
    with pytest.raises(B.OrbitQuantError):
        B.oq_check_wait_timeout(layer, 0)
    with pytest.raises(B.OrbitQuantError):
        B.oq_check_wait_timeout(layer, 2_000_000)
    _run_layer(env, 256, 256, 4, 4, x_np, Wm, label="after timeout")


def test_prepared_weight_file(env, tmp_path):
    # prepared weights saved with their layer's settings load back bit for bit
    # into a layer built the same way, give the same y, and are refused by a
    # layer with other settings or by a damaged file
    torch, B = env
    d_in, d_out, T = 1024, 256, 40
    x_np = W.custom_activations(T, d_in, seed=21)
    Wm = W.custom_weights(d_out, d_in, seed=22)
    layer = B.oq_layer_create(d_in, d_out, 5, 4, 3, 0)
    x_t, _ = _x_tensor(torch, x_np)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).cuda())
    path = str(tmp_path / "w.oqw")
    B.oq_weight_save(layer, Wc, r, path)
    again = B.oq_layer_create(d_in, d_out, 5, 4, 3, 0)
    Wc2, r2 = B.oq_weight_load(again, path)
    torch.cuda.synchronize()
    assert torch.equal(Wc2, Wc) and torch.equal(r2.view(torch.int32), r.view(torch.int32))
    np.testing.assert_array_equal(B.oq_linear_fused(again, x_t, Wc2, r2).cpu().numpy(),
                                  B.oq_linear_fused(layer, x_t, Wc, r).cpu().numpy())
    for other in (B.oq_layer_create(d_in, d_out, 6, 4, 3, 0),                    # seed
                  B.oq_layer_create(d_in, d_out, 5, 4, 4, 0),                    # weight bits
                  B.oq_layer_create(d_in, d_out, 5, 4, 3, B.OQ_FLAG_GAUSSIAN_MARGINAL),   # codebooks
                  B.oq_layer_create(d_in, 512, 5, 4, 3, 0)):                     # shape
        with pytest.raises(B.OrbitQuantError):
            B.oq_weight_load(other, path)
    raw = open(path, "rb").read()
    for bad in (raw[:-4], b"X" + raw[1:], raw + b"\0"):
        with open(path, "wb") as f:
            f.write(bad)
        with pytest.raises(B.OrbitQuantError):
            B.oq_weight_load(again, path)
    B.oq_poll_error(layer)


BF16_Y = [
    # d_in, d_out, a, w, T: the fused kernel (bf16 x, h = 1024, T >= 1024), the
    # CTA pair with weights decoded in the contraction, a small batch (which
    # takes the CTA pair for bf16 y), the one-SM kernel (d_out = 80), and the
    # packed-code route (fp32 x)
    (3072, 768, 4, 4, 1300, "bf16"),
    (2048, 512, 4, 2, 1100, "bf16"),
    (3072, 512, 4, 4, 300, "bf16"),
    (640, 512, 3, 3, 100, "bf16"),
    (192, 80, 3, 3, 129, "bf16"),
    (256, 256, 4, 4, 70, "f32"),
]


@pytest.mark.parametrize("d_in,d_out,a_bits,w_bits,T,xdt", BF16_Y)
def test_bf16_output(env, d_in, d_out, a_bits, w_bits, T, xdt):
    # y written as bf16 (round to nearest even in the epilogue): within the
    # parity bound of the oracle widened by the output rounding, |dy| <=
    # 1e-3 * bound + 2^-8 |y|; where the bf16 and fp32 calls take the same
    # kernel, bit for bit the bf16 rounding of the fp32 y; and the same through
    # the host-buffer call
    torch, B = env
    x_np = W.custom_activations(T, d_in, seed=d_in + 3 * T)
    if xdt == "f32":
        x_np = W.bf16_bits_to_f32(x_np)
    Wm = W.custom_weights(d_out, d_in, seed=d_out + 5)
    layer = B.oq_layer_create(d_in, d_out, 0, a_bits, w_bits, 0)
    x_t, x64 = _x_tensor(torch, x_np)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).cuda())
    y32 = B.oq_linear_fused(layer, x_t, Wc, r)
    y16 = B.oq_linear_fused(layer, x_t, Wc, r, y_dtype=torch.bfloat16)
    codes, s = B.oq_rotate_quantize(layer, x_t)
    y16c = B.oq_linear(layer, codes, s, Wc, r, y_dtype=torch.bfloat16)
    y32c = B.oq_linear(layer, codes, s, Wc, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    assert y16.dtype == torch.bfloat16 and y16.shape == (T, d_out)
    same_kernel = T > 256 or d_out % 256 != 0 or xdt == "f32"
    if same_kernel:
        assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
    assert torch.equal(y16c.view(torch.int16), y32c.to(torch.bfloat16).view(torch.int16))
    # against the oracle on the codes of the route that ran (the packed-code
    # kernel's codes; on the fp16-level route the fused call's operand)
    if x_np.dtype == np.uint16 and d_out % 256 == 0:
        _, a16_np, s_np = fused_with_operands(env, layer, x_t, Wc, r, y_dtype=torch.bfloat16)
        cb_a = O.lloyd_max(d_in, a_bits)
        lv = (layer.a_scale * np.asarray(cb_a.levels)).astype(np.float16).view(np.uint16)
        ca = levels_to_codes(a16_np, lv, "bf16 y")
    else:
        ca = O.unpack_codes(to_numpy_u32(codes), a_bits, d_in)
        s_np = s.cpu().numpy()
    cw = O.unpack_codes(to_numpy_u32(Wc), w_bits, d_in)
    y_or, bound = O.linear_from_codes(ca, s_np.astype(np.float64), cw, r.cpu().numpy().astype(np.float64),
                                      O.lloyd_max(d_in, a_bits).levels, O.lloyd_max(d_in, w_bits).levels)
    err = np.abs(y16.float().cpu().numpy().astype(np.float64) - y_or)
    assert np.all(err <= 1e-3 * bound + 2.0 ** -8 * np.abs(y_or) + 1e-30)
    # host buffers
    x_host = x_t.cpu().pin_memory()
    y_host = torch.empty((T, d_out), dtype=torch.bfloat16).pin_memory()
    B.oq_linear_fused_host(layer, x_host, Wc, r, y_host)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(y_host.view(torch.int16), y16.cpu().view(torch.int16))


def test_empty_batch(env):
    torch, B = env
    layer = B.oq_layer_create(256, 256, 0, 4, 4, 0)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    Wc, r = B.oq_weight_prepare(layer, torch.zeros((256, 256), device="cuda"))
    codes, s = B.oq_rotate_quantize(layer, x)
    y = B.oq_linear(layer, codes, s, Wc, r)
    assert codes.shape == (0, 32) and y.shape == (0, 256)
    B.oq_poll_error(layer)


def test_bench_config_full_size(env):
    """The image-DiT projection at its full size (9216 tokens, 3072 -> 3072,
    W4A4), in the launch configuration the benchmark times: every code and
    norm checked, y checked on 256 sampled rows."""
    torch, B = env
    wl = W.WORKLOADS["dit_image"]
    lay = wl.layers[0]
    x_np = W.activations(wl, lay.d_in)
    Wm = W.weights(wl, lay)
    rows = np.random.default_rng(0).choice(wl.tokens, 256, replace=False)
    rows.sort()
    w_rows = np.arange(0, lay.d_out, 7)
    st, lin = _run_layer(env, lay.d_in, lay.d_out, lay.a_bits, lay.w_bits, x_np, Wm, w_rows=w_rows,
                         y_rows=rows, label="dit_image full")
    print("full", st, lin)
