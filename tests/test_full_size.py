"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: one oq_linear_fused call with the workspace it asks for
(the weight codes decoded once into fp16 levels, then the fused kernel --
rotate-quantize producer warps inside the CTA-pair contraction -- where the
block size allows, else the rotate-quantize kernel and the contraction in
turn).  Needs a B200.

For every case, on the call's own operands (its workspace starts with the A
operand and the norms that gave y):
* y is the decoded-weight contraction of those operands, bit for bit;
* every activation code (read back from the fp16 A operand) and every norm
  against the fp64 oracle, with the bounds of tests/parity.py (codes exact
  outside a band of 1e-5/sqrt(d) around each threshold, excused mismatches
  one step and at most 1e-4 of all coordinates; norms to 4e-6);
* every decoded weight value is fp16(w_scale C_w[code]) of its weight code,
  and the weight codes and norms of 256 sampled rows against the oracle;
* y on 256 sampled token rows (all output columns) against the oracle's
  contraction of the GPU's codes (bound-relative 1e-3).
The oracle's row checks run in a pool of spawned worker processes, each
drawing its own rows from the seeded generator."""

import math
import multiprocessing as mp
import os

import numpy as np
import pytest

import oracle as O
from quantized_linear_token_b200 import workloads as W

from parity import CODE_RATE, NORM_RTOL, check_code_rows, check_codes, check_linear, to_numpy_u32

pytestmark = pytest.mark.gpu

ROWS_PER_JOB = 1024

FULL = [
    # workload, layer, tokens, gelu, stream (as the workload defines its layer inputs)
    ("dit_mlp", "up", 4608, False, 0),
    ("dit_mlp", "down", 4608, True, 1),
    ("video_dit", "proj_w4a4", 32760, False, 0),
    ("video_dit", "proj_w3a3", 32760, False, 0),
    ("stress", "w2a4", 4096, False, 0),
    ("stress", "w3a3", 4096, False, 0),
    ("stress", "w4a8", 4096, False, 0),
    ("stress", "w4a4", 75600, False, 0),
]


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


@pytest.fixture(scope="module")
def pool():
    n = max(1, min(16, (os.cpu_count() or 2) - 1))
    with mp.get_context("spawn").Pool(n) as p:
        yield p


def _levels_to_codes(a16_bits: np.ndarray, levels_f16: np.ndarray) -> np.ndarray:
    order = np.argsort(levels_f16)
    pos = np.minimum(np.searchsorted(levels_f16[order], a16_bits), len(order) - 1)
    bad = levels_f16[order][pos] != a16_bits
    assert not bad.any(), f"{int(bad.sum())} values of the A operand are no codebook level"
    return order[pos].astype(np.uint8)          # codes of up to 8 bits


@pytest.mark.parametrize("wl_key,layer_name,T,gelu,stream", FULL,
                         ids=[f"{c[0]}-{c[1]}-{c[2]}" for c in FULL])
def test_full_size_parity(env, pool, wl_key, layer_name, T, gelu, stream):
    torch, B = env
    wl = W.WORKLOADS[wl_key]
    lay = next(l for l in wl.layers if l.name == layer_name)
    d, dout = lay.d_in, lay.d_out
    assert T >= B.W16_MIN_T and dout % 256 == 0     # the decoded-weight route the benchmark times

    x_np = W.activations(wl, d, tokens=T, gelu=gelu, stream=stream)
    x_t = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).cuda()
    del x_np
    Wm = W.weights(wl, lay)
    layer = B.oq_layer_create(d, dout, W.ROTATION_SEED, lay.a_bits, lay.w_bits)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).cuda())
    # the benchmarked call, with its own workspace: it starts with the call's A
    # operand (fp16 levels [T, d], rounded up to 256 bytes) and its norms
    ws = torch.empty((B.oq_linear_fused_workspace_size(layer, T),), dtype=torch.uint8, device="cuda")
    y = B.oq_linear_fused(layer, x_t, Wc, r, workspace=ws)
    a_bytes = (T * d * 2 + 255) // 256 * 256
    a16 = ws[:T * d * 2].view(torch.float16).view(T, d)
    s = ws[a_bytes:a_bytes + 4 * T].view(torch.float32)
    w16 = B.oq_weight_levels(layer, Wc)
    # y is the decoded-weight contraction of those operands, bit for bit
    y2 = B.oq_linear_decoded(layer, a16, s, w16, r)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    del x_t
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32)), "fused y differs from its operands' contraction"
    del y2

    cb_a, cb_w = O.lloyd_max(d, lay.a_bits), O.lloyd_max(d, lay.w_bits)
    perm, h = O.rpbh_permutation(d, W.ROTATION_SEED), O.hadamard_block_size(d)

    # weights: codes and norms of sampled rows; every decoded level
    Wc_np, r_np = to_numpy_u32(Wc), r.cpu().numpy()
    w_rows = np.unique(np.concatenate([np.arange(64), np.arange(dout - 64, dout),
                                       np.random.default_rng(dout + d).choice(dout, 128, replace=False)]))
    check_codes(Wc_np[w_rows], Wm[w_rows].astype(np.float64), perm, h, cb_w, lay.w_bits, None, r_np[w_rows],
                f"{wl_key}/{layer_name} W")
    cw = O.unpack_codes(Wc_np, lay.w_bits, d)
    want = (layer.w_scale * np.asarray(cb_w.levels))[cw].astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(w16.cpu().numpy().view(np.uint16), want)
    del cw, want, w16

    # activations: every code (from the fp16 A operand) and every norm
    lv = (layer.a_scale * np.asarray(cb_a.levels)).astype(np.float16).view(np.uint16)
    s_np = s.cpu().numpy()
    jobs, codes_all = [], []
    for r0 in range(0, T, ROWS_PER_JOB):
        r1 = min(T, r0 + ROWS_PER_JOB)
        c = _levels_to_codes(a16[r0:r1].cpu().numpy().view(np.uint16), lv)
        codes_all.append(c)
        jobs.append((wl_key, layer_name, T, r0, r1, gelu, stream, c, s_np[r0:r1]))
    res = pool.map(check_code_rows, jobs)
    coords = sum(x["coords"] for x in res)
    mis = sum(x["mismatches"] for x in res)
    assert coords == T * d
    assert all(x["outside_band"] == 0 for x in res), [x for x in res if x["outside_band"]][:3]
    assert all(x["max_step"] <= 1 for x in res)
    assert mis / coords <= CODE_RATE, f"mismatch rate {mis / coords:.2e}"
    norm_rel = max(x["norm_rel"] for x in res)
    assert norm_rel <= NORM_RTOL, f"norms off by {norm_rel:.2e}"

    # y on sampled rows against the oracle's contraction of the GPU's codes
    rows = np.unique(np.concatenate([np.arange(8), np.arange(T - 8, T),
                                     np.random.default_rng(T + d).choice(T, 240, replace=False)]))
    ca = np.concatenate(codes_all).astype(np.int64)
    del codes_all
    words = O.pack_codes(ca[rows], lay.a_bits)
    lin = check_linear(y[torch.from_numpy(rows).cuda()].cpu().numpy(), words, s_np[rows], Wc_np, r_np,
                       cb_a, cb_w, d, f"{wl_key}/{layer_name} y")
    print(f"{wl_key}/{layer_name} T={T}: {coords} codes, {mis} excused mismatches ({mis / coords:.1e}), "
          f"norms {norm_rel:.1e}, y {lin}")
