"""Shared parity checks of the CUDA path against the oracle (test-side only).

Bounds:
* codes: bit-exact except where the oracle's fp64 coordinate u lies within
  1e-5/sqrt(d) of a decision threshold; such excused mismatches must be one
  code step and at most 1e-4 of all coordinates.
* s, r: the GPU sums d squares in fp32 (32 per thread sequentially, a 5-level
  shuffle tree, then up to 27 partials): relative error of the sum below
  ~64 * 2^-24, so 4e-6 relative on the norm.
* y: compared with the oracle evaluated on the GPU's own codes, norms and the
  oracle's fp64 codebooks; error measured against
  bound = s r sum_i |c_w c_a| (scale-free, defined at y ~ 0), max <= 1e-3.
"""

from __future__ import annotations

import math

import numpy as np

import oracle as O

CODE_BAND = 1e-5
CODE_RATE = 1e-4
NORM_RTOL = 4e-6
Y_TOL = 1e-3


def to_numpy_u32(t) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


def check_codes(words_gpu: np.ndarray, x64: np.ndarray, perm, h, cb, bits, signs=None, norms_gpu=None,
                label=""):
    """Compare packed GPU codes (and norms) with the oracle on the same rows."""
    d = x64.shape[1]
    codes_or, s_or, u_or = O.rotate_quantize(x64, perm, h, cb, signs)
    codes_gpu = O.unpack_codes(words_gpu, bits, d)
    mism = codes_gpu != codes_or
    n_mis = int(mism.sum())
    stats = {"coords": int(codes_or.size), "mismatches": n_mis, "rate": n_mis / codes_or.size}
    if n_mis:
        band = O.threshold_distance(u_or, cb.thresholds) < CODE_BAND / math.sqrt(d)
        outside = mism & ~band
        assert not outside.any(), (
            f"{label}: {int(outside.sum())} code mismatches outside the threshold band; first at "
            f"{np.argwhere(outside)[:3].tolist()}")
        assert np.all(np.abs(codes_gpu[mism] - codes_or[mism]) == 1), f"{label}: mismatch by more than one step"
        assert stats["rate"] <= CODE_RATE, f"{label}: mismatch rate {stats['rate']:.2e}"
    if norms_gpu is not None:
        np.testing.assert_allclose(norms_gpu, s_or, rtol=NORM_RTOL, atol=0, err_msg=f"{label}: norms")
    return codes_or, s_or, stats


def check_linear(y_gpu: np.ndarray, words_a: np.ndarray, s_gpu: np.ndarray, words_w: np.ndarray,
                 r_gpu: np.ndarray, cb_a, cb_w, d: int, label="", rows=None):
    """y from the GPU vs the oracle's contraction of the GPU's own codes."""
    ca = O.unpack_codes(words_a, cb_a.bits, d)
    cw = O.unpack_codes(words_w, cb_w.bits, d)
    if rows is not None:
        ca, s_gpu, y_gpu = ca[rows], s_gpu[rows], y_gpu[rows]
    y_or, bound = O.linear_from_codes(ca, s_gpu.astype(np.float64), cw, r_gpu.astype(np.float64),
                                      cb_a.levels, cb_w.levels)
    err = np.abs(y_gpu.astype(np.float64) - y_or)
    safe = np.where(bound > 0, bound, 1.0)
    rel = np.where(bound > 0, err / safe, err)
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= Y_TOL, f"{label}: max bound-relative error {worst:.3e} > {Y_TOL}"
    # the plain relative error |dy| / |y| is reported, not bounded: the levels
    # are irrational and the tensor cores multiply them as fp16 values (the
    # level rounding, up to ~1e-4 relative at 4 bits and ~3.5e-4 at 8 bits,
    # enters y scaled by bound / |y|, which grows without limit as y -> 0)
    rms = math.sqrt(float(np.mean(y_or ** 2)) + 1e-300)
    plain = {}
    for name, frac in (("max_plain_rel_at_1pct_rms", 1e-2), ("max_plain_rel_at_rms", 1.0)):
        big = np.abs(y_or) >= frac * rms
        plain[name] = float((err[big] / np.abs(y_or[big])).max()) if big.any() else 0.0
    return {"max_bound_rel": worst, **plain}


def check_code_rows(job):
    """Oracle check of one block of rows of a large batch, run in a worker
    process: draws the rows of the workload again (the generator draws any row
    block on its own), rotates and quantizes them in fp64 and compares the
    GPU's codes and norms.  Returns counts for the caller to bound."""
    from quantized_linear_token_b200 import workloads as W
    wl_key, layer_name, T, r0, r1, gelu, stream, codes_gpu, s_gpu = job
    wl = W.WORKLOADS[wl_key]
    lay = next(l for l in wl.layers if l.name == layer_name)
    d = lay.d_in
    x = W.activations(wl, d, tokens=T, gelu=gelu, stream=stream, rows=(r0, r1))
    x64 = O.bf16_bits_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)
    cb = O.lloyd_max(d, lay.a_bits)
    codes_or, s_or, u_or = O.rotate_quantize(x64, O.rpbh_permutation(d, W.ROTATION_SEED),
                                             O.hadamard_block_size(d), cb)
    mism = codes_gpu.astype(np.int64) != codes_or
    n_mis = int(mism.sum())
    outside = 0
    max_step = 0
    if n_mis:
        band = O.threshold_distance(u_or[mism], cb.thresholds) < CODE_BAND / math.sqrt(d)
        outside = int((~band).sum())
        max_step = int(np.abs(codes_gpu.astype(np.int64)[mism] - codes_or[mism]).max())
    norm_rel = float(np.max(np.abs(s_gpu.astype(np.float64) - s_or) / np.where(s_or > 0, s_or, 1.0)))
    return {"rows": (r0, r1), "coords": int(codes_or.size), "mismatches": n_mis, "outside_band": outside,
            "max_step": max_step, "norm_rel": norm_rel}
