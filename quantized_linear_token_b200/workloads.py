"""Seeded synthetic workloads for the OrbitQuant quantized linear layer.

This module only draws inputs.  It holds none of the method's arithmetic, and
both the CUDA path (tests, bench) and the oracle (tests) take their inputs from
it.  Every array comes from numpy's Philox generator with a fixed seed, so the
same call gives the same bytes on any machine.

The pages evaluate on DiT layers of FLUX.1, Z-Image-Turbo, Wan 2.1 and
CogVideoX with the GenEval and VBench suites; none of those models or suites
is available here, so these recipes stand in for their layer shapes and for
the activation structure the pages describe (per-token scale drift across
timesteps and guidance branches, a few outlier channels).

Activations are returned as bfloat16 bit patterns (uint16, round to nearest
even) except where a recipe asks for fp32; weights are fp32 N(0, 0.02^2).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

ROTATION_SEED = 0


@dataclass(frozen=True)
class LayerShape:
    name: str
    d_in: int
    d_out: int
    a_bits: int
    w_bits: int


@dataclass(frozen=True)
class Workload:
    """One workload: a token count, one or more layers, an activation recipe."""
    key: str
    title: str
    tokens: int
    layers: tuple
    recipe: str
    data_seed: int
    x_dtype: str = "bf16"
    token_sweep: tuple = field(default_factory=tuple)


WORKLOADS = {
    "pr1": Workload(
        "pr1", "one linear layer 256->256, 64 tokens, W4A4 (fp32 activations)",
        64, (LayerShape("proj", 256, 256, 4, 4),), "gauss_outlier4x30", 1001, "fp32"),
    "dit_image": Workload(
        "dit_image", "DiT image projection 3072->3072, (4096+512) tokens x 2 CFG branches, W4A4",
        9216, (LayerShape("proj", 3072, 3072, 4, 4),), "lognormal_token_t2", 1002),
    "dit_mlp": Workload(
        "dit_mlp", "DiT MLP pair 3072->12288 (W2A4) and 12288->3072 (W2A4), 4608 tokens",
        4608, (LayerShape("up", 3072, 12288, 4, 2), LayerShape("down", 12288, 3072, 4, 2)),
        "lognormal_token_t2", 1003),
    "video_dit": Workload(
        "video_dit", "video DiT projection 5120->5120, 21x39x40 = 32760 tokens, W4A4 and W3A3",
        32760, (LayerShape("proj_w4a4", 5120, 5120, 4, 4), LayerShape("proj_w3a3", 5120, 5120, 3, 3)),
        "frame_drift", 1004),
    "stress": Workload(
        "stress", "stress 13824->5120, tokens 256/4096/32760/75600, W2A4 W3A3 W4A4 W4A8",
        75600, (LayerShape("w2a4", 13824, 5120, 4, 2), LayerShape("w3a3", 13824, 5120, 3, 3),
                LayerShape("w4a4", 13824, 5120, 4, 4), LayerShape("w4a8", 13824, 5120, 8, 4)),
        "gauss_outlier_half_pct_x100", 1005, token_sweep=(256, 4096, 32760, 75600)),
}


ROW_BLOCK = 1024   # activations are drawn in independent blocks of this many tokens


def _rng(seed: int, block: int | None = None) -> np.random.Generator:
    """Philox with a key made of the seed and (for activation rows) the row
    block, so any block can be drawn without drawing the ones before it."""
    if block is None:
        return np.random.Generator(np.random.Philox(seed))
    return np.random.Generator(np.random.Philox(key=np.array([seed, block + 1], dtype=np.uint64)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (nearest, ties to even); uint16 patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _gelu_tanh(x: np.ndarray) -> np.ndarray:
    return 0.5 * x * (1.0 + np.tanh(np.float32(0.7978845608028654) * (x + np.float32(0.044715) * x * x * x)))


def activations(wl: Workload, d: int, tokens: int | None = None, gelu: bool = False,
                stream: int = 0, rows: tuple | None = None) -> np.ndarray:
    """Draw the [tokens, d] activations of a workload, or only the rows
    [rows[0], rows[1]) of that batch (the same values).  Returns fp32 values
    for fp32 recipes and bfloat16 bit patterns (uint16) otherwise.
    ``stream`` selects an independent draw (e.g. a second layer's input).

    The recipe's outlier channels come from one generator; token rows come in
    blocks of ROW_BLOCK, each from its own generator (with the per-token
    values of its rows), so a slice of a large batch costs only its rows."""
    T = wl.tokens if tokens is None else int(tokens)
    r0, r1 = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
    if not 0 <= r0 <= r1 <= T:
        raise ValueError("rows must lie inside the batch")
    seed = wl.data_seed * 1000 + stream
    meta = _rng(seed)
    if wl.recipe == "gauss_outlier4x30":
        ch = meta.choice(d, 4, replace=False)
    elif wl.recipe == "lognormal_token_t2":
        ch = meta.choice(d, int(round(0.01 * d)), replace=False)
    elif wl.recipe == "frame_drift":
        ch = meta.choice(d, 8, replace=False)
    elif wl.recipe == "gauss_outlier_half_pct_x100":
        ch = meta.choice(d, int(round(0.005 * d)), replace=False)
    else:
        raise ValueError(wl.recipe)
    out = np.empty((r1 - r0, d), dtype=np.float32 if wl.x_dtype == "fp32" else np.uint16)
    for b in range(r0 // ROW_BLOCK, (r1 + ROW_BLOCK - 1) // ROW_BLOCK):
        b0, b1 = b * ROW_BLOCK, min((b + 1) * ROW_BLOCK, T)
        rng = _rng(seed, b)
        x = rng.standard_normal((b1 - b0, d), dtype=np.float32)
        if wl.recipe == "gauss_outlier4x30":
            x[:, ch] *= np.float32(30.0)
        elif wl.recipe == "lognormal_token_t2":
            # heavy-tailed outlier channels, then a log-normal scale per token
            x[:, ch] = rng.standard_t(2.0, size=(b1 - b0, len(ch))).astype(np.float32) * np.float32(20.0)
            x *= np.exp(rng.standard_normal((b1 - b0, 1), dtype=np.float32))
            if gelu:
                x = _gelu_tanh(x)
        elif wl.recipe == "frame_drift":
            # 21 frames of equal token counts, scale drifting from x0.5 to x4
            frames = 21
            f = (np.arange(b0, b1) * frames) // max(T, 1)
            x *= (0.5 + 3.5 * f / (frames - 1)).astype(np.float32)[:, None]
            x[:, ch] *= np.float32(50.0)
        else:
            x[:, ch] *= np.float32(100.0)
        lo, hi = max(b0, r0), min(b1, r1)
        part = x[lo - b0:hi - b0]
        out[lo - r0:hi - r0] = part if wl.x_dtype == "fp32" else f32_to_bf16_bits(part)
    return out


def weights(wl: Workload, layer: LayerShape) -> np.ndarray:
    """fp32 weights [d_out, d_in] drawn as N(0, 0.02^2)."""
    idx = [l.name for l in wl.layers].index(layer.name)
    rng = _rng(wl.data_seed * 1000 + 500 + idx)
    return (rng.standard_normal((layer.d_out, layer.d_in), dtype=np.float32) * np.float32(0.02))


def custom_activations(T: int, d: int, seed: int, outliers: int = 4, scale: float = 30.0,
                       bf16: bool = True) -> np.ndarray:
    """Gaussian activations with a few scaled outlier channels, for edge cases."""
    rng = _rng(seed)
    x = rng.standard_normal((T, d), dtype=np.float32)
    if outliers:
        ch = rng.choice(d, min(outliers, d), replace=False)
        x[:, ch] *= np.float32(scale)
    return f32_to_bf16_bits(x) if bf16 else x


def custom_weights(d_out: int, d_in: int, seed: int) -> np.ndarray:
    rng = _rng(seed)
    return rng.standard_normal((d_out, d_in), dtype=np.float32) * np.float32(0.02)
