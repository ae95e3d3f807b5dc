"""Plain fp64 CPU oracle for the OrbitQuant quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or run this module.
It shares no code with the CUDA library and imports nothing from it.

Sources (web pages about "OrbitQuant: Data-Agnostic Quantization for Image and
Video Diffusion Transformers", arXiv 2607.02461), cited below by page and
section:

* "gecl notes"     -- paper.gecl.asia reading notes, sections Core Idea,
                      Method 1-5, Key Insight, Limitation.
* "llmdb summary"  -- llmdb.app summary, sections Mathematical Formulation,
                      Implementation Details.
* "hotpaper"       -- hotpaper.ai page, the paper's abstract.
* "pith"           -- pith.science review: Figure 2 caption, referee minor
                      comment 1, Supplementary A "Proof Sketch for RPBH
                      Incoherence".

Each function follows the method's steps in the pages' order, in fp64.  Where
the pages are silent, ambiguous or at odds with one another, the function
names the reading it takes; the readings are:

* D1  marginal: the exact law of one coordinate of a uniform point on
      S^{d-1} (pith referee minor comment 1); N(0, 1/d) of pith Figure 2 as
      an option.
* D2  Lloyd-Max solver: Lloyd's alternation from N(0, 3/d) quantiles until
      no level moves by 1e-11/sqrt(d).
* D3  nearest level through midpoint thresholds.
* D4  codes unsigned and ascending with the level; a value exactly on a
      threshold takes the lower code.
* D5  a zero token has s = 0 and every coordinate u = 0.
* D6  the permutation is a gather, y_i = x_{pi(i)}, drawn by SplitMix64(seed)
      driving a descending Fisher-Yates shuffle.
* D7  Rademacher signs (pith Supplementary A) optional, drawn after the
      shuffle, -1 when bit 63 of the draw is set.
* D8  Sylvester natural order, scale 1/sqrt(h), block j = rotated positions
      [j h, (j+1) h).
* D9  h = the largest power of two dividing d.
* D10 normalise, then rotate (equal to the reverse order).
* D11 weights use the same Lloyd-Max quantizer with row norm r.
* D12 no bias and no renormalisation of the dequantised directions.
* D13 32 codes per little-endian bit stream of 32*b bits, b uint32 words.
* D14 inputs read as their exact values (bf16 / fp32), all arithmetic fp64.
* D15 the codebook's dimension is d_in, not h.
* D18 AdaLN exception path: symmetric per-row INT4 round-to-nearest.
(D16 and D17, the output and code tolerances, belong to the parity tests.)

Library primitives used as single steps: ``numpy`` gathers/matmul,
``np.searchsorted`` (a sorted search), ``scipy.special.betainc`` / ``erfc``
(the regularised incomplete beta function and the complementary error
function) and ``math.lgamma``.
"""

from __future__ import annotations

import functools
import math
from dataclasses import dataclass

import numpy as np
from scipy import special

__all__ = [
    "SplitMix64",
    "rpbh_permutation",
    "rademacher_signs",
    "hadamard_block_size",
    "sylvester_hadamard",
    "fwht",
    "rpbh_rotate",
    "dense_rpbh_matrix",
    "Codebook",
    "marginal_pdf",
    "marginal_survival",
    "marginal_partial_moment",
    "lloyd_max",
    "quantize",
    "nearest_level",
    "threshold_distance",
    "pack_codes",
    "unpack_codes",
    "bf16_bits_to_f64",
    "rotate_quantize",
    "weight_prepare",
    "linear_from_codes",
    "linear_exact",
    "OQ_SIGNS",
    "OQ_GAUSSIAN_MARGINAL",
    "OQ_WEIGHT_ONLY_INT4",
    "int4_rtn_weight_prepare",
    "int4_level",
    "int4_rtn_linear",
]

# Option flags; the same numeric values as the C-ABI flags (a documented
# interface, not shared code).
OQ_SIGNS = 1              # Rademacher signs D_j before each block Hadamard
OQ_GAUSSIAN_MARGINAL = 2  # design the codebook on N(0,1/d) instead of exact f_d
OQ_WEIGHT_ONLY_INT4 = 4   # AdaLN exception path: INT4 round-to-nearest weights, 16-bit activations

_MASK64 = (1 << 64) - 1


# --------------------------------------------------------------------------
# Seeded randomness for the rotation (reading D6/D7: the pages fix no
# generator; the llmdb snippet draws a fresh randperm per call, which would
# give weights and activations different permutations, so a seeded one is
# used and shared by both sides).
# --------------------------------------------------------------------------
class SplitMix64:
    """SplitMix64 (Steele, Lea and Flood, 2014), written from its definition:
    state += 0x9E3779B97F4A7C15, then two xor-shift-multiply rounds and a
    final xor-shift.  Exact 64-bit arithmetic with Python integers."""

    def __init__(self, seed: int):
        self.state = int(seed) & _MASK64

    def next(self) -> int:
        self.state = (self.state + 0x9E3779B97F4A7C15) & _MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        return z ^ (z >> 31)


def _fisher_yates(d: int, rng: SplitMix64) -> np.ndarray:
    perm = list(range(d))
    for i in range(d - 1, 0, -1):
        # uniform j in [0, i] as the high 64 bits of next() * (i + 1)
        j = (rng.next() * (i + 1)) >> 64
        perm[i], perm[j] = perm[j], perm[i]
    return np.asarray(perm, dtype=np.int64)


def rpbh_permutation(d: int, seed: int) -> np.ndarray:
    """The random permutation Pi of RPBH as a gather: rotated position i takes
    input channel ``perm[i]`` (y = P_pi x in pith Supplementary A; the
    "random permutation first scatters outlier channels" step of gecl notes
    Method 4).  Generator: SplitMix64(seed) driving a descending Fisher-Yates
    shuffle (reading D6)."""
    if d < 1:
        raise ValueError("d must be >= 1")
    return _fisher_yates(d, SplitMix64(seed))


def rademacher_signs(d: int, seed: int) -> np.ndarray:
    """Optional Rademacher diagonal D_j of pith Supplementary A (z = H_h D_j y),
    indexed by rotated position.  Drawn from the same SplitMix64 stream after
    the permutation's d-1 draws: sign = -1 when bit 63 of the draw is set
    (reading D7; off by default)."""
    rng = SplitMix64(seed)
    _fisher_yates(d, rng)
    out = np.empty(d, dtype=np.float64)
    for i in range(d):
        out[i] = -1.0 if (rng.next() >> 63) & 1 else 1.0
    return out


# --------------------------------------------------------------------------
# Block Walsh-Hadamard transform
# --------------------------------------------------------------------------
def hadamard_block_size(d: int) -> int:
    """h = the largest power of two dividing d (gecl notes, Key Insight: the
    largest power-of-two block size; pith Supplementary A writes d = k h)."""
    if d < 1:
        raise ValueError("d must be >= 1")
    return d & -d


def sylvester_hadamard(h: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix by its recursion
    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]] (reading D8)."""
    if h < 1 or h & (h - 1):
        raise ValueError("h must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < h:
        H = np.block([[H, H], [H, -H]])
    return H


def fwht(v: np.ndarray) -> np.ndarray:
    """Orthonormal Walsh-Hadamard transform H_h v / sqrt(h) along the last axis
    (length h, a power of two) by the textbook butterfly: for each stride
    s = 1, 2, 4, ..., h/2 the pair (a, b) at distance s becomes (a + b, a - b).
    Entries of the transform are +-1/sqrt(h) as in pith Supplementary A."""
    v = np.array(v, dtype=np.float64, copy=True)
    h = v.shape[-1]
    if h & (h - 1):
        raise ValueError("last axis must be a power of two")
    lead = v.shape[:-1]
    s = 1
    while s < h:
        w = v.reshape(lead + (h // (2 * s), 2, s))
        a = w[..., 0, :].copy()
        b = w[..., 1, :].copy()
        w[..., 0, :] = a + b
        w[..., 1, :] = a - b
        v = w.reshape(lead + (h,))
        s *= 2
    return v / math.sqrt(h)


def rpbh_rotate(x: np.ndarray, perm: np.ndarray, h: int,
                signs: np.ndarray | None = None) -> np.ndarray:
    """R x for the randomized permuted block-Hadamard rotation
    R = blockdiag(H_h/sqrt(h), ..., H_h/sqrt(h)) [D] P_pi (gecl notes Method 4;
    pith Supplementary A; llmdb summary Implementation Details: permute, then a
    block Hadamard per chunk).  Block j is rotated positions [j h, (j+1) h)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    if d % h:
        raise ValueError("h must divide d")
    y = x[..., perm]
    if signs is not None:
        y = y * signs
    k = d // h
    z = fwht(y.reshape(x.shape[:-1] + (k, h)))
    return z.reshape(x.shape)


def dense_rpbh_matrix(d: int, perm: np.ndarray, h: int,
                      signs: np.ndarray | None = None) -> np.ndarray:
    """The same rotation as an explicit d x d matrix, built from the Sylvester
    recursion and a permutation matrix (brute force for tiny d)."""
    P = np.zeros((d, d))
    P[np.arange(d), perm] = 1.0
    if signs is not None:
        P = np.diag(signs) @ P
    Hn = sylvester_hadamard(h) / math.sqrt(h)
    B = np.zeros((d, d))
    for j in range(d // h):
        B[j * h:(j + 1) * h, j * h:(j + 1) * h] = Hn
    return B @ P


# --------------------------------------------------------------------------
# The marginal f_d and its Lloyd-Max codebook
# --------------------------------------------------------------------------
def _sphere_const(d: int) -> float:
    return math.exp(math.lgamma(d / 2.0) - math.lgamma((d - 1) / 2.0)) / math.sqrt(math.pi)


def marginal_pdf(t, d: int, gaussian: bool = False):
    """Density of one coordinate of a unit vector in a random basis.  Exact
    (reading D1): the coordinate of a uniform point on S^{d-1},
    f_d(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - t^2)^((d-3)/2) on
    [-1, 1] (the closed form asked for by pith referee minor comment 1).
    ``gaussian=True``: the approximation N(0, 1/d) of pith Figure 2."""
    t = np.asarray(t, dtype=np.float64)
    if gaussian:
        return np.exp(-0.5 * d * t * t) * math.sqrt(d / (2.0 * math.pi))
    m = (d - 3) / 2.0
    inside = np.abs(t) < 1.0
    tt = np.where(inside, t, 0.0)
    return np.where(inside, _sphere_const(d) * np.exp(m * np.log1p(-tt * tt)), 0.0)


def marginal_survival(x, d: int, gaussian: bool = False):
    """P(T > x) for x >= 0.  Exact: T^2 ~ Beta(1/2, (d-1)/2), so
    P(T > x) = I_{1-x^2}((d-1)/2, 1/2) / 2.  Gaussian: erfc(x sqrt(d/2)) / 2."""
    x = np.asarray(x, dtype=np.float64)
    if gaussian:
        return 0.5 * special.erfc(x * math.sqrt(d / 2.0))
    xc = np.clip(x, 0.0, 1.0)
    return 0.5 * special.betainc((d - 1) / 2.0, 0.5, 1.0 - xc * xc)


def marginal_partial_moment(a, b, d: int, gaussian: bool = False):
    """Integral of t f(t) over [a, b], 0 <= a <= b, in closed form.
    Exact: c_d [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1).
    Gaussian: (phi(a) - phi(b)) / d with phi the N(0,1/d) density."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if gaussian:
        g = lambda t: np.where(np.isinf(t), 0.0, np.exp(-0.5 * d * np.where(np.isinf(t), 0.0, t) ** 2))
        return (g(a) - g(b)) / math.sqrt(2.0 * math.pi * d)
    e = (d - 1) / 2.0

    def p(t):
        tc = np.clip(t, 0.0, 1.0)
        return np.where(tc >= 1.0, 0.0, np.exp(e * np.log1p(-np.where(tc >= 1.0, 0.0, tc) ** 2)))

    return _sphere_const(d) * (p(a) - p(b)) / (d - 1)


@dataclass(frozen=True)
class Codebook:
    """A Lloyd-Max codebook C_{d,b}: ascending ``levels`` (2^b), ``thresholds``
    (2^b - 1 midpoints) and the designed mean-squared error ``mse`` per
    coordinate, all in the units of the unit-norm coordinate u."""
    d: int
    bits: int
    gaussian: bool
    levels: np.ndarray
    thresholds: np.ndarray
    mse: float
    iterations: int


_GL_X, _GL_W = np.polynomial.legendre.leggauss(20)


def _cells_mass_moment(e: np.ndarray, d: int, gaussian: bool):
    """Probability mass P_k and first moment M_k of each cell [e_k, e_{k+1}]
    of the positive half-line.  Gaussian: closed forms (erfc, exp).  Exact f_d:
    20-point Gauss-Legendre on panels no wider than a quarter of the density's
    width 1/sqrt(d-3); a cell is integrated up to 40 widths past its lower end
    (the density there is below exp(-800) of its value at the start)."""
    a, b = e[:-1], e[1:]
    if gaussian:
        S = marginal_survival(e, d, True)
        return S[:-1] - S[1:], marginal_partial_moment(a, b, d, True)
    width = 1.0 / math.sqrt(max(d - 3, 1))
    upper = np.minimum(b, a + 40.0 * width)
    npan = np.maximum(1, np.ceil((upper - a) / (0.25 * width)).astype(np.int64))
    cell = np.repeat(np.arange(len(a)), npan)
    first = np.repeat(np.cumsum(npan) - npan, npan)
    j = np.arange(len(cell)) - first
    lo = a[cell] + (upper - a)[cell] * j / npan[cell]
    hi = a[cell] + (upper - a)[cell] * (j + 1) / npan[cell]
    half = 0.5 * (hi - lo)
    t = (0.5 * (hi + lo))[:, None] + half[:, None] * _GL_X[None, :]
    w = half[:, None] * _GL_W[None, :] * marginal_pdf(t, d)
    P = np.bincount(cell, weights=w.sum(axis=1), minlength=len(a))
    M = np.bincount(cell, weights=(w * t).sum(axis=1), minlength=len(a))
    return P, M


@functools.lru_cache(maxsize=None)
def lloyd_max(d: int, bits: int, gaussian: bool = False) -> Codebook:
    """MSE-optimal 2^b-level scalar quantizer for the fixed marginal f_d, the
    codebook C_{d,b} of gecl notes Method 3 and pith Figure 2 (one per input
    dimension and bit width, no calibration data).  Lloyd's method (Lloyd
    1982; Max 1960, both in the pith reference list): alternate
    levels <- conditional means of their cells and thresholds <- midpoints of
    adjacent levels, until no level moves by more than 1e-11/sqrt(d) (reading
    D2).  The density is symmetric and log-concave (d >= 3), so the fixed point
    is symmetric and unique; the iteration runs on the positive half-line with
    the middle threshold at 0.  Start: levels at the quantiles of N(0, 3/d)
    (the f^(1/3) point density of high-resolution theory), kept inside (0, 1)."""
    if bits < 1 or bits > 8:
        raise ValueError("bits must be in 1..8")
    if d < 3:
        raise ValueError("d must be >= 3")
    L = 1 << bits
    n = L // 2
    sigma = 1.0 / math.sqrt(d)
    top = math.inf if gaussian else 1.0
    q = (n + np.arange(n) + 0.5) / L
    c = math.sqrt(3.0) * sigma * special.ndtri(q)
    if not gaussian:
        c = np.minimum(c, 1.0 - (n - np.arange(n)) * 1e-3 / n)
    tol = 1e-11 * sigma
    maxit = 2_000_000
    it = 0
    for it in range(1, maxit + 1):
        e = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [top]])
        P, M = _cells_mass_moment(e, d, gaussian)
        c_new = M / P
        delta = float(np.max(np.abs(c_new - c)))
        c = c_new
        if delta <= tol:
            break
    else:
        raise RuntimeError("Lloyd-Max did not converge")
    e = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [top]])
    P, _ = _cells_mass_moment(e, d, gaussian)
    levels = np.concatenate([-c[::-1], c])
    thr_pos = e[1:n]
    thresholds = np.concatenate([-thr_pos[::-1], [0.0], thr_pos])
    # distortion = E[T^2] - sum_k P_k c_k^2 (centroid condition), E[T^2] = 1/d
    mse = 1.0 / d - 2.0 * float(np.sum(P * c * c))
    return Codebook(d, bits, gaussian, levels, thresholds, mse, it)


# --------------------------------------------------------------------------
# Quantizer and packing
# --------------------------------------------------------------------------
def quantize(u: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """Nearest-level code of each coordinate (gecl notes Method 3) through the
    midpoint thresholds: code = #{j : t_j < u} (readings D3, D4: ascending
    codes; a value exactly on a threshold takes the lower code)."""
    return np.searchsorted(thresholds, np.asarray(u, dtype=np.float64), side="left").astype(np.int64)


def nearest_level(u: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """Brute force argmin_k |u - c_k| (the definition the thresholds stand for)."""
    u = np.asarray(u, dtype=np.float64)
    return np.argmin(np.abs(u[..., None] - levels), axis=-1)


def threshold_distance(u: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """min_j |u - t_j|: how close each coordinate lies to a decision threshold."""
    u = np.asarray(u, dtype=np.float64)
    idx = np.searchsorted(thresholds, u)
    lo = thresholds[np.clip(idx - 1, 0, len(thresholds) - 1)]
    hi = thresholds[np.clip(idx, 0, len(thresholds) - 1)]
    return np.minimum(np.abs(u - lo), np.abs(u - hi))


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes into uint32 words (reading D13; the pages leave the index
    format open, gecl notes Limitation 3).  Each group of 32 consecutive codes
    is one little-endian bit stream of 32*bits bits -- code i of the group at
    bits [i*bits, (i+1)*bits) -- stored as ``bits`` words, low word first."""
    codes = np.asarray(codes, dtype=np.uint64)
    d = codes.shape[-1]
    if d % 32:
        raise ValueError("the last axis must be a multiple of 32")
    lead = codes.shape[:-1]
    g = codes.reshape(lead + (d // 32, 32, 1))
    bitpos = np.arange(bits, dtype=np.uint64)
    stream = (g >> bitpos) & np.uint64(1)                  # [..., G, 32, bits]
    stream = stream.reshape(lead + (d // 32, bits, 32))    # bit k of the group -> word k//32
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = np.sum(stream * weights, axis=-1, dtype=np.uint64)
    return words.reshape(lead + (d // 32 * bits,)).astype(np.uint32)


def unpack_codes(words: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    words = np.asarray(words, dtype=np.uint64)
    lead = words.shape[:-1]
    w = words.reshape(lead + (d // 32, bits, 1))
    stream = (w >> np.arange(32, dtype=np.uint64)) & np.uint64(1)   # [..., G, bits, 32]
    stream = stream.reshape(lead + (d // 32, 32, bits))
    weights = np.uint64(1) << np.arange(bits, dtype=np.uint64)
    codes = np.sum(stream * weights, axis=-1, dtype=np.uint64)
    return codes.reshape(lead + (d,)).astype(np.int64)


def bf16_bits_to_f64(bits16: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 numbers given as their uint16 bit patterns."""
    b = np.asarray(bits16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# The layer
# --------------------------------------------------------------------------
def rotate_quantize(x: np.ndarray, perm: np.ndarray, h: int, cb: Codebook,
                    signs: np.ndarray | None = None):
    """Online activation codec, per token (gecl notes Method 1, 2, 4; hotpaper
    abstract): s = ||x||_2, x~ = x / s, u = R x~, code = Q(u).  Returns
    (codes [T, d] int, s [T], u [T, d]).  A zero token has s = 0 and u = 0
    (reading D5)."""
    x = np.asarray(x, dtype=np.float64)
    s = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(s > 0, s, 1.0)
    xt = np.where((s > 0)[..., None], x / safe[..., None], 0.0)
    u = rpbh_rotate(xt, perm, h, signs)
    return quantize(u, cb.thresholds), s, u


def weight_prepare(W: np.ndarray, perm: np.ndarray, h: int, cb_w: Codebook,
                   signs: np.ndarray | None = None):
    """Offline weight rows (hotpaper abstract: the same quantizer is extended to
    weight rows with the rotation absorbed; gecl notes Method 2: W Pi^T): row
    norm r_o = ||w_o||, rotated unit row R w_o / r_o, Lloyd-Max code with the
    weight codebook (reading D11; the min-max weight quantizer in the llmdb
    summary is not used).  Returns (Wcodes [d_out, d] int, r [d_out], u)."""
    return rotate_quantize(W, perm, h, cb_w, signs)


def linear_from_codes(codes_a: np.ndarray, s: np.ndarray, codes_w: np.ndarray,
                      r: np.ndarray, levels_a: np.ndarray, levels_w: np.ndarray):
    """Codebook contraction in the shared rotated basis (llmdb summary,
    y^ = Q_w(W R^-1) Q_a(R x); gecl notes Method 2: the rotation cancels inside
    the layer, no inverse rotation; pith Figure 2: W^' x^' ~ W x) with the
    magnitudes restored (gecl notes Method 1):
        y[t, o] = s_t r_o sum_i c_w[Wc[o, i]] c_a[Xc[t, i]]
    (reading D12: no bias, no renormalisation).  Returns (y, bound) where
    bound[t, o] = s_t r_o sum_i |c_w c_a| scales the error measure."""
    A = np.asarray(levels_a, dtype=np.float64)[np.asarray(codes_a)]
    B = np.asarray(levels_w, dtype=np.float64)[np.asarray(codes_w)]
    sr = np.asarray(s, dtype=np.float64)[:, None] * np.asarray(r, dtype=np.float64)[None, :]
    y = sr * (A @ B.T)
    bound = sr * (np.abs(A) @ np.abs(B).T)
    return y, bound


def linear_exact(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """The unquantised layer y = W x for every token (llmdb summary)."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


# ------------------------------------------------------------ AdaLN exception
# gecl notes Method 5: the dynamic AdaLN modulation projection cannot absorb a
# static rotation, so it is kept at INT4 weight-only round-to-nearest (the
# podcast page says the same: INT4, not the 2-bit of the rest).  The pages do
# not say how the scale is chosen; reading D18: symmetric, one scale per
# output row, s_o = max_i |w_oi| / 7, q = round-half-even(w / s_o) in
# [-7, 7], no rotation and no activation quantization.  The decision of each
# integer is taken in fp32 (the precision the kernel takes it in: the pages
# fix none), with IEEE division and round-half-even, so the codes are exact.
# Codes use the 4-bit format of the Lloyd-Max codes: c >= 8 is the level
# c - 8, c < 8 the level c - 7 (q >= 0 -> q + 8, q < 0 -> q + 7).

def int4_rtn_weight_prepare(W: np.ndarray):
    """INT4 RTN of each weight row (reading D18).  Returns (codes [d_out, d_in]
    int in 0..15 -- 7 never occurs --, scale [d_out] float32)."""
    W32 = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W32), axis=1)
    scale = (amax / np.float32(7.0)).astype(np.float32)        # IEEE fp32 division
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.rint((W32 / safe[:, None]).astype(np.float32))       # fp32 quotient, ties to even
    q = np.where(scale[:, None] > 0, np.clip(q, -7, 7), 0).astype(np.int64)
    codes = np.where(q >= 0, q + 8, q + 7)
    return codes, scale


def int4_level(codes: np.ndarray) -> np.ndarray:
    """The integer level of an INT4 code (c >= 8: c - 8; c < 8: c - 7)."""
    codes = np.asarray(codes, dtype=np.int64)
    return np.where(codes >= 8, codes - 8, codes - 7)


def int4_rtn_linear(x: np.ndarray, codes: np.ndarray, scale: np.ndarray):
    """y = x W^T with the RTN weights (level * scale) in fp64, and the bound
    sum_i |x_i| |w^_oi| used for the bound-relative tolerance."""
    Wq = int4_level(codes).astype(np.float64) * np.asarray(scale, dtype=np.float64)[:, None]
    x = np.asarray(x, dtype=np.float64)
    return x @ Wq.T, np.abs(x) @ np.abs(Wq).T
