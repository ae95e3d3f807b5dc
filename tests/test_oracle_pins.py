"""Pins for the fp64 oracle: each test checks the oracle against something
other than itself (published values, closed forms, brute force, invariants,
library routines), chosen so that a dropped term, a wrong sign or index or a
transposed operand in the oracle fails at least one of them.  CPU only."""

import math
import os

import numpy as np
import pytest
from scipy import integrate, linalg, special, stats

import oracle as O
from quantized_linear_token_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- generator
def test_splitmix64_reference_outputs():
    # First three outputs of SplitMix64 from seed 0, as published with the
    # generator's reference implementation (Vigna, splitmix64.c test output).
    g = O.SplitMix64(0)
    assert [g.next() for _ in range(3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_permutation_is_a_permutation():
    for d in (1, 2, 32, 256, 3072, 13824):
        p = O.rpbh_permutation(d, 7)
        assert sorted(p.tolist()) == list(range(d))
    assert not np.array_equal(O.rpbh_permutation(256, 0), O.rpbh_permutation(256, 1))
    assert np.array_equal(O.rpbh_permutation(256, 5), O.rpbh_permutation(256, 5))


def test_permutation_is_uniform():
    # The pages ask for a uniform random permutation (gecl notes, Relation To
    # Prior Work: uniform random permutation, not a calibrated one).  All 24
    # permutations of 4 items must be equally likely over seeds.
    counts = {}
    n = 24000
    for seed in range(n):
        key = tuple(O.rpbh_permutation(4, seed).tolist())
        counts[key] = counts.get(key, 0) + 1
    assert len(counts) == 24
    chi2 = sum((c - n / 24) ** 2 / (n / 24) for c in counts.values())
    assert chi2 < stats.chi2.ppf(0.999, 23)


def test_rademacher_signs_balanced():
    s = O.rademacher_signs(4096, 3)
    assert set(np.unique(s).tolist()) == {-1.0, 1.0}
    assert abs(s.mean()) < 4 / math.sqrt(4096)


# ---------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("h", [1, 2, 4, 8, 16, 64, 256])
def test_sylvester_matches_library(h):
    assert np.array_equal(O.sylvester_hadamard(h), linalg.hadamard(h))


@pytest.mark.parametrize("h", [2, 8, 32, 128, 1024])
def test_fwht_is_normalised_hadamard(h):
    H = linalg.hadamard(h) / math.sqrt(h)
    rng = np.random.default_rng(h)
    v = rng.standard_normal((3, h))
    np.testing.assert_allclose(O.fwht(v), v @ H.T, rtol=0, atol=1e-12)


def test_block_size_rule():
    cases = {256: 256, 3072: 1024, 12288: 4096, 5120: 1024, 13824: 512, 96: 32, 7: 1}
    for d, h in cases.items():
        assert O.hadamard_block_size(d) == h
        assert d % h == 0 and (d // h) % 2 == 1


# P1: R is orthogonal and the fast transform equals the dense matrix
@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 96, 192, 320])
@pytest.mark.parametrize("signed", [False, True])
def test_rotation_orthogonal_and_fast_equals_dense(d, signed):
    h = O.hadamard_block_size(d)
    perm = O.rpbh_permutation(d, 11)
    sg = O.rademacher_signs(d, 11) if signed else None
    R = O.dense_rpbh_matrix(d, perm, h, sg)
    np.testing.assert_allclose(R @ R.T, np.eye(d), atol=1e-14)
    x = np.random.default_rng(d).standard_normal((5, d))
    np.testing.assert_allclose(O.rpbh_rotate(x, perm, h, sg), x @ R.T, atol=1e-13)


def test_rotation_is_not_identity_on_structure():
    # The permutation must act before the Hadamard: rotating e_{perm[0]} gives
    # the first column pattern of block 0 (all +1/sqrt(h) in block 0).
    d, h = 96, 32
    perm = O.rpbh_permutation(d, 3)
    e = np.zeros(d)
    e[perm[0]] = 1.0
    z = O.rpbh_rotate(e, perm, h)
    np.testing.assert_allclose(z[:h], np.full(h, 1 / math.sqrt(h)), atol=1e-15)
    np.testing.assert_allclose(z[h:], 0.0, atol=1e-15)


# P2: the rotation folded into the weights cancels inside the layer
@pytest.mark.parametrize("d", [64, 96, 3072])
def test_rotation_cancels_in_the_product(d):
    h = O.hadamard_block_size(d)
    perm = O.rpbh_permutation(d, 0)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, d))
    Wm = rng.standard_normal((5, d))
    Wrot = O.rpbh_rotate(Wm, perm, h)          # rows of W R^T
    xrot = O.rpbh_rotate(x, perm, h)
    y = xrot @ Wrot.T
    yx = O.linear_exact(x, Wm)
    np.testing.assert_allclose(y, yx, rtol=1e-12, atol=1e-12 * np.abs(yx).max())
    np.testing.assert_allclose(np.linalg.norm(xrot, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


# ---------------------------------------------------------------- marginal
@pytest.mark.parametrize("d", [3, 32, 256, 3072])
def test_marginal_density_normalised_with_variance_one_over_d(d):
    mass = integrate.quad(lambda t: O.marginal_pdf(t, d), -1, 1, points=[0], limit=400)[0]
    var = integrate.quad(lambda t: t * t * O.marginal_pdf(t, d), -1, 1, points=[0], limit=400)[0]
    assert mass == pytest.approx(1.0, abs=1e-10)
    assert var == pytest.approx(1.0 / d, rel=1e-9)


def test_marginal_matches_sphere_samples():
    # The exact marginal is the law of one coordinate of a uniform point on
    # S^{d-1}: compare with normalised Gaussian vectors.
    d = 64
    g = np.random.default_rng(5).standard_normal((40000, d))
    t = (g / np.linalg.norm(g, axis=1, keepdims=True)).ravel()
    cdf = lambda v: np.where(np.asarray(v) >= 0, 1 - O.marginal_survival(np.abs(v), d),
                             O.marginal_survival(np.abs(v), d))
    assert stats.kstest(t[:200000], cdf).statistic < 0.005


def test_survival_two_ways():
    # incomplete-beta survival vs direct quadrature of the density
    for d in (32, 3072, 13824):
        for x in (0.0, 0.3, 1.0, 2.5):
            xs = x / math.sqrt(d)
            q = integrate.quad(lambda t: O.marginal_pdf(t, d), xs, 1.0, limit=400, epsabs=1e-14, epsrel=1e-12,
                               points=[min(1.0, xs + k / math.sqrt(d)) for k in (1, 3, 6)])[0]
            assert float(O.marginal_survival(xs, d)) == pytest.approx(q, abs=1e-11)


# ---------------------------------------------------------------- Lloyd-Max (P3, P4)
def _golden_gaussian():
    rows = []
    with open(os.path.join(GOLDEN, "lloyd_max_gaussian_unit.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            v = line.split()
            b = int(v[0])
            rows.append((b, [float(t) for t in v[1:1 + (1 << (b - 1))]], float(v[-1])))
    return rows


@pytest.mark.parametrize("d", [256, 3072])
def test_gaussian_mode_reproduces_max_table(d):
    for b, levels, mse in _golden_gaussian():
        cb = O.lloyd_max(d, b, gaussian=True)
        pos = cb.levels[len(cb.levels) // 2:] * math.sqrt(d)
        np.testing.assert_allclose(pos, levels, atol=1e-4)
        assert cb.mse * d == pytest.approx(mse, abs=1e-3)


def test_one_bit_closed_forms():
    # 1 bit: threshold 0, level = E[|T|].  Gaussian: sqrt(2/pi)/sqrt(d).
    # Exact f_d: E|T| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)).
    for d in (3, 32, 256, 3072, 13824):
        g = O.lloyd_max(d, 1, gaussian=True)
        assert g.levels[1] == pytest.approx(math.sqrt(2 / math.pi) / math.sqrt(d), rel=1e-12)
        e = O.lloyd_max(d, 1)
        ea = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
        assert e.levels[1] == pytest.approx(ea, rel=1e-12)
        assert e.thresholds.tolist() == [0.0]


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_d3_is_the_uniform_quantizer(b):
    # For d = 3 the sphere marginal is uniform on [-1, 1]; its Lloyd-Max
    # quantizer is the uniform one: cells of width 2/L, levels at the centres,
    # MSE = (2/L)^2 / 12.
    L = 1 << b
    cb = O.lloyd_max(3, b)
    np.testing.assert_allclose(cb.levels, -1 + (2 * np.arange(L) + 1) / L, atol=1e-9)
    assert cb.mse == pytest.approx((2 / L) ** 2 / 12, rel=1e-7)


def test_exact_mode_converges_to_gaussian_table():
    # sqrt(d) c_{d,b} -> the unit-Gaussian table as d grows, gap ~ 1/d
    for b in (2, 3):
        gauss = O.lloyd_max(256, b, gaussian=True).levels * 16.0
        gaps = []
        for d in (256, 3072, 12288):
            gaps.append(np.max(np.abs(O.lloyd_max(d, b).levels * math.sqrt(d) - gauss)))
        assert gaps[0] > gaps[1] > gaps[2]
        assert gaps[0] / gaps[1] == pytest.approx(3072 / 256, rel=0.2)
        assert gaps[1] / gaps[2] == pytest.approx(12288 / 3072, rel=0.2)


@pytest.mark.parametrize("d,b", [(256, 2), (256, 4), (3072, 3), (13824, 4)])
def test_optimality_conditions_by_independent_quadrature(d, b):
    # Each level is the conditional mean of its cell (computed here with
    # adaptive quadrature, not the oracle's fixed rule), each threshold the
    # midpoint of its levels, and the codebook is symmetric.
    cb = O.lloyd_max(d, b)
    sig = 1 / math.sqrt(d)
    edges = np.concatenate([[-1.0], cb.thresholds, [1.0]])
    for k, c in enumerate(cb.levels):
        a, e = edges[k], edges[k + 1]
        if a < -0.5:
            a = max(a, e - 60 * sig)
        if e > 0.5:
            e = min(e, a + 60 * sig)
        P = integrate.quad(lambda t: O.marginal_pdf(t, d), a, e, epsabs=1e-300, epsrel=1e-13, limit=400)[0]
        M = integrate.quad(lambda t: t * O.marginal_pdf(t, d), a, e, epsabs=1e-300, epsrel=1e-13, limit=400)[0]
        assert M / P == pytest.approx(c, abs=5e-10 * sig)
    np.testing.assert_allclose(cb.thresholds, 0.5 * (cb.levels[1:] + cb.levels[:-1]), atol=1e-17)
    np.testing.assert_allclose(cb.levels, -cb.levels[::-1], atol=1e-17)
    assert np.all(np.diff(cb.levels) > 0)


def test_fixed_point_independent_of_start():
    # Run Lloyd's iteration from a uniform start with scipy quadrature and
    # compare with the oracle (log-concave density: unique fixed point).
    d, b = 256, 2
    sig = 1 / math.sqrt(d)
    c = np.array([-0.9, -0.1, 0.2, 0.7])
    for _ in range(400):
        t = 0.5 * (c[1:] + c[:-1])
        e = np.concatenate([[-1.0], t, [1.0]])
        new = []
        for k in range(4):
            P = integrate.quad(lambda v: O.marginal_pdf(v, d), e[k], e[k + 1], limit=200)[0]
            M = integrate.quad(lambda v: v * O.marginal_pdf(v, d), e[k], e[k + 1], limit=200)[0]
            new.append(M / P)
        c = np.array(new)
    np.testing.assert_allclose(c, O.lloyd_max(d, b).levels, atol=1e-9 * sig)


# ---------------------------------------------------------------- quantizer (P6)
def test_threshold_count_equals_nearest_level():
    cb = O.lloyd_max(256, 4)
    u = np.random.default_rng(2).standard_normal(200000) / 16.0
    np.testing.assert_array_equal(O.quantize(u, cb.thresholds), O.nearest_level(u, cb.levels))
    # exactly on a threshold: the lower code, which is also argmin's first
    # of two equally near levels
    ties = cb.thresholds
    np.testing.assert_array_equal(O.quantize(ties, cb.thresholds), np.arange(15))
    assert O.quantize(np.array([-1.0, 1.0]), cb.thresholds).tolist() == [0, 15]


@pytest.mark.parametrize("d", [256, 3072])
@pytest.mark.parametrize("b", [2, 3, 4, 8])
def test_threshold_distance_is_brute_force_minimum(d, b):
    # threshold_distance decides which GPU code mismatches the parity bound
    # excuses (a coordinate within 1e-5/sqrt(d) of a decision threshold).  Pin
    # it to its definition min_j |u - t_j| taken by brute force over every
    # threshold, on random coordinates, on coordinates exactly at and just
    # beside each threshold (where a wrong searchsorted side or an
    # off-by-one neighbour shows), and on coordinates past the outermost
    # thresholds and past +-1.
    cb = O.lloyd_max(d, b)
    t = cb.thresholds
    rng = np.random.default_rng(d + b)
    step = 1e-7 / math.sqrt(d)
    u = np.concatenate([
        rng.standard_normal(50000) / math.sqrt(d),
        t, t + step, t - step, np.nextafter(t, np.inf), np.nextafter(t, -np.inf),
        0.5 * (t[:-1] + t[1:]),                         # equidistant from two thresholds
        [t[0] - 1.0, t[-1] + 1.0, t[0] - step, t[-1] + step, -1.0, 1.0, -5.0, 5.0, 0.0],
    ])
    brute = np.min(np.abs(u[:, None] - t[None, :]), axis=1)
    np.testing.assert_array_equal(O.threshold_distance(u, t), brute)
    # the band test of the parity checks: exactly the coordinates whose
    # nearest threshold is closer than the band
    band = 1e-5 / math.sqrt(d)
    np.testing.assert_array_equal(O.threshold_distance(u, t) < band, brute < band)
    assert np.all(O.threshold_distance(t, t) == 0.0)


@pytest.mark.parametrize("d", [3, 4, 16, 256, 3072])
@pytest.mark.parametrize("gaussian", [False, True])
def test_partial_moment_equals_quadrature(d, gaussian):
    # the closed-form first moment of each half-line cell (exact sphere
    # marginal: the antiderivative of t (1 - t^2)^((d-3)/2); Gaussian: of
    # t phi(t)) against adaptive quadrature of t f_d(t) over the same interval
    sig = 1.0 / math.sqrt(d)
    top = 1.0 if not gaussian else 12.0 * sig
    edges = [(0.0, 0.3 * sig), (0.3 * sig, 1.1 * sig), (1.1 * sig, 2.7 * sig), (0.0, top),
             (2.7 * sig, top), (0.5 * sig, 0.5 * sig)]
    for a, b in edges:
        a, b = min(a, top), min(b, top)
        want, _ = integrate.quad(lambda t: t * O.marginal_pdf(t, d, gaussian), a, b, epsabs=0, epsrel=1e-12,
                                 limit=200)
        got = float(O.marginal_partial_moment(a, b, d, gaussian))
        assert abs(got - want) <= 1e-10 * (abs(want) + sig * 1e-3), (a, b, got, want)
    # the half-line moment E[T; T > 0] in closed form: for the sphere
    # Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2) (d-1)), for N(0, 1/d) 1/sqrt(2 pi d)
    half = float(O.marginal_partial_moment(0.0, math.inf if gaussian else 1.0, d, gaussian))
    want_half = (1.0 / math.sqrt(2 * math.pi * d) if gaussian else
                 math.exp(math.lgamma(d / 2) - math.lgamma((d - 1) / 2)) / (math.sqrt(math.pi) * (d - 1)))
    assert abs(half - want_half) <= 1e-13 * want_half


def test_quantizer_mse_matches_design():
    d = 256
    g = np.random.default_rng(9).standard_normal((20000, d))
    t = (g / np.linalg.norm(g, axis=1, keepdims=True)).ravel()
    for b in (2, 4):
        cb = O.lloyd_max(d, b)
        err = (t - cb.levels[O.quantize(t, cb.thresholds)]) ** 2
        se = err.std() / math.sqrt(err.size)
        assert abs(err.mean() - cb.mse) < 4 * se


def test_zero_token_codes():
    # s = 0: every coordinate is 0 and takes code #{t_j < 0} = L/2 - 1
    cb = O.lloyd_max(64, 3)
    codes, s, u = O.rotate_quantize(np.zeros((2, 64)), O.rpbh_permutation(64, 0), 64, cb)
    assert s.tolist() == [0.0, 0.0]
    assert np.all(codes == 3)


# ---------------------------------------------------------------- packing (P7)
@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_pack_round_trip(b):
    rng = np.random.default_rng(b)
    codes = rng.integers(0, 1 << b, size=(3, 128))
    words = O.pack_codes(codes, b)
    assert words.shape == (3, 128 * b // 32) and words.dtype == np.uint32
    np.testing.assert_array_equal(O.unpack_codes(words, b, 128), codes)


def test_pack_hand_example_3bit():
    # codes 0..7 repeated: 8 codes of 3 bits make the 24-bit value
    # 0o76543210 = 0xFAC688, four times in the 96-bit group, so the words are
    # 0x88FAC688, 0xC688FAC6, 0xFAC688FA (low word first).
    codes = np.tile(np.arange(8), 4)[None, :]
    assert O.pack_codes(codes, 3)[0].tolist() == [0x88FAC688, 0xC688FAC6, 0xFAC688FA]


def test_pack_brute_force_bitstring():
    # an independent formulation: write the bit string code by code
    rng = np.random.default_rng(4)
    for b in (2, 3, 4, 8):
        codes = rng.integers(0, 1 << b, size=64)
        bits = "".join(format(int(c), "0%db" % b)[::-1] for c in codes)   # LSB first
        words = [int(bits[32 * w:32 * w + 32][::-1], 2) for w in range(len(bits) // 32)]
        assert O.pack_codes(codes[None, :], b)[0].tolist() == words


# ---------------------------------------------------------------- layer (P5, P8)
def test_bf16_decoding():
    assert O.bf16_bits_to_f64(np.array([0x3F80, 0xBF80, 0x4049, 0x0000])).tolist() == [1.0, -1.0, 3.140625, 0.0]


@pytest.mark.parametrize("key,d,T", [("dit_image", 3072, 400), ("video_dit", 5120, 240)])
def test_rotated_coordinates_follow_the_marginal(key, d, T):
    # pith Figure 3 / "What would settle it": rotated coordinates of drifting,
    # outlier-heavy activations follow one fixed marginal ~ N(0, 1/d).  The
    # agreement is approximate: a token whose energy sits in a few outlier
    # channels gives its blocks a few large coordinates (the regime gecl
    # Limitation 1 names), so the KS distance moves with how the recipe's
    # outliers fall into blocks (0.001 to 0.024 over independent draws of
    # these recipes).  A scale or transform error gives KS distances of 0.1
    # and more.
    wl = W.WORKLOADS[key]
    x = O.bf16_bits_to_f64(W.activations(wl, d, T))
    h = O.hadamard_block_size(d)
    _, _, u = O.rotate_quantize(x, O.rpbh_permutation(d, 0), h, O.lloyd_max(d, 4))
    v = (u * math.sqrt(d)).ravel()
    assert v.size >= 10 ** 6
    assert stats.kstest(v, "norm").statistic <= 0.03
    # without the 1/sqrt(h) of the orthonormal transform the same statistic
    # is far off (the pin's sensitivity)
    assert stats.kstest(v * math.sqrt(h), "norm").statistic > 0.3


def test_signed_rotation_keeps_the_marginal():
    # pith Supplementary A adds Rademacher signs D before H; the rotated
    # coordinates of the same outlier-heavy activations still follow the one
    # fixed marginal (the signed RPBH variant of the scope's next steps)
    wl = W.WORKLOADS["dit_image"]
    d, T = 3072, 400
    x = O.bf16_bits_to_f64(W.activations(wl, d, T))
    _, _, u = O.rotate_quantize(x, O.rpbh_permutation(d, 0), O.hadamard_block_size(d), O.lloyd_max(d, 4),
                                signs=O.rademacher_signs(d, 0))
    assert stats.kstest((u * math.sqrt(d)).ravel(), "norm").statistic <= 0.03


def test_signed_and_gaussian_variants_match_the_default():
    # The two flag variants (signed RPBH; codebook on N(0, 1/d) instead of the
    # exact sphere marginal) against the default on the image-DiT recipe at
    # W4A4: at d = 3072 the two codebooks nearly coincide and the signs leave
    # the marginal unchanged, so the layer error ||y_q - W x|| / ||W x|| of all
    # four combinations agrees to within a few percent.
    wl = W.WORKLOADS["dit_image"]
    lay = wl.layers[0]
    d, T, dout = 3072, 48, 256
    x = O.bf16_bits_to_f64(W.activations(wl, d, T))
    Wm = W.weights(wl, lay)[:dout].astype(np.float64)
    h, perm = O.hadamard_block_size(d), O.rpbh_permutation(d, 0)
    yx = O.linear_exact(x, Wm)
    errs = {}
    for signed in (False, True):
        sg = O.rademacher_signs(d, 0) if signed else None
        for gauss in (False, True):
            cb = O.lloyd_max(d, 4, gauss)
            xc, s, _ = O.rotate_quantize(x, perm, h, cb, signs=sg)
            wc, r, _ = O.weight_prepare(Wm, perm, h, cb, signs=sg)
            y, _ = O.linear_from_codes(xc, s, wc, r, cb.levels, cb.levels)
            errs[(signed, gauss)] = np.linalg.norm(y - yx) / np.linalg.norm(yx)
    base = errs[(False, False)]
    assert 0.02 < base < 0.2
    for v in errs.values():
        assert abs(v / base - 1.0) < 0.05


def test_permutation_balances_block_masses():
    # gecl notes Key Insight: without the permutation, outliers sitting in one
    # block leave that block with most of the mass; Pi spreads them out.
    d, h = 5120, 1024
    k = d // h
    rng = np.random.default_rng(0)
    x = rng.standard_normal((200, d))
    x[:, :64] *= 50.0                     # all 64 outliers inside block 0
    cb = O.lloyd_max(d, 4)

    def spread(perm):
        _, _, u = O.rotate_quantize(x, perm, h, cb)
        M = (u.reshape(len(x), k, h) ** 2).sum(axis=2)
        return np.mean(np.abs(k * M - 1.0))

    assert spread(np.arange(d)) > 1.4
    assert spread(O.rpbh_permutation(d, 0)) < 0.45


def test_error_falls_with_bits():
    # P8: the quantized layer approaches W x as the bit widths grow
    d, dout, T = 512, 64, 64
    x = W.custom_activations(T, d, 3, bf16=False).astype(np.float64)
    Wm = W.custom_weights(dout, d, 4).astype(np.float64)
    h = O.hadamard_block_size(d)
    perm = O.rpbh_permutation(d, 0)
    yx = O.linear_exact(x, Wm)
    errs = []
    for wb, ab in ((2, 4), (3, 3), (4, 4), (4, 8)):
        ca, cw = O.lloyd_max(d, ab), O.lloyd_max(d, wb)
        xc, s, _ = O.rotate_quantize(x, perm, h, ca)
        wc, r, _ = O.weight_prepare(Wm, perm, h, cw)
        y, bound = O.linear_from_codes(xc, s, wc, r, ca.levels, cw.levels)
        assert np.all(np.abs(y) <= bound * (1 + 1e-12))
        errs.append(np.linalg.norm(y - yx) / np.linalg.norm(yx))
    assert errs[0] > errs[1] > errs[2] > errs[3]
    assert errs[3] < 0.15


def test_linear_exact_when_codebooks_are_fine():
    # With the exact rotated values in place of the levels the contraction is
    # W x exactly: check the s * r scaling and the shared basis by feeding
    # "levels" equal to the rotated coordinates themselves.
    d, dout = 64, 8
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, d))
    Wm = rng.standard_normal((dout, d))
    perm = O.rpbh_permutation(d, 2)
    u = O.rpbh_rotate(x / np.linalg.norm(x, axis=1, keepdims=True), perm, d)
    v = O.rpbh_rotate(Wm / np.linalg.norm(Wm, axis=1, keepdims=True), perm, d)
    levels = np.concatenate([u.ravel(), v.ravel()])
    ca = np.arange(u.size).reshape(u.shape)
    cw = u.size + np.arange(v.size).reshape(v.shape)
    y, _ = O.linear_from_codes(ca, np.linalg.norm(x, axis=1), cw, np.linalg.norm(Wm, axis=1), levels, levels)
    np.testing.assert_allclose(y, O.linear_exact(x, Wm), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- INT4 RTN (AdaLN)
def test_int4_rtn_hand_example():
    # one row, max |w| = 3.5 -> scale 0.5: w / s = [7, -2, 1.5, 0.5, -0.5, 0]
    # round half to even -> [7, -2, 2, 0, -0, 0]; codes q+8 / q+7
    codes, scale = O.int4_rtn_weight_prepare(np.array([[3.5, -1.0, 0.75, 0.25, -0.25, 0.0]]))
    assert scale.tolist() == [np.float32(0.5)]
    assert O.int4_level(codes).tolist() == [[7, -2, 2, 0, 0, 0]]
    assert codes.tolist() == [[15, 5, 10, 8, 8, 8]]


def test_int4_rtn_is_nearest_level_brute_force():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((40, 96)) * rng.uniform(0.01, 3.0, (40, 1))).astype(np.float32)
    codes, scale = O.int4_rtn_weight_prepare(W)
    assert set(np.unique(codes).tolist()) <= set(range(16)) - {7}
    lv = O.int4_level(codes)
    assert np.all(np.abs(lv).max(axis=1) == 7)                 # the largest |w| maps to +-7
    cand = np.arange(-7, 8)
    for o in range(W.shape[0]):
        t = W[o].astype(np.float64) / float(scale[o])
        best = cand[np.argmin(np.abs(t[:, None] - cand[None, :]), axis=1)]
        # away from exact ties the fp32 decision is the nearest integer level
        far = np.abs(np.abs(t - np.floor(t)) - 0.5) > 1e-5
        assert np.array_equal(lv[o][far], best[far])
    err = np.abs(W - lv * scale[:, None])
    assert np.all(err <= 0.5 * scale[:, None] * (1 + 1e-6))


def test_int4_rtn_zero_row_and_lossless_row():
    codes, scale = O.int4_rtn_weight_prepare(np.zeros((1, 8)))
    assert scale[0] == 0 and np.all(O.int4_level(codes) == 0)
    # a row already on the grid (integer multiples of max / 7) is reproduced exactly
    lv = np.array([[7, -7, 3, -2, 0, 1, -5, 6]], dtype=np.float64)
    W = lv * 0.25
    codes, scale = O.int4_rtn_weight_prepare(W)
    np.testing.assert_array_equal(O.int4_level(codes), lv)
    x = np.random.default_rng(5).standard_normal((3, 8))
    y, bound = O.int4_rtn_linear(x, codes, scale)
    np.testing.assert_allclose(y, x @ W.T, rtol=0, atol=1e-12)
    assert np.all(np.abs(y) <= bound + 1e-12)
