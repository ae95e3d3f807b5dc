"""CPU checks of the C-ABI library: it builds and loads, exports every symbol
the header declares, and its host-side math (codebook design, seeded
rotation, argument checks) agrees with the oracle.  No kernel is launched."""

import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle as O
from quantized_linear_token_b200 import binding as B
from quantized_linear_token_b200 import build as Bld

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    Bld.build()
    return B.load_library()


def _declared():
    text = open(os.path.join(ROOT, "include", "orbitquant.h")).read()
    return sorted(set(re.findall(r"^(?:oq_status|void|size_t|const char\*)\s+(oq_\w+)\s*\(", text, re.M)))


def test_header_declarations_match_binding():
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


@pytest.mark.parametrize("d", [256, 3072, 5120, 12288, 13824])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("gaussian", [False, True])
def test_codebook_matches_oracle(lib, d, bits, gaussian):
    cb = B.oq_codebook_build(d, bits, B.OQ_FLAG_GAUSSIAN_MARGINAL if gaussian else 0)
    ref = O.lloyd_max(d, bits, gaussian)
    sig = 1 / math.sqrt(d)
    # the oracle stops once no level moves by 1e-11 sigma; its error is
    # below 1e-9 sigma at these bit widths (linear convergence factor ~0.97)
    np.testing.assert_allclose(cb["levels"], ref.levels, rtol=0, atol=1e-9 * sig)
    np.testing.assert_allclose(cb["thresholds"], ref.thresholds, rtol=0, atol=1e-9 * sig)
    assert cb["mse"] == pytest.approx(ref.mse, rel=1e-8)


@pytest.mark.slow
@pytest.mark.parametrize("d", [3072, 13824])
def test_codebook_8bit_matches_oracle(lib, d):
    cb = B.oq_codebook_build(d, 8)
    ref = O.lloyd_max(d, 8)
    sig = 1 / math.sqrt(d)
    # 8 bits: the oracle's Lloyd iteration converges slowly (factor
    # ~1 - 1.5e-4 per step), so its levels carry up to ~1e-7 sigma of error
    np.testing.assert_allclose(cb["levels"], ref.levels, rtol=0, atol=5e-7 * sig)


def test_codebook_closed_forms(lib):
    # independent of the oracle: d = 3 uniform quantizer, 1-bit E|T|
    for b in (1, 2, 3, 4):
        L = 1 << b
        cb = B.oq_codebook_build(3, b)
        np.testing.assert_allclose(cb["levels"], -1 + (2 * np.arange(L) + 1) / L, atol=1e-12)
    for d in (32, 3072):
        cb = B.oq_codebook_build(d, 1)
        ea = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
        assert cb["levels"][1] == pytest.approx(ea, rel=1e-13)


@pytest.mark.parametrize("d", [32, 96, 256, 3072, 13824])
@pytest.mark.parametrize("seed", [0, 1, 12345678901234567])
def test_rotation_matches_oracle(lib, d, seed):
    perm, signs = B.oq_rotation_build(d, seed, B.OQ_FLAG_SIGNS)
    np.testing.assert_array_equal(perm.astype(np.int64), O.rpbh_permutation(d, seed))
    np.testing.assert_array_equal(signs.astype(np.float64), O.rademacher_signs(d, seed))


def test_argument_checks(lib):
    cb = B.CodebookC()
    assert lib.oq_codebook_build(256, 0, 0, ctypes.byref(cb)) == 2
    assert lib.oq_codebook_build(256, 9, 0, ctypes.byref(cb)) == 2
    assert lib.oq_codebook_build(2, 4, 0, ctypes.byref(cb)) == 1
    assert lib.oq_codebook_build(256, 4, 0, None) == 1
    h = ctypes.c_void_p()
    assert lib.oq_layer_create(100, 256, 0, 4, 4, 0, ctypes.byref(h)) == 2      # d_in % 32
    assert lib.oq_layer_create(8192, 256, 0, 4, 4, 0, ctypes.byref(h)) == 2     # h > 4096
    assert lib.oq_layer_create(256, 8, 0, 4, 4, 0, ctypes.byref(h)) == 2        # d_out % 16
    assert lib.oq_layer_create(256, 256, 0, 5, 4, 0, ctypes.byref(h)) == 2      # a_bits
    assert lib.oq_layer_create(256, 256, 0, 4, 8, 0, ctypes.byref(h)) == 2      # w_bits
    assert lib.oq_layer_create(256, 256, 0, 4, 4, 64, ctypes.byref(h)) == 1     # unknown flag
    assert lib.oq_layer_create(256, 256, 0, 4, 4, 0, None) == 1
    assert lib.oq_rotate_quantize(None, None, 1, 4, None, None, None) == 1
    assert lib.oq_linear(None, None, None, 4, None, None, None, 0, None) == 1
    assert lib.oq_linear_fused_workspace_size(None, 10) == 0
    assert lib.oq_linear_fused_host_workspace_size(None, 0, 10) == 0
    assert lib.oq_linear_fused_host(None, None, 0, 4, None, None, None, 0, None, 0, None) == 1
    assert lib.oq_rotation_build(0, 0, 0, None, None) == 1
    assert lib.oq_check_wait_timeout(None, 1000, None) == 1
    assert b"" != lib.oq_status_string(2)
    with pytest.raises(B.OrbitQuantError):
        B.oq_codebook_build(256, 9)


def test_python_names_mirror_c_names():
    for name in B.EXPORTS:
        if name in ("oq_last_error", "oq_status_string", "oq_layer_destroy", "oq_layer_get_info",
                    "oq_layer_get_perm"):
            continue
        assert callable(getattr(B, name)), name


def test_routing_thresholds_mirror_the_library():
    # bench.py labels its sweep points and the tests pick their bounds by the
    # batch sizes at which the library changes kernels; those copies must
    # follow the library's own constants
    import bench
    src = open(os.path.join(Bld.CSRC, "oq_internal.h")).read()

    def const(name):
        m = re.search(r"constexpr\s+(?:int|int64_t)\s+" + name + r"\s*=\s*(\d+)\s*;", src)
        assert m, name
        return int(m.group(1))

    assert bench.GEMV_MAX_T == const("GEMV_MAX_T")
    assert B.W16_MIN_T == const("W16_MIN_T")
    text = open(os.path.join(os.path.dirname(__file__), "test_gpu_parity.py")).read()
    assert int(re.search(r"^SKINNY_MAX_T = (\d+)", text, re.M).group(1)) == const("SKINNY_MAX_T")
    assert int(re.search(r"^W16_MIN_T = (\d+)", text, re.M).group(1)) == const("W16_MIN_T")
