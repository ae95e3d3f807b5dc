"""The index algebra of the GEMV kernel (batches of up to 24 tokens), on the CPU.

The kernel gives each CTA 16 weight rows and runs m16n8k16 warp MMAs with
the weight rows as M and a tile of 8 tokens as N.  Instead of the MMA's own K
order it maps K slots to positions so that a lane's operands are contiguous:
in a chunk of 128 positions lane q of a quad owns [32 q, 32 q + 32), and MMA
step s of a chunk maps the lane's slots {2q, 2q + 1} to positions
32 q + 4 s + {0, 1} and {2q + 8, 2q + 9} to 32 q + 4 s + {2, 3}.  A lane
decodes 8 positions of each of its two weight rows (g and g + 8) into four
fp16 pairs (.x .. .w) and loads the same 8 positions of its token 8 n + g of
each token tile n; pairs .x/.y feed step 2j and .z/.w step 2j + 1.  The
accumulator then holds rows g, g + 8 and tokens 8 n + 2q + {0, 1}.

This emulates those register maps lane by lane in numpy (the fragment
layouts of the PTX m16n8k16 instruction), with the chunks split over the
CTA's 8 warps as the kernel splits them, and checks that the assembled
result is the plain product of the weight rows and the token rows.  It pins
the derivation the kernel's indexing follows; the kernel itself is checked
against the oracle on the GPU."""

import numpy as np
import pytest

CHUNK, NWARP = 128, 8


def _lane_pairs(v, base):
    """The four value pairs (.x .. .w) a lane holds for 8 positions from
    `base` of vector v: (.x) base + 0, 1; (.y) + 2, 3; (.z) + 4, 5; (.w) + 6, 7."""
    return [(v[base + 2 * i], v[base + 2 * i + 1]) for i in range(4)]


def _gemv_emulated(Wt, X, slip=False):
    """y[t, o] for the 16 weight rows Wt [16, K] and tokens X [T, K]
    (T <= 24), assembled from per-lane MMA fragments.  slip: feed the token
    operand's two K-slot halves of every step the wrong way round (a
    plausible indexing mistake, for the check that the test can fail)."""
    K = Wt.shape[1]
    T = X.shape[0]
    NT = (T + 7) // 8
    nchunks = (K + CHUNK - 1) // CHUNK
    part = np.zeros((NWARP, NT, 16, 8))
    for warp in range(NWARP):
        for c in range(warp, nchunks, NWARP):
            for j in range(4):
                for step in (2 * j, 2 * j + 1):
                    A = np.zeros((16, 16))
                    Bs = [np.zeros((16, 8)) for _ in range(NT)]
                    for lane in range(32):
                        g, q = lane >> 2, lane & 3
                        pos0 = c * CHUNK + 32 * q
                        if pos0 >= K:          # a group past K: zeros on both sides
                            continue
                        lo = _lane_pairs(Wt[g], pos0 + 8 * j)
                        hi = _lane_pairs(Wt[g + 8], pos0 + 8 * j)
                        r0, r1 = (0, 1) if step == 2 * j else (2, 3)
                        # A fragment: a0 (row g, k 2q, 2q+1), a1 (row g+8, same k),
                        # a2 (row g, k 2q+8, 2q+9), a3 (row g+8, same k)
                        A[g, 2 * q:2 * q + 2] = lo[r0]
                        A[g + 8, 2 * q:2 * q + 2] = hi[r0]
                        A[g, 2 * q + 8:2 * q + 10] = lo[r1]
                        A[g + 8, 2 * q + 8:2 * q + 10] = hi[r1]
                        for n in range(NT):
                            t = 8 * n + g
                            if t >= T:
                                continue
                            a = _lane_pairs(X[t], pos0 + 8 * j)
                            # B fragment: b0 (k 2q, 2q+1; column g), b1 (k 2q+8, 2q+9)
                            b0, b1 = (a[r1], a[r0]) if slip else (a[r0], a[r1])
                            Bs[n][2 * q:2 * q + 2, g] = b0
                            Bs[n][2 * q + 8:2 * q + 10, g] = b1
                    for n in range(NT):
                        part[warp, n] += A @ Bs[n]
    # the warps' partial sums in warp order; lane (g, q) of warp n reads
    # d0 (row g, column 2q), d1 (g, 2q+1), d2 (g+8, 2q), d3 (g+8, 2q+1)
    y = np.zeros((T, 16))
    acc = part.sum(axis=0)
    for n in range(NT):
        for lane in range(32):
            g, q = lane >> 2, lane & 3
            for i in range(4):
                o, tk = g + 8 * (i >> 1), 8 * n + 2 * q + (i & 1)
                if tk < T:
                    y[tk, o] = acc[n, o, 2 * q + (i & 1)]
    return y


@pytest.mark.parametrize("K,T", [(128, 1), (96, 3), (1024, 8), (2048 + 96, 13), (640, 16), (4096, 24)])
def test_gemv_fragment_mapping(K, T):
    rng = np.random.default_rng(K + T)
    Wt = rng.standard_normal((16, K))
    X = rng.standard_normal((T, K))
    y = _gemv_emulated(Wt, X)
    np.testing.assert_allclose(y, X @ Wt.T, rtol=1e-12, atol=1e-9)


def test_gemv_mapping_catches_a_swapped_pair():
    # the same emulation with the token operand's K-slot halves swapped must
    # not reproduce the product, or the check above would prove nothing
    rng = np.random.default_rng(5)
    K, T = 256, 8
    Wt, X = rng.standard_normal((16, K)), rng.standard_normal((T, K))
    assert not np.allclose(_gemv_emulated(Wt, X, slip=True), X @ Wt.T)
