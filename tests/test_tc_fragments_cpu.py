"""The index algebra of the tensor-core block transform, on the CPU.

The rotate-quantize kernel for h = 512 and 1024 computes z = H_h y of one
block as Z = H_A Y H_32 (Y[a][b] = y[32 a + b], A = h / 32) with two passes of
warp MMAs, and feeds pass 1's accumulator registers to pass 2 as B
fragments after choosing pass 2's K order to match.  This emulates those
fragment layouts (the m16n8k16 and m16n8k8 register maps of the PTX warp MMA
instructions) lane by lane in numpy and checks that the assembled result is
the Sylvester transform of the flattened block.  It pins the derivation the
kernel's indexing follows; the kernel itself is checked on the GPU."""

import numpy as np
import pytest

import oracle as O


def _hb(r: int, c: int) -> float:
    return -1.0 if bin(r & c).count("1") % 2 else 1.0


@pytest.mark.parametrize("A", [16, 32])
def test_two_pass_fragment_transform(A):
    NT1, MT2 = A // 8, A // 16
    Y = np.random.default_rng(A).standard_normal((A, 32))
    H32, HA = O.sylvester_hadamard(32), O.sylvester_hadamard(A)
    # pass 1: P^T = H_32 Y^T; lane (g, q) of tile (kt, nt) holds Y[8nt + g][16kt + 2q + 8r + {0, 1}]
    D1 = {}
    for mt in range(2):
        for nt in range(NT1):
            acc = np.zeros((16, 8))
            for kt in range(2):
                Bm = np.zeros((16, 8))
                for lane in range(32):
                    g, q = lane >> 2, lane & 3
                    for r in range(2):
                        b0 = 16 * kt + 2 * q + 8 * r
                        Bm[2 * q + 8 * r][g], Bm[2 * q + 8 * r + 1][g] = Y[8 * nt + g][b0], Y[8 * nt + g][b0 + 1]
                acc += H32[16 * mt:16 * mt + 16, 16 * kt:16 * kt + 16] @ Bm
            for lane in range(32):
                g, q = lane >> 2, lane & 3
                D1[lane, mt, nt] = (acc[g][2 * q], acc[g][2 * q + 1], acc[g + 8][2 * q], acc[g + 8][2 * q + 1])
    # pass 2: Z = H_A P, k tile nt with k = q <-> a = 8nt + 2q and k = q + 4 <-> a = 8nt + 2q + 1
    z = O.sylvester_hadamard(32 * A) @ Y.reshape(-1)
    for mt2 in range(MT2):
        for nt2 in range(4):
            acc = np.zeros((16, 8))
            for nt in range(NT1):
                Am, Bm = np.zeros((16, 8)), np.zeros((8, 8))
                for lane in range(32):
                    g, q = lane >> 2, lane & 3
                    u, v = _hb(g, 2 * q), _hb(g, 2 * q + 1)
                    na = mt2 & (nt >> 1)
                    nh = na ^ (nt & 1)
                    Am[g][q], Am[g + 8][q] = (-u if na else u), (-u if nh else u)
                    Am[g][q + 4], Am[g + 8][q + 4] = (-v if na else v), (-v if nh else v)
                    d = D1[lane, nt2 >> 1, nt]
                    Bm[q][g], Bm[q + 4][g] = d[2 * (nt2 & 1)], d[2 * (nt2 & 1) + 1]
                for m in range(16):
                    for k in range(8):
                        assert Am[m][k] == HA[16 * mt2 + m][8 * nt + 2 * (k % 4) + (k >= 4)]
                acc += Am @ Bm
            for lane in range(32):
                g, q = lane >> 2, lane & 3
                for half in range(2):
                    for e2 in range(2):
                        a, b = 16 * mt2 + g + 8 * half, 8 * nt2 + 2 * q + e2
                        assert np.isclose(acc[g + 8 * half][2 * q + e2], z[32 * a + b])
