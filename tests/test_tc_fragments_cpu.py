"""The index algebra of the tensor-core block transform, on the CPU.

The rotate-quantize kernel for h = 512 and 1024 computes z = H_h y of one
block as Z = H_A Y H_32 (Y[a][b] = y[32 a + b], A = h / 32) with two passes of
warp MMAs, and feeds pass 1's accumulator registers to pass 2 as B
fragments after choosing pass 2's K order to match.  This emulates those
fragment layouts (the m16n8k16 and m16n8k8 register maps of the PTX warp MMA
instructions) lane by lane in numpy and checks that the assembled result is
the Sylvester transform of the flattened block, and that the packed-code
output (each lane placing its code pairs in the group's bit stream, the quad
OR-ing its words) assembles the packed group.  It pins the derivation the
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


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_packed_code_quad_or(bits):
    # The tensor-core kernel's packed-code output: for one row a' of the block
    # (a group of 32 positions b'), lane q of a quad holds the codes of
    # b' = 8 nt + 2q + {0, 1} (nt = 0..3); it places each pair at bit
    # bits * (8 nt + 2q) of the group's stream (bits words), the four lanes OR
    # their words together (two xor shuffles) and lane q stores the words
    # i with i % 4 == q.  The assembled words must be the packed group.
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=32)
    lanes = []
    for q in range(4):
        w = [0] * bits
        for nt in range(4):
            c0, c1 = int(codes[8 * nt + 2 * q]), int(codes[8 * nt + 2 * q + 1])
            pair = c0 | (c1 << bits)
            bit = bits * (8 * nt + 2 * q)
            for i in range(bits):
                lo = bit - 32 * i                       # the pair's offset within word i
                if 0 <= lo < 32:
                    w[i] |= (pair << lo) & 0xFFFFFFFF
                if -2 * bits < lo < 0:
                    w[i] |= pair >> (-lo)
        lanes.append(w)
    ored = [lanes[0][i] | lanes[1][i] | lanes[2][i] | lanes[3][i] for i in range(bits)]
    stored = [None] * bits
    for q in range(4):
        for i in range(bits):
            if i % 4 == q:
                stored[i] = ored[i]
    np.testing.assert_array_equal(np.array(stored, dtype=np.uint32), O.pack_codes(codes, bits))
