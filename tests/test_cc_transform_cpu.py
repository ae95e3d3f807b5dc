"""The index algebra of the CUDA-core block transform (h = 1024), on the CPU.

The fused layer kernel's producer warps transform a block of h = 1024 rotated
coordinates as Z = H_32 Y H_32 with Y[a][b] = y[32 a + b] (Sylvester's
H_1024 = H_32 (x) H_32): lane l gathers column b = l through pi, runs H_32
over a in registers, writes its column into the warp's 32 x 32 shared-memory
tile as row l of the transpose (16-byte chunk c at chunk position c ^ (l & 7)),
reads row a = l back (word b * 32 + 4 ((l >> 2) ^ (b & 7)) + (l & 3)), and
runs H_32 over b, so that it ends with Z[l][0..31], the 32 consecutive
positions 32 l .. 32 l + 31 of the block.

This emulates those steps lane by lane in numpy, with the gather table laid
out as the library builds it (entry (w * 32 + lane) * 32 + a is twice the
input channel of in-block position 32 a + lane of block w) and read as the
kernel reads it (eight 16-bit offsets per 16-byte word, low half first), and
checks the result against the Walsh-Hadamard transform of the permuted row.
It also checks that both directions of the swizzled transpose are free of
shared-memory bank conflicts.  It pins the derivation the kernel's indexing
follows; the kernel itself is checked against the oracle on the GPU."""

import numpy as np
import pytest

import oracle as O


def _fwht_rows(v):
    """In-register butterflies on the last axis, strides 16, 8, 4, 2, 1 (the
    kernel's five stages): the unnormalised Sylvester transform."""
    v = v.copy()
    for s in (16, 8, 4, 2, 1):
        for i in range(32):
            if i & s == 0:
                a, b = v[..., i].copy(), v[..., i + s].copy()
                v[..., i], v[..., i + s] = a + b, a - b
    return v


def _gather_table(d, perm):
    """Byte offsets in the staged row: entry (w * 32 + lane) * 32 + a."""
    g = np.zeros(d, dtype=np.uint16)
    for w in range(d // 1024):
        for lane in range(32):
            for a in range(32):
                g[(w * 32 + lane) * 32 + a] = 2 * perm[w * 1024 + 32 * a + lane]
    return g


def _lane_column(g, w, lane, x):
    """The 32 values lane `lane` of warp `w` gathers: words qq of its table
    row (uint4 = four uint32 = eight uint16), offsets from the low half
    first, each a bf16 value of the staged row at byte offset off."""
    words = g[(w * 32 + lane) * 32:(w * 32 + lane) * 32 + 32].astype(np.uint32)
    v = np.zeros(32)
    for qq in range(4):
        gw = [words[8 * qq + 2 * hp] | (words[8 * qq + 2 * hp + 1] << 16) for hp in range(4)]
        for hp in range(4):
            v[8 * qq + 2 * hp] = x[(gw[hp] & 0xFFFF) // 2]
            v[8 * qq + 2 * hp + 1] = x[(gw[hp] >> 16) // 2]
    return v


def _write_addr(lane, c):
    return lane * 128 + ((c ^ (lane & 7)) << 4)          # 16-byte store of chunk c of the column


def _read_addr(lane, b):
    return b * 128 + (((lane >> 2) ^ (b & 7)) << 4) + ((lane & 3) << 2)   # 4-byte load of Qt[b][lane]


@pytest.mark.parametrize("d", [1024, 3072])
def test_cc_transform_matches_block_hadamard(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal(d)
    perm = O.rpbh_permutation(d, 0)
    g = _gather_table(d, perm)
    y = x[perm]                                           # the gather the method defines
    for w in range(d // 1024):
        tile = np.zeros(32 * 32)                          # fp32 words
        for lane in range(32):
            v = _fwht_rows(_lane_column(g, w, lane, x))   # H_32 over a for column b = lane
            for c in range(8):
                at = _write_addr(lane, c) // 4
                tile[at:at + 4] = v[4 * c:4 * c + 4]
        Z = np.zeros((32, 32))
        for lane in range(32):
            row = np.array([tile[_read_addr(lane, b) // 4] for b in range(32)])
            Z[lane] = _fwht_rows(row)                     # H_32 over b: row a = lane of Z
        want = O.sylvester_hadamard(1024) @ y[w * 1024:(w + 1) * 1024]
        np.testing.assert_allclose(Z.reshape(-1), want, rtol=1e-12, atol=1e-9)


def test_cc_transpose_is_bank_conflict_free():
    # a warp's 16-byte stores of chunk c take 4 wavefronts of 8 lanes; each
    # wavefront's 8 chunks must cover all 32 banks once.  A warp's 4-byte
    # loads of row b must hit 32 distinct banks.
    for c in range(8):
        for q in range(4):
            banks = set()
            for lane in range(8 * q, 8 * q + 8):
                a = _write_addr(lane, c)
                banks.update(((a // 4) + k) % 32 for k in range(4))
            assert len(banks) == 32
    for b in range(32):
        assert len({(_read_addr(lane, b) // 4) % 32 for lane in range(32)}) == 32


def test_cc_emulation_catches_an_unswizzled_read():
    # reading the tile without the swizzle must not reproduce the transform
    d = 1024
    x = np.random.default_rng(1).standard_normal(d)
    perm = O.rpbh_permutation(d, 0)
    g = _gather_table(d, perm)
    tile = np.zeros(32 * 32)
    for lane in range(32):
        v = _fwht_rows(_lane_column(g, 0, lane, x))
        for c in range(8):
            at = _write_addr(lane, c) // 4
            tile[at:at + 4] = v[4 * c:4 * c + 4]
    Z = np.stack([_fwht_rows(np.array([tile[b * 32 + lane] for b in range(32)])) for lane in range(32)])
    assert not np.allclose(Z.reshape(-1), O.sylvester_hadamard(1024) @ x[perm])
