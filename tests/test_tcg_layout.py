"""The per-group tensor-core ring's lane layout, checked on the CPU.

The kernel's header states the mapping: lane (g, t) of a warp holds quarter t
of every group of rows g and g + 8 (G/4 codes, read from a ring stage whose
128-byte rows are stored with the 128-byte swizzle); step 2w + h of a group
takes the code pairs (n_2h, n_2h+4) as A columns (2t, 2t + 1) and
(n_2h+1, n_2h+5) as A columns (2t + 8, 2t + 9) of word w; the B fragment of
that step is {x[k0 + 2h], x[k0 + 2h + 4]}, {x[k0 + 2h + 1], x[k0 + 2h + 5]}.
Here those rules build the m16n8k16 operands lane by lane (the PTX fragment
layout of mma.sync.m16n8k16.row.col), multiply them as the MMA does and check
that every group's D equals the group's exact dot product: a wrong quarter,
pair, swizzle or fragment order fails.  Integer-valued x keeps every sum exact.
No GPU and no part of the CUDA path is used.
"""
from __future__ import annotations

import numpy as np
import pytest


def _ring_stage(codes, G, ROWS):
    """A ring stage as the tensor copies lay it out: the packed rows (LSB
    first) in 128-byte boxes, chunk c of row r at chunk c ^ (r % 8)."""
    SKB = 8 * G // 2
    packed = np.zeros((ROWS, SKB), np.uint8)
    for k in range(8 * G):
        packed[:, k // 2] |= (codes[:, k] << (4 * (k % 2))).astype(np.uint8)
    st = np.zeros((SKB // 128) * ROWS * 128, np.uint8)
    for b in range(SKB // 128):
        for r in range(ROWS):
            for c in range(8):
                dst = b * ROWS * 128 + r * 128 + (c ^ (r % 8)) * 16
                st[dst:dst + 16] = packed[r, b * 128 + c * 16: b * 128 + c * 16 + 16]
    return st


def _word(st, off):
    return int.from_bytes(bytes(st[off:off + 4]), "little")


def _pair(word, i):
    v = word >> (4 * i)
    return v & 0xF, (v >> 16) & 0xF


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("NT,M", [(1, 8), (1, 3), (2, 13), (4, 32)])
def test_fragments_give_each_groups_dot_product(G, NT, M):
    rng = np.random.default_rng(G * 100 + NT * 10 + M)
    wr, QB, NWD = 2, G // 8, G // 32
    ROWS = 16 * wr
    codes = rng.integers(0, 16, size=(ROWS, 8 * G))
    x = rng.integers(-8, 9, size=(8 * NT, 8 * G)).astype(np.float64)
    x[M:] = 0.0                                  # x rows past M are staged as zeros
    st = _ring_stage(codes, G, ROWS)
    for wrid in range(wr):
        for gl in range(8):
            D = np.zeros((NT, 16, 8))
            for w in range(NWD):
                for h in range(2):
                    A = np.full((16, 16), np.nan)
                    B = np.full((NT, 16, 8), np.nan)
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        rg = wrid * 16 + g
                        bo = gl * (G // 2) + t * QB
                        pc = ((((bo & 127) >> 4) ^ (rg & 7)) << 4) | (bo & 15)
                        pg = (bo >> 7) * ROWS * 128 + rg * 128 + pc
                        for rrow, off in ((g, pg), (g + 8, pg + 8 * 128)):
                            wd = _word(st, off + 4 * w)
                            A[rrow, 2 * t], A[rrow, 2 * t + 1] = _pair(wd, 2 * h)
                            A[rrow, 2 * t + 8], A[rrow, 2 * t + 9] = _pair(wd, 2 * h + 1)
                        k0 = gl * G + t * (G // 4) + 8 * w
                        for nt in range(NT):
                            xr = x[nt * 8 + g]
                            B[nt, 2 * t, g], B[nt, 2 * t + 1, g] = xr[k0 + 2 * h], xr[k0 + 2 * h + 4]
                            B[nt, 2 * t + 8, g], B[nt, 2 * t + 9, g] = xr[k0 + 2 * h + 1], xr[k0 + 2 * h + 5]
                    assert not np.isnan(A).any() and not np.isnan(B).any()   # every element placed once
                    for nt in range(NT):
                        D[nt] += A @ B[nt]
            rows = slice(wrid * 16, wrid * 16 + 16)
            want = codes[rows, gl * G:(gl + 1) * G] @ x[:, gl * G:(gl + 1) * G].T
            for nt in range(NT):
                assert np.array_equal(D[nt], want[:, nt * 8:(nt + 1) * 8]), (wrid, gl, nt)


def test_swizzled_reads_hit_distinct_banks():
    """The 32 lanes' 8-byte code loads of one group (G = 64) touch every
    4-byte bank exactly twice, the minimum for 256 bytes: no bank conflict."""
    G, ROWS, QB = 64, 32, 8
    for gl in range(8):
        banks = []
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            bo = gl * (G // 2) + t * QB
            pc = ((((bo & 127) >> 4) ^ (g & 7)) << 4) | (bo & 15)
            addr = (bo >> 7) * ROWS * 128 + g * 128 + pc
            banks += [(addr // 4) % 32, (addr // 4 + 1) % 32]
        assert sorted(banks) == sorted(list(range(32)) * 2), gl
