"""The parity comparator (oracle/parity.py) that the GPU tests and the benchmark use: identical
codes take the fast path; a code that differs only in a block within 1e-6 of a Voronoi boundary
is counted as a boundary disagreement; a block that differs farther from the boundary, or a
chunk that differs without such a block, fails."""
import numpy as np

import oracle
from oracle import parity
from lattice_inputs import facet_ties


def _code(u, v, meta, cw, bits, n, lattice):
    tiles = u.shape[0]
    c = oracle.Code(tiles, n, n, lattice, 1.0, 0, 0, 0, None, meta, cw, bits, 0, v, u)
    return c


def _setup(shift):
    n, lattice = 128, oracle.E8
    rng = np.random.default_rng(5)
    u = (rng.standard_normal((70, n)) * 3.0).astype(np.float32)       # 70 tiles: 3 chunks
    # one E8 block on a coset facet, pushed across it by `shift` in the second code
    tie = facet_ties(lattice, 400, 11)
    v0 = oracle.quantize_blocks(lattice, tie)
    # pick a facet point whose decision flips under a 2e-7 push along the neighbour direction
    for i in range(tie.shape[0]):
        for sgn in (1.0, -1.0):
            w = tie[i].astype(np.float64)
            g = w - np.round(w * 2) / 2
            moved = (tie[i] + np.float32(sgn * shift) * np.sign(g + 1e-12)).astype(np.float32)
            if not np.array_equal(oracle.quantize_blocks(lattice, moved[None])[0], v0[i]):
                u_a = u.copy()
                u_a[40, 16:24] = tie[i]
                u_b = u.copy()
                u_b[40, 16:24] = moved
                return n, lattice, u_a, u_b
    raise AssertionError("no flipping facet point found")


def test_identical_codes_take_the_fast_path():
    n, lattice = 128, oracle.E8
    u = (np.random.default_rng(1).standard_normal((40, n)) * 2).astype(np.float32)
    v, meta, cw, bits, _ = oracle.quantize_coeffs(u, n, lattice)
    ref = _code(u, v, meta, cw, bits, n, lattice)
    rep = parity.compare(None, meta, cw, bits, ref)
    assert rep.identical and rep.ok and rep.disagreements == 0 and rep.blocks == 40 * 16


def test_near_boundary_block_is_counted_and_far_one_fails():
    n, lattice, u_a, u_b = _setup(3e-7)
    va, ma, ca, ba, _ = oracle.quantize_coeffs(u_a, n, lattice)
    vb, mb, cb, bb, _ = oracle.quantize_coeffs(u_b, n, lattice)
    assert not np.array_equal(va, vb)
    ref = _code(u_a, va, ma, ca, ba, n, lattice)
    rep = parity.compare(None, mb, cb, bb, ref)
    assert not rep.identical
    assert rep.disagreements == 1 and not rep.failures, rep.failures
    assert rep.worst_margin <= 1e-6
    # the same device code against coefficients that put the block far from the boundary fails
    u_far = u_a.copy()
    u_far[40, 16:24] = np.round(u_a[40, 16:24] * 2) / 2 + 0.01
    vf, mf, cf, bf, _ = oracle.quantize_coeffs(u_far, n, lattice)
    rep = parity.compare(None, mb, cb, bb, _code(u_far, vf, mf, cf, bf, n, lattice))
    assert rep.failures


def test_differing_chunk_without_a_boundary_block_fails():
    n, lattice = 128, oracle.E8
    u = (np.random.default_rng(2).standard_normal((70, n)) * 3).astype(np.float32)
    v, meta, cw, bits, _ = oracle.quantize_coeffs(u, n, lattice)
    ref = _code(u, v, meta, cw, bits, n, lattice)
    bad = bits.copy()
    bad[int(cw[2]) + 3] ^= 0x10           # a flipped bit inside chunk 2
    rep = parity.compare(None, meta, cw, bad, ref)
    assert rep.failures and not rep.ok
