"""Subtractive dither for every lattice (Methodology step 4: U ~ Uniform(V(Lambda)), added before
quantization and subtracted after).  Pins that do not reuse the oracle's own arithmetic:

* every dither vector lies in the Voronoi cell of the lattice point 0 (its nearest point is 0, by
  brute force over the lattice points around it);
* the dithered error per dimension is the lattice's normalised second moment times V^(2/d), a
  closed form: Z 1/12, A2 (minimum distance 1) 5/72, D4 13/120, E8 929/12960;
* the reconstruction is unbiased per vector over independent seeds;
* the D4 dither is unchanged from the KV path's group definition.
"""
import itertools

import numpy as np
import pytest

import oracle

SQ3 = np.sqrt(3.0)
SECOND_MOMENT = {oracle.Z: 1.0 / 12.0, oracle.A2: 5.0 / 72.0, oracle.D4: 13.0 / 120.0, oracle.E8: 929.0 / 12960.0}


def _to_u(lattice, P):
    """quantizer coordinates -> u coordinates (only A2 differs: (P, Q) -> (P/2, Q sqrt(3)/2))"""
    P = np.asarray(P, dtype=np.float64)
    if lattice != oracle.A2:
        return P
    out = P.copy()
    out[..., 0::2] *= 0.5
    out[..., 1::2] *= SQ3 / 2.0
    return out


def _points(lattice, v):
    """integer embedding -> lattice point in u coordinates"""
    v = np.asarray(v, dtype=np.float64)
    if lattice == oracle.E8:
        return 0.5 * v
    return _to_u(lattice, v)


def _near_points(lattice):
    """lattice points (u coordinates) of one block within distance 1.5 of the origin"""
    d = oracle.LATTICE_DIM[lattice]
    if lattice == oracle.Z:
        return np.array([[-1.0], [0.0], [1.0]])
    if lattice == oracle.A2:
        pts = [(P / 2.0, Q * SQ3 / 2.0) for P in range(-3, 4) for Q in range(-2, 3) if (P - Q) % 2 == 0]
        return np.array(pts)
    if lattice == oracle.D4:
        pts = [p for p in itertools.product(range(-1, 2), repeat=4) if sum(p) % 2 == 0]
        return np.array(pts, dtype=np.float64)
    pts = [p for p in itertools.product(range(-1, 2), repeat=8) if sum(p) % 2 == 0]
    half = [tuple(x / 2.0 for x in p) for p in itertools.product((-1, 1), repeat=8) if sum(p) % 4 == 0]
    return np.array(pts + half, dtype=np.float64)


@pytest.mark.parametrize("lattice", [oracle.Z, oracle.A2, oracle.D4, oracle.E8])
def test_dither_lies_in_the_voronoi_cell(lattice):
    d = oracle.LATTICE_DIM[lattice]
    near = _near_points(lattice)
    for c in range(40):
        U = _to_u(lattice, oracle.dither(lattice, 11, 3, c, 128)).reshape(-1, d)
        dist = ((U[:, None, :] - near[None, :, :]) ** 2).sum(-1)
        d0 = (U ** 2).sum(-1)
        assert np.all(d0 <= dist.min(1) + 1e-6)
        assert np.max(np.abs(U)) <= 1.0


@pytest.mark.parametrize("lattice", [oracle.Z, oracle.A2, oracle.D4, oracle.E8])
def test_dithered_error_has_the_cells_second_moment(lattice):
    rng = np.random.default_rng(5)
    tiles, n = 2048, 128
    u = (rng.standard_normal((tiles, n)) * 3.0).astype(np.float32)
    v, *_ = oracle.quantize_coeffs(u, n, lattice, seed=9, kv=True, kv_S=tiles)
    U = np.stack([_to_u(lattice, oracle.dither(lattice, 9, 0, t, n)) for t in range(tiles)])
    err = _points(lattice, v) - U - u.astype(np.float64)
    mse = np.mean(err ** 2)
    assert abs(mse / SECOND_MOMENT[lattice] - 1.0) < 0.01, mse


@pytest.mark.parametrize("lattice", [oracle.Z, oracle.A2, oracle.E8])
def test_dithered_reconstruction_is_unbiased_per_vector(lattice):
    rng = np.random.default_rng(8)
    tiles, n, M = 16, 64, 400
    u = (rng.standard_normal((tiles, n)) * 1.5).astype(np.float32)
    acc = np.zeros((M, tiles, n))
    for m in range(M):
        v, *_ = oracle.quantize_coeffs(u, n, lattice, seed=1000 + m, kv=True, kv_S=tiles)
        U = np.stack([_to_u(lattice, oracle.dither(lattice, 1000 + m, 0, t, n)) for t in range(tiles)])
        acc[m] = _points(lattice, v) - U - u
    z = acc.mean(0) / (acc.std(0) / np.sqrt(M))
    assert np.mean(np.abs(z) > 4.0) < 1e-3
    # the same inputs without the dither: rounding errors are a fixed function of u
    v0, *_ = oracle.quantize_coeffs(u, n, lattice, seed=1000, kv=False)
    assert np.max(np.abs(_points(lattice, v0) - u)) > 0.1


def test_d4_group_dither_is_the_kv_block_dither():
    for g in range(8):
        assert np.array_equal(oracle.dither(oracle.D4, 7, 5, 99, 32)[4 * g:4 * g + 4], oracle.dither_d4(7, 5, 99, g))


def test_token_append_tiles_equal_the_whole_sequence_tiles():
    # appending token s0 of every (b, h) draws the dither a whole-sequence encode draws for it:
    # tile for tile, the codes and reconstructions agree (Methodology step 4, fresh U per vector)
    from post_quantization_tile_b200 import workloads as W
    B, H, S, D = 1, 3, 40, 128
    kb = W.kv_keys(B, H, S, D, seed=12)
    full = oracle.encode(kb.reshape(-1, D), D, oracle.D4, 0.9, 5, kv=True, kv_S=S, want_codes=True)
    xf, _ = oracle.decode(full)
    for s0 in (0, 7, 39):
        step = np.ascontiguousarray(kb[:, :, s0, :].reshape(-1, D))        # [B*H, D]: one token per head
        app = oracle.encode(step, D, oracle.D4, 0.9, 5, kv=True, kv_S=1, want_codes=True, kv_s0=s0)
        rows = np.arange(B * H) * S + s0
        np.testing.assert_array_equal(app.v, full.v[rows])
        np.testing.assert_array_equal(app.meta, full.meta[rows])
        xa, _ = oracle.decode(app)
        np.testing.assert_array_equal(xa, xf[rows])


def test_dither_draws_sixteen_bit_midpoints_from_one_philox_block_per_group_pair():
    """The dither reading: groups 2b and 2b + 1 of a tile share the Philox4x32-10 block with counter
    (c, c1, 0x80000000 | b, 0) (the generator pinned to curand's elsewhere); its eight 16-bit
    halves, low half first, give r = box (h + 1/2) 2^-16.  On Z (box 1) U = r - rint(r), so r is U
    taken mod 1; its 2^17 r are odd integers, the bins' midpoints."""
    seed, c1, c, n = 0x5EED, 3, 1234, 64
    U = oracle.dither(oracle.Z, seed, c1, c, n).astype(np.float64)
    r = np.where(U < 0, U + 1.0, U)
    odd = r * 2.0 ** 17
    assert np.all(odd == np.round(odd)) and np.all(np.round(odd) % 2 == 1)
    for g in range(n // 4):
        w = oracle.philox([c, c1, 0x80000000 | (g >> 1), 0], seed & 0xFFFFFFFF, seed >> 32)
        halves = [(int(w[j >> 1]) >> (16 * (j & 1))) & 0xFFFF for j in range(8)]
        want = [(2 * h + 1) * 2.0 ** -17 for h in halves[4 * (g & 1):4 * (g & 1) + 4]]
        np.testing.assert_array_equal(r[4 * g:4 * g + 4], want)
