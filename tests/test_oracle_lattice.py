"""Pins for the oracle's lattice decoders (E8, D4, A2, Z) and bit-stripping.

The oracle's closest-point rules are checked against
  * brute-force search over every lattice point in a box of neighbouring candidates (float64),
    on random inputs and on constructed near-ties;
  * textbook facts from Conway & Sloane, "Sphere Packings, Lattices and Groups" (golden file
    tests/golden/lattice_constants.json): lattice points are fixed points, the minimal vectors
    number 240 (E8), 24 (D4), 6 (A2), and the mean squared error per dimension on inputs spread
    uniformly over whole cells equals G * V^(2/d).
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "lattice_constants.json")))
SQ3_2 = np.sqrt(3.0) / 2.0


def to_points(lattice, v):
    """Integer embedding -> lattice point in u units (float64)."""
    v = np.asarray(v, dtype=np.float64)
    if lattice == oracle.E8:
        return v / 2.0
    if lattice == oracle.A2:
        p = v.copy()
        p[..., 0] *= 0.5
        p[..., 1] *= SQ3_2
        return p
    return v


# ---------------------------------------------------------------------------------------------
# brute force (float64), independent of the oracle
# ---------------------------------------------------------------------------------------------
def _box(d, lo, hi):
    return np.array(list(itertools.product(range(lo, hi + 1), repeat=d)), dtype=np.float64)


def brute_d8_union(u, half, offs):
    """nearest point of D8 (+1/2 if half) to each row of u among floor-based offsets."""
    sh = 0.5 if half else 0.0
    base = np.floor(u - sh)
    best_d = np.full(u.shape[0], np.inf)
    best_p = np.zeros_like(u)
    for i in range(u.shape[0]):
        cand = base[i] + offs + sh
        par = np.sum(cand - sh, axis=1) % 2 == 0
        cand = cand[par]
        d = np.sum((cand - u[i]) ** 2, axis=1)
        j = np.argmin(d)
        best_d[i], best_p[i] = d[j], cand[j]
    return best_d, best_p


def brute_e8(u, offs):
    dA, pA = brute_d8_union(u, False, offs)
    dB, pB = brute_d8_union(u, True, offs)
    take_b = dB < dA
    return np.where(take_b, dB, dA), np.where(take_b[:, None], pB, pA)


def brute_d4(u, offs):
    base = np.floor(u)
    best_d = np.zeros(u.shape[0])
    for i in range(u.shape[0]):
        cand = base[i] + offs
        cand = cand[np.sum(cand, axis=1) % 2 == 0]
        best_d[i] = np.min(np.sum((cand - u[i]) ** 2, axis=1))
    return best_d


def brute_a2(u):
    best = np.full(u.shape[0], np.inf)
    for i in range(u.shape[0]):
        b0 = int(np.round(u[i, 1] / SQ3_2))
        for b in range(b0 - 3, b0 + 4):
            a0 = int(np.round(u[i, 0] - b / 2.0))
            for a in range(a0 - 3, a0 + 4):
                p = np.array([a + b / 2.0, b * SQ3_2])
                best[i] = min(best[i], np.sum((p - u[i]) ** 2))
    return best


def in_lattice(lattice, v):
    v = np.asarray(v, dtype=np.int64)
    if lattice == oracle.Z:
        return np.ones(v.shape[0], dtype=bool)
    if lattice == oracle.D4:
        return np.sum(v, axis=1) % 2 == 0
    if lattice == oracle.A2:
        return (v[:, 0] - v[:, 1]) % 2 == 0
    same_parity = np.all((v % 2) == (v[:, :1] % 2), axis=1)
    return same_parity & (np.sum(v, axis=1) % 4 == 0)


def _inputs(d, count, seed, spread):
    rng = np.random.default_rng(seed)
    u = np.concatenate([
        rng.uniform(-spread, spread, size=(count, d)),
        rng.standard_normal((count, d)) * spread / 3,
        rng.uniform(-1, 1, size=(count, d)),
    ]).astype(np.float32)
    return u


def _near_ties(lattice, count, seed):
    """midpoints between a lattice point and a neighbour, nudged by +-1 ulp-ish amounts"""
    rng = np.random.default_rng(seed)
    d = oracle.LATTICE_DIM[lattice]
    base = oracle.quantize_blocks(lattice, rng.uniform(-6, 6, size=(count, d)).astype(np.float32))
    p0 = to_points(lattice, base)
    if lattice == oracle.E8:
        nbrs = [np.full(8, 0.5) * s for s in (1, -1)] + [np.eye(8)[i] + np.eye(8)[j] for i in range(8) for j in range(i + 1, 8)]
    elif lattice == oracle.D4:
        nbrs = [np.eye(4)[i] + s * np.eye(4)[j] for i in range(4) for j in range(i + 1, 4) for s in (1, -1)]
    elif lattice == oracle.A2:
        nbrs = [np.array([1.0, 0.0]), np.array([0.5, SQ3_2]), np.array([-0.5, SQ3_2])]
    else:
        nbrs = [np.array([1.0])]
    nb = np.array(nbrs)[rng.integers(0, len(nbrs), size=count)]
    mid = p0 + 0.5 * nb
    jitter = rng.choice([-1, 0, 1], size=(count, 1)) * rng.uniform(0, 1e-6, size=(count, 1)) * nb
    return (mid + jitter).astype(np.float32)


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.D4, oracle.A2, oracle.Z])
def test_nearest_point_matches_brute_force(lattice):
    d = oracle.LATTICE_DIM[lattice]
    u = np.concatenate([_inputs(d, 150, 1 + lattice, 12.0), _near_ties(lattice, 150, 50 + lattice)])
    v = oracle.quantize_blocks(lattice, u)
    assert np.all(in_lattice(lattice, v))
    p = to_points(lattice, v)
    u64 = u.astype(np.float64)
    got = np.sum((p - u64) ** 2, axis=1)
    if lattice == oracle.E8:
        best, _ = brute_e8(u64, _box(8, -1, 2))
    elif lattice == oracle.D4:
        best = brute_d4(u64, _box(4, -2, 3))
    elif lattice == oracle.A2:
        best = brute_a2(u64)
    else:
        best = (u64[:, 0] - np.round(u64[:, 0])) ** 2
    # binary32 decisions: the chosen point may lose only within rounding of a tie
    assert np.all(got <= best + 1e-6 * (1.0 + np.abs(u64).max(axis=1)))


def test_e8_many_points_corner_search():
    rng = np.random.default_rng(9)
    u = (rng.standard_normal((4000, 8)) * 4).astype(np.float32)
    v = oracle.quantize_blocks(oracle.E8, u)
    p = to_points(oracle.E8, v)
    best, bp = brute_e8(u.astype(np.float64), _box(8, 0, 1))
    got = np.sum((p - u) ** 2, axis=1)
    assert np.all(got <= best + 1e-6)
    # away from ties the point itself is the brute-force one
    np.testing.assert_array_equal(p[got < best - 0 + 1e-3], bp[got < best - 0 + 1e-3])


@pytest.mark.parametrize("name,lattice", [("E8", oracle.E8), ("D4", oracle.D4), ("A2", oracle.A2), ("Z", oracle.Z)])
def test_lattice_points_are_fixed_and_minimal_vectors_counted(name, lattice):
    d = oracle.LATTICE_DIM[lattice]
    # all lattice points with norm^2 = min norm, enumerated from the definitions
    if lattice == oracle.E8:
        ints = [np.array(c, float) for c in itertools.product([-1, 0, 1], repeat=8) if sum(map(abs, c)) == 2]
        halves = [np.array(c) * 0.5 for c in itertools.product([-1, 1], repeat=8) if sum(1 for x in c if x < 0) % 2 == 0]
        mins = np.array(ints + halves)
    elif lattice == oracle.D4:
        mins = np.array([c for c in itertools.product([-1, 0, 1], repeat=4) if sum(map(abs, c)) == 2], float)
    elif lattice == oracle.A2:
        mins = np.array([[np.cos(k * np.pi / 3), np.sin(k * np.pi / 3)] for k in range(6)])
    else:
        mins = np.array([[1.0], [-1.0]])
    assert len(mins) == GOLD["kissing"][name]
    assert np.allclose(np.sum(mins ** 2, axis=1), GOLD["min_norm_sq"][name])
    v = oracle.quantize_blocks(lattice, mins.astype(np.float32))
    np.testing.assert_allclose(to_points(lattice, v), mins, atol=1e-6)
    # slightly shrunk minimal vectors still decode to themselves; the origin to itself
    v2 = oracle.quantize_blocks(lattice, (0.9 * mins).astype(np.float32))
    np.testing.assert_allclose(to_points(lattice, v2), mins, atol=1e-6)
    assert np.all(oracle.quantize_blocks(lattice, np.zeros((1, d), np.float32)) == 0)


def _uniform_cells(lattice, count, seed):
    """u uniform over a box that is an exact union of fundamental domains"""
    rng = np.random.default_rng(seed)
    d = oracle.LATTICE_DIM[lattice]
    if lattice == oracle.A2:
        x = rng.uniform(-40, 40, size=count)
        y = rng.uniform(-40 * np.sqrt(3), 40 * np.sqrt(3), size=count)
        return np.stack([x, y], axis=1).astype(np.float32)
    return rng.uniform(-40, 40, size=(count, d)).astype(np.float32)


@pytest.mark.parametrize("name,lattice", [("E8", oracle.E8), ("D4", oracle.D4), ("A2", oracle.A2), ("Z", oracle.Z)])
def test_normalised_second_moment(name, lattice):
    d = oracle.LATTICE_DIM[lattice]
    count = 2 ** 20 // d
    u = _uniform_cells(lattice, count, 77)
    tiles = u.reshape(-1, 128)
    v, _, _, _, st = oracle.quantize_coeffs(tiles, 128, lattice)
    assert st == 0
    p = to_points(lattice, v.reshape(-1, d))
    mse = np.mean((p - u.astype(np.float64)) ** 2)
    expect = GOLD["G"][name] * GOLD["volume"][name] ** (2.0 / d)
    assert abs(mse / expect - 1.0) < 0.006, (mse, expect)


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.D4, oracle.A2, oracle.Z])
def test_strip_is_a_bijection(lattice):
    rng = np.random.default_rng(3)
    d = oracle.LATTICE_DIM[lattice]
    v = oracle.quantize_blocks(lattice, rng.uniform(-30, 30, size=(5000, d)).astype(np.float32))
    sym, cos = oracle.strip(lattice, v)
    np.testing.assert_array_equal(oracle.unstrip(lattice, sym, cos), v)
    # distinct lattice points never share symbols (lossless)
    keys = {tuple(s) + (c,) for s, c in zip(sym.tolist(), cos.tolist())}
    assert len(keys) == len({tuple(x) for x in v.tolist()})
    # stripping removes the parity-fixed bits: symbols are about half the size for the
    # checked coordinate (D4 last, E8 last) and E8 halves every coordinate
    if lattice == oracle.E8:
        assert np.all(np.abs(sym[:, :7]) <= np.abs(v[:, :7]) // 2 + 1)
        assert set(np.unique(cos)) <= {0, 1}
