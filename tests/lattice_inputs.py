"""Seeded inputs for the nearest-point tests: random points, points on and near the facets of
Voronoi cells (coset and neighbour ties), and blocks whose fix-up chooses among rounding errors
below 2^-31.  Only random draws and lattice geometry from the definitions (Conway & Sloane,
"Sphere Packings, Lattices and Groups", ch. 4); no quantizer arithmetic."""
import numpy as np

import oracle

SQ3_2 = np.sqrt(3.0) / 2.0


def random_inputs(d, count, seed):
    rng = np.random.default_rng(seed)
    k = count // 4
    return np.concatenate([
        rng.uniform(-40.0, 40.0, size=(k, d)),
        rng.standard_normal((k, d)) * 6.0,
        rng.uniform(-1.0, 1.0, size=(k, d)),
        rng.standard_normal((count - 3 * k, d)) * 300.0,
    ]).astype(np.float32)


def facet_ties(lattice, count, seed):
    """Points on (and within a few 1e-6 of) the bisector of a lattice point and a neighbour: the
    midpoint of a minimal vector r, moved within the facet by w (w . r = 0) and across it by eps r."""
    rng = np.random.default_rng(seed)
    d = oracle.LATTICE_DIM[lattice]
    if lattice == oracle.E8:
        a = rng.integers(-6, 7, size=(count, 8)).astype(np.float64)
        a[:, 7] += np.sum(a, axis=1) % 2                      # D8: even sum
        half = rng.random(count) < 0.5
        a[half] += 0.5                                        # half of them from the D8 + 1/2 coset
        kind = rng.random(count) < 0.5
        s = rng.choice([-1.0, 1.0], size=(count, 8))
        s[:, 7] *= np.prod(s, axis=1)                         # even number of -1: s / 2 in D8 + 1/2
        r = 0.5 * s                                           # half of the minimal vectors (+-1/2)^8
        ij = np.array([rng.choice(8, 2, replace=False) for _ in range(count)])
        r2 = np.zeros((count, 8))
        r2[np.arange(count), ij[:, 0]] = rng.choice([-1.0, 1.0], size=count)
        r2[np.arange(count), ij[:, 1]] = rng.choice([-1.0, 1.0], size=count)
        r = np.where(kind[:, None], r, r2)                    # and the (+-1, +-1, 0^6) ones
        base = a
    elif lattice == oracle.D4:
        base = rng.integers(-6, 7, size=(count, 4)).astype(np.float64)
        base[:, 3] += np.sum(base, axis=1) % 2
        ij = np.array([rng.choice(4, 2, replace=False) for _ in range(count)])
        r = np.zeros((count, 4))
        r[np.arange(count), ij[:, 0]] = rng.choice([-1.0, 1.0], size=count)
        r[np.arange(count), ij[:, 1]] = rng.choice([-1.0, 1.0], size=count)
    else:
        ab = rng.integers(-8, 9, size=(count, 2)).astype(np.float64)
        base = np.stack([ab[:, 0] + ab[:, 1] / 2.0, ab[:, 1] * SQ3_2], axis=1)
        ang = rng.integers(0, 6, size=count) * np.pi / 3.0
        r = np.stack([np.cos(ang), np.sin(ang)], axis=1)
    g = rng.standard_normal((count, d))
    w = g - (np.sum(g * r, axis=1) / np.sum(r * r, axis=1))[:, None] * r
    w *= (rng.uniform(0.0, 0.2, size=count) / np.maximum(np.linalg.norm(w, axis=1), 1e-30))[:, None]
    w[rng.random(count) < 0.25] = 0.0                         # facet centres
    eps = rng.choice([0.0, 1e-7, -1e-7, 5e-7, -5e-7, 2e-6, -2e-6, 1e-5, -1e-5], size=count)
    return (base + 0.5 * r + w + eps[:, None] * r).astype(np.float32)


def small_error_blocks(lattice, count, seed):
    """Blocks where a fix-up chooses among rounding errors below 2^-31 (2^-32 .. 2^-45, or 0):
    integers plus tiny offsets with an odd sum (D4, and E8's even coset), and for E8 also
    half-integer points with two or three coordinates replaced by integers plus tiny offsets, so
    that the odd coset wins and its fix-up picks among those coordinates."""
    rng = np.random.default_rng(seed)
    d = oracle.LATTICE_DIM[lattice]
    tiny = np.where(rng.random((count, d)) < 0.2, 0.0,
                    rng.choice([-1.0, 1.0], size=(count, d)) * 2.0 ** -rng.integers(32, 46, size=(count, d)))
    ints = rng.integers(-3, 4, size=(count, d)).astype(np.float64)
    ints[:, 0] += 1 - np.sum(ints, axis=1) % 2                 # odd sum
    u = ints + tiny
    if lattice == oracle.E8:
        h = np.nonzero(rng.random(count) < 0.5)[0]
        halves = rng.integers(-3, 4, size=(h.size, 8)) + 0.5
        k = rng.integers(2, 4, size=h.size)           # 2 or 3: the odd coset wins clearly
        for row, kk in zip(range(h.size), k):
            cols = rng.choice(8, kk, replace=False)
            halves[row, cols] = ints[h[row], cols] + tiny[h[row], cols]
        u[h] = halves
    return u.astype(np.float32)
