"""Pins the oracle's nearest-point rules (E8, D4, A2) against an exhaustive search on 10^6 random
inputs per lattice plus constructed near-ties.

The search (tests/lattice_search.c, binary64) enumerates every lattice point within the covering
radius of the input, so its minimum is the true nearest distance.  The oracle decides in binary32,
so it may pick another point only where the input is within rounding of a Voronoi boundary.  The
pin: every oracle point is a lattice point and is either the search's point or one whose
boundary margin (d_oracle - d_best) / (2 |p_oracle - p_best|) is at most 1e-6 max(1, |u|_max)
(u units: binary32 rounds the coordinates relative to their size, and A2's (P, Q) = (2 u0, u1 K)
change of coordinates does so before the decision); those disagreements are counted and stay a
small fraction.  A dropped fix-up, a wrong coset, an argmin for an argmax,
a wrong "toward" sign or a wrong distance weight all lose far more than 1e-6 on a large fraction of
these inputs.

Lattice: Conway & Sloane, "Sphere Packings, Lattices and Groups", ch. 4 (E8 = D8 u (D8 + 1/2),
D4, A2); the pages name E8, D4, A2 and Z as the quantizer's lattices (gist.science, Technical
Summary, Methodology: Lattice Quantization).
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from lattice_inputs import facet_ties, random_inputs, small_error_blocks

HERE = os.path.dirname(os.path.abspath(__file__))
SQ3_2 = np.sqrt(3.0) / 2.0
COUNT = 1_000_000


@pytest.fixture(scope="module")
def search():
    out = os.path.join(tempfile.mkdtemp(prefix="lattice_search_"), "liblattice_search.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", out, os.path.join(HERE, "lattice_search.c"),
                    "-lm"], check=True)
    L = ctypes.CDLL(out)
    L.ls_nearest.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p,
                             ctypes.c_void_p, ctypes.c_void_p]
    L.ls_nearest.restype = ctypes.c_int

    def run(lattice, u, tol=1e-9):
        d = oracle.LATTICE_DIM[lattice]
        u = np.ascontiguousarray(u, dtype=np.float32).reshape(-1, d)
        m = u.shape[0]
        bd = np.zeros(m, np.float64)
        bp = np.zeros((m, d), np.int32)
        cnt = np.zeros(m, np.int32)
        assert L.ls_nearest(lattice, u.ctypes.data, m, tol, bd.ctypes.data, bp.ctypes.data, cnt.ctypes.data) == 0
        return bd, bp, cnt
    return run


def to_points(lattice, v):
    v = np.asarray(v, dtype=np.float64)
    if lattice == oracle.E8:
        return v / 2.0
    if lattice == oracle.A2:
        return np.stack([v[..., 0] * 0.5, v[..., 1] * SQ3_2], axis=-1)
    return v


def in_lattice(lattice, v):
    v = np.asarray(v, dtype=np.int64)
    if lattice == oracle.D4:
        return np.sum(v, axis=1) % 2 == 0
    if lattice == oracle.A2:
        return (v[:, 0] - v[:, 1]) % 2 == 0
    same = np.all((v % 2) == (v[:, :1] % 2), axis=1)
    return same & (np.sum(v, axis=1) % 4 == 0)


def check(lattice, u, search, allow_report):
    v = oracle.quantize_blocks(lattice, u)
    assert np.all(in_lattice(lattice, v)), "oracle returned a non-lattice point"
    bd, bp, cnt = search(lattice, u)
    po = to_points(lattice, v)
    pb = to_points(lattice, bp)
    u64 = u.astype(np.float64)
    do = np.sum((po - u64) ** 2, axis=1)
    assert np.all(do >= bd - 1e-12), "the exhaustive search missed a nearer point"
    differ = np.any(v != bp, axis=1)
    sep = np.linalg.norm(po - pb, axis=1)
    margin = np.where(differ, (do - bd) / (2.0 * np.maximum(sep, 1e-30)), 0.0)
    allowed = 1e-6 * np.maximum(1.0, np.abs(u64).max(axis=1))
    bad = differ & (margin > allowed)
    assert not bad.any(), f"{bad.sum()} oracle points lose by more than the rounding margin, worst {margin.max():.3g}"
    ties = cnt > 1
    n_dis = int(np.count_nonzero(differ & ~ties))
    allow_report(lattice, n_dis, u.shape[0])
    return n_dis


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.D4, oracle.A2])
def test_random_inputs_against_exhaustive_search(search, lattice, record_property):
    d = oracle.LATTICE_DIM[lattice]
    u = random_inputs(d, COUNT, 1000 + lattice)
    report = {}
    n_dis = check(lattice, u, search, lambda lat, n, m: report.update(n=n, m=m))
    record_property("disagreements", n_dis)
    # random inputs are rarely within rounding of a boundary: a handful in 10^6 at most
    assert n_dis <= 10, n_dis


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.D4, oracle.A2])
def test_constructed_near_ties_against_exhaustive_search(search, lattice):
    u = facet_ties(lattice, 200_000, 2000 + lattice)
    check(lattice, u, search, lambda *a: None)


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.D4])
def test_fix_ups_among_tiny_rounding_errors(search, lattice):
    """Here the candidate distances differ by 2^-45 or more, which binary64 resolves: the nearest
    point is unique (apart from exact ties) and the oracle must return exactly that point."""
    u = small_error_blocks(lattice, 100_000, 3000 + lattice)
    v = oracle.quantize_blocks(lattice, u)
    bd, bp, cnt = search(lattice, u, tol=1e-15)
    unique = cnt == 1
    assert unique.mean() > 0.25
    wrong = unique & np.any(v != bp, axis=1)
    assert not wrong.any(), f"{wrong.sum()} blocks differ from the unique nearest point, e.g. u={u[wrong][0]}"
