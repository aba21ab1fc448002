"""Pins for the oracle's primitives: Philox, bf16 rounding, RMS, FWHT.

Each check compares the oracle with something other than itself: a library run (curand's host
Philox generator, torch's bf16 conversion, scipy's Sylvester Hadamard matrix), a closed form
(orthogonality, exact inverse) or a float64 reference.
"""
import ctypes
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle

CURAND = "/usr/local/cuda/lib64/libcurand.so"


def _curand_host(seed: int, count: int, offset: int = 0) -> np.ndarray:
    lib = ctypes.CDLL(CURAND)
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0  # PHILOX4_32_10
    assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
    if offset:
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
    buf = (ctypes.c_uint32 * count)()
    assert lib.curandGenerate(gen, buf, ctypes.c_size_t(count)) == 0
    lib.curandDestroyGenerator(gen)
    return np.array(buf[:], dtype=np.uint32)


@pytest.mark.skipif(not os.path.exists(CURAND), reason="curand not installed")
@pytest.mark.parametrize("seed", [0, 7, 0x0123456789ABCDEF, 0xFFFFFFFFFFFFFFFF])
def test_philox_matches_curand_host_generator(seed):
    # curand's host Philox4x32-10 generator emits block i (four words) from counter
    # (i // 65536 + offset_blocks, high word, i % 65536, 0) under key (seed_lo, seed_hi).
    k0, k1 = seed & 0xFFFFFFFF, seed >> 32
    out = _curand_host(seed, 4 * 8).reshape(-1, 4)
    for i in range(8):
        np.testing.assert_array_equal(out[i], oracle.philox([0, 0, i, 0], k0, k1))
    for x, y, c in [(5, 0, 3), (0xFFFFFFFE, 0, 9), (7, 3, 11), (123456, 77, 65535)]:
        blk = ((y << 32) | x) * 65536 + c
        got = _curand_host(seed, 4, offset=4 * blk)
        np.testing.assert_array_equal(got, oracle.philox([x, y, c, 0], k0, k1))


def test_sign_diagonal_balanced_and_seeded():
    d0 = oracle.signs(11, 4096)
    d1 = oracle.signs(12, 4096)
    assert set(np.unique(d0)) == {-1, 1}
    assert abs(int(np.sum(d0))) < 4 * np.sqrt(4096)          # ~ +-1 balanced
    assert np.mean(d0 != d1) > 0.4                              # another seed, another diagonal
    np.testing.assert_array_equal(d0[:300], oracle.signs(11, 300))  # depends on (seed, J) only


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e-38).astype(np.float32),       # subnormal range
        (rng.standard_normal(5000) * 1e30).astype(np.float32),
        # exact ties: 16 low bits = 0x8000, both parities of the kept LSB
        (np.arange(4000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38], dtype=np.float32),
    ])
    x = x[np.isfinite(x) | np.isinf(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f32_to_bf16_bits(x)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("n", [64, 128, 256])
def test_rms_matches_float64(n):
    rng = np.random.default_rng(n)
    for scale in [1e-3, 1.0, 1e3]:
        x = (rng.standard_normal(n) * scale).astype(np.float32)
        ref = np.sqrt(np.mean(x.astype(np.float64) ** 2))
        assert abs(oracle.rms(x) - ref) <= 2e-6 * ref


def _rn32_sqrt(r):
    """binary32 nearest (ties to even) to sqrt(r) for a positive Fraction r, decided exactly:
    f is the answer when the squares of the midpoints to its neighbours bracket r."""
    from fractions import Fraction
    f = np.float32(np.sqrt(float(r)))
    for _ in range(4):
        lo = np.nextafter(f, np.float32(0)); hi = np.nextafter(f, np.float32(np.inf))
        mlo = (Fraction(float(lo)) + Fraction(float(f))) / 2
        mhi = (Fraction(float(f)) + Fraction(float(hi))) / 2
        if r < mlo * mlo:
            f = lo
        elif r > mhi * mhi:
            f = hi
        else:
            assert r != mlo * mlo and r != mhi * mhi   # no tie for these inputs
            return f
    raise AssertionError("no convergence")


# One large square in the first half of the tile and n/2 equal small squares in the second half:
# the ascending pairwise tree adds the small squares among themselves first, so every partial sum
# and the total are exact, while a running (sequential) sum rounds at every step.  Found by a
# search over bf16 values for which the two sums give different bf16 scales.
RMS_ORDER_CASES = [(64, 5.15625, 0.2373046875), (64, 6.15625, 0.2060546875), (128, 5.5625, 0.1904296875),
                   (128, 5.625, 0.1591796875), (256, 7.90625, 0.2177734375), (256, 10.3125, 0.2373046875)]


@pytest.mark.parametrize("n,big,small", RMS_ORDER_CASES)
def test_rms_sums_the_squares_in_the_ascending_tree(n, big, small):
    """The scale is sqrt(mean of squares) with the squares summed by the ascending pairwise tree
    (the per-tile scaling of Methodology step 2 with the RMS statistic; the summation order is the
    reading that fixes the binary32 result).  On these inputs the tree is exact, so its result is
    the correctly rounded square root of the exact mean square, and a sequential sum is not."""
    from fractions import Fraction
    x = np.zeros(n, dtype=np.float32)
    x[0] = big
    x[n // 2:] = small
    exact = sum(Fraction(float(v)) ** 2 for v in x) / n
    want = _rn32_sqrt(exact)
    got = np.float32(oracle.rms(x))
    assert got == want, (got, want)
    # the sequential order rounds differently, down to the stored bf16 scale
    seq = np.float32(0.0)
    for v in x:
        seq = np.float32(seq + np.float32(v) * np.float32(v))
    seq_s = np.float32(np.sqrt(np.float32(seq * np.float32(1.0 / n))))
    assert oracle.f32_to_bf16_bits(np.array([seq_s]))[0] != oracle.f32_to_bf16_bits(np.array([got]))[0]


@pytest.mark.parametrize("n", [64, 128, 256])
def test_fwht_is_the_sylvester_hadamard_product(n):
    H = scipy.linalg.hadamard(n).astype(np.float64)   # natural (Sylvester) order
    rng = np.random.default_rng(100 + n)
    for _ in range(20):
        x = rng.standard_normal(n).astype(np.float32)
        ref = H @ x.astype(np.float64)
        got = oracle.fwht_f32(x).astype(np.float64)
        # binary32 butterflies: log2(n) roundings of partial sums bounded by sum |x|
        assert np.max(np.abs(got - ref)) <= np.log2(n) * 2.0 ** -23 * np.sum(np.abs(x))
        # orthogonality: |H x| = sqrt(n) |x|
        assert abs(np.linalg.norm(got) - np.sqrt(n) * np.linalg.norm(x.astype(np.float64))) <= 1e-5 * np.linalg.norm(got)
    # integer inputs: the float64 transform is exact, and H H = n I
    xi = rng.integers(-1000, 1000, size=n).astype(np.float64)
    y = oracle.fwht_f64(xi)
    np.testing.assert_array_equal(y, H @ xi)
    np.testing.assert_array_equal(oracle.fwht_f64(y), n * xi)
    # a single impulse returns the matching Hadamard column (catches index/sign slips)
    for j in [0, 1, n // 2 + 3, n - 1]:
        e = np.zeros(n, dtype=np.float32)
        e[j] = 1.0
        np.testing.assert_array_equal(oracle.fwht_f32(e), H[:, j].astype(np.float32))
