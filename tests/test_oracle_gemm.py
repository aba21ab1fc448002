"""The oracle's decode-to-int8 and grouped int8 GEMM (the method's tensor-core integration: int8
MMA on the post-RHT lattice codes).  Pins that do not reuse the oracle's arithmetic:

* the integer part is numpy's exact int64 matrix product (unit scales);
* with power-of-two scales every fma is exact, so Y is the float64 sum of scaled group sums;
* with general scales Y stays within the binary32 error bound of the exact sum;
* end to end, for activations x whose RHT is an int8 vector a (x = D H a / n per tile), the GEMM
  equals the oracle's binary64 reconstruction W_hat times x: the RHT-domain identity
  (D H p) . (D H a) / n = p . a pins signs, tile order and every scale;
* decode_int8 returns the parsed codes, the group scales, and zeros plus a range flag for
  tiles with a code outside int8.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from post_quantization_tile_b200 import workloads as W


def _int8(rng, shape, scale=40.0):
    return np.clip(np.round(rng.standard_normal(shape) * scale), -127, 127).astype(np.int8)


def test_unit_scales_give_the_exact_integer_product():
    rng = np.random.default_rng(1)
    M, N, K, n = 24, 40, 512, 128
    A, V = _int8(rng, (M, K), 20.0), _int8(rng, (N, K), 20.0)
    Y = oracle.gemm_grouped(A, np.ones(M, np.float32), V, np.ones((K // n, N), np.float32), n)
    exact = A.astype(np.int64) @ V.astype(np.int64).T
    assert np.all(np.abs(exact) < 2 ** 24)
    np.testing.assert_array_equal(Y.astype(np.int64), exact)


def test_power_of_two_scales_are_exact():
    rng = np.random.default_rng(2)
    M, N, K, n = 16, 16, 384, 128
    A, V = _int8(rng, (M, K), 10.0), _int8(rng, (N, K), 10.0)
    g = (2.0 ** rng.integers(-6, 3, size=(K // n, N))).astype(np.float32)
    sa = (2.0 ** rng.integers(-3, 3, size=M)).astype(np.float32)
    Y = oracle.gemm_grouped(A, sa, V, g, n)
    S = np.stack([A[:, t * n:(t + 1) * n].astype(np.int64) @ V[:, t * n:(t + 1) * n].astype(np.int64).T
                  for t in range(K // n)])                                  # [T, M, N]
    ref = (S * g[:, None, :].astype(np.float64)).sum(0) * sa[:, None]
    np.testing.assert_array_equal(Y.astype(np.float64), ref)


def test_general_scales_within_the_binary32_bound():
    rng = np.random.default_rng(3)
    M, N, K, n = 8, 24, 1024, 128
    A, V = _int8(rng, (M, K)), _int8(rng, (N, K))
    g = rng.uniform(1e-4, 1e-2, size=(K // n, N)).astype(np.float32)
    sa = rng.uniform(0.5, 2.0, size=M).astype(np.float32)
    Y = oracle.gemm_grouped(A, sa, V, g, n).astype(np.float64)
    S = np.stack([A[:, t * n:(t + 1) * n].astype(np.int64) @ V[:, t * n:(t + 1) * n].astype(np.int64).T
                  for t in range(K // n)])
    terms = S * g[:, None, :].astype(np.float64)
    ref = terms.sum(0) * sa[:, None]
    bound = (K // n + 1) * 2.0 ** -24 * (np.abs(terms).sum(0) * sa[:, None] + np.abs(ref))
    assert np.all(np.abs(Y - ref) <= bound)
    sample = oracle.gemm_grouped_sample(A, sa, V, g, n, [0, 7, 3], [0, 23, 11])
    np.testing.assert_array_equal(sample, Y[[0, 7, 3], [0, 23, 11]].astype(np.float32))


@pytest.mark.parametrize("lattice,beta", [(oracle.E8, 0.3), (oracle.D4, 0.45), (oracle.Z, 0.35)])
def test_gemm_equals_reconstruction_times_activations(lattice, beta):
    rng = np.random.default_rng(4)
    n, N, K, M, seed = 128, 48, 512, 6, 21
    w = W.llama_weight(N, K, seed=5)
    code = oracle.encode(w, n, lattice, beta, seed)
    v8, g, st = oracle.decode_int8(code)
    assert st == 0
    what, _ = oracle.decode(code)                       # binary64 reconstruction [N, K]
    a = _int8(rng, (M, K), 32.0)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    d = np.where(oracle.signs(seed, K) < 0, -1.0, 1.0)
    x = np.concatenate([(a[:, t * n:(t + 1) * n].astype(np.float64) @ H) / n for t in range(K // n)], axis=1) * d
    Y = oracle.gemm_grouped(a, np.ones(M, np.float32), v8, g, n).astype(np.float64)
    ref = x @ what.T
    np.testing.assert_allclose(Y, ref, rtol=2e-6, atol=2e-6 * np.abs(ref).max())


def test_decode_int8_codes_scales_and_range():
    n = 128
    u = np.random.default_rng(6).standard_normal((64, n)).astype(np.float32) * 3.0
    u[5, 7] = 80.0                                      # E8 doubled code 160: out of int8
    v, meta, cw, bits, _ = oracle.quantize_coeffs(u, n, oracle.E8)
    code = oracle.Code(64, n, n, oracle.E8, 1.0, 0, 0, 0, np.full(64, 0x3F80, np.uint16), meta, cw, bits, 0,
                       None, None)
    v8, g, st = oracle.decode_int8(code)
    assert st & oracle.ST_RANGE
    keep = np.ones(64, bool)
    keep[5] = False
    np.testing.assert_array_equal(v8[keep].astype(np.int32), v[keep])
    assert np.all(v8[5] == 0)
    assert np.all(g == np.float32(np.float32(1.0 * 0.0883883461356163) * 0.5))
