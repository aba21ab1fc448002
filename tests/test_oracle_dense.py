"""Pins of the dense-rotation KV variant of the oracle (Methodology step 4, "Bias Correction for KV
Cache": the per-layer rotation may be a dense Haar-random orthogonal matrix instead of the sign
diagonal).  None of these re-types the oracle's formulas:

* the seeded Haar matrix is orthogonal and its entries have variance 1/n;
* with Q = H_n D / sqrt(n) written out as a dense matrix, the forward rotation gives the codec's
  own RHT coefficients (pinned elsewhere) and the dense decode gives the codec's own KV decode, so
  a transposed Q, a dropped scale or a wrong dither sign fails;
* with a permutation matrix the forward chain is exact, so u equals x permuted times 1/(s beta)
  bit for bit;
* the reconstruction error of every tile is within the lattice's covering radius (dither makes
  Q(u + U) - (u + U) a point of the Voronoi cell) and the reconstruction is unbiased per vector;
* zero and non-finite head vectors, and token append, behave as in the RHT path.
"""
import numpy as np
import pytest

import oracle
from post_quantization_tile_b200 import workloads as W

N = 128
SQ3 = np.sqrt(3.0)
# covering radius of one lattice block in u coordinates (Z step 1; A2 minimum distance 1; D4 and
# E8 minimum distance sqrt 2)
COVER = {oracle.Z: 0.5, oracle.A2: 1.0 / SQ3, oracle.D4: 1.0, oracle.E8: 1.0}


def _sylvester(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def _rht_matrix(seed, n=N):
    """H_n D / sqrt(n) as a dense float32 matrix, D the codec's sign diagonal of tile column 0"""
    d = oracle.signs(seed, n).astype(np.float64)
    return (_sylvester(n) * d[None, :] / np.sqrt(n)).astype(np.float32)


def _kv_rows(B, H, S, seed=2):
    return W.kv_keys(B, H, S, N, seed=seed).reshape(B * H * S, N)


def test_haar_rotation_is_orthogonal_with_variance_one_over_n():
    for seed in (8, 9):
        Q = W.haar_rotation(N, seed=seed).astype(np.float64)
        assert np.abs(Q.T @ Q - np.eye(N)).max() < 2e-6
        assert np.abs(Q @ Q.T - np.eye(N)).max() < 2e-6
        assert abs(np.mean(Q * Q) * N - 1.0) < 1e-5   # rows of unit norm
        assert abs(np.mean(Q)) < 5.0 / N               # entries centred (sd of the mean ~ 1/n)
    assert not np.allclose(W.haar_rotation(N, seed=8), W.haar_rotation(N, seed=9))


def test_forward_rotation_with_the_rht_matrix_gives_the_codec_coefficients():
    seed, beta = 11, 0.7
    x = _kv_rows(1, 2, 40)
    ref = oracle.encode(x, N, oracle.D4, beta, seed, kv=True, kv_S=40, want_codes=True)
    Q = _rht_matrix(seed)
    u, scale, st = oracle.rotate_normalize(x, Q, beta)
    assert st == 0
    assert np.array_equal(scale, ref.scale)
    tol = 4e-6 * np.abs(ref.u).max()
    assert np.abs(u - ref.u).max() < tol
    # the transposed matrix (D H instead of H D) is a different rotation: the check above can tell
    u_t, _, _ = oracle.rotate_normalize(x, np.ascontiguousarray(Q.T), beta)
    assert np.abs(u_t - ref.u).max() > 100 * tol


def test_forward_rotation_with_a_permutation_is_exact():
    rng = np.random.default_rng(5)
    perm = rng.permutation(N)
    Q = np.zeros((N, N), dtype=np.float32)
    Q[np.arange(N), perm] = 1.0        # y_j = x_perm[j]
    x = W.gaussian_bf16(37, N, seed=4)
    beta = np.float32(1.3)
    u, scale, st = oracle.rotate_normalize(x, Q, float(beta))
    assert st == 0
    xf = W.bf16_bits_to_f32(x)
    sh = W.bf16_bits_to_f32(scale)
    g = (np.float32(1.0) / (sh * beta)).astype(np.float32)
    assert np.array_equal(u, (xf[:, perm] * g[:, None]).astype(np.float32))
    # the scale is the bf16 of the per-row RMS
    rms = np.sqrt(np.mean(xf.astype(np.float64) ** 2, axis=1))
    assert np.all(np.abs(sh - rms) <= rms * 2.0 ** -8)


@pytest.mark.parametrize("lattice", [oracle.Z, oracle.A2, oracle.D4, oracle.E8])
def test_dense_decode_with_the_rht_matrix_equals_the_codec_kv_decode(lattice):
    seed, beta, S = 21, 0.9, 50
    x = _kv_rows(1, 2, S, seed=3)
    code = oracle.encode(x, N, lattice, beta, seed, kv=True, kv_S=S)
    ref, st = oracle.decode(code)
    assert st == 0
    out, st2 = oracle.decode_dense(code, _rht_matrix(seed))
    assert st2 == 0
    # the dense matrix holds 1/sqrt(n) rounded to binary32 (relative error below 2^-24)
    assert np.abs(out - ref).max() <= 2e-7 * np.abs(ref).max()


@pytest.mark.parametrize("lattice", [oracle.Z, oracle.A2, oracle.D4, oracle.E8])
def test_dense_round_trip_error_within_the_covering_radius(lattice):
    B, H, S, beta, seed = 1, 3, 45, 0.8, 31
    x = _kv_rows(B, H, S, seed=6)
    Q = W.haar_rotation(N, seed=8)
    code = oracle.encode_dense(x, Q, lattice, beta, seed, kv_S=S)
    assert code.status == 0
    out, st = oracle.decode_dense(code, Q)
    assert st == 0
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    h = W.bf16_bits_to_f32(code.scale).astype(np.float64) * beta
    d = oracle.LATTICE_DIM[lattice]
    bound = np.sqrt(N / d) * COVER[lattice] * h * (1 + 1e-5) + 1e-5 * np.linalg.norm(xf, axis=1)
    err = np.linalg.norm(out - xf, axis=1)
    assert np.all(err <= bound)
    # and the error is not trivially small: the dither spreads it over the whole cell
    assert np.mean(err / (np.sqrt(N / d) * COVER[lattice] * h)) > 0.2


def test_dense_reconstruction_is_unbiased_per_vector():
    S, beta = 4, 1.5
    x = _kv_rows(1, 1, S, seed=7)
    Q = W.haar_rotation(N, seed=8)
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    K = 300
    acc = np.zeros_like(xf)
    for s in range(K):
        code = oracle.encode_dense(x, Q, oracle.D4, beta, 1000 + s, kv_S=S)
        acc += oracle.decode_dense(code, Q)[0]
    mean_err = acc / K - xf
    # per-coordinate error variance (s beta)^2 * 13/120 (D4 dither), so the mean over K draws has
    # standard deviation s beta sqrt(13/120 / K); 5 sigma
    h = W.bf16_bits_to_f32(oracle.encode_dense(x, Q, oracle.D4, beta, 0, kv_S=S).scale) * beta
    sd = h[:, None] * np.sqrt(13.0 / 120.0 / K)
    assert np.all(np.abs(mean_err) < 5.0 * sd)


def test_dense_zero_and_nonfinite_vectors():
    x = W.gaussian_bf16(6, N, seed=9).copy()
    x[1] = 0
    x[4, 17] = 0x7FC0   # NaN
    Q = W.haar_rotation(N, seed=8)
    code = oracle.encode_dense(x, Q, oracle.E8, 0.6, 3, kv_S=6, want_codes=True)
    assert code.status & oracle.ST_NONFINITE
    assert code.scale[1] == 0 and code.scale[4] == 0
    assert np.all(code.u[1] == 0) and np.all(code.u[4] == 0)
    out, st = oracle.decode_dense(code, Q)
    assert st == 0
    assert np.all(out[1] == 0) and np.all(out[4] == 0)
    assert np.all(np.isfinite(out))


def test_dense_token_append_matches_the_whole_sequence():
    B, H, S, s0 = 2, 2, 24, 15
    x = W.kv_keys(B, H, S, N, seed=12)
    Q = W.haar_rotation(N, seed=8)
    whole = oracle.encode_dense(x.reshape(-1, N), Q, oracle.D4, 1.1, 77, kv_S=S, want_codes=True)
    tail = np.ascontiguousarray(x[:, :, s0:, :]).reshape(-1, N)
    app = oracle.encode_dense(tail, Q, oracle.D4, 1.1, 77, kv_S=S - s0, kv_s0=s0, want_codes=True)
    v_whole = whole.v.reshape(B, H, S, N)[:, :, s0:, :].reshape(-1, N)
    assert np.array_equal(app.v, v_whole)
    assert np.array_equal(app.scale, whole.scale.reshape(B, H, S)[:, :, s0:].reshape(-1))
    # decoding the appended code gives the rows of the whole decode
    out_w = oracle.decode_dense(whole, Q)[0].reshape(B, H, S, N)[:, :, s0:, :].reshape(-1, N)
    out_a = oracle.decode_dense(app, Q)[0]
    assert np.abs(out_a - out_w).max() <= 1e-12 * np.abs(out_w).max()
