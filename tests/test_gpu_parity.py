"""GPU parity: the CUDA codec (through the C ABI) against the CPU oracle on the same seeded inputs.

Bar (from the codec's specification):
  * lattice codes, meta, chunk offsets and the bitstream are bit-exact when both sides quantize the
    same binary32 coefficients (hq_quantize_coeffs), and for whole encodes, whose binary32 chain
    (RMS tree, descending butterflies, normalisation) is defined op for op;
  * reconstructions match the oracle's float64 decode within 1e-5 relative per element, relative
    to max(|x_hat|, s_hat) of the tile (binary32 output), or one bf16 ulp (bf16 output);
  * MSE within 0.1%.
"""
import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W

pytestmark = pytest.mark.gpu

LATS = [oracle.E8, oracle.D4, oracle.A2, oracle.Z]


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


def t_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def assert_same_code(code, ref, what=""):
    """Device code against the oracle's: bit-exact, except that an index may differ for an input
    within 1e-6 of a Voronoi boundary (counted; the fraction of blocks must stay <= 1e-6, and every
    chunk without such a block must be word-identical) -- see oracle/parity.py."""
    from oracle import parity
    words = int(u32(code.chunk_word)[-1])
    scale = u16(code.scale) if (ref.scale is not None and code.scale is not None) else None
    rep = parity.compare(scale, u16(code.meta), u32(code.chunk_word), u32(code.bits)[:max(words, 1)], ref)
    assert not rep.failures, f"{what}: {rep.failures[:3]}"
    assert rep.fraction <= 1e-6, f"{what}: {rep.disagreements} boundary disagreements in {rep.blocks} blocks"
    return rep


def _coeffs(n, tiles, seed, lattice):
    rng = np.random.default_rng(seed)
    d = oracle.LATTICE_DIM[lattice]
    parts = [rng.standard_normal((tiles, n)) * s for s in (0.3, 3.0, 40.0)]
    u = np.concatenate(parts)[: tiles].astype(np.float32)
    # some rows on / near lattice points and exact ties
    pts = oracle.quantize_blocks(lattice, rng.uniform(-9, 9, size=(n // d * 8, d)).astype(np.float32))
    if lattice == oracle.E8:
        p = pts / 2.0
    elif lattice == oracle.A2:
        p = pts * np.array([0.5, np.sqrt(3.0) / 2.0])
    else:
        p = pts.astype(np.float64)
    u[:8] = p.reshape(8, n).astype(np.float32)
    u[8:12] = np.round(rng.uniform(-6, 6, size=(4, n)) * 2) / 2          # half-integers
    return u


@pytest.mark.parametrize("lattice", LATS)
@pytest.mark.parametrize("n", [64, 128, 256])
def test_quantize_coeffs_bit_exact(hq, lattice, n):
    u = _coeffs(n, 77, 100 + n + lattice, lattice)             # 77 tiles: 3 chunks, ragged
    v, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, lattice)
    st, _ = hq.status(code.ws)
    assert st == 0
    rv, rmeta, rcw, rbits, rst = oracle.quantize_coeffs(u, n, lattice)
    np.testing.assert_array_equal(v.cpu().numpy(), rv)
    np.testing.assert_array_equal(u16(code.meta), rmeta)
    np.testing.assert_array_equal(u32(code.chunk_word), rcw)
    np.testing.assert_array_equal(u32(code.bits)[: int(rcw[-1])], rbits)


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.D4, oracle.A2])
@pytest.mark.parametrize("n", [64, 128, 256])
def test_quantize_coeffs_near_ties_bit_exact(hq, lattice, n):
    """Coefficients on and within a few 1e-6 of Voronoi facets (coset ties of E8 and A2,
    neighbour ties of D4), and blocks whose fix-up chooses among rounding errors below 2^-31:
    the device's shortcut decisions hand these to the plain rule, so codes stay bit-exact."""
    from lattice_inputs import facet_ties, small_error_blocks
    d = oracle.LATTICE_DIM[lattice]
    parts = [facet_ties(lattice, 40 * n // d, 70 + n + lattice)]
    if lattice != oracle.A2:
        parts.append(small_error_blocks(lattice, 16 * n // d, 90 + n + lattice))
    u = np.ascontiguousarray(np.concatenate(parts).reshape(-1, n))
    v, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, lattice)
    assert hq.status(code.ws)[0] == 0
    rv, rmeta, rcw, rbits, rst = oracle.quantize_coeffs(u, n, lattice)
    assert rst == 0
    np.testing.assert_array_equal(v.cpu().numpy(), rv)
    np.testing.assert_array_equal(u16(code.meta), rmeta)
    np.testing.assert_array_equal(u32(code.chunk_word), rcw)
    np.testing.assert_array_equal(u32(code.bits)[: int(rcw[-1])], rbits)


@pytest.mark.parametrize("n", [64, 128, 256])
def test_quantize_coeffs_kv_dither_bit_exact(hq, n):
    u = _coeffs(n, 150, 7 + n, oracle.D4)
    v, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, oracle.D4, seed=99, kv=True, kv_S=50)
    rv, rmeta, rcw, rbits, _ = oracle.quantize_coeffs(u, n, oracle.D4, seed=99, kv=True, kv_S=50)
    np.testing.assert_array_equal(v.cpu().numpy(), rv)
    np.testing.assert_array_equal(u32(code.bits)[: int(rcw[-1])], rbits)


def _decode_check(y: torch.Tensor, ref_code, xo: np.ndarray):
    n = ref_code.n
    sh = W.bf16_bits_to_f32(ref_code.scale).astype(np.float64)
    rows, cols = xo.shape
    scale_map = np.repeat(sh.reshape(cols // n, rows).T, n, axis=1)
    if y.dtype == torch.float32:
        yh = y.cpu().numpy().astype(np.float64)
        tol = 1e-5 * np.maximum(np.abs(xo), scale_map)
        bad = np.abs(yh - xo) > tol
        assert not bad.any(), f"{bad.sum()} elements outside tolerance, max |d| {np.abs(yh - xo).max()}"
    else:
        # bf16 output: the binary32 value rounded to nearest even, so within half a bf16 ulp
        # (2^-9 relative) of a binary32 result that itself meets the tolerance above
        yb = y.float().cpu().numpy().astype(np.float64)
        tol = 2.0 ** -8 * np.abs(xo) + 1e-5 * np.maximum(np.abs(xo), scale_map)
        bad = np.abs(yb - xo) > tol
        assert not bad.any(), f"{bad.sum()} bf16 elements outside tolerance, max |d| {np.abs(yb - xo).max()}"


CASES = [
    # name, builder(rows, cols), rows, cols, n, beta
    ("tiny_fp32", lambda r, c: W.tiny_weight(0)[:r, :c], 256, 256, 64, 0.27),
    ("llama_bf16_n128", lambda r, c: W.llama_weight(4096, 4096, 1)[:r, :c], 160, 512, 128, 0.3),
    ("llama_bf16_ragged", lambda r, c: W.llama_weight(4096, 4096, 1)[:r, :c], 70, 384, 128, 0.25),
    ("llama70b_n256", lambda r, c: W.llama_70b_weight(8192, 28672, 4)[:r, :c], 100, 1024, 256, 0.3),
    ("dit_n64_bf16", lambda r, c: W.dit_linear(512, 512, 5)[:r, :c], 129, 256, 64, 0.4),
]


@pytest.mark.parametrize("lattice", LATS)
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_encode_decode_match_oracle(hq, case, lattice):
    name, build, rows, cols, n, beta = case
    x = build(rows, cols)
    seed = 1234 + lattice
    xt = torch.from_numpy(x).cuda() if x.dtype == np.float32 else t_bf16(x)
    code = hq.encode(xt, tile=n, lattice=lattice, step=beta, seed=seed)
    st, _ = hq.status(code.ws)
    assert st == 0, st
    ref = oracle.encode(x, n, lattice, beta, seed, want_codes=True)
    assert_same_code(code, ref, name)
    xo, rst = oracle.decode(ref)
    assert rst == 0
    y32 = hq.decode(code, dtype=torch.float32)
    assert hq.status(code.ws)[0] == 0
    _decode_check(y32, ref, xo)
    yb = hq.decode(code, dtype=torch.bfloat16)
    _decode_check(yb, ref, xo)
    xf = x if x.dtype == np.float32 else W.bf16_bits_to_f32(x)
    mse_gpu = np.mean((y32.cpu().numpy().astype(np.float64) - xf) ** 2)
    mse_ref = np.mean((xo - xf) ** 2)
    assert abs(mse_gpu / mse_ref - 1) < 1e-3


def test_gpu_decodes_oracle_stream(hq):
    # the decoder alone, fed with the oracle's bitstream
    x = W.llama_weight(4096, 4096, 1)[:96, :256]
    ref = oracle.encode(x, 128, oracle.E8, 0.3, seed=5)
    p = hq.params(128, hq.E8, 0.3, seed=5)
    code = hq.alloc_code(96, 256, p)
    code.scale.copy_(torch.from_numpy(ref.scale.view(np.int16)))
    code.meta.copy_(torch.from_numpy(ref.meta.view(np.int16)))
    code.chunk_word.copy_(torch.from_numpy(ref.chunk_word.view(np.int32)))
    code.bits[: ref.total_words].copy_(torch.from_numpy(ref.bits.view(np.int32)))
    y = hq.decode(code, dtype=torch.float32)
    assert hq.status(code.ws)[0] == 0
    xo, _ = oracle.decode(ref)
    _decode_check(y, ref, xo)


@pytest.mark.parametrize("bps_beta", [1.6, 0.9, 0.6])
def test_kv_encode_decode_match_oracle(hq, bps_beta):
    B, H, S, D = 2, 3, 40, 128
    kb = W.kv_keys(B, H, S, D, seed=2)
    code = hq.kv_encode(t_bf16(kb), step=bps_beta, seed=31)
    assert hq.status(code.ws)[0] == 0
    ref = oracle.encode(kb.reshape(-1, D), D, oracle.D4, bps_beta, 31, kv=True, kv_S=S, want_codes=True)
    assert_same_code(code, ref, "kv")
    y = hq.kv_decode(code, (B, H, S, D), dtype=torch.float32)
    xo, _ = oracle.decode(ref)
    _decode_check(y.reshape(-1, D), ref, xo)


def test_capacity_error_reports_needed_words(hq):
    x = t_bf16(W.llama_weight(4096, 4096, 1)[:128, :256])
    p = hq.params(128, hq.E8, 0.3)
    small = hq.alloc_code(128, 256, p, cap_words=64)
    code = hq.encode(x, 128, hq.E8, 0.3, out=small)
    st, detail = hq.status(code.ws)
    assert st == 3
    full = hq.encode(x, 128, hq.E8, 0.3)
    assert hq.status(full.ws)[0] == 0
    assert detail == full.total_words()


def test_nonfinite_tiles_flagged_and_zeroed(hq):
    x = W.llama_weight(4096, 4096, 1)[:64, :256].copy()
    x[3, 5] = 0x7FC0      # NaN
    x[40, 200] = 0x7F80   # +inf
    code = hq.encode(t_bf16(x), 128, hq.E8, 0.3, seed=3)
    st, detail = hq.status(code.ws)
    assert st == 4 and detail == 2
    ref = oracle.encode(x, 128, oracle.E8, 0.3, 3)
    assert ref.status & oracle.ST_NONFINITE
    assert_same_code(code, ref, "nonfinite")


def test_corrupt_chunk_offsets_detected(hq):
    x = t_bf16(W.llama_weight(4096, 4096, 1)[:96, :256])
    code = hq.encode(x, 128, hq.E8, 0.3, seed=3)
    assert hq.status(code.ws)[0] == 0
    code.chunk_word[1] = code.chunk_word[-1] + 100000     # offsets beyond the stream
    y = hq.decode(code, dtype=torch.float32)
    st, _ = hq.status(code.ws)
    assert st == 5
    assert torch.isfinite(y).all()


@pytest.mark.parametrize("lattice,target", [(oracle.E8, 4.0), (oracle.D4, 2.0)])
def test_rate_search_hits_target(hq, lattice, target):
    x = W.llama_weight(4096, 4096, 1)[:512, :1024]
    xt = t_bf16(x)
    beta = hq.calibrate_step(xt, 128, lattice, target, seed=2)
    code = hq.encode(xt, 128, lattice, beta, seed=2)
    assert abs(code.payload_bps() - target) <= 0.01
    ref = oracle.encode(x, 128, lattice, beta, 2)
    assert abs(oracle.payload_bps(ref) - code.payload_bps()) == 0.0
