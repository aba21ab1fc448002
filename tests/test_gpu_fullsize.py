"""GPU parity at the workloads' full sizes, in the benchmark's launch configuration.

The oracle cannot encode a 235 M-scalar matrix in test time, but tiles and chunks are
independent: the oracle encodes whole 32-row chunks taken out of the full tensor (first, a
random and the last chunk of every tile column), and the GPU's words for those chunks, their
meta and scales must be bit-identical (an index may differ only within 1e-6 of a Voronoi
boundary, counted, at most a 1e-6 fraction of the blocks); the GPU reconstruction of those rows,
decoded both to binary32 and to bf16, must match the oracle's within the tolerance, with the
same MSE.  The rate search hits the
target within 0.01 bps (Methodology step 3) on the full tensor.

Workloads: LLaMA-7B-shaped 4096x4096 and 11008x4096 (E8, 3/4/5 bps), 70B-shaped 8192x28672 with
A2/D4/E8/Z and 28672x8192 (E8), the KV keys [8, 32, 8192, 128] with the dithered D4 at 1.7/2/4 bps
and the KV values at 2 bps, and two DiT blocks (E8, 4 bps).
"""
import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


def _t(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _sample_chunks(rows, rng):
    RB = (rows + 31) // 32
    picks = sorted({0, int(rng.integers(1, max(2, RB - 1))), RB - 1})
    return picks


def _chunk_subcode(scale, meta, cw, bits, rows, n, NT, rb):
    """The device code of rows [32 rb, 32 rb + 32) as a code of its own (one chunk per tile column)."""
    RB = (rows + 31) // 32
    r0, r1 = 32 * rb, min(32 * rb + 32, rows)
    h = r1 - r0
    sub_scale = np.concatenate([scale[jt * rows + r0: jt * rows + r1] for jt in range(NT)])
    sub_meta = np.concatenate([meta[jt * rows + r0: jt * rows + r1] for jt in range(NT)])
    pieces = [bits[cw[jt * RB + rb]: cw[jt * RB + rb + 1]] for jt in range(NT)]
    sub_cw = np.zeros(NT + 1, dtype=np.uint32)
    sub_cw[1:] = np.cumsum([p.size for p in pieces])
    sub_bits = np.concatenate(pieces + [np.zeros(1, np.uint32)])
    assert sub_meta.size == NT * h
    return sub_scale, sub_meta, sub_cw, sub_bits


def _check(hq, x_host, xt, n, lattice, target, seed, kv=False, kv_S=0, rng_seed=0):
    """Sampled chunks of the full-size code against the oracle's code of the same rows: boundary-aware
    comparison (oracle/parity.py: bit-exact except counted near-boundary disagreements, fraction of
    blocks <= 1e-6), reconstructions within 1e-5 max(|x_hat|, s_hat) in binary32 and within half a
    bf16 ulp more in bf16, MSE within 0.1%."""
    from oracle import parity
    rows, cols = x_host.shape
    beta = hq.calibrate_step(xt, n, lattice, target, seed=seed, kv=kv, kv_S=kv_S)
    if kv:
        B_H = rows // kv_S
        code = hq.kv_encode(xt.view(1, B_H, kv_S, cols), step=beta, seed=seed)
    else:
        code = hq.encode(xt, n, lattice, beta, seed=seed)
    st, _ = hq.status(code.ws)
    assert st == 0
    assert abs(code.payload_bps() - target) <= 0.01
    y = hq.decode(code, dtype=torch.bfloat16)
    y32 = hq.decode(code, dtype=torch.float32)
    assert hq.status(code.ws)[0] == 0
    cw = code.chunk_word.cpu().numpy().view(np.uint32).astype(np.int64)
    bits = code.bits.cpu().numpy().view(np.uint32)
    meta = code.meta.cpu().numpy().view(np.uint16)
    scale = code.scale.cpu().numpy().view(np.uint16)
    NT = cols // n
    rng = np.random.default_rng(rng_seed)
    err_gpu = err_ref = 0.0
    blocks = disagreements = 0
    for rb in _sample_chunks(rows, rng):
        r0, r1 = 32 * rb, min(32 * rb + 32, rows)
        xs = np.ascontiguousarray(x_host[r0:r1])
        ref = oracle.encode(xs, n, lattice, beta, seed, kv, kv_S, row0=r0, want_codes=True)
        rep = parity.compare(*_chunk_subcode(scale, meta, cw, bits, rows, n, NT, rb), ref)
        assert not rep.failures, f"rows {r0}..{r1}: {rep.failures[:3]}"
        blocks += rep.blocks
        disagreements += rep.disagreements
        xo, rst = oracle.decode(ref)
        assert rst == 0
        sh = W.bf16_bits_to_f32(ref.scale).astype(np.float64)
        scale_map = np.repeat(sh.reshape(NT, r1 - r0).T, n, axis=1)
        y32s = y32[r0:r1].cpu().numpy().astype(np.float64)
        assert np.all(np.abs(y32s - xo) <= 1e-5 * np.maximum(np.abs(xo), scale_map)), "binary32 reconstruction"
        yb = y[r0:r1].float().cpu().numpy().astype(np.float64)
        tol = 2.0 ** -8 * np.abs(xo) + 1e-5 * np.maximum(np.abs(xo), scale_map)
        assert np.all(np.abs(yb - xo) <= tol)
        xf = W.bf16_bits_to_f32(xs).astype(np.float64)
        err_gpu += np.sum((yb - xf) ** 2)
        err_ref += np.sum((W.bf16_bits_to_f32(W.to_bf16_bits(xo.astype(np.float32))).astype(np.float64) - xf) ** 2)
    assert disagreements <= 1e-6 * blocks, f"{disagreements} boundary disagreements in {blocks} blocks"
    assert abs(err_gpu / err_ref - 1.0) < 1e-3
    return code


@pytest.mark.parametrize("shape,seed", [((4096, 4096), 1), ((11008, 4096), 2)], ids=["4096x4096", "11008x4096"])
def test_llama7b_shapes_e8(hq, shape, seed):
    x = W.llama_weight(*shape, seed=seed)
    xt = _t(x)
    for target in (3.0, 4.0, 5.0):
        _check(hq, x, xt, 128, hq.E8, target, seed=seed, rng_seed=int(target))


def test_llama70b_lattice_sweep(hq):
    x = W.llama_70b_weight(8192, 28672, seed=4)
    xt = _t(x)
    for lattice in (hq.A2, hq.D4, hq.E8, hq.Z):
        for target in (3.0, 4.0, 5.0):
            _check(hq, x, xt, 256, lattice, target, seed=4, rng_seed=10 * lattice + int(target))


def test_llama70b_tall_e8(hq):
    x = W.llama_70b_weight(28672, 8192, seed=5)
    _check(hq, x, _t(x), 256, hq.E8, 4.0, seed=5)


def test_kv_cache_keys_dithered_d4(hq):
    B, H, S, D = 8, 32, 8192, 128
    k = W.kv_keys(B, H, S, D, seed=2).reshape(-1, D)
    kt = _t(k)
    for target in (1.7, 2.0, 4.0):
        _check(hq, k, kt, D, hq.D4, target, seed=2, kv=True, kv_S=S, rng_seed=int(10 * target))


def test_kv_cache_values_dithered_d4(hq):
    B, H, S, D = 8, 32, 8192, 128
    v = W.kv_values(B, H, S, D, seed=2).reshape(-1, D)
    _check(hq, v, _t(v), D, hq.D4, 2.0, seed=3, kv=True, kv_S=S, rng_seed=21)


def test_dit_two_blocks_e8(hq):
    for blk in range(2):
        for i, (r, c) in enumerate(W.DIT_BLOCK_SHAPES):
            x = W.dit_linear(r, c, seed=5 + blk * 100 + i)
            _check(hq, x, _t(x), 128, hq.E8, 4.0, seed=5 + blk, rng_seed=i)
