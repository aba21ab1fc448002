"""The int8 tensor-core GEMM with the weight's decode fused into its producer warps
(hq_gemm_code), on the GPU: bit-exact against the oracle's decode_int8 + grouped GEMM -- and so
against the two-call path -- with activation row counts that are not multiples of 128, with fewer
work units (one or two 128-row activation tiles x 32-row weight slab) than SMs and with more,
with an odd number of activation tiles, for the Z, D4 and E8 codes; tiles with codes outside int8 are zero as in hq_decode_int8; chunks too long for a
decoder warp's copy are read in place; and, sampled, the 4096 x 4096 weight at M = 16 and
M = 4096."""
import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W
from test_gpu_parity import t_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


def _acts(M, K, seed):
    rng = np.random.default_rng(seed)
    a = np.clip(np.round(rng.standard_normal((M, K)) * 32.0), -127, 127).astype(np.int8)
    sa = rng.uniform(0.01, 0.05, size=M).astype(np.float32)
    return a, sa


CASES = [
    # lattice, M, N, K, beta: few units, partial activation tiles, units > SMs
    (oracle.E8, 16, 512, 1024, 0.3),
    (oracle.E8, 128, 1024, 2048, 0.29),
    (oracle.D4, 200, 384, 512, 0.45),
    (oracle.Z, 256, 256, 256, 0.35),
    (oracle.E8, 300, 256, 512, 0.3),      # three activation tiles: the second pair's second tile lies past M
    (oracle.E8, 1, 128, 128, 0.3),        # the smallest product: one row, one slab, one group
    (oracle.Z, 129, 128, 640, 0.35),      # two tiles per slab, the second holding one row
    (oracle.D4, 257, 384, 256, 0.45),     # three tiles: a partial third, a fourth past M
    (oracle.E8, 1000, 640, 512, 0.3),
    (oracle.E8, 2048, 1280, 256, 0.3),
]


@pytest.mark.parametrize("lattice,M,N,K,beta", CASES)
def test_fused_gemm_bit_exact(hq, lattice, M, N, K, beta):
    w = W.llama_weight(N, K, seed=N + K)
    code = hq.encode(t_bf16(w), 128, lattice, beta, seed=5)
    assert hq.status(code.ws)[0] == 0
    a, sa = _acts(M, K, seed=M)
    Y = hq.gemm_code(torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda(), code)
    assert hq.status(code.ws)[0] == 0
    ref_code = oracle.encode(w, 128, lattice, beta, 5)
    rv, rg, st = oracle.decode_int8(ref_code)
    assert st == 0
    ref = oracle.gemm_grouped(a, sa, rv, rg, 128)
    np.testing.assert_array_equal(Y.cpu().numpy(), ref)


def test_fused_gemm_equals_two_call_path_and_zeroes_out_of_range_tiles(hq):
    n, N, K, M = 128, 256, 512, 128
    u = np.random.default_rng(6).standard_normal((N * K // n, n)).astype(np.float32) * 3.0
    u[5, 7] = 80.0                      # one tile with a code outside int8
    _, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, hq.E8)
    # re-shape the coefficient code as a [N, K] weight code: tile (r, jt) is row jt * N + r
    code.rows, code.cols = N, K
    code.scale.fill_(0x3F80)
    code.p.step = 1.0
    a, sa = _acts(M, K, seed=9)
    At, sat = torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda()
    Y = hq.gemm_code(At, sat, code)
    assert hq.status(code.ws)[0] == 7     # HQ_ERR_RANGE
    V, g = hq.decode_int8(code)
    assert hq.status(code.ws)[0] == 7
    Y2 = hq.gemm_int8(At, sat, V, g)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


def test_fused_gemm_reads_long_chunks_in_place(hq):
    """Chunks longer than a decoder warp's 1024-word copy (about 8.5 bits per weight here: Z codes
    spread over [-120, 120]) are read where they lie; the result is the two-call path's."""
    n, N, K, M = 128, 256, 512, 128
    u = np.random.default_rng(8).uniform(-120.0, 120.0, (N * K // n, n)).astype(np.float32)
    _, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, hq.Z)
    code.rows, code.cols = N, K
    code.scale.fill_(0x3F80)
    code.p.step = 1.0
    cw = code.chunk_word.cpu().numpy().astype(np.int64)
    assert (np.diff(cw) > 1024).any()   # some chunk takes the in-place path
    a, sa = _acts(M, K, seed=10)
    At, sat = torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda()
    Y = hq.gemm_code(At, sat, code)
    assert hq.status(code.ws)[0] == 0
    V, g = hq.decode_int8(code)
    assert hq.status(code.ws)[0] == 0
    Y2 = hq.gemm_int8(At, sat, V, g)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


@pytest.mark.parametrize("M", [16, 4096])
def test_fused_gemm_full_size_sampled(hq, M):
    N = K = 4096
    w = W.llama_weight(N, K, seed=1)
    code = hq.encode(t_bf16(w), 128, hq.E8, 0.29, seed=1)
    a, sa = _acts(M, K, seed=6)
    Y = hq.gemm_code(torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda(), code)
    assert hq.status(code.ws)[0] == 0
    rv, rg, st = oracle.decode_int8(oracle.encode(w, 128, oracle.E8, 0.29, 1))
    rng = np.random.default_rng(0)
    im = rng.integers(0, M, 512)
    ir = rng.integers(0, N, 512)
    tiles_m = max(1, M // 128)
    im = np.concatenate([im, np.repeat((np.arange(tiles_m) * 128 + 77) % M, 32)])
    ir = np.concatenate([ir, np.tile(np.arange(32) * 128 + 5, tiles_m)])
    ref = oracle.gemm_grouped_sample(a, sa, rv, rg, 128, im, ir)
    np.testing.assert_array_equal(Y.cpu().numpy()[im, ir], ref)
