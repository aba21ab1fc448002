"""The int8 tensor-core GEMM over lattice codes (tcgen05) and the decode to int8 codes, on the
GPU: bit-exact against the oracle's decode_int8 and grouped GEMM (exact group sums, binary32 fma
over groups), at small shapes over several CTA tiles, with more tiles than SMs (the persistent
CTAs take several tiles each) and, sampled, at 4096 x 4096 x 4096."""
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
    """int8 activations in the RHT domain: N(0, 32^2) clipped to +-127, and per-row scales"""
    rng = np.random.default_rng(seed)
    a = np.clip(np.round(rng.standard_normal((M, K)) * 32.0), -127, 127).astype(np.int8)
    sa = rng.uniform(0.01, 0.05, size=M).astype(np.float32)
    return a, sa


@pytest.mark.parametrize("lattice,n,beta", [(oracle.E8, 128, 0.3), (oracle.D4, 256, 0.45), (oracle.Z, 128, 0.35)])
def test_decode_int8_matches_oracle(hq, lattice, n, beta):
    w = W.llama_weight(200, 512, seed=15)
    code = hq.encode(t_bf16(w), n, lattice, beta, seed=3)
    v, g = hq.decode_int8(code)
    assert hq.status(code.ws)[0] == 0
    ref = oracle.encode(w, n, lattice, beta, 3)
    rv, rg, st = oracle.decode_int8(ref)
    assert st == 0
    np.testing.assert_array_equal(v.cpu().numpy(), rv)
    np.testing.assert_array_equal(g.cpu().numpy(), rg)


def test_decode_int8_flags_codes_outside_int8(hq):
    n = 128
    u = np.random.default_rng(6).standard_normal((64, n)).astype(np.float32) * 3.0
    u[5, 7] = 80.0
    _, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, hq.E8)
    code.scale.fill_(0x3F80)
    code.p.step = 1.0
    v, g = hq.decode_int8(code)
    assert hq.status(code.ws)[0] == 7           # HQ_ERR_RANGE
    assert torch.all(v[5] == 0) and torch.any(v[4] != 0)


# tile widths: 32 columns (the first three shapes; 512 x 2048 with more tiles than SMs), 64 (1024 x
# 2048: the 128-wide tiles would leave SMs idle, the 64-wide ones fill them) and 128 (2048 x 1280)
@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 384, 1024), (384, 256, 2048), (512, 2048, 256),
                                   (1024, 2048, 256), (2048, 1280, 256)])
def test_gemm_int8_bit_exact(hq, M, N, K):
    w = W.llama_weight(N, K, seed=K + N)
    code = hq.encode(t_bf16(w), 128, hq.E8, 0.3, seed=5)
    V, g = hq.decode_int8(code)
    a, sa = _acts(M, K, seed=M)
    Y = hq.gemm_int8(torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda(), V, g)
    torch.cuda.synchronize()
    assert hq.status(hq.workspace(4096))[0] == 0
    ref = oracle.gemm_grouped(a, sa, V.cpu().numpy(), g.cpu().numpy(), 128)
    np.testing.assert_array_equal(Y.cpu().numpy(), ref)


def test_gemm_int8_full_size_sampled(hq):
    M = N = K = 4096
    w = W.llama_weight(N, K, seed=1)
    code = hq.encode(t_bf16(w), 128, hq.E8, 0.29, seed=1)
    V, g = hq.decode_int8(code)
    assert hq.status(code.ws)[0] == 0
    a, sa = _acts(M, K, seed=6)
    Y = hq.gemm_int8(torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda(), V, g)
    rng = np.random.default_rng(0)
    im = rng.integers(0, M, 512)
    ir = rng.integers(0, N, 512)
    # every 128 x 128 output tile gets a sample too
    im = np.concatenate([im, np.repeat(np.arange(32) * 128 + 77, 32)])
    ir = np.concatenate([ir, np.tile(np.arange(32) * 128 + 5, 32)])
    ref = oracle.gemm_grouped_sample(a, sa, V.cpu().numpy(), g.cpu().numpy(), 128, im, ir)
    got = Y.cpu().numpy()[im, ir]
    np.testing.assert_array_equal(got, ref)
