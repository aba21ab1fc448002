"""Subtractive dither on every lattice, on the GPU (Methodology step 4, "Subtractive Dither"):
codes and bitstreams bit-exact against the oracle for quantize_coeffs (KV rows and the weight
option), KV encodes of E8 / A2 / Z, dithered weight encodes; reconstructions within the codec's
tolerance of the oracle's binary64 decode; and, on the GPU path itself, per-vector unbiasedness
and the dithered error's closed-form second moment."""
import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W
from test_gpu_parity import _coeffs, _decode_check, assert_same_code, t_bf16, u32

pytestmark = pytest.mark.gpu

LATS = [oracle.Z, oracle.A2, oracle.D4, oracle.E8]


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("lattice", LATS)
@pytest.mark.parametrize("n", [64, 128, 256])
@pytest.mark.parametrize("kv", [1, 2])
def test_quantize_coeffs_dither_bit_exact(hq, lattice, n, kv):
    u = _coeffs(n, 150, 3 * n + lattice, lattice)
    v, code = hq.quantize_coeffs(torch.from_numpy(u).cuda(), n, lattice, seed=77, kv=kv, kv_S=50)
    assert hq.status(code.ws)[0] == 0
    rv, rmeta, rcw, rbits, _ = oracle.quantize_coeffs(u, n, lattice, seed=77, kv=kv, kv_S=50)
    np.testing.assert_array_equal(v.cpu().numpy(), rv)
    np.testing.assert_array_equal(u32(code.chunk_word), rcw)
    np.testing.assert_array_equal(u32(code.bits)[: int(rcw[-1])], rbits)


@pytest.mark.parametrize("lattice,beta", [(oracle.E8, 0.45), (oracle.A2, 0.6), (oracle.Z, 0.5), (oracle.D4, 0.9)])
def test_kv_encode_decode_every_lattice(hq, lattice, beta):
    B, H, S, D = 1, 4, 72, 128
    kb = W.kv_keys(B, H, S, D, seed=6)
    code = hq.kv_encode(t_bf16(kb), step=beta, seed=13, lattice=lattice)
    assert hq.status(code.ws)[0] == 0
    ref = oracle.encode(kb.reshape(-1, D), D, lattice, beta, 13, kv=True, kv_S=S)
    assert_same_code(code, ref, "kv")
    y = hq.kv_decode(code, (B, H, S, D), dtype=torch.float32)
    xo, _ = oracle.decode(ref)
    _decode_check(y.reshape(-1, D), ref, xo)


@pytest.mark.parametrize("lattice,n,beta", [(oracle.E8, 128, 0.3), (oracle.A2, 256, 0.4), (oracle.Z, 64, 0.35),
                                            (oracle.D4, 128, 0.5)])
def test_dithered_weight_encode_decode(hq, lattice, n, beta):
    xb = W.llama_weight(200, 512, seed=12)
    code = hq.encode(t_bf16(xb), n, lattice, beta, seed=4, dither=True)
    assert hq.status(code.ws)[0] == 0 and code.kv == 2
    ref = oracle.encode(xb, n, lattice, beta, 4, kv=2)
    assert_same_code(code, ref, "dithered weight")
    for dt in (torch.float32, torch.bfloat16):
        y = hq.decode(code, dtype=dt)
        assert hq.status(code.ws)[0] == 0
        xo, _ = oracle.decode(ref)
        _decode_check(y, ref, xo)


@pytest.mark.parametrize("lattice", [oracle.E8, oracle.A2, oracle.Z])
def test_gpu_dither_unbiased_and_cell_moment(hq, lattice):
    kb = W.kv_keys(1, 8, 64, 128, seed=2)                     # 512 key vectors
    keys = t_bf16(kb)
    x = keys.float().reshape(-1, 128).double()
    q = torch.from_numpy(W.queries(32, 128, seed=3)).cuda()
    M, beta = 192, 0.8
    E = torch.zeros(M, x.shape[0], 32, dtype=torch.float64, device="cuda")
    for m in range(M):
        code = hq.kv_encode(keys, step=beta, seed=900 + m, lattice=lattice)
        y = hq.decode(code, dtype=torch.float32).reshape(-1, 128).double()
        E[m] = (y - x) @ q.T
    z = E.mean(0) / (E.std(0) / np.sqrt(M))
    assert (z.abs() > 4.5).float().mean().item() <= 1e-3
    # per-dimension error in lattice units: the cell's second moment
    sh = ((code.scale.to(torch.int32) & 0xFFFF) << 16).view(torch.float32).double()
    mse_u = (((y - x) ** 2).sum(1) / (128 * (sh * beta) ** 2)).mean().item()
    moment = {oracle.Z: 1 / 12, oracle.A2: 5 / 72, oracle.E8: 929 / 12960}[lattice]
    assert abs(mse_u / moment - 1.0) < 0.02


@pytest.mark.parametrize("lattice", [oracle.D4, oracle.E8])
def test_token_append_matches_whole_sequence_and_oracle(hq, lattice):
    B, H, S, D = 2, 4, 48, 128
    kb = W.kv_keys(B, H, S, D, seed=21)
    full = hq.kv_encode(t_bf16(kb), step=0.8, seed=9, lattice=lattice)
    yf = hq.kv_decode(full, (B, H, S, D), dtype=torch.float32)
    for s0 in (1, 33, 47):
        step = np.ascontiguousarray(kb[:, :, s0:s0 + 1, :])               # [B, H, 1, D]
        app = hq.kv_encode(t_bf16(step), step=0.8, seed=9, lattice=lattice, s0=s0)
        assert hq.status(app.ws)[0] == 0 and app.kv_s0 == s0
        ya = hq.kv_decode(app, (B, H, 1, D), dtype=torch.float32)
        assert torch.equal(ya[:, :, 0], yf[:, :, s0])
        ref = oracle.encode(step.reshape(-1, D), D, lattice, 0.8, 9, kv=True, kv_S=1, kv_s0=s0)
        assert_same_code(app, ref, "append")
