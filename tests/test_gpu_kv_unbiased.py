"""On the GPU path, dithered KV inner products are unbiased for every single key vector, not only
on average over vectors (Subtractive Dither, Methodology step 4; the proof is Appendix A), and the
dither's error is uniform on the Voronoi cell of D4.

For 1024 key vectors of the KV workload and 64 random queries, over M = 256 seeds (each seed a
fresh sign diagonal and dither): e = <q, x_hat> - <q, x>; per pair z = mean(e) / (sd(e)/sqrt M).
Without the dither the same test at 1.7 bps shows a systematic shrinkage (negative control).
"""
import numpy as np
import pytest
import torch

from post_quantization_tile_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _errors(hq, keys, q, beta, kv, M=256):
    B, H, S, D = keys.shape
    x = keys.float().reshape(-1, D).double()
    ref = x @ q.T
    self_ref = (x * x).sum(1)
    E = torch.zeros((M,) + ref.shape, dtype=torch.float64, device="cuda")
    Es = torch.zeros((M, x.shape[0]), dtype=torch.float64, device="cuda")
    for m in range(M):
        if kv:
            code = hq.kv_encode(keys, step=beta, seed=5000 + m)
        else:
            code = hq.encode(keys.reshape(-1, D), D, hq.D4, beta, seed=5000 + m)
        y = hq.decode(code, dtype=torch.float32).reshape(-1, D).double()
        E[m] = y @ q.T - ref
        Es[m] = (y * x).sum(1) - self_ref
    assert hq.status(code.ws)[0] == 0
    z = E.mean(0) / (E.std(0) / np.sqrt(M))
    zs = Es.mean(0) / (Es.std(0) / np.sqrt(M))
    return z, zs


def test_kv_dither_unbiased_on_gpu():
    import post_quantization_tile_b200 as hq
    kb = W.kv_keys(1, 8, 128, 128, seed=2)                      # 1024 key vectors
    keys = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda()
    q = torch.from_numpy(W.queries(64, 128, seed=3)).cuda()
    for beta in (1.6, 0.6):                                       # ~1.7 and ~3 bps
        z, zs = _errors(hq, keys, q, beta, kv=True)
        assert (z.abs() > 4.5).float().mean().item() <= 1e-3     # 65536 pairs
        assert zs.abs().max().item() < 5.5
    z, zs = _errors(hq, keys, q, 1.6, kv=False)                  # deterministic quantizer
    assert zs.abs().max().item() > 10.0


def test_kv_dither_error_uniform_on_cell_gpu():
    import post_quantization_tile_b200 as hq
    kb = W.kv_keys(2, 8, 512, 128, seed=7)
    keys = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda()
    beta = 0.7
    code = hq.kv_encode(keys, step=beta, seed=11)
    y = hq.decode(code, dtype=torch.float32).reshape(-1, 128).double()
    x = keys.float().reshape(-1, 128).double()
    sh = (code.scale.to(torch.int32) << 16).view(torch.float32).double()
    mse_u = (((y - x) ** 2).sum(1) / (128 * (sh * beta) ** 2)).mean().item()
    assert abs(mse_u / (0.0766032346 * np.sqrt(2.0)) - 1.0) < 0.01
