"""Exact-rate mode on the GPU (hq_step_search; Methodology step 3: the realised rate lands about
0.01 bps from any target): the device search takes exactly the oracle's probes (the counts are
bit-exact and the update rule is the same binary64 arithmetic), so step, probe count and payload
bits match the oracle's search; at full size it lands within 0.005 bps; it replays from a CUDA
graph with the same result."""
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


def t_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("lattice,n,target,step0", [(oracle.E8, 128, 4.0, 0.25), (oracle.E8, 64, 2.5, 2.0 ** -8),
                                                    (oracle.D4, 128, 3.0, 0.6), (oracle.A2, 256, 5.0, 0.2),
                                                    (oracle.Z, 128, 1.7, 1.0)])
def test_device_search_takes_the_oracles_probes(hq, lattice, n, target, step0):
    xb = W.llama_weight(96, 1024, seed=31)
    got = hq.step_search(t_bf16(xb), n, lattice, target, seed=7, step0=step0)
    want = oracle.step_search(xb, n, lattice, target, seed=7, step0=step0)
    assert got[0] == np.float32(want[0]) and got[1:] == want[1:], (got, want)


def test_device_search_kv_matches_oracle(hq):
    kb = W.kv_keys(1, 2, 96, 128, seed=2)
    got = hq.step_search(t_bf16(kb), 128, oracle.D4, 2.0, seed=3, step0=1.0)
    want = oracle.step_search(kb.reshape(-1, 128), 128, oracle.D4, 2.0, seed=3, kv=True, kv_S=96, step0=1.0)
    assert got[0] == np.float32(want[0]) and got[1:] == want[1:], (got, want)


def test_device_search_full_size(hq):
    x = t_bf16(W.llama_weight(4096, 4096, seed=1))
    for target in (3.0, 4.0, 5.0):
        step, probes, bits = hq.step_search(x, 128, hq.E8, target, seed=1)
        assert abs(bits / x.numel() - target) <= 0.005 and probes <= 16
        code = hq.encode(x, 128, hq.E8, step, seed=1)
        assert code.payload_bits() == bits
        assert hq.status(code.ws)[0] == 0


def test_device_search_replays_from_a_cuda_graph(hq):
    import ctypes
    x = t_bf16(W.llama_weight(512, 2048, seed=8))
    p = hq.params(128, hq.E8, 0.0, 4.0, 1)
    L = hq.lib()
    ws = hq.workspace(L.hq_workspace_bytes(512, 2048, ctypes.byref(p)))
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        rc = L.hq_step_search(ctypes.c_void_p(x.data_ptr()), 0, 512, 2048, ctypes.byref(p), 0, 0, 0, 0.0,
                              ctypes.c_void_p(res.data_ptr()), ws.ptr(), ws.nbytes,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    g.replay()
    torch.cuda.synchronize()
    first = res.clone()
    res.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(res, first)
    direct = hq.step_search(x, 128, hq.E8, 4.0, seed=1)
    r = first.cpu().tolist()
    assert (r[0] >> 32, r[1]) == direct[1:]
    del g
