"""Encode / decode / KV / GEMM replayed from CUDA graphs give the direct calls' results bit for
bit; edge shapes (one row, one tile, a ragged last chunk, all-zero and constant tensors) match
the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W
from test_gpu_parity import _decode_check, assert_same_code, t_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


def test_encode_decode_replay_from_a_graph(hq):
    x = t_bf16(W.llama_weight(640, 1024, seed=3))
    direct = hq.encode(x, 128, hq.E8, 0.3, seed=2)
    yd = hq.decode(direct)
    code = hq.alloc_code(640, 1024, hq.params(128, hq.E8, 0.3, 4.0, 2))
    y = torch.empty_like(x)
    L = hq.lib()
    p = hq.params(128, hq.E8, 0.3, 4.0, 2)
    wse = hq.Workspace(L.hq_workspace_bytes(640, 1024, ctypes.byref(p)))
    wsd = hq.Workspace(4096)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        cs = code.struct()
        st = torch.cuda.current_stream().cuda_stream
        assert L.hq_encode(ctypes.c_void_p(x.data_ptr()), 0, 640, 1024, ctypes.byref(p), ctypes.byref(cs), wse.ptr(),
                           wse.nbytes, ctypes.c_void_p(st)) == 0
        assert L.hq_decode(ctypes.byref(cs), ctypes.c_void_p(y.data_ptr()), 0, wsd.ptr(), wsd.nbytes,
                           ctypes.c_void_p(st)) == 0
    for _ in range(3):
        y.zero_()
        code.bits.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert hq.status(wse)[0] == 0 and hq.status(wsd)[0] == 0
        words = direct.total_words()
        assert torch.equal(code.bits[:words], direct.bits[:words])
        assert torch.equal(code.chunk_word, direct.chunk_word)
        assert torch.equal(y, yd)
    del g


@pytest.mark.parametrize("rows,cols,n,lattice", [(1, 128, 128, oracle.E8), (1, 64, 64, oracle.D4),
                                                 (33, 256, 128, oracle.A2), (31, 512, 256, oracle.Z),
                                                 (129, 128, 128, oracle.E8)])
def test_edge_shapes_match_oracle(hq, rows, cols, n, lattice):
    xb = W.llama_weight(4096, 4096, seed=7)[:rows, :cols]
    code = hq.encode(t_bf16(np.ascontiguousarray(xb)), n, lattice, 0.3, seed=8)
    assert hq.status(code.ws)[0] == 0
    ref = oracle.encode(np.ascontiguousarray(xb), n, lattice, 0.3, 8)
    assert_same_code(code, ref, "edge")
    y = hq.decode(code, dtype=torch.float32)
    xo, _ = oracle.decode(ref)
    _decode_check(y, ref, xo)


@pytest.mark.parametrize("fill", [0x0000, 0x3F80, 0xBF80])
def test_zero_and_constant_tensors(hq, fill):
    xb = np.full((64, 256), fill, dtype=np.uint16)     # 0, +1, -1 everywhere
    code = hq.encode(t_bf16(xb), 128, hq.E8, 0.3, seed=1)
    assert hq.status(code.ws)[0] == 0
    ref = oracle.encode(xb, 128, oracle.E8, 0.3, 1)
    assert_same_code(code, ref, "constant")
    y = hq.decode(code, dtype=torch.float32)
    xo, _ = oracle.decode(ref)
    _decode_check(y, ref, xo)
