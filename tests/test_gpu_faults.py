"""Failure detection without a GPU fault: a bounded wait that runs out reports HQ_ERR_TIMEOUT and
leaves the context usable; canary words after every output buffer survive encode, decode and
the int8 GEMM; bit-flipped and truncated streams decode to a status, within bounds."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W
from test_gpu_parity import assert_same_code, t_bf16

pytestmark = pytest.mark.gpu

CANARY = 0x5A5A5A5A


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


@pytest.fixture(scope="module")
def test_lib(hq):
    """libhq_test.so: the library built with the test hooks (the product library has none)."""
    from post_quantization_tile_b200 import build
    T = ctypes.CDLL(build.TEST_LIB)
    T.hq_test_encode_silent_item.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.POINTER(hq.Params), ctypes.POINTER(hq.CodeStruct), ctypes.c_void_p,
                                             ctypes.c_size_t, ctypes.c_int64, ctypes.c_void_p]
    T.hq_test_encode_silent_item.restype = ctypes.c_int32
    T.hq_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(hq.Params)]
    T.hq_workspace_bytes.restype = ctypes.c_size_t
    return T


def test_silent_item_times_out_and_the_context_survives(hq, test_lib):
    xb = W.llama_weight(1024, 512, seed=2)
    x = t_bf16(xb)
    p = hq.params(128, hq.E8, 0.3, 4.0, 3)
    code = hq.alloc_code(1024, 512, p)
    L = test_lib
    ws = hq.Workspace(L.hq_workspace_bytes(1024, 512, ctypes.byref(p)))
    cs = code.struct()
    rc = L.hq_test_encode_silent_item(ctypes.c_void_p(x.data_ptr()), 0, 1024, 512, ctypes.byref(p), ctypes.byref(cs),
                                      ws.ptr(), ws.nbytes, 5, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    assert hq.status(ws)[0] == 6                      # HQ_ERR_TIMEOUT, read on the host
    # the context is usable: a normal encode right after matches the oracle bit for bit
    again = hq.encode(x, 128, hq.E8, 0.3, seed=3)
    assert hq.status(again.ws)[0] == 0
    assert_same_code(again, oracle.encode(xb, 128, oracle.E8, 0.3, 3), "after timeout")


def _guarded(n, dtype, device="cuda", pad=64):
    """a tensor of n elements followed by `pad` canary elements"""
    full = torch.empty(n + pad, dtype=dtype, device=device)
    full.view(torch.uint8).fill_(0x5A)
    return full, full[:n]


def _intact(full, n):
    return bool(torch.all(full[n:].contiguous().view(torch.uint8) == 0x5A).item())


def test_canaries_after_encode_and_decode_outputs(hq):
    rows, cols, n = 300, 640, 128
    xb = W.llama_weight(rows, cols, seed=4)
    p = hq.params(n, hq.E8, 0.3, 4.0, 9)
    L = hq.lib()
    T, C = L.hq_num_tiles(rows, cols, n), L.hq_num_chunks(rows, cols, n)
    cap = L.hq_encode_bound_words(rows, cols, ctypes.byref(p))
    sfull, scale = _guarded(T, torch.int16)
    mfull, meta = _guarded(T, torch.int16)
    cfull, cw = _guarded(C + 1, torch.int32)
    bfull, bits = _guarded(cap, torch.int32)
    code = hq.Code(rows, cols, p, 0, 0, scale, meta, cw, bits)
    code = hq.encode(t_bf16(xb), n, hq.E8, 0.3, seed=9, out=code)
    assert hq.status(code.ws)[0] == 0
    assert all(_intact(f, k) for f, k in ((sfull, T), (mfull, T), (cfull, C + 1), (bfull, cap)))
    assert_same_code(code, oracle.encode(xb, n, oracle.E8, 0.3, 9), "guarded")
    for dt in (torch.bfloat16, torch.float32):
        yfull, y = _guarded(rows * cols, dt)
        hq.decode(code, out=y.view(rows, cols))
        assert hq.status(code.ws)[0] == 0 and _intact(yfull, rows * cols)
    vfull, v = _guarded(rows * cols, torch.int8)
    gfull, g = _guarded(rows * cols // n, torch.float32)
    L.hq_decode_int8(ctypes.byref(code.struct()), ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                     code.ws.ptr(), code.ws.nbytes, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert hq.status(code.ws)[0] == 0 and _intact(vfull, rows * cols) and _intact(gfull, rows * cols // n)


def test_canary_after_gemm_output(hq):
    M, N, K = 256, 384, 512
    code = hq.encode(t_bf16(W.llama_weight(N, K, seed=5)), 128, hq.E8, 0.3, seed=5)
    V, g = hq.decode_int8(code)
    a = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda")
    sa = torch.full((M,), 0.5, device="cuda")
    yfull, y = _guarded(M * N, torch.float32)
    hq.gemm_int8(a, sa, V, g, out=y.view(M, N))
    torch.cuda.synchronize()
    assert hq.status(hq.workspace(4096))[0] == 0 and _intact(yfull, M * N)


@pytest.mark.parametrize("damage", ["flip", "truncate"])
def test_damaged_streams_decode_to_a_status_within_bounds(hq, damage):
    rows, cols = 256, 512
    code = hq.encode(t_bf16(W.llama_weight(rows, cols, seed=6)), 128, hq.E8, 0.3, seed=6)
    words = code.total_words()
    rng = np.random.default_rng(1)
    if damage == "flip":
        idx = torch.from_numpy(rng.integers(0, words, 64)).cuda()
        bit = torch.from_numpy((1 << rng.integers(0, 31, 64)).astype(np.int32)).cuda()
        code.bits[idx] ^= bit
    else:
        code.bits[words // 2:words] = 0                  # the second half of the stream is lost
    yfull, y = _guarded(rows * cols, torch.bfloat16)
    hq.decode(code, out=y.view(rows, cols))
    st = hq.status(code.ws)[0]
    assert st in (0, 5)                                  # ok, or HQ_ERR_CORRUPT with those tiles zeroed
    if damage == "truncate":
        assert st == 5
    assert _intact(yfull, rows * cols)
