"""The allocation-free encode entry point (hq_encode_noalloc) against the regular one.

Some callers cannot allocate GPU memory while they encode (a serving engine that owns a fixed
memory pool, code between synchronisation points where an allocation would stall the device).
hq_encode_noalloc keeps the encoder's scratch in a fixed array inside the library instead of a
caller-provided workspace.  This test calls it through the C ABI twice in a row -- the second
call finds the array holding the first call's contents -- and checks every output array bit for
bit against hq_encode on the same input.  It is collected last so a failure here leaves the
rest of the suite already run.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _noalloc_fn(hq):
    L = hq.lib()
    f = L.hq_encode_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(hq.Params),
                  ctypes.POINTER(hq.CodeStruct), ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int32
    return f


def test_noalloc_encode_matches_regular_encode_twice():
    import post_quantization_tile_b200 as hq
    from post_quantization_tile_b200 import workloads as W
    f = _noalloc_fn(hq)
    rows, cols, tile, beta, seed = 300, 1024, 128, 0.3, 17
    xb = W.llama_weight(4096, 4096, seed=1)[:rows, :cols]
    x = torch.from_numpy(np.ascontiguousarray(xb).view(np.int16)).view(torch.bfloat16).cuda()
    ref = hq.encode(x, tile, hq.E8, beta, seed=seed)
    assert hq.status(ref.ws)[0] == 0
    words = ref.total_words()
    p = hq.params(tile, hq.E8, beta, seed=seed)
    status = torch.full((1,), 0x7FFFFFFF, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = hq.alloc_code(rows, cols, p)
        cs = out.struct()
        rc = f(ctypes.c_void_p(x.data_ptr()), 0, rows, cols, ctypes.byref(p), ctypes.byref(cs),
               ctypes.c_void_p(status.data_ptr()), stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status bits {int(status.item()):#x}"
        assert cs.version == 2 and cs.rows == rows and cs.cols == cols and abs(cs.p.step - beta) < 1e-7
        assert torch.equal(out.chunk_word, ref.chunk_word)
        assert torch.equal(out.meta, ref.meta)
        assert torch.equal(out.scale, ref.scale)
        assert torch.equal(out.bits[:words], ref.bits[:words])
        # and it decodes like the regular code
        out.p = hq.Params(cs.p.tile, cs.p.lattice, cs.p.step, cs.p.bps, cs.p.seed)
        y = hq.decode(out, dtype=torch.float32)
        y_ref = hq.decode(ref, dtype=torch.float32)
        assert torch.equal(y, y_ref)


def test_noalloc_rejects_tensors_beyond_its_scratch():
    import post_quantization_tile_b200 as hq
    f = _noalloc_fn(hq)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = hq.params(128, hq.E8, 0.3)
    cs = hq.CodeStruct()
    # 65536 x 65536 at tile 128 needs 8 * 512 * 512 bytes of look-back slots, far above 128 KiB
    rc = f(ctypes.c_void_p(x.data_ptr()), 0, 65536, 65536, ctypes.byref(p), ctypes.byref(cs), None, None)
    assert rc == 7   # HQ_ERR_RANGE


def test_noalloc_accepts_managed_memory_like_the_regular_encoder():
    """A weight in CUDA managed memory (the caller's own pool may hand out managed buffers) is
    accepted like device memory, as hq_encode accepts it, and gives the same code."""
    import post_quantization_tile_b200 as hq
    from cuda.bindings import runtime as rt
    from post_quantization_tile_b200 import workloads as W
    f = _noalloc_fn(hq)
    rows, cols, tile, beta, seed = 96, 512, 128, 0.3, 5
    xb = np.ascontiguousarray(W.llama_weight(4096, 4096, seed=2)[:rows, :cols])
    err, ptr = rt.cudaMallocManaged(xb.nbytes, rt.cudaMemAttachGlobal)
    assert err == rt.cudaError_t.cudaSuccess
    try:
        err, = rt.cudaMemcpy(ptr, xb.ctypes.data, xb.nbytes, rt.cudaMemcpyKind.cudaMemcpyHostToDevice)
        assert err == rt.cudaError_t.cudaSuccess
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        ref = hq.encode(x, tile, hq.E8, beta, seed=seed)
        assert hq.status(ref.ws)[0] == 0
        p = hq.params(tile, hq.E8, beta, seed=seed)
        out = hq.alloc_code(rows, cols, p)
        cs = out.struct()
        status = torch.full((1,), 0x7FFFFFFF, dtype=torch.int32, device="cuda")
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = f(ctypes.c_void_p(int(ptr)), 0, rows, cols, ctypes.byref(p), ctypes.byref(cs),
               ctypes.c_void_p(status.data_ptr()), stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        words = ref.total_words()
        assert torch.equal(out.chunk_word, ref.chunk_word) and torch.equal(out.bits[:words], ref.bits[:words])
    finally:
        torch.cuda.synchronize()
        rt.cudaFree(ptr)
