"""The C-ABI library loads and exports every entry point the headers in include/ declare (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


def declared_functions(headers=None):
    text = "".join(open(h).read() for h in (headers or [h for h in HEADERS if not h.endswith("hq_test.h")]))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z_0-9]+)\s*\(", text)))


TEST_HEADER = os.path.join(ROOT, "include", "hq_test.h")


@pytest.fixture(scope="module")
def libhq():
    from post_quantization_tile_b200 import build
    if not os.path.exists(build.LIB):
        build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ["hq_encode", "hq_decode", "hq_kv_encode", "hq_kv_decode", "hq_quantize_coeffs", "hq_status_read"]:
        assert f in names


def test_library_exports_every_declared_symbol(libhq):
    missing = [f for f in declared_functions() if not hasattr(libhq, f)]
    assert not missing, missing


def test_test_entry_points_live_only_in_the_test_library(libhq):
    """hq_test.h's entry points are exported by libhq_test.so (built with the test hooks) and not
    by the product library; the test library also exports every product entry point."""
    from post_quantization_tile_b200 import build
    test_only = declared_functions([TEST_HEADER])
    assert test_only
    assert not [f for f in test_only if hasattr(libhq, f)]
    T = ctypes.CDLL(build.TEST_LIB)
    assert not [f for f in test_only + declared_functions() if not hasattr(T, f)]


def test_host_only_entry_points(libhq):
    import post_quantization_tile_b200 as hq
    L = hq.lib()
    p = hq.params(128, hq.E8, 0.3)
    assert L.hq_num_tiles(4096, 4096, 128) == 4096 * 32
    assert L.hq_num_chunks(4096, 4096, 128) == 32 * 128
    assert L.hq_num_chunks(70, 256, 64) == 4 * 3
    assert L.hq_num_tiles(10, 100, 64) == -1
    b = L.hq_encode_bound_words(4096, 4096, ctypes.byref(p))
    assert b % 4 == 0 and b >= 4096 * 32 * (16 * 128 + 2 * 128) // 32
    assert L.hq_workspace_bytes(4096, 4096, ctypes.byref(p)) % 256 == 0
    assert L.hq_version() == 2
    assert L.hq_status_str(3) == b"bitstream buffer too small"
    # high-resolution step: E8 at 4 bps ~ 2^(2.047 - 4)
    assert abs(L.hq_step_for_rate(hq.E8, 128, 4.0) - 2 ** (0.5 * __import__("math").log2(2 * 3.141592653589793 * 2.718281828459045) - 4)) < 1e-6


def test_calls_reject_bad_arguments_without_a_gpu(libhq):
    import post_quantization_tile_b200 as hq
    L = hq.lib()
    p = hq.params(100, hq.E8, 0.3)          # invalid tile
    cs = hq.CodeStruct()
    assert L.hq_encode(None, 0, 64, 128, ctypes.byref(p), ctypes.byref(cs), None, 0, None) == 1
    p = hq.params(128, hq.E8, 1e-4)         # step below 2^-8
    assert L.hq_encode(ctypes.c_void_p(16), 0, 64, 128, ctypes.byref(p), ctypes.byref(cs), ctypes.c_void_p(256),
                       1 << 20, None) == 1
    p = hq.params(128, hq.E8, 0.3)
    assert L.hq_kv_encode(ctypes.c_void_p(16), 0, 1, 1, 8, 64, ctypes.byref(p), ctypes.byref(cs), ctypes.c_void_p(256),
                          1 << 20, None) == 1   # head dimension != tile
    p = hq.params(100, hq.A2, 0.3)
    assert L.hq_encode_dither(None, 0, 64, 128, ctypes.byref(p), ctypes.byref(cs), None, 0, None) == 1
    p = hq.params(128, hq.Z, 0.3)
    assert L.hq_quantize_coeffs(ctypes.c_void_p(16), 8, ctypes.byref(p), 3, 0, None, ctypes.byref(cs),
                                ctypes.c_void_p(256), 1 << 20, None) == 1   # kv must be 0, 1 or 2


def test_dense_entry_points_check_arguments_without_a_gpu(libhq):
    import post_quantization_tile_b200 as hq
    L = hq.lib()
    need = L.hq_kv_dense_workspace_bytes(1000)
    assert need % 256 == 0 and need >= 1000 * 512 + 256 + L.hq_workspace_bytes(1000, 128, ctypes.byref(hq.params(128)))
    assert L.hq_kv_dense_workspace_bytes(0) == 0
    cs = hq.CodeStruct()
    q = ctypes.c_void_p(4096)
    p = hq.params(64, hq.D4, 1.0)            # head dimension 64: not provided
    assert L.hq_kv_encode_dense(ctypes.c_void_p(16), 0, 1, 1, 8, 64, 0, q, ctypes.byref(p), ctypes.byref(cs),
                                ctypes.c_void_p(256), 1 << 20, None) == 2
    p = hq.params(128, hq.D4, 1.0)
    assert L.hq_kv_encode_dense(ctypes.c_void_p(16), 0, 1, 1, 8, 64, 0, q, ctypes.byref(p), ctypes.byref(cs),
                                ctypes.c_void_p(256), 1 << 20, None) == 1   # D != tile
    assert L.hq_kv_encode_dense(ctypes.c_void_p(16), 0, 1, 1, 8, 128, -1, q, ctypes.byref(p), ctypes.byref(cs),
                                ctypes.c_void_p(256), 1 << 20, None) == 1   # negative first token
    assert L.hq_kv_encode_dense(ctypes.c_void_p(16), 0, 1, 1, 8, 128, 0, None, ctypes.byref(p), ctypes.byref(cs),
                                ctypes.c_void_p(256), 1 << 20, None) == 1   # no rotation
    cs.kv = 1                                # not a dense code
    cs.version = 2
    assert L.hq_kv_decode_dense(ctypes.byref(cs), q, ctypes.c_void_p(256), 1, ctypes.c_void_p(256), 1 << 20,
                                None) == 1


def test_fused_gemm_checks_arguments_without_a_gpu(libhq):
    import post_quantization_tile_b200 as hq
    L = hq.lib()
    # the status word only: every output element's chain stays in one CTA
    assert L.hq_gemm_code_workspace_bytes(128, 4096, 4096) >= 64
    assert L.hq_gemm_code_workspace_bytes(16, 4096, 4096) >= 64
    assert L.hq_gemm_code_workspace_bytes(16, 100, 4096) == 0      # N not a multiple of 128
    assert L.hq_gemm_code_workspace_bytes(0, 128, 128) == 0
    cs = hq.CodeStruct()
    cs.version, cs.kv, cs.rows, cs.cols = 2, 0, 128, 256
    cs.p = hq.params(256, hq.E8, 0.3)                              # tile 256: not provided
    ws = ctypes.c_void_p(256)
    assert L.hq_gemm_code(ctypes.c_void_p(16), ctypes.c_void_p(16), 16, ctypes.byref(cs), ctypes.c_void_p(16), ws,
                          1 << 20, None) == 2
    cs.p = hq.params(128, hq.A2, 0.3)                              # A2 codes: not provided
    assert L.hq_gemm_code(ctypes.c_void_p(16), ctypes.c_void_p(16), 16, ctypes.byref(cs), ctypes.c_void_p(16), ws,
                          1 << 20, None) == 2
    cs.p = hq.params(128, hq.E8, 0.3)
    cs.kv = 1                                                      # a dithered KV code
    assert L.hq_gemm_code(ctypes.c_void_p(16), ctypes.c_void_p(16), 16, ctypes.byref(cs), ctypes.c_void_p(16), ws,
                          1 << 20, None) == 1


def test_batch_entry_points_check_arguments_without_a_gpu(libhq):
    import post_quantization_tile_b200 as hq
    L = hq.lib()
    items = (hq.EncodeItem * 3)()
    for i in range(3):
        items[i].x = 16 * (i + 1)
        items[i].dtype = hq.BF16
        items[i].rows, items[i].cols = 300 + i, 512
        items[i].p = hq.params(128, hq.E8, 0.3)
    # one header and every item's look-back states: 3, 3 and 3 items of 128 rows x 4 tile columns
    per = [((300 + i + 127) // 128) * 4 for i in range(3)]
    assert L.hq_encode_batch_workspace_bytes(3, items) == 64 + 8 * sum(per)
    assert L.hq_encode_batch_workspace_bytes(0, items) == 0
    assert L.hq_encode_batch_workspace_bytes(17, items) == 0          # more than HQ_BATCH_MAX
    items[2].cols = 500                                                 # not a multiple of the tile
    assert L.hq_encode_batch_workspace_bytes(3, items) == 0
    ws = ctypes.c_void_p(256)
    assert L.hq_encode_batch(0, items, ws, 1 << 20, None) == 1
    assert L.hq_encode_batch(17, items, ws, 1 << 20, None) == 1
    assert L.hq_encode_batch(3, items, ws, 1 << 20, None) == 1         # the bad item
    dec = (hq.DecodeItem * 2)()
    assert L.hq_decode_batch(0, dec, ws, 4096, None) == 1
    assert L.hq_decode_batch(2, dec, ws, 4096, None) == 1              # no codes
