"""Dense-rotation KV variant on the GPU (Methodology step 4: the per-layer rotation as a dense
Haar-random orthogonal matrix instead of the sign diagonal) against the oracle: scales, Rice
parameters, chunk offsets and bitstreams bit for bit (the rotation is the same binary32 fma chain
on both sides, so every lattice decision agrees), reconstructions within the codec's tolerance of
the oracle's binary64 decode; ragged row counts, fp32 input, token append, zero and non-finite
head vectors, sampled rows of the full KV workload, and the calls that must refuse."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from post_quantization_tile_b200 import workloads as W
from test_gpu_parity import _decode_check, assert_same_code, t_bf16, u16

pytestmark = pytest.mark.gpu

LATS = [oracle.Z, oracle.A2, oracle.D4, oracle.E8]


@pytest.fixture(scope="module")
def hq():
    import post_quantization_tile_b200 as m
    m.lib()
    return m


@pytest.fixture(scope="module")
def Q():
    return W.haar_rotation(128, seed=8)


def _check_decode(hq, code, ref, Q, Qd):
    xo, st = oracle.decode_dense(ref, Q)
    assert st == 0
    for dt in (torch.float32, torch.bfloat16):
        y = hq.kv_decode_dense(code, Qd, dtype=dt)
        assert hq.status(code.ws)[0] == 0
        _decode_check(y, ref, xo)


@pytest.mark.parametrize("lattice,beta", [(oracle.Z, 0.5), (oracle.A2, 0.6), (oracle.D4, 0.9), (oracle.E8, 0.45)])
def test_dense_encode_bit_exact_and_decode(hq, Q, lattice, beta):
    B, H, S = 1, 3, 77                     # 231 head vectors: ragged against 64-row steps and 32-row chunks
    kb = W.kv_keys(B, H, S, 128, seed=6)
    Qd = torch.from_numpy(Q).cuda()
    code = hq.kv_encode_dense(t_bf16(kb), Qd, step=beta, seed=13, lattice=lattice)
    assert hq.status(code.ws)[0] == 0 and code.kv == hq.KV_DENSE
    ref = oracle.encode_dense(kb.reshape(-1, 128), Q, lattice, beta, 13, kv_S=S)
    assert_same_code(code, ref, "dense")
    _check_decode(hq, code, ref, Q, Qd)


def test_dense_fp32_input(hq, Q):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 2, 50, 128)).astype(np.float32)
    x[..., 5] *= 30.0
    Qd = torch.from_numpy(Q).cuda()
    code = hq.kv_encode_dense(torch.from_numpy(x).cuda(), Qd, step=0.7, seed=5, lattice=oracle.D4)
    assert hq.status(code.ws)[0] == 0
    ref = oracle.encode_dense(x.reshape(-1, 128), Q, oracle.D4, 0.7, 5, kv_S=50)
    assert_same_code(code, ref, "dense fp32")
    _check_decode(hq, code, ref, Q, Qd)


@pytest.mark.parametrize("lattice", [oracle.D4, oracle.E8])
def test_dense_token_append(hq, Q, lattice):
    B, H, S, s0 = 2, 4, 3, 1021            # a decode step of three tokens per (b, h) at position 1021
    kb = W.kv_keys(B, H, S, 128, seed=9)
    Qd = torch.from_numpy(Q).cuda()
    code = hq.kv_encode_dense(t_bf16(kb), Qd, step=1.1, seed=29, lattice=lattice, s0=s0)
    assert hq.status(code.ws)[0] == 0 and code.kv_s0 == s0
    ref = oracle.encode_dense(kb.reshape(-1, 128), Q, lattice, 1.1, 29, kv_S=S, kv_s0=s0)
    assert_same_code(code, ref, "dense append")
    _check_decode(hq, code, ref, Q, Qd)


def test_dense_zero_and_nonfinite_vectors(hq, Q):
    kb = W.kv_keys(1, 2, 40, 128, seed=4).reshape(-1, 128).copy()
    kb[3] = 0
    kb[17, 9] = 0x7F80     # +inf
    kb[50, 100] = 0x7FC0   # NaN
    Qd = torch.from_numpy(Q).cuda()
    code = hq.kv_encode_dense(t_bf16(kb.reshape(1, 2, 40, 128)), Qd, step=0.8, seed=2, lattice=oracle.E8)
    st, detail = hq.status(code.ws)
    assert st == 4 and detail == 2      # HQ_ERR_NONFINITE, two vectors
    ref = oracle.encode_dense(kb, Q, oracle.E8, 0.8, 2, kv_S=40)
    assert ref.status & oracle.ST_NONFINITE
    assert_same_code(code, ref, "dense non-finite")
    y = hq.kv_decode_dense(code, Qd, dtype=torch.float32)
    assert hq.status(code.ws)[0] == 0
    yh = y.cpu().numpy()
    assert np.all(yh[3] == 0) and np.all(yh[17] == 0) and np.all(yh[50] == 0)
    xo, _ = oracle.decode_dense(ref, Q)
    _decode_check(y, ref, xo)


def test_dense_full_kv_workload_sampled_rows(hq, Q):
    """[8, 32, 8192, 128] bf16 keys (268 M scalars), D4 at the 2-bps step: the whole tensor in one
    call; sampled 64-row windows against the oracle (scales and Rice parameters exact, decoded rows
    within tolerance; the windows' bitstreams start at other chunk offsets)."""
    B, H, S, D = 8, 32, 8192, 128
    kb = W.kv_keys(B, H, S, D, seed=2)
    x = t_bf16(kb)
    flat = kb.reshape(-1, D)
    del kb
    Qd = torch.from_numpy(Q).cuda()
    beta = 1.25
    code = hq.kv_encode_dense(x, Qd, step=beta, seed=7, lattice=oracle.D4)
    assert hq.status(code.ws)[0] == 0
    del x
    y = hq.kv_decode_dense(code, Qd, dtype=torch.float32)
    assert hq.status(code.ws)[0] == 0
    scale, meta = u16(code.scale), u16(code.meta)
    rows = B * H * S
    for r0 in (0, 64 * 12345, rows // 2 + 32 * 7, rows - 64):
        win = np.ascontiguousarray(flat[r0:r0 + 64])
        ref = oracle.encode_dense(win, Q, oracle.D4, beta, 7, kv_S=S, row0=r0)
        np.testing.assert_array_equal(scale[r0:r0 + 64], ref.scale)
        np.testing.assert_array_equal(meta[r0:r0 + 64], ref.meta)
        xo, _ = oracle.decode_dense(ref, Q)
        _decode_check(y[r0:r0 + 64], ref, xo)
    bps = code.payload_bps()
    assert 1.5 < bps < 2.6


def test_dense_codes_refuse_the_other_decoders_and_other_sizes(hq, Q):
    kb = W.kv_keys(1, 1, 8, 128, seed=1)
    Qd = torch.from_numpy(Q).cuda()
    code = hq.kv_encode_dense(t_bf16(kb), Qd, step=1.0, seed=1)
    with pytest.raises(ValueError):
        hq.decode(code)
    L = hq.lib()
    cs = code.struct()
    y = torch.empty(8, 128, dtype=torch.float32, device="cuda")
    w = hq.workspace(1 << 20)
    assert L.hq_kv_decode(ctypes.byref(cs), ctypes.c_void_p(y.data_ptr()), 1, w.ptr(), w.nbytes, None) == 1
    assert L.hq_decode(ctypes.byref(cs), ctypes.c_void_p(y.data_ptr()), 1, w.ptr(), w.nbytes, None) == 1
    # head dimension 64: not provided
    k64 = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    Q64 = torch.eye(64, dtype=torch.float32, device="cuda")
    p = hq.params(64, oracle.D4, 1.0)
    out = hq.alloc_code(8, 64, p)
    cs64 = out.struct()
    rc = L.hq_kv_encode_dense(ctypes.c_void_p(k64.data_ptr()), 0, 1, 1, 8, 64, 0, ctypes.c_void_p(Q64.data_ptr()),
                              ctypes.byref(p), ctypes.byref(cs64), w.ptr(), w.nbytes, None)
    assert rc == 2   # HQ_ERR_UNSUPPORTED
    # too small a workspace
    p128 = hq.params(128, oracle.D4, 1.0)
    out = hq.alloc_code(8, 128, p128)
    cs128 = out.struct()
    need = L.hq_kv_dense_workspace_bytes(8)
    xk = t_bf16(kb)
    rc = L.hq_kv_encode_dense(ctypes.c_void_p(xk.data_ptr()), 0, 1, 1, 8, 128, 0, ctypes.c_void_p(Qd.data_ptr()),
                              ctypes.byref(p128), ctypes.byref(cs128), w.ptr(), need - 256, None)
    assert rc == 1   # HQ_ERR_ARG


def test_dense_dither_unbiased_on_gpu(hq, Q):
    """Per key vector and query, the inner-product error over fresh dithers has mean zero (the
    dither keeps the variant unbiased whatever the rotation); 512 keys x 32 queries, 192 seeds."""
    kb = W.kv_keys(1, 4, 128, 128, seed=2)
    keys = t_bf16(kb)
    x = keys.float().reshape(-1, 128).double()
    q = torch.from_numpy(W.queries(32, 128, seed=3)).cuda()
    Qd = torch.from_numpy(Q).cuda()
    M = 192
    E = torch.zeros(M, x.shape[0], 32, dtype=torch.float64, device="cuda")
    for m in range(M):
        code = hq.kv_encode_dense(keys, Qd, step=1.6, seed=7000 + m)
        y = hq.kv_decode_dense(code, Qd, dtype=torch.float32).double()
        E[m] = (y - x) @ q.T
    assert hq.status(code.ws)[0] == 0
    z = E.mean(0) / (E.std(0) / np.sqrt(M))
    assert (z.abs() > 4.5).float().mean().item() <= 1e-3


def test_dense_replay_from_a_graph(hq, Q):
    kb = W.kv_keys(1, 2, 96, 128, seed=8)
    keys = t_bf16(kb)
    Qd = torch.from_numpy(Q).cuda()
    ref = hq.kv_encode_dense(keys, Qd, step=0.8, seed=3, lattice=oracle.E8)
    y_ref = hq.kv_decode_dense(ref, Qd, dtype=torch.float32)
    code = hq.alloc_code(keys.numel() // 128, 128, hq.params(128, oracle.E8, 0.8, seed=3))
    ws = hq.Workspace(hq.lib().hq_kv_dense_workspace_bytes(keys.numel() // 128))
    y = torch.empty_like(y_ref)
    hq.kv_encode_dense(keys, Qd, step=0.8, seed=3, lattice=oracle.E8, out=code, ws=ws)   # warm-up
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        hq.kv_encode_dense(keys, Qd, step=0.8, seed=3, lattice=oracle.E8, out=code, ws=ws)
        hq.kv_decode_dense(code, Qd, out=y, ws=ws)
    code.bits.zero_()
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert hq.status(ws)[0] == 0
    assert torch.equal(code.bits[:ref.total_words()], ref.bits[:ref.total_words()])
    assert torch.equal(code.scale, ref.scale)
    assert torch.equal(y, y_ref)


def test_dense_damaged_stream_and_canaries(hq, Q):
    """A truncated dense-rotation stream decodes to HQ_ERR_CORRUPT with finite output, and nothing
    is written past the output buffer."""
    from test_gpu_faults import _guarded, _intact
    kb = W.kv_keys(1, 2, 64, 128, seed=5)
    Qd = torch.from_numpy(Q).cuda()
    code = hq.kv_encode_dense(t_bf16(kb), Qd, step=0.9, seed=4, lattice=oracle.E8)
    assert hq.status(code.ws)[0] == 0
    words = code.total_words()
    code.bits[words // 2:words] = 0                      # the second half of the stream is lost
    rows = 128
    yfull, y = _guarded(rows * 128, torch.float32)
    hq.kv_decode_dense(code, Qd, out=y.view(rows, 128))
    assert hq.status(code.ws)[0] == 5                    # HQ_ERR_CORRUPT
    assert _intact(yfull, rows * 128)
    assert bool(torch.isfinite(y).all().item())
