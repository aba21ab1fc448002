"""Several tensors in one launch (hq_encode_batch, hq_decode_batch), on the GPU: each item's code
-- chunk offsets, meta, scales, bitstream -- is bit for bit the code of its own hq_encode call
(itself pinned to the oracle in test_gpu_parity.py), and each decoded tensor equals its own
hq_decode; ragged shapes, several tile columns, per-item steps and seeds, bf16 and fp32, the
largest batch; mixed tile sizes or lattices are refused."""
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


def _same_code(a, b):
    assert (a.rows, a.cols, a.kv) == (b.rows, b.cols, b.kv)
    assert a.p.step == b.p.step and a.p.seed == b.p.seed
    words = a.total_words()
    assert words == b.total_words()
    assert torch.equal(a.chunk_word, b.chunk_word)
    assert torch.equal(a.meta, b.meta)
    assert torch.equal(a.scale, b.scale)
    assert torch.equal(a.bits[:words], b.bits[:words])


SHAPES = [(300, 512), (77, 256), (1024, 1024), (128, 384), (513, 128)]


@pytest.mark.parametrize("lattice,n", [(oracle.E8, 128), (oracle.D4, 64), (oracle.Z, 256), (oracle.A2, 128)])
def test_encode_batch_equals_single_encodes_bf16(hq, lattice, n):
    shapes = [(r, c) for r, c in SHAPES if c % n == 0]
    xs = [t_bf16(W.llama_weight(r, c, seed=20 + i)) for i, (r, c) in enumerate(shapes)]
    steps = [0.25 + 0.05 * i for i in range(len(xs))]
    seeds = [100 + 7 * i for i in range(len(xs))]
    codes = hq.encode_batch(xs, n, lattice, steps, seeds)
    assert hq.status(codes[0].ws)[0] == 0
    for x, code, beta, seed in zip(xs, codes, steps, seeds):
        ref = hq.encode(x, n, lattice, beta, seed=seed)
        assert hq.status(ref.ws)[0] == 0
        _same_code(code, ref)
    ys = hq.decode_batch(codes)
    assert hq.status(codes[0].ws)[0] == 0
    for code, y in zip(codes, ys):
        assert torch.equal(y, hq.decode(code))


def test_encode_batch_fp32_and_fp32_output(hq):
    rng = np.random.default_rng(3)
    xs = [torch.from_numpy((rng.standard_normal((r, c)) * 0.02).astype(np.float32)).cuda() for r, c in SHAPES[:3]]
    codes = hq.encode_batch(xs, 128, oracle.E8, [0.3, 0.28, 0.31], [1, 2, 3])
    assert hq.status(codes[0].ws)[0] == 0
    for x, code, beta, seed in zip(xs, codes, [0.3, 0.28, 0.31], [1, 2, 3]):
        _same_code(code, hq.encode(x, 128, oracle.E8, beta, seed=seed))
    ys = hq.decode_batch(codes, dtype=torch.float32)
    for code, y in zip(codes, ys):
        assert torch.equal(y, hq.decode(code, dtype=torch.float32))


def test_largest_batch_with_more_items_than_blocks(hq):
    xs = [t_bf16(W.llama_weight(1024 + 64 * i, 1024, seed=40 + i)) for i in range(hq.BATCH_MAX)]
    codes = hq.encode_batch(xs, 128, oracle.E8, [0.29] * len(xs), list(range(len(xs))))
    assert hq.status(codes[0].ws)[0] == 0
    for i in (0, 7, len(xs) - 1):
        _same_code(codes[i], hq.encode(xs[i], 128, oracle.E8, 0.29, seed=i))
    ys = hq.decode_batch(codes)
    for i in (0, 9, len(xs) - 1):
        assert torch.equal(ys[i], hq.decode(codes[i]))


def test_batch_refuses_mixed_tiles_and_lattices(hq):
    import ctypes
    L = hq.lib()
    xs = [t_bf16(W.llama_weight(128, 256, seed=1)), t_bf16(W.llama_weight(128, 256, seed=2))]
    codes = [hq.alloc_code(128, 256, hq.params(128, oracle.E8, 0.3)) for _ in xs]
    structs = [c.struct() for c in codes]
    items = (hq.EncodeItem * 2)()
    for i, x in enumerate(xs):
        items[i].x = x.data_ptr()
        items[i].dtype = hq.BF16
        items[i].rows, items[i].cols = 128, 256
        items[i].p = hq.params(128 if i == 0 else 64, oracle.E8, 0.3)
        items[i].out = ctypes.pointer(structs[i])
    ws = hq.Workspace(1 << 20)
    assert L.hq_encode_batch(2, items, ws.ptr(), ws.nbytes, None) == 2     # HQ_ERR_UNSUPPORTED
    items[1].p = hq.params(128, oracle.D4, 0.3)
    assert L.hq_encode_batch(2, items, ws.ptr(), ws.nbytes, None) == 2
    items[1].p = hq.params(128, oracle.E8, 0.3)
    assert L.hq_encode_batch(2, items, ws.ptr(), 64, None) == 1            # workspace too small
    assert L.hq_encode_batch(0, items, ws.ptr(), ws.nbytes, None) == 1
    code = hq.encode(xs[0], 128, oracle.E8, 0.3)
    other = hq.encode(xs[1], 128, oracle.D4, 0.3)
    with pytest.raises(hq.HQError) as e:
        hq.decode_batch([code, other])
    assert e.value.code == 2


@pytest.mark.parametrize("lattice", [oracle.D4, oracle.E8])
def test_kv_encode_batch_equals_single_appends(hq, lattice):
    shapes = [(2, 4, 1, 128), (2, 4, 3, 128), (1, 8, 1, 128), (3, 2, 2, 128)]
    s0s = [0, 5, 17, 1000]
    kvs = [torch.from_numpy(W.kv_keys(*sh[:3], 128, seed=30 + i).view(np.int16)).view(torch.bfloat16).cuda()
           .reshape(sh) for i, sh in enumerate(shapes)]
    steps = [1.1, 1.2, 0.9, 1.05]
    seeds = [7, 8, 9, 10]
    codes = hq.kv_encode_batch(kvs, s0s, steps, seeds, lattice=lattice)
    assert hq.status(codes[0].ws)[0] == 0
    for kv, code, s0, beta, seed in zip(kvs, codes, s0s, steps, seeds):
        ref = hq.kv_encode(kv, step=beta, seed=seed, lattice=lattice, s0=s0)
        assert hq.status(ref.ws)[0] == 0
        assert (code.kv_S, code.kv_s0) == (ref.kv_S, ref.kv_s0)
        _same_code(code, ref)


def test_kv_encode_batch_fp32_and_refusals(hq):
    import ctypes
    rng = np.random.default_rng(5)
    kvs = [torch.from_numpy(rng.standard_normal((2, 2, 4, 128)).astype(np.float32)).cuda() for _ in range(3)]
    codes = hq.kv_encode_batch(kvs, [0, 4, 8], [1.1] * 3, [1, 2, 3])
    for kv, code, s0, seed in zip(kvs, codes, [0, 4, 8], [1, 2, 3]):
        _same_code(code, hq.kv_encode(kv, step=1.1, seed=seed, s0=s0))
    # head dimension other than 128: not provided in a batch
    kv64 = torch.from_numpy(rng.standard_normal((2, 2, 4, 64)).astype(np.float32)).cuda()
    with pytest.raises(hq.HQError) as e:
        hq.kv_encode_batch([kv64, kv64], [0, 0], [1.1, 1.1], [1, 1])
    assert e.value.code == 2
