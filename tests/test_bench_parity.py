"""bench.py's parity report against the oracle (the block it adds to its CPU-baseline leg), run on
CPU with the oracle's own codes standing in for the GPU's: no mismatching tile, identical
bitstreams, equal rates; then one planted difference in a copied Rice header is counted."""
import os
import sys
import types

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from post_quantization_tile_b200 import workloads as W  # noqa: E402


def _as_gpu_code(ref):
    c = types.SimpleNamespace()
    c.scale = torch.from_numpy(ref.scale.view(np.int16).copy())
    c.meta = torch.from_numpy(ref.meta.view(np.int16).copy())
    c.chunk_word = torch.from_numpy(ref.chunk_word.view(np.int32).copy())
    c.bits = torch.from_numpy(ref.bits.view(np.int32).copy())
    c.payload_bps = lambda: ref.payload_bits() / float(ref.rows * ref.cols)
    return c


def test_parity_report_on_identical_and_planted_codes():
    host = [W.llama_weight(4096, 4096, seed=1)[:64, :512].copy(), W.llama_weight(4096, 4096, seed=2)[:40, :256].copy()]
    betas = [0.29, 0.31]
    gbs, secs, elems, last = bench.oracle_sample(host, 10 ** 6, 1, betas=betas)
    assert elems == sum(h.size for h in host) and gbs > 0
    codes = [_as_gpu_code(ref) for ref, _ in last]
    mse = []
    for i, (ref, xo) in enumerate(last):
        xf = W.bf16_bits_to_f32(host[i]).astype(np.float64)
        mse.append(float(np.mean((xo - xf) ** 2) / np.mean(xf ** 2)))
    rep = bench.parity_vs_oracle(codes, host, mse, last)
    assert rep["tile_mismatches"] == [0, 0]
    assert rep["bitstream_identical"] == [True, True]
    assert rep["payload_bps_gpu"] == rep["payload_bps_oracle"]
    assert max(rep["nmse_rel_diff"]) < 1e-12
    assert rep["comparator_ok"] == [True, True] and rep["boundary_disagreements"] == [0, 0]
    codes[1].meta[5] ^= 1          # one Rice parameter changed
    codes[1].bits[3] ^= 1 << 7      # one bit flipped
    rep = bench.parity_vs_oracle(codes, host, mse, last)
    assert rep["tile_mismatches"] == [0, 1]
    assert rep["bitstream_identical"] == [True, False]
    assert rep["comparator_ok"][0] and not rep["comparator_ok"][1]
    assert rep["boundary_disagreements"][0] == 0
