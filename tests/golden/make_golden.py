"""Writes tests/golden/oracle_digests.json from the CPU oracle only.

The digests freeze the oracle's bitstream format on small seeded workloads, so that any later
change to the oracle's arithmetic or layout shows up as a failing test and has to be justified.
Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from post_quantization_tile_b200 import workloads as W  # noqa: E402

CASES = [
    # name, input builder, n, lattice, beta, seed, kv, kv_S
    ("tiny_fp32_e8", lambda: W.tiny_weight(0), 64, oracle.E8, 0.27, 0, False, 0),
    ("llama_slice_e8", lambda: W.llama_weight(4096, 4096, 1)[:96, :512], 128, oracle.E8, 0.3, 1, False, 0),
    ("llama_slice_a2_n256", lambda: W.llama_weight(4096, 4096, 1)[:40, :512], 256, oracle.A2, 0.3, 4, False, 0),
    ("llama_slice_z", lambda: W.llama_weight(4096, 4096, 1)[:33, :256], 128, oracle.Z, 0.3, 4, False, 0),
    ("kv_d4_dither", lambda: W.kv_keys(1, 2, 48, 128, 2).reshape(-1, 128), 128, oracle.D4, 1.0, 2, True, 48),
    ("llama_slice_e8_weight_dither", lambda: W.llama_weight(4096, 4096, 1)[:40, :256], 128, oracle.E8, 0.3, 5, 2, 0),
]

# the dense-rotation KV variant: name, keys [B, H, S, 128], lattice, beta, seed, first token
DENSE_CASES = [
    ("kv_dense_d4", lambda: W.kv_keys(1, 2, 48, 128, 3), oracle.D4, 1.1, 9, 0),
    ("kv_dense_e8_append", lambda: W.kv_keys(2, 2, 5, 128, 4), oracle.E8, 0.7, 11, 300),
]


def sha(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def digest(case):
    name, build, n, lat, beta, seed, kv, kv_S = case
    code = oracle.encode(build(), n, lat, beta, seed, kv, kv_S)
    return {
        "n": n, "lattice": lat, "beta": beta, "seed": seed, "kv": kv, "kv_S": kv_S,
        "status": code.status,
        "total_words": code.total_words,
        "payload_bits": code.payload_bits(),
        "bits_sha256": sha(code.bits),
        "scale_sha256": sha(code.scale),
        "meta_sha256": sha(code.meta),
        "chunk_word_sha256": sha(code.chunk_word),
    }


def digest_dense(case):
    name, build, lat, beta, seed, s0 = case
    x = build()
    S = x.shape[2]
    code = oracle.encode_dense(x.reshape(-1, 128), W.haar_rotation(128, seed=8), lat, beta, seed, kv_S=S, kv_s0=s0)
    return {
        "lattice": lat, "beta": beta, "seed": seed, "kv_S": S, "kv_s0": s0, "rotation": "haar_rotation(128, seed=8)",
        "status": code.status,
        "total_words": code.total_words,
        "payload_bits": code.payload_bits(),
        "bits_sha256": sha(code.bits),
        "scale_sha256": sha(code.scale),
        "meta_sha256": sha(code.meta),
        "chunk_word_sha256": sha(code.chunk_word),
    }


def main():
    out = {name: digest(c) for c in CASES for name in [c[0]]}
    out.update({c[0]: digest_dense(c) for c in DENSE_CASES})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_digests.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
    print("wrote", path)


if __name__ == "__main__":
    main()
