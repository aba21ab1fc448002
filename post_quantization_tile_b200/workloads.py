"""Seeded synthetic inputs for the codec workloads.

This module only draws random numbers and rounds them to bfloat16; it holds none of the codec's
arithmetic, so both the CUDA path and the CPU oracle may take their inputs from it.

The shapes and distributions stand in for the evaluation assets of the HyperQuant pages
(Llama-3.1-8B weights and KV cache, the LTX-2-19B DiT; "Experimental Results"), which are not
available: heavy-tailed weights with a few outlier input channels, Gaussian keys with per-head
outlier dimensions, Gaussian values.
"""
from __future__ import annotations

import numpy as np
import torch


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even (torch's conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_columns(rng: np.random.Generator, cols: int, count: int) -> np.ndarray:
    return rng.choice(cols, size=count, replace=False)


def tiny_weight(seed: int = 0) -> np.ndarray:
    """fp32 256x256, N(0, 0.02^2), 4 input columns scaled x20."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.02, size=(256, 256)).astype(np.float32)
    w[:, outlier_columns(rng, 256, 4)] *= 20.0
    return w


def student_t_weight(rows: int, cols: int, nu: float, std: float, outlier_frac: float, outlier_mult: float,
                     seed: int) -> np.ndarray:
    """bf16 bits [rows, cols]: Student-t(nu) scaled to the given std, a fraction of input columns
    multiplied by outlier_mult."""
    rng = np.random.default_rng(seed)
    scale = std / np.sqrt(nu / (nu - 2.0))
    w = (rng.standard_t(nu, size=(rows, cols)) * scale).astype(np.float32)
    m = max(1, int(round(outlier_frac * cols)))
    w[:, outlier_columns(rng, cols, m)] *= outlier_mult
    return to_bf16_bits(w)


def llama_weight(rows: int = 4096, cols: int = 4096, seed: int = 1) -> np.ndarray:
    """LLaMA-7B-shaped linear weight: t(5), std 0.02, 1% of input channels x20."""
    return student_t_weight(rows, cols, 5.0, 0.02, 0.01, 20.0, seed)


def llama_70b_weight(rows: int = 8192, cols: int = 28672, seed: int = 4) -> np.ndarray:
    """70B-shaped weight for the lattice sweep: t(4), std 0.015, 0.5% of input channels x30."""
    return student_t_weight(rows, cols, 4.0, 0.015, 0.005, 30.0, seed)


def dit_linear(rows: int, cols: int, seed: int) -> np.ndarray:
    """DiT-block linear: N(0, 0.02^2) with 1% of input channels x20."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.02, size=(rows, cols)).astype(np.float32)
    w[:, outlier_columns(rng, cols, max(1, cols // 100))] *= 20.0
    return to_bf16_bits(w)


DIT_BLOCK_SHAPES = [(4096, 4096)] * 4 + [(4096, 16384), (16384, 4096)]


def kv_keys(B: int = 8, H: int = 32, S: int = 8192, D: int = 128, seed: int = 2) -> np.ndarray:
    """bf16 bits [B, H, S, D]: N(0,1) with 4 outlier head dimensions per head scaled x10."""
    rng = np.random.default_rng(seed)
    k = rng.standard_normal(size=(B, H, S, D), dtype=np.float32)
    for h in range(H):
        k[:, h, :, outlier_columns(rng, D, 4)] *= 10.0
    return to_bf16_bits(k)


def kv_values(B: int = 8, H: int = 32, S: int = 8192, D: int = 128, seed: int = 2) -> np.ndarray:
    rng = np.random.default_rng(seed + 1000)
    return to_bf16_bits(rng.standard_normal(size=(B, H, S, D), dtype=np.float32))


def queries(count: int, D: int = 128, seed: int = 3) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal(size=(count, D)).astype(np.float64)


def gaussian_bf16(rows: int, cols: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.standard_normal(size=(rows, cols), dtype=np.float32))


def haar_rotation(n: int = 128, seed: int = 8) -> np.ndarray:
    """float32 [n, n] orthogonal matrix drawn from the Haar measure: the Q factor of a Gaussian
    matrix with the signs of R's diagonal moved into Q (Mezzadri's correction)."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((n, n))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return q.astype(np.float32)


def dit_linear_device(rows: int, cols: int, seed: int, device) -> torch.Tensor:
    """The DiT-block linear's distribution (N(0, 0.02^2), 1% of input channels x20) drawn on the
    device with torch's CUDA generator, for throughput runs over the whole 48-block stack where
    host generation of 9.66 G values would dominate; parity runs use dit_linear (host, numpy)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(0.02)
    cols_out = torch.randperm(cols, generator=g, device=device)[: max(1, cols // 100)]
    w[:, cols_out] *= 20.0
    return w.to(torch.bfloat16)
