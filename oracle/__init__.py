"""CPU oracle of the HyperQuant tile codec (test infrastructure only).

The oracle is a plain single-threaded C implementation (``hq_oracle.c``) of the codec described
in "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline for Large Language and Diffusion
Models" (gist.science, Technical Summary, "Methodology: The HyperQuant Pipeline").  This module
builds it with gcc and wraps it with ctypes over numpy arrays.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The product (``post_quantization_tile_b200``) never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

Z, A2, D4, E8 = 0, 1, 2, 3
LATTICE_DIM = {Z: 1, A2: 2, D4: 4, E8: 8}

ST_CAPACITY = 1 << 3
ST_NONFINITE = 1 << 4
ST_CORRUPT = 1 << 5

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle: -O2, binary32 without excess precision, no FMA contraction."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-fexcess-precision=standard", "-Wall", "-Wno-unused-function", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, u64, i32, f32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_float
        L.hqo_philox4x32_10.argtypes = [P, ctypes.c_uint32, ctypes.c_uint32, P]
        L.hqo_sign_negative.argtypes = [u64, i64]
        L.hqo_sign_negative.restype = i32
        L.hqo_f32_to_bf16.argtypes = [f32]
        L.hqo_f32_to_bf16.restype = ctypes.c_uint16
        L.hqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.hqo_bf16_to_f32.restype = f32
        L.hqo_rms.argtypes = [P, i32]
        L.hqo_rms.restype = f32
        L.hqo_fwht_f32.argtypes = [P, i32]
        L.hqo_fwht_f64.argtypes = [P, i32]
        L.hqo_quantize_block.argtypes = [i32, P, P]
        L.hqo_quantize_blocks.argtypes = [i32, P, i64, P]
        L.hqo_strip_block.argtypes = [i32, P, P, P]
        L.hqo_unstrip_block.argtypes = [i32, P, i32, P]
        L.hqo_dither_d4.argtypes = [u64, i64, i64, i32, P]
        L.hqo_dither.argtypes = [i32, u64, i64, i64, i32, P]
        L.hqo_group_scale.argtypes = [ctypes.c_uint16, ctypes.c_float, i32, i32]
        L.hqo_group_scale.restype = ctypes.c_float
        L.hqo_decode_int8.argtypes = [P, P, P, P, i64, i64, i32, i32, ctypes.c_float, P, P]
        L.hqo_decode_int8.restype = ctypes.c_uint32
        L.hqo_gemm_grouped.argtypes = [P, P, i64, P, P, i64, i64, i32, P]
        L.hqo_gemm_grouped_sample.argtypes = [P, P, P, P, i64, i64, i32, P, P, i64, P]
        L.hqo_rice_tile.argtypes = [P, i32, i32, P, i64, P, P]
        L.hqo_rice_tile.restype = i64
        L.hqo_parse_tile.argtypes = [P, i64, i32, i32, ctypes.c_uint16, P, P]
        L.hqo_parse_tile.restype = i32
        L.hqo_encode.argtypes = [P, i32, i64, i64, i32, i32, f32, u64, i32, i64, P, P, P, P, i64, P, P, i64, i64]
        L.hqo_encode.restype = ctypes.c_uint32
        L.hqo_quantize_coeffs.argtypes = [P, i64, i32, i32, i32, i64, u64, P, P, P, P, i64]
        L.hqo_quantize_coeffs.restype = ctypes.c_uint32
        L.hqo_parse.argtypes = [P, P, P, i64, i64, i32, i32, P]
        L.hqo_parse.restype = ctypes.c_uint32
        L.hqo_decode.argtypes = [P, P, P, P, i64, i64, i32, i32, f32, u64, i32, i64, P, i64, i64]
        L.hqo_decode.restype = ctypes.c_uint32
        L.hqo_rotate_normalize.argtypes = [P, i32, i64, i32, P, f32, P, P]
        L.hqo_rotate_normalize.restype = ctypes.c_uint32
        L.hqo_encode_dense.argtypes = [P, i32, i64, i32, P, i32, f32, u64, i64, i64, i64, P, P, P, P, i64, P, P]
        L.hqo_encode_dense.restype = ctypes.c_uint32
        L.hqo_decode_coeffs.argtypes = [P, P, P, i64, i32, i32, u64, i64, i64, i64, P]
        L.hqo_decode_coeffs.restype = ctypes.c_uint32
        L.hqo_unrotate.argtypes = [P, P, i64, i32, P, f32, P]
        L.hqo_decode_dense.argtypes = [P, P, P, P, i64, i32, P, i32, f32, u64, i64, i64, i64, P]
        L.hqo_decode_dense.restype = ctypes.c_uint32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------------------------
# primitives
# ----------------------------------------------------------------------------------------------
def philox(ctr, key0: int, key1: int) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().hqo_philox4x32_10(_p(c), ctypes.c_uint32(key0), ctypes.c_uint32(key1), _p(out))
    return out


def signs(seed: int, cols: int) -> np.ndarray:
    """+1/-1 diagonal for transformed-axis indices 0..cols-1."""
    L = lib()
    return np.array([-1 if L.hqo_sign_negative(seed, j) else 1 for j in range(cols)], dtype=np.int8)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(x, dtype=np.float32).ravel()
    return np.array([L.hqo_f32_to_bf16(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(x))


def rms(x: np.ndarray) -> float:
    a = np.ascontiguousarray(x, dtype=np.float32)
    return float(lib().hqo_rms(_p(a), a.size))


def fwht_f32(x: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32).copy()
    lib().hqo_fwht_f32(_p(a), a.size)
    return a


def fwht_f64(x: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float64).copy()
    lib().hqo_fwht_f64(_p(a), a.size)
    return a


def quantize_blocks(lattice: int, u: np.ndarray) -> np.ndarray:
    """Nearest lattice point of each row of u[m, d] (integer embedding, see hq_oracle.c)."""
    d = LATTICE_DIM[lattice]
    u = np.ascontiguousarray(u, dtype=np.float32).reshape(-1, d)
    v = np.zeros(u.shape, dtype=np.int32)
    lib().hqo_quantize_blocks(lattice, _p(u), u.shape[0], _p(v))
    return v


def dither_d4(seed: int, bh: int, s: int, blk: int) -> np.ndarray:
    U = np.zeros(4, dtype=np.float32)
    lib().hqo_dither_d4(seed, bh, s, blk, _p(U))
    return U


def dither(lattice: int, seed: int, c1: int, c: int, n: int) -> np.ndarray:
    """The subtractive dither of one tile (float32 [n], quantizer coordinates: (P, Q) for A2)."""
    U = np.zeros(n, dtype=np.float32)
    lib().hqo_dither(lattice, seed, c1, c, n, _p(U))
    return U


def strip(lattice: int, v: np.ndarray):
    d = LATTICE_DIM[lattice]
    v = np.ascontiguousarray(v, dtype=np.int32).reshape(-1, d)
    sym = np.zeros_like(v)
    cos = np.zeros(v.shape[0], dtype=np.int32)
    L = lib()
    c = ctypes.c_int()
    for i in range(v.shape[0]):
        L.hqo_strip_block(lattice, _p(v[i]), _p(sym[i]), ctypes.byref(c))
        cos[i] = c.value
    return sym, cos


def unstrip(lattice: int, sym: np.ndarray, cos: np.ndarray) -> np.ndarray:
    d = LATTICE_DIM[lattice]
    sym = np.ascontiguousarray(sym, dtype=np.int32).reshape(-1, d)
    v = np.zeros_like(sym)
    L = lib()
    for i in range(sym.shape[0]):
        L.hqo_unstrip_block(lattice, _p(sym[i]), int(cos[i]), _p(v[i]))
    return v


def rice_tile(v: np.ndarray, lattice: int):
    """Rice-code one tile of integer codes; returns (words, bit length, k, sum q)."""
    v = np.ascontiguousarray(v, dtype=np.int32)
    n = v.size
    cap = (n // 8 + 17 * n) // 32 + 2
    words = np.zeros(cap, dtype=np.uint32)
    k, sq = ctypes.c_int(), ctypes.c_int()
    nbits = lib().hqo_rice_tile(_p(v), n, lattice, _p(words), cap, ctypes.byref(k), ctypes.byref(sq))
    return words, int(nbits), k.value, sq.value


def parse_tile(words: np.ndarray, n: int, lattice: int, meta: int):
    words = np.ascontiguousarray(words, dtype=np.uint32)
    v = np.zeros(n, dtype=np.int32)
    bl = ctypes.c_int64()
    ok = lib().hqo_parse_tile(_p(words), words.size, n, lattice, meta, _p(v), ctypes.byref(bl))
    return bool(ok), v, int(bl.value)


# ----------------------------------------------------------------------------------------------
# whole-tensor codec
# ----------------------------------------------------------------------------------------------
def bound_words(rows: int, cols: int, n: int) -> int:
    """Worst-case words (k <= 15, sum q < 2n per tile), plus one padding word per chunk."""
    T = rows * (cols // n)
    C = (cols // n) * ((rows + 31) // 32)
    return (T * (n // 8 + 16 * n + 2 * n) + 31) // 32 + C + 4


@dataclass
class Code:
    rows: int
    cols: int
    n: int
    lattice: int
    beta: float
    seed: int
    kv: int
    kv_S: int
    scale: np.ndarray       # uint16 [T], bf16 bits
    meta: np.ndarray        # uint16 [T]
    chunk_word: np.ndarray  # uint32 [C+1]
    bits: np.ndarray        # uint32 [total words]
    status: int
    v: np.ndarray | None = None   # int32 [T, n]
    u: np.ndarray | None = None   # float32 [T, n]

    @property
    def tiles(self) -> int:
        return self.rows * (self.cols // self.n)

    @property
    def total_words(self) -> int:
        return int(self.chunk_word[-1])

    def payload_bits(self) -> int:
        k = (self.meta & 15).astype(np.int64)
        sq = (self.meta >> 4).astype(np.int64)
        cos = self.n // 8 if self.lattice == E8 else 0
        return int(np.sum(cos + self.n * k + self.n + sq))


def encode(x: np.ndarray, n: int, lattice: int, beta: float, seed: int, kv: bool = False, kv_S: int = 0,
           want_codes: bool = False, row0: int = 0, kv_s0: int = 0) -> Code:
    """x: 2-D numpy array, dtype uint16 (bf16 bits) or float32.  row0: for KV, the global row of
    x's first row when x is a slice of a larger [B*H*S, D] tensor.  kv_s0: for KV, the position of
    x's first token in every sequence (tokens appended at s0 .. s0 + kv_S - 1)."""
    assert x.ndim == 2
    if x.dtype == np.uint16:
        dtype = 0
    elif x.dtype == np.float32:
        dtype = 1
    else:
        raise TypeError("x must be uint16 (bf16 bits) or float32")
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    T = rows * (cols // n)
    C = (cols // n) * ((rows + 31) // 32)
    cap = bound_words(rows, cols, n)
    scale = np.zeros(T, dtype=np.uint16)
    meta = np.zeros(T, dtype=np.uint16)
    cw = np.zeros(C + 1, dtype=np.uint32)
    bits = np.zeros(cap, dtype=np.uint32)
    v = np.zeros((T, n), dtype=np.int32) if want_codes else None
    u = np.zeros((T, n), dtype=np.float32) if want_codes else None
    st = lib().hqo_encode(_p(x), dtype, rows, cols, n, lattice, ctypes.c_float(beta), seed, int(kv), kv_S,
                          _p(scale), _p(meta), _p(cw), _p(bits), cap,
                          _p(v) if v is not None else None, _p(u) if u is not None else None, row0, kv_s0)
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    c = Code(rows, cols, n, lattice, float(np.float32(beta)), seed, int(kv), kv_S, scale, meta, cw,
             bits[: int(cw[-1])].copy(), int(st), v, u)
    c.row0 = row0
    c.kv_s0 = kv_s0
    return c


def quantize_coeffs(u: np.ndarray, n: int, lattice: int, seed: int = 0, kv: bool = False, kv_S: int = 0):
    """u: float32 [tiles, n] normalised coefficients.  Returns (v, meta, chunk_word, bits, status)."""
    u = np.ascontiguousarray(u, dtype=np.float32)
    tiles = u.shape[0]
    C = (tiles + 31) // 32
    cap = bound_words(tiles, n, n)
    v = np.zeros((tiles, n), dtype=np.int32)
    meta = np.zeros(tiles, dtype=np.uint16)
    cw = np.zeros(C + 1, dtype=np.uint32)
    bits = np.zeros(cap, dtype=np.uint32)
    st = lib().hqo_quantize_coeffs(_p(u), tiles, n, lattice, int(kv), kv_S, seed, _p(v), _p(meta), _p(cw),
                                   _p(bits), cap)
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    return v, meta, cw, bits[: int(cw[-1])].copy(), int(st)


def parse(code: Code) -> tuple[np.ndarray, int]:
    v = np.zeros((code.tiles, code.n), dtype=np.int32)
    bits = np.ascontiguousarray(code.bits, dtype=np.uint32)
    if bits.size == 0:
        bits = np.zeros(1, dtype=np.uint32)
    st = lib().hqo_parse(_p(code.meta), _p(code.chunk_word), _p(bits), code.rows, code.cols, code.n,
                         code.lattice, _p(v))
    return v, int(st)


def decode(code: Code) -> tuple[np.ndarray, int]:
    """Reconstruction in float64 [rows, cols] and status bits."""
    out = np.zeros((code.rows, code.cols), dtype=np.float64)
    bits = np.ascontiguousarray(code.bits, dtype=np.uint32)
    if bits.size == 0:
        bits = np.zeros(1, dtype=np.uint32)
    st = lib().hqo_decode(_p(code.scale), _p(code.meta), _p(code.chunk_word), _p(bits), code.rows, code.cols,
                          code.n, code.lattice, ctypes.c_float(code.beta), code.seed, code.kv, code.kv_S, _p(out),
                          getattr(code, "row0", 0), getattr(code, "kv_s0", 0))
    return out, int(st)


def payload_bps(code: Code) -> float:
    return code.payload_bits() / float(code.rows * code.cols)


def total_bps(code: Code) -> float:
    C = code.chunk_word.size - 1
    nbytes = 4 * code.total_words + 2 * code.tiles + 2 * code.tiles + 4 * (C + 1)
    return 8.0 * nbytes / float(code.rows * code.cols)


def calibrate_step(x: np.ndarray, n: int, lattice: int, target_bps: float, seed: int = 0, kv: bool = False,
                   kv_S: int = 0, iters: int = 40) -> float:
    """Bisection on log(beta) so the oracle's payload rate on x hits target_bps."""
    lo, hi = np.log(2.0 ** -8), np.log(2.0 ** 6)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        b = float(np.float32(np.exp(mid)))
        r = payload_bps(encode(x, n, lattice, b, seed, kv, kv_S))
        if r > target_bps:
            lo = mid
        else:
            hi = mid
    return float(np.float32(np.exp(0.5 * (lo + hi))))


STEP_BITS_MIN, STEP_BITS_MAX = 0x3B800000, 0x42800000  # binary32 bit patterns of 2^-8 and 64


def _f32_bits(x: float) -> int:
    return int(np.array([x], dtype=np.float32).view(np.int32)[0])


def _bits_f32(b: int) -> float:
    return float(np.array([b], dtype=np.int32).view(np.float32)[0])


def step_search(x: np.ndarray, n: int, lattice: int, target_bps: float, seed: int = 0, kv: bool = False,
                kv_S: int = 0, step0: float = 0.0, max_probes: int = 16, tol_bps: float = 0.005):
    """Exact-rate mode: the step whose payload rate on x is target_bps, within tol_bps (the
    method lands the realised rate about 0.01 bps from any target, Methodology step 3, Rice
    coding).  Written from the rule as stated, with every quantity in binary64:

    * probe 1 is step0;
    * after each probe (payload bits c): keep the probe closest to the target; stop if
      |c - target| <= tol_bps n (tol_bps as binary32, widened); else the probe becomes the low
      end of the bracket (rate too high, c > target) or the high end;
    * with both ends known: stop when they are adjacent binary32 values; else the next probe is
      the regula-falsi point lo + floor(t (hi - lo)), t = (c_lo - target) / (c_lo - c_hi), on the
      bit patterns, or the midpoint when the same end moved twice in a row, kept strictly inside;
    * with one end known: a Newton step of floor(excess 2^23 + 1/2) bit patterns (excess = bps
      above the target, slope -1 bit per doubling of the step), at least one, clamped to
      [2^-8, 64]; stop if it cannot move;
    * stop after max_probes probes.

    Returns (step, probes, payload bits at step)."""
    N = float(x.shape[0] * x.shape[1])
    target = float(np.float32(target_bps)) * N
    tol = float(np.float32(tol_bps)) * N
    b = _f32_bits(step0)
    lo = hi = -1
    c_lo = c_hi = 0
    last_side = 0
    probes = 0
    best, c_best = b, 0
    while True:
        c = encode(x, n, lattice, _bits_f32(b), seed, kv, kv_S).payload_bits()
        probes += 1
        err = abs(float(c) - target)
        if probes == 1 or err < abs(float(c_best) - target):
            best, c_best = b, c
        if err <= tol:
            break
        if float(c) > target:
            lo, c_lo, side = b, c, 1
        else:
            hi, c_hi, side = b, c, 2
        if lo >= 0 and hi >= 0:
            if hi - lo <= 1:
                break
            if side == last_side:
                nb = lo + (hi - lo) // 2
            else:
                t = (float(c_lo) - target) / (float(c_lo) - float(c_hi))
                nb = lo + int(np.floor(t * float(hi - lo)))
            nb = min(max(nb, lo + 1), hi - 1)
        else:
            excess = (float(c) - target) / N
            d = float(np.floor(excess * 8388608.0 + 0.5))
            d = min(max(d, -134217728.0), 134217728.0)
            nb = b + int(d)
            if nb == b:
                nb += 1 if side == 1 else -1
            nb = min(max(nb, STEP_BITS_MIN), STEP_BITS_MAX)
            if nb == b:
                break
        last_side = side
        if probes >= max_probes:
            break
        b = nb
    return _bits_f32(best), probes, c_best


ST_RANGE = 1 << 6


def decode_int8(code: Code):
    """The weight's integer codes as int8 [rows, cols] (RHT domain) and its group scales
    g[cols / n, rows] (binary32 ((s_hat beta) c_n) c_L); tiles with a code outside [-127, 127]
    come back as zeros with status bit ST_RANGE.  Returns (v8, g, status)."""
    v8 = np.zeros((code.rows, code.cols), dtype=np.int8)
    g = np.zeros((code.cols // code.n, code.rows), dtype=np.float32)
    bits = np.ascontiguousarray(code.bits, dtype=np.uint32)
    if bits.size == 0:
        bits = np.zeros(1, dtype=np.uint32)
    st = lib().hqo_decode_int8(_p(code.scale), _p(code.meta), _p(code.chunk_word), _p(bits), code.rows, code.cols,
                               code.n, code.lattice, ctypes.c_float(code.beta), _p(v8), _p(g))
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    return v8, g, int(st)


def gemm_grouped(A: np.ndarray, sa: np.ndarray, V: np.ndarray, g: np.ndarray, n: int) -> np.ndarray:
    """Y[m, r] = sa_m * sum_t g[t, r] S_{m,r,t} with exact int8 group sums S, binary32 fma over t."""
    A = np.ascontiguousarray(A, dtype=np.int8)
    V = np.ascontiguousarray(V, dtype=np.int8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32)
    M, K = A.shape
    N = V.shape[0]
    Y = np.zeros((M, N), dtype=np.float32)
    lib().hqo_gemm_grouped(_p(A), _p(sa), M, _p(V), _p(g), N, K, n, _p(Y))
    return Y


def gemm_grouped_sample(A, sa, V, g, n, idx_m, idx_r) -> np.ndarray:
    A = np.ascontiguousarray(A, dtype=np.int8)
    V = np.ascontiguousarray(V, dtype=np.int8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32)
    im = np.ascontiguousarray(idx_m, dtype=np.int64)
    ir = np.ascontiguousarray(idx_r, dtype=np.int64)
    out = np.zeros(im.size, dtype=np.float32)
    lib().hqo_gemm_grouped_sample(_p(A), _p(sa), _p(V), _p(g), V.shape[0], A.shape[1], n, _p(im), _p(ir), im.size,
                                  _p(out))
    return out


# ----------------------------------------------------------------------------------------------
# dense-rotation KV variant (a caller-given orthogonal Q in place of H_n D)
# ----------------------------------------------------------------------------------------------
KV_DENSE = 3   # Code.kv of a dense-rotation KV code (dither words of KV rows)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return 0
    if x.dtype == np.float32:
        return 1
    raise TypeError("x must be uint16 (bf16 bits) or float32")


def rotate_normalize(x: np.ndarray, Q: np.ndarray, beta: float):
    """u = (Q x) / (s_hat beta) per row in binary32 (fma chain in ascending i) and the bf16 RMS
    bits.  Returns (u float32 [rows, n], scale uint16 [rows], status)."""
    x = np.ascontiguousarray(x)
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    rows, n = x.shape
    u = np.zeros((rows, n), dtype=np.float32)
    scale = np.zeros(rows, dtype=np.uint16)
    st = lib().hqo_rotate_normalize(_p(x), _dtype_code(x), rows, n, _p(Q), ctypes.c_float(beta), _p(u), _p(scale))
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    return u, scale, int(st)


def encode_dense(x: np.ndarray, Q: np.ndarray, lattice: int, beta: float, seed: int, kv_S: int,
                 row0: int = 0, kv_s0: int = 0, want_codes: bool = False) -> Code:
    """Dense-rotation KV encode of x [rows, n] (head vectors of a [B, H, S, n] tensor with S = kv_S;
    row0 the global row of x's first row, kv_s0 the first token position)."""
    x = np.ascontiguousarray(x)
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    rows, n = x.shape
    C = (rows + 31) // 32
    cap = bound_words(rows, n, n)
    scale = np.zeros(rows, dtype=np.uint16)
    meta = np.zeros(rows, dtype=np.uint16)
    cw = np.zeros(C + 1, dtype=np.uint32)
    bits = np.zeros(cap, dtype=np.uint32)
    v = np.zeros((rows, n), dtype=np.int32) if want_codes else None
    u = np.zeros((rows, n), dtype=np.float32) if want_codes else None
    st = lib().hqo_encode_dense(_p(x), _dtype_code(x), rows, n, _p(Q), lattice, ctypes.c_float(beta), seed, kv_S,
                                row0, kv_s0, _p(scale), _p(meta), _p(cw), _p(bits), cap,
                                _p(v) if v is not None else None, _p(u) if u is not None else None)
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    c = Code(rows, n, n, lattice, float(np.float32(beta)), seed, KV_DENSE, kv_S, scale, meta, cw,
             bits[: int(cw[-1])].copy(), int(st), v, u)
    c.row0 = row0
    c.kv_s0 = kv_s0
    return c


def _bits_or_pad(code: Code) -> np.ndarray:
    bits = np.ascontiguousarray(code.bits, dtype=np.uint32)
    return bits if bits.size else np.zeros(1, dtype=np.uint32)


def decode_coeffs(code: Code) -> tuple[np.ndarray, int]:
    """Lattice points minus the KV dither, in u units, float64 [rows, n] (one tile column)."""
    p = np.zeros((code.rows, code.n), dtype=np.float64)
    st = lib().hqo_decode_coeffs(_p(code.meta), _p(code.chunk_word), _p(_bits_or_pad(code)), code.rows, code.n,
                                 code.lattice, code.seed, code.kv_S, getattr(code, "row0", 0),
                                 getattr(code, "kv_s0", 0), _p(p))
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    return p, int(st)


def unrotate(p: np.ndarray, scale: np.ndarray, Q: np.ndarray, beta: float) -> np.ndarray:
    """x_hat = Q^T p (s_hat beta) per row, float64."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    scale = np.ascontiguousarray(scale, dtype=np.uint16)
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    out = np.zeros_like(p)
    lib().hqo_unrotate(_p(p), _p(scale), p.shape[0], p.shape[1], _p(Q), ctypes.c_float(beta), _p(out))
    return out


def decode_dense(code: Code, Q: np.ndarray) -> tuple[np.ndarray, int]:
    """Dense-rotation KV decode to float64 [rows, n] and status bits."""
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    out = np.zeros((code.rows, code.n), dtype=np.float64)
    st = lib().hqo_decode_dense(_p(code.scale), _p(code.meta), _p(code.chunk_word), _p(_bits_or_pad(code)),
                                code.rows, code.n, _p(Q), code.lattice, ctypes.c_float(code.beta), code.seed,
                                code.kv_S, getattr(code, "row0", 0), getattr(code, "kv_s0", 0), _p(out))
    if st & 2:
        raise ValueError("oracle rejected the arguments")
    return out, int(st)
