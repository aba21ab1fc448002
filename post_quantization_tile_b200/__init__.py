"""HyperQuant tile codec for NVIDIA B200 (sm_100a): Python binding over the C-ABI library.

Every step of the codec runs in the CUDA kernels of ``libhq.so`` (built in-tree by
``post_quantization_tile_b200.build``).  This module only marshals torch device tensors, the
current CUDA stream and the parameter structs into the C calls declared in ``include/hq.h``.
There is no CPU fallback: without the library or a CUDA device every call raises.
"""
from __future__ import annotations

import ctypes
import os
import struct
from dataclasses import dataclass

import torch

Z, A2, D4, E8 = 0, 1, 2, 3
LATTICES = {"Z": Z, "A2": A2, "D4": D4, "E8": E8}
BF16, F32 = 0, 1

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "capacity", 4: "non-finite input",
          5: "corrupt stream", 6: "timeout", 7: "range", 8: "CUDA error"}

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")


class HQError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [("tile", ctypes.c_int32), ("lattice", ctypes.c_int32), ("step", ctypes.c_float),
                ("bps", ctypes.c_float), ("seed", ctypes.c_uint64)]


class CodeStruct(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("kv_S", ctypes.c_int64), ("p", Params),
                ("kv", ctypes.c_int32), ("version", ctypes.c_int32), ("scale", ctypes.c_void_p),
                ("meta", ctypes.c_void_p), ("chunk_word", ctypes.c_void_p), ("bits", ctypes.c_void_p),
                ("cap_words", ctypes.c_int64), ("kv_s0", ctypes.c_int64)]


class EncodeItem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("p", Params), ("out", ctypes.POINTER(CodeStruct))]


class DecodeItem(ctypes.Structure):
    _fields_ = [("code", ctypes.POINTER(CodeStruct)), ("y", ctypes.c_void_p), ("dtype", ctypes.c_int32)]


class KvItem(ctypes.Structure):
    _fields_ = [("kv", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("B", ctypes.c_int64), ("H", ctypes.c_int64),
                ("S", ctypes.c_int64), ("D", ctypes.c_int64), ("s0", ctypes.c_int64), ("p", Params),
                ("out", ctypes.POINTER(CodeStruct))]


BATCH_MAX = 16

_lib = None


def lib():
    """Load libhq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m post_quantization_tile_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.hq_num_tiles.argtypes = [i64, i64, i32]
        L.hq_num_tiles.restype = i64
        L.hq_num_chunks.argtypes = [i64, i64, i32]
        L.hq_num_chunks.restype = i64
        L.hq_encode_bound_words.argtypes = [i64, i64, ctypes.POINTER(Params)]
        L.hq_encode_bound_words.restype = i64
        L.hq_workspace_bytes.argtypes = [i64, i64, ctypes.POINTER(Params)]
        L.hq_workspace_bytes.restype = ctypes.c_size_t
        L.hq_step_for_rate.argtypes = [i32, i32, ctypes.c_float]
        L.hq_step_for_rate.restype = ctypes.c_float
        L.hq_encode.argtypes = [P, i32, i64, i64, ctypes.POINTER(Params), ctypes.POINTER(CodeStruct), P,
                                ctypes.c_size_t, P]
        L.hq_encode_dither.argtypes = [P, i32, i64, i64, ctypes.POINTER(Params), ctypes.POINTER(CodeStruct), P,
                                       ctypes.c_size_t, P]
        L.hq_decode.argtypes = [ctypes.POINTER(CodeStruct), P, i32, P, ctypes.c_size_t, P]
        L.hq_kv_encode.argtypes = [P, i32, i64, i64, i64, i64, ctypes.POINTER(Params), ctypes.POINTER(CodeStruct), P,
                                   ctypes.c_size_t, P]
        L.hq_kv_decode.argtypes = [ctypes.POINTER(CodeStruct), P, i32, P, ctypes.c_size_t, P]
        L.hq_kv_encode_at.argtypes = [P, i32, i64, i64, i64, i64, i64, ctypes.POINTER(Params),
                                      ctypes.POINTER(CodeStruct), P, ctypes.c_size_t, P]
        L.hq_quantize_coeffs.argtypes = [P, i64, ctypes.POINTER(Params), i32, i64, P, ctypes.POINTER(CodeStruct), P,
                                         ctypes.c_size_t, P]
        L.hq_encode_count.argtypes = [P, i32, i64, i64, ctypes.POINTER(Params), i32, i64, P, P, ctypes.c_size_t, P]
        L.hq_decode_int8.argtypes = [ctypes.POINTER(CodeStruct), P, P, P, ctypes.c_size_t, P]
        L.hq_gemm_int8.argtypes = [P, P, i64, P, P, i64, i64, i32, P, P, ctypes.c_size_t, P]
        L.hq_gemm_code.argtypes = [P, P, i64, ctypes.POINTER(CodeStruct), P, P, ctypes.c_size_t, P]
        L.hq_encode_batch_workspace_bytes.argtypes = [i32, ctypes.POINTER(EncodeItem)]
        L.hq_encode_batch_workspace_bytes.restype = ctypes.c_size_t
        L.hq_encode_batch.argtypes = [i32, ctypes.POINTER(EncodeItem), P, ctypes.c_size_t, P]
        L.hq_decode_batch.argtypes = [i32, ctypes.POINTER(DecodeItem), P, ctypes.c_size_t, P]
        L.hq_kv_encode_batch_workspace_bytes.argtypes = [i32, ctypes.POINTER(KvItem)]
        L.hq_kv_encode_batch_workspace_bytes.restype = ctypes.c_size_t
        L.hq_kv_encode_batch.argtypes = [i32, ctypes.POINTER(KvItem), P, ctypes.c_size_t, P]
        L.hq_gemm_code_workspace_bytes.argtypes = [i64, i64, i64]
        L.hq_gemm_code_workspace_bytes.restype = ctypes.c_size_t
        L.hq_step_search.argtypes = [P, i32, i64, i64, ctypes.POINTER(Params), i32, i64, i32, ctypes.c_float, P, P,
                                     ctypes.c_size_t, P]
        L.hq_kv_dense_workspace_bytes.argtypes = [i64]
        L.hq_kv_dense_workspace_bytes.restype = ctypes.c_size_t
        L.hq_kv_encode_dense.argtypes = [P, i32, i64, i64, i64, i64, i64, P, ctypes.POINTER(Params),
                                         ctypes.POINTER(CodeStruct), P, ctypes.c_size_t, P]
        L.hq_kv_decode_dense.argtypes = [ctypes.POINTER(CodeStruct), P, P, i32, P, ctypes.c_size_t, P]
        L.hq_status_read.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
        L.hq_status_str.argtypes = [i32]
        L.hq_status_str.restype = ctypes.c_char_p
        L.hq_version.restype = i32
        for f in ["hq_encode", "hq_encode_dither", "hq_decode", "hq_kv_encode", "hq_kv_encode_at", "hq_kv_decode", "hq_quantize_coeffs",
                  "hq_encode_count", "hq_step_search", "hq_decode_int8", "hq_gemm_int8", "hq_gemm_code", "hq_status_read",
                  "hq_encode_batch", "hq_decode_batch", "hq_kv_encode_batch",
                  "hq_kv_encode_dense", "hq_kv_decode_dense"]:
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _check(code: int, where: str):
    if code != 0:
        raise HQError(code, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError("dense tensors must be bfloat16 or float32")


def _require_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def params(tile: int = 128, lattice: int | str = E8, step: float = 0.0, bps: float = 4.0, seed: int = 0) -> Params:
    if isinstance(lattice, str):
        lattice = LATTICES[lattice]
    return Params(int(tile), int(lattice), float(step), float(bps), int(seed) & ((1 << 64) - 1))


class Workspace:
    """Device scratch for one call at a time (status word, work counter, look-back states)."""

    def __init__(self, nbytes: int, device=None):
        self.nbytes = max(256, (int(nbytes) + 255) // 256 * 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


_ws_cache: dict = {}


def workspace(nbytes: int) -> Workspace:
    dev = torch.cuda.current_device()
    ws = _ws_cache.get(dev)
    if ws is None or ws.nbytes < nbytes:
        ws = Workspace(max(nbytes, 1 << 20), device=f"cuda:{dev}")
        _ws_cache[dev] = ws
    return ws


@dataclass
class Code:
    """An encoded tensor: device arrays plus the header the decoder needs."""
    rows: int
    cols: int
    p: Params
    kv: int
    kv_S: int
    scale: torch.Tensor       # uint16 view of bf16 per-tile RMS  [T]   (stored as int16)
    meta: torch.Tensor        # [T]  k | (sum q << 4)              (stored as int16)
    chunk_word: torch.Tensor  # [C+1] word offsets                 (stored as int32)
    bits: torch.Tensor        # [cap] bitstream words              (stored as int32)

    def struct(self) -> CodeStruct:
        return CodeStruct(self.rows, self.cols, self.kv_S, self.p, self.kv, lib().hq_version(),
                          self.scale.data_ptr(), self.meta.data_ptr(), self.chunk_word.data_ptr(),
                          self.bits.data_ptr(), self.bits.numel(), getattr(self, "kv_s0", 0))

    @property
    def step(self) -> float:
        return float(self.p.step)

    def total_words(self) -> int:
        return int(self.chunk_word[-1].item()) & 0xFFFFFFFF

    def payload_bits(self) -> int:
        m = self.meta.to(torch.int64) & 0xFFFF
        k = m & 15
        sq = m >> 4
        cos = self.p.tile // 8 if self.p.lattice == E8 else 0
        return int((cos + self.p.tile * (k + 1) + sq).sum().item())

    def payload_bps(self) -> float:
        return self.payload_bits() / float(self.rows * self.cols)

    def total_bps(self) -> float:
        C = self.chunk_word.numel() - 1
        T = self.scale.numel()
        return 8.0 * (4 * self.total_words() + 4 * T + 4 * (C + 1)) / float(self.rows * self.cols)


def alloc_code(rows: int, cols: int, p: Params, device=None, cap_words: int | None = None) -> Code:
    L = lib()
    T = L.hq_num_tiles(rows, cols, p.tile)
    C = L.hq_num_chunks(rows, cols, p.tile)
    if T < 0:
        raise HQError(1, "alloc_code")
    bound = L.hq_encode_bound_words(rows, cols, ctypes.byref(p))
    cap = bound if cap_words is None else int(cap_words)
    dev = device or "cuda"
    return Code(rows, cols, p, 0, 0,
                torch.zeros(T, dtype=torch.int16, device=dev), torch.zeros(T, dtype=torch.int16, device=dev),
                torch.zeros(C + 1, dtype=torch.int32, device=dev), torch.zeros(cap, dtype=torch.int32, device=dev))


def _fill(code: Code, cs: CodeStruct):
    code.rows, code.cols, code.kv_S, code.kv = cs.rows, cs.cols, cs.kv_S, cs.kv
    code.kv_s0 = cs.kv_s0
    code.p = Params(cs.p.tile, cs.p.lattice, cs.p.step, cs.p.bps, cs.p.seed)


def encode(x: torch.Tensor, tile: int = 128, lattice: int | str = E8, step: float = 0.0, bps: float = 4.0,
           seed: int = 0, out: Code | None = None, ws: Workspace | None = None, dither: bool = False) -> Code:
    """Encode a 2-D bf16/fp32 CUDA tensor (Methodology steps 1-3); dither=True adds the
    subtractive dither of each tile (the weight-path option of step 4)."""
    _require_cuda(x, "x")
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, cols]")
    p = params(tile, lattice, step, bps, seed)
    rows, cols = x.shape
    code = out if out is not None else alloc_code(rows, cols, p, device=x.device)
    L = lib()
    need = L.hq_workspace_bytes(rows, cols, ctypes.byref(p))
    w = ws or workspace(need)
    cs = code.struct()
    fn = L.hq_encode_dither if dither else L.hq_encode
    _check(fn(_ptr(x), _dtype_code(x), rows, cols, ctypes.byref(p), ctypes.byref(cs), w.ptr(), w.nbytes, _stream()),
           "hq_encode")
    _fill(code, cs)
    code.ws = w
    return code


def encode_batch(xs, tile: int = 128, lattice: int | str = E8, steps=None, seeds=None, outs=None,
                 ws: Workspace | None = None) -> list:
    """Encode several 2-D CUDA tensors of one dtype in one launch (hq_encode_batch): the same codes
    as one encode() per tensor.  steps and seeds give each tensor its step and seed."""
    n = len(xs)
    if not 1 <= n <= BATCH_MAX:
        raise ValueError(f"1 .. {BATCH_MAX} tensors per batch")
    steps = steps if steps is not None else [0.0] * n
    seeds = seeds if seeds is not None else [0] * n
    items = (EncodeItem * n)()
    codes, structs = [], []
    for i, x in enumerate(xs):
        _require_cuda(x, "x")
        if x.dim() != 2:
            raise ValueError("each tensor must be 2-D [rows, cols]")
        p = params(tile, lattice, steps[i], 4.0, seeds[i])
        rows, cols = x.shape
        code = outs[i] if outs is not None else alloc_code(rows, cols, p, device=x.device)
        cs = code.struct()
        codes.append(code)
        structs.append(cs)
        items[i].x = x.data_ptr()
        items[i].dtype = _dtype_code(x)
        items[i].rows, items[i].cols = rows, cols
        items[i].p = p
        items[i].out = ctypes.pointer(cs)
    L = lib()
    w = ws or workspace(L.hq_encode_batch_workspace_bytes(n, items))
    _check(L.hq_encode_batch(n, items, w.ptr(), w.nbytes, _stream()), "hq_encode_batch")
    for code, cs in zip(codes, structs):
        _fill(code, cs)
        code.ws = w
    return codes


def decode_batch(codes, dtype: torch.dtype = torch.bfloat16, outs=None, ws: Workspace | None = None) -> list:
    """Decode several weight codes (one tile size and lattice, no dither) in one launch
    (hq_decode_batch): the same tensors as one decode() per code."""
    n = len(codes)
    if not 1 <= n <= BATCH_MAX:
        raise ValueError(f"1 .. {BATCH_MAX} codes per batch")
    items = (DecodeItem * n)()
    ys, structs = [], []
    for i, code in enumerate(codes):
        y = outs[i] if outs is not None else torch.empty(code.rows, code.cols, dtype=dtype, device=code.bits.device)
        _require_cuda(y, "out")
        cs = code.struct()
        ys.append(y)
        structs.append(cs)
        items[i].code = ctypes.pointer(cs)
        items[i].y = y.data_ptr()
        items[i].dtype = _dtype_code(y)
    L = lib()
    w = ws or workspace(4096)
    _check(L.hq_decode_batch(n, items, w.ptr(), w.nbytes, _stream()), "hq_decode_batch")
    for code in codes:
        code.ws = w
    return ys


def decode(code: Code, dtype: torch.dtype = torch.bfloat16, out: torch.Tensor | None = None,
           ws: Workspace | None = None) -> torch.Tensor:
    """Decode to a [rows, cols] CUDA tensor (bf16 = binary32 result rounded to nearest even)."""
    y = out if out is not None else torch.empty(code.rows, code.cols, dtype=dtype, device=code.bits.device)
    _require_cuda(y, "out")
    L = lib()
    w = ws or workspace(4096)
    cs = code.struct()
    if code.kv == KV_DENSE:
        raise ValueError("a dense-rotation KV code decodes with kv_decode_dense and its rotation Q")
    fn = L.hq_kv_decode if code.kv == 1 else L.hq_decode
    _check(fn(ctypes.byref(cs), _ptr(y), _dtype_code(y), w.ptr(), w.nbytes, _stream()), "hq_decode")
    code.ws = w
    return y


def kv_encode(kv: torch.Tensor, step: float = 0.0, bps: float = 4.0, seed: int = 0, lattice: int | str = D4,
              out: Code | None = None, ws: Workspace | None = None, s0: int = 0) -> Code:
    """Encode a KV tensor [B, H, S, D] with the dither (Methodology step 4; D4 by default, any
    lattice).  s0 > 0: the tokens are positions s0 .. s0 + S - 1 of every sequence (token append)."""
    _require_cuda(kv, "kv")
    if kv.dim() != 4:
        raise ValueError("kv must be [B, H, S, D]")
    B, H, S, D = kv.shape
    p = params(D, lattice, step, bps, seed)
    rows = B * H * S
    code = out if out is not None else alloc_code(rows, D, p, device=kv.device)
    L = lib()
    w = ws or workspace(L.hq_workspace_bytes(rows, D, ctypes.byref(p)))
    cs = code.struct()
    if s0:
        _check(L.hq_kv_encode_at(_ptr(kv), _dtype_code(kv), B, H, S, D, int(s0), ctypes.byref(p), ctypes.byref(cs),
                                 w.ptr(), w.nbytes, _stream()), "hq_kv_encode_at")
    else:
        _check(L.hq_kv_encode(_ptr(kv), _dtype_code(kv), B, H, S, D, ctypes.byref(p), ctypes.byref(cs), w.ptr(),
                              w.nbytes, _stream()), "hq_kv_encode")
    _fill(code, cs)
    code.ws = w
    return code


def kv_encode_batch(kvs, s0s=None, steps=None, seeds=None, lattice: int | str = D4, outs=None,
                    ws: Workspace | None = None) -> list:
    """Encode several KV tensors [B, H, S, 128] of one dtype in one launch (hq_kv_encode_batch), item i
    as the tokens s0s[i] .. of every sequence: the same codes as one kv_encode(..., s0=s0s[i]) each."""
    n = len(kvs)
    if not 1 <= n <= BATCH_MAX:
        raise ValueError(f"1 .. {BATCH_MAX} tensors per batch")
    s0s = s0s if s0s is not None else [0] * n
    steps = steps if steps is not None else [0.0] * n
    seeds = seeds if seeds is not None else [0] * n
    items = (KvItem * n)()
    codes, structs = [], []
    for i, kv in enumerate(kvs):
        _require_cuda(kv, "kv")
        if kv.dim() != 4:
            raise ValueError("each kv must be [B, H, S, D]")
        B, H, S, D = kv.shape
        p = params(D, lattice, steps[i], 4.0, seeds[i])
        code = outs[i] if outs is not None else alloc_code(B * H * S, D, p, device=kv.device)
        cs = code.struct()
        codes.append(code)
        structs.append(cs)
        items[i].kv = kv.data_ptr()
        items[i].dtype = _dtype_code(kv)
        items[i].B, items[i].H, items[i].S, items[i].D = B, H, S, D
        items[i].s0 = int(s0s[i])
        items[i].p = p
        items[i].out = ctypes.pointer(cs)
    L = lib()
    w = ws or workspace(L.hq_kv_encode_batch_workspace_bytes(n, items))
    _check(L.hq_kv_encode_batch(n, items, w.ptr(), w.nbytes, _stream()), "hq_kv_encode_batch")
    for code, cs in zip(codes, structs):
        _fill(code, cs)
        code.ws = w
    return codes


def kv_decode(code: Code, shape, dtype: torch.dtype = torch.bfloat16, out: torch.Tensor | None = None,
              ws: Workspace | None = None) -> torch.Tensor:
    y = decode(code, dtype=dtype, out=out, ws=ws)
    return y.view(*shape)


KV_DENSE = 3  # Code.kv of a dense-rotation KV code


def _check_rotation(Q: torch.Tensor, D: int):
    _require_cuda(Q, "Q")
    if Q.dtype != torch.float32 or tuple(Q.shape) != (D, D) or not Q.is_contiguous():
        raise ValueError(f"Q must be a contiguous float32 [{D}, {D}] CUDA tensor")


def kv_encode_dense(kv: torch.Tensor, Q: torch.Tensor, step: float = 0.0, bps: float = 4.0, seed: int = 0,
                    lattice: int | str = D4, s0: int = 0, out: Code | None = None,
                    ws: Workspace | None = None) -> Code:
    """Encode a KV tensor [B, H, S, 128] with a dense orthogonal rotation Q (fp32 [128, 128], y = Q x)
    in place of the RHT, then the codec's dither, lattice and Rice coding (the Haar-rotation variant
    of Methodology step 4).  s0: first token position of every sequence (token append)."""
    _require_cuda(kv, "kv")
    if kv.dim() != 4:
        raise ValueError("kv must be [B, H, S, D]")
    B, H, S, D = kv.shape
    _check_rotation(Q, D)
    p = params(D, lattice, step, bps, seed)
    rows = B * H * S
    code = out if out is not None else alloc_code(rows, D, p, device=kv.device)
    L = lib()
    w = ws or workspace(L.hq_kv_dense_workspace_bytes(rows))
    cs = code.struct()
    _check(L.hq_kv_encode_dense(_ptr(kv), _dtype_code(kv), B, H, S, D, int(s0), _ptr(Q), ctypes.byref(p),
                                ctypes.byref(cs), w.ptr(), w.nbytes, _stream()), "hq_kv_encode_dense")
    _fill(code, cs)
    code.ws = w
    return code


def kv_decode_dense(code: Code, Q: torch.Tensor, shape=None, dtype: torch.dtype = torch.bfloat16,
                    out: torch.Tensor | None = None, ws: Workspace | None = None) -> torch.Tensor:
    """Decode a dense-rotation KV code: x_hat = Q^T (lattice point - dither) (s_hat beta)."""
    _check_rotation(Q, code.cols)
    y = out if out is not None else torch.empty(code.rows, code.cols, dtype=dtype, device=code.bits.device)
    _require_cuda(y, "out")
    L = lib()
    w = ws or workspace(L.hq_kv_dense_workspace_bytes(code.rows))
    cs = code.struct()
    _check(L.hq_kv_decode_dense(ctypes.byref(cs), _ptr(Q), _ptr(y), _dtype_code(y), w.ptr(), w.nbytes, _stream()),
           "hq_kv_decode_dense")
    code.ws = w
    return y if shape is None else y.view(*shape)


def quantize_coeffs(u: torch.Tensor, tile: int, lattice: int | str, seed: int = 0, kv: bool = False, kv_S: int = 0,
                    ws: Workspace | None = None):
    """Lattice + strip + Rice on normalised fp32 coefficients u[tiles, tile]; returns (codes, Code)."""
    _require_cuda(u, "u")
    if u.dtype != torch.float32 or u.dim() != 2 or u.shape[1] != tile:
        raise ValueError("u must be float32 [tiles, tile]")
    p = params(tile, lattice, 1.0, 0.0, seed)
    tiles = u.shape[0]
    code = alloc_code(tiles, tile, p, device=u.device)
    v = torch.empty(tiles, tile, dtype=torch.int32, device=u.device)
    L = lib()
    w = ws or workspace(L.hq_workspace_bytes(tiles, tile, ctypes.byref(p)))
    cs = code.struct()
    _check(L.hq_quantize_coeffs(_ptr(u), tiles, ctypes.byref(p), int(kv), int(kv_S), _ptr(v), ctypes.byref(cs),
                                w.ptr(), w.nbytes, _stream()), "hq_quantize_coeffs")
    _fill(code, cs)
    code.ws = w
    return v, code


def encode_count(x: torch.Tensor, tile: int, lattice: int | str, step: float, seed: int = 0, kv: bool = False,
                 kv_S: int = 0, ws: Workspace | None = None) -> torch.Tensor:
    """Total payload bits of encoding x at this step, as a device int64 scalar (no bitstream)."""
    _require_cuda(x, "x")
    rows, cols = (x.shape[0] * x.shape[1] * x.shape[2], x.shape[3]) if x.dim() == 4 else x.shape
    p = params(tile, lattice, step, 0.0, seed)
    L = lib()
    w = ws or workspace(L.hq_workspace_bytes(rows, cols, ctypes.byref(p)))
    outb = torch.zeros(1, dtype=torch.int64, device=x.device)
    _check(L.hq_encode_count(_ptr(x), _dtype_code(x), rows, cols, ctypes.byref(p), int(kv), int(kv_S), _ptr(outb),
                             w.ptr(), w.nbytes, _stream()), "hq_encode_count")
    return outb


def decode_int8(code: Code, ws: Workspace | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """The code's integer lattice codes int8 [rows, cols] and tile scales fp32 [cols / n, rows]
    (hq_decode_int8), the operands of gemm_int8."""
    dev = code.bits.device
    v = torch.empty(code.rows, code.cols, dtype=torch.int8, device=dev)
    g = torch.empty(code.cols // code.p.tile, code.rows, dtype=torch.float32, device=dev)
    w = ws or workspace(4096)
    cs = code.struct()
    _check(lib().hq_decode_int8(ctypes.byref(cs), _ptr(v), _ptr(g), w.ptr(), w.nbytes, _stream()), "hq_decode_int8")
    code.ws = w
    return v, g


def gemm_int8(A: torch.Tensor, sa: torch.Tensor, V: torch.Tensor, g: torch.Tensor, out: torch.Tensor | None = None,
              ws: Workspace | None = None) -> torch.Tensor:
    """Y = sa * sum_t g[t] (A V^T restricted to group t) on the tensor cores (hq_gemm_int8)."""
    for t, name in ((A, "A"), (sa, "sa"), (V, "V"), (g, "g")):
        _require_cuda(t, name)
    M, K = A.shape
    N = V.shape[0]
    Y = out if out is not None else torch.empty(M, N, dtype=torch.float32, device=A.device)
    w = ws or workspace(4096)
    _check(lib().hq_gemm_int8(_ptr(A), _ptr(sa), M, _ptr(V), _ptr(g), N, K, 128, _ptr(Y), w.ptr(), w.nbytes,
                              _stream()), "hq_gemm_int8")
    return Y


def gemm_code(A: torch.Tensor, sa: torch.Tensor, code: Code, out: torch.Tensor | None = None,
              ws: Workspace | None = None) -> torch.Tensor:
    """The product of decode_int8 and gemm_int8 with the decode fused into the GEMM's producer
    warps (hq_gemm_code): Y [M, code.rows] fp32."""
    for t, name in ((A, "A"), (sa, "sa")):
        _require_cuda(t, name)
    M = A.shape[0]
    Y = out if out is not None else torch.empty(M, code.rows, dtype=torch.float32, device=A.device)
    L = lib()
    w = ws or workspace(L.hq_gemm_code_workspace_bytes(M, code.rows, code.cols))
    cs = code.struct()
    _check(L.hq_gemm_code(_ptr(A), _ptr(sa), M, ctypes.byref(cs), _ptr(Y), w.ptr(), w.nbytes, _stream()),
           "hq_gemm_code")
    code.ws = w
    return Y


def step_search(x: torch.Tensor, tile: int, lattice: int | str, target_bps: float, seed: int = 0, kv: bool = False,
                kv_S: int = 0, step0: float = 0.0, max_probes: int = 0, tol_bps: float = 0.0,
                ws: Workspace | None = None) -> tuple[float, int, int]:
    """Exact-rate mode on the device (hq_step_search): (step, probes, payload bits at step).
    x: 2-D [rows, cols] or KV [B, H, S, D]; reading the result synchronises the stream."""
    _require_cuda(x, "x")
    if x.dim() == 4:
        rows, cols = x.shape[0] * x.shape[1] * x.shape[2], x.shape[3]
        kv, kv_S = True, x.shape[2]
    else:
        rows, cols = x.shape
    p = params(tile, lattice, step0, target_bps, seed)
    L = lib()
    w = ws or workspace(L.hq_workspace_bytes(rows, cols, ctypes.byref(p)))
    res = torch.zeros(2, dtype=torch.int64, device=x.device)  # {float step, int32 probes}, uint64 bits
    _check(L.hq_step_search(_ptr(x), _dtype_code(x), rows, cols, ctypes.byref(p), int(kv), int(kv_S), int(max_probes),
                            float(tol_bps), _ptr(res), w.ptr(), w.nbytes, _stream()), "hq_step_search")
    r = res.cpu().tolist()
    step = struct.unpack("<f", struct.pack("<I", r[0] & 0xFFFFFFFF))[0]
    return step, int(r[0] >> 32), int(r[1])


def calibrate_step(x: torch.Tensor, tile: int, lattice: int | str, target_bps: float, seed: int = 0,
                   kv: bool = False, kv_S: int = 0) -> float:
    """A step whose payload rate is target_bps to 1e-4 bps where the rate allows it: the device
    step search with a tight tolerance (Methodology step 3)."""
    return step_search(x, tile, lattice, target_bps, seed, kv, kv_S, max_probes=64, tol_bps=1e-4)[0]


def status(ws: Workspace) -> tuple[int, int]:
    """Synchronise the current stream and read the device status word: (code, detail)."""
    d = ctypes.c_int64(0)
    code = lib().hq_status_read(ws.ptr(), _stream(), ctypes.byref(d))
    return int(code), int(d.value)
