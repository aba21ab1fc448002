"""Comparison of a device code with the oracle's code of the same input -- TEST INFRASTRUCTURE
ONLY (used by tests/, the smoke check and the benchmark's oracle leg; never by the product).

The codec's parity bar: lattice indices and Rice bitstreams are bit-exact; an index may differ
only for an input within 1e-6 of a Voronoi boundary (u units), and such disagreements are counted
and reported as a fraction of all lattice blocks (at most 1e-6).  The boundary margin of a
disagreeing block is the distance of its quantizer input z from the bisector of the two points,
|d(z, p_device) - d(z, p_oracle)| / (2 |p_device - p_oracle|), computed in binary64.

compare() takes the fast path when every array is identical.  Otherwise it parses both codes to
integer lattice codes with the oracle's parser, requires identical scales, identical codes in
every block that is not a near-boundary disagreement, and identical chunk words in every chunk
without such a block.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import A2, E8, LATTICE_DIM, Code, dither, parse

MARGIN = 1e-6
SQ3_2 = np.sqrt(3.0) / 2.0


@dataclass
class Report:
    blocks: int
    disagreements: int = 0
    worst_margin: float = 0.0
    tiles_differing: int = 0
    identical: bool = True
    failures: list = field(default_factory=list)

    @property
    def fraction(self) -> float:
        return self.disagreements / max(1, self.blocks)

    @property
    def ok(self) -> bool:
        return not self.failures and self.fraction <= 1e-6

    def as_dict(self) -> dict:
        return {"blocks": self.blocks, "boundary_disagreements": self.disagreements,
                "disagreement_fraction": self.fraction, "worst_margin": self.worst_margin,
                "bitstream_identical": self.identical, "ok": self.ok, "failures": self.failures[:5]}


def _points(lattice: int, v: np.ndarray) -> np.ndarray:
    """integer embedding -> point in u units (A2 in its true geometry)"""
    v = v.astype(np.float64)
    if lattice == E8:
        return v / 2.0
    if lattice == A2:
        return np.stack([v[..., 0] * 0.5, v[..., 1] * SQ3_2], axis=-1)
    return v


def _input_u(lattice: int, u: np.ndarray, U: np.ndarray | None) -> np.ndarray:
    """the quantizer's input of one block in u units (the dither, if any, added as the codec adds it)"""
    z = u.astype(np.float64)
    if U is None:
        return z
    if lattice == A2:
        # A2 adds its dither in (P, Q) = (2 u0, u1 K) coordinates
        z = z.reshape(-1, 2).copy()
        z[:, 0] += U.reshape(-1, 2)[:, 0] / 2.0
        z[:, 1] += U.reshape(-1, 2)[:, 1] * SQ3_2
        return z.reshape(-1)
    return z + U.astype(np.float64)


def _tile_dither(ref: Code, t: int) -> np.ndarray | None:
    if not ref.kv:
        return None
    jt, r = divmod(t, ref.rows)
    if ref.kv == 1 and ref.kv_S:
        r_glob = r + getattr(ref, "row0", 0)
        c1, s = divmod(r_glob, ref.kv_S)
        c = s + getattr(ref, "kv_s0", 0)
    else:
        c1, c = jt, r + getattr(ref, "row0", 0)
    return dither(ref.lattice, ref.seed, c1, c, ref.n)


def compare(scale, meta, chunk_word, bits, ref: Code) -> Report:
    """Device arrays (numpy, the bf16 scale bits, meta, chunk_word and at least the words the
    device wrote) against the oracle's code `ref`, which must carry its coefficients (encode with
    want_codes=True) when the fast path does not apply."""
    d = LATTICE_DIM[ref.lattice]
    blocks = ref.tiles * (ref.n // d)
    rep = Report(blocks=blocks)
    words = int(np.asarray(chunk_word)[-1])
    same = (np.array_equal(np.asarray(chunk_word, dtype=np.uint32), ref.chunk_word)
            and np.array_equal(np.asarray(meta, dtype=np.uint16), ref.meta)
            and (ref.scale is None or scale is None or np.array_equal(np.asarray(scale, dtype=np.uint16), ref.scale))
            and words == ref.total_words
            and np.array_equal(np.asarray(bits, dtype=np.uint32)[:words], ref.bits))
    if same:
        return rep
    rep.identical = False
    if scale is not None and ref.scale is not None and not np.array_equal(np.asarray(scale, dtype=np.uint16), ref.scale):
        rep.failures.append("tile scales differ")
        return rep
    if ref.v is None or ref.u is None:
        rep.failures.append("codes differ and the oracle code carries no coefficients")
        return rep
    dev = Code(ref.rows, ref.cols, ref.n, ref.lattice, ref.beta, ref.seed, ref.kv, ref.kv_S,
               ref.scale, np.ascontiguousarray(meta, dtype=np.uint16),
               np.ascontiguousarray(chunk_word, dtype=np.uint32),
               np.ascontiguousarray(np.asarray(bits, dtype=np.uint32)[:max(words, 1)]), 0)
    v_dev, st = parse(dev)
    if st != 0:
        rep.failures.append(f"the device code does not parse (status {st})")
        return rep
    v_ref = ref.v
    diff_blocks = np.any((v_dev != v_ref).reshape(ref.tiles, ref.n // d, d), axis=2)
    tiles = np.nonzero(np.any(diff_blocks, axis=1))[0]
    rep.tiles_differing = int(tiles.size)
    for t in tiles:
        U = _tile_dither(ref, int(t))
        z = _input_u(ref.lattice, ref.u[t], U).reshape(-1, d)
        pd = _points(ref.lattice, v_dev[t].reshape(-1, d))
        pr = _points(ref.lattice, v_ref[t].reshape(-1, d))
        for b in np.nonzero(diff_blocks[t])[0]:
            dd = float(np.sum((pd[b] - z[b]) ** 2))
            dr = float(np.sum((pr[b] - z[b]) ** 2))
            margin = abs(dd - dr) / (2.0 * float(np.linalg.norm(pd[b] - pr[b])))
            rep.worst_margin = max(rep.worst_margin, margin)
            if margin > MARGIN:
                rep.failures.append(f"tile {int(t)} block {int(b)}: codes differ {margin:.3g} from the boundary")
            else:
                rep.disagreements += 1
    # chunks without a near-boundary block must be word-identical
    RB = (ref.rows + 31) // 32
    NT = ref.cols // ref.n
    bad_chunks = {(int(t) // ref.rows) * RB + (int(t) % ref.rows) // 32 for t in tiles}
    cw_dev = np.asarray(chunk_word, dtype=np.int64)
    cw_ref = ref.chunk_word.astype(np.int64)
    bits = np.asarray(bits, dtype=np.uint32)
    for c in range(NT * RB):
        if c in bad_chunks:
            continue
        a = bits[cw_dev[c]:cw_dev[c + 1]]
        b = ref.bits[cw_ref[c]:cw_ref[c + 1]]
        if not np.array_equal(a, b):
            rep.failures.append(f"chunk {c} differs without a near-boundary block")
            break
    return rep

