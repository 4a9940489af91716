"""Python face of the fp64 CPU oracle for LCSA (test infrastructure).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package. It wraps the C++ routines of ``lcsa_oracle.cpp`` with
ctypes; it shares no code with the CUDA library and never calls it.

Parity unpinned against the pages: the RoPE frequency schedule and the
block-budget reading (the pages say only "factored 3D RoPE" and print the
topk_ratio formula); the pins fix the oracle to those readings.

Rows are numbered (batch, head, query block) with the query block fastest,
blocks are numbered (frame group, block row, block column), tokens inside a
block (frame, row, column), exactly as in the C++ file.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import numpy as np

from . import build as _build


class _Geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "heads", "head_dim", "q_frames", "kv_frames", "grid_h", "grid_w",
        "block_t", "block_h", "block_w", "local_range", "topk", "kv_frame_offset",
        "norm_scope", "threads")] + [("rms_eps", ctypes.c_double), ("softmax_scale", ctypes.c_double)]


_lib = None


def lib():
    """The oracle's shared library: the in-tree build, or the build named by
    LCSA_ORACLE_LIB (the mutation tests load copies of lcsa_oracle.cpp with a
    planted mistake this way and check that the pins catch each)."""
    global _lib
    if _lib is None:
        path = os.environ.get("LCSA_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        G = ctypes.POINTER(_Geom)
        L.ora_resolve_topk.argtypes = [ctypes.c_double] + [ctypes.c_int] * 5
        L.ora_resolve_topk.restype = ctypes.c_int
        L.ora_norm_rope.argtypes = [G, P, P, ctypes.c_int, P, ctypes.c_int64, P]
        L.ora_pool.argtypes = [G, P, P, ctypes.c_int, P]
        L.ora_window_sizes.argtypes = [G, P]
        L.ora_select.argtypes = [G, P, P, P, P, ctypes.c_int, P, P]
        L.ora_attention.argtypes = [G, P, P, P, P, P, P, P, ctypes.c_int, P, ctypes.c_int64, P, P]
        L.ora_hardware_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def hardware_threads() -> int:
    return int(lib().ora_hardware_threads())


def resolve_topk(sparse_ratio: float, grid_h: int, grid_w: int, block_t: int, block_h: int, block_w: int) -> int:
    """k in blocks from topk_ratio = sparse_ratio*768*1280/(H*W) (H = 16 grid_h)."""
    return int(lib().ora_resolve_topk(float(sparse_ratio), grid_h, grid_w, block_t, block_h, block_w))


@dataclasses.dataclass
class Geometry:
    batch: int
    heads: int
    head_dim: int
    q_frames: int
    kv_frames: int
    grid_h: int
    grid_w: int
    block_t: int
    block_h: int
    block_w: int
    local_range: int
    topk: int
    kv_frame_offset: int = 0
    norm_scope: int = 0          # 0 token scope, 1 head scope
    threads: int = 0
    rms_eps: float = 1e-6
    softmax_scale: float = 0.0   # 0 -> 1/sqrt(head_dim)

    @classmethod
    def from_workload(cls, wl, **over) -> "Geometry":
        topk = wl.topk if wl.topk > 0 else resolve_topk(wl.sparse_ratio, wl.grid_h, wl.grid_w,
                                                        wl.block_t, wl.block_h, wl.block_w)
        g = cls(wl.batch, wl.heads, wl.head_dim, wl.q_frames, wl.kv_frames, wl.grid_h, wl.grid_w,
                wl.block_t, wl.block_h, wl.block_w, wl.local_range, topk, wl.kv_frame_offset)
        for k, v in over.items():
            setattr(g, k, v)
        return g

    # derived sizes
    @property
    def nb(self):
        return self.block_t * self.block_h * self.block_w

    @property
    def blocks_per_frame(self):
        return (self.grid_h // self.block_h) * (self.grid_w // self.block_w)

    @property
    def nQB(self):
        return (self.q_frames // self.block_t) * self.blocks_per_frame

    @property
    def nKB(self):
        return (self.kv_frames // self.block_t) * self.blocks_per_frame

    @property
    def Lq(self):
        return self.q_frames * self.grid_h * self.grid_w

    @property
    def Lkv(self):
        return self.kv_frames * self.grid_h * self.grid_w

    @property
    def C(self):
        return self.heads * self.head_dim

    @property
    def rows(self):
        return self.batch * self.heads * self.nQB

    def c_struct(self) -> _Geom:
        scale = self.softmax_scale if self.softmax_scale > 0 else 1.0 / math.sqrt(self.head_dim)
        return _Geom(self.batch, self.heads, self.head_dim, self.q_frames, self.kv_frames, self.grid_h,
                     self.grid_w, self.block_t, self.block_h, self.block_w, self.local_range, self.topk,
                     self.kv_frame_offset, self.norm_scope, self.threads, self.rms_eps, scale)


def norm_rope(g: Geometry, x: np.ndarray, gamma: np.ndarray, is_q: bool, tokens) -> np.ndarray:
    """fp64 normalised + rotated [ntok, heads*d] vectors; tokens are b*L + raster index."""
    tok = np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.empty((tok.size, g.C), dtype=np.float64)
    gs = g.c_struct()
    lib().ora_norm_rope(ctypes.byref(gs), _p(np.ascontiguousarray(x)), _p(np.ascontiguousarray(gamma, np.float32)),
                        int(is_q), _p(tok), tok.size, _p(out))
    return out


def pool(g: Geometry, x: np.ndarray, gamma: np.ndarray, is_q: bool) -> np.ndarray:
    """Block means [B, heads, nblocks, d] of the normalised, rotated vectors."""
    nblk = g.nQB if is_q else g.nKB
    out = np.empty((g.batch, g.heads, nblk, g.head_dim), dtype=np.float64)
    gs = g.c_struct()
    lib().ora_pool(ctypes.byref(gs), _p(np.ascontiguousarray(x)), _p(np.ascontiguousarray(gamma, np.float32)),
                   int(is_q), _p(out))
    return out


def window_sizes(g: Geometry) -> np.ndarray:
    out = np.empty(g.nQB, dtype=np.int32)
    gs = g.c_struct()
    lib().ora_window_sizes(ctypes.byref(gs), _p(out))
    return out


@dataclasses.dataclass
class Selection:
    row_len: np.ndarray   # [rows] int32
    cols: np.ndarray      # [rows, cap] int32 (entries past row_len unspecified)
    gap: np.ndarray       # [rows] float64, +inf when the whole window is kept
    scores: np.ndarray | None

    def row(self, r: int) -> np.ndarray:
        return self.cols[r, : self.row_len[r]]

    def csr(self):
        row_ptr = np.zeros(self.row_len.size + 1, dtype=np.int64)
        np.cumsum(self.row_len, out=row_ptr[1:])
        col = np.concatenate([self.row(r) for r in range(self.row_len.size)]) if self.row_len.size else \
            np.zeros(0, np.int32)
        return row_ptr, col.astype(np.int32)


def select(g: Geometry, pq: np.ndarray, pk: np.ndarray, want_scores: bool = False) -> Selection:
    rows = g.rows
    cap = max(1, min(g.topk, g.nKB))
    row_len = np.empty(rows, dtype=np.int32)
    cols = np.full((rows, cap), -1, dtype=np.int32)
    gap = np.empty(rows, dtype=np.float64)
    scores = np.empty((rows, g.nKB), dtype=np.float64) if want_scores else None
    gs = g.c_struct()
    lib().ora_select(ctypes.byref(gs), _p(np.ascontiguousarray(pq)), _p(np.ascontiguousarray(pk)), _p(row_len),
                     _p(cols), cap, _p(gap), _p(scores) if scores is not None else None)
    return Selection(row_len, cols, gap, scores)


def kth_thresholds(g: Geometry, scores: np.ndarray) -> np.ndarray:
    """Per row, the score of its k-th best admissible block (-inf when the
    budget covers the whole window): the threshold a selecting call records
    for later reuse ("FlashVSR: From 17.2 FPS to 57.3 FPS at 768x1408",
    Remove the remaining control-plane tax: the mask-generation threshold of
    the previous steady chunk, reused per DiT block). scores: [rows, nKB]
    fp64 from select(want_scores=True), non-finite where not admissible."""
    th = np.full(scores.shape[0], -np.inf)
    for r in range(scores.shape[0]):
        adm = np.sort(scores[r][np.isfinite(scores[r])])[::-1]
        if g.topk < adm.size:
            th[r] = adm[g.topk - 1]
    return th


def threshold_select(g: Geometry, scores: np.ndarray, thresholds: np.ndarray) -> Selection:
    """Selection by a reused threshold (same pages and passage): per row every
    admissible block whose score is >= the row's threshold, ascending; a row
    where none reaches it keeps its best block (the lower index among equal
    scores). Rows may keep more or fewer than k blocks."""
    rows, nkb = scores.shape
    cols = np.full((rows, nkb), -1, dtype=np.int32)
    row_len = np.zeros(rows, dtype=np.int32)
    for r in range(rows):
        sc = scores[r]
        adm = np.isfinite(sc)
        keep = np.flatnonzero(adm & (sc >= thresholds[r]))
        if keep.size == 0:
            best = np.max(sc[adm])
            keep = np.flatnonzero(adm & (sc == best))[:1]
        row_len[r] = keep.size
        cols[r, : keep.size] = keep
    return Selection(row_len, cols, np.full(rows, np.inf), scores)


def attention(g: Geometry, q, k, v, gamma_q, gamma_k, sel: Selection, rows=None):
    """fp64 outputs [nrows, nb, d] and weight sums [nrows, nb] of the given rows."""
    if rows is None:
        rows = np.arange(g.rows, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, g.nb, g.head_dim), dtype=np.float64)
    wsum = np.empty((rows.size, g.nb), dtype=np.float64)
    gs = g.c_struct()
    lib().ora_attention(ctypes.byref(gs), _p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(k)),
                        _p(np.ascontiguousarray(v)), _p(np.ascontiguousarray(gamma_q, np.float32)),
                        _p(np.ascontiguousarray(gamma_k, np.float32)), _p(np.ascontiguousarray(sel.row_len)),
                        _p(np.ascontiguousarray(sel.cols)), sel.cols.shape[1], _p(rows), rows.size, _p(out), _p(wsum))
    return out, wsum


def run(g: Geometry, inp, rows=None):
    """Whole oracle pass: pooled values, selection and the outputs of `rows`."""
    pq = pool(g, inp.q, inp.gamma_q, True)
    pk = pool(g, inp.k, inp.gamma_k, False)
    sel = select(g, pq, pk)
    out, wsum = attention(g, inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, sel, rows)
    return pq, pk, sel, out, wsum
