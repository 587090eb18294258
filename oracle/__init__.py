"""fp64 CPU oracle for NABLA block-mask building and block-masked softmax attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``block_sparse_attention_23_b200``) never does,
and this package imports nothing from it; the two share only the seeded input
generator in ``synth/``.

The arithmetic lives in ``nabla_oracle.c`` (plain fp64 loops, OpenMP across
rows, compiled with gcc -O2 and no fast-math); this module is argument
marshalling.  See that file's header for the passages each function follows and
for the readings taken where the pages are silent.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, hand-computed cases, library routines, invariants).  The overall
reading of the selection rule itself has no printed worked example on the
pages; that residual is recorded as "parity unpinned" for the rule's reading,
not for its arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nabla_oracle.c")
_LIB = os.path.join(_HERE, "libnabla_oracle.so")
_lock = threading.Lock()
_lib = None
BLOCK = 64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_pool.restype = None
            lib.oracle_pool.argtypes = [vp, i64, i64, i32, vp]
            lib.oracle_logits.restype = None
            lib.oracle_logits.argtypes = [vp, vp, i32, i32, vp]
            lib.oracle_softmax_row.restype = None
            lib.oracle_softmax_row.argtypes = [vp, i32, vp]
            lib.oracle_row_select.restype = i32
            lib.oracle_row_select.argtypes = [vp, i32, f64, vp, vp]
            lib.oracle_sta_or.restype = None
            lib.oracle_sta_or.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32]
            lib.oracle_build_mask.restype = None
            lib.oracle_build_mask.argtypes = [vp, vp, i64, i64, i32, i32, i32, i32, f64, i32,
                                              i32, i32, i32, i32, vp, vp, vp]
            lib.oracle_row_select_topk.restype = i32
            lib.oracle_row_select_topk.argtypes = [vp, i32, i32, vp, vp]
            lib.oracle_masked_attention.restype = None
            lib.oracle_masked_attention.argtypes = [vp, vp, vp, i64, i64, i32, vp, f64, i64, vp,
                                                    vp, vp]
            lib.oracle_dense_attention.restype = None
            lib.oracle_dense_attention.argtypes = [vp, vp, vp, i64, i64, i32, f64, i64, vp, vp, vp]
            lib.oracle_reorder.restype = None
            lib.oracle_reorder.argtypes = [vp, vp, i64, i32, i32, i32, i32, i32]
            lib.oracle_block_energy.restype = None
            lib.oracle_block_energy.argtypes = [vp, vp, vp, i64, i64, i32, vp, f64, i64, vp, vp,
                                                vp]
            lib.oracle_calib_accumulate.restype = None
            lib.oracle_calib_accumulate.argtypes = [vp, i64, i32, f64, vp]
            lib.oracle_calib_finalize.restype = None
            lib.oracle_calib_finalize.argtypes = [vp, i64, i32, vp]
            lib.oracle_attention_bwd.restype = None
            lib.oracle_attention_bwd.argtypes = [vp, vp, vp, vp, i64, i64, i32, vp, f64, i64, vp,
                                                 vp, i64, vp, vp, vp]
            lib.oracle_xattn_scores.restype = None
            lib.oracle_xattn_scores.argtypes = [vp, vp, i64, i64, i32, i32, i64, vp, vp]
            lib.oracle_max_threads.restype = i32
            lib.oracle_max_threads.argtypes = []
            _lib = lib
    return _lib


def _u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return a


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def pool(x: np.ndarray) -> np.ndarray:
    """[..., S, d] bf16 bits -> [..., S/64, d] fp64 block means."""
    x = _u16(x)
    S, d = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    out = np.empty(x.shape[:-2] + (S // BLOCK, d), dtype=np.float64)
    _load().oracle_pool(x.ctypes.data, BH, S, d, out.ctypes.data)
    return out


def logits(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """One head's reduced map qbar kbar^T / sqrt(d) (fp64)."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    nb, d = qbar.shape
    out = np.empty((nb, kbar.shape[0]), dtype=np.float64)
    if kbar.shape[0] != nb:
        raise ValueError("square reduced map expected")
    _load().oracle_logits(qbar.ctypes.data, kbar.ctypes.data, nb, d, out.ctypes.data)
    return out


def softmax_row(L: np.ndarray) -> np.ndarray:
    L = np.ascontiguousarray(L, dtype=np.float64)
    out = np.empty_like(L)
    _load().oracle_softmax_row(L.ctypes.data, L.shape[0], out.ctypes.data)
    return out


def row_select(p: np.ndarray, thr: float):
    """CDF binarisation of one probability row -> (keep uint8[n], count, diag[4])."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    keep = np.empty(p.shape[0], dtype=np.uint8)
    diag = np.empty(4, dtype=np.float64)
    cnt = _load().oracle_row_select(p.ctypes.data, p.shape[0], float(thr), keep.ctypes.data,
                                    diag.ctypes.data)
    return keep, int(cnt), diag


def row_select_topk(p: np.ndarray, k: int):
    """Fixed top-k selection of one probability row -> (keep uint8[n], count)."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    keep = np.empty(p.shape[0], dtype=np.uint8)
    cnt = _load().oracle_row_select_topk(p.ctypes.data, p.shape[0], int(k), keep.ctypes.data, None)
    return keep, int(cnt)


def sta_row(r: int, tile_grid, window) -> np.ndarray:
    """The clipped sliding-tile window of query tile r, as a uint8 row."""
    Tt, Th, Tw = tile_grid
    row = np.zeros(Tt * Th * Tw, dtype=np.uint8)
    _load().oracle_sta_or(row.ctypes.data, r, Tt, Th, Tw, *window)
    return row


def build_mask(q: np.ndarray, k: np.ndarray, tile_grid, thr: float, sta=None,
               with_diag: bool = False, topk: int = 0):
    """q, k: [B,H,S,d] bf16 bits -> mask [B,H,nb,nb] uint8 (and diagnostics).
    topk > 0 uses the fixed top-k rule instead of the mass rule."""
    q, k = _u16(q), _u16(k)
    B, H, S, d = q.shape
    nb = S // BLOCK
    mask = np.empty((B, H, nb, nb), dtype=np.uint8)
    diag = np.empty((B, H, nb, 4), dtype=np.float64)
    counts = np.empty((B, H, nb), dtype=np.int32)
    use_sta = sta is not None
    wt, wh, ww = sta if use_sta else (0, 0, 0)
    Tt, Th, Tw = tile_grid
    _load().oracle_build_mask(q.ctypes.data, k.ctypes.data, B * H, S, d, Tt, Th, Tw, float(thr),
                              int(topk), 1 if use_sta else 0, wt, wh, ww, mask.ctypes.data,
                              diag.ctypes.data, counts.ctypes.data)
    if with_diag:
        return mask, diag, counts
    return mask


def masked_attention(q, k, v, mask, rows=None, scale=None):
    """Block-masked softmax attention in fp64 for the given global rows (bh*S + i).

    Returns (O [nrows, d] fp64, LSE [nrows] fp64).  rows=None means every row."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, H, S, d = q.shape
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    if rows is None:
        rows = np.arange(B * H * S, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.empty((rows.shape[0], d), dtype=np.float64)
    lse = np.empty(rows.shape[0], dtype=np.float64)
    _load().oracle_masked_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, B * H, S, d,
                                    mask.ctypes.data, float(scale), rows.shape[0], rows.ctypes.data,
                                    O.ctypes.data, lse.ctypes.data)
    return O, lse


def dense_attention(q, k, v, rows=None, scale=None):
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, H, S, d = q.shape
    if rows is None:
        rows = np.arange(B * H * S, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.empty((rows.shape[0], d), dtype=np.float64)
    lse = np.empty(rows.shape[0], dtype=np.float64)
    _load().oracle_dense_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, B * H, S, d,
                                   float(scale), rows.shape[0], rows.ctypes.data, O.ctypes.data,
                                   lse.ctypes.data)
    return O, lse


def reorder(x: np.ndarray, tile_grid, to_tile_major: bool = True) -> np.ndarray:
    """[..., S, d] 16-bit rows -> the same rows moved between raster (t,h,w)
    order and tile-major order (4x4x4 tiles)."""
    x = _u16(x)
    S, d = x.shape[-2], x.shape[-1]
    Tt, Th, Tw = tile_grid
    if S != 64 * Tt * Th * Tw:
        raise ValueError("S must equal 64*Tt*Th*Tw")
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    out = np.empty_like(x)
    _load().oracle_reorder(x.ctypes.data, out.ctypes.data, BH, Tt, Th, Tw, d,
                           1 if to_tile_major else 0)
    return out


def block_energy(q, k, lse, mask, scale=None, rows=None):
    """Per-block attention energy over the listed blocks (0 elsewhere) and its
    row sums.  lse: [B,H,S], any float dtype.  rows=None: returns
    ([B,H,nb,nb], [B,H,nb]); else rows = global block-row ids bh*nb + r and
    the result is ([len(rows), nb], [len(rows)])."""
    q, k = _u16(q), _u16(k)
    B, H, S, d = q.shape
    nb = S // BLOCK
    mask = np.ascontiguousarray(mask, dtype=np.uint8).reshape(B, H, nb, nb)
    lse = np.ascontiguousarray(lse, dtype=np.float64).reshape(B, H, S)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is None:
        n, rp = B * H * nb, None
        energy = np.empty((B, H, nb, nb), dtype=np.float64)
        mass = np.empty((B, H, nb), dtype=np.float64)
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n, rp = rows.shape[0], rows.ctypes.data
        energy = np.empty((n, nb), dtype=np.float64)
        mass = np.empty(n, dtype=np.float64)
    _load().oracle_block_energy(q.ctypes.data, k.ctypes.data, lse.ctypes.data, B * H, S, d,
                                mask.ctypes.data, float(scale), n, rp, energy.ctypes.data,
                                mass.ctypes.data)
    return energy, mass


def calib_accumulate(energy: np.ndarray, eps: float, votes: np.ndarray) -> np.ndarray:
    """votes += the minimal-prefix selection (thr = eps) of each normalised energy row."""
    energy = np.ascontiguousarray(energy, dtype=np.float64)
    if votes.dtype != np.int32 or not votes.flags.c_contiguous or votes.shape != energy.shape:
        raise ValueError("votes must be a C-contiguous int32 array shaped like energy")
    nb = energy.shape[-1]
    _load().oracle_calib_accumulate(energy.ctypes.data, energy.size // nb, nb, float(eps),
                                    votes.ctypes.data)
    return votes


def calib_finalize(votes: np.ndarray, min_votes: int = 1) -> np.ndarray:
    votes = np.ascontiguousarray(votes, dtype=np.int32)
    mask = np.empty(votes.shape, dtype=np.uint8)
    _load().oracle_calib_finalize(votes.ctypes.data, votes.size, int(min_votes), mask.ctypes.data)
    return mask


def attention_bwd(q, k, v, dO, mask, scale=None, qrows=None, krows=None):
    """Gradients of block-masked softmax attention in fp64.

    q, k, v, dO: [B,H,S,d] bf16 bits; mask [B,H,nb,nb].  qrows / krows: global
    row ids (bh*S + i) for dQ and for dK, dV; None = every row, an empty array
    = none.  Returns (dQ [nq,d], dK [nk,d], dV [nk,d]) fp64."""
    q, k, v, dO = _u16(q), _u16(k), _u16(v), _u16(dO)
    B, H, S, d = q.shape
    nb = S // BLOCK
    mask = np.ascontiguousarray(mask, dtype=np.uint8).reshape(B, H, nb, nb)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    def sel(rows):
        if rows is None:
            return B * H * S, None, None
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        return rows.shape[0], rows, rows.ctypes.data
    nq, qa, qp = sel(qrows)
    nk, ka, kp = sel(krows)
    dQ = np.empty((nq, d), dtype=np.float64)
    dK = np.empty((nk, d), dtype=np.float64)
    dV = np.empty((nk, d), dtype=np.float64)
    _load().oracle_attention_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, dO.ctypes.data,
                                 B * H, S, d, mask.ctypes.data, float(scale), nq, qp,
                                 dQ.ctypes.data, nk, kp, dK.ctypes.data, dV.ctypes.data)
    return dQ, dK, dV


def xattn_scores(q, k, stride: int = 8, rows=None):
    """XAttention antidiagonal block scores in fp64: [B,H,nb,nb] (rows=None)
    or [len(rows), nb] for global block-row ids bh*nb + r."""
    q, k = _u16(q), _u16(k)
    B, H, S, d = q.shape
    nb = S // BLOCK
    if BLOCK % stride:
        raise ValueError("stride must divide 64")
    if rows is None:
        n, rp = B * H * nb, None
        out = np.empty((B, H, nb, nb), dtype=np.float64)
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n, rp = rows.shape[0], rows.ctypes.data
        out = np.empty((n, nb), dtype=np.float64)
    _load().oracle_xattn_scores(q.ctypes.data, k.ctypes.data, B * H, S, d, int(stride), n, rp,
                                out.ctypes.data)
    return out


def select_rows(weights, tile_grid, thr: float, sta=None, topk: int = 0, with_diag=False):
    """The builder's selection (a4-a6) on given block weights [B,H,nb,nb]: each
    row normalised by its sum, then the mass rule at thr (or top-k), STA OR."""
    weights = np.asarray(weights, dtype=np.float64)
    B, H, nb, _ = weights.shape
    Tt, Th, Tw = tile_grid
    mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
    diag = np.zeros((B, H, nb, 4), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r in range(nb):
                w = np.clip(weights[b, h, r], 0.0, None)
                z = w.sum()
                if z <= 0:
                    keep = np.zeros(nb, dtype=np.uint8)
                    dg = np.array([-1.0, -1.0, -1.0, -1.0])
                elif topk > 0:
                    keep, _ = row_select_topk(w / z, topk)
                    dg = np.array([-1.0, -1.0, -1.0, -1.0])
                else:
                    keep, _, dg = row_select(w / z, thr)
                if sta is not None:
                    keep = keep | sta_row(r, tile_grid, sta)
                mask[b, h, r] = keep
                diag[b, h, r] = dg
    return (mask, diag) if with_diag else mask


def near_cut_rows(diag: np.ndarray, thr: float, band: float = 1e-4) -> np.ndarray:
    """Boolean [.., nb] array: rows whose cut falls within `band` of 1 - thr
    (E_{k*} or E_{k*+1} within the band).  thr <= 0 has no cut."""
    if thr <= 0.0:
        return np.zeros(diag.shape[:-1], dtype=bool)
    t = 1.0 - thr
    return (np.abs(diag[..., 0] - t) < band) | (np.abs(diag[..., 1] - t) < band)


def near_tie_rows(diag: np.ndarray, rel: float = 1e-6) -> np.ndarray:
    """Rows whose probabilities at the cut (sorted positions k*, k*+1) differ by
    less than `rel` relative: a swap of those two blocks is within rounding."""
    a, b = diag[..., 2], diag[..., 3]
    return (b >= 0) & (np.abs(a - b) <= rel * np.maximum(np.abs(a), 1e-300))
