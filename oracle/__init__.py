"""fp64 CPU oracle for the HGA per-segment attention step (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  The product package never imports this module; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` do.  The arithmetic lives in ``hga_oracle.c`` (plain C, double
precision, sums in the written order); this file only marshals numpy arrays.

Definitions follow the HGA article ("Low-VRAM Long-Context Fine-Tuning:
Hierarchical Global Attention and Segmented Backpropagation in Practice",
sections Background / Deep analysis; fr edition, Contexte and Analyse
approfondie) with the readings stated in ``hga_oracle.c``.

Parity pins (tests/test_oracle_pins.py): every function here is checked
against something other than itself -- closed forms, hand-worked fixtures in
``tests/golden/``, brute-force subset enumeration, torch's float64
scaled-dot-product attention and autograd, and central finite differences.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

_LIB = None


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "Hq", "Hkv", "d", "blk", "S", "nblk", "topk", "qblk")]


@dataclass(frozen=True)
class Dims:
    B: int
    Hq: int
    Hkv: int
    d: int
    blk: int
    S: int
    nblk: int
    topk: int
    qblk: int = 0  # query-block size; 0 = blk (history blocks and query blocks of one size)

    @property
    def qb(self) -> int:
        return self.qblk or self.blk

    @property
    def nqb(self) -> int:
        return self.S // self.qb

    def c(self) -> _Dims:
        return _Dims(self.B, self.Hq, self.Hkv, self.d, self.blk, self.S, self.nblk, self.topk, self.qblk)


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        D = ctypes.POINTER(_Dims)
        I = ctypes.c_int
        lib.ohga_block_summaries.argtypes = [D, P, P]
        lib.ohga_query_means.argtypes = [D, P, P]
        lib.ohga_block_scores.argtypes = [D, P, P, P]
        lib.ohga_select_topk.argtypes = [D, P, P]
        lib.ohga_attn_fwd.argtypes = [D, P, P, P, P, P, P, I, I, P, P, P]
        lib.ohga_attn_bwd.argtypes = [D, P, P, P, P, P, P, P, I, I, P, P, P]
        lib.ohga_dense_causal_fwd.argtypes = [I, I, I, I, I, P, P, P, P, P]
        lib.ohga_decode_select.argtypes = [D, I, P, P, P, P]
        lib.ohga_attn_bwd_sparse.argtypes = [D, P, P, P, P, P, P, P, P, ctypes.c_double, I, I, P, P, P]
        lib.ohga_set_threads.argtypes = [I]
        lib.ohga_max_threads.restype = I
        lib.ohga_decode_attn.argtypes = [D, I, I, P, P, P, P, P, P, P, P]
        _LIB = lib
    return _LIB


def set_threads(n: int) -> None:
    """Host threads of the oracle's parallel loops (results do not depend on it)."""
    _lib().ohga_set_threads(int(n))


def max_threads() -> int:
    return int(_lib().ohga_max_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(a: np.ndarray, shape, name):
    if tuple(a.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(a.shape)}")


def block_summaries(D: Dims, k_hist) -> np.ndarray:
    k_hist = _f64(k_hist)
    _check(k_hist, (D.B, D.nblk * D.blk, D.Hkv, D.d), "k_hist")
    out = np.zeros((D.B, D.Hkv, D.nblk, D.d))
    _lib().ohga_block_summaries(ctypes.byref(D.c()), _ptr(k_hist), _ptr(out))
    return out


def query_means(D: Dims, q) -> np.ndarray:
    q = _f64(q)
    _check(q, (D.B, D.S, D.Hq, D.d), "q")
    out = np.zeros((D.B, D.Hq, D.nqb, D.d))
    _lib().ohga_query_means(ctypes.byref(D.c()), _ptr(q), _ptr(out))
    return out


def block_scores(D: Dims, qm, summ) -> np.ndarray:
    qm, summ = _f64(qm), _f64(summ)
    _check(qm, (D.B, D.Hq, D.nqb, D.d), "qm")
    _check(summ, (D.B, D.Hkv, D.nblk, D.d), "summ")
    out = np.zeros((D.B, D.Hkv, D.nqb, D.nblk))
    _lib().ohga_block_scores(ctypes.byref(D.c()), _ptr(qm), _ptr(summ), _ptr(out))
    return out


def select_topk(D: Dims, score) -> np.ndarray:
    score = _f64(score)
    _check(score, (D.B, D.Hkv, D.nqb, D.nblk), "score")
    out = np.zeros((D.B, D.Hkv, D.nqb, D.topk), dtype=np.int32)
    _lib().ohga_select_topk(ctypes.byref(D.c()), _ptr(score), _ptr(out))
    return out


def select(D: Dims, q, k_hist):
    """summaries -> query means -> scores -> top-K.  Returns (idx, score)."""
    summ = block_summaries(D, k_hist)
    score = block_scores(D, query_means(D, q), summ)
    return select_topk(D, score), score


def _attn_inputs(D: Dims, q, k_seg, v_seg, k_hist, v_hist, idx):
    q, k_seg, v_seg, k_hist, v_hist = map(_f64, (q, k_seg, v_seg, k_hist, v_hist))
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    _check(q, (D.B, D.S, D.Hq, D.d), "q")
    _check(k_seg, (D.B, D.S, D.Hkv, D.d), "k_seg")
    _check(v_seg, (D.B, D.S, D.Hkv, D.d), "v_seg")
    nb = k_hist.shape[1] // D.blk if k_hist.ndim == 4 else 0
    _check(k_hist, (D.B, nb * D.blk, D.Hkv, D.d), "k_hist")
    _check(v_hist, k_hist.shape, "v_hist")
    _check(idx, (D.B, D.Hkv, D.nqb, D.topk), "idx")
    if idx.size and (idx.max() >= nb or idx.min() < -1):
        raise ValueError("idx out of range")
    # the C code indexes history with nblk rows of blocks
    Dc = Dims(D.B, D.Hq, D.Hkv, D.d, D.blk, D.S, nb, D.topk, D.qblk)
    return Dc, q, k_seg, v_seg, k_hist, v_hist, idx


def attn_fwd(D: Dims, q, k_seg, v_seg, k_hist, v_hist, idx, kv_heads=None, rows=None):
    """O [B,S,Hq,d] and LSE [B,Hq,S] for KV heads in range(kv_heads) (default
    all) and segment positions ``rows`` (default all).  Entries not computed
    are left as NaN."""
    Dc, q, k_seg, v_seg, k_hist, v_hist, idx = _attn_inputs(D, q, k_seg, v_seg, k_hist, v_hist, idx)
    h0, h1 = (0, D.Hkv) if kv_heads is None else (kv_heads.start, kv_heads.stop)
    mask = None
    if rows is not None:
        mask = np.zeros(D.S, dtype=np.int8)
        mask[np.asarray(rows)] = 1
    o = np.full((D.B, D.S, D.Hq, D.d), np.nan)
    lse = np.full((D.B, D.Hq, D.S), np.nan)
    _lib().ohga_attn_fwd(ctypes.byref(Dc.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist), _ptr(v_hist),
                         _ptr(idx), h0, h1, None if mask is None else _ptr(mask), _ptr(o), _ptr(lse))
    return o, lse


def attn_bwd(D: Dims, q, k_seg, v_seg, k_hist, v_hist, idx, d_o, kv_heads=None):
    """dQ [B,S,Hq,d], dK_seg and dV_seg [B,S,Hkv,d] of L = <O, dO>; history gets
    no gradient.  Entries outside kv_heads are left as NaN."""
    Dc, q, k_seg, v_seg, k_hist, v_hist, idx = _attn_inputs(D, q, k_seg, v_seg, k_hist, v_hist, idx)
    d_o = _f64(d_o)
    _check(d_o, q.shape, "d_o")
    h0, h1 = (0, D.Hkv) if kv_heads is None else (kv_heads.start, kv_heads.stop)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k_seg.shape, np.nan)
    dv = np.full(v_seg.shape, np.nan)
    _lib().ohga_attn_bwd(ctypes.byref(Dc.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist), _ptr(v_hist),
                         _ptr(idx), _ptr(d_o), h0, h1, _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def attn_bwd_sparse(D: Dims, q, k_seg, v_seg, k_hist, v_hist, idx, d_o, qmask, scale: float, kv_heads=None):
    """SpaCO-style sparse backward: only query blocks with qmask[b, i] != 0
    propagate gradient, scaled by `scale` (qmask [B, S/qblk]).  Returns
    (dQ, dK_seg, dV_seg) like attn_bwd."""
    Dc, q, k_seg, v_seg, k_hist, v_hist, idx = _attn_inputs(D, q, k_seg, v_seg, k_hist, v_hist, idx)
    d_o = _f64(d_o)
    _check(d_o, q.shape, "d_o")
    qmask = np.ascontiguousarray(qmask, dtype=np.int8)
    _check(qmask, (D.B, D.nqb), "qmask")
    h0, h1 = (0, D.Hkv) if kv_heads is None else (kv_heads.start, kv_heads.stop)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k_seg.shape, np.nan)
    dv = np.full(v_seg.shape, np.nan)
    _lib().ohga_attn_bwd_sparse(ctypes.byref(Dc.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist), _ptr(v_hist),
                                _ptr(idx), _ptr(d_o), _ptr(qmask), float(scale), h0, h1, _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def dense_causal_fwd(q, k, v):
    """Textbook dense causal attention over a whole sequence: q [B,T,Hq,d],
    k/v [B,T,Hkv,d].  Returns (O, LSE[B,Hq,T])."""
    q, k, v = map(_f64, (q, k, v))
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, T))
    _lib().ohga_dense_causal_fwd(B, T, Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse))
    return o, lse


def decode_select(D: Dims, q_new, summ):
    """Decode-step selection: the nq = q_new.shape[1] new queries form one
    query group.  summ [B,Hkv,nblk,d] (oracle layout).  Returns (idx
    [B,Hkv,topk], score [B,Hkv,nblk])."""
    q_new, summ = _f64(q_new), _f64(summ)
    nq = q_new.shape[1]
    _check(q_new, (D.B, nq, D.Hq, D.d), "q_new")
    _check(summ, (D.B, D.Hkv, D.nblk, D.d), "summ")
    score = np.zeros((D.B, D.Hkv, D.nblk))
    idx = np.zeros((D.B, D.Hkv, D.topk), dtype=np.int32)
    _lib().ohga_decode_select(ctypes.byref(D.c()), nq, _ptr(q_new), _ptr(summ), _ptr(score), _ptr(idx))
    return idx, score


def decode_attn(D: Dims, t0: int, q_new, k_seg, v_seg, k_hist, v_hist, idx):
    """Decode-step attention: new query u (segment position t0+u) over the
    selected history blocks idx [B,Hkv,topk] and segment tokens 0..t0+u.
    k_seg/v_seg [B,S,Hkv,d] with S = D.S (the segment buffer's capacity).
    Returns (O [B,nq,Hq,d], LSE [B,Hq,nq])."""
    q_new, k_seg, v_seg, k_hist, v_hist = map(_f64, (q_new, k_seg, v_seg, k_hist, v_hist))
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    nq = q_new.shape[1]
    _check(q_new, (D.B, nq, D.Hq, D.d), "q_new")
    _check(k_seg, (D.B, D.S, D.Hkv, D.d), "k_seg")
    _check(v_seg, k_seg.shape, "v_seg")
    nb = k_hist.shape[1] // D.blk
    _check(k_hist, (D.B, nb * D.blk, D.Hkv, D.d), "k_hist")
    _check(v_hist, k_hist.shape, "v_hist")
    _check(idx, (D.B, D.Hkv, D.topk), "idx")
    if not (0 <= t0 and t0 + nq <= D.S):
        raise ValueError("new tokens outside the segment buffer")
    if idx.size and (idx.max() >= nb or idx.min() < -1):
        raise ValueError("idx out of range")
    Dc = Dims(D.B, D.Hq, D.Hkv, D.d, D.blk, D.S, nb, D.topk, D.qblk)
    o = np.zeros((D.B, nq, D.Hq, D.d))
    lse = np.zeros((D.B, D.Hq, nq))
    _lib().ohga_decode_attn(ctypes.byref(Dc.c()), nq, t0, _ptr(q_new), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist),
                            _ptr(v_hist), _ptr(idx), _ptr(o), _ptr(lse))
    return o, lse


def near_tie_positions(D: Dims, score, rel_tol: float = 1e-3):
    """Boolean [B,Hkv,nqb]: True where the K-th and (K+1)-th best oracle scores
    are closer than rel_tol, relative to max(|s_K|, |s_K+1|, 1e-6 * max|s|).
    At those positions a different but equally valid selection is accepted."""
    score = np.asarray(score, dtype=np.float64)
    keff = min(D.topk, D.nblk)
    out = np.zeros(score.shape[:3], dtype=bool)
    if keff >= D.nblk:
        return out
    srt = -np.sort(-score, axis=-1)
    sk, sk1 = srt[..., keff - 1], srt[..., keff]
    floor = 1e-6 * np.abs(score).max(axis=-1)
    den = np.maximum(np.maximum(np.abs(sk), np.abs(sk1)), floor)
    return (sk - sk1) / np.where(den > 0, den, 1.0) < rel_tol
