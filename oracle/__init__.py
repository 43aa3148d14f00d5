"""ORACLE — test infrastructure only.

ctypes front end of ``oracle.c``: a plain double-precision CPU statement of
the biased, block-routed attention call over MiniMax-H3's packed sequence.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library (``biased_attention_video_b200``) and never imports it.

Every function cites the page passage it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SEG_TEXT, SEG_IMAGE_REF, SEG_AUDIO, SEG_GUIDE, SEG_OUTPUT = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.oracle_penalty.argtypes = [ctypes.c_double] * 5
        L.oracle_penalty.restype = ctypes.c_double
        L.oracle_k.argtypes = [ctypes.c_int, ctypes.c_double]
        L.oracle_k.restype = ctypes.c_int
        L.oracle_block_classes.argtypes = [ctypes.c_int, ctypes.c_int, _P, _P]
        L.oracle_block_classes.restype = ctypes.c_int
        L.oracle_pool.argtypes = [ctypes.c_int] * 4 + [_P, _P]
        L.oracle_pool.restype = None
        L.oracle_route.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [_P] * 6
        L.oracle_route.restype = ctypes.c_int
        attend_args = [ctypes.c_int] * 4 + [_P, _P, _P, _P, ctypes.c_int, _P, _P, _P,
                                            ctypes.c_int, _P, _P, _P, _P]
        L.oracle_attend.argtypes = attend_args
        L.oracle_attend.restype = None
        L.oracle_attend_partitions.argtypes = attend_args
        L.oracle_attend_partitions.restype = None
        L.oracle_merge.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_int, _P, _P, _P, _P, _P]
        L.oracle_merge.restype = None
        L.oracle_tail.argtypes = [ctypes.c_int] * 4 + [_P] * 5 + [ctypes.c_int, _P, _P]
        L.oracle_tail.restype = None
        L.oracle_threads.restype = ctypes.c_int
        L.oracle_quantize_rows.argtypes = [ctypes.c_long, ctypes.c_int, _P, _P, _P]
        L.oracle_quantize_rows.restype = None
        L.oracle_attend_qk8.argtypes = [ctypes.c_int] * 4 + [_P, _P, _P, _P, ctypes.c_int] + [_P] * 5 + \
            [ctypes.c_int, _P, _P, _P, _P]
        L.oracle_attend_qk8.restype = None
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    return int(lib().oracle_threads())


def penalty(dt: float, strength=2.0, window=0.20, falloff=0.25, cap=6.0) -> float:
    """penalty(dt) = min(strength * (max(dt - window, 0) / falloff)^2, cap)."""
    return float(lib().oracle_penalty(dt, strength, window, falloff, cap))


def k_for(n_video_blocks: int, sparsity: float) -> int:
    return int(lib().oracle_k(n_video_blocks, sparsity))


def block_classes(seg: np.ndarray, B: int = 64) -> np.ndarray:
    """uint8 [nKB]: 1 if the block holds any non-video row (forced key / dense query)."""
    seg = _c(seg, np.uint8)
    nkb = (len(seg) + B - 1) // B
    out = np.empty(nkb, np.uint8)
    lib().oracle_block_classes(len(seg), B, seg.ctypes.data, out.ctypes.data)
    return out


def pool(x_bf16: np.ndarray, B: int = 64) -> np.ndarray:
    """fp64 [H][nKB][d] block means of bf16 bits x [H][S][d]."""
    x = _c(x_bf16, np.uint16)
    H, S, d = x.shape
    nkb = (S + B - 1) // B
    out = np.empty((H, nkb, d), np.float64)
    lib().oracle_pool(H, S, d, B, x.ctypes.data, out.ctypes.data)
    return out


def route(q_bf16: np.ndarray, k_bf16: np.ndarray, seg: np.ndarray, sparsity: float, B: int = 64,
          want_scores: bool = False) -> Tuple[np.ndarray, Optional[np.ndarray], np.ndarray]:
    """Routing: (sel int32 [H][nV][k], scores fp64 [H][nV][nV] or None, kth fp64 [H][nV])."""
    q = _c(q_bf16, np.uint16)
    k = _c(k_bf16, np.uint16)
    seg = _c(seg, np.uint8)
    H, S, d = q.shape
    cls = block_classes(seg, B)
    nv = int((cls == 0).sum())
    if nv == 0:
        raise ValueError("no video block")
    kk = k_for(nv, sparsity)
    sel = np.empty((H, nv, kk), np.int32)
    kth = np.empty((H, nv), np.float64)
    scores = np.empty((H, nv, nv), np.float64) if want_scores else None
    got = lib().oracle_route(H, S, d, B, sparsity, seg.ctypes.data, q.ctypes.data, k.ctypes.data,
                             sel.ctypes.data, _ptr(scores), kth.ctypes.data)
    assert got == kk
    return sel, scores, kth


def _attend(fn, q, k, v, seg, times, pen, sel, heads, rows, B):
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    seg = _c(seg, np.uint8)
    times = _c(times, np.float32)
    H, S, d = q.shape
    heads = _c(heads, np.int32)
    rows = _c(rows, np.int32)
    n = len(rows)
    assert len(heads) == n
    pen_arr = None if pen is None else _c(pen, np.float64)
    if sel is not None:
        sel = _c(sel, np.int32)
        kk = sel.shape[-1]
    else:
        kk = 0
    o = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    fn(H, S, d, B, seg.ctypes.data, times.ctypes.data, _ptr(pen_arr), _ptr(sel), kk,
       q.ctypes.data, k.ctypes.data, v.ctypes.data, n, heads.ctypes.data, rows.ctypes.data,
       o.ctypes.data, lse.ctypes.data)
    return o, lse


def attend(q, k, v, seg, times, pen=None, sel=None, heads=None, rows=None, B: int = 64):
    """Direct definition for the given (head, row) pairs (all rows of all heads if None).

    Returns (O fp64 [n][d], LSE fp64 [n]).  pen = (strength, window, falloff, cap) or None;
    sel = routed lists [H][nV][k] or None (dense)."""
    H, S, _ = np.shape(q)
    if rows is None:
        heads = np.repeat(np.arange(H), S)
        rows = np.tile(np.arange(S), H)
    return _attend(lib().oracle_attend, q, k, v, seg, times, pen, sel, heads, rows, B)


def quantize_rows(x):
    """Per-token int8 quantisation ("H3 SLA Attention", inputs table, use_int8_qk) of bf16 bit patterns
    x [..., d]: per row s = max|x| / 127 and codes rint(x * (127 / max|x|)) clamped to +-127, in fp32 with
    ties to even; a zero row gets s = 0.  Returns (codes int8 [..., d], scales float32 [...])."""
    x = _c(x, np.uint16)
    d = x.shape[-1]
    n = x.size // d
    codes = np.empty(x.shape, np.int8)
    scales = np.empty(x.shape[:-1], np.float32)
    lib().oracle_quantize_rows(n, d, x.ctypes.data, codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def attend_qk8(q, k, v, seg, times, pen=None, sel=None, heads=None, rows=None, B: int = 64):
    """As attend, with Q and K quantised per token to int8 before the QK dot product (quantize_rows); the
    score is s_q s_k (integer dot of the codes) / sqrt(d); PV uses v as given."""
    q8, sq = quantize_rows(q)
    k8, sk = quantize_rows(k)
    v = _c(v, np.uint16)
    seg = _c(seg, np.uint8)
    times = _c(times, np.float32)
    H, S, d = v.shape
    if rows is None:
        heads = np.repeat(np.arange(H), S)
        rows = np.tile(np.arange(S), H)
    heads = _c(heads, np.int32)
    rows = _c(rows, np.int32)
    n = len(rows)
    pen_arr = None if pen is None else _c(pen, np.float64)
    sel_c = None if sel is None else _c(sel, np.int32)
    kk = 0 if sel is None else sel_c.shape[-1]
    o = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    lib().oracle_attend_qk8(H, S, d, B, seg.ctypes.data, times.ctypes.data, _ptr(pen_arr), _ptr(sel_c), kk,
                            q8.ctypes.data, sq.ctypes.data, k8.ctypes.data, sk.ctypes.data, v.ctypes.data, n,
                            heads.ctypes.data, rows.ctypes.data, o.ctypes.data, lse.ctypes.data)
    return o, lse


def attend_partitions(q, k, v, seg, times, pen=None, sel=None, heads=None, rows=None, B: int = 64):
    """Flash-Partitions evaluation of the same outputs (three contributions + LSE merge)."""
    H, S, _ = np.shape(q)
    if rows is None:
        heads = np.repeat(np.arange(H), S)
        rows = np.tile(np.arange(S), H)
    return _attend(lib().oracle_attend_partitions, q, k, v, seg, times, pen, sel, heads, rows, B)


def merge(o_parts, lse_parts, log_w=None):
    """Flash-Partitions merge of normalised partition results ("Flash Partitions for H3 native temporal
    alignment", section 4): o_parts [n][rows][d], lse_parts [n][rows] (natural log), log_w [n] or None
    (every multiplier 1).  Returns (O [rows][d], L [rows]) in fp64."""
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    l = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, rows, d = o.shape
    assert l.shape == (n, rows)
    lw = None if log_w is None else np.ascontiguousarray(log_w, dtype=np.float64)
    out = np.empty((rows, d), np.float64)
    out_l = np.empty(rows, np.float64)
    lib().oracle_merge(n, rows, d, o.ctypes.data, l.ctypes.data, _ptr(lw), out.ctypes.data, out_l.ctypes.data)
    return out, out_l


def tail(q, k, v, seg, sel, B: int = 64):
    """Pooled tail term per (head, video query block) ("H3 SLA Attention", inputs table, tail_correction):
    the routed-out video key blocks as one partition, each block counted as its valid rows at its pooled
    score with its mean value.  sel: routed lists [H][nV][k].  Returns (Lt [H][nV], Ot [H][nV][d]) fp64."""
    H, S, d = np.shape(q)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    nv, kk = sel.shape[1], sel.shape[2]
    lt = np.empty((H, nv), np.float64)
    ot = np.empty((H, nv, d), np.float64)
    seg_c, q_c, k_c, v_c = _c(seg, np.uint8), _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    lib().oracle_tail(H, S, d, B, seg_c.ctypes.data, q_c.ctypes.data, k_c.ctypes.data, v_c.ctypes.data,
                      sel.ctypes.data, kk, lt.ctypes.data, ot.ctypes.data)
    return lt, ot


def attend_tail(q, k, v, seg, times, pen, sel, heads, rows, B: int = 64):
    """Routed attention with the pooled tail term merged in, for (head, row) pairs: rows of video query
    blocks merge their exact routed result with their block's tail partition; other rows are unchanged."""
    o, l = attend(q, k, v, seg, times, pen=pen, sel=sel, heads=heads, rows=rows, B=B)
    lt, ot = tail(q, k, v, seg, sel, B=B)
    fvb = int(block_classes(seg, B).sum())
    blk = np.asarray(rows) // B - fvb
    video = blk >= 0
    o2, l2 = o.copy(), l.copy()
    if video.any():
        hh = np.asarray(heads)[video]
        bb = blk[video]
        mo, ml = merge(np.stack([o[video], ot[hh, bb]]), np.stack([l[video], lt[hh, bb]]))
        o2[video], l2[video] = mo, ml
    return o2, l2
