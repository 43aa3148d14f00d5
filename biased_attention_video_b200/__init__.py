"""Python binding of libh3attn (biased, block-routed attention over MiniMax-H3's
packed sequence on B200).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch supplies device memory and the current stream.  There is no
fallback: if libh3attn.so cannot be loaded, every call raises.

Tensors: q, k, v, o bf16 [H, S, d] contiguous CUDA; seg uint8 [S]; times
float32 [S]; kv_sel int32 [H, n_video_blocks, k].
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import build as _build

OK, EINVAL, EUNSUPPORTED, EALIGN, ECUDA, ETIMEOUT, EWORKSPACE, EDATA = 0, -1, -2, -3, -4, -5, -6, -7
SEG_TEXT, SEG_IMAGE_REF, SEG_AUDIO, SEG_GUIDE, SEG_OUTPUT = 0, 1, 2, 3, 4

# every symbol the C header declares
EXPORTS = ("h3attn_plan_init", "h3attn_workspace_bytes", "h3attn_pool", "h3attn_route", "h3attn_route_static",
           "h3attn_route_static_check",
           "h3attn_forward",
           "h3attn_dense_workspace_bytes", "h3attn_dense_biased", "h3attn_check", "h3attn_selftest_timeout", "h3attn_set_wait_polls",
           "h3attn_attend_host", "h3attn_merge", "h3attn_tail_workspace_bytes", "h3attn_tail_correct",
           "h3attn_qk8_workspace_bytes", "h3attn_quantize_qk", "h3attn_forward_qk8",
           "h3attn_strerror")


class H3Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {lib().h3attn_strerror(code).decode()} ({code})")


class Plan(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("S", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32),
                ("sparsity", ctypes.c_double), ("n_blocks", ctypes.c_int32), ("prefix_rows", ctypes.c_int32),
                ("first_video_block", ctypes.c_int32), ("n_forced", ctypes.c_int32),
                ("n_video_blocks", ctypes.c_int32), ("k", ctypes.c_int32)]

    def __repr__(self):
        return "Plan(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class Penalty(ctypes.Structure):
    _fields_ = [("strength", ctypes.c_float), ("window", ctypes.c_float), ("falloff", ctypes.c_float),
                ("cap", ctypes.c_float)]


DEFAULT_PENALTY = (2.0, 0.20, 0.25, 6.0)

_lib = None
_P = ctypes.c_void_p


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libh3attn.so (building it in-tree with nvcc if it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        PP = ctypes.POINTER(Plan)
        L.h3attn_plan_init.argtypes = [PP, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _P]
        L.h3attn_plan_init.restype = ctypes.c_int
        L.h3attn_workspace_bytes.argtypes = [PP]
        L.h3attn_workspace_bytes.restype = ctypes.c_size_t
        L.h3attn_pool.argtypes = [PP, _P, ctypes.c_int, ctypes.c_int, _P, _P]
        L.h3attn_pool.restype = ctypes.c_int
        L.h3attn_route.argtypes = [PP, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.h3attn_route.restype = ctypes.c_int
        L.h3attn_route_static.argtypes = [PP, _P, _P, _P, _P]
        L.h3attn_route_static.restype = ctypes.c_int
        L.h3attn_route_static_check.argtypes = [_P]
        L.h3attn_route_static_check.restype = ctypes.c_int
        L.h3attn_forward.argtypes = [PP, _P, _P, _P, _P, _P, ctypes.POINTER(Penalty), _P, _P, _P, _P,
                                     ctypes.c_size_t, _P]
        L.h3attn_forward.restype = ctypes.c_int
        L.h3attn_dense_workspace_bytes.argtypes = [ctypes.c_int]
        L.h3attn_dense_workspace_bytes.restype = ctypes.c_size_t
        L.h3attn_dense_biased.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _P,
                                          ctypes.POINTER(Penalty), _P, _P, _P, ctypes.c_size_t, _P]
        L.h3attn_dense_biased.restype = ctypes.c_int
        L.h3attn_attend_host.argtypes = [PP, _P, _P, _P, _P, _P, ctypes.POINTER(Penalty), _P, _P, _P, _P, _P, _P,
                                         _P, _P, _P, _P, _P, ctypes.c_size_t, ctypes.c_int, _P, _P, _P]
        L.h3attn_attend_host.restype = ctypes.c_int
        L.h3attn_merge.argtypes = [ctypes.c_int, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_float),
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P]
        L.h3attn_merge.restype = ctypes.c_int
        L.h3attn_tail_workspace_bytes.argtypes = [PP]
        L.h3attn_tail_workspace_bytes.restype = ctypes.c_size_t
        L.h3attn_tail_correct.argtypes = [PP, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]
        L.h3attn_tail_correct.restype = ctypes.c_int
        L.h3attn_qk8_workspace_bytes.argtypes = [PP]
        L.h3attn_qk8_workspace_bytes.restype = ctypes.c_size_t
        L.h3attn_quantize_qk.argtypes = [PP, _P, _P, _P, ctypes.c_size_t, _P]
        L.h3attn_quantize_qk.restype = ctypes.c_int
        L.h3attn_forward_qk8.argtypes = [PP, _P, _P, _P, _P, _P, ctypes.POINTER(Penalty), _P, _P, _P, _P,
                                         ctypes.c_size_t, _P, ctypes.c_size_t, _P]
        L.h3attn_forward_qk8.restype = ctypes.c_int
        L.h3attn_check.argtypes = [_P, _P]
        L.h3attn_check.restype = ctypes.c_int
        L.h3attn_set_wait_polls.argtypes = [ctypes.c_uint32]
        L.h3attn_set_wait_polls.restype = ctypes.c_int
        L.h3attn_selftest_timeout.argtypes = [_P, ctypes.c_uint32, _P]
        L.h3attn_selftest_timeout.restype = ctypes.c_int
        L.h3attn_strerror.argtypes = [ctypes.c_int]
        L.h3attn_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _raise(code: int, what: str):
    if code != OK:
        raise H3Error(code, what)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _check_qkv(*ts):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 3):
            raise ValueError("q/k/v/o must be contiguous CUDA bf16 [H, S, d]")


def _pen(pen) -> Optional[Penalty]:
    if pen is None:
        return None
    if isinstance(pen, Penalty):
        return pen
    s, w, f, c = pen
    return Penalty(s, w, f, c)


def plan(H: int, S: int, d: int, seg_host, sparsity: float = 0.0, block: int = 64) -> Plan:
    """Block plan from the host copy of seg (numpy or CPU tensor, uint8 [S])."""
    seg = np.ascontiguousarray(seg_host.cpu().numpy() if isinstance(seg_host, torch.Tensor) else seg_host,
                               dtype=np.uint8)
    if seg.shape != (S,):
        raise ValueError("seg must have S entries")
    p = Plan()
    _raise(lib().h3attn_plan_init(ctypes.byref(p), H, S, d, block, sparsity, seg.ctypes.data), "plan_init")
    return p


def workspace(p: Plan, device="cuda") -> torch.Tensor:
    n = lib().h3attn_workspace_bytes(ctypes.byref(p))
    if n == 0:
        raise H3Error(EINVAL, "workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def dense_workspace(S: int, device="cuda") -> torch.Tensor:
    return torch.zeros(lib().h3attn_dense_workspace_bytes(S), dtype=torch.uint8, device=device)


def pool(p: Plan, x: torch.Tensor, first_block: int = 0, n_out: Optional[int] = None, out=None, stream=None):
    """Block means (fp32 [H, n_out, d]) of blocks [first_block, first_block + n_out)."""
    _check_qkv(x)
    n_out = p.n_blocks - first_block if n_out is None else n_out
    if out is None:
        out = torch.empty((p.H, n_out, p.d), dtype=torch.float32, device=x.device)
    _raise(lib().h3attn_pool(ctypes.byref(p), x.data_ptr(), first_block, n_out, out.data_ptr(), _stream(stream)),
           "pool")
    return out


def route(p: Plan, q: torch.Tensor, k: torch.Tensor, ws: torch.Tensor, kv_sel=None, stream=None) -> torch.Tensor:
    """Routed key blocks int32 [H, n_video_blocks, k] (absolute block ids, ascending)."""
    _check_qkv(q, k)
    if kv_sel is None:
        kv_sel = torch.empty((p.H, p.n_video_blocks, p.k), dtype=torch.int32, device=q.device)
    _raise(lib().h3attn_route(ctypes.byref(p), q.data_ptr(), k.data_ptr(), kv_sel.data_ptr(), ws.data_ptr(),
                              ws.numel(), _stream(stream)), "route")
    return kv_sel


def route_static(p: Plan, q: torch.Tensor, k: torch.Tensor, kv_sel=None, stream=None) -> torch.Tensor:
    """Same result as route(), for callers that cannot allocate device memory: the
    pooled centroids live in a fixed 64 MiB array inside the library (no workspace).
    The output buffer kv_sel may be passed in; concurrent calls share that array."""
    _check_qkv(q, k)
    if kv_sel is None:
        kv_sel = torch.empty((p.H, p.n_video_blocks, p.k), dtype=torch.int32, device=q.device)
    _raise(lib().h3attn_route_static(ctypes.byref(p), q.data_ptr(), k.data_ptr(), kv_sel.data_ptr(),
                                     _stream(stream)), "route_static")
    return kv_sel


def route_static_check(stream=None) -> int:
    """Synchronise and return (then clear) the status word of the route_static calls on the current device."""
    return lib().h3attn_route_static_check(_stream(stream))


def forward(p: Plan, q, k, v, seg, times, pen=DEFAULT_PENALTY, kv_sel=None, ws=None, out=None,
            lse: bool | torch.Tensor = False, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Attention over the routed tiles (kv_sel None = dense) with the temporal penalty (pen None = off)."""
    _check_qkv(q, k, v)
    if ws is None:
        ws = workspace(p, q.device)
    o = torch.empty_like(q) if out is None else out
    lse_t = lse if isinstance(lse, torch.Tensor) else (
        torch.empty((p.H, p.S), dtype=torch.float32, device=q.device) if lse else None)
    pn = _pen(pen)
    _raise(lib().h3attn_forward(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), seg.data_ptr(),
                                _dptr(times), ctypes.byref(pn) if pn is not None else None, _dptr(kv_sel),
                                o.data_ptr(), _dptr(lse_t), ws.data_ptr(), ws.numel(), _stream(stream)), "forward")
    return o, lse_t


def qk8_workspace(p: Plan, device="cuda") -> torch.Tensor:
    """Scratch of the int8-QK path: codes and per-token scales of Q and K."""
    n = lib().h3attn_qk8_workspace_bytes(ctypes.byref(p))
    if n == 0:
        raise H3Error(EINVAL, "qk8_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _align256(x: int) -> int:
    return (x + 255) // 256 * 256


def quantize_qk(p: Plan, q, k, qk8_ws=None, stream=None):
    """Per-token int8 quantisation of Q and K (h3attn_quantize_qk).  Returns views of the scratch:
    (q8 int8 [H, S, d], k8 int8 [H, S, d], q_scale float32 [H, 64 n_blocks], k_scale float32 [H, 64 n_blocks])."""
    _check_qkv(q, k, k)
    if qk8_ws is None:
        qk8_ws = qk8_workspace(p, q.device)
    _raise(lib().h3attn_quantize_qk(ctypes.byref(p), q.data_ptr(), k.data_ptr(), qk8_ws.data_ptr(), qk8_ws.numel(),
                                    _stream(stream)), "quantize_qk")
    codes = p.H * p.S * p.d
    stride = p.n_blocks * 64
    o_k8 = _align256(codes)
    o_sq = o_k8 + _align256(codes)
    o_sk = o_sq + _align256(p.H * stride * 4)
    q8 = qk8_ws[:codes].view(torch.int8).view(p.H, p.S, p.d)
    k8 = qk8_ws[o_k8:o_k8 + codes].view(torch.int8).view(p.H, p.S, p.d)
    sq = qk8_ws[o_sq:o_sq + p.H * stride * 4].view(torch.float32).view(p.H, stride)
    sk = qk8_ws[o_sk:o_sk + p.H * stride * 4].view(torch.float32).view(p.H, stride)
    return q8, k8, sq, sk


def forward_qk8(p: Plan, q, k, v, seg, times, pen=DEFAULT_PENALTY, kv_sel=None, ws=None, qk8_ws=None, out=None,
                lse: bool | torch.Tensor = False, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """forward with Q and K quantised per token to int8 before the QK product (h3attn_forward_qk8)."""
    _check_qkv(q, k, v)
    if ws is None:
        ws = workspace(p, q.device)
    if qk8_ws is None:
        qk8_ws = qk8_workspace(p, q.device)
    o = torch.empty_like(q) if out is None else out
    lse_t = lse if isinstance(lse, torch.Tensor) else (
        torch.empty((p.H, p.S), dtype=torch.float32, device=q.device) if lse else None)
    pn = _pen(pen)
    _raise(lib().h3attn_forward_qk8(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), seg.data_ptr(),
                                    _dptr(times), ctypes.byref(pn) if pn is not None else None, _dptr(kv_sel),
                                    o.data_ptr(), _dptr(lse_t), ws.data_ptr(), ws.numel(), qk8_ws.data_ptr(),
                                    qk8_ws.numel(), _stream(stream)), "forward_qk8")
    return o, lse_t


def dense_biased(q, k, v, seg, times, pen=DEFAULT_PENALTY, ws=None, out=None, lse: bool = False, stream=None):
    """Dense attention with the temporal penalty on output -> guide pairs."""
    _check_qkv(q, k, v)
    H, S, d = q.shape
    if ws is None:
        ws = dense_workspace(S, q.device)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((H, S), dtype=torch.float32, device=q.device) if lse else None
    pn = _pen(pen)
    _raise(lib().h3attn_dense_biased(H, S, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), seg.data_ptr(),
                                     _dptr(times), ctypes.byref(pn) if pn is not None else None, o.data_ptr(),
                                     _dptr(lse_t), ws.data_ptr(), ws.numel(), _stream(stream)), "dense_biased")
    return o, lse_t


def attend_host(p: Plan, q_host, k_host, v_host, seg_host, times_host, o_host, *, q, k, v, seg, times, o, ws,
                kv_sel=None, pen=DEFAULT_PENALTY, lse_host=None, lse=None, chunk_heads: int = 4, stream=None,
                copy_in_stream=None, copy_out_stream=None) -> None:
    """The whole call from (page-locked) host tensors, copies overlapped with the kernels per chunk of heads.

    Host tensors: q_host/k_host/v_host/o_host bf16 or int16 [H, S, d]; seg_host uint8 [S]; times_host float32 [S];
    device buffers q/k/v/o/seg/times (and kv_sel, lse) of the same shapes.  Streams are torch.cuda.Stream
    objects (None = the current stream)."""
    pn = _pen(pen)
    _raise(lib().h3attn_attend_host(
        ctypes.byref(p), q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), seg_host.data_ptr(),
        _dptr(times_host), ctypes.byref(pn) if pn is not None else None, o_host.data_ptr(), _dptr(lse_host),
        q.data_ptr(), k.data_ptr(), v.data_ptr(), seg.data_ptr(), _dptr(times), _dptr(kv_sel), o.data_ptr(),
        _dptr(lse), ws.data_ptr(), ws.numel(), chunk_heads, _stream(stream), _stream(copy_in_stream),
        _stream(copy_out_stream)), "attend_host")


def merge(o_parts, lse_parts, log_w=None, out=None, lse: bool | torch.Tensor = False, stream=None):
    """Merge normalised partition results (forward outputs o [H, S, d] bf16 and lse [H, S] float32 over key
    sets) with multipliers exp(log_w[i]); returns (O, LSE or None)."""
    n = len(o_parts)
    if n != len(lse_parts) or n == 0:
        raise ValueError("o_parts and lse_parts must be non-empty and of equal length")
    _check_qkv(*o_parts)
    H, S, d = o_parts[0].shape
    for t in lse_parts:
        if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (H, S)):
            raise ValueError("lse parts must be contiguous CUDA float32 [H, S]")
    o = torch.empty_like(o_parts[0]) if out is None else out
    lse_t = lse if isinstance(lse, torch.Tensor) else (
        torch.empty((H, S), dtype=torch.float32, device=o.device) if lse else None)
    op = (_P * n)(*[t.data_ptr() for t in o_parts])
    lp = (_P * n)(*[t.data_ptr() for t in lse_parts])
    lw = None if log_w is None else (ctypes.c_float * n)(*[float(x) for x in log_w])
    _raise(lib().h3attn_merge(n, op, lp, lw, H, S, d, o.data_ptr(), _dptr(lse_t), _stream(stream)), "merge")
    return o, lse_t


def tail_workspace(p: Plan, device="cuda") -> torch.Tensor:
    n = lib().h3attn_tail_workspace_bytes(ctypes.byref(p))
    if n == 0:
        raise H3Error(EINVAL, "tail_workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def tail_correct(p: Plan, v, kv_sel, o, lse, ws, tail_ws=None, stream=None) -> None:
    """Fold the routed-out video key blocks into (o, lse) as one pooled term per query block, in place.
    Call after route(p, q, k, ws, kv_sel) and forward(..., kv_sel, ws, out=o, lse=lse) with the same ws."""
    _check_qkv(v, o)
    tw = tail_workspace(p, v.device) if tail_ws is None else tail_ws
    _raise(lib().h3attn_tail_correct(ctypes.byref(p), v.data_ptr(), kv_sel.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                     ws.data_ptr(), ws.numel(), tw.data_ptr(), tw.numel(), _stream(stream)),
           "tail_correct")


def check(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return (and clear) the device status word."""
    return int(lib().h3attn_check(ws.data_ptr(), _stream(stream)))


def set_wait_polls(polls: int) -> None:
    """Test and diagnostics only: bound the attention kernels' waits of later calls to `polls` polls
    (0 = default, no poll bound)."""
    _raise(lib().h3attn_set_wait_polls(polls), "set_wait_polls")


def selftest_timeout(ws: torch.Tensor, polls: int, stream=None) -> None:
    _raise(lib().h3attn_selftest_timeout(ws.data_ptr(), polls, _stream(stream)), "selftest_timeout")
