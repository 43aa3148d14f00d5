"""Seeded synthetic inputs for the packed MiniMax-H3 attention call.

This package is shared by the oracle-side tests, ``bench.py`` and the GPU
parity tests.  It holds the input recipe only (layouts, seeds, random numbers,
cluster means, bf16 rounding) and none of the attention method's arithmetic.

Layouts follow the packed sequence ``[text | image-ref | audio | guide video |
output video]`` that the TARA / Flash-Partitions page describes (its section
"What receives the temporal bias?"): video rows are a contiguous suffix with a
fixed token count per latent frame, and latent frame k sits at t = k * 4 / 24 s
on both the guide and the output clock (24 fps, 4 video frames per latent).

Segment ids: 0 text, 1 image-ref, 2 audio, 3 guide video, 4 output video.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libinputs.so")

SEG_TEXT, SEG_IMAGE_REF, SEG_AUDIO, SEG_GUIDE, SEG_OUTPUT = 0, 1, 2, 3, 4
TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2
FRAME_SECONDS = 4.0 / 24.0


def build(force: bool = False) -> str:
    """Compile gen.c into libinputs.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.gen_tensor.argtypes = [
            ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_double,
            ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        _lib.gen_tensor.restype = None
        _lib.gen_normal.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int]
        _lib.gen_normal.restype = ctypes.c_double
        _lib.gen_threads.restype = ctypes.c_int
    return _lib


@dataclass(frozen=True)
class Segment:
    seg: int                 # segment id
    rows: int                # rows in this segment
    frames: int = 0          # latent frames (0: untimed, no cluster mean)

    @property
    def tokens_per_frame(self) -> int:
        return self.rows // self.frames if self.frames else 0


@dataclass
class Config:
    name: str
    H: int
    d: int
    segments: Tuple[Segment, ...]
    seed: int
    cluster_norm: float = 0.0           # 0: plain N(0,1) Q/K
    sparsities: Tuple[float, ...] = (0.0,)
    penalty: Optional[Tuple[float, float, float, float]] = None  # strength, window, falloff, cap
    block: int = 64

    @property
    def S(self) -> int:
        return sum(s.rows for s in self.segments)

    def layout(self) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """(seg u8[S], times f32[S], frame i32[S]); frame -1 for untimed rows."""
        S = self.S
        seg = np.empty(S, np.uint8)
        times = np.zeros(S, np.float32)
        frame = np.full(S, -1, np.int32)
        r = 0
        for s in self.segments:
            seg[r:r + s.rows] = s.seg
            if s.frames:
                tpf = s.tokens_per_frame
                assert tpf * s.frames == s.rows, (s, "rows must be frames x tokens")
                f = np.arange(s.rows, dtype=np.int64) // tpf
                frame[r:r + s.rows] = f.astype(np.int32)
                times[r:r + s.rows] = (f * FRAME_SECONDS).astype(np.float32)
            r += s.rows
        return seg, times, frame


DEFAULT_PENALTY = (2.0, 0.20, 0.25, 6.0)   # strength, window [s], falloff [s], cap

# The five workloads of the hot path (packings as stated for the H3 call).
# tiny dense biased: text 64 | audio 160 | guide 8x112 | output 8x116
TINY_DENSE = Config("tiny dense biased S=2048 H=2 d=64", H=2, d=64,
                    segments=(Segment(SEG_TEXT, 64), Segment(SEG_AUDIO, 160),
                              Segment(SEG_GUIDE, 896, 8), Segment(SEG_OUTPUT, 928, 8)),
                    seed=1001, penalty=DEFAULT_PENALTY, sparsities=(0.0,))
# routing-only: text 256 | audio 384 | video 41 frames x 384
ROUTING_ONLY = Config("routing S=16384 H=8 d=128 s=0.85", H=8, d=128,
                      segments=(Segment(SEG_TEXT, 256), Segment(SEG_AUDIO, 384),
                                Segment(SEG_OUTPUT, 15744, 41)),
                      seed=1002, cluster_norm=2.0, sparsities=(0.85,))
# mid clip: text 256 | image-ref 1024 | audio 400 | video 24 frames x 1978
MID_CLIP = Config("mid clip S=49152 H=56 d=128", H=56, d=128,
                  segments=(Segment(SEG_TEXT, 256), Segment(SEG_IMAGE_REF, 1024),
                            Segment(SEG_AUDIO, 400), Segment(SEG_OUTPUT, 47472, 24)),
                  seed=1003, cluster_norm=2.0, sparsities=(0.0, 0.60, 0.85, 0.90))
# full dense biased: text 256 | image-ref 1013 | audio 810 | guide 27x2126 | output 27x2126
FULL_DENSE = Config("full dense biased S=116883 H=56 d=128", H=56, d=128,
                    segments=(Segment(SEG_TEXT, 256), Segment(SEG_IMAGE_REF, 1013),
                              Segment(SEG_AUDIO, 810), Segment(SEG_GUIDE, 57402, 27),
                              Segment(SEG_OUTPUT, 57402, 27)),
                    seed=1004, cluster_norm=2.0, penalty=DEFAULT_PENALTY, sparsities=(0.0,))
# full combined (the benchmark's workload): the full dense packing, routed to
# the top 10 % of video KV blocks, penalty on
FULL_COMBINED = Config("full combined S=116883 H=56 d=128 s=0.90", H=56, d=128,
                       segments=(Segment(SEG_TEXT, 256), Segment(SEG_IMAGE_REF, 1013),
                                 Segment(SEG_AUDIO, 810), Segment(SEG_GUIDE, 57402, 27),
                                 Segment(SEG_OUTPUT, 57402, 27)),
                       seed=1005, cluster_norm=2.0, penalty=DEFAULT_PENALTY, sparsities=(0.90,))

WORKLOADS = (TINY_DENSE, ROUTING_ONLY, MID_CLIP, FULL_DENSE, FULL_COMBINED)


def custom(H: int, d: int, segments: Sequence[Segment], seed: int, cluster_norm: float = 0.0,
           penalty=None, sparsities=(0.0,), name: str = "custom") -> Config:
    return Config(name, H, d, tuple(segments), seed, cluster_norm, tuple(sparsities), penalty)


def tensor(cfg: Config, which: int, h0: int = 0, nh: Optional[int] = None, row0: int = 0,
           nrows: Optional[int] = None, out: Optional[np.ndarray] = None,
           seed: Optional[int] = None) -> np.ndarray:
    """bf16 bits (np.uint16) of tensor `which` for heads [h0,h0+nh), rows [row0,row0+nrows).

    Shape [nh][nrows][d].  `out` may be any C-contiguous uint16 buffer of that
    size (for example a pinned host tensor's numpy view)."""
    S, d = cfg.S, cfg.d
    nh = cfg.H - h0 if nh is None else nh
    nrows = S - row0 if nrows is None else nrows
    assert 0 <= h0 and h0 + nh <= cfg.H and 0 <= row0 and row0 + nrows <= S
    seg, _, frame = cfg.layout()
    if out is None:
        out = np.empty((nh, nrows, d), np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == nh * nrows * d
    lib().gen_tensor(ctypes.c_uint64(cfg.seed if seed is None else seed), which, S, d,
                     seg.ctypes.data, frame.ctypes.data, float(cfg.cluster_norm),
                     h0, nh, row0, nrows, out.ctypes.data)
    return out


def rows(cfg: Config, which: int, h: int, row_ids: Sequence[int]) -> np.ndarray:
    """bf16 bits [len(row_ids)][d] of tensor `which`, head h, the given rows."""
    res = np.empty((len(row_ids), cfg.d), np.uint16)
    for i, r in enumerate(row_ids):
        tensor(cfg, which, h0=h, nh=1, row0=int(r), nrows=1, out=res[i])
    return res


def bf16_bits_to_f64(x: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (finite values)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def threads() -> int:
    return int(lib().gen_threads())
