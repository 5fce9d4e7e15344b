"""Seeded synthetic Q/K/V inputs for the quantized attention path.

This module holds no step of the attention method.  It builds BF16
activations of the shapes, strides and value distributions of the five
workloads below and hands back NumPy ``uint16`` arrays holding BF16 bit
patterns, shaped ``[B, N, H, D]`` (possibly strided views into one fused
projection buffer).  The same bytes feed the CPU oracle and the GPU path.

The pages measure on real activations of a video diffusion transformer
(37,810 tokens, 56 heads, D=128; the tokens come from 1344x768 video, 124
frames).  Those activations need trained weights and are not available, so
seeded normal data of the same shape and strides stands in for them.

Element recipe (see ``synth_gen.c`` for the generator itself):
``x = scale * N(0,1) [+ K offset U(lo,hi) fixed per (head, channel)]``,
optionally ``x *= outlier_mult`` for a Bernoulli(outlier_prob) subset of Q
entries, stored as BF16 with round-to-nearest-even.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libsynth.so")
_SRC = os.path.join(_HERE, "synth_gen.c")

# stream ids: one independent counter stream per tensor / structure
STREAM_Q, STREAM_K, STREAM_V, STREAM_K_OFFSET, STREAM_Q_OUTLIER = 1, 2, 3, 4, 5

_lib = None


def build(force: bool = False) -> str:
    """Compile the generator with gcc (no GPU needed)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_fill_bf16.restype = ctypes.c_int
        lib.synth_fill_bf16.argtypes = [
            ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float,
            ctypes.c_void_p, ctypes.c_float, ctypes.c_float, ctypes.c_uint32, ctypes.c_int]
        lib.synth_uniform_f32.restype = ctypes.c_int
        lib.synth_uniform_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                          ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Config:
    """One workload: shape, layout and value distribution."""
    name: str
    B: int
    N: int
    H: int
    D: int
    layout: str = "contiguous"          # or "fused_qkv": one [B, N, 3*H*D] projection buffer
    scale: float = 1.0                  # std of Q, K, V
    k_offset: float = 2.0               # K offset ~ U(-k_offset, k_offset) per (head, channel)
    q_outlier_prob: float = 0.0
    q_outlier_mult: float = 1.0
    about: str = ""

    @property
    def ops(self) -> float:
        """Effective operation count 4*B*H*N^2*D (QK^T and PV, 2 ops per MAC)."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.D


CONFIGS = {
    "small": Config("small", 1, 256, 2, 128,
                    about="B1 N256 H2 D128 contiguous; Q,V~N(0,1), K~N(0,1)+U(-2,2)[h,d]"),
    "ragged": Config("ragged", 1, 1000, 8, 128,
                     about="B1 N1000 H8 D128; ragged tails (8-row Q32 group, 40-row K64 tile)"),
    "outlier": Config("outlier", 2, 8192, 32, 128, scale=0.5, k_offset=3.0,
                      q_outlier_prob=0.01, q_outlier_mult=8.0,
                      about="B2 N8192 H32 D128; 0.5*N(0,1), K+U(-3,3), 1% of Q entries x8"),
    "long_fused": Config("long_fused", 1, 37810, 56, 128, layout="fused_qkv",
                         about="B1 N37810 H56 D128; Q/K/V projection-strided views of one "
                               "[N, 21504] BF16 buffer at column offsets 0/7168/14336"),
    "d64_batch": Config("d64_batch", 4, 16384, 24, 64,
                        about="B4 N16384 H24 D64 contiguous; D=64 tile variant at high batch"),
}
# the order the workloads are listed in, smallest first
CONFIG_ORDER = ["small", "ragged", "outlier", "long_fused", "d64_batch"]


@dataclass
class Inputs:
    cfg: Config
    q: np.ndarray               # uint16 BF16 bits, [B, N, H, D] view
    k: np.ndarray
    v: np.ndarray
    buffers: list = field(default_factory=list)   # the arrays that own the memory
    k_offset: Optional[np.ndarray] = None          # float32 [H, D]

    def strides(self, which: str):
        """Element strides (b, n, h) of one view; d is unit stride."""
        a = getattr(self, which)
        s = [x // 2 for x in a.strides]
        assert s[3] == 1
        return s[0], s[1], s[2]


def uniform(seed: int, stream: int, count: int, lo: float, hi: float) -> np.ndarray:
    out = np.empty(count, np.float32)
    rc = _load().synth_uniform_f32(seed, stream, count, lo, hi, out.ctypes.data if count else None)
    assert rc == 0
    return out


def _fill(view: np.ndarray, seed: int, stream: int, scale: float, offset: Optional[np.ndarray],
          oprob: float, omult: float, threads: int):
    B, N, H, D = view.shape
    sb, sn, sh, sd = (s // 2 for s in view.strides)
    assert sd == 1
    off_ptr = offset.ctypes.data if offset is not None else None
    rc = _load().synth_fill_bf16(seed, stream, B, N, H, D, sb, sn, sh,
                                 view.ctypes.data if view.size else None, scale, off_ptr,
                                 oprob, omult, STREAM_Q_OUTLIER, threads)
    assert rc == 0


def make_inputs(cfg: Config, seed: int = 0, threads: Optional[int] = None) -> Inputs:
    """Generate Q, K, V for one workload (deterministic for a given seed)."""
    threads = threads or min(32, os.cpu_count() or 1)
    B, N, H, D = cfg.B, cfg.N, cfg.H, cfg.D
    if cfg.layout == "fused_qkv":
        fused = np.empty((B, N, 3 * H * D), np.uint16)
        q = fused[:, :, 0:H * D].reshape(B, N, H, D)
        k = fused[:, :, H * D:2 * H * D].reshape(B, N, H, D)
        v = fused[:, :, 2 * H * D:3 * H * D].reshape(B, N, H, D)
        buffers = [fused]
    elif cfg.layout == "contiguous":
        q = np.empty((B, N, H, D), np.uint16)
        k = np.empty((B, N, H, D), np.uint16)
        v = np.empty((B, N, H, D), np.uint16)
        buffers = [q, k, v]
    else:
        raise ValueError(cfg.layout)
    koff = uniform(seed, STREAM_K_OFFSET, H * D, -cfg.k_offset, cfg.k_offset).reshape(H, D) \
        if cfg.k_offset > 0 else None
    _fill(q, seed, STREAM_Q, cfg.scale, None, cfg.q_outlier_prob, cfg.q_outlier_mult, threads)
    _fill(k, seed, STREAM_K, cfg.scale, koff, 0.0, 1.0, threads)
    _fill(v, seed, STREAM_V, cfg.scale, None, 0.0, 1.0, threads)
    return Inputs(cfg, q, k, v, buffers, koff)


def custom(B: int, N: int, H: int, D: int, seed: int = 0, **kw) -> Inputs:
    """Inputs of an arbitrary shape with the default distribution (tests)."""
    return make_inputs(Config("custom", B, N, H, D, **kw), seed)


def bf16_to_float(a: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float32 (exact; a bit shift)."""
    return (np.ascontiguousarray(a).astype(np.uint32) << 16).view(np.float32)
