"""CPU oracle for the quantized attention path — TEST INFRASTRUCTURE ONLY.

This package is the plain single-threaded C statement of the method
(``sage_oracle.c``) plus NumPy marshalling.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg (and its
``--impl reference`` arm) may import it.  The product library never calls
into it and shares no code with it.

Every function takes and returns *logical* layouts:

* ``q8``, ``k8``: int8 ``[B, H, N, D]`` (no padding)
* ``q_scale``: float32 ``[B, H, ceil(N/32)]``; ``k_scale``: ``[B, H, ceil(N/64)]``
* ``k_mean``, ``v_scale``: float32 ``[B, H, D]``
* ``v8``: uint8 E4M3 bytes ``[B, H, N, D]`` (token-major)
* outputs: uint16 BF16 bits ``[rows, D]``

The pins that tie each function to facts outside it (library conversions,
hand-worked examples, closed forms, FP64 attention, invariants, an exact
global-maximum form) live in ``tests/pins.py``; ``tests/test_oracle_pins.py``
runs them and ``tests/test_oracle_plants.py`` shows that each planted
mistake (``ORACLE_PLANT``) fails one.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_BUILD = os.path.join(_HERE, "_build")
_SRC = os.path.join(_HERE, "sage_oracle.c")
_libs: dict = {}

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64


def build(plant: int = 0, force: bool = False) -> str:
    """Compile the oracle (plant > 0 builds a deliberately wrong variant)."""
    os.makedirs(_BUILD, exist_ok=True)
    so = os.path.join(_BUILD, "liboracle.so" if plant == 0 else f"liboracle_plant{plant}.so")
    if force or not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(_SRC):
        tmp = so + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
                               "-fno-fast-math", f"-DORACLE_PLANT={plant}", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, so)
    return so


def _lib(plant: int = 0):
    if plant not in _libs:
        lib = ctypes.CDLL(build(plant))
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_f16_round.restype = ctypes.c_uint16
        lib.oracle_f16_round.argtypes = [ctypes.c_double]
        lib.oracle_f16_decode.restype = ctypes.c_float
        lib.oracle_f16_decode.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_round.restype = ctypes.c_uint16
        lib.oracle_bf16_round.argtypes = [ctypes.c_float]
        strided = [_P, _L, _L, _L, _I, _I, _I, _I]
        lib.oracle_k_mean.argtypes = strided + [_P]
        lib.oracle_quant_q.argtypes = strided + [_P, _P]
        lib.oracle_quant_k.argtypes = strided + [_P, _P, _P]
        lib.oracle_quant_v.argtypes = strided + [_P, _P]
        lib.oracle_norm_rope.argtypes = strided + [_P, _P, _P, ctypes.c_float, _P]
        lib.oracle_attn_rows.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float,
                                         _I, _I, _I, _I, _P, _P]
        lib.oracle_qk_s32.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P]
        for f in ("oracle_k_mean", "oracle_quant_q", "oracle_quant_k", "oracle_quant_v",
                  "oracle_attn_rows", "oracle_qk_s32", "oracle_plant"):
            getattr(lib, f).restype = ctypes.c_int
        _libs[plant] = lib
    return _libs[plant]


def _ptr(a: Optional[np.ndarray]):
    return None if a is None or a.size == 0 else a.ctypes.data


def _strided(x: np.ndarray):
    assert x.dtype == np.uint16 and x.ndim == 4 and x.strides[3] == 2
    B, N, H, D = x.shape
    sb, sn, sh = (s // 2 for s in x.strides[:3])
    return [_ptr(x), sb, sn, sh, B, N, H, D]


def _ok(rc):
    if rc != 0:
        raise ValueError(f"oracle call failed with code {rc}")


# ------------------------------------------------------------------ formats
def e4m3_encode(x, plant: int = 0) -> np.ndarray:
    f = _lib(plant).oracle_e4m3_encode
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint8)


def e4m3_decode(b, plant: int = 0) -> np.ndarray:
    f = _lib(plant).oracle_e4m3_decode
    return np.array([f(int(v)) for v in np.asarray(b, np.uint8).ravel()], np.float64)


def f16_round(x, plant: int = 0) -> np.ndarray:
    f = _lib(plant).oracle_f16_round
    return np.array([f(float(v)) for v in np.asarray(x, np.float64).ravel()], np.uint16)


def bf16_round(x, plant: int = 0) -> np.ndarray:
    f = _lib(plant).oracle_bf16_round
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint16)


# --------------------------------------------------------------- prepasses
def k_mean(k: np.ndarray, plant: int = 0) -> np.ndarray:
    B, N, H, D = k.shape
    km = np.zeros((B, H, D), np.float32)
    _ok(_lib(plant).oracle_k_mean(*_strided(k), _ptr(km)))
    return km


def quant_q(q: np.ndarray, plant: int = 0):
    B, N, H, D = q.shape
    q8 = np.zeros((B, H, N, D), np.int8)
    qs = np.zeros((B, H, (N + 31) // 32), np.float32)
    _ok(_lib(plant).oracle_quant_q(*_strided(q), _ptr(q8), _ptr(qs)))
    return q8, qs


def quant_k(k: np.ndarray, km: np.ndarray, plant: int = 0):
    B, N, H, D = k.shape
    k8 = np.zeros((B, H, N, D), np.int8)
    ks = np.zeros((B, H, (N + 63) // 64), np.float32)
    _ok(_lib(plant).oracle_quant_k(*_strided(k), _ptr(np.ascontiguousarray(km, np.float32)),
                                   _ptr(k8), _ptr(ks)))
    return k8, ks


def quant_v(v: np.ndarray, plant: int = 0):
    B, N, H, D = v.shape
    v8 = np.zeros((B, H, N, D), np.uint8)
    vs = np.zeros((B, H, D), np.float32)
    _ok(_lib(plant).oracle_quant_v(*_strided(v), _ptr(v8), _ptr(vs)))
    return v8, vs


def norm_rope(x: np.ndarray, w: np.ndarray, cos_t: np.ndarray, sin_t: np.ndarray, eps: float,
              plant: int = 0) -> np.ndarray:
    """RMSNorm over D then split-half RoPE (reading R11) of a strided BF16
    [B, N, H, D] view; weights BF16 bits [D], tables FP32 [N, D/2].  Returns
    contiguous BF16 bits [B, N, H, D]."""
    B, N, H, D = x.shape
    z = np.zeros((B, N, H, D), np.uint16)
    _ok(_lib(plant).oracle_norm_rope(*_strided(x), _ptr(np.ascontiguousarray(w, np.uint16)),
                                     _ptr(np.ascontiguousarray(cos_t, np.float32)),
                                     _ptr(np.ascontiguousarray(sin_t, np.float32)), float(eps), _ptr(z)))
    return z


def quantize_normed(q, k, v, wq, wk, cos_t, sin_t, eps, plant: int = 0) -> "Quantized":
    """The producer (R11) on Q and K, then the same prepasses as quantize()."""
    return quantize(norm_rope(q, wq, cos_t, sin_t, eps, plant), norm_rope(k, wk, cos_t, sin_t, eps, plant),
                    v, plant)


@dataclass
class Quantized:
    q8: np.ndarray
    q_scale: np.ndarray
    k8: np.ndarray
    k_scale: np.ndarray
    k_mean: np.ndarray
    v8: np.ndarray
    v_scale: np.ndarray
    B: int
    N: int
    H: int
    D: int


def quantize(q: np.ndarray, k: np.ndarray, v: np.ndarray, plant: int = 0) -> Quantized:
    """The three prepasses (a1-a4) on strided BF16 [B, N, H, D] views."""
    B, N, H, D = q.shape
    km = k_mean(k, plant)
    q8, qs = quant_q(q, plant)
    k8, ks = quant_k(k, km, plant)
    v8, vs = quant_v(v, plant)
    return Quantized(q8, qs, k8, ks, km, v8, vs, B, N, H, D)


def attn_rows(qz: Quantized, b: int, h: int, row0: int, rows: int, sm_scale: float = 0.0,
              plant: int = 0, with_stats: bool = False):
    """Quantized attention (a5-a9) for rows [row0, row0+rows) of head (b, h).

    Returns BF16 bits [rows, D] (and (m, d) per row when with_stats)."""
    out = np.zeros((rows, qz.D), np.uint16)
    st = np.zeros((rows, 2), np.float32) if with_stats else None
    _ok(_lib(plant).oracle_attn_rows(_ptr(qz.q8), _ptr(qz.q_scale), _ptr(qz.k8), _ptr(qz.k_scale),
                                     _ptr(qz.v8), _ptr(qz.v_scale), qz.B, qz.N, qz.H, qz.D,
                                     float(sm_scale), b, h, row0, rows, _ptr(out), _ptr(st)))
    return (out, st) if with_stats else out


def attention(qz: Quantized, sm_scale: float = 0.0, plant: int = 0) -> np.ndarray:
    """Full quantized attention output, BF16 bits [B, N, H, D] (small shapes only)."""
    out = np.zeros((qz.B, qz.N, qz.H, qz.D), np.uint16)
    for b in range(qz.B):
        for h in range(qz.H):
            if qz.N:
                out[b, :, h, :] = attn_rows(qz, b, h, 0, qz.N, sm_scale, plant)
    return out


def qk_s32(qz: Quantized, b: int, h: int, row0: int, rows: int, key0: int, keys: int) -> np.ndarray:
    """Exact int32 QK^T block; rows/keys beyond N read as zero padding."""
    S = np.zeros((rows, keys), np.int32)
    _ok(_lib().oracle_qk_s32(_ptr(qz.q8), _ptr(qz.k8), qz.B, qz.N, qz.H, qz.D, b, h,
                             row0, rows, key0, keys, _ptr(S)))
    return S


def bf16_bits_to_float(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a).astype(np.uint32) << 16).view(np.float32)
