"""fp64 CPU oracle for cached grouped-query attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg (``bench.py``) may import this package.  It loads ``libkvattn_oracle.so``
built from ``kvattn_oracle.c`` (plain C, fp64, OpenMP) and shares nothing
with the CUDA library.  See ``kvattn_oracle.c`` for the definition computed
and the passages each step follows.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkvattn_oracle.so")
_lib = None

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")

OK, ERR_ARG, ERR_RANGE = 0, 1, 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp, no -ffast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                        "-ffp-contract=off", "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.oracle_rope_freqs.restype = ctypes.c_int
        lib.oracle_rope_freqs.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_double, _f64p]
        lib.oracle_rope_rotate_f64.restype = ctypes.c_int
        lib.oracle_rope_rotate_f64.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, ctypes.c_long,
                                               _f64p, _f64p, ctypes.c_int, ctypes.c_int]
        lib.oracle_rope_append.restype = ctypes.c_int
        lib.oracle_rope_append.argtypes = [ctypes.c_int] * 6 + [_f64p, _i32p, _u16p, _u16p, _u16p,
                                                                _u16p, _u16p, _u16p,
                                                                ctypes.c_void_p, ctypes.c_void_p,
                                                                ctypes.c_int, ctypes.c_int]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [ctypes.c_int] * 6 + [_i32p, ctypes.c_double, _u16p, _u16p,
                                                              _u16p, _f64p, ctypes.c_int]
        lib.oracle_attention_masked.restype = ctypes.c_int
        lib.oracle_attention_masked.argtypes = [ctypes.c_int] * 6 + [_i32p, ctypes.c_double, ctypes.c_int,
                                                                     ctypes.c_int, ctypes.c_void_p, _u16p,
                                                                     _u16p, _u16p, _f64p, ctypes.c_int]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def f64_to_bf16(x: float) -> int:
    return int(_load().oracle_f64_to_bf16(float(x)))


def bf16_to_f64(b: int) -> float:
    return float(_load().oracle_bf16_to_f64(int(b)))


def rope_freqs(head_dim: int = 128, theta: float = 500000.0, use_scaled: bool = False,
               factor: float = 8.0, low_freq_factor: float = 1.0, high_freq_factor: float = 4.0,
               original_max_pos: float = 8192.0) -> np.ndarray:
    out = np.zeros(head_dim // 2, dtype=np.float64)
    rc = _load().oracle_rope_freqs(head_dim, theta, int(use_scaled), factor, low_freq_factor,
                                   high_freq_factor, original_max_pos, out)
    if rc != OK:
        raise ValueError(f"oracle_rope_freqs rc={rc}")
    return out


def rope_rotate_f64(x: np.ndarray, freqs: np.ndarray, pos: int, layout: int = 0, rotary_dim: int = 0) -> np.ndarray:
    """layout 0: interleaved pairs (2i, 2i+1); 1: half-split pairs (i, i+r/2);
    the first rotary_dim elements (0: all d) rotate, the rest pass through."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    d = x.shape[-1]
    y = np.empty_like(x)
    rc = _load().oracle_rope_rotate_f64(x.size // d, d, np.ascontiguousarray(freqs), int(pos),
                                        x.reshape(-1), y.reshape(-1), int(layout), int(rotary_dim))
    if rc != OK:
        raise ValueError(f"oracle_rope_rotate_f64 rc={rc}")
    return y


def rope_append(q, k_new, v_new, cache_k, cache_v, start_pos, freqs, want_exact=False, layout=0, rotary_dim=0):
    """Rotate q and k_new, append k_rot / v_new into the caches IN PLACE.

    q [B,T,H,d], k_new/v_new [B,T,Hkv,d], caches [B,S,Hkv,d]: uint16 bf16 bits.
    Returns (q_rot, rc) or (q_rot, q_exact, k_exact, rc) when ``want_exact``.
    """
    B, T, H, d = q.shape
    Hkv = k_new.shape[2]
    S = cache_k.shape[1]
    q_rot = np.zeros_like(q)
    qe = np.zeros(q.shape, np.float64) if want_exact else None
    ke = np.zeros(k_new.shape, np.float64) if want_exact else None
    rc = _load().oracle_rope_append(
        B, T, H, Hkv, d, S, np.ascontiguousarray(freqs, np.float64),
        np.ascontiguousarray(start_pos, np.int32), np.ascontiguousarray(q),
        np.ascontiguousarray(k_new), np.ascontiguousarray(v_new), q_rot, cache_k, cache_v,
        qe.ctypes.data if want_exact else None, ke.ctypes.data if want_exact else None, int(layout),
        int(rotary_dim))
    if want_exact:
        return q_rot, qe, ke, rc
    return q_rot, rc


def attention(q_rot, cache_k, cache_v, start_pos, scale=None, n_threads=0, window=0, n_sink=0,
              sink_logits=None):
    """fp64 masked GQA softmax attention: returns (out [B,T,H,d] f64, rc).

    window > 0: token at position p sees rows p-window < r <= p, plus the
    first n_sink rows; sink_logits [H] (f64, or None): learned sink logits in
    the units of the scaled scores, added to each head's softmax denominator."""
    B, T, H, d = q_rot.shape
    S, Hkv = cache_k.shape[1], cache_k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, T, H, d), np.float64)
    args = (B, T, H, Hkv, d, S, np.ascontiguousarray(start_pos, np.int32), float(scale))
    tail = (np.ascontiguousarray(q_rot), np.ascontiguousarray(cache_k), np.ascontiguousarray(cache_v), out,
            int(n_threads))
    if window <= 0 and sink_logits is None:
        rc = _load().oracle_attention(*args, *tail)
    else:
        sl = None if sink_logits is None else np.ascontiguousarray(sink_logits, np.float64)
        if sl is not None and sl.shape != (H,):
            raise ValueError("sink_logits must have one entry per query head")
        rc = _load().oracle_attention_masked(*args, int(window), int(n_sink),
                                             None if sl is None else sl.ctypes.data, *tail)
    return out, rc


def step(q, k_new, v_new, cache_k, cache_v, start_pos, freqs, scale=None, n_threads=0, layout=0, rotary_dim=0,
         window=0, n_sink=0, sink_logits=None):
    """One whole cached-attention call: rope + append (caches updated in
    place), then attention over rows 0..start_pos+t (or the window and
    sinks).  Returns (q_rot, out, rc)."""
    q_rot, rc = rope_append(q, k_new, v_new, cache_k, cache_v, start_pos, freqs, layout=layout,
                            rotary_dim=rotary_dim)
    out, rc2 = attention(q_rot, cache_k, cache_v, start_pos, scale, n_threads, window=window, n_sink=n_sink,
                         sink_logits=sink_logits)
    return q_rot, out, max(rc, rc2)
