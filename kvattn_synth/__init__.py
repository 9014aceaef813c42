"""Seeded synthetic inputs for cached grouped-query attention.

This module holds no attention arithmetic: it only draws the numbers that
both the CUDA path and the fp64 oracle consume.  It is shared by both sides
and imports neither of them.

Generator (published definitions, implemented twice: numpy here for the
host, a CUDA kernel in ``synth.cu`` for large device-resident caches):

* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): state advance by gamma = 0x9E3779B97F4A7C15 and
  the finaliser  z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
  z *= 0x94D049BB133111EB; z ^= z>>31.
* Counter-based use: the stream key is  key = mix(seed XOR mix(stream + gamma)),
  and word i of the stream is  mix(key + (i+1)*gamma)  -- the i-th SplitMix64
  output after seeding the state with ``key``.
* Uniform: u = (word >> 11) * 2^-53 in [0, 1).
* Normal (Box and Muller, 1958): element e uses words 2e and 2e+1,
  z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2)  in fp64, rounded to fp32 (RNE) and
  then to bf16 (RNE on the bit pattern).
* Integer draws in [lo, hi]: lo + ((word >> 11) * (hi-lo+1)) >> 53, exact.

The pages' workloads draw cache contents and new q/k/v i.i.d. N(0,1) in bf16
and start positions uniform over an inclusive range; these helpers give
exactly that.  Cache rows at or beyond a sequence's start position stay zero,
as a freshly allocated cache would (the model allocates the cache with
``torch.zeros``: "Llama 3 8B · KV cache", its "storage" code excerpt).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1

# stream ids: one per tensor role; caches of layer l use 16*l + role
STREAM_Q, STREAM_K_NEW, STREAM_V_NEW, STREAM_CACHE_K, STREAM_CACHE_V = 1, 2, 3, 4, 5
STREAM_START_POS = 6

DEFAULT_SEED = 20261202


def layer_stream(role: int, layer: int = 0) -> int:
    return 16 * layer + role


def _mix_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return _mix_int((seed & _MASK) ^ _mix_int((stream + GAMMA) & _MASK))


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= np.uint64(_M1)
    z ^= z >> np.uint64(27)
    z *= np.uint64(_M2)
    z ^= z >> np.uint64(31)
    return z


def words(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """SplitMix64 words ``index`` (uint64 array) of the given stream."""
    key = np.uint64(stream_key(seed, stream))
    with np.errstate(over="ignore"):
        st = key + (index.astype(np.uint64) + np.uint64(1)) * np.uint64(GAMMA)
        return _mix_np(st)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE on the bit pattern); returns uint16."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def normal_bf16(seed: int, stream: int, offset: int, n: int) -> np.ndarray:
    """bf16 bits (uint16) of N(0,1) draws for elements offset .. offset+n-1."""
    e = np.arange(offset, offset + n, dtype=np.uint64)
    w1 = words(seed, stream, np.uint64(2) * e)
    w2 = words(seed, stream, np.uint64(2) * e + np.uint64(1))
    u1 = (w1 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    u2 = (w2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    z = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)
    return f64_to_bf16_bits(z)


def randint(seed: int, stream: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers uniform over the inclusive range [lo, hi] (exact)."""
    span = hi - lo + 1
    key = stream_key(seed, stream)
    out = np.empty(n, dtype=np.int64)
    for i in range(n):
        w = _mix_int(key + (i + 1) * GAMMA)
        out[i] = lo + (((w >> 11) * span) >> 53)
    return out


def tensor_normal(seed: int, stream: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return normal_bf16(seed, stream, 0, n).reshape(shape)


def cache_fill(seed: int, stream: int, B: int, S: int, Hkv: int, d: int,
               start_pos) -> np.ndarray:
    """Host cache [B,S,Hkv,d] (bf16 bits): rows r < start_pos[b] hold the
    N(0,1) draw of their flat element index, other rows are zero."""
    out = np.zeros((B, S, Hkv, d), dtype=np.uint16)
    row = Hkv * d
    for b in range(B):
        n = int(start_pos[b])
        if n > 0:
            off = b * S * row
            out[b, :n] = normal_bf16(seed, stream, off, n * row).reshape(n, Hkv, d)
    return out


def cache_rows(seed: int, stream: int, b: int, S: int, Hkv: int, d: int,
               r0: int, r1: int, start_pos_b: int) -> np.ndarray:
    """Rows r0..r1-1 of sequence b of a cache made by ``cache_fill``."""
    row = Hkv * d
    out = np.zeros((r1 - r0, Hkv, d), dtype=np.uint16)
    hi = min(r1, start_pos_b)
    if hi > r0:
        off = (b * S + r0) * row
        out[: hi - r0] = normal_bf16(seed, stream, off, (hi - r0) * row).reshape(hi - r0, Hkv, d)
    return out


# ---------------------------------------------------------------- device side
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkvattn_synth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the device generator (synth.cu) for sm_100a, in-tree."""
    src = os.path.join(_HERE, "synth.cu")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
               "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-o", _LIB_PATH, src]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"device generator not built: {_LIB_PATH} (run kvattn_synth.build())")
        lib = ctypes.CDLL(_LIB_PATH)
        lib.kvsynth_normal_bf16.restype = ctypes.c_int
        lib.kvsynth_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                           ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
        lib.kvsynth_cache_fill.restype = ctypes.c_int
        lib.kvsynth_cache_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


def device_normal_bf16(seed: int, stream: int, out, offset: int = 0, cuda_stream=None):
    """Fill the contiguous bf16 torch tensor ``out`` (on a GPU) in place."""
    import torch
    assert out.is_cuda and out.dtype == torch.bfloat16 and out.is_contiguous()
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream().cuda_stream
    rc = _load().kvsynth_normal_bf16(seed, stream, offset, out.numel(), out.data_ptr(), s)
    if rc != 0:
        raise RuntimeError(f"kvsynth_normal_bf16 failed ({rc})")
    return out


def device_cache_fill(seed: int, stream: int, cache, start_pos_dev, cuda_stream=None):
    """Fill the bf16 cache tensor [B,S,Hkv,d] on a GPU: rows < start_pos[b]
    get the draw of their flat index, the rest zero (same values as
    ``cache_fill``)."""
    import torch
    assert cache.is_cuda and cache.dtype == torch.bfloat16 and cache.is_contiguous()
    B, S, Hkv, d = cache.shape
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream().cuda_stream
    rc = _load().kvsynth_cache_fill(seed, stream, B, S, Hkv, d, start_pos_dev.data_ptr(),
                                    cache.data_ptr(), s)
    if rc != 0:
        raise RuntimeError(f"kvsynth_cache_fill failed ({rc})")
    return cache
