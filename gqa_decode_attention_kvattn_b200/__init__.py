"""Thin Python binding of libkvattn.so (cached GQA attention on B200).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  The function names are those of
the C ABI declared in ``include/kvattn.h``, which states each call's contract.

If the compiled library is missing the import of this package still works,
but every call raises ``KvattnLibraryMissing``: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvattn.so")

KVATTN_OK = 0
KVATTN_ERR_INVALID_ARG = 1
KVATTN_ERR_UNSUPPORTED = 2
KVATTN_ERR_OUT_OF_RANGE = 3
KVATTN_ERR_WORKSPACE = 4
KVATTN_ERR_CUDA = 5

KVATTN_DEV_START_POS_RANGE = 0x1
KVATTN_DEV_KV_LEN_HINT = 0x2
KVATTN_DEV_WAIT_TIMEOUT = 0x4
KVATTN_DEV_INTERNAL = 0x8

HEAD_DIM = 128


class KvattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class KvattnLibraryMissing(RuntimeError):
    pass


class kvattn_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_seq_len", ctypes.c_int32)]


class kvattn_attn_mask(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int32), ("n_sink", ctypes.c_int32), ("sink_logits", ctypes.c_void_p)]


class kvattn_rope_params(ctypes.Structure):
    _fields_ = [("theta", ctypes.c_double), ("use_scaled", ctypes.c_int32), ("factor", ctypes.c_double),
                ("low_freq_factor", ctypes.c_double), ("high_freq_factor", ctypes.c_double),
                ("original_max_pos", ctypes.c_double), ("layout", ctypes.c_int32), ("rotary_dim", ctypes.c_int32)]


KVATTN_ROPE_INTERLEAVED = 0
KVATTN_ROPE_HALF_SPLIT = 1


@dataclass(frozen=True)
class RopeParams:
    """RoPE settings: theta and the optional Llama-3.1 frequency scaling."""
    theta: float = 500000.0
    use_scaled: bool = False
    factor: float = 8.0
    low_freq_factor: float = 1.0
    high_freq_factor: float = 4.0
    original_max_pos: float = 8192.0
    layout: int = KVATTN_ROPE_INTERLEAVED   # or KVATTN_ROPE_HALF_SPLIT
    rotary_dim: int = 0                     # 0: the whole head

    def as_c(self) -> kvattn_rope_params:
        return kvattn_rope_params(self.theta, int(self.use_scaled), self.factor, self.low_freq_factor,
                                  self.high_freq_factor, self.original_max_pos, int(self.layout),
                                  int(self.rotary_dim))


LLAMA3 = RopeParams()                     # rope_theta 500000, use_scaled_rope False
LLAMA3_1 = RopeParams(use_scaled=True)    # rope_theta 500000, use_scaled_rope True

_lib = None

_SYMBOLS = ("kvattn_rope_append", "kvattn_decode_workspace_bytes", "kvattn_decode",
            "kvattn_prefill_workspace_bytes", "kvattn_prefill_chunk", "kvattn_status_string",
            "kvattn_version")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise KvattnLibraryMissing(
            f"{LIB_PATH} is not built; run `python -m gqa_decode_attention_kvattn_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    dims_p = ctypes.POINTER(kvattn_dims)
    rope_p = ctypes.POINTER(kvattn_rope_params)
    lib.kvattn_rope_append.restype = ctypes.c_int
    lib.kvattn_rope_append.argtypes = [dims_p, rope_p, ctypes.c_int32, P, P, P, P, P, P, P, P, P]
    lib.kvattn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.kvattn_decode_workspace_bytes.argtypes = [dims_p, ctypes.c_int32]
    lib.kvattn_decode.restype = ctypes.c_int
    lib.kvattn_decode.argtypes = [dims_p, P, P, P, P, ctypes.c_int32, ctypes.c_float, P, P, ctypes.c_size_t, P, P]
    lib.kvattn_decode_fused_workspace_bytes.restype = ctypes.c_size_t
    lib.kvattn_decode_fused_workspace_bytes.argtypes = [dims_p, ctypes.c_int32]
    lib.kvattn_decode_fused.restype = ctypes.c_int
    lib.kvattn_decode_fused.argtypes = [dims_p, rope_p, P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_float, P, P,
                                        ctypes.c_size_t, P, P]
    mask_p = ctypes.POINTER(kvattn_attn_mask)
    lib.kvattn_decode_masked_workspace_bytes.restype = ctypes.c_size_t
    lib.kvattn_decode_masked_workspace_bytes.argtypes = [dims_p, ctypes.c_int32, mask_p]
    lib.kvattn_decode_masked.restype = ctypes.c_int
    lib.kvattn_decode_masked.argtypes = [dims_p, P, P, P, P, ctypes.c_int32, ctypes.c_float, mask_p, P, P,
                                         ctypes.c_size_t, P, P]
    lib.kvattn_prefill_chunk_masked.restype = ctypes.c_int
    lib.kvattn_prefill_chunk_masked.argtypes = [dims_p, ctypes.c_int32, P, P, P, P, ctypes.c_int32, ctypes.c_float,
                                                mask_p, P, P, ctypes.c_size_t, P, P]
    lib.kvattn_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.kvattn_prefill_workspace_bytes.argtypes = [dims_p, ctypes.c_int32, ctypes.c_int32]
    lib.kvattn_prefill_chunk.restype = ctypes.c_int
    lib.kvattn_prefill_chunk.argtypes = [dims_p, ctypes.c_int32, P, P, P, P, ctypes.c_int32, ctypes.c_float, P, P,
                                         ctypes.c_size_t, P, P]
    lib.kvattn_status_string.restype = ctypes.c_char_p
    lib.kvattn_status_string.argtypes = [ctypes.c_int]
    lib.kvattn_last_cuda_error.restype = ctypes.c_int
    lib.kvattn_last_cuda_error.argtypes = []
    lib.kvattn_last_cuda_error_string.restype = ctypes.c_char_p
    lib.kvattn_last_cuda_error_string.argtypes = []
    lib.kvattn_version.restype = ctypes.c_int
    lib.kvattn_version.argtypes = []
    lib.kvattn_set_wait_policy.restype = ctypes.c_int
    lib.kvattn_set_wait_policy.argtypes = [ctypes.c_uint64, P]
    _lib = lib
    return lib


def library():
    """The loaded ctypes library (raises if it is not built)."""
    return _load()


def status_string(status: int) -> str:
    try:
        return _load().kvattn_status_string(int(status)).decode()
    except KvattnLibraryMissing:
        return f"status {status}"


def kvattn_version() -> int:
    return int(_load().kvattn_version())


def kvattn_status_string(status: int) -> str:
    return _load().kvattn_status_string(int(status)).decode()


def kvattn_set_wait_policy(limit_ns: int = 0, gate=None) -> None:
    """Limit of every in-kernel pipeline wait for later launches (0: one
    second) and an optional gate (a one-element int32 CUDA tensor) that the
    pipelined kernels wait on before issuing any copy; a gate that stays zero
    makes them give up after the limit and set KVATTN_DEV_WAIT_TIMEOUT (see
    include/kvattn.h).  kvattn_set_wait_policy() restores the defaults."""
    if gate is not None:
        import torch
        if gate.dtype != torch.int32 or not gate.is_cuda or gate.numel() < 1:
            raise ValueError("gate must be an int32 CUDA tensor")
    _check_status(_load().kvattn_set_wait_policy(int(limit_ns), _ptr(gate)), "kvattn_set_wait_policy")


# ------------------------------------------------------------------ helpers
def make_dims(batch: int, n_heads: int, n_kv_heads: int, max_seq_len: int, head_dim: int = HEAD_DIM):
    return kvattn_dims(batch, n_heads, n_kv_heads, head_dim, max_seq_len)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check_bf16(name, t, ndim):
    import torch
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == ndim):
        raise ValueError(f"{name} must be a contiguous {ndim}-D bf16 CUDA tensor, got "
                         f"{tuple(t.shape)} {t.dtype} on {t.device}")


def _check_status(rc: int, where: str):
    if rc != KVATTN_OK:
        if rc == KVATTN_ERR_CUDA:
            lib = _load()
            where = f"{where} [cuda error {lib.kvattn_last_cuda_error()}: {lib.kvattn_last_cuda_error_string().decode()}]"
        raise KvattnError(rc, where)


def _dims_from_cache(q, cache_k):
    B, _, H, d = q.shape
    _, S, Hkv, _ = cache_k.shape
    return kvattn_dims(B, H, Hkv, d, S)


# ------------------------------------------------------------------ C-ABI calls
def kvattn_rope_append(q, k_new, v_new, cache_k, cache_v, start_pos, rope: RopeParams = LLAMA3,
                       q_rot=None, dev_status=None, stream=None):
    """RoPE at positions start_pos[b]+t and cache append (see include/kvattn.h).

    q [B,T,H,d], k_new/v_new [B,T,Hkv,d], caches [B,S,Hkv,d] bf16 CUDA tensors;
    start_pos int32 [B] CUDA tensor.  Returns q_rot (a new tensor unless given;
    pass q_rot=q to rotate in place).  The caches are updated in place.
    """
    import torch
    lib = _load()
    _check_bf16("q", q, 4)
    _check_bf16("k_new", k_new, 4)
    _check_bf16("v_new", v_new, 4)
    _check_bf16("cache_k", cache_k, 4)
    _check_bf16("cache_v", cache_v, 4)
    if start_pos.dtype != torch.int32 or not start_pos.is_cuda:
        raise ValueError("start_pos must be an int32 CUDA tensor")
    if q_rot is None:
        q_rot = torch.empty_like(q)
    T = q.shape[1]
    dims = _dims_from_cache(q, cache_k)
    rope_c = rope.as_c()
    rc = lib.kvattn_rope_append(ctypes.byref(dims), ctypes.byref(rope_c), T, _ptr(q), _ptr(q_rot), _ptr(k_new),
                                _ptr(v_new), _ptr(cache_k), _ptr(cache_v), _ptr(start_pos), _ptr(dev_status),
                                _stream(stream))
    _check_status(rc, "kvattn_rope_append")
    return q_rot


def kvattn_decode_workspace_bytes(batch, n_heads, n_kv_heads, max_seq_len, max_kv_len_hint=0,
                                  head_dim=HEAD_DIM) -> int:
    dims = kvattn_dims(batch, n_heads, n_kv_heads, head_dim, max_seq_len)
    return int(_load().kvattn_decode_workspace_bytes(ctypes.byref(dims), int(max_kv_len_hint)))


def kvattn_decode_plan(batch, n_heads, n_kv_heads, max_seq_len, max_kv_len_hint=0, head_dim=HEAD_DIM) -> dict:
    """Split size, splits, persistent grid and CTAs per SM kvattn_decode
    will use on the current device."""
    lib = _load()
    fn = lib.kvattn_decode_plan
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(kvattn_dims), ctypes.c_int32] + [ctypes.POINTER(ctypes.c_int32)] * 5
    dims = kvattn_dims(batch, n_heads, n_kv_heads, head_dim, max_seq_len)
    out = [ctypes.c_int32() for _ in range(5)]
    rc = fn(ctypes.byref(dims), int(max_kv_len_hint), *[ctypes.byref(o) for o in out])
    _check_status(rc, "kvattn_decode_plan")
    return dict(rows_per_split=out[0].value, max_splits=out[1].value, grid=out[2].value,
                ctas_per_sm=out[3].value, tensor_cores=bool(out[4].value))


def kvattn_prefill_workspace_bytes(batch, n_heads, n_kv_heads, max_seq_len, T, max_kv_len_hint=0,
                                   head_dim=HEAD_DIM) -> int:
    dims = kvattn_dims(batch, n_heads, n_kv_heads, head_dim, max_seq_len)
    return int(_load().kvattn_prefill_workspace_bytes(ctypes.byref(dims), int(T), int(max_kv_len_hint)))


def alloc_workspace(nbytes: int, device=None):
    """A zeroed decode workspace (its work counter must start at zero; every
    completed call leaves it zero)."""
    import torch
    return torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device or "cuda")


def _mask(window, n_sink, sink_logits):
    """kvattn_attn_mask for the optional masks, or None when none is set.
    sink_logits: a float32 CUDA tensor [H] (learned sink logits)."""
    if window <= 0 and sink_logits is None:
        return None
    if sink_logits is not None:
        import torch
        if sink_logits.dtype != torch.float32 or not sink_logits.is_cuda or not sink_logits.is_contiguous():
            raise ValueError("sink_logits must be a contiguous float32 CUDA tensor [H]")
    return kvattn_attn_mask(int(max(window, 0)), int(n_sink), None if sink_logits is None else sink_logits.data_ptr())


def kvattn_decode(q_rot, cache_k, cache_v, start_pos, max_kv_len_hint: int = 0, scale: float = 0.0,
                  out=None, workspace=None, dev_status=None, stream=None, window: int = 0, n_sink: int = 0,
                  sink_logits=None):
    """Split-K GQA decode for one new token per sequence (see include/kvattn.h).

    q_rot [B,1,H,d]; returns out [B,1,H,d] bf16.  A workspace is allocated
    with torch when none is given.  window / n_sink / sink_logits select the
    masked entry point (sliding window, attention sinks, learned sinks)."""
    mask = _mask(window, n_sink, sink_logits)
    if mask is not None:
        return _decode_masked(q_rot, cache_k, cache_v, start_pos, max_kv_len_hint, scale, mask, out, workspace,
                              dev_status, stream)
    import torch
    lib = _load()
    _check_bf16("q_rot", q_rot, 4)
    _check_bf16("cache_k", cache_k, 4)
    _check_bf16("cache_v", cache_v, 4)
    if q_rot.shape[1] != 1:
        raise ValueError("kvattn_decode takes one token per sequence (q_rot [B,1,H,d])")
    dims = _dims_from_cache(q_rot, cache_k)
    if out is None:
        out = torch.empty_like(q_rot)
    ws_bytes = int(lib.kvattn_decode_workspace_bytes(ctypes.byref(dims), int(max_kv_len_hint)))
    if workspace is None and ws_bytes > 0:
        workspace = alloc_workspace(ws_bytes, q_rot.device)
    ws_size = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.kvattn_decode(ctypes.byref(dims), _ptr(q_rot), _ptr(cache_k), _ptr(cache_v), _ptr(start_pos),
                           int(max_kv_len_hint), float(scale), _ptr(out), _ptr(workspace), ws_size,
                           _ptr(dev_status), _stream(stream))
    _check_status(rc, "kvattn_decode")
    return out


def kvattn_decode_fused_workspace_bytes(batch, n_heads, n_kv_heads, max_seq_len, max_kv_len_hint=0,
                                        head_dim=HEAD_DIM) -> int:
    dims = kvattn_dims(batch, n_heads, n_kv_heads, head_dim, max_seq_len)
    return int(_load().kvattn_decode_fused_workspace_bytes(ctypes.byref(dims), int(max_kv_len_hint)))


def alloc_fused_workspace(nbytes: int, device=None):
    """A zeroed workspace for kvattn_decode_fused (its counters start at 0
    and every completed call leaves them at 0)."""
    import torch
    return torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device or "cuda")


def kvattn_decode_fused(q, k_new, v_new, cache_k, cache_v, start_pos, rope: RopeParams = LLAMA3,
                        max_kv_len_hint: int = 0, scale: float = 0.0, out=None, q_rot=None, workspace=None,
                        dev_status=None, stream=None):
    """RoPE + cache append + split-K decode + merge in one launch (see
    include/kvattn.h).  q [B,1,H,d], k_new/v_new [B,1,Hkv,d]; the caches are
    updated in place; returns out [B,1,H,d].  q_rot (optional, not q)
    receives the rotated q.  A zeroed workspace is allocated when none is
    given; a caller-owned one must be zeroed once before its first use."""
    import torch
    lib = _load()
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("cache_k", cache_k), ("cache_v", cache_v)):
        _check_bf16(name, t, 4)
    if q.shape[1] != 1:
        raise ValueError("kvattn_decode_fused takes one token per sequence (q [B,1,H,d])")
    if start_pos.dtype != torch.int32 or not start_pos.is_cuda:
        raise ValueError("start_pos must be an int32 CUDA tensor")
    dims = _dims_from_cache(q, cache_k)
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = int(lib.kvattn_decode_fused_workspace_bytes(ctypes.byref(dims), int(max_kv_len_hint)))
    if workspace is None and ws_bytes > 0:
        workspace = alloc_fused_workspace(ws_bytes, q.device)
    ws_size = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rope_c = rope.as_c()
    rc = lib.kvattn_decode_fused(ctypes.byref(dims), ctypes.byref(rope_c), _ptr(q), _ptr(q_rot), _ptr(k_new),
                                 _ptr(v_new), _ptr(cache_k), _ptr(cache_v), _ptr(start_pos), int(max_kv_len_hint),
                                 float(scale), _ptr(out), _ptr(workspace), ws_size, _ptr(dev_status),
                                 _stream(stream))
    _check_status(rc, "kvattn_decode_fused")
    return out


def _decode_masked(q_rot, cache_k, cache_v, start_pos, max_kv_len_hint, scale, mask, out, workspace, dev_status,
                   stream):
    import torch
    lib = _load()
    _check_bf16("q_rot", q_rot, 4)
    _check_bf16("cache_k", cache_k, 4)
    _check_bf16("cache_v", cache_v, 4)
    if q_rot.shape[1] != 1:
        raise ValueError("kvattn_decode takes one token per sequence (q_rot [B,1,H,d])")
    dims = _dims_from_cache(q_rot, cache_k)
    if out is None:
        out = torch.empty_like(q_rot)
    ws_bytes = int(lib.kvattn_decode_masked_workspace_bytes(ctypes.byref(dims), int(max_kv_len_hint),
                                                            ctypes.byref(mask)))
    if workspace is None and ws_bytes > 0:
        workspace = alloc_workspace(ws_bytes, q_rot.device)
    ws_size = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.kvattn_decode_masked(ctypes.byref(dims), _ptr(q_rot), _ptr(cache_k), _ptr(cache_v), _ptr(start_pos),
                                  int(max_kv_len_hint), float(scale), ctypes.byref(mask), _ptr(out),
                                  _ptr(workspace), ws_size, _ptr(dev_status), _stream(stream))
    _check_status(rc, "kvattn_decode_masked")
    return out


def kvattn_decode_masked_workspace_bytes(batch, n_heads, n_kv_heads, max_seq_len, max_kv_len_hint=0, window=0,
                                         n_sink=0, head_dim=HEAD_DIM) -> int:
    dims = kvattn_dims(batch, n_heads, n_kv_heads, head_dim, max_seq_len)
    mask = kvattn_attn_mask(int(window), int(n_sink), None)
    return int(_load().kvattn_decode_masked_workspace_bytes(ctypes.byref(dims), int(max_kv_len_hint),
                                                            ctypes.byref(mask)))


def kvattn_prefill_chunk(q_rot, cache_k, cache_v, start_pos, max_kv_len_hint: int = 0, scale: float = 0.0,
                         out=None, workspace=None, dev_status=None, stream=None, window: int = 0, n_sink: int = 0,
                         sink_logits=None):
    """Chunked-prefill attention with the rectangular causal mask (see
    include/kvattn.h).  q_rot [B,T,H,d]; returns out [B,T,H,d] bf16.
    window / n_sink / sink_logits select the masked entry point."""
    import torch
    lib = _load()
    mask = _mask(window, n_sink, sink_logits)
    _check_bf16("q_rot", q_rot, 4)
    _check_bf16("cache_k", cache_k, 4)
    _check_bf16("cache_v", cache_v, 4)
    T = q_rot.shape[1]
    dims = _dims_from_cache(q_rot, cache_k)
    if out is None:
        out = torch.empty_like(q_rot)
    ws_bytes = int(lib.kvattn_prefill_workspace_bytes(ctypes.byref(dims), T, int(max_kv_len_hint)))
    if workspace is None and ws_bytes > 0:
        workspace = alloc_workspace(ws_bytes, q_rot.device)
    ws_size = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if mask is not None:
        rc = lib.kvattn_prefill_chunk_masked(ctypes.byref(dims), T, _ptr(q_rot), _ptr(cache_k), _ptr(cache_v),
                                             _ptr(start_pos), int(max_kv_len_hint), float(scale), ctypes.byref(mask),
                                             _ptr(out), _ptr(workspace), ws_size, _ptr(dev_status), _stream(stream))
    else:
        rc = lib.kvattn_prefill_chunk(ctypes.byref(dims), T, _ptr(q_rot), _ptr(cache_k), _ptr(cache_v),
                                      _ptr(start_pos), int(max_kv_len_hint), float(scale), _ptr(out),
                                      _ptr(workspace), ws_size, _ptr(dev_status), _stream(stream))
    _check_status(rc, "kvattn_prefill_chunk")
    return out


# ------------------------------------------------------------ byte arithmetic
def kv_cache_bytes(n_layers: int, n_kv_heads: int, head_dim: int, tokens: int, bytes_per_elem: int = 2) -> int:
    """Bytes a KV cache holds: a key and a value per layer, KV head and channel
    for every token ("Grouped-query attention: a smaller KV cache", 8:52 and
    14:57; "Llama 3 8B · KV cache": 1 GiB per sequence at 8192 positions)."""
    return 2 * n_layers * n_kv_heads * head_dim * bytes_per_elem * tokens


def attention_kv_bytes(start_pos, T: int, n_kv_heads: int, head_dim: int = HEAD_DIM, bytes_per_elem: int = 2) -> int:
    """Algorithmic K+V bytes one attention call must read: rows
    0..start_pos[b]+T-1 of every KV head of every sequence, once."""
    rows = sum(int(s) + T for s in start_pos)
    return kv_cache_bytes(1, n_kv_heads, head_dim, rows, bytes_per_elem)


def prefill_flops(start_pos, T: int, n_heads: int, head_dim: int = HEAD_DIM) -> int:
    """Algorithmic flops of chunked-prefill attention: 2 flops per multiply-add
    of q.K and of P.V over the visible rows, i.e. 4*d*H*sum_b sum_t (sp+t+1)."""
    vis = sum(T * (int(s) + 1) + T * (T - 1) // 2 for s in start_pos)
    return 4 * head_dim * n_heads * vis


def default_scale(head_dim: int = HEAD_DIM) -> float:
    return 1.0 / math.sqrt(head_dim)


# ------------------------------------------------- allocation-free decode
_noalloc = None


def _load_noalloc():
    """ctypes handle of kvattn_decode_noalloc (argument types set once)."""
    global _noalloc
    if _noalloc is None:
        lib = _load()
        P = ctypes.c_void_p
        fn = lib.kvattn_decode_noalloc
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.POINTER(kvattn_dims), P, P, P, P, ctypes.c_int32, ctypes.c_float, P, P, P]
        lib.kvattn_decode_noalloc_scratch_bytes.restype = ctypes.c_size_t
        lib.kvattn_decode_noalloc_scratch_bytes.argtypes = []
        _noalloc = fn
    return _noalloc


def kvattn_decode_noalloc_scratch_bytes() -> int:
    _load_noalloc()
    return int(_load().kvattn_decode_noalloc_scratch_bytes())


def kvattn_decode_noalloc(q_rot, cache_k, cache_v, start_pos, max_kv_len_hint: int = 0, scale: float = 0.0,
                          out=None, dev_status=None, stream=None):
    """kvattn_decode without a workspace: for callers that cannot allocate
    device memory on the decode path (the library keeps one static 64 MiB
    array per GPU for the split partials instead).  Calls that overlap on the
    GPU share that array and race; the first call on a device looks up its
    address and should come before any stream capture.  Only ``out`` is
    allocated here, and only when it is not given."""
    import torch
    fn = _load_noalloc()
    _check_bf16("q_rot", q_rot, 4)
    _check_bf16("cache_k", cache_k, 4)
    _check_bf16("cache_v", cache_v, 4)
    if q_rot.shape[1] != 1:
        raise ValueError("kvattn_decode_noalloc takes one token per sequence (q_rot [B,1,H,d])")
    dims = _dims_from_cache(q_rot, cache_k)
    if out is None:
        out = torch.empty_like(q_rot)
    rc = fn(ctypes.byref(dims), _ptr(q_rot), _ptr(cache_k), _ptr(cache_v), _ptr(start_pos), int(max_kv_len_hint),
            float(scale), _ptr(out), _ptr(dev_status), _stream(stream))
    _check_status(rc, "kvattn_decode_noalloc")
    return out
