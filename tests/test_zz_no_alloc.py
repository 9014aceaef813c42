"""kvattn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a framework that owns every allocation, an engine
that reserved its HBM up front, a loop that cannot pay for cudaMalloc).  It
must give the same output as kvattn_decode with a caller workspace, call
after call, although every call reuses the same static device array.

This file is collected last on purpose: it runs after the rest of the GPU
suite, and it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest

import kvattn_synth as ks
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")


def _case(seed, B, H, Hkv, S, sp):
    q, _, _, ck, cv = U.host_inputs(seed, B, 1, H, Hkv, S, sp)
    return U.to_dev(q), U.to_dev(ck), U.to_dev(cv), torch.from_numpy(np.asarray(sp, np.int32)).cuda()


def _noalloc_raw(q, ck, cv, dsp, hint, out, status):
    """Call the C ABI symbol directly through ctypes."""
    lib = kv.library()
    fn = lib.kvattn_decode_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(kv.kvattn_dims)] + [ctypes.c_void_p] * 4 + \
        [ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    dims = kv.kvattn_dims(q.shape[0], q.shape[2], ck.shape[2], 128, ck.shape[1])
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.byref(dims), q.data_ptr(), ck.data_ptr(), cv.data_ptr(), dsp.data_ptr(), hint, 0.0,
              out.data_ptr(), status.data_ptr(), s)


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    cases = [
        # many splits per sequence, then a different shape and group size
        (31, 4, 32, 8, 6000, [5999, 1234, 64, 4500], 0),
        (32, 6, 64, 8, 3000, [2999, 17, 1500, 800, 2048, 1], 0),
    ]
    for seed, B, H, Hkv, S, sp, hint in cases:
        q, ck, cv, dsp = _case(seed, B, H, Hkv, S, sp)
        ref = kv.kvattn_decode(q, ck, cv, dsp, max_kv_len_hint=hint)
        out = torch.full_like(ref, 5.0)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _noalloc_raw(q, ck, cv, dsp, hint, out, status)
        torch.cuda.synchronize()
        assert rc == 0
        assert int(status.item()) == 0
        a = ks.bf16_bits_to_f64(U.to_host(out))
        b = ks.bf16_bits_to_f64(U.to_host(ref))
        err = np.abs(a - b)
        assert err.max() <= U.MAX_ABS and err.mean() <= U.MEAN_ABS


def test_noalloc_binding_and_size_limit():
    q, ck, cv, dsp = _case(33, 2, 32, 8, 512, [300, 511])
    ref = kv.kvattn_decode(q, ck, cv, dsp)
    got = kv.kvattn_decode_noalloc(q, ck, cv, dsp)
    got2 = kv.kvattn_decode_noalloc(q, ck, cv, dsp)
    torch.cuda.synchronize()
    for g in (got, got2):
        err = np.abs(ks.bf16_bits_to_f64(U.to_host(g)) - ks.bf16_bits_to_f64(U.to_host(ref)))
        assert err.max() <= U.MAX_ABS and err.mean() <= U.MEAN_ABS
    assert kv.kvattn_decode_noalloc_scratch_bytes() == 64 << 20
    # a shape whose partials exceed the static array is refused up front,
    # before anything is launched (the pointers are never touched)
    B, H, Hkv, S = 256, 64, 8, 131072
    big = kv.kvattn_decode_workspace_bytes(B, H, Hkv, S, S)
    assert big > kv.kvattn_decode_noalloc_scratch_bytes()
    dims = kv.kvattn_dims(B, H, Hkv, 128, S)
    fake = ctypes.c_void_p(0x10000)
    fn = kv.library().kvattn_decode_noalloc
    rc = fn(ctypes.byref(dims), fake, fake, fake, fake, S, 0.0, fake, None, None)
    assert rc == kv.KVATTN_ERR_WORKSPACE
