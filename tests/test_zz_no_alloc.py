"""kvattn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a framework that owns every allocation, an engine
that reserved its HBM up front, a loop that cannot pay for cudaMalloc).  Its
split partials live in one static device array that every call reuses, so
these tests run it twice in a row on each shape and check every output
against the fp64 oracle and against kvattn_decode with a caller workspace:
bit for bit where both run the same kernels (G <= 16, and G = 64), within the
attention tolerance at G = 32, where kvattn_decode takes the tensor-core split
path and this entry point the warp-MMA kernel over two 16-head groups.

This file is collected last on purpose: it runs after the rest of the GPU
suite, and it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest

import oracle
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")


def _case(seed, B, H, Hkv, S, sp):
    q, _, _, ck, cv = U.host_inputs(seed, B, 1, H, Hkv, S, sp)
    dev = (U.to_dev(q), U.to_dev(ck), U.to_dev(cv), torch.from_numpy(np.asarray(sp, np.int32)).cuda())
    return (q, ck, cv), dev


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


CASES = [
    # seed, B, H, Hkv, S, start positions, hint
    (31, 4, 32, 8, 6000, [5999, 1234, 64, 4500], 0),          # G = 4, many splits per sequence
    (32, 6, 64, 8, 3000, [2999, 17, 1500, 800, 2048, 1], 0),  # G = 8, warp-MMA kernel
    (33, 3, 32, 1, 5000, [4999, 2100, 130], 0),               # G = 32 (multi-query), split
    (34, 2, 64, 1, 2000, [1999, 700], 0),                     # G = 64: four 16-head groups
    (35, 5, 16, 16, 900, [899, 0, 31, 32, 450], 0),           # G = 1 (MHA)
]


@pytest.mark.parametrize("case", CASES)
def test_noalloc_matches_oracle_and_decode_on_two_calls_in_a_row(case):
    seed, B, H, Hkv, S, sp, hint = case
    (q, ck, cv), (dq, dck, dcv, dsp) = _case(seed, B, H, Hkv, S, sp)
    ref_o, rc = oracle.attention(q, ck, cv, np.asarray(sp, np.int32))
    assert rc == 0
    dec = kv.kvattn_decode(dq, dck, dcv, dsp, max_kv_len_hint=hint)
    outs = []
    for _ in range(2):
        out = torch.full_like(dec, 5.0)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _noalloc_raw(dq, dck, dcv, dsp, hint, out, status)
        torch.cuda.synchronize()
        assert rc == 0
        assert int(status.item()) == 0
        outs.append(U.to_host(out))
    g_dec = U.to_host(dec)
    U.assert_attention_close(g_dec, ref_o, f"kvattn_decode {case}")
    for o in outs:
        U.assert_attention_close(o, ref_o, f"kvattn_decode_noalloc {case}")
    # the two calls in a row through the shared static array agree bit for bit
    assert np.array_equal(outs[0], outs[1])
    if H // Hkv != 32:
        # the same kernels as kvattn_decode: the same bits
        assert np.array_equal(outs[0], g_dec)


def test_noalloc_binding_and_size_limit():
    (q, ck, cv), (dq, dck, dcv, dsp) = _case(36, 2, 32, 8, 512, [300, 511])
    ref_o, rc = oracle.attention(q, ck, cv, np.array([300, 511], np.int32))
    assert rc == 0
    ref = kv.kvattn_decode(dq, dck, dcv, dsp)
    got = kv.kvattn_decode_noalloc(dq, dck, dcv, dsp)
    got2 = kv.kvattn_decode_noalloc(dq, dck, dcv, dsp)
    torch.cuda.synchronize()
    for g in (got, got2):
        U.assert_attention_close(U.to_host(g), ref_o, "binding")
        assert np.array_equal(U.to_host(g), U.to_host(ref))
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
