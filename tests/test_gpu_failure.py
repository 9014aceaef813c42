"""Failure detection on the GPU, without a fault: every in-kernel pipeline
wait of the library is bounded, and a wait that runs out makes the CTA set
KVATTN_DEV_WAIT_TIMEOUT, let what it already issued finish, free its tensor
memory and exit.  These tests make the waits run out through the library's
diagnostics gate, a device flag that nothing sets (kvattn_set_wait_policy),
with a 20 ms limit; no kernel is altered.  Each case then checks that the
call returned, the context still works, the status bit is set, and that the
next ordinary call (after the recovery the header prescribes) matches the fp64
oracle."""
import time

import numpy as np
import pytest

import oracle
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")

LIMIT_NS = 20_000_000  # 20 ms per wait


def _run_with_closed_gate(call):
    gate = torch.zeros(1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    kv.kvattn_set_wait_policy(LIMIT_NS, gate)
    try:
        t0 = time.perf_counter()
        call(status)
        torch.cuda.synchronize()       # the kernels ended by themselves
        took = time.perf_counter() - t0
    finally:
        kv.kvattn_set_wait_policy()
    assert int(gate.item()) == 0
    assert int(status.item()) & kv.KVATTN_DEV_WAIT_TIMEOUT, int(status.item())
    assert took < 10.0, took
    return took


def _inputs(seed, B, T, H, Hkv, S, sp):
    q, k, v, ck, cv = U.host_inputs(seed, B, T, H, Hkv, S, sp)
    dev = dict(q=U.to_dev(q), k=U.to_dev(k), v=U.to_dev(v), ck=U.to_dev(ck), cv=U.to_dev(cv),
               sp=torch.from_numpy(np.asarray(sp, np.int32)).cuda())
    return (q, k, v, ck, cv), dev


def _oracle(host, sp, rope=kv.LLAMA3):
    q, k, v, ck, cv = (x.copy() for x in host)
    _, out, rc = oracle.step(q, k, v, ck, cv, np.asarray(sp, np.int32), U.oracle_freqs(rope))
    assert rc == 0
    return out


@pytest.mark.parametrize("case", [
    # B, T, H, Hkv, S, start positions, entry
    (3, 1, 32, 8, 2000, [1999, 700, 64], "decode"),        # G = 4, CUDA-core split kernel + merge
    (4, 1, 64, 8, 3000, [2999, 5, 1000, 2500], "decode"),  # G = 8, warp-MMA kernel + merge
    (2, 1, 32, 1, 3000, [2999, 1500], "decode"),           # G = 32, tcgen05 multi-query kernel + merge
    (3, 1, 32, 8, 2000, [1999, 700, 64], "noalloc"),
    (2, 1, 32, 8, 1500, [1499, 300], "window"),
    (2, 64, 32, 8, 600, [500, 17], "prefill"),
])
def test_wait_timeout_is_reported_and_the_next_call_is_correct(case):
    B, T, H, Hkv, S, sp, entry = case
    host, d = _inputs(41, B, T, H, Hkv, S, sp)
    q_rot = kv.kvattn_rope_append(d["q"], d["k"], d["v"], d["ck"], d["cv"], d["sp"])
    ws_bytes = kv.kvattn_decode_workspace_bytes(B, H, Hkv, S)
    ws = kv.alloc_workspace(ws_bytes)

    def attend(status):
        if entry == "decode":
            return kv.kvattn_decode(q_rot, d["ck"], d["cv"], d["sp"], workspace=ws, dev_status=status)
        if entry == "noalloc":
            return kv.kvattn_decode_noalloc(q_rot, d["ck"], d["cv"], d["sp"], dev_status=status)
        if entry == "window":
            return kv.kvattn_decode(q_rot, d["ck"], d["cv"], d["sp"], dev_status=status, window=256, n_sink=4)
        return kv.kvattn_prefill_chunk(q_rot, d["ck"], d["cv"], d["sp"], dev_status=status)

    _run_with_closed_gate(attend)
    # the next ordinary call: same workspace, nothing reset (none is needed)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = attend(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    if entry == "window":
        q, k, v, ck, cv = (x.copy() for x in host)
        q_r, rc = oracle.rope_append(q, k, v, ck, cv, np.asarray(sp, np.int32), U.oracle_freqs(kv.LLAMA3))
        assert rc == 0
        ref, rc = oracle.attention(q_r, ck, cv, np.asarray(sp, np.int32), window=256, n_sink=4)
        assert rc == 0
    else:
        ref = _oracle(host, sp)
    U.assert_attention_close(U.to_host(out), ref, f"after a timeout: {case}")
    if entry == "decode" and ws_bytes > 0:
        # the merge kernel left the work counter zero despite the timeout
        assert int(ws[:4].view(torch.int32).item()) == 0


def test_fused_decode_timeout_then_rezeroed_workspace():
    B, H, Hkv, S, sp = 3, 32, 8, 2000, [1999, 700, 64]
    host, d = _inputs(42, B, 1, H, Hkv, S, sp)
    ws = kv.alloc_fused_workspace(kv.kvattn_decode_fused_workspace_bytes(B, H, Hkv, S))
    _run_with_closed_gate(lambda st: kv.kvattn_decode_fused(d["q"], d["k"], d["v"], d["ck"], d["cv"], d["sp"],
                                                           workspace=ws, dev_status=st))
    ws.zero_()   # the header's recovery rule for the fused decode
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kv.kvattn_decode_fused(d["q"], d["k"], d["v"], d["ck"], d["cv"], d["sp"], workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    U.assert_attention_close(U.to_host(out), _oracle(host, sp), "fused after a timeout")
    # every completed call leaves the counters zero: the 16-byte header (work
    # and exit counters) and one merge counter per (sequence, KV head)
    counters = ws[:16 + B * Hkv * 4].view(torch.int32)
    assert not torch.any(counters != 0)


def test_default_policy_restored():
    # with the defaults back, an ordinary call sets no status bit
    host, d = _inputs(43, 2, 1, 32, 8, 600, [599, 10])
    q_rot = kv.kvattn_rope_append(d["q"], d["k"], d["v"], d["ck"], d["cv"], d["sp"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kv.kvattn_decode(q_rot, d["ck"], d["cv"], d["sp"], dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    U.assert_attention_close(U.to_host(out), _oracle(host, [599, 10]), "defaults")
