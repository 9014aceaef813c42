"""GPU parity of the fused decode step (rope + append + split-K attention +
merge in one launch): against the fp64 oracle, against the unfused calls bit
for bit, and its self-resetting workspace, error flags and graph replay."""
import numpy as np
import pytest

import kvattn_synth as ks
import oracle
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")


def _fused(q, k, v, ck, cv, sp, rope, hint=0, workspace=None, want_qrot=True):
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
    dsp = torch.from_numpy(np.asarray(sp, np.int32)).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_rot = torch.empty_like(dq) if want_qrot else None
    out = kv.kvattn_decode_fused(dq, dk, dv, dck, dcv, dsp, rope=rope, max_kv_len_hint=hint, q_rot=q_rot,
                                 workspace=workspace, dev_status=st)
    torch.cuda.synchronize()
    return (U.to_host(q_rot) if want_qrot else None, U.to_host(dck), U.to_host(dcv), U.to_host(out),
            int(st.item()))


def _unfused(q, k, v, ck, cv, sp, rope, hint=0):
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
    dsp = torch.from_numpy(np.asarray(sp, np.int32)).cuda()
    q_rot = kv.kvattn_rope_append(dq, dk, dv, dck, dcv, dsp, rope=rope)
    out = kv.kvattn_decode(q_rot, dck, dcv, dsp, max_kv_len_hint=hint)
    torch.cuda.synchronize()
    return U.to_host(q_rot), U.to_host(dck), U.to_host(dcv), U.to_host(out)


CASES = [
    # B, H, Hkv, S, sp, rope, hint
    (3, 32, 8, 64, [0, 17, 63], kv.LLAMA3, 0),
    (4, 32, 8, 4096, [1499, 700, 64, 1000], kv.LLAMA3, 0),          # several splits
    (4, 32, 8, 4096, [1499, 700, 64, 1000], kv.LLAMA3_1, 1500),     # another split size
    (2, 32, 8, 20000, [19999, 12345], kv.LLAMA3_1, 0),              # many splits
    (4, 16, 16, 1030, [63, 64, 65, 1029], kv.LLAMA3, 0),            # G = 1
    (3, 16, 8, 900, [0, 95, 857], kv.LLAMA3, 0),                    # G = 2
    (5, 64, 8, 2100, [1, 127, 128, 2047, 2099], kv.LLAMA3, 0),      # G = 8 (tensor cores)
    (3, 32, 2, 3000, [0, 63, 2999], kv.LLAMA3, 0),                  # G = 16 (tensor cores)
    (3, 32, 1, 2500, [0, 1000, 2499], kv.LLAMA3, 0),                # G = 32 (MQA): two groups per KV head
    (2, 32, 8, 3000, [2999, 600], kv.RopeParams(layout=1), 0),      # half-split pairs
    (2, 32, 8, 3000, [2999, 600], kv.RopeParams(rotary_dim=64, use_scaled=True), 0),  # partial rotary
]


@pytest.mark.parametrize("case", CASES)
def test_fused_matches_oracle(case):
    B, H, Hkv, S, sp, rope, hint = case
    q, k, v, ck, cv = U.host_inputs(41, B, 1, H, Hkv, S, sp)
    g_qrot, g_ck, g_cv, g_out, st = _fused(q, k, v, ck, cv, sp, rope, hint)
    assert st == 0
    o_ck, o_cv = ck.copy(), cv.copy()
    q_rot, out, rc = oracle.step(q, k, v, o_ck, o_cv, np.asarray(sp, np.int32), U.oracle_freqs(rope),
                                 layout=rope.layout, rotary_dim=rope.rotary_dim)
    assert rc == 0
    assert U.ulp_distance(g_qrot, q_rot).max() <= 1
    assert U.ulp_distance(g_ck, o_ck).max() <= 1
    assert np.array_equal(g_cv, o_cv)
    for b in range(B):  # only row sp[b] of each sequence changes
        keep = np.ones(S, bool)
        keep[sp[b]] = False
        assert np.array_equal(g_ck[b, keep], ck[b, keep])
        assert np.array_equal(g_cv[b, keep], cv[b, keep])
    U.assert_attention_close(g_out, out, f"fused B={B} H={H}/{Hkv} sp={sp}")


@pytest.mark.parametrize("case", [CASES[1], CASES[3], CASES[6], CASES[7], CASES[9]])
def test_fused_equals_unfused_bitwise(case):
    """Same rotation, same tiles, same merge order: identical bits."""
    B, H, Hkv, S, sp, rope, hint = case
    q, k, v, ck, cv = U.host_inputs(43, B, 1, H, Hkv, S, sp)
    f = _fused(q, k, v, ck, cv, sp, rope, hint)
    u = _unfused(q, k, v, ck, cv, sp, rope, hint)
    assert f[4] == 0
    for a, b, name in zip(f[:4], u, ("q_rot", "cache_k", "cache_v", "out")):
        assert np.array_equal(a, b), name


def test_fused_and_unfused_agree_at_g32():
    """At G = 32 the unfused decode of a multi-split call runs on the tcgen05
    kernel (another summation order than the fused warp-MMA kernel): the
    rotation and the cache writes are bit-identical, and both outputs match
    the oracle within the attention tolerance."""
    B, H, Hkv, S, sp, rope, hint = CASES[8]
    q, k, v, ck, cv = U.host_inputs(43, B, 1, H, Hkv, S, sp)
    f = _fused(q, k, v, ck, cv, sp, rope, hint)
    u = _unfused(q, k, v, ck, cv, sp, rope, hint)
    assert f[4] == 0
    for a, b, name in zip(f[:3], u[:3], ("q_rot", "cache_k", "cache_v")):
        assert np.array_equal(a, b), name
    o_ck, o_cv = ck.copy(), cv.copy()
    _, out, rc = oracle.step(q, k, v, o_ck, o_cv, np.asarray(sp, np.int32), U.oracle_freqs(rope),
                             layout=rope.layout, rotary_dim=rope.rotary_dim)
    assert rc == 0
    U.assert_attention_close(f[3], out, "fused G=32")
    U.assert_attention_close(u[3], out, "unfused G=32")


def test_fused_workspace_resets_and_consecutive_steps():
    """Two decode steps in a row on one workspace: the counters are zero
    after each call and the second step (position sp + 1) is right."""
    B, H, Hkv, S = 4, 32, 8, 4096
    sp = np.array([3000, 1499, 64, 2047], np.int32)
    q, k, v, ck, cv = U.host_inputs(44, B, 1, H, Hkv, S, sp)
    q2 = ks.tensor_normal(45, ks.STREAM_Q, (B, 1, H, 128))
    k2 = ks.tensor_normal(45, ks.STREAM_K_NEW, (B, 1, Hkv, 128))
    v2 = ks.tensor_normal(45, ks.STREAM_V_NEW, (B, 1, Hkv, 128))
    nbytes = kv.kvattn_decode_fused_workspace_bytes(B, H, Hkv, S)
    plan = kv.kvattn_decode_plan(B, H, Hkv, S)
    assert plan["max_splits"] > 1 and nbytes > 0
    ws = kv.alloc_fused_workspace(nbytes)
    dck, dcv = U.to_dev(ck), U.to_dev(cv)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for step, (qq, kk, vv) in enumerate(((q, k, v), (q2, k2, v2))):
        dsp = torch.from_numpy(sp + step).cuda()
        out = kv.kvattn_decode_fused(U.to_dev(qq), U.to_dev(kk), U.to_dev(vv), dck, dcv, dsp, workspace=ws,
                                     dev_status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        # the counters (16-byte header, then one per sequence and KV head) are back at zero
        head = ws[:16 + ((B * Hkv * 4 + 15) // 16) * 16].view(torch.int32)
        assert int(head.abs().sum().item()) == 0
        outs.append(U.to_host(out))
    o_ck, o_cv = ck.copy(), cv.copy()
    f = U.oracle_freqs(kv.LLAMA3)
    _, ref1, rc1 = oracle.step(q, k, v, o_ck, o_cv, sp, f)
    _, ref2, rc2 = oracle.step(q2, k2, v2, o_ck, o_cv, sp + 1, f)
    assert rc1 == 0 and rc2 == 0
    U.assert_attention_close(outs[0], ref1, "first step")
    U.assert_attention_close(outs[1], ref2, "second step")
    assert np.array_equal(U.to_host(dcv), o_cv)
    assert U.ulp_distance(U.to_host(dck), o_ck).max() <= 1


def test_fused_bad_sequences_write_nothing():
    B, H, Hkv, S = 3, 32, 8, 2048
    sp = np.array([-1, 700, 2048], np.int32)    # 2048 + 1 > S
    q, k, v, ck, cv = U.host_inputs(46, B, 1, H, Hkv, S, [0, 700, 0])
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
    dsp = torch.from_numpy(sp).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full((B, 1, H, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    out = kv.kvattn_decode_fused(dq, dk, dv, dck, dcv, dsp, out=sentinel, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & kv.KVATTN_DEV_START_POS_RANGE
    o = U.to_host(out)
    assert np.all(ks.bf16_bits_to_f64(o[0]) == 5.0) and np.all(ks.bf16_bits_to_f64(o[2]) == 5.0)
    g_ck, g_cv = U.to_host(dck), U.to_host(dcv)
    for b in (0, 2):
        assert np.array_equal(g_ck[b], ck[b]) and np.array_equal(g_cv[b], cv[b])
    qr, kr, ref = U.oracle_sequence(q[1], k[1], v[1], ck[1], cv[1], 700, 1, kv.LLAMA3)
    U.assert_attention_close(o[1], ref, "valid sequence beside bad ones")
    # the hint: a sequence above it is skipped and flagged
    st.zero_()
    sp2 = torch.tensor([100, 700, 5], dtype=torch.int32, device="cuda")
    kv.kvattn_decode_fused(dq, dk, dv, dck, dcv, sp2, max_kv_len_hint=300, out=sentinel, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & kv.KVATTN_DEV_KV_LEN_HINT


def test_fused_step_replays_in_a_cuda_graph():
    """The fused call allocates nothing and needs no memset, so a captured
    step replays to the same result as a direct call."""
    B, H, Hkv, S = 8, 32, 8, 8192
    sp = np.array([8000, 600, 4000, 1, 7999, 3333, 1024, 2500], np.int32)
    q, k, v, ck, cv = U.host_inputs(47, B, 1, H, Hkv, S, sp)
    dq, dk, dv = (U.to_dev(x) for x in (q, k, v))
    dsp = torch.from_numpy(sp).cuda()
    ws = kv.alloc_fused_workspace(kv.kvattn_decode_fused_workspace_bytes(B, H, Hkv, S))
    out_direct = torch.empty_like(dq)
    ck1, cv1 = U.to_dev(ck), U.to_dev(cv)
    kv.kvattn_decode_fused(dq, dk, dv, ck1, cv1, dsp, out=out_direct, workspace=ws)
    ck2, cv2 = U.to_dev(ck), U.to_dev(cv)
    out_graph = torch.empty_like(dq)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        kv.kvattn_decode_fused(dq, dk, dv, ck2, cv2, dsp, out=out_graph, workspace=ws, stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_direct, out_graph)
    assert torch.equal(ck1, ck2) and torch.equal(cv1, cv2)
    del g
