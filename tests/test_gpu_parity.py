"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs, at small shapes that span several tiles, ragged tails
and split boundaries, plus indexing, error-flag and schedule checks."""
import numpy as np
import pytest

import kvattn_synth as ks
import oracle
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")


def _dev_step(q, k, v, ck, cv, sp, rope, T, kind, hint=0, in_place=False):
    """Run rope_append then decode/prefill on the GPU; return host copies."""
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
    dsp = torch.from_numpy(np.asarray(sp, np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_rot = kv.kvattn_rope_append(dq, dk, dv, dck, dcv, dsp, rope=rope, q_rot=dq if in_place else None,
                                  dev_status=status)
    if kind == "decode":
        out = kv.kvattn_decode(q_rot, dck, dcv, dsp, max_kv_len_hint=hint, dev_status=status)
    else:
        out = kv.kvattn_prefill_chunk(q_rot, dck, dcv, dsp, max_kv_len_hint=hint, dev_status=status)
    torch.cuda.synchronize()
    return (U.to_host(q_rot), U.to_host(dck), U.to_host(dcv), U.to_host(out), int(status.item()))


def _check_step(seed, B, T, H, Hkv, S, sp, rope, kind, hint=0, in_place=False):
    q, k, v, ck, cv = U.host_inputs(seed, B, T, H, Hkv, S, sp)
    g_qrot, g_ck, g_cv, g_out, st = _dev_step(q, k, v, ck, cv, sp, rope, T, kind, hint, in_place)
    assert st == 0
    # the oracle on the same bits
    o_ck, o_cv = ck.copy(), cv.copy()
    q_rot, out, rc = oracle.step(q, k, v, o_ck, o_cv, np.asarray(sp, np.int32), U.oracle_freqs(rope),
                                 layout=rope.layout, rotary_dim=rope.rotary_dim)
    assert rc == 0
    assert U.ulp_distance(g_qrot, q_rot).max() <= 1
    assert U.ulp_distance(g_ck, o_ck).max() <= 1
    assert np.array_equal(g_cv, o_cv)
    for b in range(B):  # rows outside the new ones are bit-identical to the input
        keep = np.ones(S, bool)
        keep[sp[b]:sp[b] + T] = False
        assert np.array_equal(g_ck[b, keep], ck[b, keep])
    return U.assert_attention_close(g_out, out, f"{kind} B={B} T={T} H={H}/{Hkv} sp={list(sp)}")


@pytest.mark.parametrize("case", [
    (3, 32, 8, 64, [0, 17, 63], kv.LLAMA3),
    (2, 32, 8, 200, [31, 32], kv.LLAMA3),
    (2, 32, 8, 200, [33, 199], kv.LLAMA3_1),
    (4, 16, 16, 130, [63, 64, 65, 129], kv.LLAMA3),     # G = 1 (MHA)
    (3, 16, 8, 300, [0, 95, 257], kv.LLAMA3),           # G = 2
    (5, 64, 8, 520, [1, 127, 128, 511, 519], kv.LLAMA3),  # G = 8 (tensor cores)
    (3, 32, 2, 700, [0, 63, 64, 699][:3], kv.LLAMA3),     # G = 16 (tensor cores)
    (4, 64, 8, 3000, [2999, 64, 65, 1000], kv.LLAMA3_1),  # G = 8, several splits
    (8, 32, 8, 8192, [8191, 0, 63, 64, 4000, 777, 5000, 12], kv.LLAMA3),  # G = 4 on the tensor-core kernel
    (3, 32, 1, 2500, [0, 1000, 2499], kv.LLAMA3),       # G = 32 (MQA): the tcgen05 multi-query kernel
    (6, 32, 1, 6000, [5999, 127, 128, 129, 3000, 4095], kv.LLAMA3_1),  # G = 32 at key-tile edges
    (2, 64, 2, 1500, [1499, 700], kv.LLAMA3),           # G = 32 with two KV heads
    (6, 32, 1, 1000, [95, 96, 97, 191, 192, 999], kv.LLAMA3),  # G = 32, short row sets (96 to 1000 rows)
    # G = 32 with many short row sets: the multi-query kernel's even ranges of
    # key tiles cross several sequences each (Q reloaded, one partial per piece)
    (150, 32, 1, 2048, [int(x) for x in np.random.RandomState(7).randint(0, 2048, 150)], kv.LLAMA3),
    (40, 64, 2, 700, [0, 127, 128, 699] + [int(x) for x in np.random.RandomState(8).randint(0, 700, 36)],
     kv.LLAMA3_1),
    (2, 64, 1, 900, [899, 33], kv.LLAMA3_1),            # G = 64 (MQA, 64 heads)
    # fewer than four query heads, or not a multiple of four: the merge runs
    # four heads per CTA and its last CTA has heads to spare (long rows, so
    # every sequence is split)
    (3, 2, 1, 3000, [2999, 100, 1500], kv.LLAMA3),     # H = 2, G = 2
    (2, 6, 3, 4000, [3999, 2000], kv.LLAMA3_1),        # H = 6, G = 2
    (2, 1, 1, 5000, [4999, 64], kv.LLAMA3),            # H = 1 (one head)
])
def test_decode_step_small(case):
    B, H, Hkv, S, sp, rope = case
    _check_step(11, B, 1, H, Hkv, S, sp, rope, "decode")


def test_decode_step_in_place_rotation():
    _check_step(12, 2, 1, 32, 8, 96, [5, 70], kv.LLAMA3, "decode", in_place=True)


def test_prefill_step_in_place_rotation_whole_tokens():
    # 600 tokens: rope_append gives each CTA a whole token (32 query and 8 key
    # heads) and rotates q into itself in 16-byte chunks of four pairs
    _check_step(14, 2, 300, 32, 8, 1024, [100, 500], kv.LLAMA3_1, "prefill", in_place=True)


@pytest.mark.parametrize("hint", [0, 1500, 3000, 4096])
def test_decode_split_sizes_agree(hint):
    # different hints give different split sizes; each must match the oracle
    sp = [1499, 700, 64, 1000]
    _check_step(13, 4, 1, 32, 8, 4096, sp, kv.LLAMA3, "decode", hint=hint)


def test_decode_many_splits_long_rows():
    _check_step(14, 2, 1, 32, 8, 20000, [19999, 12345], kv.LLAMA3_1, "decode")


@pytest.mark.parametrize("case", [
    (2, 2, 32, 8, 80, [0, 40]),
    (2, 7, 32, 8, 120, [33, 100]),
    (1, 128, 32, 8, 400, [200]),
    (2, 9, 64, 8, 64, [0, 55]),
    (1, 33, 16, 16, 100, [31]),
])
def test_prefill_step_small(case):
    B, T, H, Hkv, S, sp = case
    _check_step(21, B, T, H, Hkv, S, sp, kv.LLAMA3, "prefill")


def test_rope_append_large_positions_scaled():
    # positions up to 131071: fp64 angles keep the rotation within one ulp
    B, T, H, Hkv, S = 2, 1, 32, 8, 131072
    sp = [131071, 65536]
    q = ks.tensor_normal(3, ks.STREAM_Q, (B, T, H, 128))
    k = ks.tensor_normal(3, ks.STREAM_K_NEW, (B, T, Hkv, 128))
    v = ks.tensor_normal(3, ks.STREAM_V_NEW, (B, T, Hkv, 128))
    dck = torch.zeros((B, S, Hkv, 128), dtype=torch.bfloat16, device="cuda")
    dcv = torch.zeros_like(dck)
    dsp = torch.tensor(sp, dtype=torch.int32, device="cuda")
    q_rot = kv.kvattn_rope_append(U.to_dev(q), U.to_dev(k), U.to_dev(v), dck, dcv, dsp, rope=kv.LLAMA3_1)
    torch.cuda.synchronize()
    g_q = U.to_host(q_rot)
    f = U.oracle_freqs(kv.LLAMA3_1)
    for b in range(B):
        ck = np.zeros((1, sp[b] + T, Hkv, 128), np.uint16)
        cv = np.zeros_like(ck)
        qr, rc = oracle.rope_append(q[b:b + 1].copy(), k[b:b + 1].copy(), v[b:b + 1].copy(), ck, cv,
                                    np.array([sp[b]], np.int32), f)
        assert rc == 0
        assert U.ulp_distance(g_q[b], qr[0]).max() <= 1
        row = U.to_host(dck[b, sp[b]:sp[b] + T])
        assert U.ulp_distance(row, ck[0, sp[b]:]).max() <= 1
        assert np.array_equal(U.to_host(dcv[b, sp[b]:sp[b] + T]), cv[0, sp[b]:])
        # Pairs 29..34 (elements 58..69) are the ones the Llama-3.1 rule
        # blends; at these positions a misread blend would turn them by far
        # more than one ulp.  Checked on their own, and shown to be sensitive:
        # the unscaled rotation differs there.
        blend = slice(58, 70)
        assert U.ulp_distance(g_q[b][..., blend], qr[0][..., blend]).max() <= 1
        assert U.ulp_distance(row[..., blend], ck[0, sp[b]:][..., blend]).max() <= 1
        ck0 = np.zeros_like(ck)
        qr0, rc = oracle.rope_append(q[b:b + 1].copy(), k[b:b + 1].copy(), v[b:b + 1].copy(), ck0,
                                     np.zeros_like(ck0), np.array([sp[b]], np.int32), U.oracle_freqs(kv.LLAMA3))
        assert rc == 0
        assert np.mean(U.ulp_distance(g_q[b][..., blend], qr0[0][..., blend]) > 1) > 0.5


@pytest.mark.parametrize("kind,T", [("decode", 1), ("prefill", 4)])
def test_planted_row_indexing(kind, T):
    # q aligned with one planted K row gives it all the weight; V rows carry
    # their index as a code, so the output names the row read, exactly.
    B, H, Hkv, S = 2, 32, 8, 300
    sp = np.array([150, 37], np.int32)
    K = np.full((B, S, Hkv, 128), -1.0 / 128)
    V = np.zeros((B, S, Hkv, 128))
    for r in range(S):
        V[:, r] = float(r % 250 + 1)
    qv = np.full((B, T, H, 128), 4.0)
    cases = []
    for b in range(B):
        for t in range(T):
            L = sp[b] + t + 1
            cases.append((b, t, L - 1, True))
    for b, t, r_star, vis in cases:
        K2 = K.copy()
        K2[b, r_star, :, :] = 1.0
        dk = U.to_dev(ks.f64_to_bf16_bits(K2))
        dv = U.to_dev(ks.f64_to_bf16_bits(V))
        dq = U.to_dev(ks.f64_to_bf16_bits(qv))
        dsp = torch.from_numpy(sp).cuda()
        if kind == "decode":
            out = kv.kvattn_decode(dq, dk, dv, dsp)
        else:
            out = kv.kvattn_prefill_chunk(dq, dk, dv, dsp)
        o = ks.bf16_bits_to_f64(U.to_host(out))
        assert np.all(o[b, t] == float(r_star % 250 + 1))
        # the next row (r_star + 1) is invisible to token t: plant there and
        # the output must stay a mean of visible codes
        if r_star + 1 < S and t == T - 1:
            K3 = K.copy()
            K3[b, r_star + 1, :, :] = 1.0
            out = (kv.kvattn_decode if kind == "decode" else kv.kvattn_prefill_chunk)(
                dq, U.to_dev(ks.f64_to_bf16_bits(K3)), dv, dsp)
            o = ks.bf16_bits_to_f64(U.to_host(out))
            vis_codes = np.array([float(r % 250 + 1) for r in range(r_star + 1)])
            assert abs(o[b, t, 0, 0] - vis_codes.mean()) < 0.02 * vis_codes.mean()


def test_out_of_range_start_pos_is_flagged_and_skipped():
    B, H, Hkv, S, T = 3, 32, 8, 64, 2
    sp = np.array([-1, 10, 63], np.int32)       # 63 + 2 > 64
    q, k, v, ck, cv = U.host_inputs(5, B, T, H, Hkv, S, [0, 10, 0])
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
    dsp = torch.from_numpy(sp).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_rot = kv.kvattn_rope_append(dq, dk, dv, dck, dcv, dsp, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & kv.KVATTN_DEV_START_POS_RANGE
    g_ck = U.to_host(dck)
    assert np.array_equal(g_ck[0], ck[0]) and np.array_equal(g_ck[2], ck[2])
    sentinel = torch.full((B, T, H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    st.zero_()
    out = kv.kvattn_prefill_chunk(q_rot, dck, dcv, dsp, out=sentinel, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & kv.KVATTN_DEV_START_POS_RANGE
    o = U.to_host(out)
    assert np.all(ks.bf16_bits_to_f64(o[0]) == 7.0) and np.all(ks.bf16_bits_to_f64(o[2]) == 7.0)
    # the valid sequence is still right
    qr, kr, ref = U.oracle_sequence(q[1], k[1], v[1], ck[1], cv[1], 10, T, kv.LLAMA3)
    U.assert_attention_close(o[1], ref, "valid sequence beside bad ones")


@pytest.mark.parametrize("seed", [101, 102, 103, 104, 105, 106])
def test_mqa_decode_random_shapes(seed):
    # multi-query decode at seeded random shapes: the call's key tiles are cut
    # into even ranges that start and end anywhere inside the sequences
    rng = np.random.RandomState(seed)
    Hkv = int(rng.choice([1, 2]))
    B = int(rng.randint(1, 60))
    S = int(rng.randint(300, 4000))
    sp = [int(x) for x in rng.randint(0, S, B)]
    assert kv.kvattn_decode_plan(B, 32 * Hkv, Hkv, S)["max_splits"] > 1  # the multi-query kernel runs
    _check_step(seed, B, 1, 32 * Hkv, Hkv, S, sp, kv.LLAMA3, "decode")


def test_mqa_decode_bad_positions_flagged_and_skipped():
    """Multi-query decode (32 heads per KV head, tcgen05): sequences whose
    start position is outside the cache or not below the hint add no key tiles
    to the call's plan, keep the caller's output and set the status bits; the
    others match the oracle."""
    B, H, Hkv, S, hint = 6, 32, 1, 3000, 2500
    sp = np.array([2499, -1, 1200, 3000, 2600, 64], np.int32)
    q, k, v, ck, cv = U.host_inputs(15, B, 1, H, Hkv, S, np.clip(sp, 0, S - 1))
    assert kv.kvattn_decode_plan(B, H, Hkv, S, max_kv_len_hint=hint)["max_splits"] > 1
    dsp = torch.from_numpy(sp).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full((B, 1, H, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    out = kv.kvattn_decode(U.to_dev(q), U.to_dev(ck), U.to_dev(cv), dsp, max_kv_len_hint=hint, out=sentinel,
                           dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & kv.KVATTN_DEV_START_POS_RANGE
    assert st.item() & kv.KVATTN_DEV_KV_LEN_HINT
    o = U.to_host(out)
    for b in (1, 3, 4):
        assert np.all(ks.bf16_bits_to_f64(o[b]) == 3.0), b
    good = [0, 2, 5]
    ref, rc = oracle.attention(q[good].copy(), ck[good].copy(), cv[good].copy(), sp[good].copy())
    assert rc == 0
    U.assert_attention_close(o[good], ref, "valid multi-query sequences beside bad ones")


def test_kv_len_hint_exceeded_is_flagged():
    B, H, Hkv, S = 2, 32, 8, 256
    sp = np.array([200, 20], np.int32)
    q, k, v, ck, cv = U.host_inputs(6, B, 1, H, Hkv, S, sp)
    dsp = torch.from_numpy(sp).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full((B, 1, H, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    out = kv.kvattn_decode(U.to_dev(q), U.to_dev(ck), U.to_dev(cv), dsp, max_kv_len_hint=100,
                           out=sentinel, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & kv.KVATTN_DEV_KV_LEN_HINT
    o = ks.bf16_bits_to_f64(U.to_host(out))
    assert np.all(o[0] == 3.0) and not np.all(o[1] == 3.0)


def test_prefill_equals_prefill_then_decode_steps():
    # 12 tokens at once vs 8 then 4 single decode steps (the schedule test of
    # "Grouped-query attention: a smaller KV cache", 9:42) on the GPU path
    B, H, Hkv, S, T, T1 = 2, 32, 8, 128, 12, 8
    sp = np.array([3, 70], np.int32)
    q, k, v, ck, cv = U.host_inputs(7, B, T, H, Hkv, S, sp)
    _, ckA, cvA, outA, st = _dev_step(q, k, v, ck, cv, sp, kv.LLAMA3, T, "prefill")
    assert st == 0
    _, ckB, cvB, outB1, st = _dev_step(q[:, :T1].copy(), k[:, :T1].copy(), v[:, :T1].copy(), ck, cv, sp,
                                       kv.LLAMA3, T1, "prefill")
    outs = [outB1]
    for t in range(T1, T):
        _, ckB, cvB, o, st = _dev_step(q[:, t:t + 1].copy(), k[:, t:t + 1].copy(), v[:, t:t + 1].copy(),
                                       ckB, cvB, sp + t, kv.LLAMA3, 1, "decode")
        assert st == 0
        outs.append(o)
    outB = np.concatenate(outs, axis=1)
    assert np.array_equal(ckA, ckB) and np.array_equal(cvA, cvB)
    a = ks.bf16_bits_to_f64(outA)
    b = ks.bf16_bits_to_f64(outB)
    assert np.abs(a - b).max() <= 2 * U.MAX_ABS / 4


@pytest.mark.parametrize("case", [
    (2, 77, 32, 8, 400, [0, 250]),      # G=4: 3 M tiles (32 tokens each), ragged tail
    (1, 300, 16, 8, 700, [123]),        # G=2: 64-token tiles, several key tiles
    (2, 20, 64, 8, 300, [0, 129]),      # G=8: 16-token tiles
    (1, 130, 8, 8, 260, [127]),         # G=1 (MHA): 128-token tiles
    (2, 11, 32, 2, 150, [0, 120]),      # G=16: 8-token tiles
    (2, 9, 32, 1, 300, [0, 200]),       # G=32 (MQA, 32 heads): 4-token tiles
    (1, 5, 64, 1, 200, [150]),          # G=64 (MQA, 64 heads): 2-token tiles
    (2, 3, 128, 1, 140, [7, 130]),      # G=128: one token per tile
    (3, 1, 32, 8, 300, [0, 127, 128]),  # one token per sequence through the prefill path
])
def test_prefill_tiles_and_groups(case):
    B, T, H, Hkv, S, sp = case
    _check_step(23, B, T, H, Hkv, S, sp, kv.LLAMA3, "prefill")


@pytest.mark.parametrize("kind,T", [("decode", 1), ("prefill", 40)])
def test_rows_past_the_sequence_may_hold_nan(kind, T):
    # cache rows at and beyond start_pos+T are outside every mask; filling them
    # with NaN must not change any output (no 0 * NaN may reach the result)
    B, H, Hkv, S = 2, 32, 8, 512
    sp = np.array([100, 300], np.int32)
    q, k, v, ck, cv = U.host_inputs(24, B, T, H, Hkv, S, sp)
    for b in range(B):
        ck[b, sp[b]:] = 0x7FC0
        cv[b, sp[b]:] = 0x7FC0
    _, g_ck, g_cv, g_out, st = _dev_step(q, k, v, ck, cv, sp, kv.LLAMA3, T, kind)
    assert st == 0
    o_ck, o_cv = ck.copy(), cv.copy()
    _, out, rc = oracle.step(q, k, v, o_ck, o_cv, sp, U.oracle_freqs(kv.LLAMA3))
    assert rc == 0
    U.assert_attention_close(g_out, out, f"{kind} with NaN past the sequence")


@pytest.mark.parametrize("layout,rotary_dim,scaled,kind,T", [
    (1, 0, False, "prefill", 3), (0, 64, False, "prefill", 3), (1, 96, True, "prefill", 3),
    (0, 2, False, "decode", 1), (1, 64, False, "decode", 1)])
def test_rope_layouts_and_partial_rotary(layout, rotary_dim, scaled, kind, T):
    """Half-split pairs (i, i + r/2) and a rotary width r < d, against the
    oracle: cache and q_rot within one ulp, the unrotated tail bit-copied."""
    B, H, Hkv, S = 2, 32, 8, 200
    sp = np.array([0, 150], np.int32)
    rope = kv.RopeParams(use_scaled=scaled, layout=layout, rotary_dim=rotary_dim)
    _check_step(37 + layout, B, T, H, Hkv, S, sp, rope, kind)
    q, k, v, ck, cv = U.host_inputs(31, B, T, H, Hkv, S, sp)
    g_qrot, _, _, _, st = _dev_step(q, k, v, ck, cv, sp, rope, T, kind)
    assert st == 0
    r = rotary_dim or 128
    assert np.array_equal(g_qrot[..., r:], q[..., r:])


def test_decode_kernel_choice():
    """G = 4 runs on the tensor-core decode for large calls and on the
    CUDA-core kernel for small ones; G >= 8 always on tensor cores."""
    assert kv.kvattn_decode_plan(8, 32, 8, 8192)["tensor_cores"]
    assert not kv.kvattn_decode_plan(1, 32, 8, 8192, max_kv_len_hint=1001)["tensor_cores"]
    assert kv.kvattn_decode_plan(1, 64, 8, 4096)["tensor_cores"]
    assert not kv.kvattn_decode_plan(64, 16, 8, 8192)["tensor_cores"]


def test_decode_workspace_shared_across_shapes_and_left_zeroed():
    """One workspace serves calls of different shapes in a row: its work
    counter sits at a fixed offset and every call leaves it zero."""
    shapes = [(8, 32, 8, 8192, [8191, 0, 63, 64, 4000, 777, 5000, 12]),
              (4, 32, 8, 4096, [1499, 700, 64, 1000]),
              (3, 64, 8, 3000, [2999, 5, 1500]),
              (2, 32, 1, 3000, [2999, 100])]
    ws = kv.alloc_workspace(max(kv.kvattn_decode_workspace_bytes(B, H, Hkv, S) for B, H, Hkv, S, _ in shapes))
    for seed, (B, H, Hkv, S, sp) in enumerate(shapes):
        q, k, v, ck, cv = U.host_inputs(70 + seed, B, 1, H, Hkv, S, sp)
        dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
        dsp = torch.from_numpy(np.asarray(sp, np.int32)).cuda()
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        q_rot = kv.kvattn_rope_append(dq, dk, dv, dck, dcv, dsp, dev_status=st)
        need = kv.kvattn_decode_workspace_bytes(B, H, Hkv, S)
        out = kv.kvattn_decode(q_rot, dck, dcv, dsp, workspace=ws[:max(need, 16)], dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert int(ws[:16].view(torch.int32).abs().sum().item()) == 0
        o_ck, o_cv = ck.copy(), cv.copy()
        _, ref, rc = oracle.step(q, k, v, o_ck, o_cv, np.asarray(sp, np.int32), U.oracle_freqs(kv.LLAMA3))
        assert rc == 0
        U.assert_attention_close(U.to_host(out), ref, f"shape {B},{H},{Hkv},{S}")
