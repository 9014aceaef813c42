"""Pins for the fp64 oracle: closed forms, invariants and special cases fixed
by the pages and by mathematics, each chosen so that a plausible slip in the
oracle (a dropped term, a flipped sign, a wrong index, a transposed operand)
fails at least one of them.  CPU only."""
import math

import numpy as np
import pytest

import kvattn_synth as ks
import oracle

RNG = np.random.default_rng(1234)


def bf16(x):
    return ks.f64_to_bf16_bits(np.asarray(x, np.float64))


# ------------------------------------------------------------- bf16 rounding
def test_bf16_rounding_is_nearest_even():
    xs = RNG.standard_normal(20000) * np.exp(RNG.uniform(-20, 20, 20000))
    for x in xs[:4000]:
        b = oracle.f64_to_bf16(x)
        r = oracle.bf16_to_f64(b)
        sign = -1.0 if x < 0 else 1.0
        mag = b & 0x7FFF
        up = oracle.bf16_to_f64((b & 0x8000) | (mag + 1))
        dn = oracle.bf16_to_f64((b & 0x8000) | (mag - 1)) if mag > 0 else 0.0
        # r is at least as close to x as both neighbours
        assert abs(x - r) <= abs(x - up)
        assert abs(x - r) <= abs(x - dn)
        assert math.copysign(1.0, r) == sign
    # ties go to the even pattern
    assert oracle.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80          # 1.0 (even) below
    assert oracle.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie -> even above
    assert oracle.f64_to_bf16(-0.0) == 0x8000
    assert oracle.f64_to_bf16(1e39) == 0x7F80
    assert oracle.f64_to_bf16(2.0 ** -133) == 0x0001              # smallest subnormal
    assert oracle.f64_to_bf16(2.0 ** -135) == 0x0000              # below half of it


def test_bf16_rounding_matches_float32_route_on_float32_inputs():
    # For values that are exactly fp32, one RNE to bf16 equals the integer
    # RNE on the fp32 bit pattern (a different, library-level route).
    f = RNG.standard_normal(5000).astype(np.float32).astype(np.float64)
    mine = np.array([oracle.f64_to_bf16(x) for x in f], np.uint16)
    assert np.array_equal(mine, ks.f64_to_bf16_bits(f))


# ---------------------------------------------------------------- frequencies
def test_freqs_closed_forms():
    th = 500000.0
    f = oracle.rope_freqs(128, th)
    assert f[0] == 1.0                                   # theta^0
    assert abs(f[32] - 1.0 / math.sqrt(th)) < 1e-18      # theta^(-64/128)
    ratio = f[1:] / f[:-1]
    assert np.allclose(ratio, th ** (-2.0 / 128), rtol=1e-13, atol=0)
    prod = f * f[::-1]                                   # theta^(-126/128) for every i
    assert np.allclose(prod, th ** (-126.0 / 128), rtol=1e-13, atol=0)
    assert np.all(np.diff(f) < 0)


def test_scaled_freqs_regions():
    base = oracle.rope_freqs(128, 500000.0)
    sc = oracle.rope_freqs(128, 500000.0, use_scaled=True)
    wl = 2 * math.pi / base
    keep = wl < 8192 / 4
    div = wl > 8192 / 1
    assert keep.sum() == 29 and div.sum() == 29        # i = 0..28 and 35..63
    assert np.array_equal(sc[keep], base[keep])
    assert np.array_equal(sc[div], base[div] / 8.0)
    mid = ~keep & ~div
    # blended values lie strictly between f/8 and f, and decrease with i
    assert np.all(sc[mid] < base[mid]) and np.all(sc[mid] > base[mid] / 8)
    assert np.all(np.diff(sc) < 0)
    # factor 1 makes scaling the identity
    assert np.allclose(oracle.rope_freqs(128, 500000.0, True, factor=1.0), base, rtol=1e-15)


# Blend weights s_i of pairs 29..34 at d = 128, theta = 500000, L0 = 8192,
# low = 1, high = 4, worked out by hand from the public Llama-3.1 rule
# (wavelength 2*pi/f_i, s = (L0/wavelength - low) / (high - low)) and written
# to three decimals; the rule itself is only named on the pages
# ("Llama 3.1 8B · Repeat heads", sku_list excerpt with use_scaled_rope True;
# "Llama 3.1 8B KV cache", section "Training details that matter": the 8x
# factor and the low and high frequency cutoffs).
BLEND_S = {29: 0.804, 30: 0.593, 31: 0.421, 32: 0.281, 33: 0.167, 34: 0.074}


def test_scaled_freqs_blend_interior_values():
    base = oracle.rope_freqs(128, 500000.0)
    sc = oracle.rope_freqs(128, 500000.0, use_scaled=True)
    for i, s in BLEND_S.items():
        # scaled f_i = ((1 - s)/8 + s) f_i, so s = (f'/f - 1/8) * 8/7
        s_oracle = (sc[i] / base[i] - 1.0 / 8.0) * 8.0 / 7.0
        assert abs(s_oracle - s) <= 1e-3, (i, s_oracle, s)


def test_scaled_freqs_blend_is_linear_in_inverse_wavelength():
    # Put pair i's wavelength at L0/2.5: the rule blends linearly in
    # L0/wavelength, so s = (2.5 - 1)/(4 - 1) = 1/2 and the scaled frequency
    # is exactly (1/16 + 1/2) f = 0.5625 f.  A blend linear in the wavelength
    # itself would give (L0/2.5 - L0/4)/(L0 - L0/4) = 0.2 and 0.825 f.
    for i in (29, 31, 40, 60):
        f = oracle.rope_freqs(128, 500000.0)[i]
        L0 = 2.5 * (2 * math.pi / f)
        got = oracle.rope_freqs(128, 500000.0, True, 8.0, 1.0, 4.0, L0)[i]
        assert abs(got / f - 0.5625) <= 1e-12, (i, got / f)


@pytest.mark.parametrize("cut", ["short", "long"])
def test_scaled_freqs_continuous_at_cutoffs(cut):
    # Move the original context L0 so that the wavelength of pair i sits just
    # below / just above a cutoff; the scaled frequency must not jump.
    i = 30
    f = oracle.rope_freqs(128, 500000.0)[i]
    wl = 2 * math.pi / f
    fac = 4.0 if cut == "short" else 1.0               # cutoff = L0 / high or L0 / low
    vals = []
    for eps in (-1e-9, 1e-9):
        L0 = fac * wl * (1 + eps)
        vals.append(oracle.rope_freqs(128, 500000.0, True, 8.0, 1.0, 4.0, L0)[i])
    assert abs(vals[0] - vals[1]) <= 1e-7 * f
    expect = f if cut == "short" else f / 8
    assert abs(vals[0] - expect) <= 1e-7 * f


# ---------------------------------------------------------------- rotation
def test_rotation_quarter_turn_counter_clockwise():
    y = oracle.rope_rotate_f64(np.array([1.0, 0.0, 0.0, 1.0]), np.array([math.pi / 2, math.pi]), 1)
    assert np.allclose(y, [0.0, 1.0, 0.0, -1.0], atol=1e-15)


def test_rotation_identity_at_zero_and_norms():
    f = oracle.rope_freqs(128, 500000.0)
    x = RNG.standard_normal((5, 128))
    assert np.array_equal(oracle.rope_rotate_f64(x, f, 0), x)
    for p in (1, 1000, 131071):
        y = oracle.rope_rotate_f64(x, f, p)
        n0 = np.hypot(x[:, 0::2], x[:, 1::2])
        n1 = np.hypot(y[:, 0::2], y[:, 1::2])
        assert np.allclose(n0, n1, rtol=1e-13)


def test_rotation_composes_and_relative_offset():
    f = oracle.rope_freqs(128, 500000.0, use_scaled=True)
    q = RNG.standard_normal(128)
    k = RNG.standard_normal(128)
    a = oracle.rope_rotate_f64(oracle.rope_rotate_f64(q, f, 700), f, 300)
    assert np.allclose(a, oracle.rope_rotate_f64(q, f, 1000), atol=1e-11)
    # <R_m q, R_n k> depends only on m - n ("The Modern Decoder Block", key ideas)
    ref = None
    for m, n in ((5, 2), (1005, 1002), (70003, 70000)):
        dot = float(oracle.rope_rotate_f64(q, f, m) @ oracle.rope_rotate_f64(k, f, n))
        ref = dot if ref is None else ref
        assert abs(dot - ref) <= 1e-9 * (1 + abs(ref))
    # and it does change with the offset
    other = float(oracle.rope_rotate_f64(q, f, 6) @ oracle.rope_rotate_f64(k, f, 2))
    assert abs(other - ref) > 1e-3


# ------------------------------------------------------- rope + cache append
def _inputs(B, T, H, Hkv, d, S, sp, seed=5):
    q = ks.tensor_normal(seed, ks.STREAM_Q, (B, T, H, d))
    k = ks.tensor_normal(seed, ks.STREAM_K_NEW, (B, T, Hkv, d))
    v = ks.tensor_normal(seed, ks.STREAM_V_NEW, (B, T, Hkv, d))
    ck = ks.cache_fill(seed, ks.STREAM_CACHE_K, B, S, Hkv, d, sp)
    cv = ks.cache_fill(seed, ks.STREAM_CACHE_V, B, S, Hkv, d, sp)
    return q, k, v, ck, cv


def test_append_writes_exactly_the_new_rows():
    B, T, H, Hkv, d, S = 3, 4, 8, 2, 16, 20
    sp = np.array([0, 7, 16], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    ck0, cv0 = ck.copy(), cv.copy()
    f = oracle.rope_freqs(d, 500000.0)
    q_rot, rc = oracle.rope_append(q, k, v, ck, cv, sp, f)
    assert rc == oracle.OK
    for b in range(B):
        rows = np.arange(S)
        new = (rows >= sp[b]) & (rows < sp[b] + T)
        assert np.array_equal(ck[b, ~new], ck0[b, ~new])
        assert np.array_equal(cv[b, ~new], cv0[b, ~new])
        assert np.array_equal(cv[b, new], v[b])          # values stored as given
    # position 0 is the identity rotation
    assert np.array_equal(ck[0, 0], k[0, 0])
    assert np.array_equal(q_rot[0, 0], q[0, 0])
    assert not np.array_equal(q_rot[1, 0], q[1, 0])


def test_append_rejects_rows_outside_the_cache():
    B, T, H, Hkv, d, S = 2, 3, 4, 2, 8, 10
    sp = np.array([8, -1], np.int32)                     # 8+3 > 10 and negative
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, [0, 0])
    ck0 = ck.copy()
    _, rc = oracle.rope_append(q, k, v, ck, cv, sp, oracle.rope_freqs(d))
    assert rc == oracle.ERR_RANGE
    assert np.array_equal(ck, ck0)


def test_append_rounding_is_one_rounding_of_the_exact_rotation():
    B, T, H, Hkv, d, S = 2, 3, 4, 2, 32, 40
    sp = np.array([5, 30], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    f = oracle.rope_freqs(d, 500000.0)
    q_rot, qe, ke, rc = oracle.rope_append(q, k, v, ck, cv, sp, f, want_exact=True)
    assert rc == 0
    assert np.array_equal(q_rot.reshape(-1), np.array([oracle.f64_to_bf16(x) for x in qe.reshape(-1)], np.uint16))
    for b in range(B):
        for t in range(T):
            y = oracle.rope_rotate_f64(ks.bf16_bits_to_f64(k[b, t]), f, int(sp[b]) + t)
            assert np.array_equal(y, ke[b, t])


# ---------------------------------------------------------------- attention
def _rope_then_attend(q, k, v, ck, cv, sp, d, scale=None):
    f = oracle.rope_freqs(d, 500000.0)
    q_rot, out, rc = oracle.step(q, k, v, ck, cv, sp, f, scale=scale)
    assert rc == 0
    return q_rot, out


def test_single_row_returns_v_exactly():
    B, T, H, Hkv, d, S = 2, 1, 8, 2, 16, 4
    sp = np.zeros(B, np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    _, out = _rope_then_attend(q, k, v, ck, cv, sp, d)
    G = H // Hkv
    for h in range(H):
        assert np.array_equal(out[:, 0, h], ks.bf16_bits_to_f64(v[:, 0, h // G]))


def test_zero_query_gives_mean_of_visible_values():
    B, T, H, Hkv, d, S = 2, 3, 4, 2, 8, 30
    sp = np.array([10, 25], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    f = oracle.rope_freqs(d)
    oracle.rope_append(q, k, v, ck, cv, sp, f)
    qz = np.zeros_like(q)
    out, rc = oracle.attention(qz, ck, cv, sp)
    assert rc == 0
    V = ks.bf16_bits_to_f64(cv)
    for b in range(B):
        for t in range(T):
            L = sp[b] + t + 1
            for h in range(H):
                assert np.allclose(out[b, t, h], V[b, :L, h // 2].mean(axis=0), atol=1e-14)


def test_equal_keys_give_mean_and_scale_zero_too():
    B, T, H, Hkv, d, S = 1, 2, 4, 1, 8, 12
    sp = np.array([6], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    f = oracle.rope_freqs(d)
    q_rot, _ = oracle.rope_append(q, k, v, ck, cv, sp, f)
    V = ks.bf16_bits_to_f64(cv)
    ck_eq = ck.copy()
    ck_eq[0, :] = ck[0, 3]
    out, _ = oracle.attention(q_rot, ck_eq, cv, sp)
    out0, _ = oracle.attention(q_rot, ck, cv, sp, scale=0.0)
    for t in range(T):
        mean = V[0, : sp[0] + t + 1, 0].mean(axis=0)
        for h in range(H):
            assert np.allclose(out[0, t, h], mean, atol=1e-14)
            assert np.allclose(out0[0, t, h], mean, atol=1e-14)


@pytest.mark.parametrize("G", [2, 4])
def test_gqa_equals_mha_with_repeated_heads(G):
    # K_G[h] = K_r[floor(h/G)]: GQA equals MHA whose KV heads are the groups'
    # heads repeated ("Llama 3.1 8B · Repeat heads"; the GQA==MHA test of
    # "Grouped-query attention: a smaller KV cache", 9:42).
    B, T, H, d, S = 2, 3, 8, 16, 24
    Hkv = H // G
    sp = np.array([4, 17], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    qr, out = _rope_then_attend(q, k, v, ck, cv, sp, d)
    ck_m = np.repeat(ck, G, axis=2)
    cv_m = np.repeat(cv, G, axis=2)
    out_m, rc = oracle.attention(qr, ck_m, cv_m, sp)
    assert rc == 0
    assert np.allclose(out, out_m, rtol=0, atol=1e-13)
    # and the map matters: a wrong grouping (h mod Hkv) gives other numbers
    perm = np.array([h % Hkv for h in range(H)])
    out_w, _ = oracle.attention(qr, ck[:, :, perm], cv[:, :, perm], sp)
    assert not np.allclose(out, out_w, atol=1e-6)


def test_mqa_all_heads_share_head_zero():
    B, T, H, d, S = 1, 2, 6, 8, 10
    sp = np.array([5], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, 1, d, S, sp)
    qr, out = _rope_then_attend(q, k, v, ck, cv, sp, d)
    for h in range(H):
        o1, _ = oracle.attention(qr[:, :, h:h + 1].copy(), ck, cv, sp)
        assert np.allclose(out[:, :, h], o1[:, :, 0], atol=1e-14)


def test_planted_row_visibility():
    # A query aligned with one cache row and scaled up puts ~all weight on it;
    # V rows carry distinct codes, so the output names the row read.
    B, T, H, Hkv, d, S = 1, 2, 4, 1, 16, 40
    sp = np.array([20], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    f = oracle.rope_freqs(d)
    oracle.rope_append(q, k, v, ck, cv, sp, f)
    V = np.zeros((B, S, Hkv, d))
    for r in range(S):
        V[0, r, 0, :] = r + 1.0
    cv2 = bf16(V)
    K = np.zeros((B, S, Hkv, d))
    K[0, :, 0, :] = -1.0 / d
    for r_star, t, visible in ((20, 0, True), (21, 0, False), (21, 1, True), (22, 1, False)):
        K2 = K.copy()
        K2[0, r_star, 0, :] = 1.0
        qv = np.zeros((B, T, H, d))
        qv[0, t, :, :] = 8.0                        # score 128*8*scale on r*, negative elsewhere
        out, rc = oracle.attention(bf16(qv), bf16(K2), cv2, sp)
        assert rc == 0
        L = sp[0] + t + 1
        if visible:
            assert np.allclose(out[0, t, :, :], r_star + 1.0, atol=1e-9)
        else:
            assert np.all(out[0, t] <= L + 1e-9)    # never sees row r* (code r*+1 > L)


def test_prefill_equals_prefill_then_single_steps():
    # 12 tokens at once == 8 at once then 4 single steps (the schedule test of
    # "Grouped-query attention: a smaller KV cache", 9:42), here with a cache
    # that already holds rows.
    B, H, Hkv, d, S = 2, 8, 2, 16, 32
    T, T1 = 12, 8
    sp = np.array([3, 9], np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp)
    f = oracle.rope_freqs(d)
    ckA, cvA = ck.copy(), cv.copy()
    _, outA, rc = oracle.step(q, k, v, ckA, cvA, sp, f)
    assert rc == 0
    ckB, cvB = ck.copy(), cv.copy()
    _, outB1, _ = oracle.step(q[:, :T1].copy(), k[:, :T1].copy(), v[:, :T1].copy(), ckB, cvB, sp, f)
    outs = [outB1]
    for t in range(T1, T):
        spt = (sp + t).astype(np.int32)
        _, o, rc = oracle.step(q[:, t:t + 1].copy(), k[:, t:t + 1].copy(), v[:, t:t + 1].copy(),
                               ckB, cvB, spt, f)
        assert rc == 0
        outs.append(o)
    outB = np.concatenate(outs, axis=1)
    assert np.array_equal(ckA, ckB) and np.array_equal(cvA, cvB)
    assert np.allclose(outA, outB, rtol=0, atol=1e-13)


def test_attention_rejects_out_of_range_start_pos():
    B, T, H, Hkv, d, S = 2, 2, 4, 2, 8, 10
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, [S, S])
    out, rc = oracle.attention(q, ck, cv, np.array([9, 1], np.int32))
    assert rc == oracle.ERR_RANGE
    assert np.all(out[0] == 0) and np.any(out[1] != 0)


# ------------------------------------------- half-split layout, partial rotary
def test_half_split_is_interleaved_under_the_pair_permutation():
    # pairs (i, i + d/2) instead of (2i, 2i+1): moving element i to 2i and
    # element i + d/2 to 2i + 1 must turn one layout into the other exactly
    d = 16
    f = oracle.rope_freqs(d, 10000.0)
    x = RNG.standard_normal((3, d))
    perm = np.empty(d, int)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    for p in (0, 7, 1234):
        half = oracle.rope_rotate_f64(x, f, p, layout=1)
        inter = oracle.rope_rotate_f64(x[:, perm], f, p, layout=0)
        assert np.array_equal(half[:, perm], inter)
        if p:
            assert not np.allclose(half, oracle.rope_rotate_f64(x, f, p, layout=0))


def test_partial_rotary_passes_the_tail_and_rotates_the_head():
    d, r = 16, 6
    f = oracle.rope_freqs(r, 10000.0)              # frequencies over the rotated width
    x = RNG.standard_normal((4, d))
    for layout in (0, 1):
        y = oracle.rope_rotate_f64(x, f, 321, layout=layout, rotary_dim=r)
        assert np.array_equal(y[:, r:], x[:, r:])
        assert np.array_equal(y[:, :r], oracle.rope_rotate_f64(x[:, :r].copy(), f, 321, layout=layout))
        # still a rotation: norms of the rotated part are kept
        assert np.allclose(np.linalg.norm(y[:, :r], axis=1), np.linalg.norm(x[:, :r], axis=1), rtol=1e-13)


def test_half_split_relative_offset():
    d = 32
    f = oracle.rope_freqs(d, 500000.0)
    q = RNG.standard_normal(d)
    k = RNG.standard_normal(d)
    a = oracle.rope_rotate_f64(q, f, 40, layout=1) @ oracle.rope_rotate_f64(k, f, 10, layout=1)
    b = oracle.rope_rotate_f64(q, f, 1030, layout=1) @ oracle.rope_rotate_f64(k, f, 1000, layout=1)
    assert abs(a - b) <= 1e-10 * (1 + abs(a))


# ---- sliding window, StreamingLLM sinks, learned sinks ("The Modern Decoder Block", L7.5 / L7.7)

def _cache_inputs(seed=7, B=2, T=3, H=4, Hkv=2, d=8, S=40, sp=(20, 33)):
    sp = np.array(sp, np.int32)
    q, k, v, ck, cv = _inputs(B, T, H, Hkv, d, S, sp, seed=seed)
    f = oracle.rope_freqs(d)
    q_rot, rc = oracle.rope_append(q, k, v, ck, cv, sp, f)
    assert rc == 0
    return q_rot, ck, cv, sp


def test_window_covering_everything_changes_nothing():
    q_rot, ck, cv, sp = _cache_inputs()
    ref, _ = oracle.attention(q_rot, ck, cv, sp)
    for W, n in ((10**6, 0), (ck.shape[1], 3), (40, 40)):
        out, rc = oracle.attention(q_rot, ck, cv, sp, window=W, n_sink=n)
        assert rc == 0 and np.array_equal(out, ref)


def test_window_one_returns_the_token_s_own_value():
    q_rot, ck, cv, sp = _cache_inputs()
    out, rc = oracle.attention(q_rot, ck, cv, sp, window=1)
    assert rc == 0
    V = ks.bf16_bits_to_f64(cv)
    for b in range(2):
        for t in range(3):
            for h in range(4):
                assert np.array_equal(out[b, t, h], V[b, sp[b] + t, h // 2])


@pytest.mark.parametrize("W,n", [(5, 0), (5, 2), (1, 3), (17, 4), (8, 30)])
def test_window_and_sinks_equal_plain_attention_over_the_gathered_rows(W, n):
    """The visible rows of token t at position p are p-W < r <= p and r < n;
    plain attention over a cache holding exactly those rows gives the same
    output (an off-by-one in either bound changes the set)."""
    q_rot, ck, cv, sp = _cache_inputs()
    out, rc = oracle.attention(q_rot, ck, cv, sp, window=W, n_sink=n)
    assert rc == 0
    B, T, H, d = q_rot.shape
    for b in range(B):
        for t in range(T):
            p = int(sp[b]) + t
            rows = [r for r in range(p + 1) if r > p - W or r < n]
            gk = ck[b:b + 1, rows]
            gv = cv[b:b + 1, rows]
            ref, rc2 = oracle.attention(q_rot[b:b + 1, t:t + 1], gk, gv, np.array([len(rows) - 1], np.int32))
            assert rc2 == 0
            assert np.allclose(out[b, t], ref[0, 0], atol=1e-15, rtol=0)


def test_learned_sink_limits_and_closed_forms():
    q_rot, ck, cv, sp = _cache_inputs()
    H = q_rot.shape[2]
    ref, _ = oracle.attention(q_rot, ck, cv, sp)
    # a sink at -infinity takes no mass
    out, rc = oracle.attention(q_rot, ck, cv, sp, sink_logits=np.full(H, -1e300))
    assert rc == 0 and np.array_equal(out, ref)
    # zero query: all scores 0, so out = mean(V) * L / (L + e^sigma)
    qz = np.zeros_like(q_rot)
    sig = np.array([-1.0, 0.0, 0.5, 2.0])
    out, rc = oracle.attention(qz, ck, cv, sp, sink_logits=sig)
    V = ks.bf16_bits_to_f64(cv)
    for b in range(2):
        for t in range(3):
            L = int(sp[b]) + t + 1
            for h in range(H):
                expect = V[b, :L, h // 2].mean(axis=0) * L / (L + math.exp(sig[h]))
                assert np.allclose(out[b, t, h], expect, atol=1e-14, rtol=1e-13)
    # one visible row (window 1): out = V_p * e^s / (e^s + e^sigma)
    out, rc = oracle.attention(q_rot, ck, cv, sp, window=1, sink_logits=sig)
    Q = ks.bf16_bits_to_f64(q_rot)
    K = ks.bf16_bits_to_f64(ck)
    for b in range(2):
        for t in range(3):
            p = int(sp[b]) + t
            for h in range(H):
                s = float(Q[b, t, h] @ K[b, p, h // 2]) / math.sqrt(8)
                wt = 1.0 / (1.0 + math.exp(sig[h] - s))
                assert np.allclose(out[b, t, h], V[b, p, h // 2] * wt, atol=1e-14, rtol=1e-12)
