"""Brute force on tiny shapes: a separately written pure-Python formula
(complex-number rotation, direct softmax with Python floats) against the C
oracle.  Nothing here calls the oracle's helpers except through its public
entry points.  CPU only."""
import cmath
import math
import random

import numpy as np
import pytest

import kvattn_synth as ks
import oracle


def _bits_to_float(b):
    return float(ks.bf16_bits_to_f64(np.array([b], np.uint16))[0])


def brute(q, k_new, v_new, cache_k, cache_v, sp, theta, scale):
    """Return (cache_k_rot_exact rows dict, q_rot_exact, out) by direct formulas."""
    B, T, H, d = q.shape
    Hkv = k_new.shape[2]
    G = H // Hkv
    n = d // 2
    freqs = [theta ** (-(2.0 * i) / d) for i in range(n)]

    def rot(vec, p):
        res = []
        for i in range(n):
            z = complex(vec[2 * i], vec[2 * i + 1]) * cmath.exp(1j * p * freqs[i])
            res += [z.real, z.imag]
        return res

    qf = [[[[_bits_to_float(q[b, t, h, c]) for c in range(d)] for h in range(H)]
           for t in range(T)] for b in range(B)]
    q_rot = [[[rot(qf[b][t][h], sp[b] + t) for h in range(H)] for t in range(T)] for b in range(B)]
    K = {}
    Vv = {}
    for b in range(B):
        for r in range(sp[b]):
            for j in range(Hkv):
                K[b, r, j] = [_bits_to_float(cache_k[b, r, j, c]) for c in range(d)]
                Vv[b, r, j] = [_bits_to_float(cache_v[b, r, j, c]) for c in range(d)]
        for t in range(T):
            for j in range(Hkv):
                kf = [_bits_to_float(k_new[b, t, j, c]) for c in range(d)]
                K[b, sp[b] + t, j] = rot(kf, sp[b] + t)
                Vv[b, sp[b] + t, j] = [_bits_to_float(v_new[b, t, j, c]) for c in range(d)]
    return q_rot, K, Vv, G


@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_tiny(seed):
    rnd = random.Random(seed)
    Hkv = rnd.choice([1, 2])
    G = rnd.choice([1, 2, 3, 4])
    H = Hkv * G
    d = rnd.choice([4, 8, 16])
    B = rnd.choice([1, 2])
    T = rnd.choice([1, 2, 3])
    S = 12
    sp = [rnd.randint(0, S - T) for _ in range(B)]
    q = ks.tensor_normal(seed, 1, (B, T, H, d))
    k = ks.tensor_normal(seed, 2, (B, T, Hkv, d))
    v = ks.tensor_normal(seed, 3, (B, T, Hkv, d))
    ck = ks.cache_fill(seed, 4, B, S, Hkv, d, sp)
    cv = ks.cache_fill(seed, 5, B, S, Hkv, d, sp)
    theta = 10000.0 if seed % 2 else 500000.0
    scale = 1.0 / math.sqrt(d)

    q_rot_b, K, Vv, _ = brute(q, k, v, ck, cv, sp, theta, scale)

    f = oracle.rope_freqs(d, theta)
    ck_o, cv_o = ck.copy(), cv.copy()
    q_rot, qe, ke, rc = oracle.rope_append(q, k, v, ck_o, cv_o, np.array(sp, np.int32), f,
                                           want_exact=True)
    assert rc == 0
    for b in range(B):
        for t in range(T):
            for h in range(H):
                assert np.allclose(qe[b, t, h], q_rot_b[b][t][h], atol=1e-12)
            for j in range(Hkv):
                assert np.allclose(ke[b, t, j], K[b, sp[b] + t, j], atol=1e-12)
                assert np.array_equal(cv_o[b, sp[b] + t, j], v[b, t, j])

    out, rc = oracle.attention(q_rot, ck_o, cv_o, np.array(sp, np.int32), scale)
    assert rc == 0
    # brute-force attention on the oracle's own bf16 q_rot and cache rows
    for b in range(B):
        for t in range(T):
            for h in range(H):
                j = h // G
                qv = [_bits_to_float(x) for x in q_rot[b, t, h]]
                L = sp[b] + t + 1
                rows_k = [[_bits_to_float(x) for x in ck_o[b, r, j]] for r in range(L)]
                rows_v = [[_bits_to_float(x) for x in cv_o[b, r, j]] for r in range(L)]
                s = [sum(a * c for a, c in zip(qv, kr)) * scale for kr in rows_k]
                mx = max(s)
                w = [math.exp(x - mx) for x in s]
                z = sum(w)
                o = [sum(w[r] * rows_v[r][c] for r in range(L)) / z for c in range(d)]
                assert np.allclose(out[b, t, h], o, atol=1e-13)


@pytest.mark.parametrize("seed", range(4))
def test_bruteforce_window_sinks(seed):
    """Direct-softmax formula over an explicitly listed row set, with a learned
    sink term in the denominator, against the oracle's masked attention."""
    rnd = random.Random(100 + seed)
    Hkv, G = rnd.choice([1, 2]), rnd.choice([1, 2, 4])
    H, d, B, T, S = Hkv * G, rnd.choice([4, 8]), 2, rnd.choice([1, 3]), 16
    sp = [rnd.randint(3, S - T) for _ in range(B)]
    W, n_sink = rnd.randint(1, 6), rnd.randint(0, 3)
    sig = [rnd.uniform(-2, 2) for _ in range(H)] if seed % 2 else None
    q = ks.tensor_normal(seed, 11, (B, T, H, d))
    ck = ks.cache_fill(seed, 14, B, S, Hkv, d, [s + T for s in sp])
    cv = ks.cache_fill(seed, 15, B, S, Hkv, d, [s + T for s in sp])
    scale = 1.0 / math.sqrt(d)
    out, rc = oracle.attention(q, ck, cv, np.array(sp, np.int32), scale, window=W, n_sink=n_sink,
                               sink_logits=None if sig is None else np.array(sig))
    assert rc == 0
    for b in range(B):
        for t in range(T):
            p = sp[b] + t
            rows = [r for r in range(0, p + 1) if (p - r) < W or r < n_sink]
            for h in range(H):
                j = h // G
                qv = [_bits_to_float(x) for x in q[b, t, h]]
                s = [sum(a * _bits_to_float(c) for a, c in zip(qv, ck[b, r, j])) * scale for r in rows]
                terms = s + ([sig[h]] if sig else [])
                mx = max(terms)
                w = [math.exp(x - mx) for x in s]
                z = sum(w) + (math.exp(sig[h] - mx) if sig else 0.0)
                o = [sum(w[i] * _bits_to_float(cv[b, r, j, c]) for i, r in enumerate(rows)) / z for c in range(d)]
                assert np.allclose(out[b, t, h], o, atol=1e-13)
