"""The polynomial 2^x that the chunked-prefill softmax evaluates on the FMA
pipes for a quarter of its exponentials (Cody and Waite's reduction x = n + f,
n = round(x), f in [-1/2, 1/2]; a cubic fitted to 2^f on that interval; n
added to the exponent field).  The coefficients are read from the kernel
source, and the fp32 steps of the device code are replayed in numpy (each
fused multiply-add rounded once), then compared with exp2 in fp64.  CPU only."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "gqa_decode_attention_kvattn_b200", "csrc", "tc_device.cuh")


def _coefficients():
    text = open(SRC).read()
    c = {}
    for i in range(4):
        m = re.search(rf"kExp2C{i}\s*=\s*([-+0-9.eE]+)f", text)
        assert m, f"kExp2C{i} not found"
        c[i] = np.float32(float(m.group(1)))
    return c


def _f32(x):
    return np.asarray(x, np.float64).astype(np.float32)


def _fma(a, b, c):
    # a*b is exact in fp64 for fp32 inputs, so one rounding to fp32 models FFMA
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def exp2_poly(x):
    c = _coefficients()
    x = np.maximum(_f32(x), np.float32(-125.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = _f32(x.astype(np.float64) + np.float64(magic))
    n = _f32(t.astype(np.float64) - np.float64(magic))
    f = _fma(n, np.full_like(n, -1.0), x)
    q = _fma(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    q = _fma(q, f, np.full_like(f, c[1]))
    q = _fma(q, f, np.full_like(f, c[0]))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) \
        & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_reduction_leaves_f_in_half_interval_and_n_exact():
    x = _f32(np.linspace(-125.0, 8.0, 200001))
    magic = np.float32(12582912.0)
    t = _f32(x.astype(np.float64) + np.float64(magic))
    n = _f32(t.astype(np.float64) - np.float64(magic))
    assert np.all(n == np.round(x))       # round to nearest even, exactly
    f = x.astype(np.float64) - n
    assert np.all(np.abs(f) <= 0.5)


def test_relative_error_against_exp2():
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-30.0, 8.0, 200000),
                        np.arange(-125, 9).astype(np.float64), np.arange(-125, 9) + 0.5])
    x = _f32(x)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()          # far below the bf16 rounding of P (2^-9)
    assert np.all(got > 0)


def test_exact_at_integers_within_bound_and_monotone():
    x = _f32(np.arange(-125, 9))
    got = exp2_poly(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 1e-4)
    xs = _f32(np.linspace(-20.0, 8.0, 100001))
    assert np.all(np.diff(exp2_poly(xs)) >= 0)


def test_clamp_below_minus_125():
    got = exp2_poly(_f32([-126.0, -500.0, -np.inf]))
    assert np.allclose(got.astype(np.float64), 2.0 ** -125, rtol=1e-4)
