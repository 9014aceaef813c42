"""The seeded input generator matches its published definitions (CPU)."""
import math

import numpy as np

import kvattn_synth as ks


def test_splitmix64_published_vector():
    # SplitMix64 seeded with state 1234567: the first five outputs of the
    # reference implementation (Vigna's splitmix64.c test values).
    key = 1234567
    got = [ks._mix_int(key + (i + 1) * ks.GAMMA) for i in range(5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]
    w = ks._mix_np(np.array([(key + (i + 1) * ks.GAMMA) & ((1 << 64) - 1) for i in range(5)],
                            dtype=np.uint64))
    assert [int(x) for x in w] == got


def test_normal_moments_and_bf16():
    x = ks.bf16_bits_to_f64(ks.normal_bf16(7, 1, 0, 200_000))
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 1.0) < 0.01
    # every value is a bf16 value: rounding it again changes nothing
    assert np.array_equal(ks.f64_to_bf16_bits(x), ks.normal_bf16(7, 1, 0, 200_000))
    # tail mass near the normal's: P(|z|>2) = 0.0455
    assert abs((np.abs(x) > 2).mean() - math.erfc(2 / math.sqrt(2))) < 0.003


def test_counter_based_offsets():
    a = ks.normal_bf16(3, 4, 0, 1000)
    b = ks.normal_bf16(3, 4, 600, 400)
    assert np.array_equal(a[600:], b)
    assert not np.array_equal(ks.normal_bf16(3, 5, 0, 1000), a)
    assert not np.array_equal(ks.normal_bf16(4, 4, 0, 1000), a)


def test_randint_range_and_uniformity():
    v = ks.randint(11, ks.STREAM_START_POS, 20000, 512, 8191)
    assert v.min() >= 512 and v.max() <= 8191
    assert abs(v.mean() - (512 + 8191) / 2) < 60
    w = ks.randint(11, ks.STREAM_START_POS, 4000, 0, 1)
    assert set(np.unique(w)) == {0, 1}


def test_cache_fill_rows():
    sp = [3, 0, 5]
    c = ks.cache_fill(1, 4, 3, 6, 2, 4, sp)
    for b, n in enumerate(sp):
        assert np.all(c[b, n:] == 0)
        if n:
            assert np.any(c[b, :n] != 0)
            assert np.array_equal(ks.cache_rows(1, 4, b, 6, 2, 4, 0, 6, n), c[b])
            assert np.array_equal(ks.cache_rows(1, 4, b, 6, 2, 4, 1, 4, n), c[b, 1:4])
