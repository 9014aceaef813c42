"""Shared helpers for the GPU parity tests: seeded inputs, host<->device
copies of bf16 bit patterns, the comparison metrics, and one oracle run per
sequence.  Test infrastructure only."""
from __future__ import annotations

import math

import numpy as np

import kvattn_synth as ks
import oracle

# Acceptance bars (stated for this path): cache rows and q_rot within one
# bf16 ulp of the fp64 result rounded once; V rows and untouched rows bit
# exact; attention outputs max-abs <= 2e-2 and mean-abs <= 2e-3 against the
# fp64 oracle.  Relative L2 <= 1e-2 is a stricter extra diagnostic: fp32
# accumulation plus one bf16 output rounding (2^-9 relative) stays well below.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_L2 = 1e-2


def to_dev(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_host(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in representable bf16 steps between two bit arrays (+0 == -0)."""
    def ordered(x):
        x = x.astype(np.int64)
        mag = x & 0x7FFF
        return np.where(x & 0x8000, -mag, mag)
    return np.abs(ordered(a) - ordered(b))


def attention_errors(gpu_bits: np.ndarray, ref: np.ndarray):
    g = ks.bf16_bits_to_f64(gpu_bits)
    err = np.abs(g - ref)
    rel = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30))
    return float(err.max()), float(err.mean()), rel


def assert_attention_close(gpu_bits, ref, what=""):
    mx, mean, rel = attention_errors(gpu_bits, ref)
    assert np.all(np.isfinite(ks.bf16_bits_to_f64(gpu_bits))), what
    assert mx <= MAX_ABS, f"{what}: max-abs {mx}"
    assert mean <= MEAN_ABS, f"{what}: mean-abs {mean}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel}"
    return mx, mean, rel


def host_inputs(seed, B, T, H, Hkv, S, sp, d=128):
    q = ks.tensor_normal(seed, ks.STREAM_Q, (B, T, H, d))
    k = ks.tensor_normal(seed, ks.STREAM_K_NEW, (B, T, Hkv, d))
    v = ks.tensor_normal(seed, ks.STREAM_V_NEW, (B, T, Hkv, d))
    ck = ks.cache_fill(seed, ks.STREAM_CACHE_K, B, S, Hkv, d, sp)
    cv = ks.cache_fill(seed, ks.STREAM_CACHE_V, B, S, Hkv, d, sp)
    return q, k, v, ck, cv


def oracle_freqs(rope):
    """f_i over the rotated width: rotary_dim (0 means the whole head)."""
    return oracle.rope_freqs(rope.rotary_dim or 128, rope.theta, rope.use_scaled, rope.factor, rope.low_freq_factor,
                             rope.high_freq_factor, rope.original_max_pos)


def oracle_sequence(q_b, k_b, v_b, ck_rows, cv_rows, sp_b, T, rope, scale=None):
    """Oracle for one sequence: q_b [T,H,d], k_b/v_b [T,Hkv,d], the cache rows
    0..sp_b-1 [sp_b,Hkv,d].  Returns (q_rot [T,H,d], k_rows [T,Hkv,d] bf16 bits,
    out [T,H,d] fp64)."""
    Hkv, d = k_b.shape[1], k_b.shape[2]
    S = sp_b + T
    ck = np.zeros((1, S, Hkv, d), np.uint16)
    cv = np.zeros((1, S, Hkv, d), np.uint16)
    ck[0, :sp_b] = ck_rows[:sp_b]
    cv[0, :sp_b] = cv_rows[:sp_b]
    spa = np.array([sp_b], np.int32)
    q_rot, out, rc = oracle.step(q_b[None].copy(), k_b[None].copy(), v_b[None].copy(), ck, cv, spa,
                                 oracle_freqs(rope), scale=scale, layout=rope.layout,
                                 rotary_dim=rope.rotary_dim)
    assert rc == 0
    return q_rot[0], ck[0, sp_b:sp_b + T], out[0]


def default_scale():
    return 1.0 / math.sqrt(128)
