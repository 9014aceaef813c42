"""The synthetic workloads: shapes, start-position draws and RoPE settings of
the cached-GQA configurations (Llama-3/3.1 head layout: 32 query heads over
8 KV heads of 128, theta 500000; "Llama 3.1 8B KV cache" and the config
excerpts of "Llama 3 8B · KV cache" / "Llama 3.1 8B · Repeat heads"; the
70B-style 64/8 layout of "Grouped-query attention: a smaller KV cache",
19:34).  Values are N(0,1) rounded to bf16 (see this package's generator);
cache rows at or beyond a sequence's start position are zero."""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import DEFAULT_SEED, STREAM_START_POS, randint


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    Hkv: int
    S: int
    sp_lo: int
    sp_hi: int
    scaled_rope: bool = False
    layers: int = 1
    kind: str = "decode"          # "decode" (T = 1) or "prefill"
    note: str = ""

    def start_pos(self, seed: int = DEFAULT_SEED) -> np.ndarray:
        if self.sp_lo == self.sp_hi:
            return np.full(self.B, self.sp_lo, np.int32)
        return randint(seed, STREAM_START_POS, self.B, self.sp_lo, self.sp_hi).astype(np.int32)

    @property
    def kv_len_hint(self) -> int:
        return self.sp_hi + self.T


WORKLOADS = {
    "decode_p1000_b1": Workload(
        "decode_p1000_b1", B=1, T=1, H=32, Hkv=8, S=8192, sp_lo=1000, sp_hi=1000,
        note="single-layer decode step at position 1000"),
    "decode_ragged_b64_l32": Workload(
        "decode_ragged_b64_l32", B=64, T=1, H=32, Hkv=8, S=8192, sp_lo=512, sp_hi=8191, layers=32,
        note="batched ragged decode, 32 layers with separate caches"),
    "prefill_b4_t512_sp3584": Workload(
        "prefill_b4_t512_sp3584", B=4, T=512, H=32, Hkv=8, S=8192, sp_lo=3584, sp_hi=3584, kind="prefill",
        note="chunked prefill of 512 tokens into a cache holding 3584 rows"),
    "decode_long_scaled_b8": Workload(
        "decode_long_scaled_b8", B=8, T=1, H=32, Hkv=8, S=131072, sp_lo=65536, sp_hi=131071, scaled_rope=True,
        note="long-context decode with Llama-3.1 scaled RoPE"),
    "decode_wide_g8_b128": Workload(
        "decode_wide_g8_b128", B=128, T=1, H=64, Hkv=8, S=4096, sp_lo=1, sp_hi=4095,
        note="70B-style 64/8 heads (groups of 8)"),
    "decode_mqa_g32_b64": Workload(
        "decode_mqa_g32_b64", B=64, T=1, H=32, Hkv=1, S=32768, sp_lo=4096, sp_hi=32767,
        note="multi-query attention: all 32 query heads share one KV head"),
    "decode_mha_g1_b16": Workload(
        "decode_mha_g1_b16", B=16, T=1, H=32, Hkv=32, S=8192, sp_lo=512, sp_hi=8191,
        note="multi-head attention: one KV head per query head (G = 1)"),
    "decode_g2_b64": Workload(
        "decode_g2_b64", B=64, T=1, H=16, Hkv=8, S=8192, sp_lo=512, sp_hi=8191,
        note="16 query heads over 8 KV heads (G = 2, the Qwen3-0.6B layout)"),
}

# the workload the headline metric is quoted on
HEADLINE = "decode_ragged_b64_l32"
