"""Host-side logic of the library, CPU only: byte arithmetic against the
pages' printed cache sizes, the exported C ABI, and argument validation that
returns before any CUDA call."""
import ctypes
import os
import re

import pytest

import gqa_decode_attention_kvattn_b200 as kv
from gqa_decode_attention_kvattn_b200 import build as kvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
UNITS = {"B": 1, "kB": 1e3, "MB": 1e6, "GB": 1e9, "MiB": 2 ** 20, "GiB": 2 ** 30}


def _golden():
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "kv_cache_bytes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fields, _, cite = line.partition("|")
            name, L, hkv, d, be, tok, val, unit, tol = fields.split()
            rows.append((name, int(L), int(hkv), int(d), int(be), int(tok), float(val), unit, float(tol), cite))
    return rows


@pytest.mark.parametrize("row", _golden(), ids=lambda r: r[0])
def test_kv_cache_bytes_match_printed_sizes(row):
    name, L, hkv, d, be, tok, val, unit, tol, _ = row
    got = kv.kv_cache_bytes(L, hkv, d, tok, be) / UNITS[unit]
    assert abs(got - val) <= tol * val + 1e-12, (name, got, val)


def test_attention_kv_bytes_and_flops():
    # decode at p = 1000 reads rows 0..1000: 1001 rows x 4096 B per layer
    assert kv.attention_kv_bytes([1000], 1, 8) == 1001 * 4096
    # prefill of T tokens sees sp+1 .. sp+T rows
    assert kv.prefill_flops([3584] * 4, 512, 32) == 4 * 128 * 32 * 4 * sum(3585 + t for t in range(512))
    assert kv.prefill_flops([0], 1, 1) == 4 * 128


@pytest.fixture(scope="module")
def lib():
    kvbuild.build()
    return kv.library()


def test_library_exports_every_header_symbol(lib):
    hdr = open(os.path.join(ROOT, "include", "kvattn.h")).read()
    names = set(re.findall(r"^\s*(?:KVATTN_API\s+)?(?:int|size_t|const char\*)\s+(kvattn_\w+)\s*\(", hdr, re.M))
    assert {"kvattn_rope_append", "kvattn_decode", "kvattn_prefill_chunk"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert lib.kvattn_version() == 100


def test_status_strings(lib):
    assert kv.kvattn_status_string(0) == "ok"
    assert "workspace" in kv.kvattn_status_string(4)
    assert kv.kvattn_status_string(99) == "unknown status"


def _dims(**kw):
    base = dict(batch=2, n_heads=32, n_kv_heads=8, head_dim=128, max_seq_len=64)
    base.update(kw)
    return kv.kvattn_dims(**base)


FAKE = ctypes.c_void_p(0x10000)  # a non-null, aligned address; never dereferenced on these paths


@pytest.mark.parametrize("dims,expect", [
    (dict(n_heads=30), kv.KVATTN_ERR_INVALID_ARG),       # H % Hkv != 0
    (dict(head_dim=64), kv.KVATTN_ERR_UNSUPPORTED),
    (dict(batch=0), kv.KVATTN_ERR_INVALID_ARG),
    (dict(max_seq_len=0), kv.KVATTN_ERR_INVALID_ARG),
])
def test_rope_append_rejects_bad_dims(lib, dims, expect):
    d = _dims(**dims)
    rope = kv.LLAMA3.as_c()
    rc = lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(rope), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                FAKE, None, None)
    assert rc == expect


def test_rope_append_rejects_bad_pointers_and_params(lib):
    d = _dims()
    rope = kv.LLAMA3.as_c()
    args = [FAKE] * 7
    for i in range(7):
        a = list(args)
        a[i] = None
        assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(rope), 1, *a, None, None) == 1
    mis = ctypes.c_void_p(0x10008)                        # 8-byte aligned only
    assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(rope), 1, mis, *args[1:], None, None) == 1
    assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(rope), 0, *args, None, None) == 1
    assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(rope), 65, *args, None, None) == 3
    bad = kv.RopeParams(theta=-1.0).as_c()
    assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(bad), 1, *args, None, None) == 1
    bad = kv.RopeParams(use_scaled=True, high_freq_factor=0.5).as_c()
    assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(bad), 1, *args, None, None) == 1


def test_attention_entry_points_reject_bad_args(lib):
    d = _dims()
    P = [FAKE] * 4
    # group sizes that are not powers of two up to 128 are not built (48, 256)
    for bad_g in (_dims(n_heads=48, n_kv_heads=1), _dims(n_heads=256, n_kv_heads=1)):
        assert lib.kvattn_decode(ctypes.byref(bad_g), *P, 0, 0.0, FAKE, None, 0, None, None) == 2
        assert lib.kvattn_prefill_chunk(ctypes.byref(bad_g), 1, *P, 0, 0.0, FAKE, None, 0, None, None) == 2
    # null output
    assert lib.kvattn_decode(ctypes.byref(d), *P, 0, 0.0, None, None, 0, None, None) == 1
    # hint beyond the cache
    assert lib.kvattn_decode(ctypes.byref(d), *P, 65, 0.0, FAKE, None, 0, None, None) == 3
    # prefill: T < 1, and a hint shorter than the chunk
    assert lib.kvattn_prefill_chunk(ctypes.byref(d), 0, *P, 0, 0.0, FAKE, None, 0, None, None) == 1
    assert lib.kvattn_prefill_chunk(ctypes.byref(d), 8, *P, 4, 0.0, FAKE, None, 0, None, None) == 3


def test_rope_layout_and_rotary_dim_validation(lib):
    d = _dims()
    args = [FAKE] * 7
    for bad in (kv.RopeParams(layout=2), kv.RopeParams(rotary_dim=3), kv.RopeParams(rotary_dim=130),
                kv.RopeParams(rotary_dim=-2)):
        rope = bad.as_c()
        assert lib.kvattn_rope_append(ctypes.byref(d), ctypes.byref(rope), 1, *args, None, None) == 1


def test_fused_decode_rejects_bad_args(lib):
    d = _dims()
    rope = kv.LLAMA3.as_c()
    P7 = [FAKE] * 6  # k_new, v_new, cache_k, cache_v, start_pos
    # q_rot aliasing q is refused (other items still read q)
    assert lib.kvattn_decode_fused(ctypes.byref(d), ctypes.byref(rope), FAKE, FAKE, *P7[:5], 0, 0.0, FAKE, None, 0,
                                   None, None) == 1
    # a null q / out
    assert lib.kvattn_decode_fused(ctypes.byref(d), ctypes.byref(rope), None, None, *P7[:5], 0, 0.0, FAKE, None, 0,
                                   None, None) == 1
    assert lib.kvattn_decode_fused(ctypes.byref(d), ctypes.byref(rope), FAKE, None, *P7[:5], 0, 0.0, None, None, 0,
                                   None, None) == 1
    # group size 32 is not built; a bad rope layout
    d32 = _dims(n_heads=48, n_kv_heads=1)
    assert lib.kvattn_decode_fused(ctypes.byref(d32), ctypes.byref(rope), FAKE, None, *P7[:5], 0, 0.0, FAKE, None,
                                   0, None, None) == 2
    bad = kv.RopeParams(layout=5).as_c()
    assert lib.kvattn_decode_fused(ctypes.byref(d), ctypes.byref(bad), FAKE, None, *P7[:5], 0, 0.0, FAKE, None, 0,
                                   None, None) == 1
    # hint beyond the cache
    assert lib.kvattn_decode_fused(ctypes.byref(d), ctypes.byref(rope), FAKE, None, *P7[:5], 65, 0.0, FAKE, None, 0,
                                   None, None) == 3


def test_masked_entry_points_validate_the_mask(lib):
    d = _dims()
    P = [FAKE] * 4
    for bad in (kv.kvattn_attn_mask(-1, 0, None), kv.kvattn_attn_mask(8, -2, None),
                kv.kvattn_attn_mask(8, 0, 0x10002)):
        assert lib.kvattn_decode_masked(ctypes.byref(d), *P, 0, 0.0, ctypes.byref(bad), FAKE, None, 0, None,
                                        None) == 1
        assert lib.kvattn_prefill_chunk_masked(ctypes.byref(d), 1, *P, 0, 0.0, ctypes.byref(bad), FAKE, None, 0,
                                               None, None) == 1
        assert lib.kvattn_decode_masked_workspace_bytes(ctypes.byref(d), 0, ctypes.byref(bad)) == 0


def test_merge_grid_limits_refused_before_launch(lib):
    # The split-K merge runs one CTA per (row set, four heads): row sets on the
    # grid's x extent (B*T at most 2^24 here), head groups on its y extent
    # (heads capped at 65535).  Larger calls are refused on the host, before
    # the split kernel could be launched without the merge that clears its
    # work counter.
    P = [FAKE] * 4
    big_b = _dims(batch=(1 << 24) + 1)
    assert lib.kvattn_decode(ctypes.byref(big_b), *P, 0, 0.0, FAKE, None, 0, None, None) == 2
    many_heads = _dims(n_heads=65536 * 2, n_kv_heads=65536 * 2 // 4)
    assert lib.kvattn_decode(ctypes.byref(many_heads), *P, 0, 0.0, FAKE, None, 0, None, None) == 2
    noalloc = kv._load_noalloc()
    assert noalloc(ctypes.byref(many_heads), *P, 0, 0.0, FAKE, None, None) == 2
    assert noalloc(ctypes.byref(big_b), *P, 0, 0.0, FAKE, None, None) == 2
    rope = kv.LLAMA3.as_c()
    assert lib.kvattn_decode_fused(ctypes.byref(many_heads), ctypes.byref(rope), FAKE, None, *[FAKE] * 5, 0, 0.0,
                                   FAKE, None, 0, None, None) == 2
