"""GPU parity of the optional masks (sliding window, attention sinks, learned
sinks) against the fp64 oracle: decode (CUDA-core and tensor-core kernels,
one and several splits) and chunked prefill, at shapes whose windows and
sink segments start and end inside and on 64-row tile boundaries."""
import numpy as np
import pytest

import oracle
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")


def _sinks(H, seed):
    rng = np.random.default_rng(seed)
    return rng.uniform(-2.0, 3.0, H)


def _run(kind, B, T, H, Hkv, S, sp, window, n_sink, sinks, seed=61, hint=0):
    q, k, v, ck, cv = U.host_inputs(seed, B, T, H, Hkv, S, sp)
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck, cv))
    dsp = torch.from_numpy(np.asarray(sp, np.int32)).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_rot = kv.kvattn_rope_append(dq, dk, dv, dck, dcv, dsp, dev_status=st)
    ds = None if sinks is None else torch.tensor(sinks, dtype=torch.float32, device="cuda")
    fn = kv.kvattn_decode if kind == "decode" else kv.kvattn_prefill_chunk
    out = fn(q_rot, dck, dcv, dsp, max_kv_len_hint=hint, dev_status=st, window=window, n_sink=n_sink,
             sink_logits=ds)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o_ck, o_cv = ck.copy(), cv.copy()
    # the oracle takes the sink logits in fp64; the GPU reads them as fp32
    sl = None if sinks is None else np.asarray(sinks, np.float32).astype(np.float64)
    _, ref, rc = oracle.step(q, k, v, o_ck, o_cv, np.asarray(sp, np.int32), U.oracle_freqs(kv.LLAMA3),
                             window=window, n_sink=n_sink, sink_logits=sl)
    assert rc == 0
    U.assert_attention_close(U.to_host(out), ref, f"{kind} W={window} sinks={n_sink} learned={sinks is not None}")


@pytest.mark.parametrize("window,n_sink,learned", [
    (100, 0, False),      # window only, not 64-aligned
    (64, 4, False),       # sinks, then the window (two segments)
    (200, 70, False),     # sink segment longer than one tile
    (1, 0, False),        # the token alone
    (1, 3, True),         # the token, three sinks, learned sinks
    (5000, 8, False),     # window longer than every sequence: all rows
    (0, 0, True),         # learned sinks only
    (300, 250, False),    # sinks and window overlap (one segment with a short gap)
])
@pytest.mark.parametrize("H,Hkv", [(32, 8), (64, 8), (32, 2), (32, 1)])
def test_decode_masks(window, n_sink, learned, H, Hkv):
    sp = [0, 63, 64, 700, 1999]
    sinks = _sinks(H, 3) if learned else None
    _run("decode", len(sp), 1, H, Hkv, 2000, sp, window, n_sink, sinks)


@pytest.mark.parametrize("window,n_sink", [(96, 4), (1500, 16), (4000, 0)])
def test_decode_masks_many_splits(window, n_sink):
    # long rows: the plan splits each sequence's visible rows across CTAs
    sp = [20000, 12345, 4096]
    _run("decode", len(sp), 1, 32, 8, 20001, sp, window, n_sink, _sinks(32, 5), seed=62)


@pytest.mark.parametrize("window,n_sink,learned", [
    (100, 0, False), (64, 4, True), (300, 130, False), (1, 2, False), (10000, 0, True), (0, 0, True),
])
@pytest.mark.parametrize("T,H,Hkv", [(77, 32, 8), (20, 64, 8), (130, 8, 8)])
def test_prefill_masks(window, n_sink, learned, T, H, Hkv):
    sp = [0, 400]
    sinks = _sinks(H, 4) if learned else None
    _run("prefill", len(sp), T, H, Hkv, 700, sp, window, n_sink, sinks, seed=63)


def test_window_reads_only_visible_rows_so_garbage_elsewhere_is_harmless():
    """Rows outside the window and the sinks may hold anything (here NaN)."""
    B, H, Hkv, S = 2, 32, 8, 3000
    sp = [2999, 1500]
    q, k, v, ck, cv = U.host_inputs(64, B, 1, H, Hkv, S, sp)
    nan_bits = np.uint16(0x7FC0)
    W, ns = 500, 10
    ck_bad, cv_bad = ck.copy(), cv.copy()
    for b in range(B):
        p = sp[b]
        ck_bad[b, ns:p - W + 1 - 64] = nan_bits   # rows neither sinks nor window, beyond the tile rounding
        cv_bad[b, ns:p - W + 1 - 64] = nan_bits
    dq, dk, dv, dck, dcv = (U.to_dev(x) for x in (q, k, v, ck_bad, cv_bad))
    dsp = torch.from_numpy(np.asarray(sp, np.int32)).cuda()
    q_rot = kv.kvattn_rope_append(dq, dk, dv, dck, dcv, dsp)
    out = kv.kvattn_decode(q_rot, dck, dcv, dsp, window=W, n_sink=ns)
    torch.cuda.synchronize()
    o_ck, o_cv = ck.copy(), cv.copy()
    _, ref, rc = oracle.step(q, k, v, o_ck, o_cv, np.asarray(sp, np.int32), U.oracle_freqs(kv.LLAMA3),
                             window=W, n_sink=ns)
    assert rc == 0
    U.assert_attention_close(U.to_host(out), ref, "garbage outside the window")
