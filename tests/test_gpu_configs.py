"""GPU parity at the full sizes of every workload, in the launch
configuration the benchmark times (same shapes, same kv-length hint, device
generated inputs), on sampled sequences the oracle computes one by one."""
import numpy as np
import pytest

import kvattn_synth as ks
from kvattn_synth.workloads import WORKLOADS
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
kv = pytest.importorskip("gqa_decode_attention_kvattn_b200")

SEED = ks.DEFAULT_SEED


def _layer_tensors(w, layer, dsp):
    dev = "cuda"
    q = torch.empty((w.B, w.T, w.H, 128), dtype=torch.bfloat16, device=dev)
    k = torch.empty((w.B, w.T, w.Hkv, 128), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    ks.device_normal_bf16(SEED, ks.layer_stream(ks.STREAM_Q, layer), q)
    ks.device_normal_bf16(SEED, ks.layer_stream(ks.STREAM_K_NEW, layer), k)
    ks.device_normal_bf16(SEED, ks.layer_stream(ks.STREAM_V_NEW, layer), v)
    ck = torch.empty((w.B, w.S, w.Hkv, 128), dtype=torch.bfloat16, device=dev)
    cv = torch.empty_like(ck)
    ks.device_cache_fill(SEED, ks.layer_stream(ks.STREAM_CACHE_K, layer), ck, dsp)
    ks.device_cache_fill(SEED, ks.layer_stream(ks.STREAM_CACHE_V, layer), cv, dsp)
    return q, k, v, ck, cv


def _sample(w, sp):
    if w.B <= 4:
        return list(range(w.B))
    rng = np.random.default_rng(0)
    pick = {0, w.B - 1, int(np.argmin(sp)), int(np.argmax(sp))}
    pick |= set(int(x) for x in rng.choice(w.B, 4, replace=False))
    limit = 3 if w.S > 100000 else 8
    return sorted(pick)[:limit]


@pytest.mark.parametrize("name,layer", [
    ("decode_p1000_b1", 0),
    ("decode_ragged_b64_l32", 0),
    ("decode_ragged_b64_l32", 31),
    ("prefill_b4_t512_sp3584", 0),
    ("decode_long_scaled_b8", 0),
    ("decode_wide_g8_b128", 0),
    ("decode_mqa_g32_b64", 0),
    ("decode_mha_g1_b16", 0),
    ("decode_g2_b64", 0),
])
def test_workload_full_size(name, layer):
    w = WORKLOADS[name]
    sp = w.start_pos(SEED)
    dsp = torch.from_numpy(sp).cuda()
    rope = kv.LLAMA3_1 if w.scaled_rope else kv.LLAMA3
    q, k, v, ck, cv = _layer_tensors(w, layer, dsp)
    seqs = _sample(w, sp) if w.kind == "decode" else [0, w.B - 1]
    # host copies of the sampled sequences' inputs before the step
    host = {}
    for b in seqs:
        spb = int(sp[b])
        host[b] = (U.to_host(q[b]), U.to_host(k[b]), U.to_host(v[b]), U.to_host(ck[b, :spb]),
                   U.to_host(cv[b, :spb]))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_rot = kv.kvattn_rope_append(q, k, v, ck, cv, dsp, rope=rope, dev_status=status)
    if w.kind == "decode":
        out = kv.kvattn_decode(q_rot, ck, cv, dsp, max_kv_len_hint=w.kv_len_hint, dev_status=status)
    else:
        out = kv.kvattn_prefill_chunk(q_rot, ck, cv, dsp, max_kv_len_hint=w.kv_len_hint, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for b in seqs:
        spb = int(sp[b])
        hq, hk, hv, hck, hcv = host[b]
        o_qrot, o_krows, o_out = U.oracle_sequence(hq, hk, hv, hck, hcv, spb, w.T, rope)
        assert U.ulp_distance(U.to_host(q_rot[b]), o_qrot).max() <= 1
        assert U.ulp_distance(U.to_host(ck[b, spb:spb + w.T]), o_krows).max() <= 1
        assert np.array_equal(U.to_host(cv[b, spb:spb + w.T]), hv)
        # the rows before start_pos are untouched
        assert np.array_equal(U.to_host(ck[b, :spb]), hck)
        U.assert_attention_close(U.to_host(out[b]), o_out, f"{name} layer {layer} seq {b} sp {spb}")
    del q, k, v, ck, cv, q_rot, out
    torch.cuda.empty_cache()
