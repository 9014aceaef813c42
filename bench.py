#!/usr/bin/env python
"""Benchmark of the cached GQA attention step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One "step" is one pass of the whole hot path over one batch: for every layer,
RoPE + cache append (kvattn_rope_append) then attention (kvattn_decode: the
split-K kernel and its LSE merge kernel, or kvattn_prefill_chunk for the
prefill workload), each layer with its own cache.  Small, latency-bound
decode workloads can run the single-launch kvattn_decode_fused instead
(--path fused; the default split path measured faster at every size).  The default workload is batched ragged decode: B=64 sequences, 32
layers with separate [64, 8192, 8, 128] bf16 caches (64 GiB in HBM, far
larger than L2, so every step streams its K/V rows from HBM), start positions
uniform in [512, 8191].

Printed: one JSON line (rank 0) with the KV-cache GB/s of the whole job, the
decode-kernel roofline, end-to-end GB/s with host buffers, the fp64 oracle's
throughput on a bounded sample of host cores, and the SM clocks seen during
the timed region.  With N > 1 (torchrun) every rank runs an independent
replica on its own GPU; the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kvattn_synth as ks  # noqa: E402
from kvattn_synth.workloads import HEADLINE, WORKLOADS  # noqa: E402

METRIC = "GQA decode: KV-cache HBM GB/s (% of peak) and decode steps/s per layer"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------- helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


KERNEL_SOURCES = {
    "decode_splitk": ("decode.cu", "kvattn_device.cuh"),
    "decode_mma": ("decode.cu", "kvattn_device.cuh"),
    # multi-query decode (G = 32): the tcgen05 multi-query kernel + the LSE merge
    "decode_tc": ("mqa_decode.cu", "tc_device.cuh", "decode.cu", "kvattn_device.cuh"),
    "decode_fused": ("decode.cu", "kvattn_device.cuh", "rope_device.cuh"),
    "prefill_chunk": ("prefill.cu", "tc_device.cuh", "kvattn_device.cuh"),
}


def kernel_source_hash(kernel_tag: str):
    """Hash of the source files a kernel is built from (its .cu and the
    shared device header), to tell whether a recorded profile still applies."""
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "gqa_decode_attention_kvattn_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_tag]:
        with open(os.path.join(pkg, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture, if the kernels have
    not changed since: profiles/<kernel>__<workload>.md holds
    `traffic_bytes_per_launch:` and `source_hash:` lines."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}__{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line:
                k, _, v = line.partition(":")
                vals[k.strip().strip("-* `")] = v.strip().strip("` ")
    try:
        if vals.get("source_hash") != kernel_source_hash(kernel_tag):
            return None
        return float(vals["traffic_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd += ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def bus_id_of(dev):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ----------------------------------------------------------------- ranks
def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank contributes its own device-timed
    milliseconds and all of them get the maximum (replicas are timed as one
    job).  A no-op for a single process."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's
    time (weak scaling: each replica does the same work)."""
    return world * steps * units_per_rank_step / (max_ms / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- state
class Layer:
    pass


def l2_bytes(device) -> int:
    import torch
    try:
        return int(torch.cuda.get_device_properties(device).L2_cache_size)
    except Exception:
        return 126 << 20


def rotation_sets(w, kv_bytes_layer, device, rotate=0) -> int:
    """How many distinct copies of the step's caches to rotate through so that
    consecutive uses of one copy are more than twice the L2 size apart (a
    cold L2 for every step); a small latency-bound step (under 16 MB of K/V)
    rotates over at least 64 caches.  rotate > 0 forces a count."""
    if rotate > 0:
        return rotate
    step_bytes = max(1, w.layers * kv_bytes_layer)
    need = math.ceil(2 * l2_bytes(device) / step_bytes)
    if need <= 1:
        return 1
    if step_bytes < (16 << 20):
        need = max(need, math.ceil(64 / w.layers))
    return need


def build_state(w, seed, device, path="auto", sets=1):
    """Device state of the step: `sets` copies of the step's layers (each
    layer with its own caches and new q/k/v), the start positions, the
    workspace and the status word."""
    import torch
    import gqa_decode_attention_kvattn_b200 as kv
    sp = w.start_pos(seed)
    dsp = torch.from_numpy(sp).to(device)
    rope = kv.LLAMA3_1 if w.scaled_rope else kv.LLAMA3
    layer_sets = []
    for r in range(sets):
        layers = []
        for l in range(w.layers):
            g = r * w.layers + l   # distinct synthetic data per copy and layer
            L = Layer()
            L.q = torch.empty((w.B, w.T, w.H, 128), dtype=torch.bfloat16, device=device)
            L.k = torch.empty((w.B, w.T, w.Hkv, 128), dtype=torch.bfloat16, device=device)
            L.v = torch.empty_like(L.k)
            ks.device_normal_bf16(seed, ks.layer_stream(ks.STREAM_Q, g), L.q)
            ks.device_normal_bf16(seed, ks.layer_stream(ks.STREAM_K_NEW, g), L.k)
            ks.device_normal_bf16(seed, ks.layer_stream(ks.STREAM_V_NEW, g), L.v)
            L.ck = torch.empty((w.B, w.S, w.Hkv, 128), dtype=torch.bfloat16, device=device)
            L.cv = torch.empty_like(L.ck)
            ks.device_cache_fill(seed, ks.layer_stream(ks.STREAM_CACHE_K, g), L.ck, dsp)
            ks.device_cache_fill(seed, ks.layer_stream(ks.STREAM_CACHE_V, g), L.cv, dsp)
            L.q_rot = torch.empty_like(L.q)
            L.out = torch.empty_like(L.q)
            layers.append(L)
        layer_sets.append(layers)
    if path == "auto":
        # the split path (rope_append, decode, merge: three launches chained by
        # programmatic dependent launch) measured faster than the one-launch
        # fused decode at every size, the single sequence at p=1000 included
        # (14.4 against 20.3 us per layer in a 32-layer graph with a cold L2)
        path = "split"
    fused = w.kind == "decode" and path == "fused"
    if fused:
        ws_bytes = kv.kvattn_decode_fused_workspace_bytes(w.B, w.H, w.Hkv, w.S, w.kv_len_hint)
        ws = kv.alloc_fused_workspace(ws_bytes, device)   # zeroed once; every call leaves it zeroed
    else:
        if w.kind == "decode":
            ws_bytes = kv.kvattn_decode_workspace_bytes(w.B, w.H, w.Hkv, w.S, w.kv_len_hint)
        else:
            ws_bytes = kv.kvattn_prefill_workspace_bytes(w.B, w.H, w.Hkv, w.S, w.T, w.kv_len_hint)
        ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=device)  # counters start at zero
    status = torch.zeros(1, dtype=torch.int32, device=device)
    torch.cuda.synchronize(device)
    return dict(sp=sp, dsp=dsp, rope=rope, sets=layer_sets, layers=layer_sets[0], ws=ws, ws_bytes=ws_bytes,
                status=status, fused=fused)


def run_layer(w, st, L, ev=None):
    """One layer of the step on the current stream; `ev` = three events:
    before the rope call, between rope and attention, after attention (the
    fused path records the first and the last)."""
    import gqa_decode_attention_kvattn_b200 as kv
    if st["fused"]:
        # one launch: rope + append + split-K attention + merge
        if ev is not None:
            ev[0].record()
        kv.kvattn_decode_fused(L.q, L.k, L.v, L.ck, L.cv, st["dsp"], rope=st["rope"],
                               max_kv_len_hint=w.kv_len_hint, out=L.out, workspace=st["ws"],
                               dev_status=st["status"])
        if ev is not None:
            ev[2].record()
        return
    if ev is not None:
        ev[0].record()
    kv.kvattn_rope_append(L.q, L.k, L.v, L.ck, L.cv, st["dsp"], rope=st["rope"], q_rot=L.q_rot,
                          dev_status=st["status"])
    if ev is not None:
        ev[1].record()
    if w.kind == "decode":
        kv.kvattn_decode(L.q_rot, L.ck, L.cv, st["dsp"], max_kv_len_hint=w.kv_len_hint, out=L.out,
                         workspace=st["ws"], dev_status=st["status"])
    else:
        kv.kvattn_prefill_chunk(L.q_rot, L.ck, L.cv, st["dsp"], max_kv_len_hint=w.kv_len_hint, out=L.out,
                                workspace=st["ws"], dev_status=st["status"])
    if ev is not None:
        ev[2].record()


def run_step(w, st, layers, events=None):
    for i, L in enumerate(layers):
        run_layer(w, st, L, None if events is None else events[i])


def work_units(w, sp):
    """(algorithmic KV bytes, flops) of the attention of one layer."""
    import gqa_decode_attention_kvattn_b200 as kv
    return kv.attention_kv_bytes(sp, w.T, w.Hkv), kv.prefill_flops(sp, w.T, w.H)


# ----------------------------------------------------------------- CPU oracle
def oracle_sample_inputs_from_device(w, st, layer, seqs):
    """Host copies (exact bf16 bits) of the inputs of some sequences of one
    layer, taken before the step rewrites nothing they depend on."""
    import torch
    L = st["layers"][layer]
    out = []
    for b in seqs:
        spb = int(st["sp"][b])
        def h(t):
            return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        out.append((b, spb, h(L.q[b]), h(L.k[b]), h(L.v[b]), h(L.ck[b, :spb]), h(L.cv[b, :spb])))
    return out


def oracle_sample_inputs_host(w, seed, layer, seqs):
    """The same bits made by the host generator (no GPU involved)."""
    sp = w.start_pos(seed)
    d = 128
    out = []
    for b in seqs:
        spb = int(sp[b])
        q = ks.normal_bf16(seed, ks.layer_stream(ks.STREAM_Q, layer), b * w.T * w.H * d, w.T * w.H * d)
        k = ks.normal_bf16(seed, ks.layer_stream(ks.STREAM_K_NEW, layer), b * w.T * w.Hkv * d, w.T * w.Hkv * d)
        v = ks.normal_bf16(seed, ks.layer_stream(ks.STREAM_V_NEW, layer), b * w.T * w.Hkv * d, w.T * w.Hkv * d)
        ck = ks.cache_rows(seed, ks.layer_stream(ks.STREAM_CACHE_K, layer), b, w.S, w.Hkv, d, 0, spb, spb)
        cv = ks.cache_rows(seed, ks.layer_stream(ks.STREAM_CACHE_V, layer), b, w.S, w.Hkv, d, 0, spb, spb)
        out.append((b, spb, q.reshape(w.T, w.H, d), k.reshape(w.T, w.Hkv, d), v.reshape(w.T, w.Hkv, d), ck, cv))
    return out


def oracle_time(w, samples, rope_scaled):
    """Run the oracle (rope + append + attention) on each sampled sequence;
    return (seconds, KV bytes, flops)."""
    import oracle
    f = oracle.rope_freqs(128, 500000.0, rope_scaled)
    secs, nbytes, flops = 0.0, 0, 0
    for (b, spb, q, k, v, ck_rows, cv_rows) in samples:
        S = spb + w.T
        ck = np.zeros((1, S, w.Hkv, 128), np.uint16)
        cv = np.zeros((1, S, w.Hkv, 128), np.uint16)
        ck[0, :spb] = ck_rows
        cv[0, :spb] = cv_rows
        spa = np.array([spb], np.int32)
        t0 = time.perf_counter()
        _, _, rc = oracle.step(q[None].copy(), k[None].copy(), v[None].copy(), ck, cv, spa, f)
        secs += time.perf_counter() - t0
        assert rc == 0
        nbytes += 2 * w.Hkv * 128 * 2 * (spb + w.T) * w.T if w.kind == "prefill" else 2 * w.Hkv * 128 * 2 * (spb + 1)
        flops += 4 * 128 * w.H * (w.T * (spb + 1) + w.T * (w.T - 1) // 2)
    return secs, nbytes, flops


def cpu_baseline_leg(w, st, seed, target_s=12.0):
    import oracle
    cores = oracle.max_threads()
    seqs = list(range(w.B))
    total_s = total_b = total_f = 0.0
    layers_done = 0
    for layer in range(w.layers):
        samples = oracle_sample_inputs_from_device(w, st, layer, seqs)
        s, b, f = oracle_time(w, samples, w.scaled_rope)
        total_s += s
        total_b += b
        total_f += f
        layers_done += 1
        if total_s >= target_s or total_s * (layers_done + 1) / layers_done > 30.0:
            break
    if w.kind == "decode":
        value, unit = total_b / total_s / 1e9, "GB/s"
    else:
        value, unit = total_f / total_s / 1e12, "TFLOP/s"
    return {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"fp64 C oracle (rope+append+attention) on all {len(seqs)} sequences of "
                      f"{layers_done} of {w.layers} layer(s) of workload {w.name}, OpenMP over {cores} host threads; "
                      f"{total_s:.2f} s of oracle time"}


# ----------------------------------------------------------------- arms
def kernel_tag(w, st):
    """Which attention kernel the step runs: the profile file name's prefix."""
    import gqa_decode_attention_kvattn_b200 as kv
    if w.kind != "decode":
        return "prefill_chunk", "kvattn_prefill_chunk (tcgen05 prefill kernel)"
    if st["fused"]:
        return "decode_fused", "kvattn_decode_fused (rope + append + split-K attention + LSE merge, one kernel)"
    if w.H == 32 * w.Hkv:
        return "decode_tc", "kvattn_decode (tcgen05 multi-query kernel + LSE merge kernel)"
    plan = kv.kvattn_decode_plan(w.B, w.H, w.Hkv, w.S, w.kv_len_hint)
    if plan["tensor_cores"]:
        return "decode_mma", "kvattn_decode (warp-MMA split-K kernel + LSE merge kernel)"
    return "decode_splitk", "kvattn_decode (CUDA-core split-K kernel + LSE merge kernel)"


def spread(samples_ms):
    """median, p10, p90 of a list of milliseconds."""
    a = np.sort(np.asarray(samples_ms, np.float64))
    return float(np.median(a)), float(np.percentile(a, 10)), float(np.percentile(a, 90))


def run_ours(args, w, rank, world, device):
    import torch
    import gqa_decode_attention_kvattn_b200 as kv

    sp = w.start_pos(args.seed)
    kv_bytes_layer, flops_layer = work_units(w, sp)
    n_sets = rotation_sets(w, kv_bytes_layer, device, args.rotate)
    st = build_state(w, args.seed, device, args.path, n_sets)
    nl = w.layers
    merge = 1 if st["ws_bytes"] > 0 else 0
    launches_per_layer = 1 if st["fused"] else 2 + merge

    # warm-up, eager, over every copy of the caches
    for k in range(max(args.warmup, n_sets)):
        run_step(w, st, st["sets"][k % n_sets])
    torch.cuda.synchronize(device)
    if int(st["status"].item()) != 0:
        raise RuntimeError(f"device status {st['status'].item()} after warm-up")

    # Capture each copy's step twice: as it runs, and with timing events
    # around each rope and attention call.  Event nodes between the kernels
    # cut the programmatic launch overlap, so the timed region replays the
    # plain graphs and the per-kernel times come from separate replays of the
    # event graphs afterwards.
    events = [[tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)) for _ in range(nl)]
              for _ in range(n_sets)]
    graphs, graphs_ev = [], []
    if not args.no_graph:
        stream = torch.cuda.Stream(device)
        stream.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(stream):
            run_step(w, st, st["sets"][0])  # one more warm-up on the capture stream
        torch.cuda.current_stream(device).wait_stream(stream)
        torch.cuda.synchronize(device)
        for r in range(n_sets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run_step(w, st, st["sets"][r])
            ge = torch.cuda.CUDAGraph()
            with torch.cuda.graph(ge):
                run_step(w, st, st["sets"][r], events[r])
            graphs.append(g)
            graphs_ev.append(ge)
        for k in range(max(args.warmup, n_sets)):
            graphs[k % n_sets].replay()
        torch.cuda.synchronize(device)

    def step(k, timed_events=False):
        r = k % n_sets
        if graphs:
            (graphs_ev if timed_events else graphs)[r].replay()
        else:
            run_step(w, st, st["sets"][r], events[r] if timed_events else None)

    # ---------------- timed region
    barrier(world)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(bus_id_of(device))
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(args.steps):
        step(k)
    t1.record()
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    barrier(world)
    ms = t0.elapsed_time(t1)
    ms = max_over_ranks(ms, world, device)
    status = int(st["status"].item())

    # ---------------- per-kernel times: at least 50 event-carrying replays
    attn_ms, rope_ms = [], []
    reps = max(50, n_sets)
    for k in range(reps):
        step(k, timed_events=True)
        torch.cuda.synchronize(device)
        for e0, e1, e2 in events[k % n_sets]:
            if st["fused"]:
                attn_ms.append(e0.elapsed_time(e2))
            else:
                rope_ms.append(e0.elapsed_time(e1))
                attn_ms.append(e1.elapsed_time(e2))
    a_med, a_p10, a_p90 = spread(attn_ms)

    secs = ms / 1e3
    ms_per_step = ms / args.steps
    hbm_peak, tf_peak, peak_src = measured_peaks()
    tag, kname = kernel_tag(w, st)
    stats = {"avg_launch_ms": round(a_med, 5), "median_ms": round(a_med, 5), "p10_ms": round(a_p10, 5),
             "p90_ms": round(a_p90, 5), "samples": len(attn_ms), "replays": reps}
    if w.kind == "decode":
        value = job_throughput(nl * kv_bytes_layer, args.steps, world, ms) / 1e9
        unit = "GB/s"
        achieved = kv_bytes_layer / (a_med / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4),
                "traffic": profiled_traffic(tag, w.name), "kernel": kname,
                "peak_source": (f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else
                                f"fallback {FALLBACK_HBM_GBS:.0f} GB/s"),
                **stats, "bytes_per_launch": kv_bytes_layer,
                "achieved_p10_p90": [round(kv_bytes_layer / (a_p90 / 1e3) / 1e9, 1),
                                     round(kv_bytes_layer / (a_p10 / 1e3) / 1e9, 1)]}
    else:
        value = job_throughput(nl * flops_layer, args.steps, world, ms) / 1e12
        unit = "TFLOP/s"
        achieved = flops_layer / (a_med / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": tf_peak, "unit": "TFLOP/s",
                "frac": round(achieved / tf_peak, 4),
                "traffic": profiled_traffic(tag, w.name), "kernel": kname,
                "peak_source": (f"{peak_src} (MEASURED_PEAKS.json bf16_tflops)" if peak_src == "measured" else
                                f"fallback {FALLBACK_BF16_TFLOPS:.0f} TFLOP/s"),
                **stats, "flops_per_launch": flops_layer,
                "achieved_p10_p90": [round(flops_layer / (a_p90 / 1e3) / 1e12, 2),
                                     round(flops_layer / (a_p10 / 1e3) / 1e12, 2)]}
    rope = None
    if rope_ms:
        r_med, r_p10, r_p90 = spread(rope_ms)
        # bytes one rope_append call moves: q in, q_rot out, k_new and v_new in,
        # the new K and V rows out
        rope_bytes = w.B * w.T * (2 * w.H + 4 * w.Hkv) * 128 * 2
        rope = {"kernel": "kvattn_rope_append", "median_ms": round(r_med, 5), "p10_ms": round(r_p10, 5),
                "p90_ms": round(r_p90, 5), "samples": len(rope_ms), "bytes_per_launch": rope_bytes,
                "achieved_gbs": round(rope_bytes / (r_med / 1e3) / 1e9, 1)}

    # ---------------- end to end with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, st, device, kv_bytes_layer, flops_layer, world)

    step_bytes = nl * kv_bytes_layer
    line = {
        "metric": METRIC if w.kind == "decode" else "GQA chunked prefill: attention TFLOP/s (% of bf16 tensor peak)",
        "value": round(value, 2), "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.B, "new_tokens": w.T, "q_heads": w.H, "kv_heads": w.Hkv,
                   "head_dim": 128, "cache_rows": w.S, "layers": nl,
                   "start_pos": f"uniform [{w.sp_lo}, {w.sp_hi}] seed {args.seed}" if w.sp_lo != w.sp_hi else w.sp_lo,
                   "rope": "llama3.1 scaled, theta 500000" if w.scaled_rope else "theta 500000",
                   "l2": (f"inputs larger than L2 ({step_bytes / 1e6:.0f} MB of K/V per step)" if n_sets == 1 else
                          f"cold L2: {n_sets} copies of the step's caches rotated, "
                          f"{n_sets * step_bytes / 1e6:.0f} MB of K/V between reuses"),
                   "cache_copies": n_sets,
                   "graph": bool(graphs),
                   "path": "fused" if st["fused"] else "rope_append + " + ("decode" if w.kind == "decode" else "prefill"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_hbm_peak": round(100 * (value / world) / hbm_peak, 2) if w.kind == "decode" else None,
        "layer_steps_per_s": round(world * args.steps * nl / secs, 1),
        "us_per_layer": round(1e3 * ms_per_step / nl, 3),
        "steps_per_s": round(world * args.steps / secs, 2),
        "roofline": roof,
        "gpu_launches": args.steps * nl * launches_per_layer,
        "clocks": clocks,
        "device_status": status,
    }
    if rope is not None:
        line["rope_append"] = rope
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(w, st, args.seed)
    return line


def run_e2e(args, w, st, device, kv_bytes_layer, flops_layer, world):
    """Same step through the C ABI with host buffers: every step copies its
    inputs (q, k_new, v_new of every layer, start_pos) from pinned host memory
    and reads every layer's output back.  The copies run on two copy streams
    (one per direction) so that they overlap the attention of other layers:
    layer i waits only for its own inputs, and its output goes back while
    layer i+1 computes; the step ends when the last copy has landed."""
    import torch
    import torch.distributed as dist
    layers = st["layers"]
    h_in = [(L.q.cpu().pin_memory(), L.k.cpu().pin_memory(), L.v.cpu().pin_memory()) for L in layers]
    h_out = [torch.empty_like(L.out, device="cpu").pin_memory() for L in layers]
    h_sp = torch.from_numpy(st["sp"]).pin_memory()

    h2d_s = torch.cuda.Stream(device)
    d2h_s = torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in layers]
    ev_done = [torch.cuda.Event() for _ in layers]

    def e2e_step():
        cur = torch.cuda.current_stream(device)
        h2d_s.wait_stream(cur)
        d2h_s.wait_stream(cur)
        with torch.cuda.stream(h2d_s):
            st["dsp"].copy_(h_sp, non_blocking=True)
            for i, ((hq, hk, hv), L) in enumerate(zip(h_in, layers)):
                L.q.copy_(hq, non_blocking=True)
                L.k.copy_(hk, non_blocking=True)
                L.v.copy_(hv, non_blocking=True)
                ev_in[i].record(h2d_s)
        for i, (ho, L) in enumerate(zip(h_out, layers)):
            cur.wait_event(ev_in[i])
            run_layer(w, st, L)
            ev_done[i].record(cur)
            d2h_s.wait_event(ev_done[i])
            with torch.cuda.stream(d2h_s):
                ho.copy_(L.out, non_blocking=True)
        cur.wait_stream(h2d_s)
        cur.wait_stream(d2h_s)

    steps = max(3, args.steps // 2)
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(stream):
        e2e_step()
    torch.cuda.current_stream(device).wait_stream(stream)
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        e2e_step()
    graph.replay()
    torch.cuda.synchronize(device)
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        graph.replay()
    t1.record()
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1)
    ms = max_over_ranks(ms, world, device)
    secs = ms / 1e3
    h2d = sum(x.numel() * x.element_size() for trip in h_in for x in trip) + h_sp.numel() * 4
    d2h = sum(x.numel() * x.element_size() for x in h_out)
    nl = len(layers)
    if w.kind == "decode":
        val, unit = world * steps * nl * kv_bytes_layer / secs / 1e9, "GB/s"
    else:
        val, unit = world * steps * nl * flops_layer / secs / 1e12, "TFLOP/s"
    return {"value": round(val, 2), "unit": unit, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": steps, "ms_per_step": round(ms / steps, 5)}


def run_reference(args, w):
    """The fp64 oracle, as it stands, on the host cores: each step runs it on
    a bounded sample (the first sequences of layer 0) of the workload."""
    import oracle
    cores = oracle.max_threads()
    nseq = min(w.B, 16 if w.kind == "decode" else 1)
    seqs = list(range(nseq))
    try:
        import torch
        if torch.cuda.is_available():
            st = build_state_sample(w, args.seed, seqs)
            samples = st
        else:
            samples = oracle_sample_inputs_host(w, args.seed, 0, seqs)
    except Exception:
        samples = oracle_sample_inputs_host(w, args.seed, 0, seqs)
    for _ in range(args.warmup):
        oracle_time(w, samples, w.scaled_rope)
    tot_s = tot_b = tot_f = 0.0
    for _ in range(args.steps):
        s, b, f = oracle_time(w, samples, w.scaled_rope)
        tot_s += s
        tot_b += b
        tot_f += f
    if w.kind == "decode":
        value, unit = tot_b / tot_s / 1e9, "GB/s"
    else:
        value, unit = tot_f / tot_s / 1e12, "TFLOP/s"
    sample = (f"fp64 C oracle (rope+append+attention) on sequences {seqs[0]}..{seqs[-1]} of layer 0 of "
              f"workload {w.name} per step, OpenMP over {cores} host threads")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": unit, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.B, "new_tokens": w.T, "q_heads": w.H, "kv_heads": w.Hkv,
                       "head_dim": 128, "cache_rows": w.S, "layers": w.layers},
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def build_state_sample(w, seed, seqs):
    """Inputs of the sampled sequences of layer 0, made by the device
    generator and copied to the host (exact bits; no product kernel runs)."""
    import torch
    dev = torch.device("cuda", 0)
    sp = w.start_pos(seed)
    d = 128
    out = []
    for b in seqs:
        spb = int(sp[b])
        def gen(stream, shape, offset):
            t = torch.empty(shape, dtype=torch.bfloat16, device=dev)
            ks.device_normal_bf16(seed, stream, t, offset=offset)
            return t.view(torch.int16).cpu().numpy().view(np.uint16)
        q = gen(ks.layer_stream(ks.STREAM_Q, 0), (w.T, w.H, d), b * w.T * w.H * d)
        k = gen(ks.layer_stream(ks.STREAM_K_NEW, 0), (w.T, w.Hkv, d), b * w.T * w.Hkv * d)
        v = gen(ks.layer_stream(ks.STREAM_V_NEW, 0), (w.T, w.Hkv, d), b * w.T * w.Hkv * d)
        row = w.Hkv * d
        ck = gen(ks.layer_stream(ks.STREAM_CACHE_K, 0), (spb, w.Hkv, d), b * w.S * row) if spb else \
            np.zeros((0, w.Hkv, d), np.uint16)
        cv = gen(ks.layer_stream(ks.STREAM_CACHE_V, 0), (spb, w.Hkv, d), b * w.S * row) if spb else \
            np.zeros((0, w.Hkv, d), np.uint16)
        out.append((b, spb, q, k, v, ck, cv))
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE)
    ap.add_argument("--seed", type=int, default=ks.DEFAULT_SEED)
    ap.add_argument("--path", choices=["auto", "fused", "split"], default="auto",
                    help="decode entry points: rope_append + decode (+ merge kernel), or one kvattn_decode_fused "
                         "launch per layer; auto takes the split path (measured faster at every size)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (small profiling cases)")
    ap.add_argument("--rotate", type=int, default=0,
                    help="copies of the step's caches to rotate through (0: enough for a cold L2 each step)")
    ap.add_argument("--all", action="store_true",
                    help="run every workload (each with these options) and print one JSON line per workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]
    if args.layers > 0:
        import dataclasses
        w = dataclasses.replace(w, layers=args.layers)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, w)), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    import gqa_decode_attention_kvattn_b200 as kv
    kv.library()  # fail loudly when the CUDA library is missing
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    names = sorted(WORKLOADS) if args.all else [w.name]
    try:
        for name in names:
            wl = WORKLOADS[name] if args.all else w
            if args.all and args.layers > 0:
                import dataclasses
                wl = dataclasses.replace(wl, layers=args.layers)
            line = run_ours(args, wl, rank, world, device)
            if rank == 0:
                print(json.dumps(line), flush=True)
            torch.cuda.empty_cache()
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
