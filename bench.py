#!/usr/bin/env python
"""Throughput benchmark of the TurboQuant-style KV-cache path on B200.

One step = the whole hot path over one decode layer shaped like
Llama-3.1-8B at 32k context (batch 8, 32 query heads, 8 KV heads, head_dim
128, bf16 K/V with Student-t(3) entries and 1% outlier channels x100):
  tq_quantize(K: 3-bit Lloyd-Max + QJL m=128), tq_quantize(V: 4-bit),
  tq_scores (logits of the 8x32 decode queries), tq_attend (decode attention).
The headline value is compressed keys processed per second (keys of the
layer / step time); per-stage figures, the roofline of the dominant kernel
and of the scoring kernel, an end-to-end figure through host buffers and the
CPU oracle's throughput on a bounded sample are reported alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]

Under torchrun (N > 1) every rank processes its own layer (independent data),
no collective touches the data path, and the step time is the maximum over
ranks (weak scaling).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "compressed keys scored/s and % of B200 HBM peak (32k ctx); tokens quantised/s"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ helpers
# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
# each stage's main kernel, from an ncu capture of that kernel, with the digest
# of the sources that capture measured.  A stage's figure is reported only while its sources (its
# kernel file plus the shared headers and host dispatch) still have that
# digest; after any change to them it is null until the capture is redone.
# (tq_kernels.cu holds the CUDA-core kernels and the attention's chunking and
# combine: it is part of the attention stage only; no measured main kernel of
# the other stages is compiled from it)
STEP_SHARED_SOURCES = ("tq_common.cuh", "tq_internal.h", "tq_tc.cuh", "tq_host.cpp", "tq_trace.h")
STAGE_SOURCES = {
    "tq_quantize_K": ("tq_quantize_tc.cu", "tq_quantize_tc.cuh"),
    "tq_quantize_V": ("tq_quantize_tc.cu", "tq_quantize_tc.cuh"),
    "tq_scores": ("tq_scores_tc.cu",),
    "tq_attend": ("tq_attend.cuh", "tq_attend_d128.cu", "tq_attend_d64.cu", "tq_kernels.cu"),
}
TRAFFIC = {  # stage: (bytes per launch, sources digest)
    "tq_quantize_K": (548_033_280 + 136_723_200, "60e1ebbf677f89535dcffe2d2e5732a96716f1153a8dd5f4d08bd95e315f0e4e"),
    "tq_quantize_V": (539_169_536 + 124_970_752, "60e1ebbf677f89535dcffe2d2e5732a96716f1153a8dd5f4d08bd95e315f0e4e"),
    "tq_scores": (152_425_216 + 16_209_152, "228a807d7a83dc7d46a04fb633a2a4483725173af5db74ea1b9696cc43088932"),
    "tq_attend": (294_011_648 + 1_265_408, "6f14879f48fe4937f67c34bdc801060ae9d7e9b9ef2b97183262a81c333d1867"),
}


def stage_sources_digest(stage: str) -> str:
    """sha256 over a stage's kernel sources, the shared headers, the host
    dispatch and tq.h (names + bytes)."""
    import hashlib
    csrc = os.path.join(ROOT, "kv_cache_vector_09_b200", "csrc")
    h = hashlib.sha256()
    for n in sorted(STEP_SHARED_SOURCES + STAGE_SOURCES[stage]):
        h.update(n.encode())
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    with open(os.path.join(ROOT, "include", "tq.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def measured_traffic(stage: str):
    if stage not in TRAFFIC:
        return None
    nbytes, digest = TRAFFIC[stage]
    return nbytes if stage_sources_digest(stage) == digest else None



def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Polls NVML for SM clock and clock-event reasons in a background thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                uuid = torch.cuda.get_device_properties(device_index).uuid
            except Exception:
                pass
            h = None
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nvml, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                mhz = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
                rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((t, mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside and self.samples:
            inside = [min(self.samples, key=lambda s: abs(s[0] - 0.5 * (t0 + t1)))]
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = sorted(v for k, v in self.REASONS.items() if bits & k and v != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


def max_over_ranks(dist, value: float, device) -> float:
    """Maximum of a per-rank scalar over all ranks (identity without a group)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """Each rank processes its own layer: same shapes, its own data seed."""
    import dataclasses
    return dataclasses.replace(w, data_seed=w.data_seed + rank)


def whole_job_value(units_per_rank: int, world: int, ms_max: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------- workload
class Layer:
    """Device-resident inputs, codecs and outputs of one decode layer."""

    def __init__(self, tq, w: synth.Workload, dev: torch.device, rank: int):
        self.w = w = rank_workload(w, rank)
        self.tq = tq
        d = w.d
        self.k_host = synth.kv_full(w, "K").reshape(-1, d)
        self.v_host = synth.kv_full(w, "V").reshape(-1, d)
        self.q_host = synth.queries(w)
        self.k = self.k_host.to(dev)
        self.v = self.v_host.to(dev)
        self.q = self.q_host.to(dev).contiguous()
        self.kc = tq.Codec(d, w.k_bits, w.k_m, w.codec_seed, device=dev.index)
        self.vc = tq.Codec(d, w.v_bits, w.v_m, w.codec_seed + 1, device=dev.index)
        n = w.n_keys
        self.K = tq.Compressed.empty(self.kc, n, dev)
        self.V = tq.Compressed.empty(self.vc, n, dev)
        self.logits = torch.empty((w.B, w.Hq, w.T), device=dev)
        self.out = torch.empty((w.B, w.Hq, d), device=dev)
        self.ws_s = tq.workspace(tq.tq_scores_workspace_size(self.kc, w.B, w.Hq, w.Hkv), dev)
        self.ws_a = tq.workspace(tq.tq_attend_workspace_size(self.kc, self.vc, w.B, w.Hq, w.Hkv, w.T), dev)

    def stages(self, k=None, v=None, q=None):
        tq, w = self.tq, self.w
        k = self.k if k is None else k
        v = self.v if v is None else v
        q = self.q if q is None else q
        return [
            ("tq_quantize_K", lambda: tq.tq_quantize(self.kc, k, self.K)),
            ("tq_quantize_V", lambda: tq.tq_quantize(self.vc, v, self.V)),
            ("tq_scores", lambda: tq.tq_scores(self.kc, q, w.B, w.Hq, w.Hkv, w.T, self.K, self.logits, self.ws_s)),
            ("tq_attend", lambda: tq.tq_attend(self.kc, self.vc, q, w.B, w.Hq, w.Hkv, w.T, self.K, self.V, self.out,
                                               self.ws_a)),
        ]

    # launches of libtq kernels per stage (quantize: 1; scores: query prep +
    # query-limb image + scoring; attend: query prep + fused attention +
    # combine)
    LAUNCHES = {"tq_quantize_K": 1, "tq_quantize_V": 1, "tq_scores": 3, "tq_attend": 3}

    def algorithmic_bytes(self):
        w, d = self.w, self.w.d
        n = w.n_keys
        esz = 2 if w.dtype == "bf16" else 4
        kc, vc = self.kc, self.vc
        krow = 4 * kc.code_words + 4 * kc.sign_words + 4 + (4 if kc.m else 0)
        vrow = 4 * vc.code_words + 4 * vc.sign_words + 4 + (4 if vc.m else 0)
        return {
            "tq_quantize_K": n * (d * esz + krow),
            "tq_quantize_V": n * (d * esz + vrow),
            "tq_scores": n * (krow + 4 * w.G),
            "tq_attend": n * (krow + vrow),
        }, {"key_row": krow, "value_row": vrow, "input_row": d * esz}


def time_steps(layer, steps: int, stream, stages=None, pre=None, post=None):
    """Times `steps` steps with CUDA events on `stream`; returns total ms and
    per-stage ms lists."""
    stages = stages or layer.stages()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(steps):
        if pre:
            pre()
        evs[s][0].record(stream)
        for i, (_, fn) in enumerate(stages):
            fn()
            evs[s][i + 1].record(stream)
        if post:
            post()
    end.record(stream)
    end.synchronize()
    total = start.elapsed_time(end)
    per = {name: [evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(steps)] for i, (name, _) in enumerate(stages)}
    return total, per


# ------------------------------------------------------------ CPU baseline
def cpu_oracle_sample(w: synth.Workload, budget_s: float, rank_seed: int = 0):
    """The oracle, as it stands, on bounded samples of the workload: whole
    (b, KV head) slabs cut to their first `tn` tokens, each quantised (K and V),
    scored for the G query heads and attended.  Returns (keys/s, seconds,
    keys, threads, description)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    d = w.d
    okc = O.make_codec(d, w.k_bits, w.k_m, w.codec_seed)
    ovc = O.make_codec(d, w.v_bits, w.v_m, w.codec_seed + 1) if w.v_bits else None
    qall = synth.queries(w).to(torch.float64).numpy()
    tn = 1024
    keys, secs, slabs = 0, 0.0, 0
    t_start = time.perf_counter()
    while secs < budget_s:
        b = slabs % w.B
        h = (slabs // w.B) % w.Hkv
        k = synth.kv_slab(w, "K", b, h, 0, tn).to(torch.float64).numpy()
        v = synth.kv_slab(w, "V", b, h, 0, tn).to(torch.float64).numpy() if ovc else None
        q = qall[b, h * w.G:(h + 1) * w.G][None]
        t0 = time.perf_counter()
        Ko = O.quantize(k, okc)
        if ovc is not None:
            Vo = O.quantize(v, ovc)
        O.estimate_scores(q, Ko, okc, 1, w.G, 1, tn)
        if ovc is not None:
            O.attend(q, Ko, Vo, okc, ovc, 1, w.G, 1, tn)
        secs += time.perf_counter() - t0
        keys += tn
        slabs += 1
        if time.perf_counter() - t_start > 4 * budget_s:
            break
    desc = (f"{slabs} (batch, KV head) slabs of the {w.name} layer cut to {tn} tokens: quantise K and V, "
            f"score {w.G} query heads, attend; keys/s = keys / oracle seconds")
    return keys / secs, secs, keys, threads, desc


# ------------------------------------------------------------ per-config
L2_FLUSH_BYTES = 256 << 20   # twice the B200's 126 MB L2


def timed_calls(fn, iters: int, stream, flush=None):
    """Per-call device times (ms) with CUDA events on `stream`; `flush` (a
    buffer larger than L2) is overwritten before every call, outside the
    timed interval."""
    out = []
    for _ in range(iters):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        out.append(a.elapsed_time(b))
    return out


def hbm_roof(nbytes: float, ms: float, hbm: float, peak_src: str):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
            "traffic": None, "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": nbytes}


def config_longctx(tq, dev, stream, flush, iters, hbm, peak_src):
    """Long-context scoring: 1 x 8 KV heads x 131072 keys (2 + 3 bits, m = 64),
    32 query heads, L2 flushed before every call."""
    w = synth.WORKLOADS["longctx"]
    kc = tq.Codec(w.d, w.k_bits, w.k_m, w.codec_seed, device=dev.index)
    K = tq.Compressed.empty(kc, w.n_keys, dev)
    for h in range(w.Hkv):
        tq.tq_quantize(kc, synth.kv_slab(w, "K", 0, h).to(dev), K.rows(h * w.T, (h + 1) * w.T))
    q = synth.queries(w).to(dev).contiguous()
    logits = torch.empty((w.B, w.Hq, w.T), device=dev)
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, w.B, w.Hq, w.Hkv), dev)
    fn = lambda: tq.tq_scores(kc, q, w.B, w.Hq, w.Hkv, w.T, K, logits, ws)
    for _ in range(3):
        fn()
    ms = statistics.median(timed_calls(fn, iters, stream, flush))
    if tq.tq_codec_device_error(kc) != 0:
        raise RuntimeError("tq_scores reported a timed-out wait (long context)")
    krow = 4 * kc.code_words + 4 * kc.sign_words + 8
    nbytes = w.n_keys * (krow + 4 * w.G)
    return {"workload": w.name, "call": "tq_scores", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T,
            "k_bits": list(w.k_bits), "k_m": w.k_m, "ms": round(ms, 5), "keys_per_s": w.n_keys / (ms * 1e-3),
            "unit": "keys/s", "key_row_bytes": krow, "l2": "256 MB written before every call (outside the timing)",
            "roofline": hbm_roof(nbytes, ms, hbm, peak_src)}


def config_esm_prefill(tq, dev, stream, flush, iters, hbm, peak_src):
    """Prefill quantisation, ESM-2-650M-shaped: K and V [4, 20, 4096, 64] bf16,
    2 bits + QJL m = 64.  Two forms: keys RoPE'd by the generator then
    tq_quantize, and raw keys through tq_quantize_rope (RoPE fused)."""
    import dataclasses
    w = synth.WORKLOADS["esm_prefill"]
    d, n = w.d, w.n_keys
    kc = tq.Codec(d, w.k_bits, w.k_m, w.codec_seed, device=dev.index)
    vc = tq.Codec(d, w.v_bits, w.v_m, w.codec_seed + 1, device=dev.index)
    k_rope = synth.kv_full(w, "K").reshape(-1, d).to(dev)
    k_raw = synth.kv_full(dataclasses.replace(w, rope=False), "K").reshape(-1, d).to(dev)
    v = synth.kv_full(w, "V").reshape(-1, d).to(dev)
    pos = (torch.arange(n, dtype=torch.int64, device=dev) % w.T).to(torch.int32)
    cs = tq.tq_rope_cache(w.rope_theta, d, w.T, device=dev)
    K, V = tq.Compressed.empty(kc, n, dev), tq.Compressed.empty(vc, n, dev)
    calls = {
        "K": lambda: tq.tq_quantize(kc, k_rope, K),
        "K_rope_fused": lambda: tq.tq_quantize_rope(kc, k_raw, cs, pos, K),
        "V": lambda: tq.tq_quantize(vc, v, V),
    }
    ms = {}
    for name, fn in calls.items():
        for _ in range(3):
            fn()
        ms[name] = statistics.median(timed_calls(fn, iters, stream, flush))
    for c in (kc, vc):
        if tq.tq_codec_device_error(c) != 0:
            raise RuntimeError("tq_quantize reported a device error (prefill)")
    tokens = w.B * w.T
    row_k = 4 * kc.code_words + 4 * kc.sign_words + 8
    row_v = 4 * vc.code_words + 4 * vc.sign_words + 8
    bytes_kv = n * (2 * d + row_k) + n * (2 * d + row_v)
    bytes_kv_fused = bytes_kv + 4 * n          # the positions
    sketch_flops = 2.0 * w.k_m * d * n + 2.0 * w.v_m * d * n
    t_plain, t_fused = ms["K"] + ms["V"], ms["K_rope_fused"] + ms["V"]
    return {"workload": w.name, "call": "tq_quantize K + V", "B": w.B, "H": w.Hkv, "T": w.T, "d": d,
            "bits": list(w.k_bits), "m": w.k_m, "tokens_per_call": tokens,
            "ms": {k: round(x, 5) for k, x in ms.items()},
            "tokens_quantised_per_s": tokens / (t_plain * 1e-3), "unit": "tokens/s",
            "tokens_quantised_per_s_rope_fused": tokens / (t_fused * 1e-3),
            "vectors_per_s": 2 * n / (t_plain * 1e-3),
            "sketch_tflops_achieved": round(sketch_flops / (t_plain * 1e-3) / 1e12, 3),
            "l2": "256 MB written before every call (outside the timing)",
            "roofline": hbm_roof(bytes_kv, t_plain, hbm, peak_src),
            "roofline_rope_fused": hbm_roof(bytes_kv_fused, t_fused, hbm, peak_src)}


def config_variants(tq, layer, dev, stream, flush, iters, hbm, peak_src):
    """The codec variants on one batch element of the Llama-8B layer (8 KV
    heads x 32768 keys, 32 query heads): tq_quantize of the keys and
    tq_scores over them, L2 flushed before every call.  Variants: the layer's
    own key codec (3 bits + QJL m = 128, randomized Hadamard), TurboESM's
    per-element residual sign (3 bits, S = I), the dense Haar rotation (3 bits
    + QJL), and FibQuant k = 2 at 2.5 bits per coordinate (32 codewords per
    2-coordinate block) + QJL."""
    w = layer.w
    d, n, Hq, Hkv = w.d, w.Hkv * w.T, w.Hq, w.Hkv
    k = layer.k[:n]                      # rows (0 * Hkv + h) * T + t: batch element 0
    q = layer.q[:1].contiguous()
    logits = torch.empty((1, Hq, w.T), device=dev)
    specs = {
        "rht_3bit_qjl128": dict(seg_bits=(3,), m=128),
        "sign_residual_3bit": dict(seg_bits=(3,), m=d, residual=tq.TQ_RESIDUAL_SIGN),
        "haar_3bit_qjl128": dict(seg_bits=(3,), m=128, rotation=tq.TQ_ROTATION_HAAR),
        "fibquant_2p5bit_qjl128": dict(seg_bits=(1,), m=128, vq_bits=5),
    }
    out = {"workload": "llama8b_decode, batch element 0", "keys": n, "Hq": Hq, "Hkv": Hkv, "T": w.T,
           "input_dtype": "bf16", "l2": "256 MB written before every call (outside the timing)"}
    for name, sp in specs.items():
        kc = tq.Codec(d, sp["seg_bits"], sp["m"], w.codec_seed, device=dev.index,
                      residual=sp.get("residual", tq.TQ_RESIDUAL_QJL), rotation=sp.get("rotation", tq.TQ_ROTATION_RHT),
                      vq_bits=sp.get("vq_bits", 0))
        K = tq.Compressed.empty(kc, n, dev)
        ws = tq.workspace(tq.tq_scores_workspace_size(kc, 1, Hq, Hkv), dev)
        fq = lambda: tq.tq_quantize(kc, k, K)
        fs = lambda: tq.tq_scores(kc, q, 1, Hq, Hkv, w.T, K, logits, ws)
        for _ in range(3):
            fq()
            fs()
        mq = statistics.median(timed_calls(fq, iters, stream, flush))
        ms = statistics.median(timed_calls(fs, iters, stream, flush))
        if tq.tq_codec_device_error(kc) != 0:
            raise RuntimeError(f"device error in the {name} variant")
        krow = 4 * kc.code_words + 4 * kc.sign_words + 8
        out[name] = {"quantize_ms": round(mq, 5), "scores_ms": round(ms, 5), "key_row_bytes": krow,
                     "keys_quantised_per_s": n / (mq * 1e-3), "keys_scored_per_s": n / (ms * 1e-3),
                     "roofline_quantize": hbm_roof(n * (2 * d + krow), mq, hbm, peak_src),
                     "roofline_scores": hbm_roof(n * (krow + 4 * (Hq // Hkv)), ms, hbm, peak_src)}
        del K, ws, kc
    return out


def config_vsearch(tq, dev, stream, iters):
    """Vector search over the 1M x 1536 compressed index, top-10 per query,
    with recall@10 against exact fp32 inner products computed on the GPU."""
    w = synth.VSEARCH
    codec = tq.Codec(w.d, w.bits, w.m, w.codec_seed, device=dev.index)
    X = tq.Compressed.empty(codec, w.n, dev)
    X32 = torch.empty((w.n, w.d), dtype=torch.float32, device=dev)
    for r0 in range(0, w.n, w.row_block):
        r1 = min(w.n, r0 + w.row_block)
        X32[r0:r1] = synth.search_rows(w, r0, r1).to(dev)
        tq.tq_quantize(codec, X32[r0:r1], X.rows(r0, r1))
    q = synth.search_queries(w).to(dev).contiguous()
    idx = torch.empty((w.nq, w.k), dtype=torch.int32, device=dev)
    sc = torch.empty((w.nq, w.k), dtype=torch.float32, device=dev)
    ws = tq.workspace(tq.tq_search_workspace_size(codec, w.nq, w.k), dev)
    fn = lambda: tq.tq_search_topk(codec, q, X, w.n, w.k, idx, sc, ws)
    for _ in range(2):
        fn()
    ms = statistics.median(timed_calls(fn, iters, stream))
    if tq.tq_codec_device_error(codec) != 0:
        raise RuntimeError("tq_search_topk reported a timed-out wait")
    # exact top-10 of the fp32 inner products, block by block
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    best_v = torch.full((w.nq, w.k), -float("inf"), device=dev)
    best_i = torch.zeros((w.nq, w.k), dtype=torch.int64, device=dev)
    for r0 in range(0, w.n, 131072):
        r1 = min(w.n, r0 + 131072)
        s = q @ X32[r0:r1].T
        v, i = torch.topk(s, w.k, dim=1)
        cv, ci = torch.cat([best_v, v], 1), torch.cat([best_i, i + r0], 1)
        best_v, sel = torch.topk(cv, w.k, dim=1)
        best_i = torch.gather(ci, 1, sel)
    torch.backends.cuda.matmul.allow_tf32 = prev
    got = idx.to(torch.int64)
    hits = (got[:, :, None] == best_i[:, None, :]).any(dim=2).sum().item()
    recall = hits / (w.nq * w.k)
    del X32
    peak, peak_src = load_tensor_peak()
    pairs = w.nq * w.n
    alg = 2.0 * (w.d + w.m) * pairs
    ach = alg / (ms * 1e-3) / 1e12
    return {"workload": w.name, "call": "tq_search_topk", "n": w.n, "nq": w.nq, "d": w.d, "bits": list(w.bits),
            "m": w.m, "k": w.k, "ms": round(ms, 4), "pairs_per_s": pairs / (ms * 1e-3), "unit": "pairs/s",
            "queries_per_s": w.nq / (ms * 1e-3), "recall_at_10": round(recall, 4),
            "recall_reference": "exact fp32 inner products of the uncompressed rows (torch.matmul on the GPU, "
                                "TF32 off), top-10 per query",
            "l2": "index 616 MB read per call, larger than L2",
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(ach / peak, 4), "traffic": None, "peak_source": peak_src,
                         "flops_per_launch": alg}}


def decode_append_step(tq, layer, dev, stream, iters, hbm, peak_src):
    """One decode step of the Llama-8B-shaped layer at 32k context: append the
    new token's key (RoPE at its position, fused) and value into their fixed
    slots, then tq_attend over the whole cache (the cache stays in HBM)."""
    w = layer.w
    d, rows = w.d, w.B * w.Hkv
    t = w.T - 1
    cs = tq.tq_rope_cache(10000.0, d, w.T, device=dev)
    kn = synth.gaussian_rows(31, rows, d, dtype=torch.bfloat16).to(dev)
    vn = synth.gaussian_rows(32, rows, d, dtype=torch.bfloat16).to(dev)

    def step():
        tq.tq_append(layer.kc, kn, t, w.T, layer.K, cs)
        tq.tq_append(layer.vc, vn, t, w.T, layer.V)
        tq.tq_attend(layer.kc, layer.vc, layer.q, w.B, w.Hq, w.Hkv, w.T, layer.K, layer.V, layer.out, layer.ws_a)

    for _ in range(3):
        step()
    ms = statistics.median(timed_calls(step, iters, stream))
    for c in (layer.kc, layer.vc):
        if tq.tq_codec_device_error(c) != 0:
            raise RuntimeError("append/attend reported a device error")
    krow = 4 * layer.kc.code_words + 4 * layer.kc.sign_words + 8
    vrow = 4 * layer.vc.code_words + 4 * layer.vc.sign_words + 4
    nbytes = w.n_keys * (krow + vrow) + rows * 2 * (2 * d + krow)
    return {"workload": w.name, "step": "tq_append K (RoPE fused) + tq_append V + tq_attend", "T": w.T,
            "ms": round(ms, 5), "decode_tokens_per_s": w.B / (ms * 1e-3), "unit": "tokens/s",
            "keys_attended_per_s": w.n_keys / (ms * 1e-3), "roofline": hbm_roof(nbytes, ms, hbm, peak_src)}


def run_configs(tq, layer, dev, stream, iters: int):
    hbm, peak_src = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {"decode_append_attend": decode_append_step(tq, layer, dev, stream, iters, hbm, peak_src)}
    out["longctx"] = config_longctx(tq, dev, stream, flush, iters, hbm, peak_src)
    out["esm_prefill"] = config_esm_prefill(tq, dev, stream, flush, iters, hbm, peak_src)
    out["variants"] = config_variants(tq, layer, dev, stream, flush, max(3, iters // 4), hbm, peak_src)
    del flush
    torch.cuda.empty_cache()
    out["vsearch"] = config_vsearch(tq, dev, stream, max(3, iters // 4))
    return out


# ------------------------------------------------------------------- main
def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 only, bounded samples per step."""
    if rank != 0:
        return 0
    if args.workload == "vsearch":
        w = synth.VSEARCH
        times, pairs_total = [], 0
        for s in range(args.warmup + args.steps):
            pps, secs, pairs, threads, desc = cpu_search_sample(w, args.ref_step_seconds)
            if s >= args.warmup:
                times.append(secs)
                pairs_total += pairs
        value = pairs_total / sum(times)
        print(json.dumps({
            "metric": SEARCH_METRIC, "value": value, "unit": "pairs/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "n": w.n, "nq": w.nq, "d": w.d, "bits": list(w.bits), "m": w.m, "k": w.k,
                       "step": "oracle top-k on a bounded sample per step"},
            "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return 0
    w = synth.WORKLOADS[args.workload]
    times, keys_total = [], 0
    for s in range(args.warmup + args.steps):
        kps, secs, keys, threads, desc = cpu_oracle_sample(w, args.ref_step_seconds)
        if s >= args.warmup:
            times.append(secs)
            keys_total += keys
    total = sum(times)
    value = keys_total / total
    line = {
        "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d,
                   "k_bits": list(w.k_bits), "k_m": w.k_m, "v_bits": list(w.v_bits), "input_dtype": w.dtype,
                   "step": "quantise K and V, score, attend (bounded sample per step)"},
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------- vector search
SEARCH_METRIC = "query-row pairs scored/s, top-10 search over a 1M-row compressed index (d=1536)"


def load_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), "measured bf16_tflops (burst; fp16 has the same dense rate)"
    except Exception:
        return 1590.0, "fallback 1.59 PFLOP/s"


def search_batches(nq: int, k: int) -> int:
    """Query batches of one tq_search_topk call: the library takes the largest
    multiple of 256 queries whose top-k lists (8k + 4 bytes per query) fit
    64 KB of shared memory, at least 256; each batch launches query prep,
    exponents, query image, search and merge (5 kernels)."""
    per = 8 * k + 4
    nb = max(256, (64 * 1024 // per) // 256 * 256)
    return -(-nq // nb)


def cpu_search_sample(w, budget_s: float):
    """The oracle's top-k on a bounded sample: a few queries against the first
    rows of the index (quantised by the oracle).  Returns (pairs/s, seconds,
    pairs, threads, description)."""
    import oracle as O
    oc = O.make_codec(w.d, w.bits, w.m, w.codec_seed)
    rows = 4096
    x = synth.search_rows(w, 0, rows).numpy()
    X = O.quantize(x, oc)
    q = synth.search_queries(w)[:64].numpy()
    t0 = time.perf_counter()
    done = 0
    while True:
        O.search_topk(q[done % 64:done % 64 + 4], X, oc, w.k)
        done += 4
        if time.perf_counter() - t0 > budget_s:
            break
    secs = time.perf_counter() - t0
    pairs = done * rows
    return pairs / secs, secs, pairs, torch.get_num_threads(), \
        f"{done} queries x {rows} rows of the index (oracle top-{w.k}, quantised by the oracle)"


def run_search(args, tq, dev, rank, world, pg):
    w = synth.VSEARCH
    codec = tq.Codec(w.d, w.bits, w.m, w.codec_seed, device=dev.index)
    X = tq.Compressed.empty(codec, w.n, dev)
    for r0 in range(0, w.n, w.row_block):
        r1 = min(w.n, r0 + w.row_block)
        tq.tq_quantize(codec, synth.search_rows(w, r0, r1).to(dev), X.rows(r0, r1))
    q_host = synth.search_queries(w)
    q = q_host.to(dev).contiguous()
    idx = torch.empty((w.nq, w.k), dtype=torch.int32, device=dev)
    sc = torch.empty((w.nq, w.k), dtype=torch.float32, device=dev)
    ws = tq.workspace(tq.tq_search_workspace_size(codec, w.nq, w.k), dev)
    stage = [("tq_search_topk", lambda: tq.tq_search_topk(codec, q, X, w.n, w.k, idx, sc, ws))]
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        stage[0][1]()
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(codec) == 0
    clocks = ClockSampler(dev.index)
    clocks.start()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    total_ms, per = time_steps(None, args.steps, stream, stage)
    t_wall1 = time.perf_counter()
    clocks.stop()
    ms_step = max_over_ranks(pg, total_ms / args.steps, dev)
    pairs = w.nq * w.n
    value = whole_job_value(pairs, world, ms_step)
    # end to end: queries from pinned host memory in, top-k lists out (the
    # index is the stored database and stays resident)
    qh = q_host.pin_memory()
    ih = torch.empty(idx.shape, dtype=torch.int32).pin_memory()
    sh = torch.empty(sc.shape, dtype=torch.float32).pin_memory()
    qd = torch.empty_like(q)

    def pre():
        qd.copy_(qh, non_blocking=True)

    def post():
        ih.copy_(idx, non_blocking=True)
        sh.copy_(sc, non_blocking=True)

    e2e_stage = [("tq_search_topk", lambda: tq.tq_search_topk(codec, qd, X, w.n, w.k, idx, sc, ws))]
    time_steps(None, 1, stream, e2e_stage, pre, post)
    e2e_steps = args.e2e_steps or args.steps
    e2e_ms, _ = time_steps(None, e2e_steps, stream, e2e_stage, pre, post)
    e2e_ms = max_over_ranks(pg, e2e_ms / e2e_steps, dev)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_src = load_tensor_peak()
    ms = statistics.mean(per["tq_search_topk"])
    alg_flops = 2.0 * (w.d + w.m) * pairs          # the dequantised contraction
    exec_flops = 3.0 * alg_flops                     # hi*hi + lo*hi + hi*lo
    ach = alg_flops / (ms * 1e-3) / 1e12
    line = {
        "metric": SEARCH_METRIC, "value": value, "unit": "pairs/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16x3 (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": w.name, "n": w.n, "nq": w.nq, "d": w.d, "bits": list(w.bits), "m": w.m, "k": w.k,
                   "parallelism": f"dp{world} (each rank searches its own copy)",
                   "l2": "index 616 MB read per step, larger than L2"},
        "queries_per_s": w.nq * world / (ms_step * 1e-3),
        "roofline": {"kernel": "tq_search_topk", "bound": "tensor", "achieved": round(ach, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None, "peak_source": peak_src,
                     "flops_per_launch": alg_flops, "executed_tensor_flops_per_launch": exec_flops},
        "gpu_launches": args.steps * 5 * search_batches(w.nq, w.k),
        "e2e": {"value": whole_job_value(pairs, world, e2e_ms), "unit": "pairs/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": qh.numel() * 4, "d2h_bytes_per_step": ih.numel() * 4 + sh.numel() * 4},
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    if world == 1 and not args.no_cpu_baseline:
        pps, secs, npairs, threads, desc = cpu_search_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": pps, "unit": "pairs/s", "cores": threads, "kind": "oracle", "sample": desc,
                                "seconds": round(secs, 2)}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", default="llama8b_decode")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0: same as --steps")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=3.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config-iters", type=int, default=20,
                    help="timed calls per per-config measurement (long context, prefill, search, decode "
                         "append); 0 skips them")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import kv_cache_vector_09_b200 as tq  # fails loudly without libtq.so
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    if args.workload == "vsearch":
        return run_search(args, tq, dev, rank, world, pg)
    w = synth.WORKLOADS[args.workload]
    layer = Layer(tq, w, dev, rank)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        for _, fn in layer.stages():
            fn()
    torch.cuda.synchronize()
    exact_k = tq.tq_codec_exact_rows(layer.kc, reset=True) / args.warmup
    exact_v = tq.tq_codec_exact_rows(layer.vc, reset=True) / args.warmup

    clocks = ClockSampler(local)
    clocks.start()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    total_ms, per = time_steps(layer, args.steps, stream)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    if pg:
        pg.barrier()
    clocks.stop()
    ms_step = max_over_ranks(pg, total_ms / args.steps, dev)
    keys_step = w.n_keys
    value = whole_job_value(keys_step, world, ms_step)

    # end to end through host buffers: pinned K, V, Q copied in, logits and the
    # attention output copied out, every step, on the same stream
    e2e_steps = args.e2e_steps or args.steps
    kh = layer.k_host.pin_memory()
    vh = layer.v_host.pin_memory()
    qh = layer.q_host.pin_memory()
    lh = torch.empty(layer.logits.shape, dtype=torch.float32).pin_memory()
    oh = torch.empty(layer.out.shape, dtype=torch.float32).pin_memory()
    kd, vd, qd = torch.empty_like(layer.k), torch.empty_like(layer.v), torch.empty_like(layer.q)

    def pre():
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        qd.copy_(qh, non_blocking=True)

    def post():
        lh.copy_(layer.logits, non_blocking=True)
        oh.copy_(layer.out, non_blocking=True)

    e2e_stages = layer.stages(kd, vd, qd)
    time_steps(layer, 1, stream, e2e_stages, pre, post)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    e2e_ms, _ = time_steps(layer, e2e_steps, stream, e2e_stages, pre, post)
    e2e_ms = max_over_ranks(pg, e2e_ms / e2e_steps, dev)
    h2d = kh.numel() * kh.element_size() + vh.numel() * vh.element_size() + qh.numel() * qh.element_size()
    d2h = lh.numel() * 4 + oh.numel() * 4
    del kd, vd
    # a kernel whose bounded wait gave up records it in its codec: such a run
    # measured nothing and must not print a number
    for c in (layer.kc, layer.vc):
        if tq.tq_codec_device_error(c) != 0:
            raise RuntimeError("a libtq kernel reported a timed-out wait during the benchmark")

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    configs = run_configs(tq, layer, dev, stream, args.config_iters) if world == 1 and args.config_iters > 0 else None

    hbm, peak_src = load_peaks()
    alg, rows = layer.algorithmic_bytes()
    stages = {}
    for name, lst in per.items():
        ms = statistics.mean(lst)
        gbs = alg[name] / (ms * 1e-3) / 1e9
        stages[name] = {"ms": round(ms, 5), "algorithmic_bytes": alg[name], "GB_s": round(gbs, 1),
                        "frac_hbm": round(gbs / hbm, 4), "launches": Layer.LAUNCHES[name]}
    dom = max(stages, key=lambda k: stages[k]["ms"])

    def roof(name):
        s = stages[name]
        return {"kernel": name, "bound": "hbm", "achieved": s["GB_s"], "peak": hbm, "unit": "GB/s",
                "frac": s["frac_hbm"], "traffic": measured_traffic(name), "peak_source": f"{peak_src} hbm_gbs",
                "bytes_per_launch": s["algorithmic_bytes"]}

    line = {
        "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d,
                   "k_bits": list(w.k_bits), "k_m": w.k_m, "v_bits": list(w.v_bits), "v_m": w.v_m,
                   "input_dtype": w.dtype, "parallelism": f"dp{world} (independent layers per rank)",
                   "step": "tq_quantize K, tq_quantize V, tq_scores, tq_attend",
                   "l2": "inputs larger than L2: 1.07 GB of bf16 K/V read per step",
                   "key_row_bytes": rows["key_row"], "value_row_bytes": rows["value_row"]},
        "stages": stages,
        "exact_rows_per_call": {"K": exact_k, "V": exact_v, "of": w.n_keys},
        "roofline": roof(dom),
        "roofline_scores": roof("tq_scores"),
        "gpu_launches": args.steps * sum(Layer.LAUNCHES.values()),
        "e2e": {"value": whole_job_value(keys_step, world, e2e_ms), "unit": "keys/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    if configs is not None:
        line["tokens_quantised_per_s"] = configs["esm_prefill"]["tokens_quantised_per_s"]
        line["configs"] = configs
    if world == 1 and not args.no_cpu_baseline:
        from threadpoolctl import threadpool_limits
        kps, secs, keys, threads, desc = cpu_oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": kps, "unit": "keys/s", "cores": threads, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2), "nproc": os.cpu_count()}
        with threadpool_limits(limits=1):
            kps1, secs1, _, _, _ = cpu_oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline_single_thread"] = {"value": kps1, "unit": "keys/s", "cores": 1, "kind": "oracle",
                                              "sample": desc, "seconds": round(secs1, 2)}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
