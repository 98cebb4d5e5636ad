#!/usr/bin/env python
"""Benchmark of the flexq hot path on B200.

Metric: decode tokens/s per OPT layer-step (and int4 compress/decompress GB/s), as a
fraction of the HBM roofline.

Default workload (``opt-1.3b``): OPT-1.3B-shaped decoder layers (h 2048, 32 heads x 64,
FFN 8192), a stack of 24 distinct layers with their own weights and int4 KV caches,
batch 32, prompt 512 then 32 decode steps; weights int4 group 64, KV int4 group 64,
seeded synthetic data. The prompt is prefilled once (setup); one benchmark *step*
is the whole decode phase of that workload - 32 new tokens for the 32 sequences
through the 24-layer stack (positions 512..543), i.e. 24,576 layer-tokens, replayed
from CUDA graphs. The stack touches ~1.6 GB per token step, more than L2, so no
flush is needed between steps.

Also measured in the same run (``parts``): the prefill of the prompt through the
stack, the codec on a 1 GiB tensor, and every kernel of the decode step timed on its
own in the launch configuration the step uses (this gives the roofline object).

``--impl reference`` times the CPU oracle (the only other implementation; there is no
installable reference) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s per OPT layer-step"
UNIT = "layer-tokens/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="flexq", choices=["flexq", "reference"])
    ap.add_argument("--workload", default="opt-1.3b", choices=["opt-125m", "opt-1.3b", "opt-30b", "opt-175b"])
    ap.add_argument("--layers", type=int, default=None, help="stack depth (default: per workload)")
    ap.add_argument("--no-parts", action="store_true", help="skip the per-part measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--codec-only", action="store_true",
                    help="measure only flexq_compress / flexq_decompress on 1 GiB and print them as one JSON line")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while it runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=2)

    def summary(self, t0=None, t1=None):
        rows = []
        for ts, line in self.lines:
            if t0 is not None and (ts < t0 or ts > t1):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if not rows and t0 is not None:
            return self.summary()
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for name, val in zip(names, r[3][1:]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------------
def max_over_ranks(ms, world, device):
    """Elapsed time of the job: the slowest rank's (an all-reduce MAX; a no-op at N=1)."""
    if world == 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, units_per_step, steps, ms):
    """Units all ranks processed per second: every replica does units_per_step per step."""
    return world * units_per_step * steps / (ms / 1e3)


def bench_config(args, cfg, world):
    L, b, s, nsteps = cfg["layers"], cfg["batch"], cfg["prompt"], cfg["decode_steps"]
    return {"workload": f"{args.workload} decode: {L} distinct layers, batch {b}, prompt {s}, "
                        f"{nsteps} decode steps (positions {s}..{s + nsteps - 1}), int4 g64 weights and KV",
            "batch": b, "prompt": s, "decode_steps": nsteps, "layers": L, "h": cfg["h"],
            "units_per_step": b * nsteps * L,
            "l2": "not flushed: each token step streams ~%.1f GB (> 126 MB L2)" %
                  (decode_bytes_per_layer_step(cfg, s) * L / 1e9),
            "parallelism": f"replicas x{world}"}


def workload_cfg(name, layers=None):
    import synth
    cfg = dict(synth.WORKLOADS[name])
    if layers is not None:
        cfg["layers"] = layers
    return cfg


def decode_bytes_per_layer_step(cfg, pos, bits=4):
    """Algorithmic HBM bytes of one decode layer-step at position pos (int4 g64):
    weights 12h^2*0.5625, KV read 2*b*pos*h*0.5625, KV write 2*b*h*0.5625,
    activations in/out 4*b*h, biases and LayerNorm ~(9h + ffn)*2."""
    h, ffn, b = cfg["h"], cfg["ffn"], cfg["batch"]
    per = 0.5 + 4 / 64 if bits == 4 else 1 + 4 / 64
    w = (3 * h * h + h * h + 2 * h * ffn) * per
    kv = 2 * b * pos * h * per + 2 * b * h * per
    act = 4 * b * h
    small = (9 * h + ffn) * 2
    return w + kv + act + small


def run_flexq(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import group_wise_int4_b200 as fq
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    peaks = measured_peaks()
    cfg = workload_cfg(args.workload, args.layers)
    L, b, s, h, nh, d = cfg["layers"], cfg["batch"], cfg["prompt"], cfg["h"], cfg["n_heads"], cfg["head_dim"]
    nsteps = cfg["decode_steps"]
    max_seq = s + nsteps
    seed = cfg["seed"]

    # ---- build the stack: compressed weights (flexq_compress on the GPU) and caches
    layers, caches = [], []
    for l in range(L):
        raw = synth.layer_params(h, cfg["ffn"], seed * 100 + l, device=dev)
        layers.append(fq.FlexLayer(raw, nh, device=dev))
        del raw
        caches.append(fq.FlexKVCache(b, nh, d, max_seq, device=dev))
    torch.cuda.synchronize()

    # ---- prefill (also measured as a part)
    ws_pre = torch.zeros(fq.flex_workspace_bytes(layers[0], b, s), dtype=torch.uint8, device=dev)
    xa = synth.activations((b, s, h), seed, device=dev)
    xb = torch.empty_like(xa)

    def prefill_stack():
        src, dst = xa, xb
        for l in range(L):
            fq.flex_prefill_layer(layers[l], caches[l], src, dst, b, s, ws_pre)
            src, dst = dst, src

    prefill_stack()
    torch.cuda.synchronize()
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"prefill failed: {fq.flex_status_string(rc)}")

    # ---- decode: one graph per position, the 24-layer stack chained through 2 buffers
    ws_dec = torch.zeros(fq.flex_workspace_bytes(layers[0], b, 1), dtype=torch.uint8, device=dev)
    inputs = torch.stack([synth.decode_inputs(b, h, t, seed, device=dev) for t in range(nsteps)])
    buf = [torch.empty((b, h), dtype=torch.float16, device=dev) for _ in range(2)]
    y_out = torch.empty((b, h), dtype=torch.float16, device=dev)

    def decode_token(t):
        src = inputs[t]
        for l in range(L):
            dst = y_out if l == L - 1 else buf[l % 2]
            fq.flex_decode_layer(layers[l], caches[l], src, dst, b, s + t, ws_dec)
            src = dst

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        decode_token(0)                        # eager first call (kernel attributes, tensor maps)
    stream.synchronize()
    graphs = []
    for t in range(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            decode_token(t)
        graphs.append(g)
    torch.cuda.synchronize()

    def decode_phase():
        for g in graphs:
            g.replay()

    # LN1, QKV (+store_cache), attention, out, LN2, fc1, fc2, plus the attention combine
    # when a (sequence, head) key range is split across CTAs (the library splits when the
    # pairs alone fill fewer than 4 CTAs per SM; a split keeps at least 128 keys)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    pairs = b * nh
    splits = [max(1, min((4 * sms + pairs - 1) // pairs, (s + t + 127) // 128)) for t in range(nsteps)]
    launches_per_token = [L * (7 if ns == 1 else 8) for ns in splits]
    units_per_step = b * nsteps * L

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            decode_phase()
    torch.cuda.synchronize()
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"decode failed: {fq.flex_status_string(rc)}")

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_uuid)
    sampler.start()
    time.sleep(0.3)

    def timed(fn, K):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(K):
                fn()
            e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    t_start = time.time()
    torch.cuda.profiler.start()               # lets an ncu launch list capture exactly the timed steps
    ms = timed(decode_phase, args.steps)
    torch.cuda.profiler.stop()
    t_end = time.time()
    value = whole_job_value(world, units_per_step, args.steps, ms)

    # ---- end to end: per step H2D of the step's inputs from pinned memory, graphs,
    #      D2H of the step's result
    host_in = inputs.cpu().pin_memory()
    host_out = torch.empty((nsteps, b, h), dtype=torch.float16).pin_memory()

    def e2e_phase():
        for t, g in enumerate(graphs):
            inputs[t].copy_(host_in[t], non_blocking=True)
            g.replay()
            host_out[t].copy_(y_out, non_blocking=True)

    for _ in range(2):
        with torch.cuda.stream(stream):
            e2e_phase()
    torch.cuda.synchronize()
    e2e_steps = max(3, args.steps // 2)
    ms_e2e = timed(e2e_phase, e2e_steps)
    e2e_value = whole_job_value(world, units_per_step, e2e_steps, ms_e2e)
    sampler.stop()
    clocks = sampler.summary(t_start, t_end)
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"timed region failed: {fq.flex_status_string(rc)}")
    assert bool(torch.isfinite(y_out).all())

    parts, roofline = {}, None
    if rank == 0 and not args.no_parts:
        parts, roofline = measure_parts(fq, torch, synth, cfg, layers, caches, ws_dec, stream, peaks, dev,
                                        prefill_stack, ws_pre)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cfg)
    if world > 1:
        dist.barrier()

    hbm_bound_ms = sum(decode_bytes_per_layer_step(cfg, s + t) for t in range(nsteps)) * L / (peaks["hbm_gbs"] * 1e6)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 x int4 (fp32 accumulate)", "data": "synthetic",
        "config": bench_config(args, cfg, world),
        "hbm_roofline_frac_of_step": hbm_bound_ms / (ms / args.steps),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(host_in.numel() * 2),
                "d2h_bytes_per_step": int(host_out.numel() * 2)},
        "gpu_launches": sum(launches_per_token) * args.steps,
        "clocks": clocks,
        "peaks": peaks,
        "parts": parts,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
    if world > 1:
        dist.destroy_process_group()


def _kernel_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "group_wise_int4_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel_key, sha):
    """Per-launch DRAM bytes of `kernel_key` from the committed ncu summary, or None when
    the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_sha") != sha:
        return None
    return e.get("dram_bytes_per_launch")


def measure_codec(fq, torch, synth, dev, hbm):
    """flexq_compress / flexq_decompress on 1 GiB of fp16 [131072, 4096], 4-bit group 64,
    grouped along the contiguous and the strided dimension: GB/s of algorithmic bytes
    (fp16 in or out, codes, metadata) over 10 back-to-back calls (the tensor is 8x L2)."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    codec = {}
    for gd in (1, 0):
        shape = (131072, 4096)
        xt = synth.codec_tensor(shape, gd, 64, 9, device=dev)
        cfgq = fq.config(4, 64, gd)
        codes, meta = fq.flexq_compress(xt, cfgq)
        yt = fq.flexq_decompress(codes, meta, shape, cfgq)
        n = xt.numel()
        nbytes = n * 2 + n // 2 + n // 64 * 4
        for opname, fn in (("compress", lambda: fq.flexq_compress(xt, cfgq, codes, meta)),
                           ("decompress", lambda: fq.flexq_decompress(codes, meta, shape, cfgq, yt))):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(10):
                fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / 10
            key = f"{opname}_{'contiguous' if gd == 1 else 'strided'}"
            codec[key] = {"gbs": nbytes / (ms * 1e6), "frac_hbm": nbytes / (ms * 1e6) / hbm, "ms": ms,
                          "bytes": nbytes}
        del xt, codes, meta, yt
        torch.cuda.empty_cache()
    return codec


def measure_parts(fq, torch, synth, cfg, layers, caches, ws_dec, stream, peaks, dev, prefill_stack, ws_pre):
    """Each kernel of the decode step on its own (same launch configuration, cycling
    over the stack so nothing stays in L2), the prefill, and the codec."""
    L, b, s, h, nh, d, ffn = cfg["layers"], cfg["batch"], cfg["prompt"], cfg["h"], cfg["n_heads"], cfg["head_dim"], cfg["ffn"]
    pos = s + cfg["decode_steps"] // 2
    hbm = peaks["hbm_gbs"]
    reps = 20

    def time_cycle(fn, reps=reps):
        """ms per call of fn, from a CUDA graph that calls fn once per layer (so the
        operands rotate through the whole stack and do not stay in L2), replayed
        `reps` times between two events on the launching stream."""
        with torch.cuda.stream(stream):
            for l in range(L):
                fn(l)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for l in range(L):
                fn(l)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / (reps * L)      # ms per launch(-group)

    x = synth.activations((b, 3 * h), 5, device=dev)
    xf = synth.activations((b, ffn), 6, device=dev)
    o = torch.empty((b, h), dtype=torch.float16, device=dev)
    yq = torch.empty((b, 3 * h), dtype=torch.float16, device=dev)
    yf = torch.empty((b, ffn), dtype=torch.float16, device=dev)
    gws = torch.zeros(max(16, max(fq.flex_gemm_ws_bytes(b, n, k) for n, k in
                                  ((3 * h, h), (h, h), (ffn, h), (h, ffn)))), dtype=torch.uint8, device=dev)
    aws = torch.zeros(fq.flex_decode_attention_ws_bytes(caches[0], b, pos), dtype=torch.uint8, device=dev)
    per = 0.5625
    kern = {}
    kern["decode_attention"] = dict(
        ms=time_cycle(lambda l: fq.flex_decode_attention(caches[l], x[:, :h], x[:, h:], x[:, 2 * h:], 3 * h, o, b,
                                                         pos, aws, stream=stream)),
        bytes=2 * b * pos * h * per + 3 * b * h * 2 + b * h * 2, launches_per_layer_step=2,
        source=["attention.cu"])
    for name, (n, k, xin, yout, epi) in {"gemm_qkv": (3 * h, h, x[:, :h], yq, 0), "gemm_out": (h, h, x[:, :h], o, 0),
                                          "gemm_fc1": (ffn, h, x[:, :h], yf, 1),
                                          "gemm_fc2": (h, ffn, xf, o, 0)}.items():
        wkey = {"gemm_qkv": "w_qkv", "gemm_out": "w_o", "gemm_fc1": "w_fc1", "gemm_fc2": "w_fc2"}[name]
        kern[name] = dict(
            # the layer hands every GEMM its activations in the interleaved 8-block order
            ms=time_cycle(lambda l, n=n, xin=xin, yout=yout, epi=epi, wkey=wkey:
                          fq.flex_dequant_gemm(xin, layers[l].w[wkey], None, None, yout, b,
                                               epi | fq.FLEX_GEMM_X_INTERLEAVED, gws, stream=stream)),
            bytes=n * k * per + b * k * 2 + b * n * 2, launches_per_layer_step=1, source=["gemm.cu", "tc.cuh"])
    kern["store_cache"] = dict(
        ms=time_cycle(lambda l: fq.flex_append_kv(caches[l], x[:, h:], x[:, 2 * h:], 3 * h, b, pos, stream=stream)),
        bytes=2 * b * h * 2 + 2 * b * h * per, launches_per_layer_step=0, source=["kv_ln.cu"],
        note="standalone store_cache entry; inside a layer it is fused into the QKV GEMM epilogue")
    kern["layernorm"] = dict(
        ms=time_cycle(lambda l: fq.flex_layernorm(x[:, :h], layers[l].vec["ln1_g"], layers[l].vec["ln1_b"], o, b, h,
                                                  stream=stream)),
        bytes=2 * b * h * 2 + 2 * h * 2, launches_per_layer_step=2, source=["kv_ln.cu"])
    for k, v in kern.items():
        v["gbs"] = v["bytes"] / (v["ms"] * 1e6)
        v["frac_hbm"] = v["gbs"] / hbm
        v["us"] = v["ms"] * 1e3
    # per kernel (the four GEMMs are launches of one kernel, gemm_tc_kernel): time per
    # layer step, and bytes and duration per launch averaged over its launches
    gemms = ["gemm_qkv", "gemm_out", "gemm_fc1", "gemm_fc2"]
    gemm_kernel = "gemv_kernel" if b <= 32 else "gemm_tc_kernel"   # the library's dispatch by batch
    per_kernel = {
        gemm_kernel: dict(launches=4, ms=sum(kern[g]["ms"] for g in gemms),
                               bytes=sum(kern[g]["bytes"] for g in gemms), source=["gemm.cu", "tc.cuh"]),
        "decode_attention": dict(launches=2, ms=kern["decode_attention"]["ms"],
                                 bytes=kern["decode_attention"]["bytes"], source=["attention.cu"]),
        "layernorm_kernel": dict(launches=2, ms=2 * kern["layernorm"]["ms"], bytes=2 * kern["layernorm"]["bytes"],
                                 source=["kv_ln.cu"]),
    }
    dom = max(per_kernel, key=lambda k: per_kernel[k]["ms"])
    dk = per_kernel[dom]
    gbs = dk["bytes"] / (dk["ms"] * 1e6)
    sha = _kernel_sha(*dk["source"])
    roofline = {"kernel": dom, "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                "frac": gbs / hbm, "traffic": _traffic(dom, sha),
                "launches_per_layer_step": dk["launches"],
                "algorithmic_bytes_per_launch": dk["bytes"] / dk["launches"],
                "avg_launch_us": dk["ms"] * 1e3 / dk["launches"],
                "share_of_layer_step_parts": dk["ms"] / sum(v["ms"] for v in per_kernel.values()),
                "peak_source": f"{peaks['source']} hbm_gbs (copy)", "source_sha": sha}

    # prefill through the stack
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    prefill_stack()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(2):
        prefill_stack()
    e1.record()
    torch.cuda.synchronize()
    pms = e0.elapsed_time(e1) / (2 * L)
    T = b * s
    flops = 2 * T * (4 * h * h + 2 * h * ffn) + 2 * b * nh * s * s * d       # causal: half of 4*b*s^2*h
    prefill = {"tokens_per_s_per_layer": T / (pms / 1e3), "ms_per_layer": pms,
               "tflops": flops / (pms * 1e9), "frac_tensor_peak": flops / (pms * 1e9) / peaks["bf16_tflops"],
               "peak_note": "fp16 tensor peak = measured bf16 cuBLAS peak (same rate)"}

    codec = measure_codec(fq, torch, synth, dev, hbm)
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"parts failed: {fq.flex_status_string(rc)}")
    return {"kernels": kern, "prefill": prefill, "codec_1gib_4bit_g64": codec}, roofline


# ---------------------------------------------------------------------------------
def _oracle_sample(cfg, nseq, nsteps_cpu, budget_s=20.0):
    """Decode of `nseq` sequences through one oracle layer, one position after another,
    until about budget_s of work. Returns (layer-tokens, seconds, threads)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import synth
    from oracle import layer as ol
    h, nh, d, s = cfg["h"], cfg["n_heads"], cfg["head_dim"], cfg["prompt"]
    raw = {k: v.numpy() for k, v in synth.layer_params(h, cfg["ffn"], cfg["seed"] * 100).items()}
    PQ = ol.compress_weights(raw)
    W = ol.dequant_all(PQ)
    cache = ol.KVCache(nseq, nh, s + cfg["decode_steps"], d)
    kh, vh = synth.kv_history(nseq, nh, s, d, cfg["seed"])
    cache.store(kh.numpy(), vh.numpy(), 0)
    done, t0 = 0, time.perf_counter()
    for t in range(nsteps_cpu):
        x = synth.decode_inputs(nseq, h, t, cfg["seed"]).numpy()
        ol.decode_layer(x, PQ, cache, s + t, nh, W=W)
        done += nseq
        if time.perf_counter() - t0 > budget_s:
            break
    secs = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return done, secs, threads


def cpu_baseline(cfg):
    nseq = min(8, cfg["batch"])
    done, secs, threads = _oracle_sample(cfg, nseq, cfg["decode_steps"], budget_s=15.0)
    return {"value": done / secs, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} layer-tokens: {nseq} sequences of the {cfg['h']}-wide layer decoded at positions "
                      f"{cfg['prompt']}.. through one oracle layer (numpy fp64, BLAS threads {threads})"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = workload_cfg(args.workload, args.layers)
    nseq = 4
    # warm-up and timed steps: each step = one decode position for `nseq` sequences
    from oracle import layer as ol  # noqa: F401  (the oracle is the reference arm)
    done, secs, threads = _oracle_sample(cfg, nseq, args.warmup + args.steps, budget_s=1e9)
    per_step = secs / (args.warmup + args.steps)
    value = nseq / per_step
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "config": bench_config(args, cfg, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"each step: {nseq} sequences of the {cfg['h']}-wide layer decoded one "
                                       f"position through one oracle layer (numpy fp64); "
                                       f"{args.warmup + args.steps} steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_codec_only():
    import torch
    import group_wise_int4_b200 as fq
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fq.lib()
    hbm = measured_peaks()["hbm_gbs"]
    codec = measure_codec(fq, torch, synth, dev, hbm)
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"codec failed: {fq.flex_status_string(rc)}")
    print(json.dumps({"mode": "codec", "unit": "GB/s", "peak_hbm_gbs": hbm, "codec_1gib_4bit_g64": codec}), flush=True)


def main():
    args = parse_args()
    if args.codec_only:
        run_codec_only()
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_flexq(args)


if __name__ == "__main__":
    main()
