#!/usr/bin/env python
"""Benchmark of the flexq hot path on B200.

Metric: decode tokens/s per OPT layer-step (and int4 compress/decompress GB/s), as a
fraction of the roofline.

Default workload (``opt-175b``): OPT-175B-shaped decoder layers (h 12288, 96 heads x
128, FFN 49152), 4 distinct layers with their own int4 weights and int4 KV caches
(about 2 GB per layer, so nothing stays in the 126 MB L2), batch 144, prompt 512 then
32 decode steps; weights int4 group 64, KV int4 group 64, seeded synthetic data. The
prompt is prefilled once (setup); one benchmark *step* is the whole decode phase - 32
new tokens for the 144 sequences through the 4 layers (positions 512..543), i.e.
18,432 layer-tokens, replayed from CUDA graphs.

``--workload opt-30b`` runs the 3 x 48 schedule of that shape (three gpu-batches of 48
sequences, each with its own caches, one layer call per gpu-batch), ``opt-1.3b`` a
24-layer stack at batch 32, ``opt-125m`` one layer at batch 4.

Also measured in the same run (``parts``): every kernel of the decode step timed on its
own in the launch configuration the step uses (this gives the roofline object), the
prefill of the prompt, the opt-30b 3 x 48 schedule (default run only) and the codec at
1 GiB. ``--codec-only`` runs the whole compress/decompress sweep instead.

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
WORKLOADS = ["opt-125m", "opt-1.3b", "opt-30b", "opt-175b"]
KERNELS = ["gemm_qkv", "gemm_out", "gemm_fc1", "gemm_fc2", "decode_attention", "layernorm", "decode_layer",
           "prefill_layer", "compress", "decompress"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="flexq", choices=["flexq", "reference"])
    ap.add_argument("--workload", default="opt-175b", choices=WORKLOADS)
    ap.add_argument("--layers", type=int, default=None, help="stack depth (default: per workload)")
    ap.add_argument("--no-parts", action="store_true", help="skip the per-part measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--codec-only", action="store_true",
                    help="measure only flexq_compress / flexq_decompress over the sweep (one JSON line)")
    ap.add_argument("--kernel", default=None, choices=KERNELS,
                    help="run only this step, 3 times, at the workload's decode shape on one layer "
                         "(a small case for ncu captures); prints one JSON line")
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


def workload_cfg(name, layers=None):
    import synth
    cfg = dict(synth.WORKLOADS[name])
    if layers is not None:
        cfg["layers"] = layers
    cfg["name"] = name
    cfg["call_batch"] = cfg.get("gpu_batch", cfg["batch"])       # sequences per layer call
    cfg["calls"] = cfg["batch"] // cfg["call_batch"]              # layer calls per layer-step
    return cfg


def bench_config(cfg, world):
    L, b, s, nsteps = cfg["layers"], cfg["batch"], cfg["prompt"], cfg["decode_steps"]
    sched = (f"{cfg['calls']} gpu-batches of {cfg['call_batch']}, each with its own caches, sharing one pass over "
             f"each layer's weights (flex_decode_layer_batches)" if cfg["calls"] > 1
             else f"batch {b} in one layer call")
    return {"workload": f"{cfg['name']} decode: {L} distinct layers (own int4 weights and KV caches), {sched}, "
                        f"prompt {s}, {nsteps} decode steps (positions {s}..{s + nsteps - 1}), int4 g64 weights "
                        f"and KV",
            "h": cfg["h"], "heads": cfg["n_heads"], "head_dim": cfg["head_dim"], "ffn": cfg["ffn"],
            "batch": b, "call_batch": cfg["call_batch"], "prompt": s, "decode_steps": nsteps, "layers": L,
            "units_per_step": b * nsteps * L,
            "l2": "not flushed: each token step streams ~%.2f GB (> 126 MB L2)" %
                  (step_cost(cfg, s, 1.0, 1.0)["bytes"] * L / 1e9),
            "parallelism": f"replicas x{world}"}


def step_cost(cfg, pos, hbm_gbs, tflops, bits=4):
    """Algorithmic cost of one decode layer-step at position pos (int4 g64) for all the
    step's sequences (with several gpu-batches the weights are streamed once for all of
    them): bytes (weights 12h^2*0.5625, KV read 2*b*pos*h*0.5625, KV write 2*b*h*0.5625,
    q/k/v in and o out 8*b*h, activations of the GEMMs and LayerNorms, biases and
    LayerNorm ~(9h + ffn)*2), flops (weight GEMMs 2*b*(4h^2 + 2h*ffn), attention
    4*b*(pos+1)*h), and two bounds: pure HBM (bytes / bandwidth) and attainable (per
    kernel the larger of bytes / bandwidth and flops / tensor peak, summed)."""
    h, ffn, b = cfg["h"], cfg["ffn"], cfg["batch"]
    per = 0.5 + 4 / 64 if bits == 4 else 1 + 4 / 64
    bw, pk = hbm_gbs * 1e9, tflops * 1e12
    tot_bytes = tot_flops = attain = 0.0
    for n, k in ((3 * h, h), (h, h), (ffn, h), (h, ffn)):
        by = n * k * per + b * k * 2 + b * n * 2
        fl = 2.0 * b * n * k
        tot_bytes += by
        tot_flops += fl
        attain += max(by / bw, fl / pk)
    kv = 2 * b * pos * h * per + 2 * b * h * per + 4 * b * h * 2      # + q, k, v in, o out
    small = (9 * h + ffn) * 2 + 2 * (2 * b * h * 2)                 # params, two LayerNorms
    tot_bytes += kv + small
    tot_flops += 4.0 * b * (pos + 1) * h
    attain += (kv + small) / bw
    return {"bytes": tot_bytes, "flops": tot_flops, "hbm_s": tot_bytes / bw, "attainable_s": attain}


# ---------------------------------------------------------------------------------
def graph_kernel_counts(g):
    """{kernel name: launches} of a captured CUDA graph (its kernel nodes), read back
    through the CUDA driver API; None if the graph cannot be inspected. A node whose
    name cannot be read is counted under "?"."""
    try:
        from cuda.bindings import driver as cd
        ok = cd.CUresult.CUDA_SUCCESS
        graph = cd.CUgraph(init_value=int(g.raw_cuda_graph()))
        err, _, n = cd.cuGraphGetNodes(graph, 0)
        if err != ok:
            return None
        err, nodes, n = cd.cuGraphGetNodes(graph, n)
        if err != ok:
            return None
        counts = {}
        for node in nodes[:n]:
            err, t = cd.cuGraphNodeGetType(node)
            if err != ok or t != cd.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
                continue
            name = "?"
            err, prm = cd.cuGraphKernelNodeGetParams(node)
            if err == ok:
                for getter, handle in ((getattr(cd, "cuFuncGetName", None), getattr(prm, "func", None)),
                                       (getattr(cd, "cuKernelGetName", None), getattr(prm, "kern", None))):
                    if getter is None or handle is None or int(handle) == 0:
                        continue
                    e2, nm = getter(handle)
                    if e2 == ok and nm:
                        name = nm.decode() if isinstance(nm, bytes) else str(nm)
                        break
            counts[name] = counts.get(name, 0) + 1
        return counts
    except Exception:
        return None


def short_kernel_name(name):
    """Kernel name without namespace, template arguments or parameters, from a plain
    ('void flexq::(anonymous namespace)::gemm_tc_kernel<4, true>(...)') or a mangled
    ('_ZN5flexq..14gemm_tc_kernelILi4ELb1EEEv...') name."""
    import re
    if name.startswith("_Z"):                 # mangled: length-prefixed identifiers
        i, found = 0, None
        while i < len(name):
            m = re.match(r"\d+", name[i:])
            if m:
                n = int(m.group(0))
                ident = name[i + len(m.group(0)):i + len(m.group(0)) + n]
                if ident.endswith("_kernel"):
                    found = ident
                i += len(m.group(0)) + (n if len(ident) == n else 0)
            else:
                i += 1
        if found:
            return found
    m = re.search(r"([A-Za-z0-9_]*_kernel)\b", name)
    return m.group(1) if m else name.split("(")[0].split("<")[0].split("::")[-1].strip()


class Stack:
    """L distinct layers of one workload on the device, each with its own compressed
    weights and, per gpu-batch, its own int4 KV cache; prefilled with the prompt."""

    def __init__(self, fq, torch, synth, cfg, dev):
        L, b, s, h = cfg["layers"], cfg["call_batch"], cfg["prompt"], cfg["h"]
        nh, d = cfg["n_heads"], cfg["head_dim"]
        self.fq, self.torch, self.cfg, self.dev = fq, torch, cfg, dev
        self.max_seq = s + cfg["decode_steps"]
        self.layers, self.caches = [], []
        for l in range(L):
            raw = synth.layer_params(h, cfg["ffn"], cfg["seed"] * 100 + l, device=dev)
            self.layers.append(fq.FlexLayer(raw, nh, device=dev))
            del raw
            self.caches.append([fq.FlexKVCache(b, nh, d, self.max_seq, device=dev) for _ in range(cfg["calls"])])
        torch.cuda.synchronize()
        nc = cfg["calls"]
        self.ws_pre = torch.zeros(fq.flex_workspace_bytes(self.layers[0], nc * b, s), dtype=torch.uint8, device=dev)
        self.x_pre = synth.activations((nc, b, s, h), cfg["seed"] * 10, device=dev)
        self.y_pre = torch.empty_like(self.x_pre)
        self.ws_dec = torch.zeros(fq.flex_workspace_bytes(self.layers[0], nc * b, 1), dtype=torch.uint8, device=dev)

    def prefill(self, stream=None, events=None):
        """Prompt of every gpu-batch through the stack (writes cache slots [0, prompt));
        several gpu-batches share one pass over each layer's weights. With `events`
        (a list), a pair of CUDA events on `stream` brackets each layer call."""
        fq, cfg, torch = self.fq, self.cfg, self.torch
        src, dst = self.x_pre, self.y_pre
        for l in range(cfg["layers"]):
            if events is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            if cfg["calls"] == 1:
                fq.flex_prefill_layer(self.layers[l], self.caches[l][0], src, dst, cfg["call_batch"], cfg["prompt"],
                                      self.ws_pre, stream=stream)
            else:
                fq.flex_prefill_layer_batches(self.layers[l], self.caches[l], src, dst, cfg["call_batch"],
                                              cfg["prompt"], self.ws_pre, stream=stream)
            if events is not None:
                e1.record(stream)
                events.append((e0, e1))
            src, dst = dst, src
        # the last layer's output is not kept: a synthetic stack has no LM head

    def free_prefill(self):
        del self.ws_pre, self.x_pre, self.y_pre
        self.torch.cuda.empty_cache()


def build_decode_graphs(fq, torch, stack, stream, inputs, y_outs, positions):
    """One CUDA graph per position: all sequences through every layer, chained through
    two activation buffers. With several gpu-batches (the pages' gpu_batch_size x
    num_gpu_batches block) each layer is one flex_decode_layer_batches call, so its
    weights are streamed once for all gpu-batches. inputs [T][batch][h]; the graph of
    position t writes its output to y_outs[t % len(y_outs)] ([batch][h] each), so that a
    copy of one token's output can run while the next token computes."""
    cfg = stack.cfg
    L, b, calls = cfg["layers"], cfg["call_batch"], cfg["calls"]
    bufs = [torch.empty((calls * b, cfg["h"]), dtype=torch.float16, device=stack.dev) for _ in range(2)]

    def token(t, pos):
        src = inputs[t]
        for l in range(L):
            dst = y_outs[t % len(y_outs)] if l == L - 1 else bufs[l % 2]
            if calls == 1:
                fq.flex_decode_layer(stack.layers[l], stack.caches[l][0], src, dst, b, pos, stack.ws_dec)
            else:
                fq.flex_decode_layer_batches(stack.layers[l], stack.caches[l], src, dst, b, pos, stack.ws_dec)
            src = dst

    with torch.cuda.stream(stream):
        token(0, positions[0])                     # eager first call (kernel attributes, tensor maps)
    stream.synchronize()
    graphs = []
    for t, pos in enumerate(positions):
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=stream):
            token(t, pos)
        g.instantiate()
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs, bufs


def run_flexq(args):
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
    L, b, s, h = cfg["layers"], cfg["batch"], cfg["prompt"], cfg["h"]
    nsteps = cfg["decode_steps"]

    stack = Stack(fq, torch, synth, cfg, dev)
    stack.prefill()
    torch.cuda.synchronize()
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"prefill failed: {fq.flex_status_string(rc)}")

    stream = torch.cuda.Stream(device=dev)
    inputs = torch.stack([synth.decode_inputs(b, h, t, cfg["seed"], device=dev) for t in range(nsteps)])
    y_outs = [torch.empty((b, h), dtype=torch.float16, device=dev) for _ in range(2)]
    positions = [s + t for t in range(nsteps)]
    graphs, _bufs = build_decode_graphs(fq, torch, stack, stream, inputs, y_outs, positions)

    # kernels per decode phase, read back from the captured graphs
    launch_counts = {}
    for g in graphs:
        c = graph_kernel_counts(g)
        if c is None:
            launch_counts = None
            break
        for k, v in c.items():
            launch_counts[k] = launch_counts.get(k, 0) + v

    def decode_phase():
        for g in graphs:
            g.replay()

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

    # ---- end to end: every token's inputs copied from pinned host memory and its output
    #      copied back, inside the timed region. The copies run on their own stream:
    #      token t + 1's inputs while token t computes, token t's output while token t + 1
    #      computes (outputs alternate between two buffers). Each graph waits for its
    #      inputs, and a graph reuses an output buffer only once its earlier copy is done.
    host_in = inputs.cpu().pin_memory()
    host_out = torch.empty((nsteps, b, h), dtype=torch.float16).pin_memory()
    copy_stream = torch.cuda.Stream(device=dev)
    T = len(graphs)

    def e2e_phase():
        ev_in = [torch.cuda.Event() for _ in range(T)]
        ev_out = [torch.cuda.Event() for _ in range(T)]
        start = torch.cuda.Event()
        start.record(stream)                       # every earlier graph has finished here
        copy_stream.wait_event(start)
        with torch.cuda.stream(copy_stream):
            inputs[0].copy_(host_in[0], non_blocking=True)
            ev_in[0].record(copy_stream)
        for t, g in enumerate(graphs):
            stream.wait_event(ev_in[t])
            if t >= 2:
                stream.wait_event(ev_out[t - 2])   # y_outs[t % 2] has been copied out
            ev_run = torch.cuda.Event()
            ev_run.record(stream)                  # graph t - 1, the last reader of inputs[t + 1] before, is done
            g.replay()
            ev_done = torch.cuda.Event()
            ev_done.record(stream)
            with torch.cuda.stream(copy_stream):
                if t + 1 < T:
                    copy_stream.wait_event(ev_run)
                    inputs[t + 1].copy_(host_in[t + 1], non_blocking=True)
                    ev_in[t + 1].record(copy_stream)
                copy_stream.wait_event(ev_done)
                host_out[t].copy_(y_outs[t % 2], non_blocking=True)
                ev_out[t].record(copy_stream)
        stream.wait_event(ev_out[T - 1])           # the timed region ends after the last copy

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
    assert all(bool(torch.isfinite(y).all()) for y in y_outs)
    del graphs

    # ---- bounds of the step (summed over its positions and layers)
    costs = [step_cost(cfg, p, peaks["hbm_gbs"], peaks["bf16_tflops"]) for p in positions]
    step_s = ms / args.steps / 1e3
    hbm_s = sum(c["hbm_s"] for c in costs) * L
    att_s = sum(c["attainable_s"] for c in costs) * L
    step_bounds = {"hbm_bound_ms": hbm_s * 1e3, "attainable_bound_ms": att_s * 1e3, "measured_ms": step_s * 1e3,
                   "frac_of_hbm_bound": hbm_s / step_s, "frac_of_attainable_bound": att_s / step_s,
                   "note": "hbm: algorithmic bytes / measured copy bandwidth; attainable: per kernel max(bytes / "
                           "bandwidth, flops / tensor peak), summed"}

    parts, roofline = {}, None
    if rank == 0 and not args.no_parts:
        parts, roofline = measure_parts(fq, torch, synth, cfg, stack, stream, peaks, dev)
        if args.workload == "opt-175b":
            del stack
            torch.cuda.empty_cache()
            parts["opt-30b_3x48"] = measure_secondary_decode(fq, torch, synth, "opt-30b", peaks, dev)
        codec = measure_codec(fq, torch, synth, dev, peaks["hbm_gbs"], points=CODEC_POINTS_DEFAULT)
        parts["codec"] = codec
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cfg)
        if "codec" in parts:
            parts["codec"]["cpu_baseline"] = codec_cpu_baseline()
    if world > 1:
        dist.barrier()

    ours = None
    if launch_counts is not None:
        # every kernel node of the decode graphs is one of the library's; names show which
        ours = {short_kernel_name(k) if k != "?" else "unnamed kernel node": v for k, v in launch_counts.items()}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 x int4 (fp32 accumulate)", "data": "synthetic",
        "config": bench_config(cfg, world),
        "roofline": roofline,
        "step_bounds": step_bounds,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(host_in.numel() * 2),
                "d2h_bytes_per_step": int(host_out.numel() * 2)},
        "gpu_launches": (sum(ours.values()) * args.steps) if ours else None,
        "gpu_launches_per_step_by_kernel": ours,
        "gpu_launches_source": "kernel nodes of the captured decode graphs replayed in the timed region",
        "clocks": clocks,
        "peaks": peaks,
        "parts": parts,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
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


# ---- codec ---------------------------------------------------------------------------
# (rows of [R, 4096] fp16 or a 3-D shape, group_dim, bits, group size)
CODEC_POINTS_DEFAULT = [((131072, 4096), 1, 4, 64), ((131072, 4096), 0, 4, 64), ((131072, 4096), 1, 8, 64),
                        ((131072, 4096), 1, 4, 32), ((131072, 4096), 1, 4, 128)]


def codec_sweep_points():
    pts = []
    for mb in (16, 256, 1024, 4096):
        rows = mb * (1 << 20) // (2 * 4096)
        for gd in (1, 0):
            for bits in (4, 8):
                for gs in (32, 64, 128):
                    pts.append(((rows, 4096), gd, bits, gs))
    pts.append(((544, 144 * 96, 128), 2, 4, 64))         # KV-shaped: [tokens][seq x heads][head_dim]
    # codec variants (the generic kernels), 1 GiB: 3-bit codes, the symmetric form, and a
    # group dimension that is not a multiple of the group size (last group padded)
    rows = 1024 * (1 << 20) // (2 * 4096)
    pts += [((rows, 4096), 1, 3, 64, 0), ((rows, 4096), 1, 4, 64, 1), ((rows, 4096), 1, 8, 64, 1),
            ((rows, 4000), 1, 4, 64, 0)]
    return pts


def measure_codec(fq, torch, synth, dev, hbm, points):
    """flexq_compress / flexq_decompress: GB/s of algorithmic bytes (fp16 in or out,
    codes, metadata) over 10 back-to-back calls per point (each input is at least 2x L2,
    except the 16 MB points, which are L2-resident and marked so)."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    out = {}
    for shape, gd, bits, gs, *rest in points:
        sym = rest[0] if rest else 0
        if shape[gd] % gs:                     # partial last group: a slice of a whole-group tensor
            full = list(shape)
            full[gd] = (shape[gd] + gs - 1) // gs * gs
            xt = synth.codec_tensor(tuple(full), gd, gs, 9, device=dev).narrow(gd, 0, shape[gd]).contiguous()
        else:
            xt = synth.codec_tensor(shape, gd, gs, 9, device=dev)
        cfgq = fq.config(bits, gs, gd, sym)
        codes, meta = fq.flexq_compress(xt, cfgq)
        yt = fq.flexq_decompress(codes, meta, shape, cfgq)
        n = xt.numel()
        nbytes = n * 2 + codes.numel() + meta.numel() * meta.element_size()
        layout = {1: "contiguous", 0: "strided"}.get(gd, f"dim{gd}") if len(shape) == 2 else f"kv-dim{gd}"
        key = f"{'x'.join(map(str, shape))}_{layout}_{bits}bit_g{gs}" + ("_symmetric" if sym else "")
        entry = {"mb": round(n * 2 / (1 << 20)), "bytes": nbytes}
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
            entry[opname] = {"gbs": nbytes / (ms * 1e6), "frac_hbm": nbytes / (ms * 1e6) / hbm, "us": ms * 1e3}
        if n * 2 < 2 * 126 * (1 << 20):
            entry["note"] = "L2-resident"
        out[key] = entry
        del xt, codes, meta, yt
        torch.cuda.empty_cache()
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"codec failed: {fq.flex_status_string(rc)}")
    return out


# ---- parts ---------------------------------------------------------------------------
def measure_parts(fq, torch, synth, cfg, stack, stream, peaks, dev):
    """Each kernel of the decode step on its own (same launch configuration, cycling
    over the stack so nothing stays in L2) and the prefill."""
    L, b, s, h, nh, d, ffn = (cfg["layers"], cfg["call_batch"], cfg["prompt"], cfg["h"], cfg["n_heads"],
                              cfg["head_dim"], cfg["ffn"])
    calls = cfg["calls"]
    pos = s + cfg["decode_steps"] // 2
    hbm, tpk = peaks["hbm_gbs"], peaks["bf16_tflops"]
    ridge = tpk * 1e12 / (hbm * 1e9)               # flop per byte where the two bounds meet
    reps = 20
    layers = stack.layers
    caches = [cs[0] for cs in stack.caches]

    def time_cycle(fn, reps=reps):
        """(ms per call of fn, {kernel: launches per call}), from a CUDA graph that calls
        fn once per layer (so the operands rotate through the whole stack and do not
        stay in L2), replayed `reps` times between two events on the launching stream;
        the kernel names are read from the captured graph (None if it cannot be read)."""
        with torch.cuda.stream(stream):
            for l in range(L):
                fn(l)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)        # the graph stays readable after capture
        with torch.cuda.graph(g, stream=stream):
            for l in range(L):
                fn(l)
        g.instantiate()
        counts = graph_kernel_counts(g)
        names = None if counts is None else {short_kernel_name(k): v / L for k, v in counts.items()}
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
        return e0.elapsed_time(e1) / (reps * L), names      # ms per launch(-group)

    def main_kernel(names, expected):
        """The part's working kernel: its most-launched kernel that is not a combine
        step (the expected name when the graph could not be read)."""
        if not names:
            return expected
        work = {k: v for k, v in names.items() if "combine" not in k} or names
        return max(sorted(work), key=lambda k: work[k])

    x = synth.activations((b, 3 * h), 5, device=dev)
    x[:, :h] *= d ** -0.5
    xf = synth.activations((b, ffn), 6, device=dev)
    o = torch.empty((b, h), dtype=torch.float16, device=dev)
    yq = torch.empty((b, 3 * h), dtype=torch.float16, device=dev)
    yf = torch.empty((b, ffn), dtype=torch.float16, device=dev)
    gws = torch.zeros(max(16, max(fq.flex_gemm_ws_bytes(b, n, k) for n, k in
                                  ((3 * h, h), (h, h), (ffn, h), (h, ffn)))), dtype=torch.uint8, device=dev)
    aws = torch.zeros(max(16, fq.flex_decode_attention_ws_bytes(caches[0], b, pos)), dtype=torch.uint8, device=dev)
    per = 0.5625
    # the library splits a (sequence, head) key range over CTAs only when the pairs alone
    # fill fewer than 4 CTAs per SM; then a combine kernel merges the splits
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kern = {}
    ms, names = time_cycle(lambda l: fq.flex_decode_attention(caches[l], x[:, :h], x[:, h:], x[:, 2 * h:], 3 * h, o,
                                                              b, pos, aws, stream=stream))
    kern["decode_attention"] = dict(
        ms=ms, bytes=2 * b * pos * h * per + 3 * b * h * 2 + b * h * 2, flops=4.0 * b * (pos + 1) * h,
        launches_per_call=int(round(sum(names.values()))) if names else (1 if b * nh >= 4 * sms else 2),
        kernel=main_kernel(names, "decode_attn_tc_kernel"), kernels=names, source=["attention.cu"])
    gemm_kernel = "gemv_kernel" if b <= 32 else "gemm_tc_kernel"   # only if the graph cannot be read
    for name, (n, k, xin, yout, epi) in {"gemm_qkv": (3 * h, h, x[:, :h], yq, 0), "gemm_out": (h, h, x[:, :h], o, 0),
                                          "gemm_fc1": (ffn, h, x[:, :h], yf, 1),
                                          "gemm_fc2": (h, ffn, xf, o, 0)}.items():
        wkey = {"gemm_qkv": "w_qkv", "gemm_out": "w_o", "gemm_fc1": "w_fc1", "gemm_fc2": "w_fc2"}[name]
        # the layer hands every GEMM its activations in the interleaved 8-block order
        ms, names = time_cycle(lambda l, xin=xin, yout=yout, epi=epi, wkey=wkey:
                               fq.flex_dequant_gemm(xin, layers[l].w[wkey], None, None, yout, b,
                                                    epi | fq.FLEX_GEMM_X_INTERLEAVED, gws, stream=stream))
        kern[name] = dict(ms=ms, bytes=n * k * per + b * k * 2 + b * n * 2, flops=2.0 * b * n * k, launches_per_call=1,
                          kernel=main_kernel(names, gemm_kernel), kernels=names, source=["gemm.cu", "tc.cuh"])
    ms, names = time_cycle(lambda l: fq.flex_append_kv(caches[l], x[:, h:], x[:, 2 * h:], 3 * h, b, pos,
                                                       stream=stream))
    kern["store_cache"] = dict(
        ms=ms, bytes=2 * b * h * 2 + 2 * b * h * per, flops=0.0, launches_per_call=0, kernels=names,
        source=["kv_ln.cu"], note="standalone store_cache entry; inside a layer it is fused into the QKV GEMM epilogue")
    ms, names = time_cycle(lambda l: fq.flex_layernorm(x[:, :h], layers[l].vec["ln1_g"], layers[l].vec["ln1_b"], o, b,
                                                       h, stream=stream))
    kern["layernorm"] = dict(ms=ms, bytes=2 * b * h * 2 + 2 * h * 2, flops=0.0, launches_per_call=2,
                             kernel=main_kernel(names, "layernorm_kernel"), kernels=names, source=["kv_ln.cu"])
    # left padding (valid_from): sequence i starts at key (i % 4) * 128, so its first keys
    # are neither read nor attended (the same kernel, fewer keys)
    vf = torch.clamp((torch.arange(b, device=dev, dtype=torch.int32) % 4) * 128, max=pos)
    for c in caches:
        c.valid_from = vf
    ms, names = time_cycle(lambda l: fq.flex_decode_attention(caches[l], x[:, :h], x[:, h:], x[:, 2 * h:], 3 * h, o,
                                                              b, pos, aws, stream=stream))
    for c in caches:
        c.valid_from = None
    kept = float(torch.clamp(pos - vf, min=0).sum().item())
    kern["decode_attention_padded"] = dict(
        ms=ms, bytes=2 * kept * h * per + 3 * b * h * 2 + b * h * 2, flops=4.0 * (kept + b) * h,
        launches_per_call=int(round(sum(names.values()))) if names else 1, kernels=names, source=["attention.cu"],
        note="left-padded batch: sequence i skips its first (i % 4) * 128 keys; bytes count the keys read")
    # the model around the layers: input embedding of the next tokens, then the output head
    # (final LayerNorm, logits over the 4-bit token table, greedy choice) - OPT vocabulary
    vocab = synth.OPT_VOCAB
    vpad = (vocab + 255) // 256 * 256
    mp = synth.model_params(vocab, h, 2048, cfg["seed"], vpad, device=dev)
    E = fq.CompressedWeight(mp.pop("E"))
    tok = synth.token_ids((b,), vocab, 7, device=dev)
    tpos = torch.full((b,), pos, dtype=torch.int32, device=dev)
    xe = torch.empty((b, h), dtype=torch.float16, device=dev)
    ids = torch.empty(b, dtype=torch.int32, device=dev)
    hws = torch.zeros(max(16, fq.flex_lm_head_ws_bytes(E, vocab, b)), dtype=torch.uint8, device=dev)

    def model_io(_l):
        fq.flex_embed(E, vocab, mp["P"], tok, tpos, xe, stream=stream)
        fq.flex_lm_head_argmax(E, vocab, mp["lnf_g"], mp["lnf_b"], xe, hws, ids, stream=stream)
    ms, names = time_cycle(model_io)
    kern["embed_and_head"] = dict(
        ms=ms, bytes=vpad * h * per + b * h * (per + 2 + 2) + 3 * b * h * 2 + b * vpad * 2 * 2,
        flops=2.0 * b * vpad * h, launches_per_call=int(round(sum(names.values()))) if names else 4, kernels=names,
        source=["model.cu", "gemm.cu"],
        note="flex_embed of the next tokens + flex_lm_head_argmax (final LayerNorm, logits over the 4-bit token "
             "table, greedy id) for the whole batch; not part of the layer step")
    del E, mp, hws
    # the whole layer call in the same regime (a graph of one call per layer, replayed):
    # against the sum of its kernels' parts it shows what the kernel boundaries cost
    xl = synth.decode_inputs(b * calls, h, 0, cfg["seed"], device=dev)
    yl = torch.empty((b * calls, h), dtype=torch.float16, device=dev)
    ms_layer, names = time_cycle(lambda l: (fq.flex_decode_layer(layers[l], caches[l], xl, yl, b, pos, stack.ws_dec,
                                                                  stream=stream) if calls == 1 else
                                            fq.flex_decode_layer_batches(layers[l], stack.caches[l], xl, yl, b, pos,
                                                                         stack.ws_dec, stream=stream)))
    layer_call = {"us": ms_layer * 1e3, "kernels": names,
                  "note": "one decode layer call (all its kernels, programmatic-launch chained), graph-timed "
                          "like the parts"}
    for k, v in kern.items():
        v["us"] = v["ms"] * 1e3
        v["gbs"] = v["bytes"] / (v["ms"] * 1e6)
        v["frac_hbm"] = v["gbs"] / hbm
        if v["flops"]:
            v["tflops"] = v["flops"] / (v["ms"] * 1e9)
            v["frac_tensor"] = v["tflops"] / tpk
    # per kernel (the four GEMMs are launches of one kernel): time per layer call, and
    # bytes / flops / duration per launch averaged over its launches
    # each part's time goes to its working kernel (the attention's combine step, when the
    # key range is split, is timed with it); one layer call runs 4 GEMMs, 1 attention, 2 LNs
    per_kernel = {}
    for part, per_call in (("gemm_qkv", 1), ("gemm_out", 1), ("gemm_fc1", 1), ("gemm_fc2", 1),
                           ("decode_attention", 1), ("layernorm", 2)):
        v = kern[part]
        e = per_kernel.setdefault(v["kernel"], dict(launches=0, ms=0.0, bytes=0.0, flops=0.0, parts=[],
                                                    source=v["source"]))
        e["launches"] += per_call
        e["ms"] += per_call * v["ms"]
        e["bytes"] += per_call * v["bytes"]
        e["flops"] += per_call * v["flops"]
        e["parts"].append(part)
    dom = max(per_kernel, key=lambda k: per_kernel[k]["ms"])
    dk = per_kernel[dom]
    sha = _kernel_sha(*dk["source"])
    intensity = dk["flops"] / dk["bytes"]
    tensor_bound = intensity > ridge
    achieved = dk["flops"] / (dk["ms"] * 1e9) if tensor_bound else dk["bytes"] / (dk["ms"] * 1e6)
    peak = tpk if tensor_bound else hbm
    roofline = {"kernel": dom, "bound": "tensor" if tensor_bound else "hbm", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s" if tensor_bound else "GB/s", "frac": achieved / peak,
                "traffic": _traffic(f"{dom}@{cfg['name']}", sha),
                "launches_per_layer_call": dk["launches"],
                "algorithmic_bytes_per_launch": dk["bytes"] / dk["launches"],
                "algorithmic_flops_per_launch": dk["flops"] / dk["launches"],
                "intensity_flop_per_byte": intensity, "ridge_flop_per_byte": ridge,
                "avg_launch_us": dk["ms"] * 1e3 / dk["launches"],
                "frac_hbm": dk["bytes"] / (dk["ms"] * 1e6) / hbm,
                "frac_tensor": dk["flops"] / (dk["ms"] * 1e9) / tpk,
                "share_of_layer_step_parts": dk["ms"] / sum(v["ms"] for v in per_kernel.values()),
                "peak_source": f"{peaks['source']} " + ("bf16_tflops (cuBLAS burst; fp16 dense has the same rate)"
                                                        if tensor_bound else "hbm_gbs (copy)"),
                "timing": "CUDA events around a graph of one launch per layer of the stack, replayed 20 times",
                "source_sha": sha}

    # prefill through the stack
    torch.cuda.synchronize()
    stack_ok = hasattr(stack, "ws_pre")
    prefill = None
    if stack_ok:
        stack.prefill(stream)
        torch.cuda.synchronize()
        evs = []
        with torch.cuda.stream(stream):
            stack.prefill(stream, evs)
        torch.cuda.synchronize()
        each = [e_a.elapsed_time(e_b) for e_a, e_b in evs]             # ms per layer call
        pms = sum(each) / (L * calls)
        T = b * s
        flops = 2 * T * (4 * h * h + 2 * h * ffn) + 2 * b * nh * s * s * d       # causal: half of 4*b*s^2*h
        prefill = {"tokens_per_s_per_layer": T / (pms / 1e3), "ms_per_layer_call": pms,
                   "ms_each_layer_call": each,
                   "tflops": flops / (pms * 1e9), "frac_tensor_peak": flops / (pms * 1e9) / tpk,
                   "peak_note": "fp16 tensor peak = measured bf16 cuBLAS peak (same rate)"}
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"parts failed: {fq.flex_status_string(rc)}")
    return {"kernels": kern, "per_kernel_per_layer_call": per_kernel, "layer_call": layer_call,
            "prefill": prefill}, roofline


def measure_secondary_decode(fq, torch, synth, name, peaks, dev, ntok=8, reps=5):
    """Decode of another workload's schedule (e.g. opt-30b as 3 gpu-batches of 48): a
    1-layer stack prefilled with the prompt, then graphs of `ntok` positions replayed
    `reps` times. layer-tokens/s and the step bounds."""
    cfg = workload_cfg(name)
    stack = Stack(fq, torch, synth, cfg, dev)
    stack.prefill()
    stack.free_prefill()
    stream = torch.cuda.Stream(device=dev)
    b, h, s = cfg["batch"], cfg["h"], cfg["prompt"]
    inputs = torch.stack([synth.decode_inputs(b, h, t, cfg["seed"], device=dev) for t in range(ntok)])
    y_out = torch.empty((b, h), dtype=torch.float16, device=dev)
    positions = [s + t for t in range(ntok)]
    graphs, _ = build_decode_graphs(fq, torch, stack, stream, inputs, [y_out], positions)
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            for g in graphs:
                g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"{name} decode failed: {fq.flex_status_string(rc)}")
    ms = e0.elapsed_time(e1) / (reps * ntok * cfg["layers"])          # per layer-step
    costs = [step_cost(cfg, p, peaks["hbm_gbs"], peaks["bf16_tflops"]) for p in positions]
    hbm_s = sum(c["hbm_s"] for c in costs) / ntok
    att_s = sum(c["attainable_s"] for c in costs) / ntok
    out = {"workload": bench_config(cfg, 1)["workload"], "layer_tokens_per_s": b / (ms / 1e3),
           "ms_per_layer_step": ms, "frac_of_hbm_bound": hbm_s / (ms / 1e3),
           "frac_of_attainable_bound": att_s / (ms / 1e3), "positions": f"{s}..{s + ntok - 1}"}
    del graphs, stack
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------------
def _oracle_sample(cfg, nseq, nsteps_cpu, budget_s=15.0, nthreads=None):
    """Decode of `nseq` sequences through one layer of the C++ fp32 oracle, one position
    after another from `prompt` on, until about budget_s of work (at least one step).
    Returns (layer-tokens, seconds, threads, steps)."""
    import synth
    from oracle import cpp
    h, nh, d, s = cfg["h"], cfg["n_heads"], cfg["head_dim"], cfg["prompt"]
    nthreads = nthreads or cpp.threads()
    raw = {k: v.numpy() for k, v in synth.layer_params(h, cfg["ffn"], cfg["seed"] * 100).items()}
    layer = cpp.Layer(raw, nh, nthreads=nthreads)
    del raw
    cache = cpp.KVCache(nseq, nh, s + cfg["decode_steps"], d)
    kh, vh = synth.kv_history(nseq, nh, s, d, cfg["seed"])
    for name, t in (("k", kh), ("v", vh)):
        c, m = cpp.compress(t.numpy(), 4, 64, 3, nthreads)
        getattr(cache, f"{name}_codes")[:, :, :s] = c
        getattr(cache, f"{name}_meta")[:, :, :s] = m
    done, steps, t0 = 0, 0, time.perf_counter()
    for t in range(nsteps_cpu):
        x = synth.decode_inputs(nseq, h, t, cfg["seed"]).numpy()
        cpp.decode_layer(x, layer, cache, s + t % cfg["decode_steps"], nthreads)
        done += nseq
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return done, time.perf_counter() - t0, nthreads, steps


def cpu_baseline(cfg):
    nseq = min(16, cfg["call_batch"])
    done, secs, threads, _ = _oracle_sample(cfg, nseq, cfg["decode_steps"], budget_s=12.0)
    return {"value": done / secs, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} layer-tokens: {nseq} sequences of the {cfg['h']}-wide layer decoded at positions "
                      f"{cfg['prompt']}.. through one layer of the C++ fp32 oracle ({threads} threads)"}


def codec_cpu_baseline():
    """The C++ oracle's compress / decompress of a 256 MiB fp16 [32768, 4096] tensor (4-bit
    g64, contiguous groups), on one thread and on every host core: GB/s with the GPU's
    byte accounting."""
    import synth
    from oracle import cpp
    x = synth.codec_tensor((32768, 4096), 1, 64, 9).numpy()
    n = x.size
    nbytes = n * 2 + n // 2 + n // 64 * 4
    out = {}
    for th in (1, cpp.threads()):
        t0 = time.perf_counter()
        c, m = cpp.compress(x, 4, 64, 1, nthreads=th)
        t1 = time.perf_counter()
        cpp.decompress(c, m, x.shape, 4, 64, 1, nthreads=th)
        t2 = time.perf_counter()
        out[f"threads_{th}"] = {"compress_gbs": nbytes / (t1 - t0) / 1e9, "decompress_gbs": nbytes / (t2 - t1) / 1e9}
    out["kind"] = "oracle"
    out["sample"] = "256 MiB fp16 [32768, 4096], 4-bit g64 along the contiguous dim, C++ fp32 oracle"
    out["cores"] = cpp.threads()
    return out


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = workload_cfg(args.workload, args.layers)
    nseq = min(16, cfg["call_batch"])
    # warm-up and timed steps: each step = one decode position for `nseq` sequences
    n_all = args.warmup + args.steps
    done, secs, threads, steps = _oracle_sample(cfg, nseq, n_all, budget_s=1e9)
    per_step = secs / steps
    value = nseq / per_step
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 (C++ oracle)", "data": "synthetic",
            "config": bench_config(cfg, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"each step: {nseq} sequences of the {cfg['h']}-wide layer decoded one "
                                       f"position through one layer of the C++ fp32 oracle ({threads} threads); "
                                       f"{n_all} steps"},
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
    codec = measure_codec(fq, torch, synth, dev, hbm, points=codec_sweep_points())
    print(json.dumps({"mode": "codec", "unit": "GB/s", "peak_hbm_gbs": hbm, "codec": codec}), flush=True)


def run_kernel_only(args):
    """One step of the decode layer (or the codec on 1 GiB) 3 times on one layer of the
    workload, with a device synchronisation after each call: the small case that the
    ncu captures under profiles/ run."""
    import torch
    import group_wise_int4_b200 as fq
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = workload_cfg(args.workload, 1)
    b, s, h, nh, d, ffn = cfg["call_batch"], cfg["prompt"], cfg["h"], cfg["n_heads"], cfg["head_dim"], cfg["ffn"]
    pos = s + cfg["decode_steps"] // 2
    k = args.kernel
    if k in ("compress", "decompress"):
        shape, cfgq = (131072, 4096), fq.config(4, 64, 1)
        xt = synth.codec_tensor(shape, 1, 64, 9, device=dev)
        codes, meta = fq.flexq_compress(xt, cfgq)
        fn = ((lambda: fq.flexq_compress(xt, cfgq, codes, meta)) if k == "compress"
              else (lambda: fq.flexq_decompress(codes, meta, shape, cfgq, xt)))
    else:
        layer = fq.FlexLayer(synth.layer_params(h, ffn, cfg["seed"], device=dev), nh, device=dev)
        cache = fq.FlexKVCache(b, nh, d, s + cfg["decode_steps"], device=dev)
        kh, vh = synth.kv_history(b, nh, pos, d, cfg["seed"], device=dev)
        cache.fill_from(kh, vh)
        del kh, vh
        x = synth.activations((b, 3 * h), 5, device=dev)
        x[:, :h] *= d ** -0.5
        xf = synth.activations((b, ffn), 6, device=dev)
        y = torch.empty((b, max(3 * h, ffn)), dtype=torch.float16, device=dev)
        if k.startswith("gemm_"):
            wkey, xin, n, epi = {"gemm_qkv": ("w_qkv", x[:, :h], 3 * h, 0), "gemm_out": ("w_o", x[:, :h], h, 0),
                                 "gemm_fc1": ("w_fc1", x[:, :h], ffn, 1), "gemm_fc2": ("w_fc2", xf, h, 0)}[k]
            kk = xin.shape[1]
            ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(b, n, kk)), dtype=torch.uint8, device=dev)
            yo = y[:, :n].contiguous()
            fn = lambda: fq.flex_dequant_gemm(xin.contiguous(), layer.w[wkey], None, None, yo, b,
                                              epi | fq.FLEX_GEMM_X_INTERLEAVED, ws)
        elif k == "decode_attention":
            ws = torch.zeros(max(16, fq.flex_decode_attention_ws_bytes(cache, b, pos)), dtype=torch.uint8, device=dev)
            o = torch.empty((b, h), dtype=torch.float16, device=dev)
            fn = lambda: fq.flex_decode_attention(cache, x[:, :h], x[:, h:], x[:, 2 * h:], 3 * h, o, b, pos, ws)
        elif k == "layernorm":
            o = torch.empty((b, h), dtype=torch.float16, device=dev)
            fn = lambda: fq.flex_layernorm(x[:, :h], layer.vec["ln1_g"], layer.vec["ln1_b"], o, b, h)
        elif k == "decode_layer":
            ws = torch.zeros(fq.flex_workspace_bytes(layer, b, 1), dtype=torch.uint8, device=dev)
            xin = synth.decode_inputs(b, h, 0, cfg["seed"], device=dev)
            o = torch.empty((b, h), dtype=torch.float16, device=dev)
            fn = lambda: fq.flex_decode_layer(layer, cache, xin, o, b, pos, ws)
        else:                                            # prefill_layer, a 128-token prompt
            sp = 128
            ws = torch.zeros(fq.flex_workspace_bytes(layer, b, sp), dtype=torch.uint8, device=dev)
            xin = synth.activations((b, sp, h), cfg["seed"], device=dev)
            o = torch.empty_like(xin)
            fn = lambda: fq.flex_prefill_layer(layer, cache, xin, o, b, sp, ws)
    times = []
    for _ in range(3):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    rc = fq.flex_get_status()
    if rc != 0:
        raise RuntimeError(f"{k} failed: {fq.flex_status_string(rc)}")
    print(json.dumps({"mode": "kernel", "kernel": k, "workload": cfg["name"], "call_batch": b, "pos": pos,
                      "us_per_call_cold": times}), flush=True)


def main():
    args = parse_args()
    if args.kernel:
        run_kernel_only(args)
    elif args.codec_only:
        run_codec_only()
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_flexq(args)


if __name__ == "__main__":
    main()
