#!/usr/bin/env python
"""Decode-step benchmark of the quantised-KV decode-attention path on B200.

Workload (default): B=16, 32 layers, 32 query / 8 KV heads, head_dim 128,
8K context (8191 cached + 1 appended per step), per-(token, head) fp16 scales.
One step = for every layer: quantize-on-append of the new token's K and V,
split-KV decode attention, merge of the partials -- captured in one CUDA graph.
The headline variant is K8V8; K8V4, K4V4, F8 (FP8 e4m3 keys and values), A8
(asymmetric INT8 with zero-points) and T8 (per-tensor INT8) are reported under
"variants".

value  = KV bytes read per step (codes + scales of every attended token, all
         layers and sequences, summed over ranks) / device time per step.
e2e    = the same metric through the public API (eager C-ABI calls) with the
         step's inputs copied from pinned host memory and the outputs copied
         back inside the timed region.
roofline = the decode-attention kernel alone, timed live by CUDA event nodes
         inside the step graph, against the measured HBM copy bandwidth.
cpu_baseline = the CPU oracle (fp64 attention) on one layer of one step.

Multi-GPU: replicas only (every rank runs the full workload on its own GPU; no
data-path collective); launched with torch.distributed.run, max time over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn KV GB/s (% of HBM peak) and steps/s at 8K ctx, K8V8/K8V4/K4V4"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
# (k_bits, v_bits, k_group, v_group, kv_format); F8: FP8 e4m3 keys and values; A8:
# asymmetric INT8 (scale + zero-point per (token, head)); T8: per-tensor INT8 (one
# scale per K / V tensor of a layer, set from the tensor's absmax before the prefill)
VARIANTS = {"K8V8": (8, 8, 128, 128, 0), "K8V4": (8, 4, 128, 128, 0), "K4V4": (4, 4, 128, 128, 0),
            "F8": (8, 8, 128, 128, 1), "A8": (8, 8, 128, 128, 2), "T8": (8, 8, 128, 128, 3)}


def tensor_scale_bits(x) -> int:
    """fp16 bits of a per-tensor INT8 scale max|x| / 127, as a caller would calibrate it."""
    import numpy as np
    return int(np.float16(float(x.float().abs().max()) / 127.0).view(np.uint16))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def bf16_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 1590.0, 1400.0, "fallback"


def decode_kernel_sha() -> str:
    """sha256 over the decode kernels' device sources (kernels, PTX wrappers, quantiser)."""
    import hashlib
    h = hashlib.sha256()
    for name in ("kvq_decode_kernel.cuh", "kvq_decode_common.cuh", "kvq_decode_tc.cu",
                 "kvq_ptx.cuh", "kvq_quant.cuh"):
        with open(os.path.join(ROOT, "quantized_kv_cache_22_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def decode_traffic(variant: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on
    the current decode kernel sources (decode_kernel_sha); otherwise None."""
    f = os.path.join(ROOT, "profiles", "decode_kernel_traffic.txt")
    if not os.path.exists(f):
        return None
    vals = {}
    for line in open(f):
        parts = line.split()
        if len(parts) == 2 and not line.startswith("#"):
            vals[parts[0]] = parts[1]
    if vals.get("sha256") != decode_kernel_sha():
        return None
    return float(vals[variant]) if variant in vals else None


def bench_config(w, head: str, world: int) -> dict:
    """The workload description both arms print (identical dicts)."""
    return {"workload": w.name, "kv": head, "batch": w.batch, "layers": w.n_layers,
            "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "context": w.context, "scales": "fp16 per (token, head)",
            "l2": "inputs larger than L2 (cache >= 4.4 GB per variant)",
            "parallelism": f"replicas x{world}"}


def l2_rotation(bytes_per_step: int, device) -> int:
    """Copies of a workload's caches to rotate through so that the bytes read between
    two reads of the same copy are at least twice the L2 size."""
    import torch
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    return max(1, -(-2 * l2 // bytes_per_step))


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a scalar over ranks (identity without a process group)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm

def build_variant(w, fmt, device):
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs

    kb, vb, kg, vg, kf = fmt
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=kb, v_bits=vb,
                 k_group=kg, v_group=vg, n_layers=w.n_layers, kv_format=kf)
    L = w.context
    caches = []
    pos0 = torch.zeros(w.batch, dtype=torch.int32, device=device)
    for layer in range(w.n_layers):
        c = LayerCache(cfg, device)
        k, v = inputs.kv_tokens(w, layer, L - 1, device)
        if kf == kvq.KVQ_FMT_TENSOR:
            for t, x in ((c.k_scales, k), (c.v_scales, v)):
                t.view(torch.int16)[0] = (tensor_scale_bits(x) ^ 0x8000) - 0x8000
        kvq.kvq_append(cfg, c, k, v, pos0, 0, L - 1)
        del k, v
        caches.append(c)
    torch.cuda.synchronize(device)
    st = {"cfg": cfg, "caches": caches,
          "d_pos": torch.full((w.batch,), L - 1, dtype=torch.int32, device=device),
          "d_len": torch.full((w.batch,), L, dtype=torch.int32, device=device),
          "ws": Workspace(cfg, 0, device)}
    knew, vnew, qs = [], [], []
    for layer in range(w.n_layers):
        k1, v1 = inputs.kv_tokens(w, layer, 1, device, offset_seed=1)
        knew.append(k1)
        vnew.append(v1)
        qs.append(inputs.queries(w, layer, 0, device))
    st["k_new"] = torch.stack(knew)
    st["v_new"] = torch.stack(vnew)
    st["q"] = torch.stack(qs)
    st["out"] = torch.empty_like(st["q"])
    return st


def capture_step(w, st):
    import torch
    import quantized_kv_cache_22_b200 as kvq
    cfg, L = st["cfg"], w.context
    ev_s = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(w.n_layers)]
    ev_e = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(w.n_layers)]

    def step(timed_events: bool):
        # one launch per layer: append the new token, attend, merge
        for layer in range(w.n_layers):
            if timed_events:
                ev_s[layer].record()
            kvq.kvq_append_decode_attn(cfg, st["caches"][layer], st["k_new"][layer],
                                       st["v_new"][layer], st["q"][layer], st["d_len"], L,
                                       st["out"][layer], st["ws"])
            if timed_events:
                ev_e[layer].record()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(False)   # warm the host-side memos outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    # the step as a user runs it: consecutive layers' kernels are programmatic
    # dependents, so each is scheduled while the previous one drains
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(False)
    # the same step with an event pair around each launch, for the kernel's own
    # duration (the event nodes serialise the launches)
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge):
        step(True)
    torch.cuda.synchronize()
    return g, ge, ev_s, ev_e, step


def time_graph(g, steps, warmup, world, device, sampler=None):
    import torch
    import torch.distributed as dist
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.start()
        time.sleep(0.25)
    a.record()
    for _ in range(steps):
        g.replay()
    b.record()
    b.synchronize()
    clocks = sampler.stop() if sampler else None
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = a.elapsed_time(b) / steps
    return reduce_max(ms, world, device), clocks


def time_e2e(w, st, steps, warmup, world, device):
    """Public-API step with host buffers: H2D inputs, eager ABI calls, D2H outputs."""
    import torch
    import torch.distributed as dist
    import quantized_kv_cache_22_b200 as kvq
    cfg, L = st["cfg"], w.context
    h_q = st["q"].cpu().pin_memory()
    h_k = st["k_new"].cpu().pin_memory()
    h_v = st["v_new"].cpu().pin_memory()
    h_out = torch.empty(st["out"].shape, dtype=st["out"].dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v))
    d2h = h_out.numel() * h_out.element_size()

    # Inputs go up on a copy stream in growing chunks of layers (layer 0 alone, then
    # 1-3, 4-11, 12-): the compute stream waits only at a chunk's first layer, by which
    # time the chunk has long landed, so the programmatic launches between layers break
    # three times per step.  Each layer's output goes back on the copy stream as soon
    # as its kernel ends.  The step ends when its last output is on the host.
    copy = torch.cuda.Stream()
    done = [torch.cuda.Event() for _ in range(w.n_layers)]
    bounds = [0] + [b for b in (1, 4, 12) if b < w.n_layers] + [w.n_layers]
    chunks = list(zip(bounds[:-1], bounds[1:]))
    landed = [torch.cuda.Event() for _ in chunks]
    first = {a: i for i, (a, _) in enumerate(chunks)}

    def one():
        cur = torch.cuda.current_stream()
        copy.wait_stream(cur)   # the previous step is done with the input buffers
        with torch.cuda.stream(copy):
            for i, (a, b) in enumerate(chunks):
                st["q"][a:b].copy_(h_q[a:b], non_blocking=True)
                st["k_new"][a:b].copy_(h_k[a:b], non_blocking=True)
                st["v_new"][a:b].copy_(h_v[a:b], non_blocking=True)
                landed[i].record(copy)
        for layer in range(w.n_layers):
            if layer in first:
                cur.wait_event(landed[first[layer]])
            kvq.kvq_append_decode_attn(cfg, st["caches"][layer], st["k_new"][layer],
                                       st["v_new"][layer], st["q"][layer], st["d_len"], L,
                                       st["out"][layer], st["ws"])
            done[layer].record(cur)
            copy.wait_event(done[layer])
            with torch.cuda.stream(copy):
                h_out[layer].copy_(st["out"][layer], non_blocking=True)
        cur.wait_stream(copy)   # the step ends when its outputs are on the host

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        one()
    b.record()
    b.synchronize()
    ms = reduce_max(a.elapsed_time(b) / steps, world, device)
    return ms, h2d, d2h


def cpu_oracle_layer(w, fmt, st=None, device=None, reps=1, budget_s=0.0, single=False):
    """Time the oracle on one layer of one decode step: quantize the new token's K/V,
    then fp64 attention for every (sequence, query head) over the 8K context.
    Runs `reps` times, and more until `budget_s` seconds of CPU work have passed, on
    every host core; with `single`, also once on one thread (returned third)."""
    import numpy as np
    import torch
    import oracle
    from quantized_kv_cache_22_b200 import inputs

    kb, vb, kg, vg, kf = fmt
    # the oracle's width arguments
    kb_o, vb_o = {1: ("e4m3", "e4m3"), 2: ("asym8", "asym8")}.get(kf, (kb, vb))
    L = w.context
    gen_dev = device if device is not None else "cpu"
    k, v = inputs.kv_tokens(w, 0, L - 1, gen_dev)
    k1, v1 = inputs.kv_tokens(w, 0, 1, gen_dev, offset_seed=1)
    q = inputs.queries(w, 0, 0, gen_dev)
    s16 = (tensor_scale_bits(k), tensor_scale_bits(v)) if kf == 3 else (0, 0)
    k_f = k.float().cpu().numpy().transpose(0, 2, 1, 3)
    v_f = v.float().cpu().numpy().transpose(0, 2, 1, 3)
    del k, v

    def quant(x, grp, bits_o, sc):
        if kf == 3:   # per-tensor: the per-head layout with every row's scale equal to sc
            return (oracle.quantize_rows_tensor(x, sc),
                    np.full(x.shape[:-1] + (1,), sc, np.uint16))
        return oracle.quantize_rows(x, grp, bits_o)

    kc = np.zeros((w.batch, w.n_kv_heads, L, w.head_dim * kb // 8), np.uint8)
    vc = np.zeros((w.batch, w.n_kv_heads, L, w.head_dim * vb // 8), np.uint8)
    a, b = quant(np.ascontiguousarray(k_f), kg, kb_o, s16[0])
    ks = np.zeros((w.batch, w.n_kv_heads, L) + b.shape[3:], np.uint16)
    kc[:, :, : L - 1], ks[:, :, : L - 1] = a, b
    a, b = quant(np.ascontiguousarray(v_f), vg, vb_o, s16[1])
    vs = np.zeros((w.batch, w.n_kv_heads, L) + b.shape[3:], np.uint16)
    vc[:, :, : L - 1], vs[:, :, : L - 1] = a, b
    del k_f, v_f
    k1f = np.ascontiguousarray(k1.float().cpu().numpy().transpose(0, 2, 1, 3))
    v1f = np.ascontiguousarray(v1.float().cpu().numpy().transpose(0, 2, 1, 3))
    qf = q.float().cpu().numpy()
    lens = np.full(w.batch, L, np.int32)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()

    def one(threads):
        t0 = time.perf_counter()
        a, b = quant(k1f, kg, kb_o, s16[0])
        kc[:, :, L - 1:], ks[:, :, L - 1:] = a, b
        a, b = quant(v1f, vg, vb_o, s16[1])
        vc[:, :, L - 1:], vs[:, :, L - 1:] = a, b
        oracle.decode_layer(qf, lens, kc, ks, kb_o, kg, vc, vs, vb_o, vg, w.n_kv_heads, 0.0, threads)
        return time.perf_counter() - t0

    times = []
    while len(times) < reps or (sum(times) < budget_s and len(times) < 1000):
        times.append(one(cores))
    if single:
        return times, cores, one(1)
    return times, cores


def time_cpu(fn, budget_s: float, max_reps: int = 50):
    """Mean wall time of fn() over repetitions until about budget_s has passed."""
    times = []
    while not times or (sum(times) < budget_s and len(times) < max_reps):
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    return statistics.mean(times), len(times)


def host_cores() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def run_tiny(args, world, device, cpu: bool):
    """mni-ml benchmark shape: B=1, 1 layer, 4 heads x 64, fp32 inputs, INT8 per (token,
    head); a 4-token prompt, then 252 decode steps, each one kvq_append_decode_attn
    (append the new token, attend over all cached tokens).  Launch-bound: steps/s."""
    import numpy as np
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs

    w = inputs.WORKLOADS[1]
    n_prompt, n_gen = 4, 252
    cfg = Config(batch=1, capacity=w.capacity, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                 head_dim=w.head_dim, k_bits=8, v_bits=8, k_group=w.head_dim,
                 v_group=w.head_dim)
    k, v = inputs.kv_tokens(w, 0, n_prompt + n_gen, device)          # [1, 256, 4, 64] fp32
    qs = torch.stack([inputs.queries(w, 0, s, device) for s in range(n_gen)])
    k_new = k[:, n_prompt:].transpose(0, 1).contiguous()              # [252, 1, 4, 64]
    v_new = v[:, n_prompt:].transpose(0, 1).contiguous()
    lens = torch.arange(n_prompt + 1, n_prompt + n_gen + 1, dtype=torch.int32,
                        device=device).view(n_gen, 1)
    cache = LayerCache(cfg, device)
    ws = Workspace(cfg, 0, device)
    out = torch.empty(n_gen, 1, w.n_q_heads, w.head_dim, dtype=torch.float32, device=device)
    kvq.kvq_append(cfg, cache, k[:, :n_prompt].contiguous(), v[:, :n_prompt].contiguous(),
                   torch.zeros(1, dtype=torch.int32, device=device), 0, n_prompt)

    def generate():
        for s in range(n_gen):
            kvq.kvq_append_decode_attn(cfg, cache, k_new[s], v_new[s], qs[s], lens[s],
                                       n_prompt + 1 + s, out[s], ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        generate()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        generate()
    reps = max(3, min(args.steps, 50))
    gms, _ = time_graph(g, reps, args.warmup, world, device)
    # the same generation as eager ABI calls (host launch cost included)
    for _ in range(args.warmup):
        generate()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        generate()
    b.record()
    b.synchronize()
    ems = reduce_max(a.elapsed_time(b) / reps, world, device)
    assert kvq.kvq_workspace_status(ws) == 0
    res = {"workload": w.name, "kv": "K8V8", "prompt": n_prompt, "generated": n_gen,
           "graph": {"ms_per_generation": round(gms, 4),
                     "steps_per_s": round(world * n_gen * 1e3 / gms, 1),
                     "us_per_step": round(gms * 1e3 / n_gen, 3)},
           "eager": {"ms_per_generation": round(ems, 4),
                     "steps_per_s": round(world * n_gen * 1e3 / ems, 1),
                     "us_per_step": round(ems * 1e3 / n_gen, 3)},
           "bound": "launch latency (about 1 KB of KV per step)", "gpu_launches": n_gen}
    if cpu:
        import oracle
        kf = k.float().cpu().numpy().transpose(0, 2, 1, 3).copy()   # [1, 4, 256, 64]
        vf = v.float().cpu().numpy().transpose(0, 2, 1, 3).copy()
        qn = qs.float().cpu().numpy()
        kc = np.zeros((1, w.n_kv_heads, w.capacity, w.head_dim), np.uint8)
        vc = np.zeros_like(kc)
        ks = np.zeros((1, w.n_kv_heads, w.capacity, 1), np.uint16)
        vs = np.zeros_like(ks)

        def gen_cpu(threads):
            kc[:, :, :n_prompt], ks[:, :, :n_prompt] = oracle.quantize_rows(
                kf[:, :, :n_prompt].copy(), w.head_dim, 8)
            vc[:, :, :n_prompt], vs[:, :, :n_prompt] = oracle.quantize_rows(
                vf[:, :, :n_prompt].copy(), w.head_dim, 8)
            for s_ in range(n_gen):
                t = n_prompt + s_
                kc[:, :, t:t + 1], ks[:, :, t:t + 1] = oracle.quantize_rows(
                    kf[:, :, t:t + 1].copy(), w.head_dim, 8)
                vc[:, :, t:t + 1], vs[:, :, t:t + 1] = oracle.quantize_rows(
                    vf[:, :, t:t + 1].copy(), w.head_dim, 8)
                oracle.decode_layer(qn[s_], np.array([t + 1], np.int32), kc, ks, 8, w.head_dim,
                                    vc, vs, 8, w.head_dim, w.n_kv_heads, 0.0, threads)

        cores = host_cores()
        t_all, n_all = time_cpu(lambda: gen_cpu(cores), 2.0)
        t_one, n_one = time_cpu(lambda: gen_cpu(1), 2.0)
        res["cpu_baseline"] = {"kind": "oracle", "unit": "steps/s", "cores": cores,
                               "value": round(n_gen / t_all, 1),
                               "single_thread": {"value": round(n_gen / t_one, 1), "cores": 1,
                                                 "sample": f"{n_one} whole generations"},
                               "sample": f"{n_all} whole generations (prompt + 252 steps)"}
    return res


def _rotated_caches(w, cfg, copies, device):
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import LayerCache, inputs
    L = w.context
    pos0 = torch.zeros(w.batch, dtype=torch.int32, device=device)
    out = []
    for _ in range(copies):
        caches = []
        for layer in range(w.n_layers):
            c = LayerCache(cfg, device)
            k, v = inputs.kv_tokens(w, layer, L - 1, device)
            kvq.kvq_append(cfg, c, k, v, pos0, 0, L - 1)
            caches.append(c)
        out.append(caches)
    torch.cuda.synchronize()
    return out


def _oracle_step_timer(w, fmt, device):
    """A closure that runs one whole decode step (every layer: quantise the new token,
    fp64 attention) through the oracle, on the given number of threads."""
    import numpy as np
    import oracle
    from quantized_kv_cache_22_b200 import inputs
    kb, vb, kg, vg = fmt
    L = w.context
    layers = []
    for layer in range(w.n_layers):
        k, v = inputs.kv_tokens(w, layer, L, device)
        kf = k.float().cpu().numpy().transpose(0, 2, 1, 3).copy()
        vf = v.float().cpu().numpy().transpose(0, 2, 1, 3).copy()
        kc, ks = oracle.quantize_rows(kf[:, :, :L - 1].copy(), kg, kb)
        vc, vs = oracle.quantize_rows(vf[:, :, :L - 1].copy(), vg, vb)
        pad = lambda a: np.concatenate([a, np.zeros(a.shape[:2] + (1,) + a.shape[3:], a.dtype)], 2)
        q = inputs.queries(w, layer, 0, device).float().cpu().numpy()
        layers.append((pad(kc), pad(ks), pad(vc), pad(vs), kf[:, :, L - 1:].copy(),
                       vf[:, :, L - 1:].copy(), q))
    lens = np.full(w.batch, L, np.int32)

    def step(threads):
        for kc, ks, vc, vs, k1, v1, q in layers:
            kc[:, :, L - 1:], ks[:, :, L - 1:] = oracle.quantize_rows(k1, kg, kb)
            vc[:, :, L - 1:], vs[:, :, L - 1:] = oracle.quantize_rows(v1, vg, vb)
            oracle.decode_layer(q, lens, kc, ks, kb, kg, vc, vs, vb, vg, w.n_kv_heads, 0.0, threads)
    return step


def run_rotated(args, world, device, widx: int, fmt, label: str, cpu: bool):
    """A whole decode step (every layer: append the new token, attend, merge; one
    kvq_append_decode_attn per layer) of a workload whose caches are near the L2
    size: the timed graph rotates over copies of the caches totalling at least
    twice the L2, so that every step reads its KV bytes from HBM."""
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import Config, Workspace, inputs

    w = inputs.WORKLOADS[widx]
    kb, vb, kg, vg = fmt
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=kb, v_bits=vb,
                 k_group=kg, v_group=vg, n_layers=w.n_layers)
    L = w.context
    per_tok_layer = kvq.kvq_cache_bytes(cfg)[0]
    per_layer = per_tok_layer * w.batch * L
    step_bytes = per_layer * w.n_layers
    R = l2_rotation(step_bytes, device)
    copies = _rotated_caches(w, cfg, R, device)
    knew, vnew, qs = [], [], []
    for layer in range(w.n_layers):
        k1, v1 = inputs.kv_tokens(w, layer, 1, device, offset_seed=1)
        knew.append(k1[:, 0])
        vnew.append(v1[:, 0])
        qs.append(inputs.queries(w, layer, 0, device))
    k_new, v_new, q = torch.stack(knew), torch.stack(vnew), torch.stack(qs)
    out = torch.empty_like(q)
    d_len = torch.full((w.batch,), L, dtype=torch.int32, device=device)
    ws = Workspace(cfg, 0, device)

    def steps():
        for caches in copies:
            for layer in range(w.n_layers):
                kvq.kvq_append_decode_attn(cfg, caches[layer], k_new[layer], v_new[layer],
                                           q[layer], d_len, L, out[layer], ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        steps()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        steps()
    reps = max(3, min(args.steps, 100))
    ms_r, _ = time_graph(g, reps, args.warmup, world, device)
    ms = ms_r / R
    assert kvq.kvq_workspace_status(ws) == 0
    hbm_peak, peak_kind = measured_peaks()
    launch_gbs = per_layer / (ms / w.n_layers * 1e-3) / 1e9
    res = {"workload": w.name, "kv": label, "batch": w.batch, "layers": w.n_layers,
           "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "context": L,
           "bytes_per_token_layer": per_tok_layer, "kv_bytes_per_step": step_bytes,
           "l2": f"{R} copies of the caches rotated ({R * step_bytes / 1e6:.1f} MB >= 2 x L2)",
           "ms_per_step": round(ms, 5), "steps_per_s": round(world * 1e3 / ms, 1),
           "kv_gbs": round(world * step_bytes / (ms * 1e-3) / 1e9, 1),
           "roofline": {"bound": "hbm", "kernel": "decode_kernel (append + attention + merge)",
                        "achieved": round(launch_gbs, 1), "peak": hbm_peak,
                        "peak_kind": peak_kind, "unit": "GB/s",
                        "frac": round(launch_gbs / hbm_peak, 4),
                        "launch_ms": round(ms / w.n_layers, 5),
                        "timing": f"in step: ms_per_step / {w.n_layers}"},
           "gpu_launches_per_step": w.n_layers}
    del copies
    if cpu:
        step = _oracle_step_timer(w, fmt, device)
        cores = host_cores()
        t_all, n_all = time_cpu(lambda: step(cores), 5.0)
        t_one, n_one = time_cpu(lambda: step(1), 5.0)
        res["cpu_baseline"] = {"kind": "oracle", "unit": "steps/s", "cores": cores,
                               "value": round(1.0 / t_all, 3),
                               "kv_gbs": round(step_bytes / t_all / 1e9, 4),
                               "single_thread": {"value": round(1.0 / t_one, 3), "cores": 1,
                                                 "kv_gbs": round(step_bytes / t_one / 1e9, 4),
                                                 "sample": f"{n_one} whole steps"},
                               "sample": f"{n_all} whole steps ({w.n_layers} layers each)"}
    torch.cuda.empty_cache()
    return res



def run_hmode(args, world, device, cpu: bool = False):
    """h-mode workload: INT4-h cache of B=8 x 1024 tokens, D=2048, 16 heads x 128;
    one call = rebuild K/V with the tcgen05 GEMM (137.4 GFLOP) + decode attention."""
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs

    w = inputs.WORKLOADS[5]
    S, D, H = w.context, w.d_model, w.n_kv_heads
    cfg = Config(batch=w.batch, capacity=w.capacity, mode=kvq.KVQ_MODE_H, d_model=D, h_bits=4,
                 h_groups=16, n_q_heads=w.n_q_heads, n_kv_heads=H, head_dim=w.head_dim)
    h, W = inputs.hmode_inputs(w, S, device)
    cache = LayerCache(cfg, device)
    kvq.kvq_append(cfg, cache, h, None, torch.zeros(w.batch, dtype=torch.int32, device=device), 0, S)
    del h
    q = inputs.queries(w, 0, 0, device)
    out = torch.empty_like(q)
    ws = Workspace(cfg, 0, device)
    scratch = torch.empty(kvq.kvq_h_scratch_bytes(cfg, S) // 2, dtype=torch.float16, device=device)
    nkv = w.batch * H * S * w.head_dim
    k_out = scratch[:nkv].view(w.batch, H, S, w.head_dim)
    v_out = scratch[nkv:2 * nkv].view(w.batch, H, S, w.head_dim)
    d_len = torch.full((w.batch,), S, dtype=torch.int32, device=device)
    flops = 2.0 * w.batch * S * (2 * H * w.head_dim) * D

    operand = torch.empty(kvq.kvq_h_operand_bytes(cfg, S) // 2, dtype=torch.bfloat16, device=device)

    def gemm():
        kvq.kvq_h_reconstruct(cfg, cache, W, S, k_out, v_out, S, operand)

    def step():
        kvq.kvq_decode_attn(cfg, cache, q, d_len, S, out, ws, w_kv=W, kv_scratch=scratch)

    res = {"workload": w.name, "h_bits": 4, "gflop_per_call": round(flops / 1e9, 2)}
    for name, fn in (("gemm", gemm), ("step", step)):
        for _ in range(max(args.warmup, 3)):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        n = max(3, min(args.steps, 100))
        a.record()
        for _ in range(n):
            fn()
        b.record()
        b.synchronize()
        res[f"{name}_ms"] = round(reduce_max(a.elapsed_time(b) / n, world, device), 5)
    assert kvq.kvq_workspace_status(ws) == 0
    burst, sustained, kind = bf16_peaks()
    tf = flops / (res["gemm_ms"] * 1e-3) / 1e12
    res["gemm_tflops"] = round(tf, 1)
    res["roofline"] = {"bound": "tensor", "kernel": "hgemm_kernel (tcgen05 bf16, fp32 acc)",
                       "achieved": round(tf, 1), "peak": burst, "peak_kind": kind + " burst",
                       "unit": "TFLOP/s", "frac": round(tf / burst, 4),
                       "frac_of_sustained": round(tf / sustained, 4)}
    res["steps_per_s"] = round(world * 1e3 / res["step_ms"], 2)

    # the attention half alone (over the K/V the reconstruction just wrote, as the
    # h-mode decode runs it): 16-bit K and V, G = 1; its 67 MB fit in L2, so every
    # timed call follows a 256 MB write that flushes L2
    gemm()
    cfg16 = Config(batch=w.batch, capacity=S, n_q_heads=w.n_q_heads, n_kv_heads=H,
                   head_dim=w.head_dim, k_bits=16, v_bits=16)
    kv16 = LayerCache.__new__(LayerCache)
    kv16.cfg, kv16.block_table = cfg16, None
    kv16.k_codes, kv16.k_scales = k_out.reshape(-1).view(torch.uint8), None
    kv16.v_codes, kv16.v_scales = v_out.reshape(-1).view(torch.uint8), None
    ws16 = Workspace(cfg16, 0, device)
    flush_a6 = torch.empty(256 * 1024 * 1024 // 4, device=device)

    def attn():
        kvq.kvq_decode_attn(cfg16, kv16, q, d_len, S, out, ws16)

    for _ in range(max(args.warmup, 3)):
        attn()
    na = max(3, min(args.steps, 100))
    evs_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(na)]
    for a, b in evs_a:
        flush_a6.fill_(1.0)
        a.record()
        attn()
        b.record()
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws16) == 0
    a6_ms = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in evs_a), world, device)
    a6_bytes = 2 * k_out.numel() * k_out.element_size()
    hbm_a6, hkind_a6 = measured_peaks()
    a6_gbs = a6_bytes / (a6_ms * 1e-3) / 1e9
    res["attention"] = {"kernel": "decode_kernel<16-bit K, 16-bit V>", "ms": round(a6_ms, 5),
                        "bytes": a6_bytes, "l2": "flushed before each call",
                        "roofline": {"bound": "hbm", "achieved": round(a6_gbs, 1),
                                     "peak": hbm_a6, "peak_kind": hkind_a6, "unit": "GB/s",
                                     "frac": round(a6_gbs / hbm_a6, 4)},
                        "share_of_step": round(a6_ms / res["step_ms"], 3)}
    del flush_a6

    # the reconstruction fused into the attention (tcgen05 tiles of K_j | V_j attended
    # in the GEMM epilogue, nothing written back): tensor-bound like the GEMM
    fz_scratch = torch.zeros(kvq.kvq_h_fused_scratch_bytes(cfg, S) // 4, device=device)

    def fused():
        kvq.kvq_h_decode_fused(cfg, cache, W, q, d_len, S, out, fz_scratch)

    for _ in range(max(args.warmup, 3)):
        fused()
    torch.cuda.synchronize()
    fa = torch.cuda.Event(enable_timing=True)
    fb = torch.cuda.Event(enable_timing=True)
    nf = max(3, min(args.steps, 100))
    fa.record()
    for _ in range(nf):
        fused()
    fb.record()
    fb.synchronize()
    fms = reduce_max(fa.elapsed_time(fb) / nf, world, device)
    assert kvq.kvq_workspace_status(fz_scratch) == 0
    ftf = flops / (fms * 1e-3) / 1e12
    res["fused"] = {"kernels": "dequant_h, hgemm_kernel<fused>, fused_merge", "ms": round(fms, 5),
                    "steps_per_s": round(world * 1e3 / fms, 1),
                    "roofline": {"bound": "tensor", "achieved": round(ftf, 1), "peak": burst,
                                 "peak_kind": kind + " burst", "unit": "TFLOP/s",
                                 "frac": round(ftf / burst, 4)},
                    "speedup_vs_reconstruction_step": round(res["step_ms"] / fms, 2)}

    # the same attention by query absorption (W_k^T q against the h codes, W_v on
    # sum p h^): HBM-bound on the h codes + scales and W; the inputs (25 MB) fit in
    # L2, so every timed call follows a 256 MB L2 flush and is bracketed alone
    ab_scratch = torch.empty(kvq.kvq_h_absorbed_scratch_bytes(cfg, S) // 4, device=device)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=device)

    def absorbed():
        kvq.kvq_h_decode_absorbed(cfg, cache, W, q, d_len, S, out, ab_scratch)

    for _ in range(max(args.warmup, 3)):
        absorbed()
    n = max(3, min(args.steps, 100))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        flush.fill_(1.0)
        a.record()
        absorbed()
        b.record()
    torch.cuda.synchronize()
    ams = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in evs), world, device)
    h_bytes = kvq.kvq_cache_bytes(cfg)[0] * w.batch * S
    w_bytes = W.numel() * W.element_size()
    hbm, hkind = measured_peaks()
    gbs = (h_bytes + w_bytes) / (ams * 1e-3) / 1e9
    res["absorbed"] = {"kernels": "absorb_q, absorb_scores, absorb_pv, absorb_out",
                       "ms": round(ams, 5), "steps_per_s": round(world * 1e3 / ams, 1),
                       "bytes": h_bytes + w_bytes, "l2": "flushed before each call",
                       "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                                    "peak_kind": hkind, "unit": "GB/s",
                                    "frac": round(gbs / hbm, 4)},
                       "speedup_vs_reconstruction_step": round(res["step_ms"] / ams, 2)}
    if cpu:
        # the oracle's reconstruction (fp64 K, V = W bf16(h^)) and fp64 attention for one
        # of the 8 sequences: a bounded sample of the same call
        import numpy as np
        import oracle
        hc = cache.k_codes.cpu().numpy()[: w.batch * S * D // 2].reshape(w.batch, S, D // 2)
        hs = cache.k_scales.cpu().numpy().view(np.uint16)[: w.batch * S * 16].reshape(
            w.batch, S, 16)
        Wb = W.cpu().view(torch.int16).numpy().view(np.uint16)
        qn = q.float().cpu().numpy()

        def one_seq(threads, n_tok, b=0):
            _, y16 = oracle.h_reconstruct(hc[b, :n_tok], hs[b, :n_tok], D, 16, 4, Wb, True,
                                          threads)
            kv = y16.reshape(n_tok, 2, H, w.head_dim)
            kk = np.ascontiguousarray(kv[:, 0].transpose(1, 0, 2))[None]
            vv = np.ascontiguousarray(kv[:, 1].transpose(1, 0, 2))[None]
            oracle.decode_layer(qn[b:b + 1], np.array([n_tok], np.int32), kk, None, 16,
                                w.head_dim, vv, None, 16, w.head_dim, H, 0.0, threads)

        cores = host_cores()
        t_all, n_all = time_cpu(lambda: one_seq(cores, S), 5.0, 5)
        t_one, _ = time_cpu(lambda: one_seq(1, 128), 0.0, 1)
        per_step_one = t_one * (S / 128) * w.batch
        res["cpu_baseline"] = {"kind": "oracle", "unit": "steps/s", "cores": cores,
                               "value": round(1.0 / (t_all * w.batch), 5),
                               "single_thread": {"value": round(1.0 / per_step_one, 6),
                                                 "cores": 1,
                                                 "sample": "1 run over the first 128 tokens of "
                                                           "1 sequence, scaled to the call"},
                               "sample": f"{n_all} runs of 1 of the {w.batch} sequences "
                                         f"(reconstruction + attention), {t_all:.2f} s each; "
                                         "steps/s scaled to all sequences"}
    return res


def run_window(args, world, device):
    """Sliding-window workload: B=64 sequences that have seen 8192 tokens, each
    caching 64 anchors + the 1536 most recent (1600 tokens), K4V8; a step of a few
    layers, one kvq_append_decode_attn per layer (ring slot of the new token)."""
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs

    w = dataclasses.replace(inputs.WORKLOADS[6], n_layers=4)
    kb, vb, kg, vg = w.kv_variants[0]
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=kb, v_bits=vb,
                 k_group=kg, v_group=vg, n_layers=w.n_layers, window=w.window,
                 n_anchor=w.n_anchor)
    L = w.context                                  # tokens seen, the newest at L - 1
    first_win = L - 1 - w.window                   # window tokens cached before the step
    caches = []
    for layer in range(w.n_layers):
        c = LayerCache(cfg, device)
        k, v = inputs.kv_tokens(w, layer, w.capacity, device)
        kvq.kvq_append(cfg, c, k[:, :w.n_anchor].contiguous(), v[:, :w.n_anchor].contiguous(),
                       torch.zeros(w.batch, dtype=torch.int32, device=device), 0, w.n_anchor)
        kvq.kvq_append(cfg, c, k[:, w.n_anchor:].contiguous(), v[:, w.n_anchor:].contiguous(),
                       torch.full((w.batch,), first_win, dtype=torch.int32, device=device),
                       first_win, w.window)
        del k, v
        caches.append(c)
    st = {"cfg": cfg, "caches": caches,
          "d_len": torch.full((w.batch,), L, dtype=torch.int32, device=device),
          "ws": Workspace(cfg, 0, device)}
    kn, vn, qs = [], [], []
    for layer in range(w.n_layers):
        k1, v1 = inputs.kv_tokens(w, layer, 1, device, offset_seed=1)
        kn.append(k1[:, 0])
        vn.append(v1[:, 0])
        qs.append(inputs.queries(w, layer, 0, device))
    st["k_new"], st["v_new"], st["q"] = torch.stack(kn), torch.stack(vn), torch.stack(qs)
    st["out"] = torch.empty_like(st["q"])
    g, ge, ev_s, ev_e, _ = capture_step(w, st)
    ms, _ = time_graph(g, max(3, min(args.steps, 100)), args.warmup, world, device)
    for _ in range(args.warmup + 3):
        ge.replay()
    torch.cuda.synchronize()
    dec_ms = reduce_max(statistics.mean(ev_s[i].elapsed_time(ev_e[i]) for i in range(w.n_layers)),
                        world, device)
    assert kvq.kvq_workspace_status(st["ws"]) == 0
    per_layer = kvq.kvq_cache_bytes(cfg)[0] * w.batch * w.capacity
    return {"workload": w.name, "kv": "K4V8", "window": w.window, "n_anchor": w.n_anchor,
            "tokens_seen": L, "tokens_attended": w.capacity, "layers_timed": w.n_layers,
            "kv_bytes_per_layer": per_layer, "ms_per_layer": round(ms / w.n_layers, 5),
            "kv_gbs": round(world * per_layer * w.n_layers / (ms * 1e-3) / 1e9, 1),
            "roofline": step_roofline("decode_kernel (ring-slot append + attention + merge)",
                                      per_layer, ms, w.n_layers, dec_ms, decode_traffic("window"))}


def step_roofline(kernel, per_layer, ms, n_layers, dec_ms, traffic=None):
    """Roofline of a step that is nothing but n_layers decode launches chained by
    programmatic dependent launch: achieved = bytes per layer / (step time / layers);
    `isolated` keeps the event-bracketed time of each launch in a serialised copy."""
    hbm_peak, peak_kind = measured_peaks()
    in_step = ms / n_layers
    gbs = per_layer / (in_step * 1e-3) / 1e9
    iso = per_layer / (dec_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": round(gbs, 1), "peak": hbm_peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
            "traffic": traffic, "launch_ms": round(in_step, 5),
            "timing": "in step: ms_per_step / layers",
            "isolated": {"launch_ms": round(dec_ms, 5), "achieved": round(iso, 1),
                         "frac": round(iso / hbm_peak, 4),
                         "timing": "an event pair around each launch in a copy of the step "
                                   "graph (serialised launches, no programmatic overlap)"}}


def run_paged(args, world, device):
    """Paged layout of the 8K workload: each layer's cache is a pool of 1024 pages of
    128 tokens (16 sequences x 64 pages, shuffled by a seeded permutation) behind a
    block table; a step of four layers, one kvq_append_decode_attn per layer."""
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs

    w = dataclasses.replace(inputs.WORKLOADS[4], n_layers=4)
    kb, vb, kg, vg, _ = VARIANTS["K8V8"]
    pages = w.batch * (w.capacity // 128)
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=kb, v_bits=vb,
                 k_group=kg, v_group=vg, n_layers=w.n_layers, page_tokens=128, n_pages=pages)
    g = torch.Generator().manual_seed(w.seed)
    table = torch.randperm(pages, generator=g).view(w.batch, -1).to(torch.int32).to(device)
    L = w.context
    caches = []
    for layer in range(w.n_layers):
        c = LayerCache(cfg, device, block_table=table)
        k, v = inputs.kv_tokens(w, layer, L - 1, device)
        kvq.kvq_append(cfg, c, k, v, torch.zeros(w.batch, dtype=torch.int32, device=device), 0,
                       L - 1)
        del k, v
        caches.append(c)
    st = {"cfg": cfg, "caches": caches,
          "d_len": torch.full((w.batch,), L, dtype=torch.int32, device=device),
          "ws": Workspace(cfg, 0, device)}
    kn, vn, qs = [], [], []
    for layer in range(w.n_layers):
        k1, v1 = inputs.kv_tokens(w, layer, 1, device, offset_seed=1)
        kn.append(k1[:, 0])
        vn.append(v1[:, 0])
        qs.append(inputs.queries(w, layer, 0, device))
    st["k_new"], st["v_new"], st["q"] = torch.stack(kn), torch.stack(vn), torch.stack(qs)
    st["out"] = torch.empty_like(st["q"])
    g, ge, ev_s, ev_e, _ = capture_step(w, st)
    ms, _ = time_graph(g, max(3, min(args.steps, 100)), args.warmup, world, device)
    for _ in range(args.warmup + 3):
        ge.replay()
    torch.cuda.synchronize()
    dec_ms = reduce_max(statistics.mean(ev_s[i].elapsed_time(ev_e[i]) for i in range(w.n_layers)),
                        world, device)
    assert kvq.kvq_workspace_status(st["ws"]) == 0
    per_layer = kvq.kvq_cache_bytes(cfg)[0] * w.batch * w.context
    return {"workload": w.name + "-paged128", "kv": "K8V8", "page_tokens": 128, "pages": pages,
            "layers_timed": w.n_layers, "kv_bytes_per_layer": per_layer,
            "ms_per_layer": round(ms / w.n_layers, 5),
            "kv_gbs": round(world * per_layer * w.n_layers / (ms * 1e-3) / 1e9, 1),
            "roofline": step_roofline("decode_kernel (paged: block-table tiles)", per_layer, ms,
                                      w.n_layers, dec_ms)}


def run_gpu(args):
    import torch
    import quantized_kv_cache_22_b200 as kvq
    from quantized_kv_cache_22_b200 import inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    w = inputs.WORKLOADS[args.workload]
    if args.layers:
        w = dataclasses.replace(w, n_layers=args.layers)
    hbm_peak, peak_kind = measured_peaks()
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"

    results = {}
    main_state = None
    variants = args.variants if "kv" in args.sections else []
    for name in variants:
        fmt = VARIANTS[name]
        st = build_variant(w, fmt, device)
        g, ge, ev_s, ev_e, _ = capture_step(w, st)
        sampler = ClockSampler(gpu_id) if name == args.variants[0] else None
        ms, clocks = time_graph(g, args.steps, args.warmup, world, device, sampler)
        # kernel duration: mean over the layers of the last of a few event-graph replays
        for _ in range(args.warmup + 3):
            ge.replay()
        torch.cuda.synchronize()
        dec_ms = statistics.mean(ev_s[i].elapsed_time(ev_e[i]) for i in range(w.n_layers))
        dec_ms = reduce_max(dec_ms, world, device)
        per_tok_layer = kvq.kvq_cache_bytes(st["cfg"])[0]
        kv_bytes_layer = per_tok_layer * w.batch * w.context
        kv_bytes_step = kv_bytes_layer * w.n_layers
        results[name] = {
            "ms_per_step": ms,
            "steps_per_s": 1e3 / ms,
            "kv_bytes_per_step": kv_bytes_step,
            "kv_gbs": world * kv_bytes_step / (ms * 1e-3) / 1e9,
            "decode_kernel_ms": dec_ms,
            "decode_kernel_gbs": kv_bytes_layer / (dec_ms * 1e-3) / 1e9,
            "clocks": clocks,
            "plan": kvq.kvq_decode_plan_info(st["cfg"], 0),
        }
        # per decode launch inside the step (the step is only these launches)
        results[name]["in_step_gbs"] = kv_bytes_layer / (ms / w.n_layers * 1e-3) / 1e9
        results[name]["pct_hbm_measured"] = 100.0 * results[name]["in_step_gbs"] / hbm_peak
        results[name]["pct_hbm_nominal_8tbs"] = 100.0 * results[name]["in_step_gbs"] / NOMINAL_HBM_GBS
        results[name]["pct_hbm_measured_isolated"] = (100.0 * results[name]["decode_kernel_gbs"]
                                                      / hbm_peak)
        if name == args.variants[0]:
            main_state = (st, g, ge)
            if not args.no_e2e:
                e2e_steps = max(3, min(args.steps, 50))
                ems, h2d, d2h = time_e2e(w, st, e2e_steps, max(args.warmup, 3), world, device)
                results[name]["e2e"] = {"value": world * kv_bytes_step / (ems * 1e-3) / 1e9,
                                        "unit": "GB/s", "ms_per_step": ems,
                                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                                        "steps": e2e_steps}
        else:
            del g, ge, st
            torch.cuda.synchronize()
            torch.cuda.empty_cache()

    cpu_legs = rank == 0 and world == 1 and not args.no_cpu_baseline
    hmode = run_hmode(args, world, device, cpu_legs) if "hmode" in args.sections else None
    window = run_window(args, world, device) if "window" in args.sections else None
    paged = run_paged(args, world, device) if "paged" in args.sections else None
    tiny = run_tiny(args, world, device, cpu_legs) if "tiny" in args.sections else None
    int8kv = (run_rotated(args, world, device, 2, (8, 8, 128, 128), "K8V8", cpu_legs)
              if "int8kv" in args.sections else None)
    mixed = ([run_rotated(args, world, device, 3, f, n, cpu_legs)
              for f, n in (((8, 4, 128, 32), "K8V4"), ((4, 8, 32, 128), "K4V8"))]
             if "mixed" in args.sections else None)
    extra = {"hmode": hmode, "window": window, "paged": paged, "tiny": tiny, "int8kv": int8kv,
             "mixed": mixed}
    if not variants:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": None, **extra}), flush=True)
        return
    head = args.variants[0]
    r = results[head]
    line = {
        "metric": METRIC,
        "value": round(r["kv_gbs"], 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(r["ms_per_step"], 5),
        "steps_per_s": round(r["steps_per_s"], 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": bench_config(w, head, world),
        "execution": {"graph": "one CUDA graph per step",
                      "launch": "programmatic dependent launch between layers",
                      "decode_plan": r["plan"]},
        "pct_hbm_measured": round(r["pct_hbm_measured"], 2),
        "pct_hbm_nominal_8tbs": round(r["pct_hbm_nominal_8tbs"], 2),
        "roofline": {"bound": "hbm", "kernel": "decode_kernel (append + split-KV attention + merge)",
                     "achieved": round(r["in_step_gbs"], 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(r["in_step_gbs"] / hbm_peak, 4),
                     "traffic": args.traffic_bytes if args.traffic_bytes else decode_traffic(head),
                     "bytes_per_launch": r["kv_bytes_per_step"] // w.n_layers,
                     "launch_ms": round(r["ms_per_step"] / w.n_layers, 5),
                     "timing": f"in step: ms_per_step / {w.n_layers}; the step is nothing but the "
                               f"{w.n_layers} decode launches (one per layer), chained by "
                               "programmatic dependent launch",
                     "isolated": {"launch_ms": round(r["decode_kernel_ms"], 5),
                                  "achieved": round(r["decode_kernel_gbs"], 1),
                                  "frac": round(r["decode_kernel_gbs"] / hbm_peak, 4),
                                  "timing": "an event pair around each launch in a copy of the "
                                            "step graph (serialised launches, no programmatic "
                                            "overlap); mean over the layers"}},
        "variants": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv)
                         for kk, vv in v.items() if kk not in ("clocks", "e2e")}
                     for k, v in results.items()},
        "gpu_launches": args.steps * w.n_layers,   # one decode-step kernel per layer
        **extra,
        "clocks": r["clocks"],
    }
    if "e2e" in r:
        line["e2e"] = {k: (round(v, 3) if isinstance(v, float) else v) for k, v in r["e2e"].items()}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a bounded sample: the same layer of the step repeated for ~10 s of CPU work
        times, cores, t1 = cpu_oracle_layer(w, VARIANTS[head], device=device, reps=1,
                                            budget_s=10.0, single=True)
        t = statistics.mean(times)
        per_layer = r["kv_bytes_per_step"] / w.n_layers
        line["cpu_baseline"] = {"value": round(per_layer / t / 1e9, 4), "unit": "GB/s",
                                "single_thread": {"value": round(per_layer / t1 / 1e9, 4),
                                                  "unit": "GB/s", "cores": 1,
                                                  "sample": f"1 run of the same layer, {t1:.3f} s"},
                                "steps_per_s": round(1.0 / (t * w.n_layers), 5),
                                "cores": cores, "kind": "oracle",
                                "sample": f"{len(times)} runs of 1 of the {w.n_layers} layers of "
                                          f"one {head} step (quantize {w.batch}x{w.n_kv_heads} new "
                                          f"rows + fp64 attention for {w.batch}x{w.n_q_heads} heads "
                                          f"over {w.context} tokens), {sum(times):.1f} s in all, "
                                          f"{t:.3f} s per layer"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del main_state
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The CPU oracle as it stands, on the same workload and metric (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from quantized_kv_cache_22_b200.inputs import WORKLOADS
    import quantized_kv_cache_22_b200 as kvq
    w = WORKLOADS[args.workload]
    head = args.variants[0]
    fmt = VARIANTS[head]
    cfg = kvq.Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                     n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=fmt[0], v_bits=fmt[1],
                     k_group=fmt[2], v_group=fmt[3], n_layers=w.n_layers, kv_format=fmt[4])
    per_layer = kvq.kvq_cache_bytes(cfg)[0] * w.batch * w.context
    times, cores = cpu_oracle_layer(w, fmt, reps=args.warmup + args.steps)
    t = statistics.mean(times[args.warmup:]) if len(times) > args.warmup else statistics.mean(times)
    value = per_layer / t / 1e9
    sample = (f"each step = 1 of {w.n_layers} layers of one {head} decode step (quantize "
              f"{w.batch}x{w.n_kv_heads} new rows + fp64 attention, {w.batch}x{w.n_q_heads} heads "
              f"x {w.context} tokens)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(w, head, world),
            "step": f"a bounded CPU sample: each timed step is 1 of the {w.n_layers} layers of "
                    f"one decode step (ms_per_step is that layer's measured time; a whole "
                    f"{w.n_layers}-layer step would take {w.n_layers}x as long)",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("kvq", "reference"), default="kvq")
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--variants", default="K8V8,K8V4,K4V4,F8,A8,T8")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sections", default="kv,hmode,window,paged,tiny,int8kv,mixed",
                    help="kv: the 8K K/V decode step (headline); hmode: the h-mode workload; "
                         "window: the sliding-window workload; paged: the 8K step on a paged "
                         "cache; tiny: 4-token prompt + 252 steps (B=1, 4 heads x 64); int8kv: "
                         "INT8 KV at D=2048, 34 layers x 1024; mixed: K8V4 / K4V8 GQA 24/8, "
                         "28 layers x 2048 with outlier channels")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (small profiling captures only)")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="dram bytes per decode launch from an ncu capture of this kernel build")
    args = ap.parse_args()
    args.variants = [v.strip() for v in args.variants.split(",") if v.strip()]
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
