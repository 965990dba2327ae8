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
    """sha256 over the decode kernel's device sources (kernel, PTX wrappers, quantiser)."""
    import hashlib
    h = hashlib.sha256()
    for name in ("kvq_decode_kernel.cuh", "kvq_ptx.cuh", "kvq_quant.cuh"):
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


def run_hmode(args, world, device):
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
    hbm_peak, peak_kind = measured_peaks()
    gbs = per_layer / (dec_ms * 1e-3) / 1e9
    return {"workload": w.name, "kv": "K4V8", "window": w.window, "n_anchor": w.n_anchor,
            "tokens_seen": L, "tokens_attended": w.capacity, "layers_timed": w.n_layers,
            "kv_bytes_per_layer": per_layer, "ms_per_layer": round(ms / w.n_layers, 5),
            "kv_gbs": round(world * per_layer * w.n_layers / (ms * 1e-3) / 1e9, 1),
            "roofline": {"bound": "hbm", "kernel": "decode_kernel (ring-slot append + attention "
                         "+ merge)", "achieved": round(gbs, 1), "peak": hbm_peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
                         "launch_ms": round(dec_ms, 5)}}


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
    hbm_peak, peak_kind = measured_peaks()
    gbs = per_layer / (dec_ms * 1e-3) / 1e9
    return {"workload": w.name + "-paged128", "kv": "K8V8", "page_tokens": 128, "pages": pages,
            "layers_timed": w.n_layers, "kv_bytes_per_layer": per_layer,
            "ms_per_layer": round(ms / w.n_layers, 5),
            "kv_gbs": round(world * per_layer * w.n_layers / (ms * 1e-3) / 1e9, 1),
            "roofline": {"bound": "hbm", "kernel": "decode_kernel (paged: block-table tiles)",
                         "achieved": round(gbs, 1), "peak": hbm_peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
                         "launch_ms": round(dec_ms, 5)}}


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
        }
        results[name]["pct_hbm_measured"] = 100.0 * results[name]["decode_kernel_gbs"] / hbm_peak
        results[name]["pct_hbm_nominal_8tbs"] = 100.0 * results[name]["decode_kernel_gbs"] / NOMINAL_HBM_GBS
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

    hmode = run_hmode(args, world, device) if "hmode" in args.sections else None
    window = run_window(args, world, device) if "window" in args.sections else None
    paged = run_paged(args, world, device) if "paged" in args.sections else None
    if not variants:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": None, "hmode": hmode, "window": window,
                              "paged": paged}), flush=True)
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
        "config": {"workload": w.name, "kv": head, "batch": w.batch, "layers": w.n_layers,
                   "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                   "context": w.context, "scales": "fp16 per (token, head)",
                   "l2": "inputs larger than L2 (cache >= 4.4 GB per variant)",
                   "parallelism": f"replicas x{world}", "graph": "one CUDA graph per step",
                   "launch": "programmatic dependent launch between layers"},
        "pct_hbm_measured": round(r["pct_hbm_measured"], 2),
        "pct_hbm_nominal_8tbs": round(r["pct_hbm_nominal_8tbs"], 2),
        "roofline": {"bound": "hbm", "kernel": "decode_kernel (append + split-KV attention + merge)",
                     "achieved": round(r["decode_kernel_gbs"], 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(r["decode_kernel_gbs"] / hbm_peak, 4),
                     "traffic": args.traffic_bytes if args.traffic_bytes else decode_traffic(head),
                     "bytes_per_launch": r["kv_bytes_per_step"] // w.n_layers,
                     "launch_ms": round(r["decode_kernel_ms"], 5)},
        "variants": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv)
                         for kk, vv in v.items() if kk not in ("clocks", "e2e")}
                     for k, v in results.items()},
        "gpu_launches": args.steps * w.n_layers,   # one decode-step kernel per layer
        "hmode": hmode,
        "window": window,
        "paged": paged,
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
            "ms_per_step": round(t * 1e3 * w.n_layers, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "kv": head, "batch": w.batch, "layers": w.n_layers,
                       "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                       "head_dim": w.head_dim, "context": w.context},
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
    ap.add_argument("--sections", default="kv,hmode,window,paged",
                    help="kv: the 8K K/V decode step (headline); hmode: the h-mode workload; "
                         "window: the sliding-window workload; paged: the 8K step on a paged cache")
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
