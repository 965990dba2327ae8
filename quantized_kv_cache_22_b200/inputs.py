"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle runs.

This module holds no arithmetic of the method (no quantisation, no attention):
it only draws seeded random tensors with the shapes, dtypes and value
distributions of the workloads below, so that the CUDA path and the CPU oracle
can be fed the very same numbers.

The pages measure on trained models and text corpora (TinyStories, perplexity
sets, TinyLlama, Llama 3.2 3B, a 12M and a 407M model) that are not available
here; these synthetic tensors stand in for their KV activations, with the
cache shapes those pages imply.

Workloads (seed = 1000 + index):
  1 tiny      B=1, 1 layer, 4 heads (G=1), head_dim 64, fp32 q/k/v ~ N(0,1);
              INT8 per-(token,head); 4-token prompt then 252 append+attend steps
              (the mni-ml page's benchmark: 4-token prompt, 252 generated).
  2 int8kv    B=1, 34 layers, 16 heads x 128 (D=2048, G=1), capacity 1024
              filled, fp16 ~ N(0,1), K8V8 per-(token,head): 4160 B/token/layer
              (TinyLoop page, INT8 KV row).
  3 mixed     B=1, 28 layers, 24 query / 8 KV heads (G=3), head_dim 128,
              context 2048, fp16; K8V4 and K4V8 with INT4 group 32 and INT8
              per-(token,head); keys ~ N(0,1) with 4 of 128 channels per
              (layer, KV head), fixed across tokens, scaled x10 (outliers).
  4 long      B=16, 32 layers, 32 query / 8 KV heads (G=4), head_dim 128,
              context 8192 (8191 prefilled + 1 appended per step), fp16
              ~ N(0,1); K8V8, K8V4, K4V4 per-(token,head).
  5 h-mode    B=8, S=1024, D=2048, 16 heads x 128; residual ~ N(0,1),
              h = LayerNorm(residual) without affine, eps 1e-5; W_k, W_v bf16
              ~ N(0, 1/D); INT4-h with 16 fp16 scales per token.
  6 window    sliding-window cache (on-device page: 1536 recent tokens plus the
              first 64 as anchors; INT4 keys, INT8 values; 24 query / 8 KV
              heads x 128, 28 layers as the page's 3B model), B=64, 8192 tokens
              seen, so 1600 cached tokens per sequence; fp16 ~ N(0,1); keys INT4
              with 32-element groups, values INT8 per (token, head).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    batch: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int          # tokens attended per decode step
    capacity: int
    in_dtype: torch.dtype
    kv_variants: tuple = field(default_factory=tuple)  # ((k_bits, v_bits, k_group, v_group), ...)
    outliers: int = 0     # key channels per (layer, kv head) scaled by outlier_scale
    outlier_scale: float = 10.0
    d_model: int = 0      # h-mode
    window: int = 0       # sliding window (capacity = n_anchor + window)
    n_anchor: int = 0

    @property
    def seed(self) -> int:
        return 1000 + self.index


WORKLOADS = {
    1: Workload("tiny-int8-h4-d64", 1, 1, 1, 4, 4, 64, 256, 256, torch.float32,
                ((8, 8, 64, 64),)),
    2: Workload("int8kv-d2048-34L-1k", 2, 1, 34, 16, 16, 128, 1024, 1024, torch.float16,
                ((8, 8, 128, 128),)),
    3: Workload("mixed-gqa24x8-28L-2k", 3, 1, 28, 24, 8, 128, 2048, 2048, torch.float16,
                ((8, 4, 128, 32), (4, 8, 32, 128)), outliers=4),
    4: Workload("long-b16-gqa32x8-32L-8k", 4, 16, 32, 32, 8, 128, 8192, 8192, torch.float16,
                ((8, 8, 128, 128), (8, 4, 128, 128), (4, 4, 128, 128))),
    5: Workload("hmode-int4h-b8-s1k-d2048", 5, 8, 1, 16, 16, 128, 1024, 1024, torch.float16,
                (), d_model=2048),
    6: Workload("window-gqa24x8-b64-w1536a64-8k", 6, 64, 28, 24, 8, 128, 8192, 1600,
                torch.float16, ((4, 8, 32, 128),), window=1536, n_anchor=64),
}


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, device="cpu", dtype=torch.float16) -> torch.Tensor:
    """N(0,1) draws in fp32 from a seeded generator on `device`, cast to `dtype`."""
    g = generator(seed, device)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    return x.to(dtype)


def layer_seed(w: Workload, layer: int, stream: int) -> int:
    """Distinct seed per (workload, layer, stream); stream 0=K, 1=V, 2=Q, 3=outliers."""
    return w.seed * 1_000_003 + layer * 101 + stream


def kv_tokens(w: Workload, layer: int, n_tokens: int, device="cpu", offset_seed: int = 0):
    """Keys and values for `n_tokens` tokens: two tensors [B, n_tokens, Hkv, Dh]."""
    shape = (w.batch, n_tokens, w.n_kv_heads, w.head_dim)
    k = normal(shape, layer_seed(w, layer, 0) + 7919 * offset_seed, device, torch.float32)
    v = normal(shape, layer_seed(w, layer, 1) + 7919 * offset_seed, device, torch.float32)
    if w.outliers:
        g = generator(layer_seed(w, layer, 3), "cpu")
        mult = torch.ones(w.n_kv_heads, w.head_dim)
        for h in range(w.n_kv_heads):
            ch = torch.randperm(w.head_dim, generator=g)[: w.outliers]
            mult[h, ch] = w.outlier_scale
        k = k * mult.to(k.device)
    return k.to(w.in_dtype), v.to(w.in_dtype)


def queries(w: Workload, layer: int, step: int = 0, device="cpu") -> torch.Tensor:
    """Decode queries [B, Hq, Dh]."""
    shape = (w.batch, w.n_q_heads, w.head_dim)
    return normal(shape, layer_seed(w, layer, 2) + 7919 * step, device, w.in_dtype)


def hmode_inputs(w: Workload, n_tokens: int, device="cpu"):
    """h = LayerNorm(residual) [B, n_tokens, D] fp16 and W_kv bf16 [2*Hkv*Dh, D].

    The layer norm has no affine parameters and eps 1e-5 (the pages do not give
    them).  W_kv stacks W_k (rows 0..Hkv*Dh-1) over W_v, ~ N(0, 1/D).
    """
    D = w.d_model
    r = normal((w.batch, n_tokens, D), w.seed * 7 + 1, device, torch.float32)
    mu = r.mean(dim=-1, keepdim=True)
    var = r.var(dim=-1, unbiased=False, keepdim=True)
    h = ((r - mu) / torch.sqrt(var + 1e-5)).to(torch.float16)
    n_out = 2 * w.n_kv_heads * w.head_dim
    W = (normal((n_out, D), w.seed * 7 + 2, device, torch.float32) / math.sqrt(D)).to(torch.bfloat16)
    return h, W
