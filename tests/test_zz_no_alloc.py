"""kvq_decode_attn_noalloc: decode attention without a caller-provided workspace.

Some callers of this library may not allocate device memory (a host framework
that owns every allocation, a real-time loop that forbids cudaMalloc after
start-up); this entry point keeps its split-KV partials in a fixed device array
inside libkvq instead.  These tests call it through the C ABI and check it
against kvq_decode_attn with a regular workspace, on two calls in a row (the
array keeps the previous call's contents), and check its size limit.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config
from _helpers import TOL, gpu_cache, gpu_decode, oracle_cache, vmax_per_batch

pytestmark = pytest.mark.gpu

LIMIT = 8 * 1024 * 1024  # KVQ_NOALLOC_SCRATCH_BYTES


def _noalloc_fn():
    f = kvq.lib().kvq_decode_attn_noalloc
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [ctypes.POINTER(kvq.KvqConfig), ctypes.POINTER(kvq.KvqLayer), P, i32, P, i32,
                  ctypes.c_float, P, i32, i32, P]
    f.restype = ctypes.c_int
    return f


def _call(cfg, cache, q, d_len, max_len, out):
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.c_void_p(q.data_ptr()),
             kvq.KVQ_F16, ctypes.c_void_p(d_len.data_ptr()), max_len, ctypes.c_float(0.0),
             ctypes.c_void_p(out.data_ptr()), kvq.KVQ_F32, 0, stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    B, Hkv, G, dh, cap = 3, 2, 4, 128, 512
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                 k_bits=8, v_bits=4, k_group=128, v_group=32)
    g = torch.Generator().manual_seed(91)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half()
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    for call, lens in enumerate(([512, 77, 300], [129, 512, 1])):
        q = torch.randn(B, Hkv * G, dh, generator=g).half()
        want = gpu_decode(cfg, cache, q, lens)          # kvq_decode_attn, own workspace
        d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
        qd = q.cuda()
        out = torch.full((B, Hkv * G, dh), float("nan"), dtype=torch.float32, device="cuda")
        rc = _call(cfg, cache, qd, d_len, max(lens), out)
        assert rc == 0, kvq.status_string(rc)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        vmax = vmax_per_batch(oc[2], oc[3], cfg, lens)
        err = np.abs(got - want).max(axis=(1, 2))
        assert np.all(err <= TOL * vmax), (call, err, TOL * vmax)


def test_noalloc_rejects_configs_beyond_its_scratch(cuda_device):
    # B*Hkv = 4096 sequences x heads needs far more than 8 MiB of partials
    B, Hkv, G, dh, cap = 512, 8, 8, 128, 64
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh)
    assert kvq.kvq_workspace_bytes(cfg) > LIMIT
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    layer = kvq.KvqLayer(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr())
    f = _noalloc_fn()
    rc = f(ctypes.byref(cfg.c()), ctypes.byref(layer), ctypes.c_void_p(dummy.data_ptr()),
           kvq.KVQ_F16, ctypes.c_void_p(dummy.data_ptr()), 1, ctypes.c_float(0.0),
           ctypes.c_void_p(dummy.data_ptr()), kvq.KVQ_F32, 0,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -5   # KVQ_ERR_WORKSPACE, nothing launched
