"""kvq_decode_attn_noalloc: decode attention without a caller-provided workspace.

Some callers of this library may not allocate device memory (a host framework
that owns every allocation, a real-time loop that forbids cudaMalloc after
start-up); this entry point keeps its split-KV partials in a fixed device array
inside libkvq instead.  These tests call it through the C ABI and check it
against the CPU oracle and against kvq_decode_attn with a regular workspace, on
two calls in a row (the array keeps the previous call's contents); they check
its size limit at and beyond the edge, that a timed-out call is visible through
kvq_noalloc_status and that the next call recovers, and a paged cache.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache
from _helpers import (TOL, assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache,
                      oracle_decode, vmax_per_batch)

pytestmark = pytest.mark.gpu

LIMIT = 8 * 1024 * 1024  # KVQ_NOALLOC_SCRATCH_BYTES
KVQ_ERR_TIMEOUT = -8
KVQ_ERR_WORKSPACE = -5


def _noalloc_fn():
    f = kvq.lib().kvq_decode_attn_noalloc
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [ctypes.POINTER(kvq.KvqConfig), ctypes.POINTER(kvq.KvqLayer), P, i32, P, i32,
                  ctypes.c_float, P, i32, i32, P]
    f.restype = ctypes.c_int
    return f


def _call(cfg, cache, q, d_len, max_len, out, num_ctas=0):
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.c_void_p(q.data_ptr()),
             kvq.KVQ_F16, ctypes.c_void_p(d_len.data_ptr()), max_len, ctypes.c_float(0.0),
             ctypes.c_void_p(out.data_ptr()), kvq.KVQ_F32, num_ctas, stream)


def _setup(B, Hkv, G, dh, cap, seed, fmt=(8, 4, 128, 32)):
    kb, vb, kg, vg = fmt
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                 k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half()
    return cfg, g, k, v


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    B, Hkv, G, dh, cap = 3, 2, 4, 128, 512
    cfg, g, k, v = _setup(B, Hkv, G, dh, cap, 91)
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
        assert kvq.kvq_noalloc_status() == 0
        got = out.cpu().numpy()
        vmax = vmax_per_batch(oc[2], oc[3], cfg, lens)
        err = np.abs(got - want).max(axis=(1, 2))
        assert np.all(err <= TOL * vmax), (call, err, TOL * vmax)
        # and against the CPU oracle directly
        assert_close_to_oracle(got, oracle_decode(cfg, oc, q, lens), vmax, G, f"call {call}")


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
    assert rc == KVQ_ERR_WORKSPACE   # nothing launched


def test_noalloc_at_the_edge_of_its_scratch(cuda_device):
    """An explicit CTA count whose workspace is just under the array's size runs and
    matches the workspace entry point with the same count (same partition, same
    bits) and the oracle; one CTA more per step past the limit is rejected."""
    B, Hkv, G, dh, cap = 3, 2, 4, 128, 1024
    cfg, g, k, v = _setup(B, Hkv, G, dh, cap, 93, fmt=(8, 8, 128, 128))
    n = 1
    while kvq.kvq_workspace_bytes(cfg, 2 * n) <= LIMIT:
        n *= 2
    lo, hi = n, 2 * n   # bytes(lo) <= LIMIT < bytes(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if kvq.kvq_workspace_bytes(cfg, mid) <= LIMIT else (lo, mid)
    assert LIMIT - kvq.kvq_workspace_bytes(cfg, lo) < 4096
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    lens = [1024, 1000, 3]
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hkv * G, dh), float("nan"), dtype=torch.float32, device="cuda")
    assert _call(cfg, cache, q.cuda(), d_len, max(lens), out, num_ctas=lo) == 0
    torch.cuda.synchronize()
    assert kvq.kvq_noalloc_status() == 0
    got = out.cpu().numpy()
    assert np.array_equal(got, gpu_decode(cfg, cache, q, lens, num_ctas=lo))
    assert_close_to_oracle(got, oracle_decode(cfg, oc, q, lens),
                           vmax_per_batch(oc[2], oc[3], cfg, lens), G, f"num_ctas={lo}")
    assert _call(cfg, cache, q.cuda(), d_len, max(lens), out, num_ctas=hi) == KVQ_ERR_WORKSPACE


def test_noalloc_timeout_is_reported_and_the_next_call_recovers(cuda_device):
    """The stalled-producer decode kernel on the library's array: every wait gives up,
    kvq_noalloc_status reads KVQ_ERR_TIMEOUT (and clears it); the next regular call
    clears the merge counters the timed-out call may have left and is correct."""
    B, Hkv, G, dh, cap = 3, 2, 4, 128, 384
    cfg, g, k, v = _setup(B, Hkv, G, dh, cap, 95)
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    lens = [384, 200, 0]
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hkv * G, dh), float("nan"), dtype=torch.float32, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    kvq.kvq_selftest_noalloc_timeout(cfg, cache, q.cuda(), d_len, out, 20_000_000)
    b.record()
    torch.cuda.synchronize()
    assert 18.0 <= a.elapsed_time(b) < 1000.0, a.elapsed_time(b)
    assert kvq.kvq_noalloc_status() == KVQ_ERR_TIMEOUT
    assert kvq.kvq_noalloc_status() == 0          # the read cleared it
    for call in range(2):
        out.fill_(float("nan"))
        kvq.kvq_decode_attn_noalloc(cfg, cache, q.cuda(), d_len, max(lens), out)
        torch.cuda.synchronize()
        assert kvq.kvq_noalloc_status() == 0
        assert_close_to_oracle(out.cpu().numpy(), oracle_decode(cfg, oc, q, lens),
                               vmax_per_batch(oc[2], oc[3], cfg, lens), G,
                               f"call {call} after a timeout")


def test_noalloc_paged_cache(cuda_device):
    """A paged cache (128-token pages behind a shuffled block table) through the
    noalloc entry point equals the workspace entry point bit for bit and the oracle."""
    lens = [1000, 129, 513]
    B, Hkv, G, dh, cap, n_pages = len(lens), 2, 4, 128, 1024, 30
    base = dict(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                k_bits=4, v_bits=4, k_group=32, v_group=32)
    cfg = Config(**base, page_tokens=128, n_pages=n_pages)
    g = torch.Generator().manual_seed(97)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half()
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    table = torch.randperm(n_pages, generator=g)[: B * (cap // 128)].view(B, -1).to(torch.int32)
    cache = LayerCache(cfg, block_table=table.cuda())
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    n = max(lens)
    kvq.kvq_append(cfg, cache, k[:, :n].contiguous().cuda(), v[:, :n].contiguous().cuda(), pos, 0, n)
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hkv * G, dh), float("nan"), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attn_noalloc(cfg, cache, q.cuda(), d_len, max(lens), out)
    torch.cuda.synchronize()
    assert kvq.kvq_noalloc_status() == 0
    got = out.cpu().numpy()
    assert np.array_equal(got, gpu_decode(cfg, cache, q, lens))
    flat = Config(**base)
    oc = oracle_cache(k, v, flat)
    assert_close_to_oracle(got, oracle_decode(flat, oc, q, lens),
                           vmax_per_batch(oc[2], oc[3], flat, lens), G, "paged")
