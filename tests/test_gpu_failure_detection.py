"""Failure detection without a GPU fault: every wait in the library's kernels is a
bounded mbarrier wait that, after its limit, records KVQ_ERR_TIMEOUT in the workspace
status word and returns.  kvq_selftest_bounded_wait runs that wait on a barrier that
nothing completes (a flag nobody sets); the status must read KVQ_ERR_TIMEOUT after
about the limit, and the context and the workspace must stay usable."""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, Workspace
from _helpers import assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache, oracle_decode, vmax_per_batch

pytestmark = pytest.mark.gpu

KVQ_ERR_TIMEOUT = -8


def test_bounded_wait_gives_up_and_the_context_stays_usable(cuda_device):
    B, Hkv, G, dh, cap = 2, 2, 4, 128, 256
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                 k_bits=8, v_bits=8)
    ws = Workspace(cfg)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    kvq.kvq_selftest_bounded_wait(ws, 20_000_000)            # 20 ms
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    assert 18.0 <= ms < 1000.0, ms
    assert kvq.kvq_workspace_status(ws) == KVQ_ERR_TIMEOUT
    assert kvq.kvq_workspace_status(ws) == 0                 # read clears it
    # the same context decodes correctly afterwards
    g = torch.Generator().manual_seed(5)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half()
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    lens = [256, 100]
    got = gpu_decode(cfg, gpu_cache(cfg, k, v), q, lens)
    oc = oracle_cache(k, v, cfg)
    assert_close_to_oracle(got, oracle_decode(cfg, oc, q, lens),
                           vmax_per_batch(oc[2], oc[3], cfg, lens), G, "after a timeout")


def test_decode_kernel_wait_runs_out_and_reports_timeout(cuda_device):
    """The decode kernel with a producer that copies nothing: every consumer's wait for
    its first tile runs out after the limit, the kernel reports KVQ_ERR_TIMEOUT and
    returns; after zero-filling the workspace the same context decodes correctly."""
    B, Hkv, G, dh, cap = 3, 2, 4, 128, 384
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                 k_bits=8, v_bits=4, k_group=128, v_group=32)
    g = torch.Generator().manual_seed(9)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half()
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    lens = [384, 200, 0]
    cache = gpu_cache(cfg, k, v)
    ws = Workspace(cfg)
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hkv * G, dh), float("nan"), device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    kvq.kvq_selftest_decode_timeout(cfg, cache, q.cuda(), d_len, out, ws, 20_000_000)
    b.record()
    torch.cuda.synchronize()
    assert 18.0 <= a.elapsed_time(b) < 1000.0, a.elapsed_time(b)
    assert kvq.kvq_workspace_status(ws) == KVQ_ERR_TIMEOUT
    ws.buf.zero_()
    got = gpu_decode(cfg, cache, q, lens)
    oc = oracle_cache(k, v, cfg)
    assert_close_to_oracle(got, oracle_decode(cfg, oc, q, lens),
                           vmax_per_batch(oc[2], oc[3], cfg, lens), G, "after a decode timeout")
    # and the workspace itself is usable again
    kvq.kvq_decode_attn(cfg, cache, q.cuda(), d_len, max(lens), out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    assert np.array_equal(out.cpu().numpy(), got)
