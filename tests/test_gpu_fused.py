"""GPU parity for the one-launch decode step and the merge paths.

kvq_append_decode_attn quantises each sequence's newest token into the cache and
attends over the cache that includes it, in one launch: its codes must match the
oracle quantiser bit for bit and its outputs the oracle within 2e-3 * max|V^|.
The in-kernel merge (arrival counters in the workspace) must give the same bits
as the separate partials + merge launches, and a workspace must stay usable
from one call to the next.  Every call goes through the C ABI.
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs
from _helpers import (assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache, oracle_decode,
                      read_gpu_cache, vmax_per_batch)

pytestmark = pytest.mark.gpu


def _cfg(B, cap, Hkv, G, dh, fmt):
    kb, vb, kg, vg = fmt
    return Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                  k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)


def _raw(B, L, Hkv, G, dh, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, L, Hkv, dh, generator=g).to(dtype)
    v = torch.randn(B, L, Hkv, dh, generator=g).to(dtype)
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    return k, v, q


def _fused_step(cfg, k, v, q, lens, seed, out_dtype=torch.float32):
    """Cache holds k/v everywhere except a decoy at each sequence's newest
    position; the fused call must overwrite it with the real newest token."""
    B, cap = cfg.batch, cfg.capacity
    cache = gpu_cache(cfg, k, v)
    decoy = torch.randn(B, 1, cfg.n_kv_heads, cfg.head_dim,
                        generator=torch.Generator().manual_seed(seed)).to(k.dtype) * 5
    pos = torch.tensor([L - 1 for L in lens], dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, decoy.cuda(), decoy.cuda(), pos, max(lens) - 1, 1)
    idx = torch.tensor([max(L - 1, 0) for L in lens])
    k_new = k[torch.arange(B), idx].contiguous()            # [B, Hkv, dh]
    v_new = v[torch.arange(B), idx].contiguous()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, cfg.n_q_heads, cfg.head_dim), float("nan"), dtype=out_dtype, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k_new.cuda(), v_new.cuda(), q.cuda(), d_len, max(lens),
                               out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    return cache, out.float().cpu().numpy()


@pytest.mark.parametrize("fmt", [(8, 8, 0, 0), (8, 4, 0, 32), (4, 4, 32, 32), (4, 8, 0, 64),
                                 (16, 16, 0, 0), (8, 16, 0, 0), (16, 4, 0, 0)])
@pytest.mark.parametrize("dh", [64, 128])
def test_append_decode_attn_matches_oracle(cuda_device, fmt, dh):
    B, Hkv, G, cap = 4, 2, 4, 320
    lens = [300, 1, 0, 129]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 7 + dh + fmt[0] + fmt[1])
    cfg = _cfg(B, cap, Hkv, G, dh, fmt)
    cache, got = _fused_step(cfg, k, v, q, lens, 99)
    oc = oracle_cache(k, v, cfg)
    gc = read_gpu_cache(cache, cfg)
    for i, name in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        if oc[i] is None:
            continue
        for b, L in enumerate(lens):
            assert np.array_equal(gc[i][b, :, :L], oc[i][b, :, :L]), (name, b)
    want = oracle_decode(cfg, oc, q, lens)
    assert np.all(got[2] == 0)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, str(fmt))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_append_decode_attn_input_dtypes(cuda_device, dtype):
    B, Hkv, G, dh, cap = 2, 3, 2, 128, 256
    lens = [256, 77]
    k, v, q = _raw(B, cap, Hkv, G, dh, dtype, 61)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 4, 0, 32))
    cache, got = _fused_step(cfg, k, v, q, lens, 62, out_dtype=torch.float16)
    oc = oracle_cache(k, v, cfg)
    gc = read_gpu_cache(cache, cfg)
    for i in range(4):
        for b, L in enumerate(lens):
            assert np.array_equal(gc[i][b, :, :L], oc[i][b, :, :L]), (i, b)
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, str(dtype))


def test_fused_tiny_workload_prompt_then_252_steps(cuda_device):
    """The mni-ml benchmark shape (4-token prompt, 252 generated tokens) with every
    step a single append+attend launch, checked against the oracle each step."""
    w = inputs.WORKLOADS[1]
    cfg = Config(batch=1, capacity=w.capacity, n_q_heads=4, n_kv_heads=4, head_dim=64,
                 k_bits=8, v_bits=8, k_group=64, v_group=64)
    k, v = inputs.kv_tokens(w, 0, 256)
    cache = LayerCache(cfg)
    ws = Workspace(cfg)
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, k[:, :4].cuda().contiguous(), v[:, :4].cuda().contiguous(), pos, 0, 4)
    oc = oracle_cache(k, v, cfg)
    d_len = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(1, 4, 64, dtype=torch.float32, device="cuda")
    for step in range(252):
        L = 5 + step
        d_len.fill_(L)
        q = inputs.queries(w, 0, step)
        kvq.kvq_append_decode_attn(cfg, cache, k[:, L - 1].cuda().contiguous(),
                                   v[:, L - 1].cuda().contiguous(), q.cuda(), d_len, L, out, ws)
        want = oracle_decode(cfg, oc, q, [L])
        vmax = vmax_per_batch(oc[2], oc[3], cfg, [L])
        assert_close_to_oracle(out.cpu().numpy(), want, vmax, 1, f"step {step}")
    gc = read_gpu_cache(cache, cfg)
    for i in range(4):
        assert np.array_equal(gc[i][:, :, :256], oc[i][:, :, :256]), i
    assert kvq.kvq_workspace_status(ws) == 0


@pytest.mark.parametrize("num_ctas", [0, 3, 40])
def test_partials_then_merge_equal_one_launch(cuda_device, num_ctas):
    B, Hkv, G, dh, cap = 3, 2, 4, 128, 1024
    lens = [1000, 5, 513]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 71)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 8, 0, 0))
    cache = gpu_cache(cfg, k, v)
    fused = gpu_decode(cfg, cache, q, lens, num_ctas=num_ctas)
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = Workspace(cfg, num_ctas)
    out = torch.empty(B, Hkv * G, dh, dtype=torch.float32, device="cuda")
    kvq.kvq_decode_partials(cfg, cache, q.cuda(), d_len, max(lens), ws, num_ctas=num_ctas)
    kvq.kvq_merge_partials(cfg, d_len, out, ws, num_ctas=num_ctas)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    # the same partials merged in the same order: identical bits
    assert np.array_equal(out.cpu().numpy(), fused)


def test_workspace_reused_across_calls(cuda_device):
    B, Hkv, G, dh, cap = 2, 4, 2, 128, 640
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 81)
    cfg = _cfg(B, cap, Hkv, G, dh, (4, 4, 0, 0))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    ws = Workspace(cfg)
    out = torch.empty(B, Hkv * G, dh, dtype=torch.float32, device="cuda")
    for lens in ([640, 300], [1, 639], [0, 128], [640, 640]):
        d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
        kvq.kvq_decode_attn(cfg, cache, q.cuda(), d_len, max(lens), out, ws)
        want = oracle_decode(cfg, oc, q, lens)
        assert_close_to_oracle(out.cpu().numpy(), want, vmax_per_batch(oc[2], oc[3], cfg, lens),
                               G, str(lens))
    assert kvq.kvq_workspace_status(ws) == 0


def test_many_ctas_per_sequence_head(cuda_device):
    # one (sequence, KV head) pair spread over many CTAs: tens of partials merged
    B, Hkv, G, dh, cap = 1, 1, 8, 128, 8192
    lens = [8192]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 91)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 4, 0, 0))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    vmax = vmax_per_batch(oc[2], oc[3], cfg, lens)
    for n in (0, 64, 200):
        got = gpu_decode(cfg, cache, q, lens, num_ctas=n)
        assert_close_to_oracle(got, want, vmax, G, f"num_ctas={n}")
