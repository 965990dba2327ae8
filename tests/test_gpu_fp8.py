"""GPU parity for the FP8 e4m3 cache format (the mni-ml page's comparison with
production stacks: vLLM and TensorRT-LLM keep FP8 KV caches).

Keys and values are one e4m3 byte per element with an fp16 scale per group,
s = fp16(absmax / 448) and code = e4m3(x / s) rounded to nearest even and
saturating at 448.  Codes and scales must match the oracle quantiser bit for
bit (every input dtype, every group size, outliers past the fp16 scale range,
all-zero groups); attention outputs must be within 2e-3 * max|V^| of the
oracle's fp64 attention over the dequantised cache.  Every call goes through
the C ABI.
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace
from _helpers import (assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache, oracle_decode,
                      read_gpu_cache, vmax_per_batch)
from test_gpu_kv import _sampled_full_size

pytestmark = pytest.mark.gpu

F8 = kvq.KVQ_FMT_E4M3
GROUPS = [(0, 0), (32, 32), (64, 128), (0, 32), (128, 64)]   # (k_group, v_group); 0: per head
CASES = [(kg, vg, dh) for dh in (64, 128) for kg, vg in GROUPS if max(kg, vg) <= dh]


def _cfg(B, cap, Hkv, G, dh, kg, vg, **kw):
    return Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                  k_bits=8, v_bits=8, k_group=kg, v_group=vg, kv_format=F8, **kw)


def _raw(B, L, Hkv, G, dh, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, L, Hkv, dh, generator=g)
    v = torch.randn(B, L, Hkv, dh, generator=g)
    q = torch.randn(B, Hkv * G, dh, generator=g)
    return k.to(dtype), v.to(dtype), q


def _compare_codes(cfg, cache, oc, lens):
    got = read_gpu_cache(cache, cfg)
    for i, name in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        for b, L in enumerate(lens):
            assert np.array_equal(got[i][b, :, :L], oc[i][b, :, :L]), (name, b)


@pytest.mark.parametrize("kg,vg,dh", CASES)
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32, torch.bfloat16])
def test_fp8_append_codes_bit_exact(cuda_device, kg, vg, dh, dtype):
    B, L, Hkv, cap = 2, 77, 3, 128
    k, v, _ = _raw(B, L, Hkv, 1, dh, dtype, 11 + dh + kg + vg)
    # outliers, tiny values (e4m3 subnormals after scaling) and an all-zero row
    k[0, 3, 1, 5] = 300.0
    v[1, 10, 2] = 0.0
    v[1, 11, 0, :8] = 1e-3
    if dtype != torch.float16:
        k[1, 20, 0, 7] = 1e8   # scale saturates to 65504, codes to 448
    cfg = _cfg(B, cap, Hkv, 1, dh, kg, vg)
    cache = gpu_cache(cfg, k, v)
    _compare_codes(cfg, cache, oracle_cache(k, v, cfg), [L] * B)


@pytest.mark.parametrize("kg,vg,dh", CASES)
@pytest.mark.parametrize("G", [1, 4, 8])
def test_fp8_decode_matches_oracle(cuda_device, kg, vg, dh, G):
    B, Hkv, cap = 4, 2, 320
    lens = [300, 1, 0, 129]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 5 + dh + G + kg + vg)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, kg, vg)
    cache = gpu_cache(cfg, k, v)
    got = gpu_decode(cfg, cache, q, lens)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    assert np.all(got[2] == 0)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, f"{kg},{vg}")


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("G", [1, 3, 4])
def test_fp8_decode_f32_bf16_queries(cuda_device, qdtype, G):
    """f32 / bf16 queries take an fp16 pair (value + residual) per head."""
    B, Hkv, dh, cap = 2, 2, 128, 256
    lens = [256, 77]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 40 + G)
    q = (q * 3).to(qdtype)
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 0)
    cache = gpu_cache(cfg, k, v)
    got = gpu_decode(cfg, cache, q, lens)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q.float(), lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, str(qdtype))


def test_fp8_f32_query_with_more_than_4_heads_per_group_is_rejected(cuda_device):
    B, Hkv, G, dh, cap = 1, 1, 8, 64, 128
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 0)
    cache = LayerCache(cfg)
    q = torch.zeros(B, G, dh, device="cuda")
    out = torch.empty(B, G, dh, device="cuda")
    with pytest.raises(RuntimeError):
        kvq.kvq_decode_attn(cfg, cache, q, torch.ones(1, dtype=torch.int32, device="cuda"), 1,
                            out, Workspace(cfg))


def test_fp8_stale_nan_codes_past_the_length_are_ignored(cuda_device):
    """Slots past a sequence's length may hold any byte, e4m3 NaN (0x7f) included,
    and any scale."""
    B, Hkv, G, dh, cap = 2, 1, 4, 128, 256
    lens = [130, 5]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 8)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 32)
    cache = gpu_cache(cfg, k, v)
    kc = cache.k_codes[: B * cap * dh].view(B, cap, dh)
    vc = cache.v_codes[: B * cap * dh].view(B, cap, dh)
    ks = cache.k_scales[: B * cap].view(B, cap)
    vs = cache.v_scales[: B * cap * (dh // 32)].view(B, cap, dh // 32)
    for b, L in enumerate(lens):
        kc[b, L:] = 0x7F
        vc[b, L:] = 0xFF
        ks[b, L:] = 65504.0
        vs[b, L:] = 65504.0
    got = gpu_decode(cfg, cache, q, lens)
    assert np.all(np.isfinite(got))
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, "stale")


def _fused_step(cfg, k, v, q, lens, seed):
    """Cache holds k/v everywhere except a decoy at each sequence's newest
    position; the fused call must overwrite it with the real newest token."""
    B = cfg.batch
    cache = gpu_cache(cfg, k, v)
    decoy = torch.randn(B, 1, cfg.n_kv_heads, cfg.head_dim,
                        generator=torch.Generator().manual_seed(seed)).to(k.dtype) * 5
    pos = torch.tensor([max(L - 1, 0) for L in lens], dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, decoy.cuda(), decoy.cuda(), pos, max(lens) - 1, 1)
    idx = torch.tensor([max(L - 1, 0) for L in lens])
    k_new = k[torch.arange(B), idx].contiguous()
    v_new = v[torch.arange(B), idx].contiguous()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, cfg.n_q_heads, cfg.head_dim), float("nan"), device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k_new.cuda(), v_new.cuda(), q.cuda(), d_len, max(lens),
                               out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    return cache, out.cpu().numpy()


@pytest.mark.parametrize("kg,vg", [(0, 0), (32, 64)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fp8_append_decode_step_matches_oracle(cuda_device, kg, vg, dtype):
    """One launch: quantise the newest token in FP8 and attend over the cache with it."""
    B, Hkv, G, dh, cap = 4, 2, 4, 128, 384
    lens = [384, 1, 200, 129]
    k, v, q = _raw(B, cap, Hkv, G, dh, dtype, 21 + kg + vg)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, kg, vg)
    cache, got = _fused_step(cfg, k, v, q, lens, 3)
    oc = oracle_cache(k, v, cfg)
    _compare_codes(cfg, cache, oc, lens)
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, f"{kg},{vg}")


def test_fp8_paged_matches_contiguous(cuda_device):
    """The paged FP8 cache gives the bits of the contiguous one."""
    B, Hkv, G, dh, cap, n_pages = 2, 2, 4, 128, 512, 9
    lens = [500, 130]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 31)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 0)
    pcfg = _cfg(B, cap, Hkv, G, dh, 0, 0, page_tokens=128, n_pages=n_pages)
    table = torch.tensor([[3, 0, 7, 5], [1, 8, 2, 6]], dtype=torch.int32, device="cuda")
    paged = LayerCache(pcfg, block_table=table)
    kvq.kvq_append(pcfg, paged, k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"),
                   0, cap)
    got = gpu_decode(pcfg, paged, q, lens)
    ref = gpu_decode(cfg, gpu_cache(cfg, k, v), q, lens)
    assert np.array_equal(got, ref)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, "paged")


def test_fp8_full_size_long_context_8k(cuda_device):
    """B=16, 32 query / 8 KV heads x 128, 8192 tokens, FP8 keys and values per
    (token, head): sampled (sequence, KV head) pairs against the oracle."""
    _sampled_full_size(4, (8, 8, 0, 0), 2, [(0, 0), (9, 4), (15, 7)], kv_format=F8)
