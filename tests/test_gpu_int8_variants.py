"""GPU parity for the two other INT8 cache formats of the mni-ml page ("Tại sao INT8
mà không mất tốc": scale/zero-point metadata; "Limitations": symmetric per-tensor
scaling).

Asymmetric (KVQ_FMT_ASYM): per group lo = min(0, min x), hi = max(0, max x),
s = fp16((hi - lo)/255), z = clamp(rne(-lo/s), 0, 255), code = clamp(rne(x/s) + z,
0, 255) as a uint8 with the pair (s, z) per group.  Per-tensor (KVQ_FMT_TENSOR): one
caller-set fp16 scale per K / V tensor, code = clamp(rne(x/s), -127, 127).

Codes, scales and zero-points must match the oracle bit for bit; attention outputs
must be within 2e-3 * max|V^| of the oracle.  Every call goes through the C ABI.
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

ASYM, TENSOR = kvq.KVQ_FMT_ASYM, kvq.KVQ_FMT_TENSOR
GROUPS = [(0, 0), (32, 32), (64, 128), (0, 32), (128, 64)]   # (k_group, v_group); 0: per head
CASES = [(kg, vg, dh) for dh in (64, 128) for kg, vg in GROUPS if max(kg, vg) <= dh]


def _cfg(B, cap, Hkv, G, dh, kg, vg, fmt, **kw):
    return Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                  k_bits=8, v_bits=8, k_group=kg, v_group=vg, kv_format=fmt, **kw)


def _raw(B, L, Hkv, G, dh, dtype, seed, offset=0.0):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, L, Hkv, dh, generator=g) + offset
    v = torch.randn(B, L, Hkv, dh, generator=g) - offset
    q = torch.randn(B, Hkv * G, dh, generator=g)
    return k.to(dtype), v.to(dtype), q


def _compare_codes(cfg, cache, oc, lens):
    got = read_gpu_cache(cache, cfg)
    for i, name in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        for b, L in enumerate(lens):
            assert np.array_equal(got[i][b, :, :L], oc[i][b, :, :L]), (name, b)


def _tensor_s16(x, margin=1.0):
    """A per-tensor scale as a caller would set it: fp16(max|x| * margin / 127)."""
    return int(np.float16(float(x.float().abs().max()) * margin / 127).view(np.uint16))


def _tensor_cache(cfg, k, v, sk, sv, block_table=None):
    cache = LayerCache(cfg, block_table=block_table)
    cache.k_scales.view(torch.int16)[0] = np.int16(np.uint16(sk).view(np.int16))
    cache.v_scales.view(torch.int16)[0] = np.int16(np.uint16(sv).view(np.int16))
    B, L = k.shape[0], k.shape[1]
    kvq.kvq_append(cfg, cache, k.cuda().contiguous(), v.cuda().contiguous(),
                   torch.zeros(B, dtype=torch.int32, device="cuda"), 0, L)
    return cache


# --- asymmetric ----------------------------------------------------------------------

@pytest.mark.parametrize("kg,vg,dh", CASES)
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32, torch.bfloat16])
def test_asym_append_codes_bit_exact(cuda_device, kg, vg, dh, dtype):
    B, L, Hkv, cap = 2, 77, 3, 128
    k, v, _ = _raw(B, L, Hkv, 1, dh, dtype, 13 + dh + kg + vg, offset=1.5)
    k[0, 4] = k[0, 4].abs() + 0.1      # all-positive rows: zero-point 0
    v[1, 6] = -v[1, 6].abs() - 0.1     # all-negative rows: zero-point 255
    v[1, 7] = 0.0
    k[1, 9, 2, 3] = 250.0
    cfg = _cfg(B, cap, Hkv, 1, dh, kg, vg, ASYM)
    cache = gpu_cache(cfg, k, v)
    _compare_codes(cfg, cache, oracle_cache(k, v, cfg), [L] * B)


@pytest.mark.parametrize("kg,vg,dh", CASES)
@pytest.mark.parametrize("G", [1, 4, 8])
def test_asym_decode_matches_oracle(cuda_device, kg, vg, dh, G):
    B, Hkv, cap = 4, 2, 320
    lens = [300, 1, 0, 129]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 9 + dh + G + kg + vg, offset=0.7)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, kg, vg, ASYM)
    cache = gpu_cache(cfg, k, v)
    got = gpu_decode(cfg, cache, q, lens)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    assert np.all(got[2] == 0)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, f"{kg},{vg}")


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
def test_asym_decode_f32_bf16_queries(cuda_device, qdtype):
    B, Hkv, G, dh, cap = 2, 2, 8, 128, 256
    lens = [256, 77]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 50, offset=-2.0)
    q = (q * 3).to(qdtype)
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 64, ASYM)
    cache = gpu_cache(cfg, k, v)
    got = gpu_decode(cfg, cache, q, lens)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q.float(), lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, str(qdtype))


@pytest.mark.parametrize("vg", [0, 32])
def test_asym_stale_scales_and_zero_points_past_the_length(cuda_device, vg):
    """Scale and zero-point slots past a sequence's length may hold NaN or inf."""
    B, Hkv, G, dh, cap = 2, 1, 4, 128, 256
    lens = [131, 6]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 18, offset=0.3)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, 0, vg, ASYM)
    cache = gpu_cache(cfg, k, v)
    nv = 2 * (dh // (vg or dh))
    ks = cache.k_scales[: B * cap * 2].view(B, cap, 2)
    vs = cache.v_scales[: B * cap * nv].view(B, cap, nv)
    for b, L in enumerate(lens):
        ks[b, L:] = float("nan")
        vs[b, L:, 0::2] = float("inf")
        vs[b, L:, 1::2] = float("nan")
    got = gpu_decode(cfg, cache, q, lens)
    assert np.all(np.isfinite(got))
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, "stale")


def test_asym_append_decode_step_and_paged(cuda_device):
    """The fused step writes the newest token's codes and (s, z); the paged cache
    gives the bits of the contiguous one."""
    B, Hkv, G, dh, cap, n_pages = 2, 2, 4, 128, 384, 7
    lens = [384, 200]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.bfloat16, 23, offset=1.0)
    q = q.half()
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 32, ASYM)
    cache = gpu_cache(cfg, k, v)
    decoy = (torch.randn(B, 1, Hkv, dh, generator=torch.Generator().manual_seed(2)) * 4).to(k.dtype)
    kvq.kvq_append(cfg, cache, decoy.cuda(), decoy.cuda(),
                   torch.tensor([L - 1 for L in lens], dtype=torch.int32, device="cuda"),
                   max(lens) - 1, 1)
    idx = torch.tensor([L - 1 for L in lens])
    out = torch.empty(B, Hkv * G, dh, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k[torch.arange(B), idx].cuda().contiguous(),
                               v[torch.arange(B), idx].cuda().contiguous(), q.cuda(),
                               torch.tensor(lens, dtype=torch.int32, device="cuda"), max(lens),
                               out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    oc = oracle_cache(k, v, cfg)
    _compare_codes(cfg, cache, oc, lens)
    got = out.cpu().numpy()
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, "fused")
    pcfg = _cfg(B, cap, Hkv, G, dh, 0, 32, ASYM, page_tokens=128, n_pages=n_pages)
    table = torch.tensor([[4, 0, 6], [1, 5, 2]], dtype=torch.int32, device="cuda")
    paged = LayerCache(pcfg, block_table=table)
    kvq.kvq_append(pcfg, paged, k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"),
                   0, cap)
    assert np.array_equal(gpu_decode(pcfg, paged, q, lens), gpu_decode(cfg, gpu_cache(cfg, k, v), q, lens))


def test_asym_full_size_long_context_8k(cuda_device):
    """B=16, 32 query / 8 KV heads x 128, 8192 tokens, asymmetric INT8 per (token,
    head): sampled (sequence, KV head) pairs against the oracle."""
    _sampled_full_size(4, (8, 8, 0, 0), 3, [(0, 0), (6, 2), (15, 7)], kv_format=ASYM)


# --- per-tensor ----------------------------------------------------------------------

@pytest.mark.parametrize("dh", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32, torch.bfloat16])
@pytest.mark.parametrize("margin", [1.0, 0.5])   # 0.5: the scale clips the largest values
def test_tensor_append_and_decode_match_oracle(cuda_device, dh, dtype, margin):
    B, Hkv, G, cap = 3, 2, 4, 256
    lens = [256, 0, 70]
    k, v, q = _raw(B, cap, Hkv, G, dh, dtype, 31 + dh, offset=0.2)
    q = q.half()
    sk, sv = _tensor_s16(k, margin), _tensor_s16(v, margin)
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 0, TENSOR)
    cache = _tensor_cache(cfg, k, v, sk, sv)
    # the library reads the tensor scales and never writes them
    assert int(cache.k_scales.view(torch.int16)[0]) & 0xFFFF == sk
    assert int(cache.v_scales.view(torch.int16)[0]) & 0xFFFF == sv
    oc = oracle_cache(k, v, cfg, tensor_s16=(sk, sv))
    _compare_codes(cfg, cache, oc, [cap] * B)
    got = gpu_decode(cfg, cache, q, lens)
    want = oracle_decode(cfg, oc, q, lens)
    assert np.all(got[1] == 0)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, f"{margin}")


def test_tensor_append_decode_step(cuda_device):
    B, Hkv, G, dh, cap = 2, 2, 4, 128, 384
    lens = [384, 129]
    k, v, q = _raw(B, cap, Hkv, G, dh, torch.float16, 40)
    q = q.half()
    sk, sv = _tensor_s16(k), _tensor_s16(v)
    cfg = _cfg(B, cap, Hkv, G, dh, 0, 0, TENSOR)
    decoy_k = k.clone()
    decoy_k[torch.arange(B), torch.tensor([L - 1 for L in lens])] = 3.0
    cache = _tensor_cache(cfg, decoy_k, decoy_k, sk, sv)
    idx = torch.tensor([L - 1 for L in lens])
    # the cache holds decoy_k as keys and values; the fused step replaces the newest token
    kk = decoy_k.clone()
    vv = decoy_k.clone()
    kk[torch.arange(B), idx] = k[torch.arange(B), idx]
    vv[torch.arange(B), idx] = v[torch.arange(B), idx]
    out = torch.empty(B, Hkv * G, dh, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k[torch.arange(B), idx].cuda().contiguous(),
                               v[torch.arange(B), idx].cuda().contiguous(), q.cuda(),
                               torch.tensor(lens, dtype=torch.int32, device="cuda"), max(lens),
                               out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    oc = oracle_cache(kk, vv, cfg, tensor_s16=(sk, sv))
    _compare_codes(cfg, cache, oc, lens)
    want = oracle_decode(cfg, oc, q, lens)
    assert_close_to_oracle(out.cpu().numpy(), want, vmax_per_batch(oc[2], oc[3], cfg, lens), G,
                           "fused")


def test_tensor_full_size_long_context_8k(cuda_device):
    """B=16, 32 query / 8 KV heads x 128, 8192 tokens, per-tensor INT8 with the scale
    a caller calibrates from the whole tensor: sampled pairs against the oracle."""
    from quantized_kv_cache_22_b200 import inputs
    w = inputs.WORKLOADS[4]
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=8, v_bits=8,
                 kv_format=TENSOR)
    L = w.context
    k, v = inputs.kv_tokens(w, 5, L, "cuda")
    sk, sv = _tensor_s16(k), _tensor_s16(v)
    cache = _tensor_cache(cfg, k, v, sk, sv)
    q = inputs.queries(w, 5, 0, "cuda")
    got = gpu_decode(cfg, cache, q, [L] * w.batch)
    gc = read_gpu_cache(cache, cfg)
    G = w.n_q_heads // w.n_kv_heads
    for (b, kvh) in ((0, 0), (8, 5), (15, 7)):
        sub = Config(**{**cfg.__dict__, "batch": 1, "n_kv_heads": 1, "n_q_heads": G})
        oc = oracle_cache(k[b:b + 1, :, kvh:kvh + 1].cpu(), v[b:b + 1, :, kvh:kvh + 1].cpu(), sub,
                          tensor_s16=(sk, sv))
        assert np.array_equal(gc[0][b, kvh], oc[0][0, 0]) and np.array_equal(gc[2][b, kvh], oc[2][0, 0])
        want = oracle_decode(sub, oc, q[b:b + 1, kvh * G:(kvh + 1) * G].cpu(), [L])
        vmax = vmax_per_batch(oc[2], oc[3], sub, [L])
        assert_close_to_oracle(got[b:b + 1, kvh * G:(kvh + 1) * G], want, vmax, G, f"{(b, kvh)}")
