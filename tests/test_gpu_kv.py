"""GPU parity: quantize-on-append and split-KV decode attention vs the CPU oracle.

Codes and scales must match the oracle bit for bit; attention outputs must be
within 2e-3 * max|V^| (fp32 accumulation).  Every call goes through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace
from quantized_kv_cache_22_b200 import inputs
from _helpers import (assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache, oracle_decode,
                      read_gpu_cache, to_np32, vmax_per_batch)

pytestmark = pytest.mark.gpu

FORMATS = [  # (k_bits, v_bits, k_group, v_group)
    (8, 8, 0, 0), (8, 4, 0, 32), (4, 8, 32, 0), (4, 4, 0, 0), (4, 4, 32, 32), (8, 8, 32, 64),
    (16, 16, 0, 0), (8, 16, 0, 0), (16, 4, 0, 32), (8, 8, 64, 64), (4, 8, 64, 0)]


def _inputs(B, L, Hkv, G, dh, dtype, seed, scale_v=1.0):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, L, Hkv, dh, generator=g).to(dtype)
    v = (torch.randn(B, L, Hkv, dh, generator=g) * scale_v).to(dtype)
    q = torch.randn(B, Hkv * G, dh, generator=g).to(dtype)
    return k, v, q


def _cfg(B, cap, Hkv, G, dh, fmt):
    kb, vb, kg, vg = fmt
    return Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                  k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)


def _compare_codes(cfg, cache, oc, L):
    got = read_gpu_cache(cache, cfg)
    for g, w, name in zip(got, oc, ("k_codes", "k_scales", "v_codes", "v_scales")):
        if w is None:
            continue
        assert np.array_equal(g[:, :, :L], w[:, :, :L]), name


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("dh", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32, torch.bfloat16])
def test_append_codes_bit_exact(cuda_device, fmt, dh, dtype):
    B, L, Hkv, cap = 2, 77, 3, 128
    k, v, _ = _inputs(B, L, Hkv, 1, dh, dtype, 1 + dh + fmt[0] * 3 + fmt[1])
    cfg = _cfg(B, cap, Hkv, 1, dh, fmt)
    cache = gpu_cache(cfg, k, v)
    _compare_codes(cfg, cache, oracle_cache(k, v, cfg), L)


def test_append_at_positions_and_skip_out_of_range(cuda_device):
    B, Hkv, dh, cap = 3, 2, 128, 64
    cfg = _cfg(B, cap, Hkv, 1, dh, (8, 4, 0, 32))
    k, v, _ = _inputs(B, 40, Hkv, 1, dh, torch.float16, 5)
    cache = gpu_cache(cfg, k, v)
    k2, v2, _ = _inputs(B, 3, Hkv, 1, dh, torch.float16, 6)
    before = read_gpu_cache(cache, cfg)
    # device positions 40, 10 and 62: the last sequence's third token (position 64) is skipped
    pos = torch.tensor([40, 10, 62], dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, k2.cuda(), v2.cuda(), pos, 61, 3)
    torch.cuda.synchronize()
    after = read_gpu_cache(cache, cfg)
    o2 = oracle_cache(k2, v2, Config(**{**cfg.__dict__, "capacity": 16}))
    for b, p in enumerate([40, 10, 62]):
        n = min(3, cap - p)
        for i in range(4):
            if after[i] is None:
                continue
            assert np.array_equal(after[i][b, :, p:p + n], o2[i][b, :, :n])
            # rows outside the written range are untouched
            mask = np.ones(cap, bool)
            mask[p:p + n] = False
            assert np.array_equal(after[i][b, :, mask], before[i][b, :, mask])


def test_append_rejects_capacity_overflow(cuda_device):
    cfg = _cfg(1, 32, 1, 1, 128, (8, 8, 0, 0))
    cache = LayerCache(cfg)
    k = torch.zeros(1, 4, 1, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append(cfg, cache, k, k, torch.zeros(1, dtype=torch.int32, device="cuda"), 30, 4)
    assert e.value.status == -3


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("dh,G", [(128, 4), (128, 1), (64, 3), (128, 8)])
def test_decode_matches_oracle(cuda_device, fmt, dh, G):
    B, Hkv, cap = 3, 2, 320
    lens = [300, 1, 129]
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 11 + G + dh)
    cfg = _cfg(B, cap, Hkv, G, dh, fmt)
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    _compare_codes(cfg, cache, oc, cap)
    want = oracle_decode(cfg, oc, q, lens)
    vmax = vmax_per_batch(oc[2], oc[3], cfg, lens)
    got = gpu_decode(cfg, cache, q, lens)
    assert_close_to_oracle(got, want, vmax, G, f"fmt={fmt} dh={dh} G={G}")
    got16 = gpu_decode(cfg, cache, q, lens, out_dtype=torch.float16)
    assert_close_to_oracle(got16, want, vmax, G, "fp16 out")


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("G", [1, 4])
def test_decode_f32_bf16_queries(cuda_device, qdtype, G):
    B, Hkv, dh, cap = 2, 2, 128, 192
    lens = [192, 70]
    k, v, _ = _inputs(B, cap, Hkv, G, dh, torch.float16, 21)
    q = torch.randn(B, Hkv * G, dh, generator=torch.Generator().manual_seed(22)).to(qdtype) * 3
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 8, 0, 0))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    got = gpu_decode(cfg, cache, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, str(qdtype))


def test_decode_split_count_invariance(cuda_device):
    B, Hkv, G, dh, cap = 2, 2, 4, 128, 1024
    lens = [1024, 700]
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 31)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 4, 0, 32))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    vmax = vmax_per_batch(oc[2], oc[3], cfg, lens)
    outs = []
    for n in (1, 2, 7, 19, 64, 0):
        got = gpu_decode(cfg, cache, q, lens, num_ctas=n)
        assert_close_to_oracle(got, want, vmax, G, f"num_ctas={n}")
        outs.append(got)
    # p * s_V enters the MMA rounded to fp16 relative to the running max, and the
    # running max depends on where the split boundaries fall: outputs of different
    # split counts agree to fp16 rounding of the weights, 2^-11 * max|V^|.
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2.0 ** -11 * vmax.max()


@pytest.mark.parametrize("B", [256, 257])
def test_decode_batch_at_and_past_early_range_limit(cuda_device, B):
    """Up to 256 sequences the kernel finds its work range from lengths it reads
    before the wait for the preceding launch (and reads again after it); past 256 it
    reads them after the wait only.  Both sides of that limit match the oracle, with
    ragged lengths (zero included)."""
    Hkv, G, dh, cap = 1, 2, 64, 48
    rng = np.random.default_rng(B)
    lens = [int(x) for x in rng.integers(0, cap + 1, size=B)]
    lens[0], lens[-1] = 0, cap
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 61)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 4, 0, 0))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    got = gpu_decode(cfg, cache, q, lens)
    assert np.all(got[0] == 0)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, f"B={B}")


def test_decode_lengths_rewritten_on_device_between_calls(cuda_device):
    """A length changed on the device by the launch right before the decode call (the
    kernel's early read of the lengths may see the old ones) gives the new lengths'
    result, call after call."""
    B, Hkv, G, dh, cap = 4, 2, 4, 128, 512
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 67)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 8, 0, 0))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    vmaxs = {}
    d_len = torch.tensor([512, 300, 1, 129], dtype=torch.int32, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    ws = Workspace(cfg, 0, torch.device("cuda"))
    qd = q.cuda()
    for step, delta in enumerate([0, -37, 90, -200, 64]):
        d_len.add_(delta).clamp_(0, cap)          # a device kernel right before the call
        kvq.kvq_decode_attn(cfg, cache, qd, d_len, cap, out, ws)
        torch.cuda.synchronize()
        lens = [int(x) for x in d_len.cpu()]
        want = oracle_decode(cfg, oc, q, lens)
        assert_close_to_oracle(out.cpu().numpy(), want, vmax_per_batch(oc[2], oc[3], cfg, lens), G,
                               f"step {step} lens {lens}")
    assert kvq.kvq_workspace_status(ws) == 0


def test_decode_edge_lengths_and_capacity_tail(cuda_device):
    # capacity 80 is not a multiple of the 64-token tile: the last tile runs past it
    B, Hkv, G, dh, cap = 6, 1, 2, 128, 80
    lens = [0, 1, 63, 64, 65, 80]
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 41)
    for fmt in ((8, 8, 0, 0), (4, 4, 32, 32), (16, 16, 0, 0)):
        cfg = _cfg(B, cap, Hkv, G, dh, fmt)
        cache = gpu_cache(cfg, k, v)
        oc = oracle_cache(k, v, cfg)
        want = oracle_decode(cfg, oc, q, lens)
        got = gpu_decode(cfg, cache, q, lens)
        assert np.all(got[0] == 0)
        assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, lens), G, str(fmt))


def test_decode_nan_past_length_is_ignored(cuda_device):
    # 16-bit cache with NaN/Inf in positions past the attended length
    B, Hkv, G, dh, cap = 1, 1, 1, 128, 64
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 43)
    k[:, 30:] = float("nan")
    v[:, 30:] = float("inf")
    cfg = _cfg(B, cap, Hkv, G, dh, (16, 16, 0, 0))
    cache = gpu_cache(cfg, k, v)
    got = gpu_decode(cfg, cache, q, [30])
    oc = oracle_cache(k[:, :30], v[:, :30], Config(**{**cfg.__dict__}))
    want = oracle_decode(cfg, oc, q, [30])
    assert np.all(np.isfinite(got))
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, [30]), G, "nan tail")


def test_decode_value_scale_range(cuda_device):
    # tiny and huge value magnitudes: p * s_V must stay representable
    B, Hkv, G, dh, cap = 2, 1, 4, 128, 256
    for sv in (1e-4, 30.0):
        k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float32, 47, scale_v=sv)
        cfg = _cfg(B, cap, Hkv, G, dh, (8, 8, 0, 0))
        cache = gpu_cache(cfg, k, v)
        oc = oracle_cache(k, v, cfg)
        want = oracle_decode(cfg, oc, q.half(), [256, 100])
        got = gpu_decode(cfg, cache, q.half(), [256, 100])
        assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, [256, 100]), G, str(sv))


def test_decode_softmax_scale_override(cuda_device):
    B, Hkv, G, dh, cap = 1, 2, 2, 128, 128
    k, v, q = _inputs(B, cap, Hkv, G, dh, torch.float16, 53)
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 8, 0, 0))
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    for sc in (0.02, 0.3):
        want = oracle_decode(cfg, oc, q, [128], scale=sc)
        got = gpu_decode(cfg, cache, q, [128], scale=sc)
        assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], cfg, [128]), G, str(sc))


def test_tiny_workload_prompt_then_252_steps(cuda_device):
    """mni-ml page benchmark shape: 4-token prompt, then 252 append+attend steps,
    every step checked against the oracle (B=1, 4 heads, head_dim 64, fp32, INT8)."""
    w = inputs.WORKLOADS[1]
    cfg = Config(batch=1, capacity=w.capacity, n_q_heads=4, n_kv_heads=4, head_dim=64,
                 k_bits=8, v_bits=8, k_group=64, v_group=64)
    k, v = inputs.kv_tokens(w, 0, 256)
    cache = LayerCache(cfg)
    ws = Workspace(cfg)
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, k[:, :4].cuda().contiguous(), v[:, :4].cuda().contiguous(), pos, 0, 4)
    oc = oracle_cache(k, v, cfg)
    worst = 0.0
    for step in range(252):
        # each step appends the newest token (position 4 + step), then attends over all
        L = 5 + step
        pos.fill_(L - 1)
        kvq.kvq_append(cfg, cache, k[:, L - 1:L].cuda().contiguous(),
                       v[:, L - 1:L].cuda().contiguous(), pos, L - 1, 1)
        q = inputs.queries(w, 0, step)
        d_len = torch.tensor([L], dtype=torch.int32, device="cuda")
        out = torch.empty(1, 4, 64, dtype=torch.float32, device="cuda")
        kvq.kvq_decode_attn(cfg, cache, q.cuda(), d_len, L, out, ws)
        want = oracle_decode(cfg, oc, q, [L])
        vmax = vmax_per_batch(oc[2], oc[3], cfg, [L])
        worst = max(worst, assert_close_to_oracle(out.cpu().numpy(), want, vmax, 1, f"step {step}"))
    _compare_codes(cfg, cache, oc, 256)
    assert kvq.kvq_workspace_status(ws) == 0


def _sampled_full_size(widx, fmt, layer, pairs, device="cuda", kv_format=0):
    w = inputs.WORKLOADS[widx]
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=fmt[0], v_bits=fmt[1],
                 k_group=fmt[2], v_group=fmt[3], kv_format=kv_format)
    L = w.context
    k, v = inputs.kv_tokens(w, layer, L, device)
    cache = gpu_cache(cfg, k, v, device)
    q = inputs.queries(w, layer, 0, device)
    got = gpu_decode(cfg, cache, q, [L] * w.batch)
    gc = read_gpu_cache(cache, cfg)
    G = w.n_q_heads // w.n_kv_heads
    for (b, kvh) in pairs:
        sub = Config(**{**cfg.__dict__, "batch": 1, "n_kv_heads": 1, "n_q_heads": G})
        kk, vv = k[b:b + 1, :, kvh:kvh + 1].cpu(), v[b:b + 1, :, kvh:kvh + 1].cpu()
        oc = oracle_cache(kk, vv, sub)
        for i in range(4):
            if oc[i] is not None:
                assert np.array_equal(gc[i][b, kvh, :L], oc[i][0, 0, :L]), (b, kvh, i)
        qq = q[b:b + 1, kvh * G:(kvh + 1) * G].cpu()
        want = oracle_decode(sub, oc, qq, [L])
        vmax = vmax_per_batch(oc[2], oc[3], sub, [L])
        assert_close_to_oracle(got[b:b + 1, kvh * G:(kvh + 1) * G], want, vmax, G, f"{(b, kvh)}")


def test_full_size_int8kv_d2048(cuda_device):
    _sampled_full_size(2, (8, 8, 0, 0), 0, [(0, 0), (0, 7), (0, 15)])


@pytest.mark.parametrize("fmt", [(8, 4, 0, 32), (4, 8, 32, 0)])
def test_full_size_mixed_gqa_outliers(cuda_device, fmt):
    _sampled_full_size(3, fmt, 5, [(0, 0), (0, 3), (0, 7)])


@pytest.mark.parametrize("fmt", [(8, 8, 0, 0), (8, 4, 0, 0), (4, 4, 0, 0)])
def test_full_size_long_context_8k(cuda_device, fmt):
    _sampled_full_size(4, fmt, 1, [(0, 0), (7, 3), (15, 7)])
