"""GPU parity for the sliding-window cache (on-device page, "Sliding Window
Eviction": keep the most recent tokens plus the first tokens as anchors).

The cache holds n_anchor anchor slots and a ring of `window` slots; token t sits
in slot t (t < n_anchor) or n_anchor + (t - n_anchor) mod window.  The oracle is
the plain definition: attention over the anchor tokens and the last `window`
tokens of the sequence, quantised exactly like any other token.  Codes in their
ring slots must match bit for bit; outputs within 2e-3 * max|V^|.
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace
from _helpers import (assert_close_to_oracle, oracle_cache, oracle_decode, read_gpu_cache,
                      vmax_per_batch)

pytestmark = pytest.mark.gpu

N_ANCHOR, WINDOW = 64, 1536


def _slot(t):
    return t if t < N_ANCHOR else N_ANCHOR + (t - N_ANCHOR) % WINDOW


def _kept(L):
    """Token positions a window cache holds after L tokens (anchors, then the window)."""
    return sorted(set(range(min(N_ANCHOR, L))) | set(range(max(N_ANCHOR, L - WINDOW), L)))


def _sub_layer(cache, cfg, b):
    """KvqLayer-compatible view of sequence b's part of every buffer."""
    sub = LayerCache.__new__(LayerCache)
    rows = cfg.n_kv_heads * cfg.capacity
    for name, bits, grp in (("k_codes", cfg.k_bits, None), ("k_scales", cfg.k_bits, cfg.k_group),
                            ("v_codes", cfg.v_bits, None), ("v_scales", cfg.v_bits, cfg.v_group)):
        t = getattr(cache, name)
        if t is None:
            setattr(sub, name, None)
            continue
        pairs = 2 if cfg.kv_format == kvq.KVQ_FMT_ASYM else 1     # (scale, zero-point)
        per = rows * (cfg.head_dim * bits // 8 if grp is None else 2 * pairs * (cfg.head_dim // grp))
        per //= t.element_size()
        setattr(sub, name, t[b * per:(b + 1) * per])
    return sub


@pytest.mark.parametrize("fmt", [(4, 8, 32, 128), (8, 8, 128, 128), (8, 4, 128, 32),
                                 (8, 8, 128, 32, kvq.KVQ_FMT_E4M3), (8, 8, 32, 128, kvq.KVQ_FMT_ASYM)])
def test_window_cache_decode_step_matches_oracle(cuda_device, fmt):
    lens = [100, 1600, 1700, 4000]
    B, Hkv, G, dh = len(lens), 2, 4, 128
    cap = N_ANCHOR + WINDOW
    kb, vb, kg, vg = fmt[:4]
    kf = fmt[4] if len(fmt) > 4 else kvq.KVQ_FMT_INT
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                 k_bits=kb, v_bits=vb, k_group=kg, v_group=vg, window=WINDOW, n_anchor=N_ANCHOR,
                 kv_format=kf)
    g = torch.Generator().manual_seed(5 + kb + vb)
    Lmax = max(lens)
    k = torch.randn(B, Lmax, Hkv, dh, generator=g).half()
    v = torch.randn(B, Lmax, Hkv, dh, generator=g).half()
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    cache = LayerCache(cfg)
    cfg1 = Config(**{**cfg.__dict__, "batch": 1})
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b, L in enumerate(lens):
        # prefill tokens 0 .. L-2 in one call (earlier ring passes are skipped)
        if L > 1:
            kvq.kvq_append(cfg1, _sub_layer(cache, cfg, b), k[b:b + 1, :L - 1].cuda().contiguous(),
                           v[b:b + 1, :L - 1].cuda().contiguous(), zero, 0, L - 1)
    # one decode step: append token L-1 into its ring slot and attend
    k_new = torch.stack([k[b, L - 1] for b, L in enumerate(lens)]).cuda()
    v_new = torch.stack([v[b, L - 1] for b, L in enumerate(lens)]).cuda()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hkv * G, dh), float("nan"), dtype=torch.float32, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k_new, v_new, q.cuda(), d_len, Lmax, out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    got = out.cpu().numpy()
    gc = read_gpu_cache(cache, cfg)
    for b, L in enumerate(lens):
        kept = _kept(L)
        kk = k[b:b + 1, kept].contiguous()
        vv = v[b:b + 1, kept].contiguous()
        sub = Config(**{**cfg.__dict__, "batch": 1, "capacity": len(kept), "window": 0,
                        "n_anchor": 0})
        oc = oracle_cache(kk, vv, sub)
        # every kept token's codes and scales sit in its ring slot
        slots = [_slot(t) for t in kept]
        for i in range(4):
            if oc[i] is not None:
                assert np.array_equal(gc[i][b][:, slots], oc[i][0]), (L, i)
        want = oracle_decode(sub, oc, q[b:b + 1], [len(kept)])
        vmax = vmax_per_batch(oc[2], oc[3], sub, [len(kept)])
        assert_close_to_oracle(got[b:b + 1], want, vmax, G, f"{fmt} L={L}")


def test_window_steps_across_the_wrap(cuda_device):
    """Decode steps one token at a time across the first wrap of the ring."""
    B, Hkv, G, dh = 1, 1, 2, 64
    cap = N_ANCHOR + WINDOW
    cfg = Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                 k_bits=8, v_bits=4, k_group=64, v_group=32, window=WINDOW, n_anchor=N_ANCHOR)
    g = torch.Generator().manual_seed(77)
    steps = list(range(cap - 3, cap + 4))
    Lmax = steps[-1]
    k = torch.randn(B, Lmax, Hkv, dh, generator=g).half()
    v = torch.randn(B, Lmax, Hkv, dh, generator=g).half()
    cache = LayerCache(cfg)
    kvq.kvq_append(cfg, cache, k[:, :steps[0] - 1].cuda().contiguous(),
                   v[:, :steps[0] - 1].cuda().contiguous(),
                   torch.zeros(1, dtype=torch.int32, device="cuda"), 0, steps[0] - 1)
    ws = Workspace(cfg)
    d_len = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hkv * G, dh, dtype=torch.float32, device="cuda")
    for L in steps:
        d_len.fill_(L)
        q = torch.randn(B, Hkv * G, dh, generator=g).half()
        kvq.kvq_append_decode_attn(cfg, cache, k[:, L - 1].cuda().contiguous(),
                                   v[:, L - 1].cuda().contiguous(), q.cuda(), d_len, L, out, ws)
        kept = _kept(L)
        sub = Config(**{**cfg.__dict__, "capacity": len(kept), "window": 0, "n_anchor": 0})
        oc = oracle_cache(k[:, kept].contiguous(), v[:, kept].contiguous(), sub)
        want = oracle_decode(sub, oc, q, [len(kept)])
        vmax = vmax_per_batch(oc[2], oc[3], sub, [len(kept)])
        assert_close_to_oracle(out.cpu().numpy(), want, vmax, G, f"L={L}")
    assert kvq.kvq_workspace_status(ws) == 0


def test_window_workload_full_size_sampled(cuda_device):
    """Sliding-window workload at full size (B=64, 8 KV heads, 1536 + 64 slots, 8192
    tokens seen, K4V8): one decode step, sampled (sequence, KV head) pairs checked."""
    from quantized_kv_cache_22_b200 import inputs
    w = inputs.WORKLOADS[6]
    kb, vb, kg, vg = w.kv_variants[0]
    cfg = Config(batch=w.batch, capacity=w.capacity, n_q_heads=w.n_q_heads,
                 n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, k_bits=kb, v_bits=vb,
                 k_group=kg, v_group=vg, window=w.window, n_anchor=w.n_anchor)
    L = w.context
    first_win = L - 1 - w.window
    k, v = inputs.kv_tokens(w, 0, w.capacity, "cuda")
    cache = LayerCache(cfg)
    kvq.kvq_append(cfg, cache, k[:, :w.n_anchor].contiguous(), v[:, :w.n_anchor].contiguous(),
                   torch.zeros(w.batch, dtype=torch.int32, device="cuda"), 0, w.n_anchor)
    kvq.kvq_append(cfg, cache, k[:, w.n_anchor:].contiguous(), v[:, w.n_anchor:].contiguous(),
                   torch.full((w.batch,), first_win, dtype=torch.int32, device="cuda"),
                   first_win, w.window)
    k1, v1 = inputs.kv_tokens(w, 0, 1, "cuda", offset_seed=1)
    q = inputs.queries(w, 0, 0, "cuda")
    d_len = torch.full((w.batch,), L, dtype=torch.int32, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k1[:, 0].contiguous(), v1[:, 0].contiguous(), q, d_len,
                               L, out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    # logical tokens now cached: anchors 0..63, positions first_win+1 .. L-1 (the
    # token at first_win shared its slot with the newest one)
    kept_k = torch.cat([k[:, :w.n_anchor], k[:, w.n_anchor + 1:], k1], 1).cpu()
    kept_v = torch.cat([v[:, :w.n_anchor], v[:, w.n_anchor + 1:], v1], 1).cpu()
    positions = list(range(w.n_anchor)) + list(range(first_win + 1, L))
    slots = [_slot(t) for t in positions]
    gc = read_gpu_cache(cache, cfg)
    G = w.n_q_heads // w.n_kv_heads
    got = out.cpu().numpy()
    for (b, kvh) in ((0, 0), (31, 5), (63, 7)):
        sub = Config(**{**cfg.__dict__, "batch": 1, "n_kv_heads": 1, "n_q_heads": G,
                        "window": 0, "n_anchor": 0})
        oc = oracle_cache(kept_k[b:b + 1, :, kvh:kvh + 1], kept_v[b:b + 1, :, kvh:kvh + 1], sub)
        for i in range(4):
            assert np.array_equal(gc[i][b, kvh][slots], oc[i][0, 0]), (b, kvh, i)
        qq = q[b:b + 1, kvh * G:(kvh + 1) * G].cpu()
        want = oracle_decode(sub, oc, qq, [w.capacity])
        vmax = vmax_per_batch(oc[2], oc[3], sub, [w.capacity])
        assert_close_to_oracle(got[b:b + 1, kvh * G:(kvh + 1) * G], want, vmax, G, f"{(b, kvh)}")
