"""GPU parity for h-mode: quantize-on-append of h, the tcgen05 reconstruction GEMM
K = W_k bf16(h^), V = W_v bf16(h^), and decode attention over the rebuilt K/V.

The oracle computes the GEMM in fp64 from the same bf16 operands and rounds to
fp16; the GPU accumulates in fp32, so a rebuilt element may differ from the
oracle's fp16 by one rounding step when the exact value sits near a rounding
boundary: the tests bound the error by the fp16 step plus a small fp32
accumulation term and require almost every element to match bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs
from _helpers import TOL, assert_close_to_oracle

pytestmark = pytest.mark.gpu


def _hcfg(B, cap, D, hbits, hgroups, G=1):
    H = D // 128
    return Config(batch=B, capacity=cap, mode=kvq.KVQ_MODE_H, d_model=D, h_bits=hbits,
                  h_groups=hgroups, n_q_heads=H * G, n_kv_heads=H, head_dim=128)


def _h_and_w(B, n, D, seed):
    g = torch.Generator().manual_seed(seed)
    r = torch.randn(B, n, D, generator=g)
    h = ((r - r.mean(-1, keepdim=True)) / torch.sqrt(r.var(-1, unbiased=False, keepdim=True) + 1e-5)).half()
    W = (torch.randn(2 * D, D, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    return h, W


def _oracle_kv(h, W, cfg, L):
    """Oracle rebuild of K, V for tokens < L: returns (f64 [B, 2, Hkv, L, 128], fp16 bits)."""
    B, n, D = h.shape
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    out64, out16 = [], []
    for b in range(B):
        hb = h[b, :L].float().numpy()
        if cfg.h_bits == 16:
            codes, scales = hb.astype(np.float16).view(np.uint16), None
        else:
            codes, scales = oracle.quantize_rows(hb, D // cfg.h_groups, cfg.h_bits)
        y64, y16 = oracle.h_reconstruct(codes, scales, D, max(cfg.h_groups, 1), cfg.h_bits, Wb, True)
        H = cfg.n_kv_heads
        out64.append(y64.reshape(L, 2, H, 128).transpose(1, 2, 0, 3))
        out16.append(y16.reshape(L, 2, H, 128).transpose(1, 2, 0, 3))
    return np.stack(out64), np.stack(out16)


def _gpu_kv(cfg, h, W, L, out_cap):
    cache = LayerCache(cfg)
    B, n, D = h.shape
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, h.cuda(), None, pos, 0, n)
    H = cfg.n_kv_heads
    k_out = torch.full((B, H, out_cap, 128), float("nan"), dtype=torch.float16, device="cuda")
    v_out = torch.full_like(k_out, float("nan"))
    operand = torch.full((kvq.kvq_h_operand_bytes(cfg, L) // 2,), float("nan"),
                         dtype=torch.bfloat16, device="cuda")
    kvq.kvq_h_reconstruct(cfg, cache, W.cuda(), L, k_out, v_out, out_cap, operand)
    torch.cuda.synchronize()
    return cache, k_out.cpu(), v_out.cpu()


def _check_kv(gk, gv, o64, o16, L):
    got = np.stack([gk[:, :, :L].float().numpy(), gv[:, :, :L].float().numpy()], 1)
    want16 = o16.view(np.float16).astype(np.float32)
    # one fp16 rounding step of the value plus fp32 accumulation over D terms
    step = np.abs(want16) * 2.0 ** -10 + 2.0 ** -24
    bound = step + 1e-5 * np.abs(o64).max()
    assert np.all(np.abs(got - o64) <= bound + np.abs(want16 - o64)), np.abs(got - o64).max()
    exact = np.mean(got.view(np.int32) == want16.view(np.int32))
    assert exact > 0.995, exact


@pytest.mark.parametrize("hbits,hgroups", [(4, 4), (8, 4), (16, 0), (4, 16)])
def test_h_reconstruct_matches_oracle(cuda_device, hbits, hgroups):
    B, n, D, cap, L = 2, 200, 512, 256, 200
    cfg = _hcfg(B, cap, D, hbits, hgroups)
    h, W = _h_and_w(B, n, D, 3 + hbits + hgroups)
    cache, gk, gv = _gpu_kv(cfg, h, W, L, 256)
    # the h codes themselves are bit-exact with the oracle quantiser
    if hbits != 16:
        codes, scales = oracle.quantize_rows(h.float().numpy(), D // hgroups, hbits)
        row, ng = codes.shape[-1], scales.shape[-1]
        gc = cache.k_codes.cpu().numpy()[: B * cap * row].reshape(B, cap, row)[:, :n]
        gs = cache.k_scales.cpu().numpy().view(np.uint16)[: B * cap * ng].reshape(B, cap, ng)[:, :n]
        assert np.array_equal(gc, codes) and np.array_equal(gs, scales)
    o64, o16 = _oracle_kv(h, W, cfg, L)
    _check_kv(gk, gv, o64, o16, L)
    # rows past the length are left untouched
    assert torch.isnan(gk[:, :, L:]).all() and torch.isnan(gv[:, :, L:]).all()


def test_h_reconstruct_short_and_partial_tiles(cuda_device):
    B, D, cap = 3, 256, 128
    cfg = _hcfg(B, cap, D, 4, 2)
    h, W = _h_and_w(B, 128, D, 77)
    for L in (1, 64, 127, 128):
        cache, gk, gv = _gpu_kv(cfg, h, W, L, 128)
        o64, o16 = _oracle_kv(h, W, cfg, L)
        _check_kv(gk, gv, o64, o16, L)


@pytest.mark.parametrize("hbits,G", [(4, 1), (8, 2)])
def test_hmode_decode_matches_oracle(cuda_device, hbits, G):
    B, n, D, cap = 2, 300, 512, 320
    lens = [300, 129]
    cfg = _hcfg(B, cap, D, hbits, 4, G)
    h, W = _h_and_w(B, n, D, 11 + hbits)
    cache = LayerCache(cfg)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, h.cuda(), None, pos, 0, n)
    H = cfg.n_kv_heads
    q = torch.randn(B, H * G, 128, generator=torch.Generator().manual_seed(5)).half()
    out = torch.empty(B, H * G, 128, dtype=torch.float32, device="cuda")
    ws = Workspace(cfg)
    scratch = torch.empty(kvq.kvq_h_scratch_bytes(cfg, max(lens)) // 2, dtype=torch.float16,
                          device="cuda")
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_attn(cfg, cache, q.cuda(), d_len, max(lens), out, ws, w_kv=W.cuda(),
                        kv_scratch=scratch)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    o64, o16 = _oracle_kv(h, W, cfg, max(lens))
    kc = np.zeros((B, H, cap, 128), np.uint16)
    vc = np.zeros((B, H, cap, 128), np.uint16)
    kc[:, :, :n] = o16[:, 0]
    vc[:, :, :n] = o16[:, 1]
    want = oracle.decode_layer(q.float().numpy(), np.array(lens, np.int32), kc, None, 16, 128,
                               vc, None, 16, 128, H)
    vmax = np.array([np.abs(vc[b, :, :L].view(np.float16).astype(np.float64)).max()
                     for b, L in enumerate(lens)])
    assert_close_to_oracle(out.cpu().numpy(), want, vmax, G, f"h{hbits}")


def test_hmode_full_size_sampled(cuda_device):
    """h-mode workload (B=8, S=1024, D=2048, 16 heads x 128, INT4-h with 16 scales):
    rebuild on the GPU, check sampled (sequence, head) pairs against the oracle."""
    w = inputs.WORKLOADS[5]
    B, S, D = w.batch, w.context, w.d_model
    cfg = _hcfg(B, w.capacity, D, 4, 16)
    h, W = inputs.hmode_inputs(w, S, "cuda")
    cache = LayerCache(cfg)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, h, None, pos, 0, S)
    H = cfg.n_kv_heads
    k_out = torch.empty(B, H, S, 128, dtype=torch.float16, device="cuda")
    v_out = torch.empty_like(k_out)
    operand = torch.empty(kvq.kvq_h_operand_bytes(cfg, S) // 2, dtype=torch.bfloat16, device="cuda")
    kvq.kvq_h_reconstruct(cfg, cache, W, S, k_out, v_out, S, operand)
    torch.cuda.synchronize()
    Wb = W.cpu().view(torch.int16).numpy().view(np.uint16)
    for b, head in ((0, 0), (5, 9), (7, 15)):
        codes, scales = oracle.quantize_rows(h[b].float().cpu().numpy(), D // 16, 4)
        rows = np.concatenate([Wb[head * 128:(head + 1) * 128], Wb[(H + head) * 128:(H + head + 1) * 128]])
        y64, y16 = oracle.h_reconstruct(codes, scales, D, 16, 4, rows, True)
        o64 = y64.reshape(S, 2, 1, 128).transpose(1, 2, 0, 3)[None]
        o16 = y16.reshape(S, 2, 1, 128).transpose(1, 2, 0, 3)[None]
        gk = k_out[b:b + 1, head:head + 1].cpu()
        gv = v_out[b:b + 1, head:head + 1].cpu()
        _check_kv(gk, gv, o64, o16, S)
