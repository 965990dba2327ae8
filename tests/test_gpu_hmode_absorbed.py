"""GPU parity for h-mode decode by query absorption (kvq_h_decode_absorbed).

The reconstruction path of the TinyLoop page ("運作原理") rebuilds K = W_k h^ and
V = W_v h^ for every cached token; by linearity the same attention is
qa = W_k,j^T q, s_t = tau qa . h^_t, out = W_v,j sum_t p_t h^_t.  The oracle
computes that in fp64 from the same codes and bf16 W (no bf16/fp16 roundings);
outputs must be within 2e-3 * max|V| of it, V = W_v h^ over the attended tokens.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs
from _helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu


def _cfg(B, cap, D, Dh, hbits, hgroups, G):
    H = D // Dh
    return Config(batch=B, capacity=cap, mode=kvq.KVQ_MODE_H, d_model=D, h_bits=hbits,
                  h_groups=hgroups, n_q_heads=H * G, n_kv_heads=H, head_dim=Dh)


def _h_and_w(B, n, D, seed):
    g = torch.Generator().manual_seed(seed)
    r = torch.randn(B, n, D, generator=g)
    h = ((r - r.mean(-1, keepdim=True)) / torch.sqrt(r.var(-1, unbiased=False, keepdim=True) + 1e-5)).half()
    W = (torch.randn(2 * D, D, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    return h, W


def _oracle(cfg, h, W, q, lens):
    """Oracle codes of h (per sequence), the absorbed attention, and max|V| per sequence."""
    B, n, D = h.shape
    codes = np.zeros((B, cfg.capacity, D * cfg.h_bits // 8), np.uint8)
    scales = np.zeros((B, cfg.capacity, cfg.h_groups), np.uint16)
    for b in range(B):
        c, s = oracle.quantize_rows(h[b].float().numpy(), D // cfg.h_groups, cfg.h_bits)
        codes[b, :n], scales[b, :n] = c, s
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    want = oracle.h_absorbed_decode(codes, scales, cfg.h_bits, cfg.h_groups, Wb, q.float().numpy(),
                                    np.array(lens, np.int32), cfg.n_kv_heads)
    Wv = W.double().numpy()[D:]
    vmax = []
    for b, L in enumerate(lens):
        if L == 0:
            vmax.append(1.0)
            continue
        hd = oracle.dequantize_rows(codes[b, :L], scales[b, :L], D, D // cfg.h_groups, cfg.h_bits)
        vmax.append(float(np.abs(hd @ Wv.T).max()))
    return codes, scales, want, np.array(vmax)


def _gpu(cfg, h, W, q, lens, out_dtype=torch.float32, scale=0.0):
    cache = LayerCache(cfg)
    B, n, _ = h.shape
    kvq.kvq_append(cfg, cache, h.cuda(), None, torch.zeros(B, dtype=torch.int32, device="cuda"), 0, n)
    L = max(lens)
    scratch = torch.full((kvq.kvq_h_absorbed_scratch_bytes(cfg, L) // 4,), float("nan"),
                         device="cuda")
    out = torch.full((B, cfg.n_q_heads, cfg.head_dim), float("nan"), dtype=out_dtype, device="cuda")
    kvq.kvq_h_decode_absorbed(cfg, cache, W.cuda(), q.cuda(), torch.tensor(lens, dtype=torch.int32,
                              device="cuda"), L, out, scratch, softmax_scale=scale)
    torch.cuda.synchronize()
    return cache, out.float().cpu().numpy()


@pytest.mark.parametrize("hbits,hgroups,G,Dh,D", [
    (4, 4, 1, 128, 512), (8, 4, 2, 128, 512), (4, 16, 1, 128, 2048), (4, 8, 4, 64, 512),
    (8, 16, 1, 64, 512), (4, 2, 8, 128, 256),
    # 128-element groups with more than 16 query heads (two m-tiles of heads)
    (4, 4, 3, 64, 512), (8, 4, 3, 64, 512)])
def test_absorbed_decode_matches_oracle(cuda_device, hbits, hgroups, G, Dh, D):
    B, n, cap = 3, 300, 320
    lens = [300, 1, 129]
    cfg = _cfg(B, cap, D, Dh, hbits, hgroups, G)
    h, W = _h_and_w(B, n, D, 3 + hbits + G + Dh)
    q = torch.randn(B, cfg.n_q_heads, Dh, generator=torch.Generator().manual_seed(9)).half()
    _, got = _gpu(cfg, h, W, q, lens)
    _, _, want, vmax = _oracle(cfg, h, W, q, lens)
    assert_close_to_oracle(got, want, vmax, G, f"h{hbits} g{hgroups} G{G} Dh{Dh}")


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
def test_absorbed_query_dtypes_scale_and_fp16_out(cuda_device, qdtype):
    B, n, cap, D = 2, 200, 256, 512
    lens = [200, 0]                 # an empty sequence gets zeros
    cfg = _cfg(B, cap, D, 128, 4, 4, 2)
    h, W = _h_and_w(B, n, D, 21)
    q = (torch.randn(B, cfg.n_q_heads, 128, generator=torch.Generator().manual_seed(4)) * 2).to(qdtype)
    _, got = _gpu(cfg, h, W, q, lens, out_dtype=torch.float16, scale=0.05)
    codes, scales = _oracle(cfg, h, W, q, lens)[:2]
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    want = oracle.h_absorbed_decode(codes, scales, 4, 4, Wb, q.float().numpy(),
                                    np.array(lens, np.int32), cfg.n_kv_heads, tau=0.05)
    vmax = _oracle(cfg, h, W, q, lens)[3]
    assert np.all(got[1] == 0)
    # fp16 output, held to the same 2e-3 * max|V^| as every other output
    err = np.abs(got[:1].astype(np.float64) - want[:1]).max()
    assert err <= 2e-3 * vmax[0], err


def test_absorbed_agrees_with_reconstruction_path(cuda_device):
    """Both h-mode paths approximate the same attention: their outputs agree within
    the sum of their tolerances."""
    B, n, cap, D = 2, 256, 256, 512
    lens = [256, 97]
    cfg = _cfg(B, cap, D, 128, 4, 4, 1)
    h, W = _h_and_w(B, n, D, 33)
    q = torch.randn(B, cfg.n_q_heads, 128, generator=torch.Generator().manual_seed(8)).half()
    cache, got = _gpu(cfg, h, W, q, lens)
    out = torch.empty(B, cfg.n_q_heads, 128, device="cuda")
    ws = Workspace(cfg)
    scratch = torch.empty(kvq.kvq_h_scratch_bytes(cfg, max(lens)) // 2, dtype=torch.float16,
                          device="cuda")
    kvq.kvq_decode_attn(cfg, cache, q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"),
                        max(lens), out, ws, w_kv=W.cuda(), kv_scratch=scratch)
    torch.cuda.synchronize()
    vmax = _oracle(cfg, h, W, q, lens)[3]
    err = np.abs(out.cpu().numpy() - got).max(axis=(1, 2))
    assert np.all(err <= 4e-3 * vmax), err


def test_absorbed_full_size_hmode_workload(cuda_device):
    """h-mode workload (B=8, S=1024, D=2048, 16 heads x 128, INT4-h, 16 scales per
    token): every (sequence, head) against the oracle."""
    w = inputs.WORKLOADS[5]
    B, S, D = w.batch, w.context, w.d_model
    cfg = _cfg(B, w.capacity, D, 128, 4, 16, 1)
    h, W = inputs.hmode_inputs(w, S, "cuda")
    q = inputs.queries(w, 0, 0, "cuda")
    _, got = _gpu(cfg, h, W, q, [S] * B)
    _, _, want, vmax = _oracle(cfg, h.cpu(), W.cpu(), q.cpu(), [S] * B)
    assert_close_to_oracle(got, want, vmax, 1, "full size")
