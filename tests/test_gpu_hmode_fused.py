"""GPU parity for h-mode decode with the reconstruction fused into the attention
(kvq_h_decode_fused): the tcgen05 GEMM computes each 128-token tile's K_j, V_j in
tensor memory and the epilogue attends over them; nothing is written back.

Oracle: the reconstruction of the TinyLoop page ("運作原理") in fp64 from the bf16(h^)
operand and the bf16 W (oracle.h_reconstruct before its fp16 rounding), then fp64
attention (oracle.attend) over the attended tokens.  Outputs within 2e-3 * max|V|.
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


def _cfg(B, cap, D, hbits, hgroups, G):
    H = D // 128
    return Config(batch=B, capacity=cap, mode=kvq.KVQ_MODE_H, d_model=D, h_bits=hbits,
                  h_groups=hgroups, n_q_heads=H * G, n_kv_heads=H, head_dim=128)


def _h_and_w(B, n, D, seed):
    g = torch.Generator().manual_seed(seed)
    r = torch.randn(B, n, D, generator=g)
    h = ((r - r.mean(-1, keepdim=True)) / torch.sqrt(r.var(-1, unbiased=False, keepdim=True) + 1e-5)).half()
    W = (torch.randn(2 * D, D, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    return h, W


def _oracle(cfg, h, W, q, lens, seqs=None, tau=0.0):
    """fp64 attention over K, V = W bf16(h^) (no fp16 rounding); [B, Hq, 128] and max|V|."""
    B, n, D = h.shape
    H, G = cfg.n_kv_heads, cfg.n_q_heads // cfg.n_kv_heads
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    want = np.zeros((B, cfg.n_q_heads, 128))
    vmax = np.ones(B)
    tau = tau or 1 / np.sqrt(128)
    for b in (range(B) if seqs is None else seqs):
        L = lens[b]
        if L == 0:
            continue
        hb = h[b, :L].float().numpy()
        if cfg.h_bits == 16:
            codes, scales = hb.astype(np.float16).view(np.uint16), None
        else:
            codes, scales = oracle.quantize_rows(hb, D // cfg.h_groups, cfg.h_bits)
        y64, _ = oracle.h_reconstruct(codes, scales, D, max(cfg.h_groups, 1), cfg.h_bits, Wb, True)
        K = y64[:, :D].reshape(L, H, 128)
        V = y64[:, D:].reshape(L, H, 128)
        vmax[b] = np.abs(V).max()
        qb = q[b].float().numpy().astype(np.float64)
        for hq in range(cfg.n_q_heads):
            want[b, hq] = oracle.attend(qb[hq], K[:, hq // G], V[:, hq // G], tau)
    return want, vmax


def _gpu(cfg, h, W, q, lens, out_dtype=torch.float32, scale=0.0):
    cache = LayerCache(cfg)
    B, n, _ = h.shape
    kvq.kvq_append(cfg, cache, h.cuda(), None, torch.zeros(B, dtype=torch.int32, device="cuda"), 0, n)
    L = max(lens)
    scratch = torch.zeros(kvq.kvq_h_fused_scratch_bytes(cfg, L) // 4, device="cuda")
    out = torch.full((B, cfg.n_q_heads, 128), float("nan"), dtype=out_dtype, device="cuda")
    kvq.kvq_h_decode_fused(cfg, cache, W.cuda(), q.cuda(),
                           torch.tensor(lens, dtype=torch.int32, device="cuda"), L, out, scratch,
                           softmax_scale=scale)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(scratch) == 0
    return cache, out.float().cpu().numpy()


@pytest.mark.parametrize("hbits,hgroups,G", [(4, 4, 1), (8, 4, 2), (16, 0, 1), (4, 2, 8)])
def test_fused_decode_matches_oracle(cuda_device, hbits, hgroups, G):
    B, n, cap, D = 3, 300, 320, 512 if G < 8 else 256
    lens = [300, 129, 0]
    cfg = _cfg(B, cap, D, hbits, hgroups, G)
    h, W = _h_and_w(B, n, D, 7 + hbits + G)
    q = torch.randn(B, cfg.n_q_heads, 128, generator=torch.Generator().manual_seed(3)).half()
    _, got = _gpu(cfg, h, W, q, lens)
    want, vmax = _oracle(cfg, h, W, q, lens)
    assert np.all(got[2] == 0)
    assert_close_to_oracle(got, want, vmax, G, f"h{hbits} G{G}")


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
def test_fused_query_dtypes_scale_fp16_out_and_one_token(cuda_device, qdtype):
    B, n, cap, D = 2, 140, 256, 512
    lens = [1, 140]
    cfg = _cfg(B, cap, D, 4, 4, 2)
    h, W = _h_and_w(B, n, D, 29)
    q = (torch.randn(B, cfg.n_q_heads, 128, generator=torch.Generator().manual_seed(6)) * 2).to(qdtype)
    _, got = _gpu(cfg, h, W, q, lens, out_dtype=torch.float16, scale=0.04)
    want, vmax = _oracle(cfg, h, W, q, lens, tau=0.04)
    # fp16 output, held to the same 2e-3 * max|V^| as every other output
    err = np.abs(got.astype(np.float64) - want).max(axis=(1, 2))
    assert np.all(err <= 2e-3 * vmax), err


def test_fused_agrees_with_reconstruction_and_absorbed_paths(cuda_device):
    B, n, cap, D = 2, 256, 256, 512
    lens = [256, 200]
    cfg = _cfg(B, cap, D, 4, 4, 1)
    h, W = _h_and_w(B, n, D, 41)
    q = torch.randn(B, cfg.n_q_heads, 128, generator=torch.Generator().manual_seed(2)).half()
    cache, got = _gpu(cfg, h, W, q, lens)
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    rec = torch.empty(B, cfg.n_q_heads, 128, device="cuda")
    scratch = torch.empty(kvq.kvq_h_scratch_bytes(cfg, max(lens)) // 2, dtype=torch.float16, device="cuda")
    kvq.kvq_decode_attn(cfg, cache, q.cuda(), d_len, max(lens), rec, Workspace(cfg), w_kv=W.cuda(),
                        kv_scratch=scratch)
    ab = torch.empty_like(rec)
    abs_scratch = torch.empty(kvq.kvq_h_absorbed_scratch_bytes(cfg, max(lens)) // 4, device="cuda")
    kvq.kvq_h_decode_absorbed(cfg, cache, W.cuda(), q.cuda(), d_len, max(lens), ab, abs_scratch)
    torch.cuda.synchronize()
    _, vmax = _oracle(cfg, h, W, q, lens)
    for other in (rec, ab):
        err = np.abs(other.cpu().numpy() - got).max(axis=(1, 2))
        assert np.all(err <= 4e-3 * vmax), err


def test_fused_full_size_hmode_workload(cuda_device):
    """h-mode workload (B=8, S=1024, D=2048, 16 heads x 128, INT4-h, 16 scales per
    token): sequences 0 and 7 against the oracle, every head."""
    w = inputs.WORKLOADS[5]
    B, S, D = w.batch, w.context, w.d_model
    cfg = _cfg(B, w.capacity, D, 4, 16, 1)
    h, W = inputs.hmode_inputs(w, S, "cuda")
    q = inputs.queries(w, 0, 0, "cuda")
    _, got = _gpu(cfg, h, W, q, [S] * B)
    want, vmax = _oracle(cfg, h.cpu(), W.cpu(), q.cpu(), [S] * B, seqs=(0, 7))
    for b in (0, 7):
        assert_close_to_oracle(got[b:b + 1], want[b:b + 1], vmax[b:b + 1], 1, f"seq {b}")
