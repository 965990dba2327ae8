"""GPU parity for the paged cache: a pool of 128-token pages per layer and a block
table that maps each sequence's logical pages to pool pages.

Codes and scales of every token must sit, bit-exact with the oracle quantiser, at
slot t % 128 of page block_table[b][t / 128]; attention outputs must match the
oracle within 2e-3 * max|V^| and match the contiguous layout bit for bit (same
partition, same arithmetic).
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace
from _helpers import (assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache, oracle_decode,
                      vmax_per_batch)

pytestmark = pytest.mark.gpu

PAGE = 128


def _gather_pool(cache, cfg, table):
    """Pool buffers -> logical [B][Hkv][capacity][...] arrays (codes, scales) like the oracle's."""
    B, H, cap, dh = cfg.batch, cfg.n_kv_heads, cfg.capacity, cfg.head_dim
    npg = cap // PAGE
    res = []
    for codes, scales, bits, grp in ((cache.k_codes, cache.k_scales, cfg.k_bits, cfg.k_group or dh),
                                     (cache.v_codes, cache.v_scales, cfg.v_bits, cfg.v_group or dh)):
        row = dh * bits // 8
        c = codes.cpu().numpy()[: cfg.n_pages * H * PAGE * row].reshape(cfg.n_pages, H, PAGE, row)
        if bits == 16:
            c = c.view(np.uint16).reshape(cfg.n_pages, H, PAGE, dh)
        out_c = np.stack([np.concatenate([c[table[b, j]] for j in range(npg)], axis=1)
                          for b in range(B)])
        res.append(out_c)
        if bits == 16:
            res.append(None)
            continue
        ng = dh // grp
        sc = scales.cpu().numpy().view(np.uint16)[: cfg.n_pages * H * PAGE * ng].reshape(
            cfg.n_pages, H, PAGE, ng)
        res.append(np.stack([np.concatenate([sc[table[b, j]] for j in range(npg)], axis=1)
                             for b in range(B)]))
    return res


@pytest.mark.parametrize("fmt", [(8, 8, 0, 0), (4, 4, 32, 32), (8, 4, 0, 32), (16, 16, 0, 0)])
def test_paged_decode_step_matches_oracle_and_contiguous(cuda_device, fmt):
    lens = [1000, 129, 513]
    B, Hkv, G, dh, cap, n_pages = len(lens), 2, 4, 128, 1024, 30
    kb, vb, kg, vg = fmt
    base = dict(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)
    cfg = Config(**base, page_tokens=PAGE, n_pages=n_pages)
    g = torch.Generator().manual_seed(13 + kb + vb)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half()
    q = torch.randn(B, Hkv * G, dh, generator=g).half()
    perm = torch.randperm(n_pages, generator=g)[: B * (cap // PAGE)]
    table = perm.view(B, cap // PAGE).to(torch.int32)
    cache = LayerCache(cfg, block_table=table.cuda())
    # prefill every sequence's positions 0 .. max-2, then a decoy at each newest position
    n_pre = max(lens) - 1
    kvq.kvq_append(cfg, cache, k[:, :n_pre].cuda().contiguous(), v[:, :n_pre].cuda().contiguous(),
                   torch.zeros(B, dtype=torch.int32, device="cuda"), 0, n_pre)
    decoy = (torch.randn(B, 1, Hkv, dh, generator=g) * 7).half().cuda()
    kvq.kvq_append(cfg, cache, decoy, decoy,
                   torch.tensor([L - 1 for L in lens], dtype=torch.int32, device="cuda"),
                   max(lens) - 1, 1)
    k_new = torch.stack([k[b, L - 1] for b, L in enumerate(lens)]).cuda()
    v_new = torch.stack([v[b, L - 1] for b, L in enumerate(lens)]).cuda()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hkv * G, dh), float("nan"), dtype=torch.float32, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k_new, v_new, q.cuda(), d_len, max(lens), out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    got = out.cpu().numpy()

    oc = oracle_cache(k, v, Config(**base))
    gathered = _gather_pool(cache, cfg, table.numpy())
    for i, name in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        if oc[i] is None:
            continue
        for b, L in enumerate(lens):
            assert np.array_equal(gathered[i][b, :, :L], oc[i][b, :, :L]), (name, b)
    want = oracle_decode(Config(**base), oc, q, lens)
    assert_close_to_oracle(got, want, vmax_per_batch(oc[2], oc[3], Config(**base), lens), G,
                           str(fmt))
    # the contiguous layout of the same tokens gives the same bits
    contiguous = gpu_cache(Config(**base), k, v)
    ref = gpu_decode(Config(**base), contiguous, q, lens)
    assert np.array_equal(got, ref)


def test_paged_shared_pages_and_partial_table(cuda_device):
    """Two sequences whose tables name the same pool pages read the same tokens; pages
    past a sequence's length need no valid entry (only attended pages are read)."""
    B, Hkv, G, dh, cap, n_pages = 2, 1, 2, 64, 512, 4
    base = dict(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                k_bits=8, v_bits=8, k_group=64, v_group=64)
    cfg = Config(**base, page_tokens=PAGE, n_pages=n_pages)
    g = torch.Generator().manual_seed(3)
    k = torch.randn(1, 300, Hkv, dh, generator=g).half()
    v = torch.randn(1, 300, Hkv, dh, generator=g).half()
    q = torch.randn(1, Hkv * G, dh, generator=g).half()
    table = torch.tensor([[2, 0, 3, 1], [2, 0, 3, 1]], dtype=torch.int32)
    cache = LayerCache(cfg, block_table=table.cuda())
    one = Config(**{**cfg.__dict__, "batch": 1})
    kvq.kvq_append(one, cache, k.cuda(), v.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"),
                   0, 300)
    d_len = torch.tensor([300, 300], dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hkv * G, dh, dtype=torch.float32, device="cuda")
    ws = Workspace(cfg)
    kvq.kvq_decode_attn(cfg, cache, q.repeat(2, 1, 1).cuda(), d_len, 300, out, ws)
    torch.cuda.synchronize()
    oc = oracle_cache(k, v, Config(**{**base, "batch": 1, "capacity": 300}))
    want = oracle_decode(Config(**{**base, "batch": 1, "capacity": 300}), oc, q, [300])
    vmax = vmax_per_batch(oc[2], oc[3], Config(**{**base, "batch": 1, "capacity": 300}), [300])
    got = out.cpu().numpy()
    assert_close_to_oracle(got[:1], want, vmax, G, "seq 0")
    assert np.array_equal(got[0], got[1])
