"""Bounds evidence for the kernels' global-memory writes (in place of a memory checker).

Every buffer a call writes -- the cache (codes and scales, written by the append
kernel and by the decode kernel's producer warp), the workspace (status word,
arrival counters, split partials) and the output -- is placed between two 4 KiB
guard regions filled with a seeded byte pattern.  After the call the guards must
hold the same bytes: a write one element before or past any of these buffers would
change them.  Contiguous, sliding-window (ring wrap) and paged (shuffled block
table) caches, several code formats and CTA counts, and the noalloc entry point.
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace

pytestmark = pytest.mark.gpu

PAD = 4096


class Guarded:
    """A device buffer of `nbytes` between two PAD-byte guards of seeded bytes."""

    def __init__(self, nbytes: int, dtype, seed: int, zero: bool = False):
        nbytes = max(int(nbytes), 16)
        nbytes = (nbytes + 15) // 16 * 16
        g = torch.Generator().manual_seed(seed)
        host = torch.randint(0, 256, (nbytes + 2 * PAD,), generator=g, dtype=torch.uint8)
        if zero:
            host[PAD:PAD + nbytes] = 0
        self.full = host.cuda()
        self.guard = torch.cat([host[:PAD], host[PAD + nbytes:]])
        self.nbytes = nbytes
        self.view = self.full[PAD:PAD + nbytes].view(dtype)

    def check(self, what: str):
        torch.cuda.synchronize()
        f = self.full.cpu()
        now = torch.cat([f[:PAD], f[PAD + self.nbytes:]])
        bad = (now != self.guard).nonzero().flatten()
        assert bad.numel() == 0, f"{what}: {bad.numel()} guard bytes changed, first at {int(bad[0])}"


def _guarded_layer(cfg: Config, seed: int, block_table=None):
    layer = LayerCache.__new__(LayerCache)
    layer.cfg = cfg
    layer.block_table = block_table
    kc, ks, vc, vs = kvq.kvq_layer_buffer_bytes(cfg)
    guards = []
    for i, (name, nb, dt) in enumerate((("k_codes", kc, torch.uint8), ("k_scales", ks, torch.float16),
                                        ("v_codes", vc, torch.uint8), ("v_scales", vs, torch.float16))):
        if nb == 0:
            setattr(layer, name, None)
            continue
        # the interior starts zeroed: rows the test never appends hold code 0, scale 0
        gb = Guarded(nb, dt, seed + i, zero=True)
        setattr(layer, name, gb.view)
        guards.append((name, gb))
    return layer, guards


def _guarded_ws(cfg: Config, seed: int, num_ctas: int = 0):
    ws = Workspace.__new__(Workspace)
    ws.nbytes = kvq.kvq_workspace_bytes(cfg, num_ctas)
    gb = Guarded(ws.nbytes, torch.float32, seed, zero=True)
    ws.buf = gb.view
    return ws, gb


def _check_all(guards, what):
    for name, gb in guards:
        gb.check(f"{what} {name}")


FORMATS = [(8, 8, 128, 128, 0), (4, 4, 32, 32, 0), (8, 4, 128, 32, 0), (4, 8, 64, 128, 0),
           (16, 16, 128, 128, 0), (8, 8, 128, 128, kvq.KVQ_FMT_E4M3),
           (8, 8, 32, 128, kvq.KVQ_FMT_ASYM), (8, 8, 128, 128, kvq.KVQ_FMT_TENSOR)]


def _cfg(B, cap, Hkv, G, dh, fmt, **kw):
    kb, vb, kg, vg, kf = fmt
    return Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                  k_bits=kb, v_bits=vb, k_group=kg, v_group=vg, kv_format=kf, **kw)


def _set_tensor_scales(layer, cfg):
    if cfg.kv_format == kvq.KVQ_FMT_TENSOR:
        layer.k_scales[0] = 0.02
        layer.v_scales[0] = 0.02


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("num_ctas", [0, 7])
def test_append_and_fused_step_stay_in_bounds(cuda_device, fmt, num_ctas):
    lens = [640, 1, 257, 0, 639]
    B, Hkv, G, dh, cap = len(lens), 2, 4, 128, 640
    cfg = _cfg(B, cap, Hkv, G, dh, fmt)
    layer, guards = _guarded_layer(cfg, 11 + fmt[0] + fmt[1])
    _set_tensor_scales(layer, cfg)
    g = torch.Generator().manual_seed(3)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half().cuda()
    v = torch.randn(B, cap, Hkv, dh, generator=g).half().cuda()
    q = torch.randn(B, Hkv * G, dh, generator=g).half().cuda()
    # prefill all but the newest token; the last sequence's device position lies
    # above the host bound, so its rows past the capacity must be skipped
    pos = torch.tensor([0, 0, 0, 0, 5], dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, layer, k[:, :cap - 1].contiguous(), v[:, :cap - 1].contiguous(), pos, 1,
                   cap - 1)
    _check_all(guards, "append")
    ws, wg = _guarded_ws(cfg, 21, num_ctas)
    og = Guarded(B * Hkv * G * dh * 2, torch.float16, 31)
    out = og.view.view(B, Hkv * G, dh)
    idx = torch.tensor([max(L - 1, 0) for L in lens])
    k_new = k[torch.arange(B), idx].contiguous()
    v_new = v[torch.arange(B), idx].contiguous()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for _ in range(2):
        kvq.kvq_append_decode_attn(cfg, layer, k_new, v_new, q, d_len, max(lens), out, ws,
                                   num_ctas=num_ctas)
    _check_all(guards + [("workspace", wg), ("out", og)], "append_decode_attn")
    assert kvq.kvq_workspace_status(ws) == 0
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("fmt", [(4, 8, 32, 128, 0), (8, 8, 128, 128, kvq.KVQ_FMT_ASYM)])
def test_window_ring_wrap_stays_in_bounds(cuda_device, fmt):
    n_anchor, window = 64, 448
    lens = [100, 512, 513, 3000, 1]
    B, Hkv, G, dh = len(lens), 2, 4, 128
    cfg = _cfg(B, n_anchor + window, Hkv, G, dh, fmt, window=window, n_anchor=n_anchor)
    layer, guards = _guarded_layer(cfg, 41)
    g = torch.Generator().manual_seed(4)
    q = torch.randn(B, Hkv * G, dh, generator=g).half().cuda()
    ws, wg = _guarded_ws(cfg, 51)
    og = Guarded(B * Hkv * G * dh * 4, torch.float32, 61)
    out = og.view.view(B, Hkv * G, dh)
    # every sequence runs 40 decode steps from lens - 40 (ring slots wrap around)
    for step in range(40):
        d_len = torch.tensor([max(L - 39 + step, 1) for L in lens], dtype=torch.int32,
                             device="cuda")
        k_new = torch.randn(B, Hkv, dh, generator=g).half().cuda()
        v_new = torch.randn(B, Hkv, dh, generator=g).half().cuda()
        kvq.kvq_append_decode_attn(cfg, layer, k_new, v_new, q, d_len, max(lens) + 1, out, ws)
    # and a prefill that wraps the ring several times
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    kk = torch.randn(B, 1200, Hkv, dh, generator=g).half().cuda()
    kvq.kvq_append(cfg, layer, kk, kk, pos, 0, 1200)
    _check_all(guards + [("workspace", wg), ("out", og)], "window")
    assert kvq.kvq_workspace_status(ws) == 0


@pytest.mark.parametrize("fmt", [(8, 8, 128, 128, 0), (4, 4, 32, 32, 0)])
def test_paged_shuffled_table_stays_in_bounds(cuda_device, fmt):
    lens = [1000, 129, 513, 1024]
    B, Hkv, G, dh, cap = len(lens), 2, 4, 128, 1024
    n_pages = B * (cap // 128)
    cfg = _cfg(B, cap, Hkv, G, dh, fmt, page_tokens=128, n_pages=n_pages)
    g = torch.Generator().manual_seed(5)
    table = torch.randperm(n_pages, generator=g).view(B, -1).to(torch.int32).cuda()
    layer, guards = _guarded_layer(cfg, 71, block_table=table)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half().cuda()
    q = torch.randn(B, Hkv * G, dh, generator=g).half().cuda()
    kvq.kvq_append(cfg, layer, k[:, :cap - 1].contiguous(), k[:, :cap - 1].contiguous(),
                   torch.zeros(B, dtype=torch.int32, device="cuda"), 0, cap - 1)
    ws, wg = _guarded_ws(cfg, 81)
    og = Guarded(B * Hkv * G * dh * 2, torch.float16, 91)
    out = og.view.view(B, Hkv * G, dh)
    idx = torch.tensor([L - 1 for L in lens])
    k_new = k[torch.arange(B), idx].contiguous()
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    kvq.kvq_append_decode_attn(cfg, layer, k_new, k_new, q, d_len, max(lens), out, ws)
    _check_all(guards + [("workspace", wg), ("out", og)], "paged")
    assert kvq.kvq_workspace_status(ws) == 0


def test_noalloc_output_stays_in_bounds(cuda_device):
    lens = [512, 77, 300]
    B, Hkv, G, dh, cap = len(lens), 2, 4, 128, 512
    cfg = _cfg(B, cap, Hkv, G, dh, (8, 4, 128, 32, 0))
    layer, guards = _guarded_layer(cfg, 101)
    g = torch.Generator().manual_seed(6)
    k = torch.randn(B, cap, Hkv, dh, generator=g).half().cuda()
    q = torch.randn(B, Hkv * G, dh, generator=g).half().cuda()
    kvq.kvq_append(cfg, layer, k, k, torch.zeros(B, dtype=torch.int32, device="cuda"), 0, cap)
    og = Guarded(B * Hkv * G * dh * 4, torch.float32, 111)
    out = og.view.view(B, Hkv * G, dh)
    d_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for _ in range(2):
        kvq.kvq_decode_attn_noalloc(cfg, layer, q, d_len, max(lens), out)
    _check_all(guards + [("out", og)], "noalloc")
    assert kvq.kvq_noalloc_status() == 0
    assert np.isfinite(out.cpu().numpy()).all()
