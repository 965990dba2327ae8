"""GPU parity of the symmetric INT8 / INT4 quantiser on constructed edge cases.

The TinyLoop mode table fixes only the level counts (255 levels for INT8, 15 for
INT4, one fp16 scale per head); the readings taken where it is silent are the
ones the oracle pins: scale = fp16(absmax / qmax) saturating at 65504 with
binary16 subnormals kept, codes by IEEE fp32 division and round-half-to-even,
an all-zero group giving scale 0 and codes 0.  Random N(0,1) data almost never
reaches those cases, so these rows are built to: all-zero groups, absmax that
saturates the scale, subnormal scales, exact ties x/s = k + 1/2 (also next to
+-qmax), mixed signs with a negative absmax.  The GPU quantiser must give the
oracle's codes and scales bit for bit, through kvq_append and through the
append fused into the decode kernel (kvq_append_decode_attn), per (token, head)
and per 32-element group.
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace
from _helpers import oracle_cache, read_gpu_cache

pytestmark = pytest.mark.gpu

DH = 128


def _edge_rows(bits: int, n_rows: int, seed: int) -> np.ndarray:
    """[n_rows, 128] fp32 rows, each of one edge kind, valid for per-head scales and
    for 32-element groups alike (every 32-element group holds its own absmax)."""
    qmax = 127 if bits == 8 else 7
    rng = np.random.default_rng(seed)
    rows = []
    kinds = ("zero", "zero_groups", "saturate", "subnormal", "ties_unit", "ties_quarter",
             "neg_absmax", "normal")
    for i in range(n_rows):
        kind = kinds[i % len(kinds)]
        x = np.zeros(DH, np.float32)
        if kind == "zero":
            pass
        elif kind == "zero_groups":
            # groups 1 and 3 all zero, groups 0 and 2 ordinary
            x[0:32] = rng.standard_normal(32)
            x[64:96] = rng.standard_normal(32) * 3
        elif kind == "saturate":
            # absmax / qmax > 65504: the fp16 scale saturates, codes clamp at +-qmax
            x[:] = rng.uniform(-5e6, 5e6, DH)
            x[::32] = 1e7 * rng.choice([-1.0, 1.0], DH // 32)
        elif kind == "subnormal":
            # absmax / qmax below 2^-14: the scale is a binary16 subnormal
            x[:] = rng.standard_normal(DH) * (2e-4 if bits == 8 else 2e-5)
        elif kind in ("ties_unit", "ties_quarter"):
            # s = fp32(absmax / qmax) is exactly 1 (or 1/4), so every x = s (k + 1/2) is an
            # exact tie; k reaches qmax - 1 (ties next to +-qmax) and 0 (+-1/2)
            s = 1.0 if kind == "ties_unit" else 0.25
            k = rng.integers(-qmax, qmax, DH)
            k[1::32] = qmax - 1
            k[2::32] = -qmax
            k[3::32] = 0
            k[4::32] = -1
            x[:] = (k + 0.5) * s
            x[::32] = qmax * s * rng.choice([-1.0, 1.0], DH // 32)
        elif kind == "neg_absmax":
            # mixed signs, the group's largest magnitude negative
            x[:] = rng.standard_normal(DH)
            x[::32] = -(np.abs(x).reshape(4, 32).max(1) + 0.75)
        else:
            x[:] = rng.standard_normal(DH) * 2
        rows.append(x)
    return np.stack(rows).astype(np.float32)


def _kv(bits_k, bits_v, B, L, Hkv, seed):
    n = B * L * Hkv
    k = _edge_rows(bits_k, n, seed).reshape(B, L, Hkv, DH)
    v = _edge_rows(bits_v, n, seed + 1).reshape(B, L, Hkv, DH)
    # shuffle the kinds over tokens so every tile and head sees all of them
    perm = np.random.default_rng(seed + 2).permutation(L)
    return torch.from_numpy(k[:, perm].copy()), torch.from_numpy(v[:, perm].copy())


FMTS = [(8, 8, 128, 128), (4, 4, 128, 128), (8, 4, 128, 32), (4, 8, 32, 128), (8, 8, 32, 32),
        (4, 4, 32, 32)]


@pytest.mark.parametrize("fmt", FMTS)
def test_edge_groups_append_bit_exact(cuda_device, fmt):
    kb, vb, kg, vg = fmt
    B, L, Hkv = 2, 48, 2
    k, v = _kv(kb, vb, B, L, Hkv, 300 + kb * 10 + vb + kg)
    cfg = Config(batch=B, capacity=64, n_q_heads=Hkv, n_kv_heads=Hkv, head_dim=DH,
                 k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)
    cache = LayerCache(cfg)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    kvq.kvq_append(cfg, cache, k.cuda(), v.cuda(), pos, 0, L)
    torch.cuda.synchronize()
    oc = oracle_cache(k, v, cfg)
    gc = read_gpu_cache(cache, cfg)
    for i, name in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        assert np.array_equal(gc[i][:, :, :L], oc[i][:, :, :L]), name
    # the edge kinds really occur in the oracle's scales
    for s in (oc[1], oc[3]):
        assert np.any(s == 0) and np.any(s == 0x7BFF) and np.any((s > 0) & (s < 0x0400))


@pytest.mark.parametrize("fmt", FMTS)
def test_edge_groups_fused_append_bit_exact(cuda_device, fmt):
    """Token by token through the decode kernel's fused append: after L steps the
    cache holds the oracle's codes and scales.  The outputs are only checked to be
    finite here: keys of 1e7 make the softmax one-hot, and the attention's accuracy
    is the business of the other parity tests."""
    kb, vb, kg, vg = fmt
    B, L, Hkv, G = 2, 40, 2, 4
    k, v = _kv(kb, vb, B, L, Hkv, 400 + kb * 10 + vb + kg)
    cfg = Config(batch=B, capacity=48, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=DH,
                 k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)
    cache = LayerCache(cfg, zero=True)
    ws = Workspace(cfg)
    q = torch.randn(B, Hkv * G, DH, generator=torch.Generator().manual_seed(kb + vb)).half()
    qd = q.cuda()
    d_len = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hkv * G, DH, dtype=torch.float32, device="cuda")
    oc = oracle_cache(k, v, cfg)
    for t in range(L):
        d_len.fill_(t + 1)
        kvq.kvq_append_decode_attn(cfg, cache, k[:, t].contiguous().cuda(),
                                   v[:, t].contiguous().cuda(), qd, d_len, t + 1, out, ws)
        if t % 8 == 7 or t == L - 1:
            assert torch.isfinite(out).all(), t
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    gc = read_gpu_cache(cache, cfg)
    for i, name in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        assert np.array_equal(gc[i][:, :, :L], oc[i][:, :, :L]), name
