"""Shared helpers for the GPU parity tests: build the GPU cache through the C ABI,
build the oracle's own cache from the same raw inputs, compare."""
import numpy as np
import torch

import oracle
import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace

TOL = 2e-3   # max-abs error <= TOL * max|V^| (fp32 accumulation, fp16 output)


def to_np32(t):
    return t.detach().to("cpu").float().numpy()


def obits(cfg: Config, bits: int):
    """The oracle's bit-width argument for a cache width: "e4m3" / "asym8" for those
    8-bit formats (per-tensor INT8 codes are INT8 codes)."""
    if bits == 8 and cfg.kv_format == kvq.KVQ_FMT_E4M3:
        return "e4m3"
    if bits == 8 and cfg.kv_format == kvq.KVQ_FMT_ASYM:
        return "asym8"
    return bits


def oracle_cache(k, v, cfg: Config, tensor_s16=None):
    """k, v: [B, L, Hkv, dh] tensors -> oracle codes/scales in the cache layout [B, Hkv, cap, ...].
    Per-tensor INT8: tensor_s16 = (K scale, V scale) fp16 bits; the scales come back
    broadcast to one per (token, head), the per-head layout of the same values."""
    B, L, H, dh = k.shape
    cap = cfg.capacity
    out = []
    for i, (x, bits, grp) in enumerate(((k, cfg.k_bits, cfg.k_group or dh),
                                        (v, cfg.v_bits, cfg.v_group or dh))):
        xf = np.ascontiguousarray(to_np32(x).transpose(0, 2, 1, 3))   # [B, H, L, dh]
        if cfg.kv_format == kvq.KVQ_FMT_TENSOR:
            c = np.zeros((B, H, cap, dh), np.uint8)
            c[:, :, :L] = oracle.quantize_rows_tensor(xf, tensor_s16[i])
            out += [c, np.full((B, H, cap, 1), tensor_s16[i], np.uint16)]
            continue
        if bits == 16:
            c = np.zeros((B, H, cap, dh), np.float16)
            c[:, :, :L] = xf.astype(np.float16)
            out += [c.view(np.uint16), None]
        else:
            cc, ss = oracle.quantize_rows(xf, grp, obits(cfg, bits))
            c = np.zeros((B, H, cap, dh * bits // 8), np.uint8)
            s = np.zeros((B, H, cap) + ss.shape[3:], np.uint16)
            c[:, :, :L] = cc
            s[:, :, :L] = ss
            out += [c, s]
    return out


def gpu_cache(cfg: Config, k, v, device="cuda"):
    cache = LayerCache(cfg, device)
    B, L = k.shape[0], k.shape[1]
    pos = torch.zeros(B, dtype=torch.int32, device=device)
    kvq.kvq_append(cfg, cache, k.to(device).contiguous(), v.to(device).contiguous(), pos, 0, L)
    return cache


def read_gpu_cache(cache: LayerCache, cfg: Config):
    """The GPU cache as numpy arrays in the oracle_cache layout."""
    B, H, cap, dh = cfg.batch, cfg.n_kv_heads, cfg.capacity, cfg.head_dim
    res = []
    for codes, scales, bits, grp in ((cache.k_codes, cache.k_scales, cfg.k_bits, cfg.k_group or dh),
                                     (cache.v_codes, cache.v_scales, cfg.v_bits, cfg.v_group or dh)):
        c = codes.cpu().numpy()
        if bits == 16:
            res += [c[: B * H * cap * dh * 2].view(np.uint16).reshape(B, H, cap, dh), None]
            continue
        c = c[: B * H * cap * dh * bits // 8].reshape(B, H, cap, dh * bits // 8)
        sc = scales.cpu().numpy().view(np.uint16)
        if cfg.kv_format == kvq.KVQ_FMT_TENSOR:
            res += [c, np.full((B, H, cap, 1), sc[0], np.uint16)]
        elif cfg.kv_format == kvq.KVQ_FMT_ASYM:
            res += [c, sc[: B * H * cap * (dh // grp) * 2].reshape(B, H, cap, dh // grp, 2)]
        else:
            res += [c, sc[: B * H * cap * (dh // grp)].reshape(B, H, cap, dh // grp)]
    return res


def vmax_per_batch(vc, vs, cfg: Config, lens):
    """max |v^| per sequence over its attended tokens, from the oracle cache."""
    dh = cfg.head_dim
    out = []
    for b, L in enumerate(lens):
        if L == 0:
            out.append(1.0)
            continue
        vd = oracle.dequantize_rows(vc[b, :, :L], None if vs is None else vs[b, :, :L], dh,
                                    cfg.v_group or dh, obits(cfg, cfg.v_bits))
        out.append(float(np.abs(vd).max()))
    return np.array(out)


def gpu_decode(cfg: Config, cache, q, lens, out_dtype=torch.float32, num_ctas=0, scale=0.0):
    dev = cache.k_codes.device
    d_len = torch.tensor(lens, dtype=torch.int32, device=dev)
    out = torch.empty(q.shape, dtype=out_dtype, device=dev)
    ws = Workspace(cfg, num_ctas, dev)
    kvq.kvq_decode_attn(cfg, cache, q.to(dev).contiguous(), d_len, max(lens), out, ws,
                        softmax_scale=scale, num_ctas=num_ctas)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    return out.float().cpu().numpy()


def oracle_decode(cfg: Config, oc, q, lens, scale=0.0):
    kc, ks, vc, vs = oc
    return oracle.decode_layer(to_np32(q), np.array(lens, np.int32), kc, ks, obits(cfg, cfg.k_bits),
                               cfg.k_group or cfg.head_dim, vc, vs, obits(cfg, cfg.v_bits),
                               cfg.v_group or cfg.head_dim, cfg.n_kv_heads, scale)


def assert_close_to_oracle(got, want, vmax, G, what=""):
    """got/want [B, Hq, dh]; per-sequence bound TOL * max|V^|."""
    err = np.abs(got.astype(np.float64) - want).max(axis=(1, 2))
    bound = TOL * vmax
    assert np.all(err <= bound), f"{what}: err {err} bound {bound}"
    return float((err / bound).max())
