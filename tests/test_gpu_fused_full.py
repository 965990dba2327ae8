"""Parity of the benchmarked call at the benchmark's own shape and launch configuration.

The decode step that the benchmark times is one kvq_append_decode_attn per layer
on the long-context workload: B=16 sequences, 32 query / 8 KV heads, head_dim 128,
8191 cached tokens plus the one appended by the call itself (8192 attended), fp16
queries and outputs, the default CTA count (a stream-K split over all SMs).  This
test runs that call once per KV format the benchmark reports and checks
  * the appended row of every (sequence, KV head) -- written by the decode
    kernel's producer warp -- bit for bit against the oracle quantiser;
  * the whole cache row range and the fp16 outputs of sampled (sequence, KV head)
    pairs against the oracle, within 2e-3 * max|V^| of that pair.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, LayerCache, Workspace, inputs
from _helpers import (assert_close_to_oracle, obits, oracle_cache, oracle_decode, read_gpu_cache,
                      to_np32, vmax_per_batch)

pytestmark = pytest.mark.gpu

# (k_bits, v_bits, kv_format): the benchmark's variants at per-(token, head) scales
VARIANTS = {"K8V8": (8, 8, 0), "K8V4": (8, 4, 0), "K4V4": (4, 4, 0),
            "F8": (8, 8, kvq.KVQ_FMT_E4M3), "A8": (8, 8, kvq.KVQ_FMT_ASYM),
            "T8": (8, 8, kvq.KVQ_FMT_TENSOR)}
PAIRS = [(0, 0), (7, 3), (15, 7), (10, 5)]


def _tensor_scale_bits(x: torch.Tensor) -> int:
    # a caller's calibration of a per-tensor INT8 scale: fp16(max|x| / 127)
    return int(np.float16(float(x.float().abs().max()) / 127.0).view(np.uint16))


@pytest.mark.parametrize("name", list(VARIANTS))
def test_benchmarked_step_at_full_size(cuda_device, name):
    kb, vb, kf = VARIANTS[name]
    w = inputs.WORKLOADS[4]
    layer = 1
    L, B, Hkv, dh = w.context, w.batch, w.n_kv_heads, w.head_dim
    G = w.n_q_heads // Hkv
    cfg = Config(batch=B, capacity=w.capacity, n_q_heads=w.n_q_heads, n_kv_heads=Hkv,
                 head_dim=dh, k_bits=kb, v_bits=vb, k_group=dh, v_group=dh, kv_format=kf)
    k, v = inputs.kv_tokens(w, layer, L - 1, "cuda")
    k1, v1 = inputs.kv_tokens(w, layer, 1, "cuda", offset_seed=1)
    cache = LayerCache(cfg)
    s16 = None
    if kf == kvq.KVQ_FMT_TENSOR:
        s16 = (_tensor_scale_bits(k), _tensor_scale_bits(v))
        for t, bits in ((cache.k_scales, s16[0]), (cache.v_scales, s16[1])):
            t.view(torch.int16)[0] = (bits ^ 0x8000) - 0x8000
    kvq.kvq_append(cfg, cache, k, v, torch.zeros(B, dtype=torch.int32, device="cuda"), 0, L - 1)
    q = inputs.queries(w, layer, 0, "cuda")
    d_len = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))                    # fp16, as the benchmark
    ws = Workspace(cfg)
    kvq.kvq_append_decode_attn(cfg, cache, k1[:, 0].contiguous(), v1[:, 0].contiguous(), q,
                               d_len, L, out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_workspace_status(ws) == 0
    gc = read_gpu_cache(cache, cfg)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()

    # every appended row: the decode kernel's producer quantised it into position L - 1
    one = Config(**{**cfg.__dict__, "capacity": 1})
    onew = oracle_cache(k1.cpu(), v1.cpu(), one, s16)
    for i, nm in enumerate(("k_codes", "k_scales", "v_codes", "v_scales")):
        assert np.array_equal(gc[i][:, :, L - 1], onew[i][:, :, 0]), nm

    # sampled pairs: all 8192 rows and the outputs of their G query heads
    sub = Config(**{**cfg.__dict__, "batch": 1, "n_kv_heads": 1, "n_q_heads": G})
    for b, kvh in PAIRS:
        kk = torch.cat([k[b:b + 1, :, kvh:kvh + 1], k1[b:b + 1, :, kvh:kvh + 1]], 1).cpu()
        vv = torch.cat([v[b:b + 1, :, kvh:kvh + 1], v1[b:b + 1, :, kvh:kvh + 1]], 1).cpu()
        oc = oracle_cache(kk, vv, sub, s16)
        for i in range(4):
            assert np.array_equal(gc[i][b, kvh], oc[i][0, 0]), (b, kvh, i)
        qq = q[b:b + 1, kvh * G:(kvh + 1) * G].cpu()
        want = oracle_decode(sub, oc, qq, [L])
        vmax = vmax_per_batch(oc[2], oc[3], sub, [L])
        assert_close_to_oracle(got[b:b + 1, kvh * G:(kvh + 1) * G], want, vmax, G,
                               f"{name} {(b, kvh)}")
