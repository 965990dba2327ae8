"""The tcgen05 decode kernel (selected by KVQ_DECODE_TC=1) against the oracle.

The warp-MMA kernel serves every format by default, so the rest of the suite tests
that one.  Here the environment variable selects the tcgen05/TMEM kernel for the
formats it takes (head_dim 128, INT8 / INT4 codes, value scales per (token, head),
key scales per (token, head) or per 32/64-element group, per-tensor INT8), the plan
query confirms that it is the kernel launched, and its outputs meet the same bound,
2e-3 * max|V^| per sequence.  The last test reruns the decode parity modules as a
whole under the variable in a child process: formats the kernel does not take fall
back to the warp-MMA kernel there, the others run on tcgen05.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import quantized_kv_cache_22_b200 as kvq
from _helpers import (assert_close_to_oracle, gpu_cache, gpu_decode, oracle_cache, oracle_decode,
                      vmax_per_batch)
from quantized_kv_cache_22_b200 import Config

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (k_bits, v_bits, k_group, v_group): 0 = one scale per (token, head)
TC_FORMATS = [(8, 8, 0, 0), (8, 4, 0, 0), (4, 8, 0, 0), (4, 4, 0, 0), (8, 8, 32, 0),
              (4, 4, 64, 0), (8, 4, 32, 0)]


@pytest.fixture
def tc_engine(monkeypatch):
    monkeypatch.setenv("KVQ_DECODE_TC", "1")


def _cfg(B, cap, Hkv, G, fmt, dh=128):
    kb, vb, kg, vg = fmt
    return Config(batch=B, capacity=cap, n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=dh,
                  k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)


def _inputs(B, L, Hkv, G, dh, seed, scale_v=1.0, dtype=torch.float16):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, L, Hkv, dh, generator=g).to(dtype)
    v = (torch.randn(B, L, Hkv, dh, generator=g) * scale_v).to(dtype)
    q = torch.randn(B, Hkv * G, dh, generator=g).to(dtype)
    return k, v, q


def _check(cfg, k, v, q, lens, what, num_ctas=0, out_dtype=torch.float32):
    assert kvq.kvq_decode_plan_info(cfg, num_ctas)["engine"] == kvq.KVQ_ENGINE_TCGEN05, what
    cache = gpu_cache(cfg, k, v)
    oc = oracle_cache(k, v, cfg)
    want = oracle_decode(cfg, oc, q, lens)
    vmax = vmax_per_batch(oc[2], oc[3], cfg, lens)
    got = gpu_decode(cfg, cache, q, lens, num_ctas=num_ctas, out_dtype=out_dtype)
    assert_close_to_oracle(got, want, vmax, cfg.n_q_heads // cfg.n_kv_heads, what)
    return got, want, vmax


@pytest.mark.parametrize("fmt", TC_FORMATS)
@pytest.mark.parametrize("G", [1, 4, 8])
def test_tc_decode_matches_oracle(cuda_device, tc_engine, fmt, G):
    # several 128-token tiles, a one-token sequence and a ragged tail
    B, Hkv, cap = 3, 2, 384
    lens = [384, 1, 257]
    k, v, q = _inputs(B, cap, Hkv, G, 128, 7 + G + 3 * fmt[0] + fmt[1] + fmt[2])
    _check(_cfg(B, cap, Hkv, G, fmt), k, v, q, lens, f"{fmt} G={G}")


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
def test_tc_decode_f32_bf16_queries_and_f16_out(cuda_device, tc_engine, qdtype):
    B, Hkv, G, cap = 2, 2, 4, 256
    lens = [256, 130]
    k, v, _ = _inputs(B, cap, Hkv, G, 128, 61)
    q = torch.randn(B, Hkv * G, 128, generator=torch.Generator().manual_seed(62)).to(qdtype) * 3
    cfg = _cfg(B, cap, Hkv, G, (8, 4, 0, 0))
    _check(cfg, k, v, q, lens, str(qdtype))
    _check(cfg, k, v, q, lens, f"{qdtype} fp16 out", out_dtype=torch.float16)


def test_tc_decode_edge_lengths(cuda_device, tc_engine):
    # capacity 144: the last tile runs past it; lengths 0, 1, one tile +- 1, capacity
    B, Hkv, G, cap = 6, 1, 4, 144
    lens = [0, 1, 127, 128, 129, 144]
    k, v, q = _inputs(B, cap, Hkv, G, 128, 71)
    for fmt in ((8, 8, 0, 0), (4, 4, 0, 0), (8, 4, 32, 0)):
        got, _, _ = _check(_cfg(B, cap, Hkv, G, fmt), k, v, q, lens, str(fmt))
        assert np.all(got[0] == 0)


def test_tc_decode_split_count_invariance(cuda_device, tc_engine):
    # every split of the same work gives the oracle's result; the P.V sums are exact
    # integers per epoch, so splits differ only by the fp32 rounding of the merge
    B, Hkv, G, cap = 2, 2, 4, 2048
    lens = [2048, 1500]
    k, v, q = _inputs(B, cap, Hkv, G, 128, 73)
    cfg = _cfg(B, cap, Hkv, G, (4, 4, 0, 0))
    outs = []
    for n in (1, 2, 7, 19, 64, 0):
        got, _, vmax = _check(cfg, k, v, q, lens, f"num_ctas={n}", num_ctas=n)
        outs.append(got)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2.0 ** -16 * vmax.max()


def test_tc_decode_value_scale_range(cuda_device, tc_engine):
    # tiny and huge value magnitudes: P = 2^(s - m) * s_V stays inside its fixed point
    B, Hkv, G, cap = 2, 1, 4, 256
    for sv in (1e-4, 30.0):
        k, v, q = _inputs(B, cap, Hkv, G, 128, 79, scale_v=sv, dtype=torch.float32)
        _check(_cfg(B, cap, Hkv, G, (8, 8, 0, 0)), k, v, q.half(), [256, 100], str(sv))


def test_decode_parity_modules_under_tc_engine(cuda_device):
    mods = ["test_gpu_kv.py", "test_gpu_fused.py", "test_gpu_fused_full.py",
            "test_gpu_window.py", "test_gpu_paged.py", "test_gpu_int8_variants.py",
            "test_gpu_quant_edges.py", "test_gpu_bounds.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider"] + [os.path.join(ROOT, "tests", m) for m in mods],
                       capture_output=True, text=True, timeout=1200, cwd=ROOT,
                       env=dict(os.environ, KVQ_DECODE_TC="1"))
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
