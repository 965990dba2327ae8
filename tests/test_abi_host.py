"""C-ABI tests that need no GPU: symbols, byte formulas, host-side validation."""
import ctypes
import json
import os
import re

import pytest

import oracle
import quantized_kv_cache_22_b200 as kvq
from quantized_kv_cache_22_b200 import Config, KvqConfig, KvqLayer

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]*?\b(kvq_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 9
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(kvq.EXPORTED)


def test_status_strings():
    assert kvq.status_string(0) == "ok"
    for rc in range(-8, 0):
        assert kvq.status_string(rc) != "unknown status"


def _mib(x):
    return x / float(1 << 20)


@pytest.mark.parametrize("kb,vb,kg,vg,H,dh", [
    (8, 8, 128, 128, 16, 128), (16, 16, 0, 0, 16, 128), (8, 4, 128, 32, 8, 128),
    (4, 8, 32, 128, 8, 128), (4, 4, 32, 32, 4, 64), (8, 8, 64, 64, 4, 64), (4, 16, 64, 0, 2, 128)])
def test_cache_bytes_matches_oracle(kb, vb, kg, vg, H, dh):
    cfg = Config(batch=3, capacity=1024, n_q_heads=H, n_kv_heads=H, head_dim=dh, k_bits=kb,
                 v_bits=vb, k_group=kg, v_group=vg, n_layers=5)
    per_tok, per_layer, total = kvq.kvq_cache_bytes(cfg)
    want = oracle.bytes_per_token_layer(0, H, dh, kb, vb, kg or dh, vg or dh)
    assert per_tok == want
    assert per_layer == want * 3 * 1024
    assert total == per_layer * 5
    kc, ks, vc, vs = kvq.kvq_layer_buffer_bytes(cfg)
    assert kc + ks + vc + vs == per_layer


def test_cache_bytes_tinyloop_figures():
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "tinyloop_bytes.json")))
    b = g["bytes_per_token_per_layer"]
    kv = dict(batch=1, capacity=1024, n_q_heads=16, n_kv_heads=16, head_dim=128, n_layers=34)
    assert kvq.kvq_cache_bytes(Config(k_bits=16, v_bits=16, **kv))[0] == b["fp16_kv"]
    int8 = kvq.kvq_cache_bytes(Config(k_bits=8, v_bits=8, **kv))
    assert int8[0] == b["int8_kv"]
    assert round(_mib(int8[2])) == g["footprint"]["mib"]["int8_kv"]
    for name, bits in (("fp16_h", 16), ("int8_h", 8), ("int4_h", 4)):
        cfg = Config(batch=1, capacity=1024, mode=kvq.KVQ_MODE_H, d_model=2048, h_bits=bits,
                     h_groups=16, n_q_heads=16, n_kv_heads=16, head_dim=128, n_layers=34)
        assert kvq.kvq_cache_bytes(cfg)[0] == b[name]


def test_cache_bytes_kvsplit_figures():
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "kvsplit_mib.json")))
    for name, (kb, vb) in {"K8V8": (8, 8), "K8V4": (8, 4), "K4V4": (4, 4)}.items():
        cfg = Config(batch=1, capacity=g["tokens"], n_q_heads=32, n_kv_heads=g["n_kv_heads"],
                     head_dim=g["head_dim"], k_bits=kb, v_bits=vb, k_group=g["group"],
                     v_group=g["group"], n_layers=g["n_layers"])
        assert _mib(kvq.kvq_cache_bytes(cfg)[2]) == g["mib"][name]


def test_workspace_bytes_explicit_ctas_without_device():
    cfg = Config(batch=16, capacity=8192, n_q_heads=32, n_kv_heads=8, head_dim=128)
    a = kvq.kvq_workspace_bytes(cfg, num_ctas=296)
    b = kvq.kvq_workspace_bytes(cfg, num_ctas=300)
    # header + B*Hkv arrival counters (rounded up to 64) + (CTAs + B*Hkv)
    # partial slots of G*(Dh+4) floats
    assert a == 256 + 128 * 4 + (296 + 128) * 4 * 132 * 4
    assert b - a == 4 * 4 * 132 * 4


def _rc(fn, *args):
    return getattr(kvq.lib(), fn)(*args)


def test_validation_errors_are_returned_on_the_host():
    good = Config(batch=2, capacity=64, n_q_heads=4, n_kv_heads=2, head_dim=128).c()
    lay = KvqLayer(16, 16, 32, 48)
    P = ctypes.c_void_p
    # bad configs
    for field, val, want in (("capacity", 40, -2), ("head_dim", 96, -2), ("k_bits", 6, -2),
                             ("n_q_heads", 3, -1), ("batch", 0, -1), ("k_group", 48, -2),
                             ("mode", 7, -1), ("window", 100, -1), ("n_anchor", 4, -1),
                             ("window", -1, -1)):
        c = Config(batch=2, capacity=64, n_q_heads=4, n_kv_heads=2, head_dim=128).c()
        setattr(c, field, val)
        out = ctypes.c_uint64()
        assert _rc("kvq_cache_bytes", ctypes.byref(c), ctypes.byref(out), None, None) == want, field
    # append: capacity overflow, null input, misaligned pointer, bad dtype
    assert _rc("kvq_append", ctypes.byref(good), ctypes.byref(lay), P(16), P(32), 0, P(64), 60, 8,
               None) == -3
    assert _rc("kvq_append", ctypes.byref(good), ctypes.byref(lay), None, P(32), 0, P(64), 0, 1,
               None) == -1
    assert _rc("kvq_append", ctypes.byref(good), ctypes.byref(lay), P(17), P(32), 0, P(64), 0, 1,
               None) == -4
    assert _rc("kvq_append", ctypes.byref(good), ctypes.byref(lay), P(16), P(32), 9, P(64), 0, 1,
               None) == -1
    assert _rc("kvq_append", ctypes.byref(good), ctypes.byref(lay), P(16), P(32), 0, P(64), 0, 0,
               None) == 0   # zero tokens: nothing to do
    # decode: length beyond capacity, bad dtype, misaligned out, KV mode with h-mode args
    args = lambda **kw: [ctypes.byref(good), ctypes.byref(lay), kw.get("q", P(16)), kw.get("qd", 0),
                         P(64), kw.get("ml", 8), ctypes.c_float(0.0), kw.get("out", P(128)),
                         kw.get("od", 0), P(256), ctypes.c_uint64(1 << 20), 4, kw.get("w", None),
                         None, ctypes.c_uint64(0), None]
    assert _rc("kvq_decode_attn", *args(ml=65)) == -3
    assert _rc("kvq_decode_attn", *args(qd=5)) == -1
    assert _rc("kvq_decode_attn", *args(od=2)) == -1
    assert _rc("kvq_decode_attn", *args(out=P(130))) == -4
    assert _rc("kvq_decode_attn", *args(q=P(18))) == -4   # the kernels load queries 16 bytes at a time
    assert _rc("kvq_decode_attn", *args(w=P(512))) == -1
    assert _rc("kvq_decode_attn", *args(q=None)) == -1
    # h-mode reconstruction argument checks
    hc = Config(batch=1, capacity=64, mode=kvq.KVQ_MODE_H, d_model=256, h_bits=4, h_groups=2,
                n_q_heads=2, n_kv_heads=2, head_dim=128).c()
    hl = KvqLayer(16, 32, None, None)
    assert _rc("kvq_h_reconstruct", ctypes.byref(hc), ctypes.byref(hl), P(64), 65, P(128), P(256),
               128, P(512), ctypes.c_uint64(1 << 20), None) == -3
    assert _rc("kvq_h_reconstruct", ctypes.byref(hc), ctypes.byref(hl), P(64), 10, P(128), P(256),
               100, P(512), ctypes.c_uint64(1 << 20), None) == -1
    # operand scratch smaller than kvq_h_operand_bytes
    need = ctypes.c_uint64()
    assert _rc("kvq_h_operand_bytes", ctypes.byref(hc), 10, ctypes.byref(need)) == 0
    assert need.value == 1 * 128 * 256 * 2
    assert _rc("kvq_h_reconstruct", ctypes.byref(hc), ctypes.byref(hl), P(64), 10, P(128), P(256),
               64, P(512), ctypes.c_uint64(need.value - 16), None) == -5


def test_window_config_validation_and_bytes():
    # capacity must be n_anchor + window; the cache bytes are those of `capacity` slots
    ok = Config(batch=2, capacity=1600, n_q_heads=4, n_kv_heads=2, head_dim=128, k_bits=4,
                v_bits=8, k_group=32, v_group=128, window=1536, n_anchor=64)
    plain = Config(batch=2, capacity=1600, n_q_heads=4, n_kv_heads=2, head_dim=128, k_bits=4,
                   v_bits=8, k_group=32, v_group=128)
    assert kvq.kvq_cache_bytes(ok) == kvq.kvq_cache_bytes(plain)
    bad = Config(**{**ok.__dict__, "n_anchor": 63})
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(bad)
    assert e.value.status == -1
    h = Config(batch=1, capacity=64, mode=kvq.KVQ_MODE_H, d_model=2048, h_bits=4, h_groups=16,
               n_q_heads=16, n_kv_heads=16, head_dim=128, window=48, n_anchor=16)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(h)
    assert e.value.status == -2


def test_paged_config_validation_and_bytes():
    base = dict(batch=3, capacity=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, k_bits=8,
                v_bits=4, k_group=128, v_group=32)
    paged = Config(**base, page_tokens=128, n_pages=30)
    per_tok = kvq.kvq_cache_bytes(Config(**base))[0]
    t, layer, _ = kvq.kvq_cache_bytes(paged)
    assert t == per_tok and layer == per_tok * 30 * 128
    kc, ks, vc, vs = kvq.kvq_layer_buffer_bytes(paged)
    assert kc == 30 * 2 * 128 * 128 and ks == 30 * 2 * 128 * 2
    assert vc == 30 * 2 * 128 * 64 and vs == 30 * 2 * 128 * 4 * 2
    for over, want in (({"page_tokens": 64}, -2), ({"n_pages": 0}, -1), ({"capacity": 1040}, -1),
                       ({"window": 896, "n_anchor": 128}, -2)):
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_cache_bytes(Config(**{**paged.__dict__, **over}))
        assert e.value.status == want, over
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(Config(**base, n_pages=4))
    assert e.value.status == -1
    # a paged layer without a block table is rejected before anything runs
    lay = KvqLayer(16, 16, 32, 48, None)
    P = ctypes.c_void_p
    assert _rc("kvq_append", ctypes.byref(paged.c()), ctypes.byref(lay), P(16), P(32), 0, P(64),
               0, 1, None) == -1


def test_fp8_config_validation_and_bytes():
    # FP8 e4m3 codes take one byte per element like INT8: same cache bytes
    base = dict(batch=2, capacity=256, n_q_heads=8, n_kv_heads=2, head_dim=128, k_bits=8,
                v_bits=8, k_group=32, v_group=128)
    f8 = Config(**base, kv_format=kvq.KVQ_FMT_E4M3)
    assert kvq.kvq_cache_bytes(f8) == kvq.kvq_cache_bytes(Config(**base))
    assert kvq.kvq_layer_buffer_bytes(f8) == kvq.kvq_layer_buffer_bytes(Config(**base))
    for over, want in (({"k_bits": 4}, -2), ({"v_bits": 16}, -2), ({"kv_format": 4}, -1),
                       ({"kv_format": -1}, -1)):
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_cache_bytes(Config(**{**f8.__dict__, **over}))
        assert e.value.status == want, over
    h = Config(batch=1, capacity=64, mode=kvq.KVQ_MODE_H, d_model=2048, h_bits=4, h_groups=16,
               n_q_heads=16, n_kv_heads=16, head_dim=128, kv_format=kvq.KVQ_FMT_E4M3)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(h)
    assert e.value.status == -2


def test_asym_and_tensor_config_bytes_and_validation():
    base = dict(batch=2, capacity=256, n_q_heads=8, n_kv_heads=2, head_dim=128, k_bits=8,
                v_bits=8, k_group=32, v_group=128)
    sym = kvq.kvq_cache_bytes(Config(**base))[0]
    asym = Config(**base, kv_format=kvq.KVQ_FMT_ASYM)
    # a (scale, zero-point) pair per group: the scale bytes double
    scale_bytes = 2 * (128 // 32 + 128 // 128) * 2
    assert kvq.kvq_cache_bytes(asym)[0] == sym + scale_bytes
    kc, ks, vc, vs = kvq.kvq_layer_buffer_bytes(asym)
    assert ks == 2 * 256 * 2 * 4 * 2 * 2 and vs == 2 * 256 * 2 * 1 * 2 * 2
    tensor = Config(**{**base, "k_group": 0, "v_group": 0}, kv_format=kvq.KVQ_FMT_TENSOR)
    per_tok, layer, _ = kvq.kvq_cache_bytes(tensor)
    assert per_tok == 2 * 2 * 128 and layer == per_tok * 2 * 256 + 4
    assert kvq.kvq_layer_buffer_bytes(tensor) == (2 * 256 * 2 * 128, 2, 2 * 256 * 2 * 128, 2)
    for cfg, want in ((Config(**{**base, "k_bits": 4}, kv_format=kvq.KVQ_FMT_ASYM), -2),
                      (Config(**base, kv_format=kvq.KVQ_FMT_TENSOR), -2),      # grouped
                      (Config(**{**base, "v_bits": 16, "k_group": 0, "v_group": 0},
                              kv_format=kvq.KVQ_FMT_TENSOR), -2),
                      (Config(**base, kv_format=4), -1)):
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_cache_bytes(cfg)
        assert e.value.status == want


def test_absorbed_scratch_bytes_and_validation():
    cfg = Config(batch=8, capacity=1024, mode=kvq.KVQ_MODE_H, d_model=2048, h_bits=4, h_groups=16,
                 n_q_heads=16, n_kv_heads=16, head_dim=128)
    # q fragments B*(D/32)*NT*512 + factors B*ng*NT*8*4 + scores B*Hq*capP*4 + tile
    # statistics B*Hq*(capP/64)*8 + ob B*Hq*D*4 (the token splits add into one)
    want = (8 * 64 * 2 * 512 + 8 * 16 * 16 * 4 + 8 * 16 * 1024 * 4 + 8 * 16 * 16 * 8 +
            8 * 16 * 2048 * 4)
    assert kvq.kvq_h_absorbed_scratch_bytes(cfg, 1024) == want
    assert kvq.kvq_h_absorbed_scratch_bytes(cfg, 1000) == want
    for over, st in (({"h_bits": 16, "h_groups": 0}, -2), ({"n_q_heads": 64}, -2),
                     ({"n_kv_heads": 8}, -1)):
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_h_absorbed_scratch_bytes(Config(**{**cfg.__dict__, **over}), 1024)
        assert e.value.status == st, over
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_h_absorbed_scratch_bytes(cfg, 1025)
    assert e.value.status == -3
    kv = Config(batch=1, capacity=64, n_q_heads=4, n_kv_heads=4, head_dim=128)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_h_absorbed_scratch_bytes(kv, 64)
    assert e.value.status == -1


def test_fused_scratch_bytes_and_validation():
    cfg = Config(batch=8, capacity=1024, mode=kvq.KVQ_MODE_H, d_model=2048, h_bits=4, h_groups=16,
                 n_q_heads=16, n_kv_heads=16, head_dim=128)
    # header 256 + bf16 operand B*round_up(len,128)*D*2 + partials B*Hq*m_tiles*4*(Dh+2)*4
    assert kvq.kvq_h_fused_scratch_bytes(cfg, 1000) == 256 + 8 * 1024 * 2048 * 2 + 8 * 16 * 8 * 4 * 130 * 4
    for over, st in (({"n_q_heads": 256}, -2), ({"n_kv_heads": 8}, -1)):
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_h_fused_scratch_bytes(Config(**{**cfg.__dict__, **over}), 1024)
        assert e.value.status == st, over


def test_selftest_bounded_wait_argument_checks():
    P = ctypes.c_void_p
    f = kvq.lib().kvq_selftest_bounded_wait
    assert f(None, 1000, None) == -1                 # no workspace
    assert f(P(256), 0, None) == -1                  # no limit
    assert f(P(256), 3_000_000_000, None) == -1      # above 2 s
    assert f(P(8), 1000, None) == -4                 # not 16-byte aligned


def test_decode_plan_info_without_device(monkeypatch):
    # explicit CTA counts plan without a device: the warp-MMA kernel by default, two
    # CTAs per SM where a ring of two or more stages fits beside another CTA; the
    # tcgen05 kernel only when KVQ_DECODE_TC=1 and the format is one it takes
    def cfg(kb, vb, vg=128, dh=128):
        return Config(batch=16, capacity=8192, n_q_heads=32, n_kv_heads=8, head_dim=dh,
                      k_bits=kb, v_bits=vb, k_group=dh, v_group=vg if vb != 16 else dh)
    monkeypatch.delenv("KVQ_DECODE_TC", raising=False)
    # (16-bit keys and values: a two-stage ring of 64 KB tiles fits one CTA per SM)
    for kb, vb, per_sm in ((8, 8, 2), (8, 4, 2), (4, 4, 2), (4, 8, 2), (16, 16, 1)):
        info = kvq.kvq_decode_plan_info(cfg(kb, vb), 296)
        assert info["engine"] == kvq.KVQ_ENGINE_WARP_MMA and info["num_ctas"] == 296
        assert info["ctas_per_sm_planned"] == per_sm and info["threads"] == 192
        assert info["stages"] >= 2 and info["stage_bytes"] * info["stages"] < info["smem_bytes"]
        # the plan's shared memory leaves room for that many CTAs on a 228 KB SM (1 KB
        # reserved per CTA, 1 KB of static shared memory before the aligned dynamic part)
        assert per_sm * (info["smem_bytes"] + 1024 + 1024) <= 233472
    assert kvq.kvq_decode_plan_info(cfg(4, 4, vg=64, dh=64), 10)["ctas_per_sm_planned"] == 2
    # packed score columns for G <= 4 at head_dim 128 with INT4 / INT8 keys
    assert kvq.kvq_decode_plan_info(cfg(8, 4), 296)["packed_columns"] == 1
    assert kvq.kvq_decode_plan_info(cfg(4, 8, vg=32), 296)["packed_columns"] == 1
    assert kvq.kvq_decode_plan_info(cfg(16, 16), 296)["packed_columns"] == 0
    assert kvq.kvq_decode_plan_info(cfg(4, 4, vg=64, dh=64), 10)["packed_columns"] == 0
    f8 = Config(batch=16, capacity=8192, n_q_heads=32, n_kv_heads=8, head_dim=128, k_bits=8,
                v_bits=8, k_group=128, v_group=128, kv_format=kvq.KVQ_FMT_E4M3)
    assert kvq.kvq_decode_plan_info(f8, 296)["packed_columns"] == 1
    a8 = Config(**{**f8.__dict__, "kv_format": kvq.KVQ_FMT_ASYM})
    assert kvq.kvq_decode_plan_info(a8, 296)["packed_columns"] == 1
    a8g = Config(**{**a8.__dict__, "k_group": 32})   # grouped zero-points: unpacked
    assert kvq.kvq_decode_plan_info(a8g, 296)["packed_columns"] == 0
    g8 = Config(batch=2, capacity=256, n_q_heads=16, n_kv_heads=2, head_dim=128, k_bits=8, v_bits=8,
                k_group=128, v_group=128)
    assert kvq.kvq_decode_plan_info(g8, 10)["packed_columns"] == 0
    monkeypatch.setenv("KVQ_DECODE_TC", "1")
    for kb, vb in ((8, 8), (8, 4), (4, 4), (4, 8)):
        info = kvq.kvq_decode_plan_info(cfg(kb, vb), 296)
        assert info["engine"] == kvq.KVQ_ENGINE_TCGEN05 and info["stages"] >= 2
    # grouped value scales and 16-bit codes stay on the warp-MMA kernel
    assert kvq.kvq_decode_plan_info(cfg(8, 4, vg=32), 296)["engine"] == kvq.KVQ_ENGINE_WARP_MMA
    assert kvq.kvq_decode_plan_info(cfg(16, 16), 296)["engine"] == kvq.KVQ_ENGINE_WARP_MMA
    with pytest.raises(kvq.KvqError):
        kvq.kvq_decode_plan_info(cfg(8, 8), -1)
