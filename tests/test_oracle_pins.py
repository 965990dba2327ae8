"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-types the oracle's own formulas.  They use library routines
(numpy float16, torch bfloat16, numpy matmul, torch scaled_dot_product_attention),
closed forms, invariants, and the figures the pages print (tests/golden/).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MIB = float(1 << 20)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# number formats, pinned to library conversions
# ----------------------------------------------------------------------------

def _edge_floats():
    v = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e30, -1e30,
         2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -26, 6.1e-5, 1e-8, 1e-45,
         float("inf"), -float("inf")]
    # exact binary16 ties: halfway between neighbours at several binades
    for e in (-20, -14, -3, 0, 5, 14, 15):
        ulp = 2.0 ** (e - 10) if e >= -14 else 2.0 ** -24
        for k in (1024, 1025, 1500, 2046, 2047):
            base = k * ulp if e >= -14 else (k - 1024) * ulp
            v += [base + ulp / 2, -(base + ulp / 2)]
    return np.array(v, np.float32)


def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, size=60000, dtype=np.uint64).astype(np.uint32)
    vals = np.concatenate([bits.view(np.float32), _edge_floats(),
                           rng.standard_normal(20000).astype(np.float32) * 1e-5,
                           rng.standard_normal(20000).astype(np.float32) * 3e4])
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f32_to_f16_bits(x) for x in vals], np.uint16)
    nan = np.isnan(vals)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


def test_f64_to_f16_matches_numpy():
    rng = np.random.default_rng(12)
    vals = np.concatenate([rng.standard_normal(30000) * s for s in (1e-7, 1e-3, 1.0, 1e3, 7e4)])
    vals = np.concatenate([vals, _edge_floats().astype(np.float64),
                           np.array([1 + 2.0 ** -11 + 2.0 ** -40, 1 + 2.0 ** -11 - 2.0 ** -40])])
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f64_to_f16_bits(x) for x in vals], np.uint16)
    assert np.array_equal(got, ref)


def test_f16_to_f32_matches_numpy_all_codes():
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_bits_to_f32(int(c)) for c in codes], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_bf16_matches_torch():
    rng = np.random.default_rng(13)
    bits = rng.integers(0, 2 ** 32, size=50000, dtype=np.uint64).astype(np.uint32)
    vals = bits.view(np.float32)
    vals = vals[~np.isnan(vals)]
    ties = (np.arange(1, 3000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    vals = np.concatenate([vals, ties, -ties])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16_bits(x) for x in vals], np.uint16)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------------------
# quantiser
# ----------------------------------------------------------------------------

def _scale_f32(s_bits):
    return np.asarray(s_bits, np.uint16).view(np.float16).astype(np.float32)


def _signed_codes(codes, bits, dim):
    if bits == 8:
        return codes.view(np.int8).astype(np.int32)
    lo = (codes & 0xF).astype(np.int32)
    hi = (codes >> 4).astype(np.int32)
    out = np.empty(codes.shape[:-1] + (dim,), np.int32)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out)


@pytest.mark.parametrize("bits,group", [(8, 128), (8, 32), (4, 32), (4, 128), (8, 64)])
def test_quantizer_error_bound_and_code_range(bits, group):
    rng = np.random.default_rng(100 + bits + group)
    dim = 128
    mags = np.array([1e-3, 0.1, 1.0, 7.0, 300.0], np.float32)
    x = (rng.standard_normal((400, dim)).astype(np.float32)
         * mags[rng.integers(0, len(mags), 400)][:, None]).astype(np.float16).astype(np.float32)
    codes, scales = oracle.quantize_rows(x, group, bits)
    qmax = 127 if bits == 8 else 7
    c = _signed_codes(codes, bits, dim)
    s = np.repeat(_scale_f32(scales), group, axis=-1)
    assert np.all(np.abs(c) <= qmax)
    # error bound |x - c*s| <= s/2 (plus fp32 rounding of the quotient)
    err = np.abs(x.astype(np.float64) - c.astype(np.float64) * s.astype(np.float64))
    assert np.all(err <= s.astype(np.float64) * 0.5 * (1 + 2.0 ** -20))
    # the scale is the binary16 nearest to fp32(absmax / qmax) (numpy's conversion)
    a = np.abs(x).reshape(400, dim // group, group).max(-1)
    want = (a.astype(np.float32) / np.float32(qmax)).astype(np.float16).view(np.uint16)
    assert np.array_equal(scales, want)
    # the absmax element of every group maps to +-qmax (normal-range scales)
    xg = x.reshape(400, dim // group, group)
    cg = c.reshape(400, dim // group, group)
    idx = np.abs(xg).argmax(-1)
    top = np.take_along_axis(cg, idx[..., None], -1)[..., 0]
    normal = _scale_f32(scales) >= 2.0 ** -14
    assert np.all(np.abs(top[normal]) == qmax)


def test_quantizer_ties_round_half_even_int8():
    # absmax 127 gives s32 = 1.0 exactly, s16 = 1.0: codes are rne(x)
    x = np.zeros((1, 32), np.float32)
    x[0, :10] = [127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 126.5, -1.5]
    codes, scales = oracle.quantize_rows(x, 32, 8)
    assert scales[0, 0] == 0x3C00
    c = codes.view(np.int8)[0, :10].tolist()
    assert c == [127, 2, 4, -2, -4, 0, 2, 0, 126, -2]


def test_quantizer_ties_round_half_even_int4_and_nibble_order():
    x = np.zeros((1, 32), np.float32)
    x[0, :8] = [7, 2.5, -0.5, 6.5, 1, -2, -7, 5.5]
    codes, scales = oracle.quantize_rows(x, 32, 4)
    assert scales[0, 0] == 0x3C00
    # codes 7, 2, 0, 6, 1, -2, -7, 6 ; element 2j low nibble, 2j+1 high nibble
    assert codes[0, :4].tolist() == [0x27, 0x60, 0xE1, 0x69]


def test_quantizer_zero_group_and_saturation_and_subnormal():
    x = np.zeros((3, 32), np.float32)
    x[1, 0] = 1e7          # absmax/127 > 65504: scale saturates to 65504
    x[1, 1] = -5e6
    x[2, 0] = 1e-5         # scale is a binary16 subnormal
    x[2, 1] = -3e-6
    codes, scales = oracle.quantize_rows(x, 32, 8)
    assert scales[0, 0] == 0 and np.all(codes[0] == 0)
    assert scales[1, 0] == 0x7BFF
    c = codes.view(np.int8)
    assert c[1, 0] == 127 and c[1, 1] == -76          # 5e6/65504 = 76.3
    assert 0 < scales[2, 0] < 0x0400                  # subnormal scale kept
    assert c[2, 0] == 127                              # clamped


def test_quantizer_idempotent_when_a_code_reaches_qmax():
    rng = np.random.default_rng(7)
    for bits, group in ((8, 128), (4, 32), (8, 32)):
        x = rng.standard_normal((64, 128)).astype(np.float16).astype(np.float32)
        codes, scales = oracle.quantize_rows(x, group, bits)
        xr = oracle.dequantize_rows(codes, scales, 128, group, bits).astype(np.float32)
        codes2, scales2 = oracle.quantize_rows(xr, group, bits)
        assert np.array_equal(codes, codes2) and np.array_equal(scales, scales2)


def test_dequantize_is_exact_product():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    codes, scales = oracle.quantize_rows(x, 32, 4)
    xr = oracle.dequantize_rows(codes, scales, 128, 32, 4)
    c = _signed_codes(codes, 4, 128).astype(np.float64)
    s = np.repeat(_scale_f32(scales).astype(np.float64), 32, axis=-1)
    assert np.array_equal(xr, c * s)


# ----------------------------------------------------------------------------
# attention: closed forms, invariants, library cross-check
# ----------------------------------------------------------------------------

def _cache(k, v, kb, vb, kg, vg):
    """k, v: [B, Hkv, L, dh] float32 -> oracle cache arrays in the ABI layout."""
    def q(x, bits, g):
        if bits == 16:
            return x.astype(np.float16).view(np.uint16), None
        return oracle.quantize_rows(x, g, bits)
    kc, ks = q(k, kb, kg)
    vc, vs = q(v, vb, vg)
    return kc, ks, vc, vs


def _deq(c, s, bits, g, dh):
    if bits == 16:
        return c.view(np.float16).astype(np.float64)
    return oracle.dequantize_rows(c, s, dh, g, bits)


def _run(q, lens, k, v, kb=8, vb=8, kg=None, vg=None, tau=0.0):
    B, Hkv, L, dh = k.shape
    kg = kg or dh
    vg = vg or dh
    kc, ks, vc, vs = _cache(k, v, kb, vb, kg, vg)
    out = oracle.decode_layer(q, lens, kc, ks, kb, kg, vc, vs, vb, vg, Hkv, tau)
    return out, _deq(kc, ks, kb, kg, dh), _deq(vc, vs, vb, vg, dh)


@pytest.mark.parametrize("kb,vb", [(8, 8), (4, 8), (8, 4), (16, 16)])
def test_single_token_returns_its_value(kb, vb):
    rng = np.random.default_rng(20)
    k = rng.standard_normal((2, 3, 1, 64)).astype(np.float32)
    v = rng.standard_normal((2, 3, 1, 64)).astype(np.float32)
    q = rng.standard_normal((2, 6, 64)).astype(np.float32)
    out, _, vh = _run(q, np.array([1, 1], np.int32), k, v, kb, vb, 32, 32)
    for h in range(6):
        assert np.array_equal(out[:, h], vh[:, h // 2, 0])


def test_zero_query_returns_mean_of_values():
    rng = np.random.default_rng(21)
    k = rng.standard_normal((1, 2, 37, 128)).astype(np.float32)
    v = rng.standard_normal((1, 2, 37, 128)).astype(np.float32)
    q = np.zeros((1, 2, 128), np.float32)
    out, _, vh = _run(q, np.array([37], np.int32), k, v, 8, 4, 128, 32)
    np.testing.assert_allclose(out[0], vh[0].mean(axis=1), rtol=0, atol=1e-13)


def test_equal_keys_return_mean_of_values():
    rng = np.random.default_rng(22)
    row = rng.standard_normal(64).astype(np.float32)
    k = np.broadcast_to(row, (1, 1, 50, 64)).copy()
    v = rng.standard_normal((1, 1, 50, 64)).astype(np.float32)
    q = rng.standard_normal((1, 1, 64)).astype(np.float32) * 5
    out, _, vh = _run(q, np.array([50], np.int32), k, v)
    np.testing.assert_allclose(out[0, 0], vh[0, 0].mean(axis=0), rtol=0, atol=1e-13)


def test_two_tokens_closed_form_with_softmax_scale():
    # out = v0 + (v1 - v0) * logistic(tau * (q.k1 - q.k0)); catches a missing or wrong tau
    rng = np.random.default_rng(23)
    k = rng.standard_normal((1, 1, 2, 64)).astype(np.float32)
    v = rng.standard_normal((1, 1, 2, 64)).astype(np.float32)
    q = rng.standard_normal((1, 1, 64)).astype(np.float32)
    for tau in (0.0, 0.37):
        out, kh, vh = _run(q, np.array([2], np.int32), k, v, 8, 8, tau=tau)
        t = tau if tau > 0 else 1 / math.sqrt(64)
        d = t * (q[0, 0].astype(np.float64) @ (kh[0, 0, 1] - kh[0, 0, 0]))
        w = 1.0 / (1.0 + math.exp(-d))
        np.testing.assert_allclose(out[0, 0], vh[0, 0, 0] + (vh[0, 0, 1] - vh[0, 0, 0]) * w,
                                   rtol=0, atol=1e-13)


def test_dominant_key_returns_its_value():
    rng = np.random.default_rng(24)
    L = 200
    k = rng.standard_normal((1, 1, L, 128)).astype(np.float32) * 0.01
    k[0, 0, 77] = 1.0
    v = rng.standard_normal((1, 1, L, 128)).astype(np.float32)
    q = np.full((1, 1, 128), 60.0, np.float32)
    out, _, vh = _run(q, np.array([L], np.int32), k, v)
    np.testing.assert_allclose(out[0, 0], vh[0, 0, 77], rtol=0, atol=1e-12)


def test_gqa_query_head_reads_kv_head_floor_h_over_g():
    # value heads are constant per KV head; q = 0 averages, so out[h] names its KV head
    Hkv, G, L = 3, 4, 9
    k = np.random.default_rng(25).standard_normal((1, Hkv, L, 64)).astype(np.float32)
    v = np.zeros((1, Hkv, L, 64), np.float32)
    for j in range(Hkv):
        v[0, j] = j + 1
    q = np.zeros((1, Hkv * G, 64), np.float32)
    out, _, vh = _run(q, np.array([L], np.int32), k, v)
    for h in range(Hkv * G):
        np.testing.assert_allclose(out[0, h], vh[0, h // G, 0], rtol=0, atol=1e-12)
        assert abs(out[0, h, 0] - (h // G + 1)) < 0.01


def test_replicated_kv_heads_equal_shared_head():
    rng = np.random.default_rng(26)
    k = rng.standard_normal((1, 1, 40, 64)).astype(np.float32)
    v = rng.standard_normal((1, 1, 40, 64)).astype(np.float32)
    q = rng.standard_normal((1, 4, 64)).astype(np.float32)
    shared, _, _ = _run(q, np.array([40], np.int32), k, v, 4, 8, 32, 64)
    rep, _, _ = _run(q, np.array([40], np.int32), np.repeat(k, 4, 1), np.repeat(v, 4, 1), 4, 8, 32, 64)
    np.testing.assert_allclose(shared, rep, rtol=0, atol=1e-14)


def test_token_permutation_and_duplication_invariance():
    rng = np.random.default_rng(27)
    L = 33
    k = rng.standard_normal((1, 2, L, 64)).astype(np.float32)
    v = rng.standard_normal((1, 2, L, 64)).astype(np.float32)
    q = rng.standard_normal((1, 2, 64)).astype(np.float32)
    base, _, _ = _run(q, np.array([L], np.int32), k, v, 8, 4, 64, 32)
    perm = rng.permutation(L)
    p, _, _ = _run(q, np.array([L], np.int32), k[:, :, perm], v[:, :, perm], 8, 4, 64, 32)
    dup, _, _ = _run(q, np.array([2 * L], np.int32), np.concatenate([k, k], 2),
                     np.concatenate([v, v], 2), 8, 4, 64, 32)
    np.testing.assert_allclose(p, base, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dup, base, rtol=0, atol=1e-13)


def test_lengths_truncate_and_empty_sequence_is_zero():
    rng = np.random.default_rng(28)
    k = rng.standard_normal((2, 1, 20, 64)).astype(np.float32)
    v = rng.standard_normal((2, 1, 20, 64)).astype(np.float32)
    q = rng.standard_normal((2, 1, 64)).astype(np.float32)
    out, _, _ = _run(q, np.array([0, 7], np.int32), k, v)
    assert np.all(out[0] == 0)
    short, _, _ = _run(q[1:], np.array([7], np.int32), k[1:, :, :7], v[1:, :, :7])
    np.testing.assert_allclose(out[1], short[0], rtol=0, atol=1e-14)


def test_16bit_mode_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(29)
    B, Hkv, G, L, dh = 2, 2, 3, 45, 128
    k = rng.standard_normal((B, Hkv, L, dh)).astype(np.float16).astype(np.float32)
    v = rng.standard_normal((B, Hkv, L, dh)).astype(np.float16).astype(np.float32)
    q = rng.standard_normal((B, Hkv * G, dh)).astype(np.float32)
    out, _, _ = _run(q, np.array([L, L], np.int32), k, v, 16, 16)
    kk = torch.from_numpy(np.repeat(k, G, 1)).double()
    vv = torch.from_numpy(np.repeat(v, G, 1)).double()
    qq = torch.from_numpy(q).double()[:, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, :, 0].numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# h-mode reconstruction
# ----------------------------------------------------------------------------

def _h_setup(n_tok=48, D=512, N=256, seed=30):
    rng = np.random.default_rng(seed)
    r = rng.standard_normal((n_tok, D))
    h = ((r - r.mean(-1, keepdims=True)) / np.sqrt(r.var(-1, keepdims=True) + 1e-5)).astype(np.float16)
    W = torch.from_numpy(rng.standard_normal((N, D)) / math.sqrt(D)).float().to(torch.bfloat16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    return h, Wb, W.double().numpy()


def test_h_reconstruct_fp16_h_equals_matmul():
    h, Wb, W = _h_setup()
    y64, y16 = oracle.h_reconstruct(h.view(np.uint16), None, 512, 4, 16, Wb, round_bf16=False)
    ref = h.astype(np.float64) @ W.T
    np.testing.assert_allclose(y64, ref, rtol=1e-13, atol=1e-13)
    assert np.array_equal(y16, ref.astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("bits,lo,hi", [(8, 0.003, 0.012), (4, 0.05, 0.20)])
def test_h_quantized_kv_error_band(bits, lo, hi):
    # TinyLoop docs, mode table: INT8-h K/V relative L2 error ~0.6 %, INT4-h ~10 %
    h, Wb, W = _h_setup(n_tok=64, D=2048, N=512, seed=31)
    groups = 16
    codes, scales = oracle.quantize_rows(h.astype(np.float32), 2048 // groups, bits)
    y64, _ = oracle.h_reconstruct(codes, scales, 2048, groups, bits, Wb, round_bf16=False)
    ref = h.astype(np.float64) @ W.T
    rel = np.linalg.norm(y64 - ref) / np.linalg.norm(ref)
    assert lo < rel < hi, rel


# ----------------------------------------------------------------------------
# bytes per token per layer: the printed figures
# ----------------------------------------------------------------------------

def test_tinyloop_bytes_per_token_layer():
    g = _golden("tinyloop_bytes.json")
    D, H = g["d_model"], g["n_heads"]
    dh = D // H
    b = g["bytes_per_token_per_layer"]
    assert oracle.bytes_per_token_layer(0, H, dh, 16, 16) == b["fp16_kv"]
    assert oracle.bytes_per_token_layer(0, H, dh, 8, 8, dh, dh) == b["int8_kv"]
    assert oracle.bytes_per_token_layer(1, d_model=D, h_bits=16, h_groups=H) == b["fp16_h"]
    assert oracle.bytes_per_token_layer(1, d_model=D, h_bits=8, h_groups=H) == b["int8_h"]
    assert oracle.bytes_per_token_layer(1, d_model=D, h_bits=4, h_groups=H) == b["int4_h"]
    fp = g["footprint"]
    n = fp["n_layers"] * fp["max_seq_len"]
    assert round(b["fp16_kv"] * n / MIB) == fp["mib"]["fp16_kv"]
    assert round(b["int8_kv"] * n / MIB) == fp["mib"]["int8_kv"]
    assert round(b["fp16_h"] * n / MIB) == fp["mib"]["fp16_h"]
    assert round(1 - b["int4_h"] / b["fp16_kv"], 2) == g["h_limit"]["saving"]


def test_kvsplit_mib_at_8k_tokens():
    g = _golden("kvsplit_mib.json")
    n = g["n_layers"] * g["tokens"]
    H, dh, grp = g["n_kv_heads"], g["head_dim"], g["group"]
    assert oracle.bytes_per_token_layer(0, H, dh, 16, 16) * n / MIB == g["mib"]["fp16"]
    for name, (kb, vb) in {"K8V8": (8, 8), "K8V4": (8, 4), "K4V4": (4, 4)}.items():
        got = oracle.bytes_per_token_layer(0, H, dh, kb, vb, grp, grp) * n / MIB
        assert got == g["mib"][name], (name, got)


def test_ondevice_mib_k4v8_codes():
    g = _golden("ondevice_mib.json")
    n = g["n_layers"] * g["tokens"]
    H, dh = g["n_kv_heads"], g["head_dim"]
    assert oracle.bytes_per_token_layer(0, H, dh, 16, 16) * n / MIB == g["mib"]["fp16"]
    with_scales = oracle.bytes_per_token_layer(0, H, dh, 4, 8, dh, dh)
    codes_only = with_scales - 2 * H * 2          # one fp16 scale per head per tensor
    assert codes_only * n / MIB == g["mib"]["K4V8_codes"]
    assert round(1 - g["mib"]["K4V8_codes"] / g["mib"]["fp16"], 2) in (0.62, 0.63)


def test_h_reconstruct_rounds_operand_to_bf16():
    # the GEMM operand is bf16(h^): pinned against torch's bfloat16 conversion
    h, Wb, W = _h_setup(n_tok=32, D=512, N=128, seed=32)
    codes, scales = oracle.quantize_rows(h.astype(np.float32), 128, 4)
    hd = oracle.dequantize_rows(codes, scales, 512, 128, 4)
    hb = torch.from_numpy(hd).float().to(torch.bfloat16).double().numpy()
    assert not np.array_equal(hb, hd)
    y64, y16 = oracle.h_reconstruct(codes, scales, 512, 4, 4, Wb, round_bf16=True)
    ref = hb @ W.T
    np.testing.assert_allclose(y64, ref, rtol=1e-13, atol=1e-13)
    assert np.array_equal(y16, ref.astype(np.float16).view(np.uint16))


# --- FP8 e4m3 codes ------------------------------------------------------------

def test_e4m3_decode_matches_torch_for_every_code():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    want = codes.view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_to_f32(c) for c in range(256)], np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2   # 0x7f, 0xff
    assert np.array_equal(got[~nan], want[~nan])
    assert oracle.e4m3_to_f32(0x7e) == 448.0 and oracle.e4m3_to_f32(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_torch_rounding():
    # every representable value, every midpoint between neighbours (ties), values
    # just off the midpoints, random magnitudes over the whole range, saturation
    vals = np.array([oracle.e4m3_to_f32(c) for c in range(0x7f)], np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(4)
    x = np.concatenate([vals, mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20),
                        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(600.0), 4000)),
                        [448.0, 460.0, 464.0, 470.0, 1e6, 2.0 ** -10, 2.0 ** -10 * 1.01]])
    x = np.concatenate([x, -x]).astype(np.float32)
    want = torch.from_numpy(np.clip(x, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8)
    got = np.array([oracle.f32_to_e4m3(v) for v in x], np.uint8)
    assert np.array_equal(got, want.numpy())


def test_e4m3_quantiser_scale_codes_and_error_bound():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 128)) * rng.uniform(0.01, 50, (64, 1))).astype(np.float32)
    x[3] = 0.0
    for group in (32, 128):
        codes, scales = oracle.quantize_rows(x, group, "e4m3")
        assert codes.shape == (64, 128) and scales.shape == (64, 128 // group)
        g = x.reshape(64, -1, group)
        amax = np.abs(g).max(-1)
        want_s = (amax / np.float32(448.0)).astype(np.float32).astype(np.float16).view(np.uint16)
        assert np.array_equal(scales, want_s)
        assert np.all(codes[3] == 0)
        s = scales.view(np.float16).astype(np.float64)
        xhat = oracle.dequantize_rows(codes, scales, 128, group, "e4m3").reshape(64, -1, group)
        y = g / np.where(s == 0, 1, s)[..., None]
        # half a unit in the last place of e4m3 at |x / s| (normal range: 2^(e-4)),
        # never below half the smallest subnormal
        e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6)))
        bound = np.maximum(2.0 ** (e - 4), 2.0 ** -10) * s[..., None]
        assert np.all(np.abs(xhat - g) <= bound * (1 + 1e-6))
        # the largest element lands within one step of 448
        top = np.abs(xhat).max(-1)
        ok = amax > 0
        assert np.all(np.abs(top[ok] / s[ok] - 448) <= 32)


def test_e4m3_decode_layer_matches_dequantised_attention():
    rng = np.random.default_rng(6)
    B, H, G, L, dh = 2, 2, 2, 40, 64
    k = rng.standard_normal((B, H, L, dh)).astype(np.float32)
    v = rng.standard_normal((B, H, L, dh)).astype(np.float32)
    q = rng.standard_normal((B, H * G, dh)).astype(np.float32)
    kc, ks = oracle.quantize_rows(k, 32, "e4m3")
    vc, vs = oracle.quantize_rows(v, 64, "e4m3")
    got = oracle.decode_layer(q, np.array([L, 17], np.int32), kc, ks, "e4m3", 32, vc, vs, "e4m3", 64, H)
    kd = oracle.dequantize_rows(kc, ks, dh, 32, "e4m3")
    vd = oracle.dequantize_rows(vc, vs, dh, 64, "e4m3")
    for b, n in ((0, L), (1, 17)):
        for h in range(H * G):
            want = oracle.attend(q[b, h], kd[b, h // G, :n], vd[b, h // G, :n], 1 / np.sqrt(dh))
            assert np.allclose(got[b, h], want, rtol=0, atol=1e-12)


# --- asymmetric INT8 (zero-point) and per-tensor INT8 ----------------------------

def _asym(x, group):
    codes, sz = oracle.quantize_rows(x, group, "asym8")
    return codes, sz[..., 0], sz[..., 1]


def test_asym8_arithmetic_progression_closed_form():
    # x_i = (i - 100) / 4, i = 0..255: lo = -25, hi = 38.75, s = 63.75 / 255 = 1/4 exactly,
    # z = 100 and q_i = i
    x = ((np.arange(256) - 100) / 4.0).astype(np.float32)[None]
    codes, s, z = _asym(x, 256)
    assert np.array_equal(codes[0], np.arange(256))
    assert s[0, 0] == np.float16(0.25).view(np.uint16) and z[0, 0] == np.float16(100).view(np.uint16)
    # shuffled order, same codes per element
    perm = np.random.default_rng(0).permutation(256)
    c2, _, _ = _asym(np.ascontiguousarray(x[:, perm]), 256)
    assert np.array_equal(c2[0], perm)


def test_asym8_one_sided_groups_and_zero_group():
    rng = np.random.default_rng(1)
    pos = rng.uniform(0.5, 3.0, (4, 64)).astype(np.float32)
    c, s, z = _asym(pos, 64)
    assert np.all(z == 0) and np.all(c.max(-1) >= 254)          # lo = 0: the max near 255
    c, s, z = _asym(-pos, 64)
    assert np.all(z == np.float16(255).view(np.uint16)) and np.all(c.min(-1) <= 1)
    c, s, z = _asym(np.zeros((2, 64), np.float32), 32)
    assert not c.any() and not s.any() and not z.any()


@pytest.mark.parametrize("group", [32, 64, 128])
def test_asym8_error_bound_and_exact_zero(group):
    rng = np.random.default_rng(2 + group)
    x = (rng.standard_normal((96, 128)) * rng.uniform(0.01, 40, (96, 1))
         + rng.uniform(-30, 30, (96, 1))).astype(np.float32)
    x[5, :: 7] = 0.0
    codes, sz = oracle.quantize_rows(x, group, "asym8")
    xhat = oracle.dequantize_rows(codes, sz, 128, group, "asym8")
    s = sz[..., 0].view(np.float16).astype(np.float64)
    srow = np.repeat(s, group, axis=-1)
    # unclipped: |x - x^| <= s/2; fp16 rounding of s can clip the ends by at most 1/8 step
    assert np.all(np.abs(xhat - x) <= 0.625 * srow * (1 + 1e-6))
    assert np.all(xhat[5, ::7] == 0.0)
    zr = sz[..., 1].view(np.float16).astype(np.float64)
    assert np.all(zr == np.round(zr)) and zr.min() >= 0 and zr.max() <= 255


def test_asym8_codes_match_torch_affine_quantiser():
    """torch.quantize_per_tensor (quint8, the oracle's own scale and zero-point per
    group) computes the same codes, up to one step where x / s sits on a tie (torch
    multiplies by 1/s)."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 128)) * 3 + 1).astype(np.float32)
    codes, s, z = _asym(x, 32)
    n_eq = 0
    for r in range(64):
        for g in range(4):
            sc = float(s[r, g:g + 1].view(np.float16)[0])
            zp = int(z[r, g:g + 1].view(np.float16)[0])
            t = torch.quantize_per_tensor(torch.from_numpy(x[r, 32 * g:32 * g + 32].copy()), sc, zp,
                                          torch.quint8).int_repr().numpy()
            d = np.abs(t.astype(int) - codes[r, 32 * g:32 * g + 32].astype(int))
            assert d.max() <= 1
            n_eq += int((d == 0).sum())
    assert n_eq >= 0.99 * x.size


def test_asym8_decode_with_zero_point_128_equals_symmetric_codes():
    # symmetric int8 codes c with scale s are the asymmetric codes c + 128 with (s, 128)
    rng = np.random.default_rng(7)
    B, H, G, L, dh = 2, 2, 2, 33, 64
    k = rng.standard_normal((B, H, L, dh)).astype(np.float32)
    v = rng.standard_normal((B, H, L, dh)).astype(np.float32)
    q = rng.standard_normal((B, H * G, dh)).astype(np.float32)
    kc, ks = oracle.quantize_rows(k, 64, 8)
    vc, vs = oracle.quantize_rows(v, 32, 8)
    z128 = np.float16(128).view(np.uint16)

    def to_asym(c, s):
        pairs = np.stack([s, np.full_like(s, z128)], -1)
        return (c.view(np.int8).astype(np.int16) + 128).astype(np.uint8), pairs

    kca, ksa = to_asym(kc, ks)
    vca, vsa = to_asym(vc, vs)
    lens = np.array([L, 9], np.int32)
    want = oracle.decode_layer(q, lens, kc, ks, 8, 64, vc, vs, 8, 32, H)
    got = oracle.decode_layer(q, lens, kca, ksa, "asym8", 64, vca, vsa, "asym8", 32, H)
    assert np.array_equal(got, want)


def test_per_tensor_int8_equals_per_head_codes_at_the_same_scale():
    # rows whose per-head scale is exactly s = 1/16 (absmax 127/16) get the same codes
    rng = np.random.default_rng(8)
    x = rng.uniform(-7.9, 7.9, (16, 128)).astype(np.float32)
    x[:, 3] = 127 / 16
    s16 = int(np.float16(1 / 16).view(np.uint16))
    c_head, s_head = oracle.quantize_rows(x, 128, 8)
    assert np.all(s_head == s16)
    assert np.array_equal(oracle.quantize_rows_tensor(x, s16), c_head)


def test_per_tensor_int8_clips_and_matches_torch_qint8():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((32, 64)) * 4).astype(np.float32)
    s = 0.03125
    c = oracle.quantize_rows_tensor(x, int(np.float16(s).view(np.uint16))).view(np.int8)
    assert c.min() == -127 and c.max() == 127                      # |x| reaches past 127 s
    xc = np.clip(x, -127 * s, 127 * s)
    t = torch.quantize_per_tensor(torch.from_numpy(xc), s, 0, torch.qint8).int_repr().numpy()
    assert np.array_equal(t, c)                                   # s a power of two: no ties differ
    assert not oracle.quantize_rows_tensor(x, 0).any()


# --- h-mode query absorption -------------------------------------------------------

def _h_case(bits, seed, B=2, Hkv=2, G=2, Dh=32, cap=20, h_groups=2):
    rng = np.random.default_rng(seed)
    D = Hkv * Dh
    h = rng.standard_normal((B, cap, D)).astype(np.float32)
    if bits == 16:
        codes, scales = h.astype(np.float16).view(np.uint16), None
    else:
        codes, scales = oracle.quantize_rows(h, D // h_groups, bits)
    w = torch.from_numpy(rng.standard_normal((2 * D, D)).astype(np.float32) / np.sqrt(D))
    wb = w.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q = rng.standard_normal((B, Hkv * G, Dh)).astype(np.float32)
    hd = oracle.dequantize_rows(codes, scales, D, D // h_groups, bits)     # [B, cap, D] fp64
    W = w.to(torch.bfloat16).double().numpy()
    return codes, scales, wb, q, hd, W, D, Dh, G, Hkv


@pytest.mark.parametrize("bits", [4, 8, 16])
def test_h_absorbed_equals_reconstruction_attention_in_fp64(bits):
    codes, scales, wb, q, hd, W, D, Dh, G, Hkv = _h_case(bits, 11)
    lens = np.array([20, 7], np.int32)
    got = oracle.h_absorbed_decode(codes, scales, bits, 2, wb, q, lens, Hkv)
    for b, L in enumerate(lens):
        K = hd[b, :L] @ W[:D].T          # [L, Hkv*Dh], numpy matmul
        V = hd[b, :L] @ W[D:].T
        for h in range(Hkv * G):
            j = h // G
            want = oracle.attend(q[b, h].astype(np.float64), K[:, j * Dh:(j + 1) * Dh],
                                 V[:, j * Dh:(j + 1) * Dh], 1 / np.sqrt(Dh))
            assert np.allclose(got[b, h], want, rtol=1e-10, atol=1e-12), (b, h)


def test_h_absorbed_single_token_and_zero_query():
    codes, scales, wb, q, hd, W, D, Dh, G, Hkv = _h_case(4, 12)
    one = oracle.h_absorbed_decode(codes, scales, 4, 2, wb, q, np.array([1, 0], np.int32), Hkv)
    V0 = W[D:] @ hd[0, 0]
    for h in range(Hkv * G):
        j = h // G
        assert np.allclose(one[0, h], V0[j * Dh:(j + 1) * Dh], rtol=1e-12, atol=1e-12)
    assert not one[1].any()                                              # empty sequence
    zq = oracle.h_absorbed_decode(codes, scales, 4, 2, wb, np.zeros_like(q),
                                  np.array([20, 9], np.int32), Hkv)
    for b, L in ((0, 20), (1, 9)):
        Vm = W[D:] @ hd[b, :L].mean(0)
        for h in range(Hkv * G):
            j = h // G
            assert np.allclose(zq[b, h], Vm[j * Dh:(j + 1) * Dh], rtol=1e-10, atol=1e-12)
