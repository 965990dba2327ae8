"""CPU oracle for quantized-KV decode attention (test infrastructure).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``quantized_kv_cache_22_b200``) never imports it and
shares no code, header, table or helper with it.

Everything numeric happens in ``kvq_oracle.c`` (plain C, fp64 attention); this
module only loads it with ctypes and marshals numpy arrays.  See the C file's
header for the passages each function follows.

Parity status of each function (what pins it, in ``tests/test_oracle_pins.py``):
  f32_to_f16 / f64_to_f16 / bf16: pinned against numpy float16 / torch bfloat16.
  quantize_rows: pinned by the error bound |x - x^| <= s/2, |code| <= qmax,
      absmax -> +-qmax, idempotence, RNE ties and nibble-order fixtures.
  quantize_rows "e4m3": every code and every tie against torch float8_e4m3fn, the
      scale formula and the half-ulp error bound.
  quantize_rows "asym8": an exact arithmetic progression (codes 0..255), one-sided
      and all-zero groups, the error bound and exact zero, torch's quint8 affine
      quantiser at the same scale and zero-point; its decode equals the symmetric
      INT8 decode when the zero-point is 128.
  quantize_rows_tensor: equal to the per-head INT8 codes at the same scale,
      clipping, torch's qint8 quantiser.
  attend / decode_layer: pinned by closed forms (L=1, q=0, two tokens, equal
      keys, dominant key), GQA head mapping, permutation/duplication
      invariance, and torch scaled_dot_product_attention in fp64.
  h_reconstruct: pinned against a numpy matmul (library primitive) and the
      INT8-h / INT4-h quality bands of the TinyLoop page.
  h_absorbed_decode: pinned to the reconstruction attention in fp64 (numpy matmuls of
      W and the dequantised h, then attend), to out = W_v h^ for one token, and to
      W_v mean(h^) for a zero query.
  bytes_per_token_layer: pinned to the printed TinyLoop, KVSplit and
      on-device figures (tests/golden/).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, IEEE arithmetic, OpenMP) into oracle/."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.kvqo_f32_to_f16.argtypes = [ctypes.c_float]
    lib.kvqo_f32_to_f16.restype = ctypes.c_uint16
    lib.kvqo_f64_to_f16.argtypes = [ctypes.c_double]
    lib.kvqo_f64_to_f16.restype = ctypes.c_uint16
    lib.kvqo_f16_to_f32.argtypes = [ctypes.c_uint16]
    lib.kvqo_f16_to_f32.restype = ctypes.c_float
    lib.kvqo_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.kvqo_f32_to_bf16.restype = ctypes.c_uint16
    lib.kvqo_f32_to_e4m3.argtypes = [ctypes.c_float]
    lib.kvqo_f32_to_e4m3.restype = ctypes.c_uint8
    lib.kvqo_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    lib.kvqo_e4m3_to_f32.restype = ctypes.c_float
    lib.kvqo_quantize_rows.argtypes = [P, i64, i32, i32, i32, P, P]
    lib.kvqo_dequantize_rows.argtypes = [P, P, i64, i32, i32, i32, P]
    lib.kvqo_quantize_rows_tensor.argtypes = [P, i64, i32, ctypes.c_uint16, P]
    lib.kvqo_h_absorbed_decode.argtypes = [i32, i32, i32, i32, i32, i32, P, P, i32, i32, P, P, P,
                                           f64, P, i32]
    lib.kvqo_attend.argtypes = [P, P, P, i64, i32, f64, P]
    lib.kvqo_decode_layer.argtypes = [i32, i32, i32, i32, i32, P, P, i32, i32, P, P, i32, i32,
                                      P, P, f64, P, i32]
    lib.kvqo_h_reconstruct.argtypes = [P, P, i64, i32, i32, i32, P, i32, i32, P, P, i32]
    lib.kvqo_bytes_per_token_layer.argtypes = [i32] * 10 + [ctypes.POINTER(ctypes.c_uint64)]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _chk(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with status {rc}")


# --- scalar conversions -------------------------------------------------------

def f32_to_f16_bits(x: float) -> int:
    return int(_load().kvqo_f32_to_f16(float(x)))


def f64_to_f16_bits(x: float) -> int:
    return int(_load().kvqo_f64_to_f16(float(x)))


def f16_bits_to_f32(h: int) -> float:
    return float(_load().kvqo_f16_to_f32(int(h)))


def f32_to_bf16_bits(x: float) -> int:
    return int(_load().kvqo_f32_to_bf16(float(x)))


E4M3 = 228   # bit-width code of FP8 e4m3 codes (one byte per element)
ASYM8 = 208  # bit-width code of asymmetric INT8: uint8 codes, (scale, zero-point) fp16 pairs


def f32_to_e4m3(x: float) -> int:
    """e4m3 byte of x: round to nearest even, saturating at +-448."""
    return int(_load().kvqo_f32_to_e4m3(float(x)))


def e4m3_to_f32(c: int) -> float:
    return float(_load().kvqo_e4m3_to_f32(int(c)))


def _bits_arg(bits):
    if bits in ("e4m3", E4M3):
        return E4M3
    if bits in ("asym8", ASYM8):
        return ASYM8
    return int(bits)


def _row_bytes(dim: int, bits: int) -> int:
    return dim if bits in (E4M3, ASYM8) else dim * bits // 8


def _scales_per_group(bits: int) -> int:
    return 2 if bits == ASYM8 else 1


# --- quantiser ----------------------------------------------------------------

def quantize_rows(x, group: int, bits):
    """x: [..., dim] float32 (fp16/bf16 inputs must be widened exactly first).
    bits: 4, 8, "e4m3" or "asym8".

    Returns (codes uint8 [..., dim*bits/8], scales uint16 fp16-bits [..., dim/group]);
    "asym8": codes [..., dim], scales [..., dim/group, 2] = (scale, zero-point) per group.
    """
    bits = _bits_arg(bits)
    x = np.ascontiguousarray(x, dtype=np.float32)
    dim = x.shape[-1]
    rows = int(np.prod(x.shape[:-1])) if x.ndim > 1 else 1
    codes = np.zeros(x.shape[:-1] + (_row_bytes(dim, bits),), np.uint8)
    scales = np.zeros(x.shape[:-1] + (dim // group,) + ((2,) if bits == ASYM8 else ()), np.uint16)
    _chk(_load().kvqo_quantize_rows(_ptr(x), rows, dim, group, bits, _ptr(codes), _ptr(scales)),
         "quantize_rows")
    return codes, scales


def quantize_rows_tensor(x, s16: int):
    """Per-tensor INT8: every element of x with the one fp16 scale s16 (bits);
    returns int8 codes as uint8 [..., dim]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    dim = x.shape[-1]
    codes = np.zeros(x.shape, np.uint8)
    _chk(_load().kvqo_quantize_rows_tensor(_ptr(x), x.size // dim, dim, int(s16), _ptr(codes)),
         "quantize_rows_tensor")
    return codes


def dequantize_rows(codes, scales, dim: int, group: int, bits):
    """Inverse of quantize_rows in fp64.  bits == 16: codes hold fp16 values."""
    bits = _bits_arg(bits)
    codes = np.ascontiguousarray(codes)
    if bits == 16:
        codes = codes.view(np.uint8) if codes.dtype != np.uint8 else codes
        rows = codes.size // (dim * 2)
        lead = codes.shape[:-1]
    else:
        rows = codes.size // _row_bytes(dim, bits)
        lead = codes.shape[:-1]
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.zeros(lead + (dim,), np.float64)
    _chk(_load().kvqo_dequantize_rows(_ptr(codes), _ptr(scales) if bits != 16 else None, rows, dim,
                                      group, bits, _ptr(out)), "dequantize_rows")
    return out


# --- attention ----------------------------------------------------------------

def attend(q, K, V, tau: float):
    """q [dh], K/V [L, dh] float64 -> out [dh] float64."""
    q = np.ascontiguousarray(q, np.float64)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    out = np.zeros(q.shape[-1], np.float64)
    _chk(_load().kvqo_attend(_ptr(q), _ptr(K), _ptr(V), K.shape[0], q.shape[-1], tau, _ptr(out)),
         "attend")
    return out


def decode_layer(q, lens, k_codes, k_scales, k_bits, k_group, v_codes, v_scales, v_bits, v_group,
                 n_kv_heads: int, tau: float = 0.0, n_threads: int = 0):
    """Decode attention of one layer in the cache layout.

    q: [B, Hq, dh] float32 values; lens: [B] int32;
    k_codes: [B, Hkv, cap, row] uint8 (bits 16: [B, Hkv, cap, dh] float16/uint16);
    k_scales: [B, Hkv, cap, dh/group] uint16 or None.  Returns [B, Hq, dh] float64.
    """
    k_bits, v_bits = _bits_arg(k_bits), _bits_arg(v_bits)
    q = np.ascontiguousarray(q, np.float32)
    B, Hq, dh = q.shape
    lens = np.ascontiguousarray(lens, np.int32)
    cap = k_codes.shape[2]

    def prep(c, s, bits):
        c = np.ascontiguousarray(c)
        if bits == 16:
            c = c.view(np.uint8)
            return c, None
        return c, np.ascontiguousarray(s, np.uint16)

    kc, ks = prep(k_codes, k_scales, k_bits)
    vc, vs = prep(v_codes, v_scales, v_bits)
    out = np.zeros((B, Hq, dh), np.float64)
    _chk(_load().kvqo_decode_layer(B, Hq, n_kv_heads, dh, cap, _ptr(kc), _ptr(ks), k_bits,
                                   k_group if k_bits != 16 else dh, _ptr(vc), _ptr(vs), v_bits,
                                   v_group if v_bits != 16 else dh, _ptr(q), _ptr(lens), tau,
                                   _ptr(out), n_threads), "decode_layer")
    return out


def h_reconstruct(h_codes, h_scales, D: int, h_groups: int, h_bits: int, w_bf16_bits,
                  round_bf16: bool = True, n_threads: int = 0):
    """Rebuild [K|V] rows from an h cache.

    h_codes: [n_tok, D*bits/8] uint8 (bits 16: fp16 [n_tok, D]); h_scales [n_tok, h_groups];
    w_bf16_bits: [N, D] uint16 (bf16 bit patterns).
    Returns (y_f64 [n_tok, N], y_f16_bits [n_tok, N] uint16).
    """
    hc = np.ascontiguousarray(h_codes).view(np.uint8)
    n_tok = h_codes.shape[0]
    hs = None if h_bits == 16 else np.ascontiguousarray(h_scales, np.uint16)
    W = np.ascontiguousarray(w_bf16_bits, np.uint16)
    N = W.shape[0]
    y64 = np.zeros((n_tok, N), np.float64)
    y16 = np.zeros((n_tok, N), np.uint16)
    _chk(_load().kvqo_h_reconstruct(_ptr(hc), _ptr(hs), n_tok, D, h_groups, h_bits, _ptr(W), N,
                                    1 if round_bf16 else 0, _ptr(y64), _ptr(y16), n_threads),
         "h_reconstruct")
    return y64, y16


def h_absorbed_decode(h_codes, h_scales, h_bits: int, h_groups: int, w_bf16_bits, q, lens,
                      n_kv_heads: int, tau: float = 0.0, n_threads: int = 0):
    """h-mode decode attention by query absorption, fp64 (see the C header).

    h_codes: [B, cap, D*bits/8] uint8 (bits 16: fp16 [B, cap, D]); h_scales [B, cap, h_groups];
    w_bf16_bits: [2*Hkv*Dh, D] uint16; q: [B, Hq, Dh] float32; lens [B].
    Returns out [B, Hq, Dh] float64.
    """
    hc = np.ascontiguousarray(h_codes)
    hc = hc.view(np.uint8) if hc.dtype != np.uint8 else hc
    B, cap = h_codes.shape[0], h_codes.shape[1]
    hs = None if h_bits == 16 else np.ascontiguousarray(h_scales, np.uint16)
    W = np.ascontiguousarray(w_bf16_bits, np.uint16)
    q = np.ascontiguousarray(q, np.float32)
    _, Hq, Dh = q.shape
    D = W.shape[1]
    lens = np.ascontiguousarray(lens, np.int32)
    out = np.zeros((B, Hq, Dh), np.float64)
    _chk(_load().kvqo_h_absorbed_decode(B, Hq, n_kv_heads, Dh, D, cap, _ptr(hc), _ptr(hs), h_bits,
                                        h_groups, _ptr(W), _ptr(q), _ptr(lens), tau, _ptr(out),
                                        n_threads), "h_absorbed_decode")
    return out


def bytes_per_token_layer(mode=0, n_kv_heads=0, head_dim=0, k_bits=16, v_bits=16, k_group=0,
                          v_group=0, d_model=0, h_bits=16, h_groups=0) -> int:
    out = ctypes.c_uint64(0)
    _chk(_load().kvqo_bytes_per_token_layer(mode, n_kv_heads, head_dim, k_bits, v_bits,
                                            k_group or head_dim, v_group or head_dim, d_model,
                                            h_bits, h_groups, ctypes.byref(out)),
         "bytes_per_token_layer")
    return int(out.value)
