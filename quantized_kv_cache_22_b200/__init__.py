"""Python binding of libkvq (quantised KV cache + decode attention on B200).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libkvq.so``; PyTorch tensors only provide device memory and streams.  The
functions carry the C ABI's names (``include/kvq.h``) and raise ``KvqError``
on a non-zero status.  If the shared library is missing the import fails: there
is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
KVQ_MODE_KV, KVQ_MODE_H = 0, 1
KVQ_FMT_INT, KVQ_FMT_E4M3, KVQ_FMT_ASYM, KVQ_FMT_TENSOR = 0, 1, 2, 3
KVQ_F16, KVQ_F32, KVQ_BF16 = 0, 1, 2

EXPORTED = ("kvq_cache_bytes", "kvq_layer_buffer_bytes", "kvq_append", "kvq_workspace_bytes",
            "kvq_h_scratch_bytes", "kvq_decode_attn", "kvq_decode_partials", "kvq_merge_partials",
            "kvq_h_reconstruct", "kvq_workspace_status", "kvq_status_string",
            "kvq_last_error_detail", "kvq_decode_attn_noalloc", "kvq_h_operand_bytes",
            "kvq_append_decode_attn", "kvq_h_absorbed_scratch_bytes", "kvq_h_decode_absorbed",
            "kvq_h_fused_scratch_bytes", "kvq_h_decode_fused", "kvq_selftest_bounded_wait",
            "kvq_selftest_decode_timeout", "kvq_noalloc_status", "kvq_selftest_noalloc_timeout",
            "kvq_decode_plan_info")


class KvqError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        detail = _lib.kvq_last_error_detail().decode() if status == -6 else ""
        super().__init__(f"{fn} failed: {status} ({status_string(status)}) {detail}".rstrip())


class KvqConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "mode", "batch", "capacity", "n_layers", "n_q_heads", "n_kv_heads", "head_dim",
        "k_bits", "v_bits", "k_group", "v_group", "d_model", "h_bits", "h_groups",
        "window", "n_anchor", "page_tokens", "n_pages", "kv_format")]


class KvqDecodePlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "engine", "num_ctas", "ctas_per_sm_planned", "stages", "stage_bytes", "smem_bytes",
        "threads", "packed_columns")]


KVQ_ENGINE_WARP_MMA, KVQ_ENGINE_TCGEN05 = 0, 1


class KvqLayer(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so not built ({LIB_PATH}); run quantized_kv_cache_22_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64
    pu64 = ctypes.POINTER(u64)
    cfgp = ctypes.POINTER(KvqConfig)
    layp = ctypes.POINTER(KvqLayer)
    sig = {
        "kvq_cache_bytes": [cfgp, pu64, pu64, pu64],
        "kvq_layer_buffer_bytes": [cfgp, pu64, pu64, pu64, pu64],
        "kvq_append": [cfgp, layp, P, P, i32, P, i32, i32, P],
        "kvq_workspace_bytes": [cfgp, i32, pu64],
        "kvq_h_scratch_bytes": [cfgp, i32, pu64],
        "kvq_decode_attn": [cfgp, layp, P, i32, P, i32, ctypes.c_float, P, i32, P, u64, i32, P, P,
                            u64, P],
        "kvq_decode_partials": [cfgp, layp, P, i32, P, i32, ctypes.c_float, P, u64, i32, P],
        "kvq_append_decode_attn": [cfgp, layp, P, P, i32, P, i32, P, i32, ctypes.c_float, P, i32,
                                   P, u64, i32, P],
        "kvq_merge_partials": [cfgp, P, P, i32, P, u64, i32, P],
        "kvq_h_operand_bytes": [cfgp, i32, pu64],
        "kvq_h_reconstruct": [cfgp, layp, P, i32, P, P, i32, P, u64, P],
        "kvq_workspace_status": [P, ctypes.POINTER(i32), P],
        "kvq_h_absorbed_scratch_bytes": [cfgp, i32, pu64],
        "kvq_h_fused_scratch_bytes": [cfgp, i32, pu64],
        "kvq_selftest_bounded_wait": [P, u64, P],
        "kvq_selftest_decode_timeout": [cfgp, layp, P, i32, P, P, i32, P, u64, u64, P],
        "kvq_h_decode_fused": [cfgp, layp, P, P, i32, P, i32, ctypes.c_float, P, i32, P, u64, P],
        "kvq_h_decode_absorbed": [cfgp, layp, P, P, i32, P, i32, ctypes.c_float, P, i32, P, u64, P],
        "kvq_decode_attn_noalloc": [cfgp, layp, P, i32, P, i32, ctypes.c_float, P, i32, i32, P],
        "kvq_noalloc_status": [ctypes.POINTER(i32), P],
        "kvq_selftest_noalloc_timeout": [cfgp, layp, P, i32, P, P, i32, u64, P],
        "kvq_decode_plan_info": [cfgp, i32, ctypes.POINTER(KvqDecodePlan)],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.kvq_status_string.argtypes = [ctypes.c_int]
    lib.kvq_status_string.restype = ctypes.c_char_p
    lib.kvq_last_error_detail.argtypes = []
    lib.kvq_last_error_detail.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def status_string(status: int) -> str:
    return _lib.kvq_status_string(int(status)).decode()


def _check(fn, rc):
    if rc != KVQ_OK:
        raise KvqError(fn, rc)


def _ptr(t):
    # plain ints: ctypes converts them for c_void_p arguments
    return None if t is None else t.data_ptr()


_DTYPE_CODES = {torch.float16: KVQ_F16, torch.float32: KVQ_F32, torch.bfloat16: KVQ_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    return _DTYPE_CODES[t.dtype]


def _stream(stream):
    if stream is None:
        # the current stream's handle without building a Stream object
        return torch._C._cuda_getCurrentRawStream(torch.cuda.current_device())
    return stream.cuda_stream


_CFG_MEMO = {}   # field tuple -> (KvqConfig, byref); the library only reads the struct


@dataclass
class Config:
    """Python view of ``kvq_config`` (see include/kvq.h for the meaning of each field)."""
    batch: int
    capacity: int
    n_q_heads: int = 0
    n_kv_heads: int = 0
    head_dim: int = 128
    k_bits: int = 8
    v_bits: int = 8
    k_group: int = 0
    v_group: int = 0
    n_layers: int = 1
    mode: int = KVQ_MODE_KV
    d_model: int = 0
    h_bits: int = 4
    h_groups: int = 0
    window: int = 0       # sliding window: ring of recent tokens (capacity = n_anchor + window)
    n_anchor: int = 0     # tokens kept at the start of the sequence
    page_tokens: int = 0  # 128: paged cache (a pool of n_pages pages, block table per layer)
    n_pages: int = 0
    kv_format: int = 0    # KVQ_FMT_INT; or, with k_bits = v_bits = 8, KVQ_FMT_E4M3 (FP8),
    #                       KVQ_FMT_ASYM (zero-point) or KVQ_FMT_TENSOR (one scale per tensor)

    def _key(self):
        return (self.mode, self.batch, self.capacity, self.n_layers, self.n_q_heads,
                self.n_kv_heads, self.head_dim, self.k_bits, self.v_bits,
                self.k_group or self.head_dim, self.v_group or self.head_dim,
                self.d_model, self.h_bits, self.h_groups, self.window, self.n_anchor,
                self.page_tokens, self.n_pages, self.kv_format)

    def c(self) -> KvqConfig:
        """A new ``kvq_config`` struct with these fields."""
        return KvqConfig(*self._key())

    def _ref(self):
        """byref() of a shared struct with these fields (read-only use by the wrappers)."""
        key = self._key()
        r = _CFG_MEMO.get(key)
        if r is None:
            if len(_CFG_MEMO) > 256:
                _CFG_MEMO.clear()
            c = KvqConfig(*key)
            r = _CFG_MEMO[key] = (c, ctypes.byref(c))
        return r[1]


# ----------------------------------------------------------------------------- host-only calls

def kvq_cache_bytes(cfg: Config):
    a, b, c = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check("kvq_cache_bytes", _lib.kvq_cache_bytes(ctypes.byref(cfg.c()), ctypes.byref(a),
                                                   ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def kvq_layer_buffer_bytes(cfg: Config):
    v = [ctypes.c_uint64() for _ in range(4)]
    _check("kvq_layer_buffer_bytes",
           _lib.kvq_layer_buffer_bytes(ctypes.byref(cfg.c()), *[ctypes.byref(x) for x in v]))
    return tuple(x.value for x in v)


def kvq_workspace_bytes(cfg: Config, num_ctas: int = 0) -> int:
    v = ctypes.c_uint64()
    _check("kvq_workspace_bytes", _lib.kvq_workspace_bytes(ctypes.byref(cfg.c()), num_ctas,
                                                           ctypes.byref(v)))
    return v.value


def kvq_decode_plan_info(cfg: Config, num_ctas: int = 0) -> dict:
    """The decode launch the library makes for cfg: engine, CTAs, ring depth, shared memory."""
    v = KvqDecodePlan()
    _check("kvq_decode_plan_info", _lib.kvq_decode_plan_info(ctypes.byref(cfg.c()), num_ctas,
                                                             ctypes.byref(v)))
    return {n: getattr(v, n) for n, _ in KvqDecodePlan._fields_}


def kvq_h_scratch_bytes(cfg: Config, max_len: int) -> int:
    v = ctypes.c_uint64()
    _check("kvq_h_scratch_bytes", _lib.kvq_h_scratch_bytes(ctypes.byref(cfg.c()), max_len,
                                                           ctypes.byref(v)))
    return v.value


# ----------------------------------------------------------------------------- device buffers

class LayerCache:
    """One layer's cache buffers, allocated with torch on `device` (caller-owned memory).
    A paged config allocates the page pool; `block_table` (int32 [B][capacity/128] on
    the device) then maps each sequence's logical pages to pool pages."""

    block_table = None

    def __init__(self, cfg: Config, device="cuda", zero: bool = False, block_table=None):
        kc, ks, vc, vs = kvq_layer_buffer_bytes(cfg)
        alloc = torch.zeros if zero else torch.empty
        self.k_codes = alloc(max(kc, 16), dtype=torch.uint8, device=device)
        self.k_scales = alloc(max(ks // 2, 8), dtype=torch.float16, device=device) if ks else None
        self.v_codes = alloc(max(vc, 16), dtype=torch.uint8, device=device) if vc else None
        self.v_scales = alloc(max(vs // 2, 8), dtype=torch.float16, device=device) if vs else None
        self.cfg = cfg
        self.block_table = block_table

    def c(self) -> KvqLayer:
        """A new ``kvq_layer`` struct with these buffers."""
        return KvqLayer(*(None if t is None else t.data_ptr()
                          for t in (self.k_codes, self.k_scales, self.v_codes, self.v_scales,
                                    self.block_table)))

    def _ref(self):
        """byref() of a struct kept for these buffers (read-only use by the wrappers)."""
        ts = (self.k_codes, self.k_scales, self.v_codes, self.v_scales, self.block_table)
        memo = self.__dict__.get("_c_memo")
        if memo is None or any(a is not b for a, b in zip(memo[0], ts)):
            c = self.c()
            memo = (ts, c, ctypes.byref(c))
            self.__dict__["_c_memo"] = memo
        return memo[2]


class Workspace:
    """Split-KV partials and merge counters, sized by kvq_workspace_bytes and zero-filled
    (a call leaves it ready for the next; zero it again after a timeout status)."""

    def __init__(self, cfg: Config, num_ctas: int = 0, device="cuda"):
        self.nbytes = kvq_workspace_bytes(cfg, num_ctas)
        self.buf = torch.zeros(self.nbytes // 4 + 64, dtype=torch.float32, device=device)


# ----------------------------------------------------------------------------- device calls

def kvq_append(cfg: Config, layer: LayerCache, k: torch.Tensor, v, d_pos: torch.Tensor,
               max_pos: int, n_new: int, stream=None):
    _check("kvq_append", _lib.kvq_append(cfg._ref(), layer._ref(), _ptr(k),
                                         _ptr(v), _dtype_code(k), _ptr(d_pos), int(max_pos),
                                         int(n_new), _stream(stream)))


def kvq_decode_attn(cfg: Config, layer: LayerCache, q: torch.Tensor, d_len: torch.Tensor,
                    max_len: int, out: torch.Tensor, ws: Workspace, softmax_scale: float = 0.0,
                    num_ctas: int = 0, w_kv=None, kv_scratch=None, stream=None):
    scratch_bytes = 0 if kv_scratch is None else kv_scratch.numel() * kv_scratch.element_size()
    _check("kvq_decode_attn",
           _lib.kvq_decode_attn(cfg._ref(), layer._ref(), _ptr(q),
                                _dtype_code(q), _ptr(d_len), int(max_len), float(softmax_scale),
                                _ptr(out), _dtype_code(out), _ptr(ws.buf), ws.nbytes,
                                int(num_ctas), _ptr(w_kv), _ptr(kv_scratch), scratch_bytes,
                                _stream(stream)))


def kvq_append_decode_attn(cfg: Config, layer: LayerCache, k_new: torch.Tensor,
                           v_new: torch.Tensor, q: torch.Tensor, d_len: torch.Tensor, max_len: int,
                           out: torch.Tensor, ws: Workspace, softmax_scale: float = 0.0,
                           num_ctas: int = 0, stream=None):
    """One decode step: quantise k_new/v_new ([B][Hkv][Dh]) into position d_len-1, then attend."""
    if k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share a dtype")
    _check("kvq_append_decode_attn",
           _lib.kvq_append_decode_attn(cfg._ref(), layer._ref(), _ptr(k_new),
                                       _ptr(v_new), _dtype_code(k_new), _ptr(q), _dtype_code(q),
                                       _ptr(d_len), int(max_len), float(softmax_scale), _ptr(out),
                                       _dtype_code(out), _ptr(ws.buf), ws.nbytes, int(num_ctas),
                                       _stream(stream)))


def kvq_decode_partials(cfg: Config, layer: LayerCache, q: torch.Tensor, d_len: torch.Tensor,
                        max_len: int, ws: Workspace, softmax_scale: float = 0.0, num_ctas: int = 0,
                        stream=None):
    _check("kvq_decode_partials",
           _lib.kvq_decode_partials(cfg._ref(), layer._ref(), _ptr(q),
                                    _dtype_code(q), _ptr(d_len), int(max_len), float(softmax_scale),
                                    _ptr(ws.buf), ws.nbytes, int(num_ctas), _stream(stream)))


def kvq_merge_partials(cfg: Config, d_len: torch.Tensor, out: torch.Tensor, ws: Workspace,
                       num_ctas: int = 0, stream=None):
    _check("kvq_merge_partials",
           _lib.kvq_merge_partials(cfg._ref(), _ptr(d_len), _ptr(out), _dtype_code(out),
                                   _ptr(ws.buf), ws.nbytes, int(num_ctas), _stream(stream)))


def kvq_h_operand_bytes(cfg: Config, max_len: int) -> int:
    v = ctypes.c_uint64()
    _check("kvq_h_operand_bytes", _lib.kvq_h_operand_bytes(cfg._ref(), max_len,
                                                           ctypes.byref(v)))
    return v.value


def kvq_h_reconstruct(cfg: Config, layer: LayerCache, w_kv: torch.Tensor, max_len: int,
                      k_out: torch.Tensor, v_out: torch.Tensor, out_capacity: int,
                      operand: torch.Tensor, stream=None):
    _check("kvq_h_reconstruct",
           _lib.kvq_h_reconstruct(cfg._ref(), layer._ref(), _ptr(w_kv),
                                  int(max_len), _ptr(k_out), _ptr(v_out), int(out_capacity),
                                  _ptr(operand), operand.numel() * operand.element_size(),
                                  _stream(stream)))


def kvq_h_absorbed_scratch_bytes(cfg: Config, max_len: int) -> int:
    v = ctypes.c_uint64()
    _check("kvq_h_absorbed_scratch_bytes",
           _lib.kvq_h_absorbed_scratch_bytes(cfg._ref(), int(max_len), ctypes.byref(v)))
    return v.value


def kvq_h_decode_absorbed(cfg: Config, layer: LayerCache, w_kv: torch.Tensor, q: torch.Tensor,
                          d_len: torch.Tensor, max_len: int, out: torch.Tensor,
                          scratch: torch.Tensor, softmax_scale: float = 0.0, stream=None):
    """h-mode decode attention by query absorption (W_k^T q against the h codes)."""
    _check("kvq_h_decode_absorbed",
           _lib.kvq_h_decode_absorbed(cfg._ref(), layer._ref(), _ptr(w_kv), _ptr(q),
                                      _dtype_code(q), _ptr(d_len), int(max_len),
                                      float(softmax_scale), _ptr(out), _dtype_code(out),
                                      _ptr(scratch), scratch.numel() * scratch.element_size(),
                                      _stream(stream)))


def kvq_h_fused_scratch_bytes(cfg: Config, max_len: int) -> int:
    v = ctypes.c_uint64()
    _check("kvq_h_fused_scratch_bytes",
           _lib.kvq_h_fused_scratch_bytes(cfg._ref(), int(max_len), ctypes.byref(v)))
    return v.value


def kvq_h_decode_fused(cfg: Config, layer: LayerCache, w_kv: torch.Tensor, q: torch.Tensor,
                       d_len: torch.Tensor, max_len: int, out: torch.Tensor, scratch: torch.Tensor,
                       softmax_scale: float = 0.0, stream=None):
    """h-mode decode attention with the K/V reconstruction fused into the GEMM epilogue.
    `scratch` starts with a status word (zero it once; read it with kvq_workspace_status)."""
    _check("kvq_h_decode_fused",
           _lib.kvq_h_decode_fused(cfg._ref(), layer._ref(), _ptr(w_kv), _ptr(q),
                                   _dtype_code(q), _ptr(d_len), int(max_len),
                                   float(softmax_scale), _ptr(out), _dtype_code(out),
                                   _ptr(scratch), scratch.numel() * scratch.element_size(),
                                   _stream(stream)))


def kvq_selftest_bounded_wait(ws, timeout_ns: int, stream=None):
    """Run the kernels' bounded wait on a barrier nothing completes (see kvq.h)."""
    buf = ws.buf if isinstance(ws, Workspace) else ws
    _check("kvq_selftest_bounded_wait",
           _lib.kvq_selftest_bounded_wait(_ptr(buf), int(timeout_ns), _stream(stream)))


def kvq_selftest_decode_timeout(cfg: Config, layer: LayerCache, q: torch.Tensor,
                                d_len: torch.Tensor, out: torch.Tensor, ws: Workspace,
                                timeout_ns: int, stream=None):
    """The decode kernel with a producer that copies nothing: its waits run out (see kvq.h)."""
    _check("kvq_selftest_decode_timeout",
           _lib.kvq_selftest_decode_timeout(cfg._ref(), layer._ref(), _ptr(q), _dtype_code(q),
                                            _ptr(d_len), _ptr(out), _dtype_code(out),
                                            _ptr(ws.buf), ws.nbytes, int(timeout_ns),
                                            _stream(stream)))


def kvq_decode_attn_noalloc(cfg: Config, layer: LayerCache, q: torch.Tensor, d_len: torch.Tensor,
                            max_len: int, out: torch.Tensor, softmax_scale: float = 0.0,
                            num_ctas: int = 0, stream=None):
    """kvq_decode_attn with the library's own fixed device array as the workspace
    (for callers that may not allocate device memory; see kvq.h)."""
    _check("kvq_decode_attn_noalloc",
           _lib.kvq_decode_attn_noalloc(cfg._ref(), layer._ref(), _ptr(q), _dtype_code(q),
                                        _ptr(d_len), int(max_len), float(softmax_scale), _ptr(out),
                                        _dtype_code(out), int(num_ctas), _stream(stream)))


def kvq_noalloc_status(stream=None) -> int:
    """Read and clear the status word of the noalloc entry point's device array."""
    st = ctypes.c_int32()
    _check("kvq_noalloc_status", _lib.kvq_noalloc_status(ctypes.byref(st), _stream(stream)))
    return st.value


def kvq_selftest_noalloc_timeout(cfg: Config, layer: LayerCache, q: torch.Tensor,
                                 d_len: torch.Tensor, out: torch.Tensor, timeout_ns: int,
                                 stream=None):
    """The stalled-producer decode kernel run on the noalloc array (see kvq.h)."""
    _check("kvq_selftest_noalloc_timeout",
           _lib.kvq_selftest_noalloc_timeout(cfg._ref(), layer._ref(), _ptr(q), _dtype_code(q),
                                             _ptr(d_len), _ptr(out), _dtype_code(out),
                                             int(timeout_ns), _stream(stream)))


def kvq_workspace_status(ws, stream=None) -> int:
    """Read and clear the status word of a Workspace (or of a scratch tensor that starts
    with one, as the fused h-mode path's)."""
    st = ctypes.c_int32()
    buf = ws.buf if isinstance(ws, Workspace) else ws
    _check("kvq_workspace_status", _lib.kvq_workspace_status(_ptr(buf), ctypes.byref(st),
                                                             _stream(stream)))
    return st.value
