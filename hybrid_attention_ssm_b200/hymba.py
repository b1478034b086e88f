"""ctypes binding of libhymba.so (argument marshalling only).

Every computation happens in the library's CUDA kernels; this module only turns torch
tensors (device memory allocated by PyTorch) into the pointers and structs of the C ABI
declared in include/hymba.h.  It raises if the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhymba.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "hymba.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_FP16_RANGE = range(7)
KV_OWN, KV_PRODUCER, KV_CONSUMER = 0, 1, 2
CACHE_SWA, CACHE_GLOBAL = 0, 1
MODE_PREFILL, MODE_DECODE, MODE_PREFILL_HOST = 0, 1, 2

_c_int, _c_size, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p


class HymbaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"hymba error {code}: {msg}")
        self.code = code


class LayerCfg(ctypes.Structure):
    _fields_ = [(n, _c_int) for n in ("d_model", "n_q_heads", "n_kv_heads", "head_dim", "d_inner",
                                       "d_state", "d_conv", "dt_rank", "window", "n_meta",
                                       "is_global", "kv_role")] + \
               [("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("meta", _vp), ("w_in", _vp), ("conv_w", _vp), ("conv_b", _vp), ("w_x", _vp),
                ("w_dt", _vp), ("w_dt_ld", _c_int), ("dt_bias", _vp), ("A", _vp),
                ("g_attn", _vp), ("g_ssm", _vp), ("w_out", _vp)]


class KVCache(ctypes.Structure):
    _fields_ = [(n, _c_int) for n in ("kind", "batch", "n_kv_heads", "head_dim", "n_meta",
                                       "window", "max_tokens")] + \
               [(n, _vp) for n in ("meta_k", "meta_v", "ring_k", "ring_v", "k", "v")]


class ProfRecord(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("ms", ctypes.c_float)]


class StageLayout(ctypes.Structure):
    _fields_ = [(n, _c_size) for n in ("q", "xz", "xc", "xbc", "dt_pre", "y", "o", "u")] + \
               [("ld_xbc", _c_int), ("scan_chunks", _c_int), ("scan_chunk_len", _c_int)]


class MetaPrefix(ctypes.Structure):
    _fields_ = [("k", _vp), ("v", _vp), ("ssm_state", _vp), ("conv_state", _vp)]


class DecodeStageLayout(ctypes.Structure):
    _fields_ = [(n, _c_size) for n in ("proj", "xc", "xbc_part", "y")] + \
               [("proj_slice_stride", ctypes.c_longlong), ("xbc_slice_stride", ctypes.c_longlong)] + \
               [(n, _c_int) for n in ("in_split", "xproj_split", "ld_proj", "ld_xbc")]


_LIB = None


def header_functions():
    """Names of the functions include/hymba.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^(?:int|const char\*)\s+(hymba_\w+)\s*\(", text, flags=re.M)))


def lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "hymba_version": ([], _c_int),
            "hymba_last_error": ([], ctypes.c_char_p),
            "hymba_mixer_workspace_size": ([ctypes.POINTER(LayerCfg), _c_int, _c_int, _c_int, _c_int,
                                            ctypes.POINTER(_c_size)], _c_int),
            "hymba_workspace_init": ([_vp, _c_size, _vp], _c_int),
            "hymba_status_read": ([_vp, _vp, ctypes.POINTER(_c_int)], _c_int),
            "hymba_kv_share_alloc": ([ctypes.POINTER(LayerCfg), _c_int, ctypes.POINTER(ctypes.c_uint8),
                                      _c_int, _c_int, _vp, _c_size, ctypes.POINTER(_c_size),
                                      ctypes.POINTER(_c_int), ctypes.POINTER(_c_int),
                                      ctypes.POINTER(KVCache), _c_int, ctypes.POINTER(_c_int)], _c_int),
            "hymba_mixer_prefill": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                     _c_int, _c_int, ctypes.POINTER(KVCache), _vp, _vp, _vp, _vp, _vp,
                                     _c_size, _vp], _c_int),
            "hymba_mixer_decode": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                    _c_int, ctypes.POINTER(KVCache), _vp, _vp, _vp, _vp, _vp, _c_size,
                                    _vp], _c_int),
            "hymba_mixer_prefill_host": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                          _c_int, _c_int, ctypes.POINTER(KVCache), _vp, _vp, _vp, _vp, _c_size,
                                          _vp], _c_int),
            "hymba_meta_prefix_size": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(_c_size)], _c_int),
            "hymba_meta_prefix_build": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _vp, _c_size,
                                         ctypes.POINTER(MetaPrefix), ctypes.POINTER(MetaPrefix), _vp, _vp, _c_size,
                                         _vp], _c_int),
            "hymba_mixer_prefill_prefix": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                            _c_int, ctypes.POINTER(MetaPrefix), ctypes.POINTER(KVCache), _vp, _vp,
                                            _vp, _vp, _vp, _c_size, _vp], _c_int),
            "hymba_mixer_decode_norm": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                         _c_int, ctypes.POINTER(KVCache), _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                                         _vp, _vp, _c_size, _vp], _c_int),
            "hymba_ffn_swiglu_decode_norm": ([_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, ctypes.c_float,
                                              _vp, _vp, _c_size, _vp], _c_int),
            "hymba_mixer_decode_ragged": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                           _vp, _c_int, ctypes.POINTER(KVCache), _vp, _vp, _vp, _vp, _vp, _c_size,
                                           _vp], _c_int),
            "hymba_mixer_stage_layout": ([ctypes.POINTER(LayerCfg), _c_int, _c_int, _c_int,
                                          ctypes.POINTER(StageLayout)], _c_int),
            "hymba_decode_stage_layout": ([ctypes.POINTER(LayerCfg), _c_int, _c_int,
                                           ctypes.POINTER(DecodeStageLayout)], _c_int),
            "hymba_gemm_bf16": ([_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
            "hymba_rmsnorm": ([_vp, _vp, _c_int, _c_int, ctypes.c_float, _vp, _vp], _c_int),
            "hymba_ffn_swiglu": ([_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp], _c_int),
            "hymba_ffn_workspace_size": ([_c_int, _c_int, _c_int, ctypes.POINTER(_c_size)], _c_int),
            "hymba_ffn_swiglu_decode": ([_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_size, _vp], _c_int),
            "hymba_l2_prefetch": ([ctypes.POINTER(_vp), ctypes.POINTER(_c_size), _c_int, _vp], _c_int),
            "hymba_set_wait_limit_ns": ([ctypes.c_ulonglong], _c_int),
            "hymba_prepend_meta": ([_vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
            "hymba_selftest_wait_timeout": ([_vp, _c_size, _vp], _c_int),
            "hymba_mixer_decode_noalloc": ([ctypes.POINTER(LayerCfg), ctypes.POINTER(LayerWeights), _vp, _c_int,
                                            _c_int, ctypes.POINTER(KVCache), _vp, _vp, _vp, _vp, _vp], _c_int),
            "hymba_profile_begin": ([_c_int], _c_int),
            "hymba_profile_read": ([ctypes.POINTER(ProfRecord), _c_int, ctypes.POINTER(_c_int)], _c_int),
            "hymba_profile_end": ([ctypes.POINTER(ProfRecord), _c_int, ctypes.POINTER(_c_int)], _c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def check(rc):
    if rc != OK:
        raise HymbaError(rc, lib().hymba_last_error().decode())
    return rc


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def stream_handle(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------------------------------
# configuration / weights / caches
# ---------------------------------------------------------------------------------------
def make_cfg(dims) -> LayerCfg:
    return LayerCfg(dims.d_model, dims.n_q_heads, dims.n_kv_heads, dims.head_dim, dims.d_inner,
                    dims.d_state, dims.d_conv, dims.dt_rank, dims.window, dims.n_meta,
                    int(dims.is_global), int(dims.kv_role), float(dims.rope_base), float(dims.norm_eps))


_BF16_W = ("meta", "w_in", "w_x")
_F32_W = ("conv_w", "conv_b", "dt_bias", "A", "g_attn", "g_ssm")


class DeviceWeights:
    """A layer's weights in device memory plus the C struct pointing at them."""

    def __init__(self, w: dict, device="cuda"):
        """w: numpy arrays (as synth.layer_weights returns them) or float32 torch tensors."""
        def dev(a, dtype):
            if isinstance(a, torch.Tensor):
                return a.to(device=device, dtype=torch.float32).contiguous().to(dtype)
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device).to(dtype)

        self.t = {}
        for k in _BF16_W:
            self.t[k] = dev(w[k], torch.bfloat16)
        self.t["w_out"] = dev(w["w_out"], torch.float16)
        for k in _F32_W:
            self.t[k] = dev(w[k], torch.float32)
        wdt = dev(w["w_dt"], torch.float32)
        ld = (wdt.shape[1] + 3) // 4 * 4
        pad = torch.zeros(wdt.shape[0], ld, dtype=torch.float32, device=device)
        pad[:, :wdt.shape[1]] = wdt
        self.t["w_dt"] = pad
        self.c = LayerWeights(ptr(self.t["meta"]), ptr(self.t["w_in"]), ptr(self.t["conv_w"]),
                              ptr(self.t["conv_b"]), ptr(self.t["w_x"]), ptr(self.t["w_dt"]), ld,
                              ptr(self.t["dt_bias"]), ptr(self.t["A"]), ptr(self.t["g_attn"]),
                              ptr(self.t["g_ssm"]), ptr(self.t["w_out"]))


class Cache:
    """A KV cache (SWA meta + ring + prefill view, or global) owned by torch tensors."""

    def __init__(self, dims, batch, max_tokens, kind=None, device="cuda", view=None):
        kind = (CACHE_GLOBAL if dims.is_global else CACHE_SWA) if kind is None else kind
        Hkv, D = dims.n_kv_heads, dims.head_dim
        z = lambda *s: torch.zeros(*s, Hkv, D, dtype=torch.float16, device=device)
        self.t = {}
        if view is None:
            self.t["k"], self.t["v"] = z(batch, max_tokens), z(batch, max_tokens)
        else:
            self.t["k"], self.t["v"] = view
        if kind == CACHE_SWA:
            self.t["meta_k"], self.t["meta_v"] = z(batch, max(dims.n_meta, 1)), z(batch, max(dims.n_meta, 1))
            self.t["ring_k"], self.t["ring_v"] = z(batch, dims.window), z(batch, dims.window)
        g = lambda n: ptr(self.t[n]) if n in self.t else None
        self.c = KVCache(kind, batch, Hkv, D, dims.n_meta, dims.window, max_tokens,
                         g("meta_k"), g("meta_v"), g("ring_k"), g("ring_v"), g("k"), g("v"))


def workspace_size(dims, batch, n_tokens, x_has_meta=0, mode=MODE_PREFILL):
    n = ctypes.c_size_t()
    cfg = make_cfg(dims)
    check(lib().hymba_mixer_workspace_size(ctypes.byref(cfg), batch, n_tokens, x_has_meta, mode, ctypes.byref(n)))
    return n.value


def alloc_workspace(nbytes, device="cuda", stream=None):
    ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    view = ws[off:off + nbytes]
    check(lib().hymba_workspace_init(ptr(view), nbytes, stream_handle(stream)))
    return view


def stage_layout(dims, batch, n_tokens, x_has_meta=0) -> StageLayout:
    out = StageLayout()
    cfg = make_cfg(dims)
    check(lib().hymba_mixer_stage_layout(ctypes.byref(cfg), batch, n_tokens, x_has_meta, ctypes.byref(out)))
    return out


def decode_stage_layout(dims, batch, max_tokens) -> DecodeStageLayout:
    out = DecodeStageLayout()
    cfg = make_cfg(dims)
    check(lib().hymba_decode_stage_layout(ctypes.byref(cfg), batch, max_tokens, ctypes.byref(out)))
    return out


def status_read(ws, stream=None) -> int:
    s = ctypes.c_int()
    check(lib().hymba_status_read(ptr(ws), stream_handle(stream), ctypes.byref(s)))
    return s.value


def kv_share_alloc(base_dims, is_global, batch, max_tokens, dev_buf=None):
    """Returns (bytes_needed, cache_id list, role list, caches list)."""
    n = len(is_global)
    cfg = make_cfg(base_dims)
    g = (ctypes.c_uint8 * n)(*[int(v) for v in is_global])
    cid, role = (ctypes.c_int * n)(), (ctypes.c_int * n)()
    need = ctypes.c_size_t()
    caches = (KVCache * n)()
    nc = ctypes.c_int()
    buf_bytes = 0 if dev_buf is None else dev_buf.numel() * dev_buf.element_size()
    check(lib().hymba_kv_share_alloc(ctypes.byref(cfg), n, g, batch, max_tokens, ptr(dev_buf), buf_bytes,
                                     ctypes.byref(need), cid, role, caches, n, ctypes.byref(nc)))
    return need.value, list(cid), list(role), [caches[i] for i in range(nc.value)]


# ---------------------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------------------
def mixer_prefill(dims, dw: DeviceWeights, x, kv: Cache, out, ws, x_has_meta=0, ssm_state=None,
                  conv_state=None, residual=None, stream=None, cfg=None):
    cfg = make_cfg(dims) if cfg is None else cfg
    B, n_tokens = x.shape[0], x.shape[1]
    check(lib().hymba_mixer_prefill(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x), x_has_meta, B, n_tokens,
                                    ctypes.byref(kv.c), ptr(ssm_state), ptr(conv_state), ptr(residual), ptr(out),
                                    ptr(ws), ws.numel(), stream_handle(stream)))


def mixer_prefill_host(dims, dw: DeviceWeights, x_host, kv: Cache, out_host, ws, x_has_meta=0, ssm_state=None,
                       conv_state=None, stream=None, cfg=None):
    """hymba_mixer_prefill from host buffers: x_host [B, n, d] and out_host [B, T, d] are CPU
    bf16 tensors (pinned for asynchronous copies); ws sized with MODE_PREFILL_HOST."""
    assert not x_host.is_cuda and not out_host.is_cuda
    cfg = make_cfg(dims) if cfg is None else cfg
    B, n_tokens = x_host.shape[0], x_host.shape[1]
    check(lib().hymba_mixer_prefill_host(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x_host), x_has_meta, B, n_tokens,
                                         ctypes.byref(kv.c), ptr(ssm_state), ptr(conv_state), ptr(out_host), ptr(ws),
                                         ws.numel(), stream_handle(stream)))


class Prefix:
    """A layer's precomputed meta-token prefix (hymba_meta_prefix_build), owned by a torch buffer."""

    def __init__(self, dims, dw: DeviceWeights, meta_rows, meta_out, ws, producer=None, stream=None, device="cuda"):
        cfg = make_cfg(dims)
        n = ctypes.c_size_t()
        check(lib().hymba_meta_prefix_size(ctypes.byref(cfg), ctypes.byref(n)))
        raw = torch.empty(n.value + 256, dtype=torch.uint8, device=device)
        off = (-raw.data_ptr()) % 256
        self._raw = raw
        self.buf = raw[off:off + n.value]
        self.c = MetaPrefix()
        self.producer = producer
        check(lib().hymba_meta_prefix_build(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(meta_rows), ptr(self.buf),
                                            n.value, None if producer is None else ctypes.byref(producer.c),
                                            ctypes.byref(self.c), ptr(meta_out), ptr(ws), ws.numel(),
                                            stream_handle(stream)))
        self.dims = dims

    def tensor(self, name):
        """Device view of the prefix's k / v [M, Hkv, D] fp16, ssm_state [Di, S] or conv_state
        [Di, 3] fp32 (a consumer's k / v live in its producer's buffer)."""
        d = self.dims
        shapes = {"k": ((d.n_meta, d.n_kv_heads, d.head_dim), torch.float16),
                  "v": ((d.n_meta, d.n_kv_heads, d.head_dim), torch.float16),
                  "ssm_state": ((d.d_inner, d.d_state), torch.float32),
                  "conv_state": ((d.d_inner, d.d_conv - 1), torch.float32)}
        shape, dt = shapes[name]
        owner = self.producer if name in ("k", "v") and self.producer is not None else self
        off = getattr(self.c, name) - owner.buf.data_ptr()
        n = int(np.prod(shape)) * torch.tensor([], dtype=dt).element_size()
        return owner.buf[off:off + n].view(dt).view(*shape)


def mixer_prefill_prefix(dims, dw: DeviceWeights, x, prefix: Prefix, kv: Cache, out, ws, ssm_state=None,
                         conv_state=None, residual=None, stream=None, cfg=None):
    """hymba_mixer_prefill of the input rows only, from a precomputed meta-token prefix."""
    cfg = make_cfg(dims) if cfg is None else cfg
    B, n_tokens = x.shape[0], x.shape[1]
    check(lib().hymba_mixer_prefill_prefix(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x), B, n_tokens,
                                           ctypes.byref(prefix.c), ctypes.byref(kv.c), ptr(ssm_state),
                                           ptr(conv_state), ptr(residual), ptr(out), ptr(ws), ws.numel(),
                                           stream_handle(stream)))


def mixer_decode(dims, dw: DeviceWeights, x, position, kv: Cache, ssm_state, conv_state, out, ws, residual=None,
                 stream=None, cfg=None):
    cfg = make_cfg(dims) if cfg is None else cfg
    check(lib().hymba_mixer_decode(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x), x.shape[0], position,
                                   ctypes.byref(kv.c), ptr(ssm_state), ptr(conv_state), ptr(residual), ptr(out),
                                   ptr(ws), ws.numel(), stream_handle(stream)))


def mixer_decode_norm(dims, dw: DeviceWeights, x, position, kv: Cache, ssm_state, conv_state, out, norm_gain,
                      norm_eps, norm_out, ws, residual=None, stream=None, cfg=None):
    """hymba_mixer_decode_norm: the decode step, and norm_out = RMSNorm(out) * norm_gain."""
    cfg = make_cfg(dims) if cfg is None else cfg
    check(lib().hymba_mixer_decode_norm(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x), x.shape[0], position,
                                        ctypes.byref(kv.c), ptr(ssm_state), ptr(conv_state), ptr(residual), ptr(out),
                                        ptr(norm_gain), norm_eps, ptr(norm_out), ptr(ws), ws.numel(),
                                        stream_handle(stream)))


def mixer_decode_ragged(dims, dw: DeviceWeights, x, positions, max_position, kv: Cache, ssm_state, conv_state, out,
                        ws, residual=None, stream=None, cfg=None):
    """hymba_mixer_decode with a position per sequence: positions is an int32 device tensor [B]."""
    assert positions.dtype == torch.int32 and positions.is_cuda and positions.numel() == x.shape[0]
    cfg = make_cfg(dims) if cfg is None else cfg
    check(lib().hymba_mixer_decode_ragged(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x), x.shape[0], ptr(positions),
                                          max_position, ctypes.byref(kv.c), ptr(ssm_state), ptr(conv_state),
                                          ptr(residual), ptr(out), ptr(ws), ws.numel(), stream_handle(stream)))


def mixer_decode_noalloc(dims, dw: DeviceWeights, x, position, kv: Cache, ssm_state, conv_state, out,
                         residual=None, stream=None, cfg=None):
    """hymba_mixer_decode with the library's built-in scratch instead of a workspace."""
    cfg = make_cfg(dims) if cfg is None else cfg
    check(lib().hymba_mixer_decode_noalloc(ctypes.byref(cfg), ctypes.byref(dw.c), ptr(x), x.shape[0], position,
                                           ctypes.byref(kv.c), ptr(ssm_state), ptr(conv_state), ptr(residual),
                                           ptr(out), stream_handle(stream)))


def gemm_bf16(A, B, C, status_ws, residual=None, stream=None):
    M, K = A.shape
    N = B.shape[0]
    check(lib().hymba_gemm_bf16(ptr(A), ptr(B), ptr(residual), ptr(C), M, N, K, ptr(status_ws),
                                stream_handle(stream)))


def rmsnorm(x, gain, eps, out, stream=None):
    rows, d = x.shape
    check(lib().hymba_rmsnorm(ptr(x), ptr(gain), rows, d, eps, ptr(out), stream_handle(stream)))


def ffn_swiglu(h, w_gate_up, w_down, act, out, status_ws, residual=None, stream=None):
    rows, d = h.shape
    F = w_down.shape[1]
    check(lib().hymba_ffn_swiglu(ptr(h), ptr(w_gate_up), ptr(w_down), rows, d, F, ptr(act), ptr(residual),
                                 ptr(out), ptr(status_ws), stream_handle(stream)))


def prepend_meta(meta, x, out, stream=None):
    """out[b] = [meta; x[b]] (bf16, on the device)."""
    B, N, d = x.shape
    M = 0 if meta is None else meta.shape[0]
    check(lib().hymba_prepend_meta(ptr(meta), ptr(x), B, M, N, d, ptr(out), stream_handle(stream)))


def interleave_gate_up(w_gate, w_up):
    """Stack gate and up rows in blocks of 32, the layout hymba_ffn_swiglu reads."""
    F, d = w_gate.shape
    g = w_gate.reshape(F // 32, 32, d)
    u = w_up.reshape(F // 32, 32, d)
    return np.concatenate([g, u], axis=1).reshape(2 * F, d)


def ffn_workspace_size(rows, d, F) -> int:
    n = ctypes.c_size_t()
    check(lib().hymba_ffn_workspace_size(rows, d, F, ctypes.byref(n)))
    return n.value


def ffn_swiglu_decode(h, w_gate_up, w_down, out, ws, residual=None, stream=None):
    """hymba_ffn_swiglu_decode: the SwiGLU FFN of a few rows (decode), ws sized by ffn_workspace_size."""
    rows, d = h.shape
    F = w_down.shape[1]
    check(lib().hymba_ffn_swiglu_decode(ptr(h), ptr(w_gate_up), ptr(w_down), rows, d, F, ptr(residual), ptr(out),
                                        ptr(ws), ws.numel(), stream_handle(stream)))


def l2_prefetch(tensors, stream=None):
    """hymba_l2_prefetch: an L2 prefetch hint for up to 8 device tensors (read-only ranges)."""
    n = len(tensors)
    ptrs = (_vp * n)(*[t.data_ptr() for t in tensors])
    sizes = (_c_size * n)(*[t.numel() * t.element_size() for t in tensors])
    check(lib().hymba_l2_prefetch(ptrs, sizes, n, stream_handle(stream)))


def ffn_swiglu_decode_norm(h, w_gate_up, w_down, out, norm_gain, norm_eps, norm_out, ws, residual=None,
                           stream=None):
    """hymba_ffn_swiglu_decode_norm: the decode FFN, and norm_out = RMSNorm(out) * norm_gain."""
    rows, d = h.shape
    F = w_down.shape[1]
    check(lib().hymba_ffn_swiglu_decode_norm(ptr(h), ptr(w_gate_up), ptr(w_down), rows, d, F, ptr(residual), ptr(out),
                                             ptr(norm_gain), norm_eps, ptr(norm_out), ptr(ws), ws.numel(),
                                             stream_handle(stream)))


def profile_begin(max_records=8192):
    check(lib().hymba_profile_begin(max_records))


def profile_read(max_records=8192):
    """The records so far without clearing them (recording stops); after a captured CUDA
    graph replays, these are that replay's kernel times."""
    recs = (ProfRecord * max_records)()
    n = ctypes.c_int()
    check(lib().hymba_profile_read(recs, max_records, ctypes.byref(n)))
    return [(recs[i].name.decode(), float(recs[i].ms)) for i in range(n.value)]


def profile_end(max_records=8192):
    """[(kernel name, milliseconds)] of every launch since profile_begin, in launch order."""
    recs = (ProfRecord * max_records)()
    n = ctypes.c_int()
    check(lib().hymba_profile_end(recs, max_records, ctypes.byref(n)))
    return [(recs[i].name.decode(), float(recs[i].ms)) for i in range(n.value)]


def set_wait_limit_ns(ns):
    check(lib().hymba_set_wait_limit_ns(int(ns)))


def selftest_wait_timeout(ws, stream=None):
    check(lib().hymba_selftest_wait_timeout(ptr(ws), ws.numel(), stream_handle(stream)))
