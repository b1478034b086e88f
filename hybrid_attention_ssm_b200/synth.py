"""Seeded synthetic inputs for the Hymba hybrid-head mixer.

This module only draws random tensors with the shapes and value distributions of the
workloads (and rounds the ones stored in bf16 to bf16).  It holds none of the method's
arithmetic, so that both the CUDA path and the fp64 oracle can consume the same inputs
without sharing any computation.

Every tensor gets its own child generator ``default_rng([seed, layer, k])`` where ``k`` is
the tensor's index in a fixed name list, so adding a tensor never shifts the others.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np

# Fixed order of tensor names; the index is part of each tensor's child seed.
_NAMES = [
    "meta", "w_in", "conv_w", "conv_b", "w_x", "w_dt", "dt_bias", "A", "g_attn", "g_ssm",
    "w_out", "x", "residual", "meta_k", "meta_v", "ring_k", "ring_v", "ssm_state",
    "conv_state", "x_new", "g_norm1", "g_norm2", "w_gate", "w_up", "w_down", "embed",
    "kv_k", "kv_v",
]
KV_OWN, KV_PRODUCER, KV_CONSUMER = 0, 1, 2


@dataclass
class LayerDims:
    """Per-layer sizes, named after the pages' problem statement."""
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_inner: int
    d_state: int
    d_conv: int
    dt_rank: int
    window: int
    n_meta: int
    is_global: int = 0
    kv_role: int = KV_OWN
    rope_base: float = 10000.0
    norm_eps: float = 1e-6

    @property
    def attn_width(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_width(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def in_width(self) -> int:
        """Rows of W_in: [Q | K | V | x | z], without K/V for a consumer layer."""
        kv = 0 if self.kv_role == KV_CONSUMER else 2 * self.kv_width
        return self.attn_width + kv + 2 * self.d_inner

    @property
    def out_in_width(self) -> int:
        return self.attn_width + self.d_inner

    def replace(self, **kw) -> "LayerDims":
        return dataclasses.replace(self, **kw)


@dataclass
class Workload:
    name: str
    dims: LayerDims
    batch: int
    n_tokens: int               # input tokens N per sequence (meta excluded)
    dt_bias_mean: float = 0.0
    dt_bias_std: float = 0.02
    n_layers: int = 1
    global_layers: tuple = ()
    ffn_dim: int = 0
    decode_position: int = 0    # position p of the new token (decode workloads)
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def seq_len(self) -> int:
        return self.dims.n_meta + self.n_tokens


def _hymba_dims(**kw) -> LayerDims:
    base = dict(d_model=1600, n_q_heads=25, n_kv_heads=5, head_dim=64, d_inner=3200,
                d_state=16, d_conv=4, dt_rank=100, window=1024, n_meta=128)
    base.update(kw)
    return LayerDims(**base)


def workloads() -> dict:
    """The five workloads: tiny parity layer, Hymba-1.5B-shaped SWA and global prefill
    layers, the shared-KV SWA decode pair, and the 32-layer stack."""
    tiny = LayerDims(d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64, d_inner=512,
                     d_state=16, d_conv=4, dt_rank=16, window=32, n_meta=8)
    return {
        "tiny": Workload("tiny", tiny, batch=1, n_tokens=120),
        "tiny_full": Workload("tiny_full", tiny.replace(window=128), batch=1, n_tokens=120),
        "swa": Workload("swa", _hymba_dims(), batch=1, n_tokens=2048,
                        dt_bias_mean=-4.0, dt_bias_std=1.0),
        "global": Workload("global", _hymba_dims(is_global=1), batch=4, n_tokens=8192,
                           dt_bias_mean=-4.0, dt_bias_std=1.0),
        "decode_pair": Workload("decode_pair", _hymba_dims(kv_role=KV_PRODUCER), batch=64,
                                n_tokens=4000, dt_bias_mean=-4.0, dt_bias_std=1.0,
                                decode_position=128 + 4000),
        "stack": Workload("stack", _hymba_dims(), batch=8, n_tokens=4096,
                          dt_bias_mean=-4.0, dt_bias_std=1.0, n_layers=32,
                          global_layers=(0, 15, 31), ffn_dim=5504),
    }


def _rng(seed: int, layer: int, name: str) -> np.random.Generator:
    return np.random.default_rng([seed, layer, _NAMES.index(name)])


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), returned as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32)
    return np.where(np.isfinite(a), out, a).astype(np.float32)


def normal(seed, layer, name, shape, mean=0.0, std=1.0, bf16=True) -> np.ndarray:
    a = _rng(seed, layer, name).normal(mean, std, size=shape).astype(np.float32)
    return bf16_round(a) if bf16 else a


def layer_weights(dims: LayerDims, seed: int = 0, layer: int = 0,
                  dt_bias_mean: float = 0.0, dt_bias_std: float = 0.02) -> dict:
    """Weights of one mixer layer.  bf16 tensors come back bf16-rounded in float32.

    Shapes: meta [M,d]; w_in [P,d] rows [Q|K|V|x|z]; conv_w [Di,kc]; conv_b [Di];
    w_x [R+2S, Di] rows [dt_low|B|C]; w_dt [Di,R]; dt_bias [Di]; A [Di,S];
    g_attn [Hq*D]; g_ssm [Di]; w_out [d, Hq*D+Di].
    """
    d, Di, S, R = dims.d_model, dims.d_inner, dims.d_state, dims.dt_rank
    s = 0.02
    w = {
        "meta": normal(seed, layer, "meta", (dims.n_meta, d), std=s),
        "w_in": normal(seed, layer, "w_in", (dims.in_width, d), std=s),
        "conv_w": normal(seed, layer, "conv_w", (Di, dims.d_conv), std=s, bf16=False),
        "conv_b": normal(seed, layer, "conv_b", (Di,), std=s, bf16=False),
        "w_x": normal(seed, layer, "w_x", (R + 2 * S, Di), std=s),
        "w_dt": normal(seed, layer, "w_dt", (Di, R), std=s),
        "dt_bias": normal(seed, layer, "dt_bias", (Di,), mean=dt_bias_mean,
                          std=dt_bias_std, bf16=False),
        "A": np.tile(-np.arange(1, S + 1, dtype=np.float32), (Di, 1)),
        "g_attn": 1.0 + normal(seed, layer, "g_attn", (dims.attn_width,), std=s, bf16=False),
        "g_ssm": 1.0 + normal(seed, layer, "g_ssm", (Di,), std=s, bf16=False),
        "w_out": normal(seed, layer, "w_out", (d, dims.out_in_width), std=s),
    }
    return w


def prefill_input(wl: Workload, seed: int = 0, layer: int = 0) -> np.ndarray:
    """X [B, N, d] drawn N(0,1), bf16-rounded."""
    return normal(seed, layer, "x", (wl.batch, wl.n_tokens, wl.dims.d_model))


def decode_state(wl: Workload, seed: int = 0, layer: int = 0) -> dict:
    """Decode-step inputs and cache contents, all N(0,1): new token x [B,d]; meta K/V
    [B,M,Hkv,D]; ring K/V [B,W,Hkv,D]; SSM state [B,Di,S] fp32; conv state [B,Di,kc-1] fp32."""
    dm = wl.dims
    B, M, W, Hkv, D = wl.batch, dm.n_meta, dm.window, dm.n_kv_heads, dm.head_dim
    return {
        "x_new": normal(seed, layer, "x_new", (B, dm.d_model)),
        "meta_k": normal(seed, layer, "meta_k", (B, M, Hkv, D)),
        "meta_v": normal(seed, layer, "meta_v", (B, M, Hkv, D)),
        "ring_k": normal(seed, layer, "ring_k", (B, W, Hkv, D)),
        "ring_v": normal(seed, layer, "ring_v", (B, W, Hkv, D)),
        "ssm_state": normal(seed, layer, "ssm_state", (B, dm.d_inner, dm.d_state), bf16=False),
        "conv_state": normal(seed, layer, "conv_state", (B, dm.d_inner, dm.d_conv - 1),
                             bf16=False),
    }


def global_cache(wl: Workload, max_tokens: int, seed: int = 0, layer: int = 0) -> dict:
    """Full-length K/V cache contents [B, max_tokens, Hkv, D], N(0,1)."""
    dm = wl.dims
    shape = (wl.batch, max_tokens, dm.n_kv_heads, dm.head_dim)
    return {"k": normal(seed, layer, "kv_k", shape), "v": normal(seed, layer, "kv_v", shape)}


def block_weights(dims: LayerDims, ffn_dim: int, seed: int = 0, layer: int = 0) -> dict:
    """Block extras around the mixer: two RMSNorm gains and the SwiGLU FFN."""
    d, s = dims.d_model, 0.02
    return {
        "g_norm1": 1.0 + normal(seed, layer, "g_norm1", (d,), std=s, bf16=False),
        "g_norm2": 1.0 + normal(seed, layer, "g_norm2", (d,), std=s, bf16=False),
        "w_gate": normal(seed, layer, "w_gate", (ffn_dim, d), std=s),
        "w_up": normal(seed, layer, "w_up", (ffn_dim, d), std=s),
        "w_down": normal(seed, layer, "w_down", (d, ffn_dim), std=s),
    }


def stack_embeddings(wl: Workload, seed: int = 0) -> np.ndarray:
    """Token embeddings [B, N, d] N(0,1) for the stack workload."""
    return normal(seed, 0, "embed", (wl.batch, wl.n_tokens, wl.dims.d_model))
