"""A stack of Hymba blocks on the C ABI (the 32-layer harness): prefill and decode steps.

Each block is norm -> hybrid-head mixer -> norm -> FFN with pre-norm residuals (juejin post
"NVIDIA提出Hymba网络…", §Hymba 的整体架构).  The meta tokens are prepended once, to the
residual stream, and every layer sees them as the first rows of its input; the first,
middle and last layers attend globally, the others use a sliding window, and adjacent SWA
layers share one KV cache (hymba_kv_share_alloc plans the pairs).  A decode step runs one
new token per sequence through the same 32 blocks from the caches and the per-layer SSM and
conv states that the prefill left (model card Hymba-1.5B-Base, §步骤2: generation with the
cache).  This module only allocates device memory and calls the library: every step runs in
libhymba's kernels.
"""
from __future__ import annotations

import torch

from . import hymba as H
from . import synth


def _device_weights(dl, F, seed, layer, dt_mean, dt_std, device):
    """Random-init layer and block weights drawn on the device (same distributions as
    synth.layer_weights / synth.block_weights, a torch generator instead of numpy's), for
    timing runs where drawing 32 layers on the host would dominate."""
    g = torch.Generator(device=device)
    g.manual_seed(1000003 * (seed + 1) + layer)
    d, Di, S, R = dl.d_model, dl.d_inner, dl.d_state, dl.dt_rank
    n = lambda *shape, std=0.02, mean=0.0: torch.randn(*shape, generator=g, device=device) * std + mean
    w = {
        "meta": n(dl.n_meta, d), "w_in": n(dl.in_width, d), "conv_w": n(Di, dl.d_conv), "conv_b": n(Di),
        "w_x": n(R + 2 * S, Di), "w_dt": n(Di, R), "dt_bias": n(Di, std=dt_std, mean=dt_mean),
        "A": -torch.arange(1, S + 1, dtype=torch.float32, device=device).repeat(Di, 1),
        "g_attn": n(dl.attn_width, mean=1.0), "g_ssm": n(Di, mean=1.0), "w_out": n(d, dl.out_in_width),
    }
    gate, up = n(F, d), n(F, d)
    gu = torch.cat([gate.view(F // 32, 32, d), up.view(F // 32, 32, d)], dim=1).view(2 * F, d)
    blk = {"g1": n(d, mean=1.0), "g2": n(d, mean=1.0), "w_gu": gu.to(torch.bfloat16),
           "w_down": n(d, F).to(torch.float16)}
    return w, blk


class HymbaStack:
    def __init__(self, wl: synth.Workload, seed: int = 0, device="cuda", keep_host_weights=False,
                 device_init=False, decode_room=0):
        """decode_room > 0 sizes the caches for that many decode steps after the prefill and
        keeps each layer's SSM and conv state for them."""
        self.wl = wl
        dims = wl.dims
        self.B, self.N = wl.batch, wl.n_tokens
        self.T = dims.n_meta + self.N
        self.max_tokens = self.T + decode_room
        self.L = wl.n_layers
        self.F = wl.ffn_dim
        self.device = device
        is_global = [1 if i in wl.global_layers else 0 for i in range(self.L)]
        need, _, _, _ = H.kv_share_alloc(dims, is_global, self.B, self.max_tokens)
        raw = torch.empty(need + 256, dtype=torch.uint8, device=device)
        off = (-raw.data_ptr()) % 256
        self._cache_raw = raw
        self.cache_buf = raw[off:off + need]
        _, self.cache_id, self.role, caches = H.kv_share_alloc(dims, is_global, self.B, self.max_tokens,
                                                              self.cache_buf)
        self.caches = []
        for c in caches:
            holder = H.Cache.__new__(H.Cache)
            holder.t = {}
            holder.c = c
            self.caches.append(holder)
        self.layers = []
        self.host = [] if keep_host_weights else None
        for l in range(self.L):
            dl = dims.replace(is_global=is_global[l], kv_role=self.role[l])
            if device_init:
                w, dev = _device_weights(dl, self.F, seed, l, wl.dt_bias_mean, wl.dt_bias_std, device)
                self.layers.append((dl, H.DeviceWeights(w, device), dev))
                continue
            w = synth.layer_weights(dl, seed=seed, layer=l, dt_bias_mean=wl.dt_bias_mean, dt_bias_std=wl.dt_bias_std)
            bw = synth.block_weights(dl, self.F, seed=seed, layer=l)
            dev = {
                "g1": torch.from_numpy(bw["g_norm1"]).to(device),
                "g2": torch.from_numpy(bw["g_norm2"]).to(device),
                "w_gu": torch.from_numpy(H.interleave_gate_up(bw["w_gate"], bw["w_up"])).to(device).to(torch.bfloat16),
                "w_down": torch.from_numpy(bw["w_down"]).to(device).to(torch.float16),
            }
            self.layers.append((dl, H.DeviceWeights(w), dev))
            if keep_host_weights:
                self.host.append((dl, w, bw))
        # the stack's meta tokens R (those of layer 0's parameter set)
        if device_init:
            self.meta = self.layers[0][1].t["meta"]
        else:
            self.meta = torch.from_numpy(synth.layer_weights(dims, seed=seed, layer=0)["meta"]).to(device).to(
                torch.bfloat16)
        rows = self.B * self.T
        bf = dict(dtype=torch.bfloat16, device=device)
        # flat buffers, viewed as [B, T_run, d] for a prefill of T_run <= T rows
        self._hs = [torch.empty(rows * dims.d_model, **bf) for _ in range(2)]
        self._h1 = torch.empty(rows * dims.d_model, **bf)
        self._hn = torch.empty(rows * dims.d_model, **bf)
        self.act = torch.empty(rows, self.F, dtype=torch.float16, device=device)
        ws_bytes = max(H.workspace_size(dl, self.B, self.T, 1) for dl, _, _ in self.layers)
        self.ws = H.alloc_workspace(ws_bytes)
        self.ssm = self.conv = None
        if decode_room > 0:
            f32 = dict(dtype=torch.float32, device=device)
            self.ssm = [torch.zeros(self.B, dims.d_inner, dims.d_state, **f32) for _ in range(self.L)]
            self.conv = [torch.zeros(self.B, dims.d_inner, dims.d_conv - 1, **f32) for _ in range(self.L)]
            dec = max(H.workspace_size(dl, self.B, self.max_tokens, 0, H.MODE_DECODE) for dl, _, _ in self.layers)
            self.dws = H.alloc_workspace(dec)
            self.dh = [torch.empty(self.B, dims.d_model, **bf) for _ in range(2)]
            self.dh1 = torch.empty(self.B, dims.d_model, **bf)
            self.dhn = torch.empty(self.B, dims.d_model, **bf)
            self.dhn2 = torch.empty(self.B, dims.d_model, **bf)
            self.fws = H.alloc_workspace(H.ffn_workspace_size(self.B, dims.d_model, self.F))

    def cache_view(self, ptr_value, max_tokens, dl):
        """fp16 view [B, max_tokens, Hkv, D] of a K or V buffer carved out of cache_buf."""
        off = ptr_value - self.cache_buf.data_ptr()
        n = self.B * max_tokens * dl.n_kv_heads * dl.head_dim * 2
        return self.cache_buf[off:off + n].view(torch.float16).view(self.B, max_tokens, dl.n_kv_heads, dl.head_dim)

    def forward(self, E, record=None):
        """E [B, n, d] bf16 on the device (n <= N input tokens) -> residual stream after the
        last layer [B, M + n, d].  record: optional dict layer -> list, filled with (H_in,
        H_mid, H_out) copies of sequence 0 and, for consumer layers, the producer K/V they
        read.  With decode_room > 0 the prefill leaves each layer's SSM and conv state for a
        decode step at position M + n."""
        d = self.wl.dims.d_model
        T = self.wl.dims.n_meta + E.shape[1]
        assert T <= self.T
        self.T_run = T
        rows = self.B * T
        hs = [b[:rows * d].view(self.B, T, d) for b in self._hs]
        h1, hn = self._h1[:rows * d].view(self.B, T, d), self._hn[:rows * d].view(self.B, T, d)
        cur = 0
        H.prepend_meta(self.meta, E, hs[cur])
        for l, (dl, dw, dev) in enumerate(self.layers):
            Hin = hs[cur]
            Hout = hs[1 - cur]
            kv = self.caches[self.cache_id[l]]
            if record is not None and l in record and dl.kv_role == H.KV_CONSUMER:
                view_k = self.cache_view(kv.c.k, kv.c.max_tokens, dl)
                view_v = self.cache_view(kv.c.v, kv.c.max_tokens, dl)
                record[l].append(("kv", view_k[0, :T].float().cpu().numpy(),
                                  view_v[0, :T].float().cpu().numpy()))
            H.rmsnorm(Hin.view(rows, d), dev["g1"], dl.norm_eps, hn.view(rows, d))
            st = {} if self.ssm is None else dict(ssm_state=self.ssm[l], conv_state=self.conv[l])
            H.mixer_prefill(dl, dw, hn, kv, h1, self.ws, x_has_meta=1, residual=Hin, **st)
            H.rmsnorm(h1.view(rows, d), dev["g2"], dl.norm_eps, hn.view(rows, d))
            H.ffn_swiglu(hn.view(rows, d), dev["w_gu"], dev["w_down"], self.act[:rows], Hout.view(rows, d), self.ws,
                         residual=h1.view(rows, d))
            if record is not None and l in record:
                record[l].append(("h", Hin[0].float().cpu().numpy(), h1[0].float().cpu().numpy(),
                                  Hout[0].float().cpu().numpy()))
            cur = 1 - cur
        return hs[cur]

    def layer_cache_tensors(self, l):
        """Device views of layer l's cache: SWA meta_k/meta_v [B, M, Hkv, D] and ring_k/ring_v
        [B, W, Hkv, D], or a global layer's k/v [B, max_tokens, Hkv, D]."""
        dl = self.layers[l][0]
        c = self.caches[self.cache_id[l]].c

        def view(ptr_value, rows):
            off = ptr_value - self.cache_buf.data_ptr()
            n = self.B * rows * dl.n_kv_heads * dl.head_dim * 2
            return self.cache_buf[off:off + n].view(torch.float16).view(self.B, rows, dl.n_kv_heads, dl.head_dim)

        if dl.is_global:
            return {"k": view(c.k, c.max_tokens), "v": view(c.v, c.max_tokens)}
        return {"meta_k": view(c.meta_k, dl.n_meta), "meta_v": view(c.meta_v, dl.n_meta),
                "ring_k": view(c.ring_k, dl.window), "ring_v": view(c.ring_v, dl.window)}

    def decode_step(self, x, position, record=None):
        """One new token per sequence through all layers: x [B, d] bf16 (its embedding) at
        `position` (meta rows counted; the first decode step after a prefill of T rows is at
        position T).  Returns the residual stream after the last layer [B, d] (a view that the
        next step overwrites).  record: optional dict layer -> dict, filled with host copies
        of the layer's normalised mixer input, caches and states before its step, and of the
        stream after its mixer and after its FFN."""
        assert self.ssm is not None, "build the stack with decode_room > 0"
        assert self.wl.dims.n_meta < position < self.max_tokens
        cur = 0
        self.dh[cur].copy_(x)
        # only the first layer's input norm runs on its own: each later norm is fused into the
        # last kernel of the sublayer before it (hymba_*_decode_norm)
        L = len(self.layers)
        H.rmsnorm(self.dh[cur], self.layers[0][2]["g1"], self.layers[0][0].norm_eps, self.dhn)
        for l, (dl, dw, dev) in enumerate(self.layers):
            hin, hout = self.dh[cur], self.dh[1 - cur]
            kv = self.caches[self.cache_id[l]]
            if record is not None and l in record:
                cache = {k: v.float().cpu().numpy() for k, v in self.layer_cache_tensors(l).items()}
                record[l].update(h_in=hin.float().cpu().numpy(), hn=self.dhn.float().cpu().numpy(), cache=cache,
                                 ssm=self.ssm[l].cpu().numpy(), conv=self.conv[l].cpu().numpy())
            H.mixer_decode_norm(dl, dw, self.dhn, position, kv, self.ssm[l], self.conv[l], self.dh1, dev["g2"],
                                dl.norm_eps, self.dhn2, self.dws, residual=hin)
            if l + 1 < L:
                ndl, _, ndev = self.layers[l + 1]
                H.ffn_swiglu_decode_norm(self.dhn2, dev["w_gu"], dev["w_down"], hout, ndev["g1"], ndl.norm_eps,
                                         self.dhn, self.fws, residual=self.dh1)
            else:
                H.ffn_swiglu_decode(self.dhn2, dev["w_gu"], dev["w_down"], hout, self.fws, residual=self.dh1)
            if record is not None and l in record:
                record[l].update(h_mid=self.dh1.float().cpu().numpy(), hn2=self.dhn2.float().cpu().numpy(),
                                 h_out=hout.float().cpu().numpy())
            cur = 1 - cur
        return self.dh[cur]
