"""fp64 CPU oracle for the Hymba hybrid-head mixer (test infrastructure only).

This is the plain, slow, obviously-correct statement of what the mixer computes.  Only the
tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  It shares no code with the CUDA path, and the CUDA path never
calls it.

Sources (cited by page title and section):
  [JJ]  juejin.cn post "NVIDIA提出Hymba网络，Mamba+Attenation解决transformer的长序列低效难题":
        §深入理解混合头模块 (hybrid-head module), §深入理解元 Tokens (meta tokens),
        §Hymba 的整体架构 (block layout, global/SWA layers, cross-layer KV sharing),
        §数学表示 1-6 (the equations: meta prefix, input projection, eq. (1) attention,
        eq. (2) SSM heads, output fusion with normalisation and beta rescale).
  [MC]  model card "Hymba-1.5B-Base" (model.aibase.cn), §模型概述 / §模型架构: sizes, GQA,
        RoPE, 16 SSM states, 3 full-attention layers, meta tokens visible to every token.
Where the pages are silent the reading used is named in the docstring (R-numbers refer to
the readings list kept with the design notes).

All arithmetic is float64 on the given (bf16-rounded) inputs.  Matrix products use numpy's
matmul as a library primitive; nothing is blocked, fused or reordered beyond the
definitions.

Parity pins: every function here, the SwiGLU FFN and the block composition included, is
pinned by tests/test_oracle_pins.py except the RoPE pairing convention, the 1/2 of the
average, the eps of the RMSNorm and the omitted D skip term, which are readings of silent
passages (parity unpinned for those choices only).
"""
from __future__ import annotations

import numpy as np

KV_OWN, KV_PRODUCER, KV_CONSUMER = 0, 1, 2


# ----------------------------------------------------------------------------------------
# elementwise pieces
# ----------------------------------------------------------------------------------------
def silu(x):
    """SiLU(x) = x * sigmoid(x) (the gate nonlinearity the SSM output gate G uses)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def softplus(x):
    """softplus(x) = log(1 + e^x), evaluated stably: max(x,0) + log1p(e^-|x|)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def rmsnorm(v, gain, eps):
    """RMSNorm over the last axis: v / sqrt(mean(v^2) + eps) * gain.
    [JJ] §数学表示 5: each branch output is normalised, then rescaled by a learnable
    vector (beta1 for attention, beta2 for SSM).  Reading R11: RMSNorm over the whole
    branch vector of a token."""
    v = np.asarray(v, dtype=np.float64)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * np.asarray(gain, dtype=np.float64)


# ----------------------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------------------
def rope(x, positions, base):
    """Rotary position embedding on the last axis (head dim D).

    [MC] §模型架构 names RoPE.  Reading R4: half-split pairing (x_j, x_{j+D/2}) rotated by
    angle pos * base^(-2j/D), j < D/2; positions index the meta-prefixed sequence.
    x: [..., L, H, D]; positions: [L].
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    j = np.arange(half, dtype=np.float64)
    theta = np.power(float(base), -2.0 * j / D)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]   # [L, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------------------
# attention, eq. (1)
# ----------------------------------------------------------------------------------------
def visibility_mask(n_q_pos, n_k_pos, n_meta, window, is_global):
    """Boolean [Lq, Lk] mask: whether key position j is visible to query position i.

    [JJ] §Hymba 的整体架构: the first, middle and last blocks attend globally, the rest
    use sliding-window attention.  [JJ] §Hymba简介 and [MC] §模型架构: meta tokens take
    part in every later token's attention, even under SWA.  Readings R1-R3: causal; under
    SWA key j is visible iff j <= i and (j < n_meta or i - j < window).
    """
    qi = np.asarray(n_q_pos)[:, None]
    kj = np.asarray(n_k_pos)[None, :]
    causal = kj <= qi
    if is_global:
        return causal
    return causal & ((kj < n_meta) | ((qi - kj) < window))


def attention(Q, K, V, q_pos, k_pos, n_meta, window, is_global):
    """Y_attn = softmax(Q K^T / sqrt(D)) V over the visible set, per query head.

    [JJ] §数学表示 3, eq. (1) prints softmax(QK^T)V; reading R1 adds the 1/sqrt(D) scale
    and the causal/window mask.  GQA ([MC] §模型概述: KV shared between the heads of a
    layer): query head h reads KV head floor(h * Hkv / Hq) (reading R5).
    Q: [Lq, Hq, D]; K, V: [Lk, Hkv, D]; returns [Lq, Hq, D].  Dense two-pass softmax: the
    scores of every visible pair are formed explicitly, invisible ones are dropped.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Lq, Hq, D = Q.shape
    Hkv = K.shape[1]
    mask = visibility_mask(q_pos, k_pos, n_meta, window, is_global)
    out = np.zeros((Lq, Hq, D), dtype=np.float64)
    scale = 1.0 / np.sqrt(D)
    for h in range(Hq):
        g = (h * Hkv) // Hq
        s = (Q[:, h, :] @ K[:, g, :].T) * scale              # [Lq, Lk]
        s = np.where(mask, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)                  # pass 1: row max
        p = np.where(mask, np.exp(s - m), 0.0)                # pass 2: weights
        p /= np.sum(p, axis=1, keepdims=True)
        out[:, h, :] = p @ V[:, g, :]
    return out


# ----------------------------------------------------------------------------------------
# SSM branch, eq. (2)
# ----------------------------------------------------------------------------------------
def causal_conv1d_silu(x, w, b, x_prev=None):
    """Depthwise causal conv1d over time followed by SiLU.

    Not on the pages (the workload fixes a kernel of 4).  xc[t,c] =
    SiLU(b_c + sum_k w[c,k] * x[t-(kc-1)+k, c]); times before the start read x_prev (the
    last kc-1 inputs of an earlier call) or zero.  x: [L, Di]; w: [Di, kc]; x_prev:
    [Di, kc-1] or None.  Returns (xc [L, Di], last kc-1 inputs [Di, kc-1]).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    L, Di = x.shape
    kc = w.shape[1]
    if x_prev is None:
        head = np.zeros((kc - 1, Di))
    else:
        head = np.asarray(x_prev, dtype=np.float64).T          # [kc-1, Di]
    xp = np.concatenate([head, x], axis=0)                      # [kc-1+L, Di]
    acc = np.zeros((L, Di)) + np.asarray(b, dtype=np.float64)[None, :]
    for k in range(kc):
        acc += w[None, :, k] * xp[k:k + L, :]
    return silu(acc), xp[L:, :].T.copy()


def ssm_params(xc, w_x, w_dt, dt_bias, dt_rank, d_state):
    """Delta, B, C of the selective SSM from the conv output (reading R8).

    [JJ] §数学表示 4 calls B, C and Delta learnable parameters of the SSM heads; the
    workload fixes dt_rank.  [dt_low | B | C] = xc W_x^T; Delta = softplus(dt_low W_dt^T +
    dt_bias).  xc: [L, Di]; returns Delta [L, Di], B [L, S], C [L, S].
    """
    xc = np.asarray(xc, dtype=np.float64)
    proj = xc @ np.asarray(w_x, dtype=np.float64).T
    dt_low = proj[:, :dt_rank]
    Bm = proj[:, dt_rank:dt_rank + d_state]
    Cm = proj[:, dt_rank + d_state:dt_rank + 2 * d_state]
    delta = softplus(dt_low @ np.asarray(w_dt, dtype=np.float64).T
                     + np.asarray(dt_bias, dtype=np.float64)[None, :])
    return delta, Bm, Cm, dt_low


def selective_scan(xc, delta, A, Bm, Cm, z, h0=None):
    """Sequential selective scan with the output gate.

    [JJ] §数学表示 4, eq. (2): y_i = sum_{j<=i} C_i (prod_{k=j+1..i} exp(A Delta_k)) B_j
    Delta_j x_j, which is the recurrence h_t = exp(Delta_t A) * h_{t-1} + Delta_t B_t x_t,
    y_t = C_t . h_t (reading R7: this Euler form, no D skip term R9).  Then
    Y_ssm = G * y with G = SiLU(z) (reading R10).
    xc, delta, z: [L, Di]; A: [Di, S]; Bm, Cm: [L, S]; h0: [Di, S] or None.
    Returns (y_gated [L, Di], h_L [Di, S]).
    """
    xc = np.asarray(xc, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    Cm = np.asarray(Cm, dtype=np.float64)
    L, Di = xc.shape
    h = np.zeros_like(A) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.zeros((L, Di))
    for t in range(L):
        a = np.exp(delta[t][:, None] * A)                                  # [Di, S]
        h = a * h + (delta[t] * xc[t])[:, None] * Bm[t][None, :]
        y[t] = h @ Cm[t]
    return y * silu(z), h


# ----------------------------------------------------------------------------------------
# the mixer
# ----------------------------------------------------------------------------------------
def split_in_proj(proj, dims):
    """Columns of X~ W_in^T in the order [Q | K | V | x | z] ([JJ] §数学表示 2)."""
    Hq, Hkv, D, Di = dims.n_q_heads, dims.n_kv_heads, dims.head_dim, dims.d_inner
    o = 0
    Q = proj[..., o:o + Hq * D]; o += Hq * D
    if dims.kv_role == KV_CONSUMER:
        K = V = None
    else:
        K = proj[..., o:o + Hkv * D]; o += Hkv * D
        V = proj[..., o:o + Hkv * D]; o += Hkv * D
    xs = proj[..., o:o + Di]; o += Di
    z = proj[..., o:o + Di]
    return Q, K, V, xs, z


def fuse_and_project(O_flat, y_ssm, w, dims, residual=None):
    """Y = W_out * 1/2 [beta1 * norm(Y_attn) ; beta2 * norm(Y_ssm)] (+ residual).

    [JJ] §深入理解混合头模块 and §数学表示 5: both branch outputs are normalised, rescaled
    by beta1 / beta2, averaged, and passed through the output projection.  Reading R12:
    the two branches have different widths (Hq*D vs Di), so W_out has Hq*D + Di columns
    and each branch is projected by its own slice before the two are averaged (R13: 1/2).
    """
    ua = rmsnorm(O_flat, w["g_attn"], dims.norm_eps)
    us = rmsnorm(y_ssm, w["g_ssm"], dims.norm_eps)
    u = 0.5 * np.concatenate([ua, us], axis=-1)
    out = u @ np.asarray(w["w_out"], dtype=np.float64).T
    if residual is not None:
        out = out + np.asarray(residual, dtype=np.float64)
    return out, u


def ring_slot(pos, n_meta, window):
    """Ring-buffer slot of input position pos (>= n_meta) in an SWA cache (reading R3)."""
    return (pos - n_meta) % window


def mixer_prefill(dims, w, X, x_has_meta=False, kv_in=None, residual=None):
    """One hybrid-head mixer layer over a batch of sequences (prefill).

    [JJ] §数学表示 1-6: X~ = [R, X] (meta prefix), in_proj, attention heads (eq. 1) in
    parallel with SSM heads (eq. 2), per-branch norm + beta, average, out_proj.
    X: [B, N, d] (or [B, T, d] with the prefix already in place when x_has_meta).
    kv_in: for a consumer layer, the producer's post-RoPE (K, V), each [B, T, Hkv, D]
    ([JJ] §Hymba 的整体架构: adjacent SWA blocks share one KV cache; reading R16).
    Returns a dict with out [B,T,d], K/V [B,T,Hkv,D] used by attention, ssm_state
    [B,Di,S], conv_state [B,Di,kc-1], the SWA decode cache (meta_k/v [B,M,Hkv,D],
    ring_k/v [B,W,Hkv,D]) and the intermediates of every stage.
    """
    X = np.asarray(X, dtype=np.float64)
    Bsz = X.shape[0]
    M, Hq, Hkv, D = dims.n_meta, dims.n_q_heads, dims.n_kv_heads, dims.head_dim
    if x_has_meta:
        Xt = X
    else:
        R = np.asarray(w["meta"], dtype=np.float64)
        Xt = np.concatenate([np.broadcast_to(R, (Bsz,) + R.shape), X], axis=1)
    T = Xt.shape[1]
    pos = np.arange(T)

    proj = Xt @ np.asarray(w["w_in"], dtype=np.float64).T          # [B, T, P]
    Qf, Kf, Vf, xs, z = split_in_proj(proj, dims)
    Q = rope(Qf.reshape(Bsz, T, Hq, D), pos, dims.rope_base)
    if dims.kv_role == KV_CONSUMER:
        if kv_in is None:
            raise ValueError("a consumer layer needs the producer's K/V")
        K = np.asarray(kv_in[0], dtype=np.float64)
        V = np.asarray(kv_in[1], dtype=np.float64)
    else:
        K = rope(Kf.reshape(Bsz, T, Hkv, D), pos, dims.rope_base)
        V = Vf.reshape(Bsz, T, Hkv, D)

    O = np.stack([attention(Q[b], K[b], V[b], pos, pos, M, dims.window, dims.is_global)
                  for b in range(Bsz)])                               # [B, T, Hq, D]
    O_flat = O.reshape(Bsz, T, Hq * D)

    ys, states, convs, xcs, deltas, Bms, Cms, dtl = [], [], [], [], [], [], [], []
    for b in range(Bsz):
        xc, conv_last = causal_conv1d_silu(xs[b], w["conv_w"], w["conv_b"])
        delta, Bm, Cm, dt_low = ssm_params(xc, w["w_x"], w["w_dt"], w["dt_bias"],
                                           dims.dt_rank, dims.d_state)
        y, h = selective_scan(xc, delta, w["A"], Bm, Cm, z[b])
        ys.append(y); states.append(h); convs.append(conv_last)
        xcs.append(xc); deltas.append(delta); Bms.append(Bm); Cms.append(Cm); dtl.append(dt_low)
    y_ssm = np.stack(ys)

    out, u = fuse_and_project(O_flat, y_ssm, w, dims, residual)

    res = dict(out=out, K=K, V=V, Q=Q, O=O_flat, y_ssm=y_ssm, u=u, proj=proj,
               xc=np.stack(xcs), delta=np.stack(deltas), Bm=np.stack(Bms),
               Cm=np.stack(Cms), dt_low=np.stack(dtl), z=z, x_ssm=xs,
               ssm_state=np.stack(states), conv_state=np.stack(convs))
    if not dims.is_global:
        W = dims.window
        ring_k = np.zeros((Bsz, W, Hkv, D)); ring_v = np.zeros((Bsz, W, Hkv, D))
        for p in range(max(M, T - W), T):
            s = ring_slot(p, M, W)
            ring_k[:, s] = K[:, p]; ring_v[:, s] = V[:, p]
        res.update(meta_k=K[:, :M].copy(), meta_v=V[:, :M].copy(),
                   ring_k=ring_k, ring_v=ring_v)
    return res


def mixer_decode(dims, w, x_new, position, cache, ssm_state, conv_state, residual=None):
    """One decode step of the mixer for B sequences that all sit at the same position.

    The new token (position p = M + context length, meta included) goes through the same
    stages as a prefill row: in_proj, RoPE at p, attention over the meta keys plus the
    last `window` positions (SWA) or every position <= p (global), the conv/SSM step from
    the carried conv and SSM states, norm, average and out_proj.
    cache (SWA): dict meta_k/meta_v [B,M,Hkv,D], ring_k/ring_v [B,W,Hkv,D] holding
    input position q at slot (q - M) mod W; an own/producer layer writes its new K/V into
    the ring before attending, a consumer only reads it ([JJ] §Hymba 的整体架构).
    cache (global): dict k/v [B, Lmax, Hkv, D] indexed by position.
    Returns dict(out [B,d], ssm_state, conv_state, cache) with copies of the updated state.
    """
    x_new = np.asarray(x_new, dtype=np.float64)
    Bsz = x_new.shape[0]
    M, Hq, Hkv, D, W = dims.n_meta, dims.n_q_heads, dims.n_kv_heads, dims.head_dim, dims.window
    p = int(position)
    cache = {k: np.array(v, dtype=np.float64) for k, v in cache.items()}
    proj = x_new @ np.asarray(w["w_in"], dtype=np.float64).T          # [B, P]
    Qf, Kf, Vf, xs, z = split_in_proj(proj, dims)
    Q = rope(Qf.reshape(Bsz, 1, Hq, D), [p], dims.rope_base)[:, 0]     # [B, Hq, D]
    if dims.kv_role != KV_CONSUMER:
        k_new = rope(Kf.reshape(Bsz, 1, Hkv, D), [p], dims.rope_base)[:, 0]
        v_new = Vf.reshape(Bsz, Hkv, D)
        if dims.is_global:
            cache["k"][:, p] = k_new; cache["v"][:, p] = v_new
        else:
            s = ring_slot(p, M, W)
            cache["ring_k"][:, s] = k_new; cache["ring_v"][:, s] = v_new

    O = np.zeros((Bsz, Hq, D))
    for b in range(Bsz):
        if dims.is_global:
            kpos = np.arange(p + 1)
            Kb, Vb = cache["k"][b, :p + 1], cache["v"][b, :p + 1]
        else:
            win = np.arange(max(M, p - W + 1), p + 1)
            kpos = np.concatenate([np.arange(M), win])
            slots = ring_slot(win, M, W)
            Kb = np.concatenate([cache["meta_k"][b], cache["ring_k"][b, slots]], axis=0)
            Vb = np.concatenate([cache["meta_v"][b], cache["ring_v"][b, slots]], axis=0)
        O[b] = attention(Q[b][None], Kb, Vb, [p], kpos, M, W, dims.is_global)[0]
    O_flat = O.reshape(Bsz, Hq * D)

    y = np.zeros((Bsz, dims.d_inner))
    new_ssm = np.zeros_like(np.asarray(ssm_state, dtype=np.float64))
    new_conv = np.zeros_like(np.asarray(conv_state, dtype=np.float64))
    for b in range(Bsz):
        xc, conv_last = causal_conv1d_silu(xs[b][None, :], w["conv_w"], w["conv_b"],
                                           x_prev=conv_state[b])
        delta, Bm, Cm, _ = ssm_params(xc, w["w_x"], w["w_dt"], w["dt_bias"],
                                      dims.dt_rank, dims.d_state)
        yb, h = selective_scan(xc, delta, w["A"], Bm, Cm, z[b][None, :], h0=ssm_state[b])
        y[b] = yb[0]; new_ssm[b] = h; new_conv[b] = conv_last

    out, _ = fuse_and_project(O_flat, y, w, dims, residual)
    return dict(out=out, ssm_state=new_ssm, conv_state=new_conv, cache=cache,
                O=O_flat, y_ssm=y)


# ----------------------------------------------------------------------------------------
# cross-layer KV sharing plan and the block (stack harness)
# ----------------------------------------------------------------------------------------
def kv_share_plan(is_global):
    """Pair adjacent SWA layers so each pair keeps one KV cache.

    [JJ] §Hymba 的整体架构: for SWA blocks, neighbouring blocks share their KV cache
    instead of each keeping its own; global blocks keep their own.  Reading R16: walk the
    layers in order; an SWA layer whose predecessor is an SWA layer that opened a pair
    becomes that pair's consumer; any other SWA layer opens a pair as producer (and stays
    an own-KV layer if its successor cannot join).  Returns (cache_id[], role[]).
    """
    n = len(is_global)
    cache_id, role = [0] * n, [KV_OWN] * n
    next_id = 0
    i = 0
    while i < n:
        if is_global[i]:
            cache_id[i], role[i] = next_id, KV_OWN
            next_id += 1; i += 1
            continue
        if i + 1 < n and not is_global[i + 1]:
            cache_id[i] = cache_id[i + 1] = next_id
            role[i], role[i + 1] = KV_PRODUCER, KV_CONSUMER
            next_id += 1; i += 2
        else:
            cache_id[i], role[i] = next_id, KV_OWN
            next_id += 1; i += 1
    return cache_id, role


def ffn_swiglu(v, bw):
    """SwiGLU feed-forward: W_down (SiLU(W_gate v) * (W_up v)) ([JJ] §Hymba 的整体架构
    names the FFN; the workload fixes SwiGLU with the model card's intermediate size)."""
    v = np.asarray(v, dtype=np.float64)
    g = v @ np.asarray(bw["w_gate"], dtype=np.float64).T
    u = v @ np.asarray(bw["w_up"], dtype=np.float64).T
    return (silu(g) * u) @ np.asarray(bw["w_down"], dtype=np.float64).T


def hymba_block(dims, w, bw, H, kv_in=None):
    """One Hymba block on the residual stream H [B, T, d] (meta rows included):
    H1 = H + mixer(norm(H)); out = H1 + FFN(norm(H1)).  [JJ] §Hymba 的整体架构 lists
    norm, hybrid-head module, norm, FFN; reading R15: pre-norm residuals."""
    h_in = rmsnorm(H, bw["g_norm1"], dims.norm_eps)
    r = mixer_prefill(dims, w, h_in, x_has_meta=True, kv_in=kv_in, residual=H)
    H1 = r["out"]
    out = H1 + ffn_swiglu(rmsnorm(H1, bw["g_norm2"], dims.norm_eps), bw)
    return out, r
