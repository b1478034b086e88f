"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these tests re-types the oracle's formulas: each compares the oracle with a hand
derivation, a brute-force evaluation of a printed equation, a library routine, or an
invariant, chosen so that a dropped term, a wrong sign or index, or a transposed operand
in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from hybrid_attention_ssm_b200 import synth
from oracle import hymba_oracle as orc

TINY = synth.workloads()["tiny"]


def _small_dims(**kw):
    base = dict(d_model=32, n_q_heads=4, n_kv_heads=2, head_dim=8, d_inner=16, d_state=4,
                d_conv=4, dt_rank=4, window=5, n_meta=3)
    base.update(kw)
    return synth.LayerDims(**base)


def _weights(dims, seed=1, dt_mean=0.0, dt_std=0.5):
    return {k: v.astype(np.float64) for k, v in
            synth.layer_weights(dims, seed=seed, dt_bias_mean=dt_mean, dt_bias_std=dt_std).items()}


def _x(B, N, d, seed=2):
    return np.random.default_rng(seed).normal(size=(B, N, d))


# ---------------------------------------------------------------------------------------
# SSM: eq. (2) by brute force, hand-derived cases, state carry
# ---------------------------------------------------------------------------------------
def _scan_bruteforce(xc, delta, A, Bm, Cm, z):
    """Eq. (2) written as the unrolled double sum with an explicit product, loops only."""
    L, Di = xc.shape
    S = A.shape[1]
    y = np.zeros((L, Di))
    for c in range(Di):
        for i in range(L):
            acc = 0.0
            for j in range(i + 1):
                for s in range(S):
                    prod = 1.0
                    for k in range(j + 1, i + 1):
                        prod *= math.exp(A[c, s] * delta[k, c])
                    acc += Cm[i, s] * prod * Bm[j, s] * delta[j, c] * xc[j, c]
            g = z[i, c] / (1.0 + math.exp(-z[i, c]))
            y[i, c] = acc * g
    return y


def test_scan_matches_bruteforce_eq2():
    rng = np.random.default_rng(5)
    L, Di, S = 11, 3, 4
    xc = rng.normal(size=(L, Di))
    delta = rng.uniform(0.05, 1.5, size=(L, Di))
    A = -rng.uniform(0.2, 3.0, size=(Di, S))
    Bm, Cm, z = rng.normal(size=(L, S)), rng.normal(size=(L, S)), rng.normal(size=(L, Di))
    y, _ = orc.selective_scan(xc, delta, A, Bm, Cm, z)
    np.testing.assert_allclose(y, _scan_bruteforce(xc, delta, A, Bm, Cm, z), rtol=1e-12, atol=1e-12)


def test_scan_hand_derived(golden_dir):
    with open(os.path.join(golden_dir, "scan_closed_form.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        y, h = orc.selective_scan(np.array(c["x"]), np.array(c["delta"]), np.array(c["A"]),
                                  np.array(c["B"]), np.array(c["C"]), np.array(c["z"]))
        np.testing.assert_allclose(y, np.array(c["y"]), rtol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(h, np.array(c["h_last"]), rtol=1e-13, err_msg=c["name"])


def test_scan_state_carry_is_associative():
    """Scanning [0,t) then [t,L) from the carried state equals one scan over [0,L), for
    every split point (the composition (a,b)o(a',b') = (aa', a'b+b') is associative)."""
    rng = np.random.default_rng(6)
    L, Di, S = 17, 5, 3
    xc, delta = rng.normal(size=(L, Di)), rng.uniform(0.01, 1.0, size=(L, Di))
    A = -rng.uniform(0.5, 4.0, size=(Di, S))
    Bm, Cm, z = rng.normal(size=(L, S)), rng.normal(size=(L, S)), rng.normal(size=(L, Di))
    y_full, h_full = orc.selective_scan(xc, delta, A, Bm, Cm, z)
    for t in (1, 4, 9, 16):
        y1, h1 = orc.selective_scan(xc[:t], delta[:t], A, Bm[:t], Cm[:t], z[:t])
        y2, h2 = orc.selective_scan(xc[t:], delta[t:], A, Bm[t:], Cm[t:], z[t:], h0=h1)
        np.testing.assert_allclose(np.concatenate([y1, y2]), y_full, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(h2, h_full, rtol=1e-12)


def test_scan_zero_delta_keeps_state():
    """Delta = 0: exp(0)=1 keeps the state and the input term vanishes."""
    rng = np.random.default_rng(7)
    h0 = rng.normal(size=(3, 4))
    y, h = orc.selective_scan(rng.normal(size=(5, 3)), np.zeros((5, 3)), -np.ones((3, 4)),
                              rng.normal(size=(5, 4)), np.ones((5, 4)), np.full((5, 3), 30.0), h0=h0)
    np.testing.assert_allclose(h, h0)
    np.testing.assert_allclose(y, np.tile(h0.sum(1), (5, 1)) * 30.0, rtol=1e-12)


# ---------------------------------------------------------------------------------------
# conv1d, softplus, SiLU, RMSNorm
# ---------------------------------------------------------------------------------------
def test_conv_one_hot_is_shift():
    rng = np.random.default_rng(8)
    L, Di, kc = 9, 3, 4
    x = rng.normal(size=(L, Di))
    for k in range(kc):
        w = np.zeros((Di, kc)); w[:, k] = 1.0
        xc, _ = orc.causal_conv1d_silu(x, w, np.zeros(Di))
        lag = kc - 1 - k
        shifted = np.concatenate([np.zeros((lag, Di)), x[:L - lag]])
        np.testing.assert_allclose(xc, shifted / (1 + np.exp(-shifted)), rtol=1e-14)


def test_conv_state_carry():
    rng = np.random.default_rng(9)
    x, w, b = rng.normal(size=(12, 4)), rng.normal(size=(4, 4)), rng.normal(size=4)
    full, last_full = orc.causal_conv1d_silu(x, w, b)
    a, st = orc.causal_conv1d_silu(x[:7], w, b)
    c, last = orc.causal_conv1d_silu(x[7:], w, b, x_prev=st)
    np.testing.assert_allclose(np.concatenate([a, c]), full, rtol=1e-14)
    np.testing.assert_allclose(last, last_full)
    np.testing.assert_allclose(last_full, x[-3:].T)


def test_x_proj_column_layout():
    """The boundary fixes the rows of W_x as [dt_low (R) | B (S) | C (S)].  With W_x a row
    selection the projection hands out xc's own columns, so each output must be the
    corresponding slice of xc; with W_dt = 0, Delta is softplus(bias) in every row."""
    rng = np.random.default_rng(13)
    L, Di, R, S = 5, 12, 3, 4
    xc = rng.normal(size=(L, Di))
    w_x = np.eye(R + 2 * S, Di)
    bias = rng.normal(size=Di)
    delta, Bm, Cm, dt_low = orc.ssm_params(xc, w_x, np.zeros((Di, R)), bias, R, S)
    np.testing.assert_array_equal(dt_low, xc[:, :R])
    np.testing.assert_array_equal(Bm, xc[:, R:R + S])
    np.testing.assert_array_equal(Cm, xc[:, R + S:R + 2 * S])
    np.testing.assert_allclose(delta, np.log1p(np.exp(bias))[None, :].repeat(L, axis=0), rtol=1e-15)


def test_elementwise_closed_forms():
    assert orc.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert orc.softplus(50.0) == pytest.approx(50.0, rel=1e-15)
    assert orc.softplus(-50.0) == pytest.approx(math.exp(-50.0), rel=1e-12)
    assert orc.softplus(math.log(3.0)) == pytest.approx(math.log(4.0), rel=1e-15)
    assert orc.silu(0.0) == 0.0
    assert orc.silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    v = np.array([3.0, 4.0])
    np.testing.assert_allclose(orc.rmsnorm(v, [1.0, 2.0], 0.0),
                               [3.0 / math.sqrt(12.5), 8.0 / math.sqrt(12.5)], rtol=1e-15)


# ---------------------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------------------
def _mask_loops(T, M, W, is_global):
    m = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for j in range(T):
            if j <= i and (is_global or j < M or i - j < W):
                m[i, j] = True
    return m


@pytest.mark.parametrize("is_global,W,M", [(1, 0, 3), (0, 4, 3), (0, 1, 2), (0, 7, 0)])
def test_attention_matches_torch_sdpa(is_global, W, M):
    """GQA with replicated KV heads == MHA; MHA with the mask == torch SDPA in fp64."""
    rng = np.random.default_rng(10)
    T, Hq, Hkv, D = 13, 6, 2, 8
    Q, K, V = rng.normal(size=(T, Hq, D)), rng.normal(size=(T, Hkv, D)), rng.normal(size=(T, Hkv, D))
    pos = np.arange(T)
    o = orc.attention(Q, K, V, pos, pos, M, W, is_global)
    rep = Hq // Hkv
    Kr = np.repeat(K, rep, axis=1)     # query head h -> kv head h // rep
    Vr = np.repeat(V, rep, axis=1)
    mask = torch.from_numpy(_mask_loops(T, M, W, is_global))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q).permute(1, 0, 2), torch.from_numpy(Kr).permute(1, 0, 2),
        torch.from_numpy(Vr).permute(1, 0, 2), attn_mask=mask)
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_hand_derived(golden_dir):
    with open(os.path.join(golden_dir, "attention_meta_window1.json")) as f:
        g = json.load(f)
    q, k, v = (np.array(g[n])[:, None, :] for n in ("q", "k", "v"))
    pos = np.arange(q.shape[0])
    o = orc.attention(q, k, v, pos, pos, g["n_meta"], g["window"], 0)
    np.testing.assert_allclose(o[:, 0, :], np.array(g["o"]), rtol=1e-13, atol=1e-15)


def test_window_one_sees_meta_and_self():
    """W=1: an input row attends to exactly {meta} U {self}; brute-force softmax."""
    rng = np.random.default_rng(11)
    T, M, D = 9, 3, 4
    Q, K, V = rng.normal(size=(T, 1, D)), rng.normal(size=(T, 1, D)), rng.normal(size=(T, 1, D))
    o = orc.attention(Q, K, V, np.arange(T), np.arange(T), M, 1, 0)
    for i in range(M, T):
        keys = list(range(M)) + [i]
        sc = [float(Q[i, 0] @ K[j, 0]) / 2.0 for j in keys]
        e = [math.exp(s - max(sc)) for s in sc]
        want = sum(ei * V[j, 0] for ei, j in zip(e, keys)) / sum(e)
        np.testing.assert_allclose(o[i, 0], want, rtol=1e-12)


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(12)
    D, L = 16, 6
    q, k = rng.normal(size=(L, 1, D)), rng.normal(size=(L, 1, D))
    pos = np.arange(L) * 37
    for shift in (1, 250, 4096):
        a = orc.rope(q, pos, 10000.0)[:, 0] @ orc.rope(k, pos, 10000.0)[:, 0].T
        b = orc.rope(q, pos + shift, 10000.0)[:, 0] @ orc.rope(k, pos + shift, 10000.0)[:, 0].T
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)
    r = orc.rope(q, pos, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(orc.rope(q, np.zeros(L), 10000.0), q)
    # position 1 rotates pair j by base^(-2j/D) radians: check pair 0 (angle 1 rad)
    e = np.zeros((1, 1, D)); e[0, 0, 0] = 1.0
    r1 = orc.rope(e, [1], 10000.0)[0, 0]
    assert r1[0] == pytest.approx(math.cos(1.0)) and r1[D // 2] == pytest.approx(math.sin(1.0))


# ---------------------------------------------------------------------------------------
# whole mixer: special cases and invariants
# ---------------------------------------------------------------------------------------
def test_window_covering_sequence_equals_global():
    dims = _small_dims(window=64)
    w = _weights(dims)
    X = _x(2, 10, dims.d_model)
    a = orc.mixer_prefill(dims, w, X)["out"]
    b = orc.mixer_prefill(dims.replace(is_global=1), w, X)["out"]
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)
    c = orc.mixer_prefill(dims.replace(window=3), w, X)["out"]
    assert np.max(np.abs(c - b)) > 1e-3        # a real window changes the result


def test_meta_rows_independent_of_input():
    dims = _small_dims()
    w = _weights(dims)
    X1, X2 = _x(1, 12, dims.d_model, seed=3), _x(1, 12, dims.d_model, seed=4)
    r1, r2 = orc.mixer_prefill(dims, w, X1), orc.mixer_prefill(dims, w, X2)
    M = dims.n_meta
    assert np.array_equal(r1["out"][:, :M], r2["out"][:, :M])
    # the SSM state after the meta prefix does not depend on X
    s1 = orc.selective_scan(r1["xc"][0, :M], r1["delta"][0, :M], w["A"], r1["Bm"][0, :M],
                            r1["Cm"][0, :M], r1["z"][0, :M])[1]
    s2 = orc.selective_scan(r2["xc"][0, :M], r2["delta"][0, :M], w["A"], r2["Bm"][0, :M],
                            r2["Cm"][0, :M], r2["z"][0, :M])[1]
    assert np.array_equal(s1, s2)
    assert not np.array_equal(r1["out"][:, M:], r2["out"][:, M:])


def test_consumer_reuses_producer_kv():
    dims = _small_dims()
    prod = dims.replace(kv_role=synth.KV_PRODUCER)
    cons = dims.replace(kv_role=synth.KV_CONSUMER)
    wp, wc = _weights(prod, seed=1), _weights(cons, seed=2)
    X = _x(1, 11, dims.d_model)
    rp = orc.mixer_prefill(prod, wp, X)
    rc = orc.mixer_prefill(cons, wc, X, kv_in=(rp["K"], rp["V"]))
    T = X.shape[1] + dims.n_meta
    pos = np.arange(T)
    want = orc.attention(rc["Q"][0], rp["K"][0], rp["V"][0], pos, pos, dims.n_meta, dims.window, 0)
    np.testing.assert_allclose(rc["O"][0], want.reshape(T, -1), rtol=1e-13)
    # perturbing the producer's W_K changes what the consumer computes
    wp2 = dict(wp); wp2["w_in"] = wp["w_in"].copy()
    wp2["w_in"][dims.attn_width:dims.attn_width + dims.kv_width] *= 1.5
    rp2 = orc.mixer_prefill(prod, wp2, X)
    rc2 = orc.mixer_prefill(cons, wc, X, kv_in=(rp2["K"], rp2["V"]))
    assert np.max(np.abs(rc2["out"] - rc["out"])) > 1e-4
    assert cons.in_width == prod.in_width - 2 * dims.kv_width


def test_norm_scale_invariances():
    """Scaling W_V (attention branch) or the C rows of W_x (SSM branch) by c>0 scales only
    that branch's output, which the RMSNorm removes (eps aside)."""
    dims = _small_dims(norm_eps=0.0)
    w = _weights(dims)
    X = _x(1, 9, dims.d_model)
    base = orc.mixer_prefill(dims, w, X)["out"]
    wv = dict(w); wv["w_in"] = w["w_in"].copy()
    a0 = dims.attn_width + dims.kv_width
    wv["w_in"][a0:a0 + dims.kv_width] *= 3.0
    np.testing.assert_allclose(orc.mixer_prefill(dims, wv, X)["out"], base, rtol=1e-11, atol=1e-12)
    wc = dict(w); wc["w_x"] = w["w_x"].copy()
    wc["w_x"][dims.dt_rank + dims.d_state:] *= 0.25
    np.testing.assert_allclose(orc.mixer_prefill(dims, wc, X)["out"], base, rtol=1e-11, atol=1e-12)
    # ... and scaling the SSM input side (B rows) is not invisible through Delta-free paths:
    wb = dict(w); wb["w_x"] = w["w_x"].copy()
    wb["w_x"][:dims.dt_rank] *= 3.0               # dt_low feeds Delta nonlinearly
    assert np.max(np.abs(orc.mixer_prefill(dims, wb, X)["out"] - base)) > 1e-6


def test_tied_out_proj_reduces_to_printed_fusion():
    """With Hq*D == Di and tied W_out slices, Y = W (beta1 norm(Ya) + beta2 norm(Ys)) / 2,
    the fusion formula of §数学表示 5 with the average's 1/2."""
    dims = _small_dims(d_inner=32)              # Hq*D = 4*8 = 32
    w = _weights(dims)
    Wt = np.random.default_rng(13).normal(size=(dims.d_model, 32))
    w["w_out"] = np.concatenate([Wt, Wt], axis=1)
    X = _x(1, 7, dims.d_model)
    r = orc.mixer_prefill(dims, w, X)
    ya, ys = r["O"][0], r["y_ssm"][0]
    na = ya / np.sqrt(np.mean(ya ** 2, axis=-1, keepdims=True) + dims.norm_eps)
    ns = ys / np.sqrt(np.mean(ys ** 2, axis=-1, keepdims=True) + dims.norm_eps)
    want = 0.5 * (w["g_attn"] * na + w["g_ssm"] * ns) @ Wt.T
    np.testing.assert_allclose(r["out"][0], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("is_global", [0, 1])
def test_prefill_then_decode_equals_longer_prefill(is_global):
    """prefill(T) + decode(position T) == the last row of prefill(T+1); covers the ring
    wrap (T > M + W), the conv state and the SSM state carried across the calls."""
    dims = _small_dims(is_global=is_global, window=4)
    w = _weights(dims)
    N = 9
    X = _x(2, N + 1, dims.d_model)
    T = dims.n_meta + N
    r = orc.mixer_prefill(dims, w, X[:, :N])
    if is_global:
        Lmax = T + 1
        k = np.zeros((2, Lmax, dims.n_kv_heads, dims.head_dim)); v = np.zeros_like(k)
        k[:, :T], v[:, :T] = r["K"], r["V"]
        cache = dict(k=k, v=v)
    else:
        cache = {n: r[n] for n in ("meta_k", "meta_v", "ring_k", "ring_v")}
    d = orc.mixer_decode(dims, w, X[:, N], T, cache, r["ssm_state"], r["conv_state"])
    full = orc.mixer_prefill(dims, w, X)
    np.testing.assert_allclose(d["out"], full["out"][:, -1], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(d["ssm_state"], full["ssm_state"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(d["conv_state"], full["conv_state"], rtol=1e-14)


def test_consumer_decode_reads_producer_ring():
    dims = _small_dims(window=4)
    prod, cons = dims.replace(kv_role=synth.KV_PRODUCER), dims.replace(kv_role=synth.KV_CONSUMER)
    wp, wc = _weights(prod, seed=1), _weights(cons, seed=2)
    N = 8
    X = _x(1, N + 1, dims.d_model)
    T = dims.n_meta + N
    rp = orc.mixer_prefill(prod, wp, X[:, :N])
    rc = orc.mixer_prefill(cons, wc, X[:, :N], kv_in=(rp["K"], rp["V"]))
    cache = {n: rp[n] for n in ("meta_k", "meta_v", "ring_k", "ring_v")}
    dp = orc.mixer_decode(prod, wp, X[:, N], T, cache, rp["ssm_state"], rp["conv_state"])
    dc = orc.mixer_decode(cons, wc, X[:, N], T, dp["cache"], rc["ssm_state"], rc["conv_state"])
    fp = orc.mixer_prefill(prod, wp, X)
    fc = orc.mixer_prefill(cons, wc, X, kv_in=(fp["K"], fp["V"]))
    np.testing.assert_allclose(dc["out"], fc["out"][:, -1], rtol=1e-11, atol=1e-12)


def test_kv_share_plan_hymba_layout():
    is_global = [1 if i in (0, 15, 31) else 0 for i in range(32)]
    cid, role = orc.kv_share_plan(is_global)
    pairs = [(i, i + 1) for i in range(1, 15, 2)] + [(i, i + 1) for i in range(16, 30, 2)]
    for a, b in pairs:
        assert cid[a] == cid[b] and role[a] == synth.KV_PRODUCER and role[b] == synth.KV_CONSUMER
    for i in (0, 15, 31, 30):
        assert role[i] == synth.KV_OWN and cid.count(cid[i]) == 1
    assert len(set(cid)) == 3 + 14 + 1


def test_block_residual_identity():
    """Zero mixer and FFN outputs leave the residual stream unchanged (pre-norm residual)."""
    dims = _small_dims()
    w = _weights(dims); w["w_out"] = np.zeros_like(w["w_out"])
    bw = {k: v.astype(np.float64) for k, v in synth.block_weights(dims, 12).items()}
    bw["w_down"] = np.zeros_like(bw["w_down"])
    H = _x(1, 8, dims.d_model)
    out, _ = orc.hymba_block(dims, w, bw, H)
    np.testing.assert_array_equal(out, H)


def test_ffn_swiglu_hand_derived(golden_dir):
    """SwiGLU on a d = 2, F = 2 case whose SiLU values have closed forms (ln 3 inputs):
    the gate branch goes through SiLU, the up branch does not, the two multiply, and
    W_down maps the product back (an asymmetric W_down, so a transposed one fails)."""
    with open(os.path.join(golden_dir, "ffn_swiglu_closed_form.json")) as f:
        c = json.load(f)
    bw = {k: np.array(c[k]) for k in ("w_gate", "w_up", "w_down")}
    np.testing.assert_allclose(orc.ffn_swiglu(np.array(c["v"]), bw), np.array(c["out"]), rtol=1e-13, atol=1e-15)


def _block_case(eps=1e-6):
    dims = _small_dims(norm_eps=eps)
    w = _weights(dims)
    bw = {k: v.astype(np.float64) for k, v in synth.block_weights(dims, 24, seed=3).items()}
    # FFN weights large enough that its update is far above rounding
    for k in ("w_gate", "w_up", "w_down"):
        bw[k] = bw[k] * 25.0
    return dims, w, bw, _x(1, 8, dims.d_model, seed=4)


def test_block_is_its_two_sublayers_in_order():
    """[JJ] §Hymba 的整体架构: norm -> mixer -> norm -> FFN, each sublayer adding to the
    residual stream.  The whole block must equal its mixer sublayer alone (FFN output
    zeroed) followed by its FFN sublayer alone (mixer output zeroed): the FFN reads the
    stream after the mixer's update, not the block's input."""
    dims, w, bw, H = _block_case()
    full, _ = orc.hymba_block(dims, w, bw, H)
    bw_no_ffn = dict(bw); bw_no_ffn["w_down"] = np.zeros_like(bw["w_down"])
    w_no_mix = dict(w); w_no_mix["w_out"] = np.zeros_like(w["w_out"])
    H1, _ = orc.hymba_block(dims, w, bw_no_ffn, H)
    two_step, _ = orc.hymba_block(dims, w_no_mix, bw, H1)
    assert np.max(np.abs(H1 - H)) > 1e-3 and np.max(np.abs(two_step - H1)) > 1e-3   # both sublayers act
    np.testing.assert_allclose(full, two_step, rtol=1e-12, atol=1e-13)


def test_block_sublayers_read_normalised_stream():
    """Pre-norm: each sublayer reads RMSNorm of the stream, so with eps = 0 its update does
    not change when the stream is scaled by c > 0 (the residual itself scales)."""
    dims, w, bw, H = _block_case(eps=0.0)
    bw_no_ffn = dict(bw); bw_no_ffn["w_down"] = np.zeros_like(bw["w_down"])
    w_no_mix = dict(w); w_no_mix["w_out"] = np.zeros_like(w["w_out"])
    for ww, bb in ((w, bw_no_ffn), (w_no_mix, bw)):
        upd1 = orc.hymba_block(dims, ww, bb, H)[0] - H
        upd7 = orc.hymba_block(dims, ww, bb, 7.5 * H)[0] - 7.5 * H
        assert np.max(np.abs(upd1)) > 1e-3
        np.testing.assert_allclose(upd7, upd1, rtol=1e-9, atol=1e-11)


def test_tiny_workload_runs_and_is_finite():
    w = synth.layer_weights(TINY.dims, seed=0)
    X = synth.prefill_input(TINY, seed=0)
    r = orc.mixer_prefill(TINY.dims, w, X)
    assert r["out"].shape == (1, 128, 256) and np.all(np.isfinite(r["out"]))
