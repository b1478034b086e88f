"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on seeded inputs.

Tolerances: bf16 paths max|err| <= 2e-2 * RMS(ref); the fp32 scan state <= 1e-4 relative
(inf-norm) when the scan stage is fed the GPU's own inputs.
"""
import numpy as np
import pytest
import torch

from hybrid_attention_ssm_b200 import hymba as H
from hybrid_attention_ssm_b200 import synth
from oracle import hymba_oracle as orc

from tests.helpers import (PrefillRun, assert_elem, assert_rel_inf, assert_rms, bf16_dev, f32_dev,
                           to_np)

pytestmark = pytest.mark.gpu

WL = synth.workloads()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.lib()


def _w(dims, seed=0, layer=0, wl=None):
    mean, std = (wl.dt_bias_mean, wl.dt_bias_std) if wl is not None else (0.0, 0.02)
    return synth.layer_weights(dims, seed=seed, layer=layer, dt_bias_mean=mean, dt_bias_std=std)


# ---------------------------------------------------------------------------------------
# tcgen05 GEMM against a plain fp32 PyTorch product
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 200, 1600), (2176, 1600, 4800), (64, 8640, 1600),
                                   (1, 8, 8), (513, 136, 72)])
def test_gemm_matches_fp32_reference(M, N, K):
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16).cuda()
    R = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = H.alloc_workspace(256)
    H.gemm_bf16(A, B, C, ws, residual=R)
    ref = A.float() @ B.float().T + R.float()
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0
    assert_rms(to_np(C), to_np(ref), name=f"gemm {M}x{N}x{K}")


# ---------------------------------------------------------------------------------------
# prefill: end to end and stage by stage
# ---------------------------------------------------------------------------------------
def _check_stages(run, ref, dims, w):
    """Each stage against the oracle fed the GPU's own stage inputs.  Stages stored in 16
    bits are checked elementwise against their unit roundoff; attention (bf16 P inside the
    PV product) against the bf16-path bound."""
    B, T = run.B, run.T
    Di, R, S = dims.d_inner, dims.dt_rank, dims.d_state
    pos = np.arange(T)
    # in_proj + RoPE, from the exact inputs
    assert_elem(run.stage("q"), ref["Q"], name="Q")
    xz = run.stage("xz")
    assert_elem(xz[..., :Di], ref["x_ssm"], name="x_ssm")
    assert_elem(xz[..., Di:], ref["z"], name="z")
    k = v = None
    if dims.kv_role != synth.KV_CONSUMER:
        k, v = run.kv()
        assert_elem(k, ref["K"], name="K")
        assert_elem(v, ref["V"], name="V")
    xc, xbc, delta = run.stage("xc"), run.stage("xbc"), run.stage("delta")
    y, o, u, q = run.stage("y"), run.stage("o"), run.stage("u"), run.stage("q")
    out = to_np(run.out)
    for b in range(B):
        xc_ref, cst = orc.causal_conv1d_silu(xz[b, :, :Di], w["conv_w"], w["conv_b"])
        assert_elem(xc[b], xc_ref, name="conv")
        assert_rel_inf(to_np(run.conv[b]), cst, tol=1e-6, name="conv state")
        proj = xc[b] @ w["w_x"].astype(np.float64).T
        assert_rms(xbc[b, :, :R + 2 * S], proj, tol=1e-3, name="x_proj")
        d_ref = orc.softplus(xbc[b, :, :R] @ w["w_dt"].astype(np.float64).T + w["dt_bias"])
        assert_rel_inf(delta[b], d_ref, tol=5e-3, name="delta")
        # scan fed the GPU's own xc, delta, B, C, z (the scan reads B and C as fp16)
        zb = xz[b, :, Di:]
        bm16 = xbc[b, :, R:R + S].astype(np.float16).astype(np.float64)
        cm16 = xbc[b, :, R + S:R + 2 * S].astype(np.float16).astype(np.float64)
        y_ref, h_ref = orc.selective_scan(xc[b], delta[b], w["A"], bm16, cm16, zb)
        assert_rel_inf(to_np(run.ssm[b]), h_ref, tol=1e-4, name="scan state")
        assert_elem(y[b] * orc.silu(zb), y_ref, name="scan y")
        if k is not None:
            o_ref = orc.attention(q[b], k[b], v[b], pos, pos, dims.n_meta, dims.window, dims.is_global)
            assert_rms(o[b], o_ref.reshape(T, -1), name="attention")
        _, u_ref = orc.fuse_and_project(o[b], y[b] * orc.silu(zb), w, dims)
        assert_elem(u[b], u_ref, rel=2e-3, abs_rms=1e-4, name="norm/avg")
        assert_elem(out[b], u[b] @ w["w_out"].astype(np.float64).T, name="out_proj")


@pytest.mark.parametrize("name", ["tiny", "tiny_full"])
def test_prefill_tiny(name):
    wl = WL[name]
    w = _w(wl.dims, wl=wl)
    X = synth.prefill_input(wl)
    run = PrefillRun(wl.dims, w, X)
    ref = orc.mixer_prefill(wl.dims, w, X)
    assert_rms(to_np(run.out), ref["out"], name="out")
    assert_rel_inf(to_np(run.ssm), ref["ssm_state"], tol=2e-2, name="ssm state (end to end)")
    _check_stages(run, ref, wl.dims, w)
    # SWA cache after prefill
    if not wl.dims.is_global:
        for n in ("meta_k", "meta_v", "ring_k", "ring_v"):
            got = to_np(run.cache.t[n])
            want = ref[n]
            if n.startswith("ring"):
                filled = [orc.ring_slot(p, wl.dims.n_meta, wl.dims.window)
                          for p in range(max(wl.dims.n_meta, run.T - wl.dims.window), run.T)]
                got, want = got[:, filled], want[:, filled]
            assert_rms(got, want, name=n)


def test_prefill_window_at_least_sequence_equals_global():
    wl = WL["tiny_full"]
    w = _w(wl.dims)
    X = synth.prefill_input(wl)
    a = PrefillRun(wl.dims, w, X)
    b = PrefillRun(wl.dims.replace(is_global=1), w, X)
    assert torch.equal(a.out, b.out)


@pytest.mark.parametrize("kw", [dict(n_meta=8, n_tokens=117, B=1),      # ragged T
                                dict(n_meta=0, n_tokens=200, B=2),      # no meta tokens
                                dict(n_meta=5, n_tokens=1, B=3),        # one token
                                dict(n_meta=8, n_tokens=300, B=1, window=1),
                                dict(n_meta=130, n_tokens=140, B=2, window=100),
                                dict(n_meta=8, n_tokens=250, B=1, heads=(4, 4))])
def test_prefill_edge_shapes(kw):
    hq, hkv = kw.get("heads", (4, 2))
    dims = WL["tiny"].dims.replace(n_meta=kw["n_meta"], window=kw.get("window", 32), n_q_heads=hq,
                                   n_kv_heads=hkv)
    w = _w(dims, seed=3)
    X = np.random.default_rng(4).normal(size=(kw["B"], kw["n_tokens"], dims.d_model)).astype(np.float32)
    X = synth.bf16_round(X)
    run = PrefillRun(dims, w, X)
    ref = orc.mixer_prefill(dims, w, X)
    assert_rms(to_np(run.out), ref["out"], name="out")
    _check_stages(run, ref, dims, w)


def test_prefill_with_meta_in_input_and_residual():
    wl = WL["tiny"]
    dims = wl.dims
    w = _w(dims, seed=5)
    rng = np.random.default_rng(6)
    Hs = synth.bf16_round(rng.normal(size=(2, 128, dims.d_model)).astype(np.float32))
    res = synth.bf16_round(rng.normal(size=(2, 128, dims.d_model)).astype(np.float32))
    run = PrefillRun(dims, w, Hs, x_has_meta=1, residual=res)
    ref = orc.mixer_prefill(dims, w, Hs, x_has_meta=True, residual=res)
    assert_rms(to_np(run.out), ref["out"], name="out")


def test_prefill_shared_kv_pair():
    wl = WL["tiny"]
    prod = wl.dims.replace(kv_role=synth.KV_PRODUCER)
    cons = wl.dims.replace(kv_role=synth.KV_CONSUMER)
    wp, wc = _w(prod, seed=1), _w(cons, seed=2)
    X = synth.prefill_input(wl)
    rp = PrefillRun(prod, wp, X)
    rc = PrefillRun(cons, wc, X, cache=rp.cache)
    op = orc.mixer_prefill(prod, wp, X)
    oc = orc.mixer_prefill(cons, wc, X, kv_in=(op["K"], op["V"]))
    assert_rms(to_np(rp.out), op["out"], name="producer")
    assert_rms(to_np(rc.out), oc["out"], name="consumer")
    # the consumer's attention reads exactly the producer's cached K/V
    k, v = rp.kv()
    pos = np.arange(rc.T)
    o_ref = orc.attention(rc.stage("q")[0], k[0], v[0], pos, pos, cons.n_meta, cons.window, 0)
    assert_rms(rc.stage("o")[0], o_ref.reshape(rc.T, -1), name="consumer attention")


def test_prefill_swa_hymba_layer():
    wl = WL["swa"]
    w = _w(wl.dims, wl=wl)
    X = synth.prefill_input(wl)
    run = PrefillRun(wl.dims, w, X)
    ref = orc.mixer_prefill(wl.dims, w, X)
    assert_rms(to_np(run.out), ref["out"], name="out")
    _check_stages(run, ref, wl.dims, w)


# ---------------------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------------------
def _decode(dims, w, cache, x, position, ssm, conv, residual=None):
    B = x.shape[0]
    dw = H.DeviceWeights(w)
    out = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
    nbytes = H.workspace_size(dims, B, cache.c.max_tokens, 0, H.MODE_DECODE)
    ws = H.alloc_workspace(nbytes)
    H.mixer_decode(dims, dw, bf16_dev(x), position, cache, ssm, conv, out, ws,
                   residual=None if residual is None else bf16_dev(residual))
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0
    return out


@pytest.mark.parametrize("is_global", [0, 1])
def test_prefill_then_decode_matches_longer_prefill(is_global):
    dims = WL["tiny"].dims.replace(is_global=is_global, window=16)
    w = _w(dims, seed=7)
    N = 60
    X = synth.bf16_round(np.random.default_rng(8).normal(size=(2, N + 1, dims.d_model)).astype(np.float32))
    T = dims.n_meta + N
    run = PrefillRun(dims, w, X[:, :N], max_tokens=T + 1)
    out = _decode(dims, w, run.cache, X[:, N], T, run.ssm, run.conv)
    full = PrefillRun(dims, w, X)
    ref = orc.mixer_prefill(dims, w, X)
    assert_rms(to_np(out), ref["out"][:, -1], name="decode vs oracle prefill(T+1)")
    assert_rms(to_np(out), to_np(full.out[:, -1]), name="decode vs GPU prefill(T+1)")
    assert_rel_inf(to_np(run.ssm), ref["ssm_state"], tol=2e-2, name="state after decode")


def test_prefill_and_decode_at_the_size_limits():
    """Every width at the largest value the library accepts: d_inner 4096 and Hq*D 2048 (the
    norm's per-thread chunks full), dt_rank 224 (dt_low | B | C = 256 columns: the widest
    x_proj tile and the largest decode SSM staging), 4 query heads per KV head."""
    dims = WL["tiny"].dims.replace(d_model=1024, n_q_heads=32, n_kv_heads=8, d_inner=4096, dt_rank=224,
                                   n_meta=8, window=48)
    w = _w(dims, seed=21)
    N = 60
    X = synth.bf16_round(np.random.default_rng(22).normal(size=(2, N + 1, dims.d_model)).astype(np.float32))
    T = dims.n_meta + N
    run = PrefillRun(dims, w, X[:, :N], max_tokens=T + 1)
    ref_n = orc.mixer_prefill(dims, w, X[:, :N])
    assert_rms(to_np(run.out), ref_n["out"], name="prefill out at the limits")
    assert_rel_inf(to_np(run.ssm), ref_n["ssm_state"], tol=2e-2, name="ssm state at the limits")
    out = _decode(dims, w, run.cache, X[:, N], T, run.ssm, run.conv)
    ref = orc.mixer_prefill(dims, w, X)
    assert_rms(to_np(out), ref["out"][:, -1], name="decode at the limits vs oracle prefill(T+1)")


def test_decode_pair_hymba():
    wl = WL["decode_pair"]
    prod = wl.dims
    cons = wl.dims.replace(kv_role=synth.KV_CONSUMER)
    wp, wc = _w(prod, layer=0, wl=wl), _w(cons, layer=1, wl=wl)
    st_p, st_c = synth.decode_state(wl, layer=0), synth.decode_state(wl, layer=1)
    p = wl.decode_position
    cache = H.Cache(prod, wl.batch, 1)
    for n in ("meta_k", "meta_v", "ring_k", "ring_v"):
        cache.t[n].copy_(f32_dev(st_p[n]).to(torch.float16))
    ssm_p, conv_p = f32_dev(st_p["ssm_state"]), f32_dev(st_p["conv_state"])
    ssm_c, conv_c = f32_dev(st_c["ssm_state"]), f32_dev(st_c["conv_state"])
    out_p = _decode(prod, wp, cache, st_p["x_new"], p, ssm_p, conv_p)
    out_c = _decode(cons, wc, cache, st_c["x_new"], p, ssm_c, conv_c)
    ocache = {n: st_p[n] for n in ("meta_k", "meta_v", "ring_k", "ring_v")}
    rp = orc.mixer_decode(prod, wp, st_p["x_new"], p, ocache, st_p["ssm_state"], st_p["conv_state"])
    rc = orc.mixer_decode(cons, wc, st_c["x_new"], p, rp["cache"], st_c["ssm_state"], st_c["conv_state"])
    assert_rms(to_np(out_p), rp["out"], name="producer out")
    assert_rms(to_np(out_c), rc["out"], name="consumer out")
    assert_rel_inf(to_np(ssm_p), rp["ssm_state"], tol=1e-3, name="producer ssm state")
    assert_rel_inf(to_np(conv_p), rp["conv_state"], tol=1e-2, name="producer conv state")
    slot = orc.ring_slot(p, prod.n_meta, prod.window)
    assert_rms(to_np(cache.t["ring_k"][:, slot]), rp["cache"]["ring_k"][:, slot], name="new ring k")
    assert_rms(to_np(cache.t["ring_v"][:, slot]), rp["cache"]["ring_v"][:, slot], name="new ring v")


# ---------------------------------------------------------------------------------------
# bounded waits: the timeout path reports an error instead of hanging
# ---------------------------------------------------------------------------------------
def test_bounded_wait_reports_timeout():
    ws = H.alloc_workspace(256)
    H.set_wait_limit_ns(20_000_000)
    try:
        H.selftest_wait_timeout(ws)
        assert H.status_read(ws) == H.ERR_TIMEOUT
    finally:
        H.set_wait_limit_ns(2_000_000_000)
    assert H.status_read(ws) == 0
