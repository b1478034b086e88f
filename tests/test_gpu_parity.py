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
    xc, xbc, dt_pre = run.stage("xc"), run.stage("xbc"), run.stage("dt_pre")
    y, o, u, q = run.stage("y"), run.stage("o"), run.stage("u"), run.stage("q")
    out = to_np(run.out)
    for b in range(B):
        xc_ref, cst = orc.causal_conv1d_silu(xz[b, :, :Di], w["conv_w"], w["conv_b"])
        assert_elem(xc[b], xc_ref, name="conv")
        assert_rel_inf(to_np(run.conv[b]), cst, tol=1e-6, name="conv state")
        proj = xc[b] @ w["w_x"].astype(np.float64).T
        assert_rms(xbc[b, :, :R + 2 * S], proj, tol=1e-3, name="x_proj")
        # dt_proj (tf32): dt_low W_dt^T, before the bias and softplus that the scan applies
        assert_rel_inf(dt_pre[b], xbc[b, :, :R] @ w["w_dt"].astype(np.float64).T, tol=5e-3, name="dt_proj")
        # the scan fed its own inputs (dt_pre, xc, B, C, z): delta = softplus(dt_pre + bias) in fp64
        delta = orc.softplus(dt_pre[b] + w["dt_bias"])
        zb = xz[b, :, Di:]
        y_ref, h_ref = orc.selective_scan(xc[b], delta, w["A"], xbc[b, :, R:R + S], xbc[b, :, R + S:R + 2 * S], zb)
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


@pytest.mark.parametrize("is_global,window", [(1, 32), (0, 200)])
def test_attention_running_max_growth(is_global, window):
    """Scores that grow along each row, so the running maximum of the online softmax rises
    by more than the kernel's lazy-rescale threshold (2^8) from one key tile to the next: the
    attention output, fed the GPU's own Q, K, V, against the oracle's dense softmax.  The
    test checks on the CPU that its inputs do reach that path."""
    dims = WL["tiny"].dims.replace(is_global=is_global, window=window)
    w = _w(dims, seed=61)
    qk = dims.attn_width + 2 * dims.n_kv_heads * dims.head_dim     # Q and K rows of W_in
    w_in = w["w_in"].copy()
    w_in[:qk] = synth.bf16_round(w_in[:qk] * 10.0)
    w = dict(w, w_in=w_in)
    N = 500
    T = dims.n_meta + N
    rng = np.random.default_rng(62)
    grow = (0.5 + 3.0 * np.arange(N) / N)[None, :, None]            # later rows larger
    X = synth.bf16_round((rng.normal(size=(1, N, dims.d_model)) * grow).astype(np.float32))
    run = PrefillRun(dims, w, X)
    q, o = run.stage("q")[0], run.stage("o")[0]
    k, v = run.kv()
    k, v = k[0], v[0]
    pos = np.arange(T)
    o_ref = orc.attention(q, k, v, pos, pos, dims.n_meta, dims.window, dims.is_global)
    assert_rms(o, o_ref.reshape(T, -1), name="attention, growing scores")
    # the case is the intended one: some row's running max (log2 units, per 128-key tile in
    # the order the kernel visits them) grows by more than 8 at some tile
    g = dims.n_q_heads // dims.n_kv_heads
    vis = orc.visibility_mask(pos, pos, dims.n_meta, dims.window, dims.is_global)
    s = np.einsum("thd,shd->hts", q, np.repeat(k, g, axis=1)) * (np.log2(np.e) / np.sqrt(dims.head_dim))
    s = np.where(vis[None], s, -np.inf)
    tile_max = np.stack([s[:, :, j:j + 128].max(axis=2) for j in range(0, T, 128)], axis=2)
    run_max = np.maximum.accumulate(tile_max, axis=2)
    jumps = np.diff(np.where(np.isfinite(run_max), run_max, np.nan), axis=2)
    assert np.nanmax(jumps) > 8.0, f"largest running-max step {np.nanmax(jumps):.1f} (log2 units)"


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


def test_prefill_from_host_buffers_equals_device_path():
    """hymba_mixer_prefill_host (input and output in pinned host memory, copies enqueued by
    the library) gives the device-buffer prefill's output bit for bit, on its own stream."""
    wl = WL["tiny"]
    dims = wl.dims
    w = _w(dims, seed=51)
    X = synth.bf16_round(np.random.default_rng(52).normal(size=(2, 77, dims.d_model)).astype(np.float32))
    run = PrefillRun(dims, w, X)
    xh = torch.from_numpy(X).to(torch.bfloat16).pin_memory()
    oh = torch.zeros(2, run.T, dims.d_model, dtype=torch.bfloat16).pin_memory()
    ws = H.alloc_workspace(H.workspace_size(dims, 2, 77, 0, H.MODE_PREFILL_HOST))
    s = torch.cuda.Stream()
    H.mixer_prefill_host(dims, run.dw, xh, H.Cache(dims, 2, run.T), oh, ws, stream=s)
    s.synchronize()
    assert H.status_read(ws, s) == 0
    assert torch.equal(oh, run.out.cpu())


# ---------------------------------------------------------------------------------------
# meta-token prefix computed once, then prefills of the input rows only
# ---------------------------------------------------------------------------------------
def _prefix_run(dims, w, X, producer_prefix=None, cache=None, max_tokens=None):
    """Build the layer's prefix from its meta tokens, then prefill X's rows from it."""
    B, N = X.shape[0], X.shape[1]
    M, T = dims.n_meta, dims.n_meta + X.shape[1]
    dw = H.DeviceWeights(w)
    meta_out = torch.zeros(M, dims.d_model, dtype=torch.bfloat16, device="cuda")
    bws = H.alloc_workspace(H.workspace_size(dims, 1, M, 1))
    pre = H.Prefix(dims, dw, dw.t["meta"], meta_out, bws, producer=producer_prefix)
    cache = cache if cache is not None else H.Cache(dims, B, max_tokens or T)
    out = torch.zeros(B, N, dims.d_model, dtype=torch.bfloat16, device="cuda")
    ssm = torch.zeros(B, dims.d_inner, dims.d_state, device="cuda")
    conv = torch.zeros(B, dims.d_inner, dims.d_conv - 1, device="cuda")
    ws = H.alloc_workspace(H.workspace_size(dims, B, N))
    H.mixer_prefill_prefix(dims, dw, bf16_dev(X), pre, cache, out, ws, ssm_state=ssm, conv_state=conv)
    torch.cuda.synchronize()
    assert H.status_read(bws) == 0 and H.status_read(ws) == 0
    return dict(prefix=pre, meta_out=meta_out, cache=cache, out=out, ssm=ssm, conv=conv, ws=ws)


@pytest.mark.parametrize("kw", [dict(B=1, N=120), dict(B=2, N=77, M=130, W=100), dict(B=3, N=1),
                                dict(B=2, N=200, is_global=1), dict(B=1, N=300, W=1)])
def test_prefill_from_meta_prefix(kw):
    """[JJ] §深入理解元 Tokens: the meta tokens' work is done once.  A prefill of the input
    rows from the layer's prefix equals rows M..T-1 of the full prefill: against the oracle
    (bf16 bound) and against the full GPU prefill (the rows, the final states, the cache);
    the prefix itself (meta output rows, meta K/V, states after the meta rows) equals the
    full prefill's meta rows."""
    dims = WL["tiny"].dims.replace(n_meta=kw.get("M", 8), window=kw.get("W", 32), is_global=kw.get("is_global", 0))
    w = _w(dims, seed=61)
    X = synth.bf16_round(np.random.default_rng(62).normal(size=(kw["B"], kw["N"], dims.d_model)).astype(np.float32))
    M = dims.n_meta
    full = PrefillRun(dims, w, X)
    r = _prefix_run(dims, w, X)
    ref = orc.mixer_prefill(dims, w, X)
    assert_rms(to_np(r["out"]), ref["out"][:, M:], name="prefix prefill vs oracle rows M..T-1")
    assert_rms(to_np(r["out"]), to_np(full.out[:, M:]), name="prefix prefill vs full prefill")
    assert torch.equal(r["meta_out"], full.out[0, :M]), "meta rows of the output"
    assert_rel_inf(to_np(r["ssm"]), to_np(full.ssm), tol=1e-4, name="final ssm state")
    assert torch.equal(r["conv"], full.conv), "final conv state"
    for n in (("k", "v") if dims.is_global else ("k", "v", "meta_k", "meta_v", "ring_k", "ring_v")):
        a, b = r["cache"].t[n], full.cache.t[n]
        if n in ("k", "v"):
            a, b = a[:, :full.T], b[:, :full.T]
        assert torch.equal(a, b), f"cache {n}"
    # the prefix against the oracle's meta rows alone (meta rows never see X: P6)
    om = orc.mixer_prefill(dims, w, w["meta"][None], x_has_meta=True)
    pre = r["prefix"]
    assert_rms(to_np(r["meta_out"]), om["out"][0], name="meta rows vs oracle")
    assert_rms(to_np(pre.tensor("k")), om["K"][0], name="prefix K vs oracle")
    assert_rms(to_np(pre.tensor("v")), om["V"][0], name="prefix V vs oracle")
    assert_rel_inf(to_np(pre.tensor("ssm_state")), om["ssm_state"][0], tol=2e-2, name="prefix ssm state vs oracle")
    assert_rel_inf(to_np(pre.tensor("conv_state")), om["conv_state"][0], tol=1e-2, name="prefix conv state vs oracle")


def test_prefill_from_meta_prefix_shared_kv_pair():
    """A consumer layer's prefix reads its producer's meta K/V; prefills of both layers from
    their prefixes equal the full prefills of the pair."""
    wl = WL["tiny"]
    prod = wl.dims.replace(kv_role=synth.KV_PRODUCER)
    cons = wl.dims.replace(kv_role=synth.KV_CONSUMER)
    wp, wc = _w(prod, seed=63), _w(cons, seed=64)
    X = synth.prefill_input(wl)
    M = prod.n_meta
    fp = PrefillRun(prod, wp, X)
    fc = PrefillRun(cons, wc, X, cache=fp.cache)
    rp = _prefix_run(prod, wp, X)
    rc = _prefix_run(cons, wc, X, producer_prefix=rp["prefix"], cache=rp["cache"])
    assert_rms(to_np(rp["out"]), to_np(fp.out[:, M:]), name="producer")
    assert_rms(to_np(rc["out"]), to_np(fc.out[:, M:]), name="consumer")
    assert torch.equal(rc["meta_out"], fc.out[0, :M]), "consumer meta rows"


def test_prefill_from_meta_prefix_hymba_layer():
    """The Hymba-shaped SWA layer (128 meta + 2048 tokens) from its prefix."""
    wl = WL["swa"]
    w = _w(wl.dims, wl=wl)
    X = synth.prefill_input(wl)
    M = wl.dims.n_meta
    full = PrefillRun(wl.dims, w, X)
    r = _prefix_run(wl.dims, w, X)
    assert_rms(to_np(r["out"]), to_np(full.out[:, M:]), name="prefix prefill vs full prefill (swa)")
    assert_rel_inf(to_np(r["ssm"]), to_np(full.ssm), tol=1e-4, name="final ssm state (swa)")


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


@pytest.mark.parametrize("B,N", [(1, 120), (3, 700)])
def test_prefill_scan_general_decays(B, N):
    """A rows that are not the progression A[s] = (s+1) A[0] take the scan's general path
    (one exponential per state); here half of the channels (whole warps) have such rows, the
    rest the progression, so both paths run in one launch and against the oracle."""
    dims = WL["tiny"].dims
    w = _w(dims, seed=11)
    rng = np.random.default_rng(12)
    A = w["A"].copy()
    A[dims.d_inner // 2:] = -rng.uniform(0.3, 6.0, size=(dims.d_inner // 2, dims.d_state)).astype(np.float32)
    w["A"] = A
    X = synth.bf16_round(rng.normal(size=(B, N, dims.d_model)).astype(np.float32))
    run = PrefillRun(dims, w, X)
    ref = orc.mixer_prefill(dims, w, X)
    assert_rms(to_np(run.out), ref["out"], name="out")
    _check_stages(run, ref, dims, w)


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
def _decode(dims, w, cache, x, position, ssm, conv, residual=None, keep_ws=False):
    B = x.shape[0]
    dw = H.DeviceWeights(w)
    out = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
    nbytes = H.workspace_size(dims, B, cache.c.max_tokens, 0, H.MODE_DECODE)
    ws = H.alloc_workspace(nbytes)
    H.mixer_decode(dims, dw, bf16_dev(x), position, cache, ssm, conv, out, ws,
                   residual=None if residual is None else bf16_dev(residual))
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0
    return (out, ws) if keep_ws else out


def _check_decode_ssm_step(dims, w, ws, B, max_tokens, h0, h_gpu):
    """The decode SSM step against the oracle fed the step's own inputs from the workspace
    (xc, x_proj's dt_low | B | C summed over its split-K slices in order, z from in_proj):
    the fp32 state within 1e-4 (inf-norm relative), the gated output y likewise."""
    from tests.helpers import ws_view
    L = H.decode_stage_layout(dims, B, max_tokens)
    Di, R, S = dims.d_inner, dims.dt_rank, dims.d_state
    proj = sum(to_np(ws_view(ws, L.proj + 4 * i * L.proj_slice_stride, (B, L.ld_proj), torch.float32))
               for i in range(L.in_split))
    xbc = sum(to_np(ws_view(ws, L.xbc_part + 4 * i * L.xbc_slice_stride, (B, L.ld_xbc), torch.float32))
              for i in range(L.xproj_split))
    xc = to_np(ws_view(ws, L.xc, (B, Di), torch.bfloat16))
    y_gpu = to_np(ws_view(ws, L.y, (B, Di), torch.float32))
    z = proj[:, L.ld_proj - Di:]
    for b in range(B):
        delta = orc.softplus(xbc[b:b + 1, :R] @ w["w_dt"].astype(np.float64).T + w["dt_bias"])
        y_ref, h_ref = orc.selective_scan(xc[b:b + 1], delta, w["A"], xbc[b:b + 1, R:R + S],
                                          xbc[b:b + 1, R + S:R + 2 * S], z[b:b + 1], h0=h0[b])
        assert_rel_inf(h_gpu[b], h_ref, tol=1e-4, name=f"decode ssm state, own inputs (b={b})")
        assert_rel_inf(y_gpu[b], y_ref[0], tol=1e-4, name=f"decode ssm y, own inputs (b={b})")


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
    out_p, ws_p = _decode(prod, wp, cache, st_p["x_new"], p, ssm_p, conv_p, keep_ws=True)
    out_c = _decode(cons, wc, cache, st_c["x_new"], p, ssm_c, conv_c)
    _check_decode_ssm_step(prod, wp, ws_p, wl.batch, cache.c.max_tokens,
                           st_p["ssm_state"].astype(np.float64), to_np(ssm_p))
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


def test_decode_global_layer_hymba_width():
    """A global (full-attention) layer's decode step at Hymba width: 25/5 heads, d_inner 3200,
    batch 8, new token at position 128 + 4096 over a full-length cache of N(0,1) keys and
    values, against the oracle's decode over the same cache; the new K/V row and the SSM
    step (own inputs, 1e-4) too."""
    import dataclasses
    wl = dataclasses.replace(WL["decode_pair"], batch=8)
    dims = wl.dims.replace(is_global=1, kv_role=synth.KV_OWN)
    B, p = wl.batch, 128 + 4096
    Lmax = p + 1
    w = _w(dims, layer=2, wl=wl)
    st = synth.decode_state(wl, layer=2)
    kv = synth.global_cache(wl, Lmax, layer=2)
    cache = H.Cache(dims, B, Lmax, kind=H.CACHE_GLOBAL)
    cache.t["k"].copy_(f32_dev(kv["k"]).to(torch.float16))
    cache.t["v"].copy_(f32_dev(kv["v"]).to(torch.float16))
    ssm, conv = f32_dev(st["ssm_state"]), f32_dev(st["conv_state"])
    out, ws = _decode(dims, w, cache, st["x_new"], p, ssm, conv, keep_ws=True)
    ref = orc.mixer_decode(dims, w, st["x_new"], p, {"k": kv["k"], "v": kv["v"]}, st["ssm_state"],
                           st["conv_state"])
    assert_rms(to_np(out), ref["out"], name="global decode out")
    assert_rms(to_np(cache.t["k"][:, p]), ref["cache"]["k"][:, p], name="new k row")
    assert_rms(to_np(cache.t["v"][:, p]), ref["cache"]["v"][:, p], name="new v row")
    assert_rel_inf(to_np(conv), ref["conv_state"], tol=1e-2, name="conv state")
    _check_decode_ssm_step(dims, w, ws, B, Lmax, st["ssm_state"].astype(np.float64), to_np(ssm))


# ---------------------------------------------------------------------------------------
# the SwiGLU FFN of the stack harness, for a few rows (decode) and many (prefill)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("rows", [1, 8, 64, 200])
def test_ffn_swiglu_decode(rows):
    """The decode-shaped FFN (weights as the M operand, split-K) against the oracle's SwiGLU
    and against the prefill-shaped FFN, at the stack's sizes (d 1600, F 5504), with a
    residual."""
    d, F = 1600, 5504
    dims = WL["stack"].dims
    bw = synth.block_weights(dims, F, seed=5, layer=3)
    rng = np.random.default_rng(70 + rows)
    hx = synth.bf16_round(rng.normal(size=(rows, d)).astype(np.float32))
    res = synth.bf16_round(rng.normal(size=(rows, d)).astype(np.float32))
    w_gu = torch.from_numpy(H.interleave_gate_up(bw["w_gate"], bw["w_up"])).cuda().to(torch.bfloat16)
    w_dn = torch.from_numpy(bw["w_down"]).cuda().to(torch.float16)
    h, r = bf16_dev(hx), bf16_dev(res)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    ws = H.alloc_workspace(H.ffn_workspace_size(rows, d, F))
    H.ffn_swiglu_decode(h, w_gu, w_dn, out, ws, residual=r)
    out2 = torch.empty_like(out)
    act = torch.empty(rows, F, dtype=torch.float16, device="cuda")
    ws2 = H.alloc_workspace(256)
    H.ffn_swiglu(h, w_gu, w_dn, act, out2, ws2, residual=r)
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0 and H.status_read(ws2) == 0
    # the output is bf16(residual + FFN): compare the sum, whose rounding is what is stored
    ref = orc.ffn_swiglu(hx, bw) + res
    assert_rms(to_np(out), ref, name=f"decode FFN ({rows} rows) vs oracle")
    assert_rms(to_np(out), to_np(out2), name=f"decode FFN vs prefill FFN ({rows} rows)")


@pytest.mark.parametrize("rows,d", [(1, 8), (7, 1600), (1000, 1600), (33, 4096), (9, 4104)])
def test_rmsnorm_against_oracle(rows, d):
    """hymba_rmsnorm (a warp per row up to d 4096, a CTA per row beyond) against the oracle's
    RMSNorm of the same bf16 rows, elementwise at the bf16 unit roundoff."""
    rng = np.random.default_rng(rows + d)
    x = synth.bf16_round(rng.normal(size=(rows, d)).astype(np.float32) * 3.0)
    g = rng.normal(1.0, 0.2, size=d).astype(np.float32)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    H.rmsnorm(bf16_dev(x), torch.from_numpy(g).cuda(), 1e-6, out)
    torch.cuda.synchronize()
    assert_elem(to_np(out), orc.rmsnorm(x, g, 1e-6), name=f"rmsnorm {rows}x{d}")


@pytest.mark.parametrize("is_global", [False, True])
def test_decode_norm_variants_equal_the_plain_calls_then_rmsnorm(is_global):
    """hymba_mixer_decode_norm and hymba_ffn_swiglu_decode_norm: out bit for bit what the plain
    calls write, and norm_out what hymba_rmsnorm computes from it (the same bf16 row; only the
    order of the sum of squares differs)."""
    dims = WL["tiny"].dims.replace(is_global=is_global, window=16)
    w = _w(dims, seed=31)
    N = 60
    X = synth.bf16_round(np.random.default_rng(32).normal(size=(2, N + 1, dims.d_model)).astype(np.float32))
    T = dims.n_meta + N
    run = PrefillRun(dims, w, X[:, :N], max_tokens=T + 1)
    ssm0, conv0 = run.ssm.clone(), run.conv.clone()
    dw = H.DeviceWeights(w)
    B, d = 2, dims.d_model
    x, res = bf16_dev(X[:, N]), bf16_dev(X[:, N - 1])
    g = torch.from_numpy(np.random.default_rng(33).normal(1.0, 0.1, size=d).astype(np.float32)).cuda()
    ws = H.alloc_workspace(H.workspace_size(dims, B, T + 1, 0, H.MODE_DECODE))
    out_a = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    H.mixer_decode(dims, dw, x, T, run.cache, run.ssm, run.conv, out_a, ws, residual=res)
    norm_a = torch.empty_like(out_a)
    H.rmsnorm(out_a, g, 1e-6, norm_a)
    ssm_a = run.ssm.clone()
    run.ssm.copy_(ssm0)
    run.conv.copy_(conv0)
    out_b, norm_b = torch.empty_like(out_a), torch.empty_like(out_a)
    H.mixer_decode_norm(dims, dw, x, T, run.cache, run.ssm, run.conv, out_b, g, 1e-6, norm_b, ws, residual=res)
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0
    assert torch.equal(out_a, out_b)
    assert torch.equal(ssm_a, run.ssm)
    assert_rms(to_np(norm_b), to_np(norm_a), tol=1e-2, name="mixer decode fused norm vs rmsnorm")
    # the FFN of the same rows (stack sizes d 1600 need not apply: tiny d_model, F a multiple of 64)
    F = 256
    bw = synth.block_weights(dims, F, seed=34, layer=0)
    w_gu = torch.from_numpy(H.interleave_gate_up(bw["w_gate"], bw["w_up"])).cuda().to(torch.bfloat16)
    w_dn = torch.from_numpy(bw["w_down"]).cuda().to(torch.float16)
    fws = H.alloc_workspace(H.ffn_workspace_size(B, d, F))
    f_a, f_b = torch.empty_like(out_a), torch.empty_like(out_a)
    H.ffn_swiglu_decode(norm_a, w_gu, w_dn, f_a, fws, residual=out_a)
    fn_a = torch.empty_like(out_a)
    H.rmsnorm(f_a, g, 1e-6, fn_a)
    fn_b = torch.empty_like(out_a)
    H.ffn_swiglu_decode_norm(norm_a, w_gu, w_dn, f_b, g, 1e-6, fn_b, fws, residual=out_a)
    torch.cuda.synchronize()
    assert H.status_read(fws) == 0
    assert torch.equal(f_a, f_b)
    assert_rms(to_np(fn_b), to_np(fn_a), tol=1e-2, name="FFN decode fused norm vs rmsnorm")


def test_l2_prefetch_hint_runs_and_writes_nothing():
    """hymba_l2_prefetch enqueues its bulk L2 prefetches for up to 8 ranges (odd sizes
    included) on a stream and leaves every byte as it was."""
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    ts = [torch.randn(n, generator=g, device="cuda") for n in (1, 1000, 8192 + 3, 1 << 20, 5 << 20)]
    before = [t.clone() for t in ts]
    s = torch.cuda.Stream()
    H.l2_prefetch(ts, stream=s)
    H.l2_prefetch(ts[:1])
    s.synchronize()
    torch.cuda.synchronize()
    for a, b in zip(ts, before):
        assert torch.equal(a, b)


# ---------------------------------------------------------------------------------------
# decode with a position per sequence
# ---------------------------------------------------------------------------------------
def _ragged_case(dims, B, positions, seed, Lmax=None):
    rng = np.random.default_rng(seed)
    Hkv, D, M, W = dims.n_kv_heads, dims.head_dim, dims.n_meta, dims.window
    r = lambda *shape: synth.bf16_round(rng.normal(size=shape).astype(np.float32))
    st = {"x_new": r(B, dims.d_model), "ssm_state": rng.normal(size=(B, dims.d_inner, dims.d_state)).astype(np.float32),
          "conv_state": rng.normal(size=(B, dims.d_inner, dims.d_conv - 1)).astype(np.float32)}
    if dims.is_global:
        cache = {"k": r(B, Lmax, Hkv, D), "v": r(B, Lmax, Hkv, D)}
    else:
        cache = {"meta_k": r(B, M, Hkv, D), "meta_v": r(B, M, Hkv, D), "ring_k": r(B, W, Hkv, D),
                 "ring_v": r(B, W, Hkv, D)}
    return st, cache


def _ragged_run(dims, w, st, cache, positions, Lmax, dev_cache=None):
    B = len(positions)
    if dev_cache is None:
        dev_cache = H.Cache(dims, B, Lmax)
        for n, a in cache.items():
            dev_cache.t[n].copy_(f32_dev(a).to(torch.float16))
    ssm, conv = f32_dev(st["ssm_state"]), f32_dev(st["conv_state"])
    out = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
    ws = H.alloc_workspace(H.workspace_size(dims, B, Lmax, 0, H.MODE_DECODE))
    pos = torch.tensor(positions, dtype=torch.int32, device="cuda")
    H.mixer_decode_ragged(dims, H.DeviceWeights(w), bf16_dev(st["x_new"]), pos, max(positions), dev_cache, ssm,
                          conv, out, ws)
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0
    return out, ssm, conv, dev_cache


def _ragged_oracle(dims, w, st, cache, positions):
    outs, states, caches = [], [], []
    for b, p in enumerate(positions):
        cb = {n: a[b:b + 1] for n, a in cache.items()}
        r = orc.mixer_decode(dims, w, st["x_new"][b:b + 1], p, cb, st["ssm_state"][b:b + 1], st["conv_state"][b:b + 1])
        outs.append(r["out"][0]); states.append(r["ssm_state"][0]); caches.append(r["cache"])
    return np.stack(outs), np.stack(states), {n: np.concatenate([c[n] for c in caches]) for n in cache}


@pytest.mark.parametrize("is_global", [0, 1])
def test_decode_ragged_positions(is_global):
    """Sequences at different positions in one decode call: the first input token (one
    filled ring slot), a partly filled ring, a ring exactly full, a wrapped ring, and for a
    global layer caches filled to different lengths; each sequence against the oracle's
    decode at its own position, then a consumer layer reading the producer's ring."""
    dims = WL["tiny"].dims.replace(window=32, is_global=is_global,
                                   kv_role=synth.KV_OWN if is_global else synth.KV_PRODUCER)
    M, W = dims.n_meta, dims.window
    positions = [M, M + 5, M + W - 1, M + W, M + 3 * W + 7, M + 1]
    Lmax = max(positions) + 1 if is_global else 1
    w = _w(dims, seed=41)
    st, cache = _ragged_case(dims, len(positions), positions, seed=42, Lmax=Lmax)
    out, ssm, conv, dcache = _ragged_run(dims, w, st, cache, positions, Lmax)
    ref_out, ref_state, ref_cache = _ragged_oracle(dims, w, st, cache, positions)
    assert_rms(to_np(out), ref_out, name="ragged decode out")
    assert_rel_inf(to_np(ssm), ref_state, tol=1e-3, name="ragged decode ssm state")
    for b, p in enumerate(positions):   # the one cache row each sequence wrote
        if is_global:
            assert_rms(to_np(dcache.t["k"][b, p]), ref_cache["k"][b, p], name=f"k row (b={b})")
        else:
            slot = orc.ring_slot(p, M, W)
            assert_rms(to_np(dcache.t["ring_k"][b, slot]), ref_cache["ring_k"][b, slot], name=f"ring k (b={b})")
            assert_rms(to_np(dcache.t["ring_v"][b, slot]), ref_cache["ring_v"][b, slot], name=f"ring v (b={b})")
    if not is_global:   # the consumer of the pair reads the producer's updated ring
        cons = dims.replace(kv_role=synth.KV_CONSUMER)
        wc = _w(cons, seed=43)
        stc, _ = _ragged_case(cons, len(positions), positions, seed=44)
        outc, _, _, _ = _ragged_run(cons, wc, stc, None, positions, Lmax, dev_cache=dcache)
        refc, _, _ = _ragged_oracle(cons, wc, stc, ref_cache, positions)
        assert_rms(to_np(outc), refc, name="ragged decode consumer out")


def test_decode_ragged_equal_positions_is_the_uniform_step():
    """With every sequence at the same position the per-sequence step is the uniform step,
    bit for bit (Hymba-width SWA producer, batch 16)."""
    wl = WL["decode_pair"]
    dims = wl.dims
    B, p = 16, wl.decode_position
    w = _w(dims, wl=wl)
    st, cache = _ragged_case(dims, B, [p] * B, seed=45)
    out_r, ssm_r, _, cache_r = _ragged_run(dims, w, st, cache, [p] * B, 1)
    c2 = H.Cache(dims, B, 1)
    for n, a in cache.items():
        c2.t[n].copy_(f32_dev(a).to(torch.float16))
    ssm, conv = f32_dev(st["ssm_state"]), f32_dev(st["conv_state"])
    out = _decode(dims, w, c2, st["x_new"], p, ssm, conv)
    assert torch.equal(out, out_r) and torch.equal(ssm, ssm_r)
    assert torch.equal(c2.t["ring_k"], cache_r.t["ring_k"])


def test_decode_ragged_hymba_width():
    """Hymba-width SWA layer, batch 12, positions spread from the first input token to far
    past the window."""
    wl = WL["decode_pair"]
    dims = wl.dims
    rng = np.random.default_rng(46)
    positions = sorted(int(v) for v in rng.integers(dims.n_meta, dims.n_meta + 4000, size=10)) + [dims.n_meta, 1151]
    w = _w(dims, wl=wl, layer=3)
    st, cache = _ragged_case(dims, len(positions), positions, seed=47)
    out, ssm, _, _ = _ragged_run(dims, w, st, cache, positions, 1)
    ref_out, ref_state, _ = _ragged_oracle(dims, w, st, cache, positions)
    assert_rms(to_np(out), ref_out, name="ragged decode out (Hymba width)")
    assert_rel_inf(to_np(ssm), ref_state, tol=1e-3, name="ragged decode ssm state (Hymba width)")


# ---------------------------------------------------------------------------------------
# fp16 range: a layer input far outside the normalised range is reported, not hidden
# ---------------------------------------------------------------------------------------
def test_fp16_overflow_is_reported():
    """Queries, keys and values are stored in fp16.  With inputs scaled by 1e6 the
    projections exceed fp16's range (|v| >= 65520 rounds to inf); prefill and decode must
    then report HYMBA_ERR_FP16_RANGE in the status word, and a normal call must not."""
    dims = WL["tiny"].dims.replace(window=16)
    w = _w(dims, seed=31)
    rng = np.random.default_rng(32)
    X = synth.bf16_round(rng.normal(size=(1, 40, dims.d_model)).astype(np.float32))
    dw = H.DeviceWeights(w)
    for scale, want in ((1.0, H.OK), (1e6, H.ERR_FP16_RANGE)):
        x = bf16_dev(X * scale)
        T = dims.n_meta + 40
        cache = H.Cache(dims, 1, T + 1)
        out = torch.zeros(1, T, dims.d_model, dtype=torch.bfloat16, device="cuda")
        ws = H.alloc_workspace(H.workspace_size(dims, 1, 40))
        ssm = torch.zeros(1, dims.d_inner, dims.d_state, device="cuda")
        conv = torch.zeros(1, dims.d_inner, dims.d_conv - 1, device="cuda")
        H.mixer_prefill(dims, dw, x, cache, out, ws, ssm_state=ssm, conv_state=conv)
        assert H.status_read(ws) == want, f"prefill, input scale {scale}"
        if scale == 1.0:   # decode from the finite state, with a new token scaled up
            dws = H.alloc_workspace(H.workspace_size(dims, 1, T + 1, 0, H.MODE_DECODE))
            o1 = torch.zeros(1, dims.d_model, dtype=torch.bfloat16, device="cuda")
            xn = bf16_dev(synth.bf16_round(rng.normal(size=(1, dims.d_model)).astype(np.float32)) * 1e6)
            H.mixer_decode(dims, dw, xn, T, cache, ssm, conv, o1, dws)
            assert H.status_read(dws) == H.ERR_FP16_RANGE, "decode, input scale 1e6"
    assert H.status_read(ws) == 0   # read-and-clear


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
