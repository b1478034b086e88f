"""Full-size parity: the Hymba-1.5B-shaped global layer (batch 4, 128 meta + 8192 tokens)
and the 32-layer stack (batch 8, 128 meta + 4096 tokens), on outputs the fp64 oracle can
compute at these sizes: sampled rows of the global layer (every stage the rows depend on is
computed in full), and, for the stack, the mixer and FFN of selected layers teacher-forced on
the GPU's own layer inputs (sequence 0)."""
import numpy as np
import pytest
import torch

from hybrid_attention_ssm_b200 import hymba as H
from hybrid_attention_ssm_b200 import synth
from hybrid_attention_ssm_b200.stack import HymbaStack
from oracle import hymba_oracle as orc
from tests.helpers import PrefillRun, assert_elem, assert_rel_inf, assert_rms, to_np

pytestmark = pytest.mark.gpu

WL = synth.workloads()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.lib()


def _sampled_rows(T, M, n, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, M - 1, M, M + 1, T // 2, T - 2, T - 1]
    extra = rng.choice(np.arange(T), size=n - len(fixed), replace=False)
    return np.unique(np.concatenate([fixed, extra]))


def _oracle_rows(dims, w, Xt_b, rows):
    """Oracle output rows of one sequence: in_proj, conv and scan over every row, attention
    and the output projection for the sampled rows only."""
    T = Xt_b.shape[0]
    pos = np.arange(T)
    proj = Xt_b @ w["w_in"].astype(np.float64).T
    Qf, Kf, Vf, xs, z = orc.split_in_proj(proj, dims)
    Hq, Hkv, D = dims.n_q_heads, dims.n_kv_heads, dims.head_dim
    Q = orc.rope(Qf.reshape(T, Hq, D), pos, dims.rope_base)
    K = orc.rope(Kf.reshape(T, Hkv, D), pos, dims.rope_base)
    V = Vf.reshape(T, Hkv, D)
    O = orc.attention(Q[rows], K, V, rows, pos, dims.n_meta, dims.window, dims.is_global).reshape(len(rows), -1)
    xc, _ = orc.causal_conv1d_silu(xs, w["conv_w"], w["conv_b"])
    delta, Bm, Cm, _ = orc.ssm_params(xc, w["w_x"], w["w_dt"], w["dt_bias"], dims.dt_rank, dims.d_state)
    y, h = orc.selective_scan(xc, delta, w["A"], Bm, Cm, z)
    out, _ = orc.fuse_and_project(O, y[rows], w, dims)
    return out, h


def test_global_layer_full_size_sampled_rows():
    wl = WL["global"]
    dims = wl.dims
    w = synth.layer_weights(dims, dt_bias_mean=wl.dt_bias_mean, dt_bias_std=wl.dt_bias_std)
    X = synth.prefill_input(wl)
    run = PrefillRun(dims, w, X)
    T = run.T
    out = to_np(run.out)
    R = w["meta"].astype(np.float64)
    for b in (0, wl.batch - 1):
        rows = _sampled_rows(T, dims.n_meta, 40, seed=b)
        Xt_b = np.concatenate([R, X[b].astype(np.float64)], axis=0)
        ref, h = _oracle_rows(dims, w, Xt_b, rows)
        assert_rms(out[b, rows], ref, name=f"global layer rows (b={b})")
        assert_rel_inf(to_np(run.ssm[b]), h, tol=2e-2, name=f"global layer ssm state (b={b})")
        # the scan over all 8320 steps, fed its own inputs (dt_pre, xc, B, C): fp32 state at 1e-4
        xc, dt_pre, xbc = run.stage("xc", b), run.stage("dt_pre", b), run.stage("xbc", b)
        R_, S = dims.dt_rank, dims.d_state
        delta = orc.softplus(dt_pre + w["dt_bias"])
        _, h_own = orc.selective_scan(xc, delta, w["A"], xbc[:, R_:R_ + S], xbc[:, R_ + S:R_ + 2 * S],
                                      np.zeros_like(xc))
        assert_rel_inf(to_np(run.ssm[b]), h_own, tol=1e-4, name=f"global layer scan state, own inputs (b={b})")


def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return np.exp2(e - 7)


def test_stack_32_layers_teacher_forced():
    wl = WL["stack"]
    st = HymbaStack(wl, seed=0, keep_host_weights=True)
    E = torch.from_numpy(synth.stack_embeddings(wl)).cuda().to(torch.bfloat16)
    check_layers = [0, 1, 2, 15, 16, 30, 31]
    record = {l: [] for l in check_layers}
    out = st.forward(E, record=record)
    torch.cuda.synchronize()
    assert H.status_read(st.ws) == 0
    assert torch.isfinite(out.float()).all().item()
    T, d = st.T, wl.dims.d_model
    ws = H.alloc_workspace(H.workspace_size(wl.dims, 1, T, 1))
    for l in check_layers:
        dl, w, bw = st.host[l]
        _, dw, dev = st.layers[l]
        items = record[l]
        _, h_in, h_mid, h_out = items[-1]
        # the stack's residual adds: h_mid = h_in + mixer, h_out = h_mid + FFN, in bf16
        # mixer and FFN of this layer, rerun without the residual on the recorded input
        x = torch.from_numpy(h_in[None].astype(np.float32)).cuda().to(torch.bfloat16)
        hn = torch.empty_like(x)
        H.rmsnorm(x.view(T, d), dev["g1"], dl.norm_eps, hn.view(T, d))
        cache = H.Cache(dl, 1, T, kind=H.CACHE_GLOBAL if dl.is_global else H.CACHE_SWA)
        kv_in = None
        if dl.kv_role == synth.KV_CONSUMER:
            _, k, v = items[0]
            cache.t["k"][0].copy_(torch.from_numpy(k.astype(np.float32)).cuda().to(torch.float16))
            cache.t["v"][0].copy_(torch.from_numpy(v.astype(np.float32)).cuda().to(torch.float16))
            kv_in = (k[None], v[None])
        mix = torch.empty_like(x)
        H.mixer_prefill(dl, dw, hn, cache, mix, ws, x_has_meta=1)
        x2 = torch.from_numpy(h_mid.astype(np.float32)).cuda().to(torch.bfloat16)
        hn2 = torch.empty_like(x2)
        H.rmsnorm(x2, dev["g2"], dl.norm_eps, hn2)
        act = torch.empty(T, st.F, dtype=torch.float16, device="cuda")
        ffn = torch.empty_like(x2)
        H.ffn_swiglu(hn2, dev["w_gu"], dev["w_down"], act, ffn, ws)
        torch.cuda.synchronize()
        assert H.status_read(ws) == 0
        mix_np, ffn_np = to_np(mix)[0], to_np(ffn)
        hn_np, hn2_np = to_np(hn)[0], to_np(hn2)
        tag = f"layer {l} (kv role {dl.kv_role}, global {dl.is_global})"
        # RMSNorm against the oracle, elementwise (bf16 output)
        assert_elem(hn_np, orc.rmsnorm(h_in, bw["g_norm1"], dl.norm_eps), name=f"{tag} norm 1")
        assert_elem(hn2_np, orc.rmsnorm(h_mid, bw["g_norm2"], dl.norm_eps), name=f"{tag} norm 2")
        # mixer and FFN teacher-forced on the GPU's normed inputs
        ref_mix = orc.mixer_prefill(dl, w, hn_np[None], x_has_meta=True, kv_in=kv_in)["out"][0]
        assert_rms(mix_np, ref_mix, name=f"{tag} mixer")
        assert_rms(ffn_np, orc.ffn_swiglu(hn2_np, bw), name=f"{tag} FFN")
        # residual adds of the stack, within one bf16 step of the stored stream
        assert np.all(np.abs(h_mid - (h_in + mix_np)) <= _bf16_ulp(h_mid) + _bf16_ulp(mix_np)), f"{tag}: mixer residual"
        assert np.all(np.abs(h_out - (h_mid + ffn_np)) <= _bf16_ulp(h_out) + _bf16_ulp(ffn_np)), f"{tag}: FFN residual"


def test_stack_32_layers_decode_step():
    """The 32-layer decode step (first, middle and last layers global with full-length
    caches; SWA pairs sharing one ring; each layer's FFN): prefill of the first N-1 tokens,
    then one decode step for token N at position M + N - 1 for all 8 sequences.
    - Every checked layer's mixer and FFN, rerun on copies of the inputs, caches and states
      that layer saw inside the step, against the oracle's decode (bf16 bound), and the
      stack's residual adds within one bf16 step.
    - End to end, the decoded stream equals the last row of the 32-layer prefill of all N
      tokens (different kernels and summation orders on the two paths; a wrong cache slot,
      state or pairing would be an O(1) error): max|err| <= 1e-1 RMS."""
    wl = WL["stack"]
    st = HymbaStack(wl, seed=0, keep_host_weights=True, decode_room=1)
    E = torch.from_numpy(synth.stack_embeddings(wl)).cuda().to(torch.bfloat16)
    N, d = wl.n_tokens, wl.dims.d_model
    check_layers = [0, 1, 2, 15, 16, 30, 31]
    frec = {l: [] for l in check_layers}
    full_last = to_np(st.forward(E, record=frec)[:, -1])
    st.forward(E[:, :N - 1].contiguous())
    rec = {l: {} for l in check_layers}
    p = wl.dims.n_meta + N - 1
    h = to_np(st.decode_step(E[:, N - 1].contiguous(), p, record=rec))
    torch.cuda.synchronize()
    assert H.status_read(st.dws) == 0 and H.status_read(st.ws) == 0 and H.status_read(st.fws) == 0
    # drift of the decode path from the prefill path, layer by layer (sequence 0): it starts
    # at zero (same embedding) and grows by the two paths' independent bf16 roundings
    for l in check_layers:
        h_pre = [it for it in frec[l] if it[0] == "h"][-1][1][-1]
        assert_rms(rec[l]["h_in"][0], h_pre, tol=5e-2 if l <= 2 else 1.5e-1,
                           name=f"decode vs prefill stream entering layer {l}")
    assert_rms(h, full_last, tol=1.5e-1, name="32-layer decode step vs last row of the 32-layer prefill")
    B = wl.batch
    for l in check_layers:
        dl, w, bw = st.host[l]
        _, dw, dev = st.layers[l]
        r = rec[l]
        tag = f"decode layer {l} (kv role {dl.kv_role}, global {dl.is_global})"
        # the mixer, rerun without the residual on copies of what the layer saw
        cache = H.Cache(dl, B, st.max_tokens)
        for n, arr in r["cache"].items():
            cache.t[n].copy_(torch.from_numpy(arr.astype(np.float32)).cuda().to(torch.float16))
        ssm = torch.from_numpy(r["ssm"]).cuda()
        conv = torch.from_numpy(r["conv"]).cuda()
        ws = H.alloc_workspace(H.workspace_size(dl, B, st.max_tokens, 0, H.MODE_DECODE))
        mix = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
        H.mixer_decode(dl, dw, torch.from_numpy(r["hn"].astype(np.float32)).cuda().to(torch.bfloat16), p, cache,
                       ssm, conv, mix, ws)
        ffn = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
        fws = H.alloc_workspace(H.ffn_workspace_size(B, d, st.F))
        H.ffn_swiglu_decode(torch.from_numpy(r["hn2"].astype(np.float32)).cuda().to(torch.bfloat16), dev["w_gu"],
                            dev["w_down"], ffn, fws)
        torch.cuda.synchronize()
        assert H.status_read(ws) == 0 and H.status_read(fws) == 0
        ocache = r["cache"] if dl.is_global else {n: r["cache"][n] for n in ("meta_k", "meta_v", "ring_k", "ring_v")}
        ref = orc.mixer_decode(dl, w, r["hn"], p, ocache, r["ssm"], r["conv"])
        mix_np, ffn_np = to_np(mix), to_np(ffn)
        assert_rms(mix_np, ref["out"], name=f"{tag} mixer")
        assert_rms(ffn_np, orc.ffn_swiglu(r["hn2"], bw), name=f"{tag} FFN")
        assert_elem(r["hn"], orc.rmsnorm(r["h_in"], bw["g_norm1"], dl.norm_eps), name=f"{tag} norm 1")
        assert_elem(r["hn2"], orc.rmsnorm(r["h_mid"], bw["g_norm2"], dl.norm_eps), name=f"{tag} norm 2")
        assert np.all(np.abs(r["h_mid"] - (r["h_in"] + mix_np)) <= _bf16_ulp(r["h_mid"]) + _bf16_ulp(mix_np)), \
            f"{tag}: mixer residual"
        assert np.all(np.abs(r["h_out"] - (r["h_mid"] + ffn_np)) <= _bf16_ulp(r["h_out"]) + _bf16_ulp(ffn_np)), \
            f"{tag}: FFN residual"
        # the layer's states after the step agree with the oracle's
        # (through the bf16 conv output of the new token, as every end-to-end state check)
        assert_rel_inf(st.ssm[l].cpu().numpy(), ref["ssm_state"], tol=2e-2, name=f"{tag} ssm state")
