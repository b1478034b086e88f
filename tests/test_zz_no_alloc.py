"""hymba_mixer_decode_noalloc: the decode step for callers that cannot allocate device
memory (a serving loop that must not take cudaMalloc's device synchronisation between
tokens, or a plugin whose host runtime owns all device memory).  It
keeps its scratch in a built-in device array instead of a caller workspace, so it must give
the same results as hymba_mixer_decode with a workspace, call after call, although the
array keeps the previous call's contents.

This file is collected last on purpose: it runs after every other test in a full run and
must also pass alone in a fresh process."""
import numpy as np
import pytest
import torch

from hybrid_attention_ssm_b200 import hymba as H
from hybrid_attention_ssm_b200 import synth
from tests.helpers import assert_rel_inf, assert_rms, to_np

pytestmark = pytest.mark.gpu


def _layer_state(wl, dims, layer, cache_src):
    st = synth.decode_state(wl, layer=layer)
    cache = H.Cache(dims, wl.batch, 1)
    for n in ("meta_k", "meta_v", "ring_k", "ring_v"):
        cache.t[n].copy_(torch.from_numpy(cache_src[n]).cuda().to(torch.float16))
    return (st, cache, torch.from_numpy(st["ssm_state"]).cuda(), torch.from_numpy(st["conv_state"]).cuda())


def test_decode_noalloc_matches_workspace_path_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = synth.workloads()["decode_pair"]
    dims = wl.dims
    B, p = wl.batch, wl.decode_position
    w = synth.layer_weights(dims, seed=0, dt_bias_mean=wl.dt_bias_mean, dt_bias_std=wl.dt_bias_std)
    dw = H.DeviceWeights(w)
    src = synth.decode_state(wl, layer=0)
    rng = np.random.default_rng(11)
    xs = [torch.from_numpy(synth.bf16_round(rng.normal(size=(B, dims.d_model)).astype(np.float32))).cuda().to(
        torch.bfloat16) for _ in range(2)]

    # existing entry point, caller workspace
    _, cache_a, ssm_a, conv_a = _layer_state(wl, dims, 0, src)
    ws = H.alloc_workspace(H.workspace_size(dims, B, cache_a.c.max_tokens, 0, H.MODE_DECODE))
    outs_a = []
    for i in range(2):
        o = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
        H.mixer_decode(dims, dw, xs[i], p + i, cache_a, ssm_a, conv_a, o, ws)
        outs_a.append(o)
    torch.cuda.synchronize()
    assert H.status_read(ws) == 0

    # built-in scratch, same inputs, two calls in a row
    _, cache_b, ssm_b, conv_b = _layer_state(wl, dims, 0, src)
    outs_b = []
    for i in range(2):
        o = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
        H.mixer_decode_noalloc(dims, dw, xs[i], p + i, cache_b, ssm_b, conv_b, o)
        outs_b.append(o)
    torch.cuda.synchronize()

    for i in range(2):
        assert_rms(to_np(outs_b[i]), to_np(outs_a[i]), name=f"noalloc decode call {i}")
    assert_rel_inf(to_np(ssm_b), to_np(ssm_a), tol=1e-4, name="ssm state after two calls")
    assert_rel_inf(to_np(conv_b), to_np(conv_a), tol=1e-6, name="conv state after two calls")
    for n in ("ring_k", "ring_v"):
        assert torch.equal(cache_a.t[n], cache_b.t[n]), n


def test_decode_noalloc_rejects_oversized_steps():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dims = synth.workloads()["decode_pair"].dims.replace(is_global=1, kv_role=synth.KV_OWN)
    B, max_tokens = 64, 16384            # partials for 16384 keys exceed the built-in scratch
    need = H.workspace_size(dims, B, max_tokens, 0, H.MODE_DECODE)
    assert need > 32 << 20
    w = synth.layer_weights(dims, seed=1)
    dw = H.DeviceWeights(w)
    cache = H.Cache(dims, B, max_tokens)
    ssm = torch.zeros(B, dims.d_inner, 16, device="cuda")
    conv = torch.zeros(B, dims.d_inner, 3, device="cuda")
    x = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HymbaError) as e:
        H.mixer_decode_noalloc(dims, dw, x, 200, cache, ssm, conv, out)
    assert e.value.code == H.ERR_WORKSPACE
