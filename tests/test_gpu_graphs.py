"""Stream capture of the C-ABI calls.

Prefill at small batch and every decode step fork the attention onto a second stream and
join it again before the norm. A call captured into a CUDA graph must therefore be a
two-branch graph that replays to exactly the bytes of the eager call: every sum in the
path has a fixed order, so the comparison is bitwise.
"""
import numpy as np
import pytest
import torch

from hybrid_attention_ssm_b200 import hymba as H
from hybrid_attention_ssm_b200 import synth

from tests.helpers import PrefillRun, bf16_dev

pytestmark = pytest.mark.gpu

WL = synth.workloads()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.lib()


def _clone_cache(dims, batch, src, max_tokens):
    c = H.Cache(dims, batch, max_tokens)
    for n, t in src.t.items():
        c.t[n].copy_(t)
    return c


def _capture(fn):
    """Capture fn() on a side stream into a graph, then replay it once."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("is_global", [0, 1])
def test_decode_graph_replay_matches_eager(is_global):
    dims = WL["tiny"].dims.replace(is_global=is_global, window=16)
    w = synth.layer_weights(dims, seed=11)
    B, N = 3, 40
    X = synth.bf16_round(np.random.default_rng(12).normal(size=(B, N + 1, dims.d_model)).astype(np.float32))
    T = dims.n_meta + N
    run = PrefillRun(dims, w, X[:, :N], max_tokens=T + 1)
    x_new = bf16_dev(X[:, N])
    nbytes = H.workspace_size(dims, B, T + 1, 0, H.MODE_DECODE)

    def fresh():
        return (_clone_cache(dims, B, run.cache, T + 1), run.ssm.clone(), run.conv.clone(),
                torch.zeros(B, dims.d_model, dtype=torch.bfloat16, device="cuda"), H.alloc_workspace(nbytes))

    ce, se, ke, oe, wse = fresh()
    H.mixer_decode(dims, run.dw, x_new, T, ce, se, ke, oe, wse)
    torch.cuda.synchronize()
    cg, sg, kg, og, wsg = fresh()
    _capture(lambda: H.mixer_decode(dims, run.dw, x_new, T, cg, sg, kg, og, wsg))
    assert H.status_read(wse) == 0 and H.status_read(wsg) == 0
    assert torch.equal(og, oe), "decode output"
    assert torch.equal(sg, se), "SSM state"
    assert torch.equal(kg, ke), "conv state"
    for n in ce.t:
        assert torch.equal(cg.t[n], ce.t[n]), f"cache {n}"


@pytest.mark.parametrize("B", [1, 2])
def test_prefill_graph_replay_matches_eager(B):
    dims = WL["tiny"].dims.replace(window=32)
    w = synth.layer_weights(dims, seed=13)
    N = 120
    X = synth.bf16_round(np.random.default_rng(14).normal(size=(B, N, dims.d_model)).astype(np.float32))
    eager = PrefillRun(dims, w, X)
    T = dims.n_meta + N
    x = bf16_dev(X)
    cache = H.Cache(dims, B, T)
    out = torch.zeros(B, T, dims.d_model, dtype=torch.bfloat16, device="cuda")
    ssm = torch.zeros(B, dims.d_inner, dims.d_state, dtype=torch.float32, device="cuda")
    conv = torch.zeros(B, dims.d_inner, dims.d_conv - 1, dtype=torch.float32, device="cuda")
    ws = H.alloc_workspace(H.workspace_size(dims, B, N, 0))
    _capture(lambda: H.mixer_prefill(dims, eager.dw, x, cache, out, ws, ssm_state=ssm, conv_state=conv))
    assert H.status_read(ws) == 0
    assert torch.equal(out, eager.out), "prefill output"
    assert torch.equal(ssm, eager.ssm), "SSM state"
    assert torch.equal(conv, eager.conv), "conv state"
    for n in cache.t:
        assert torch.equal(cache.t[n], eager.cache.t[n]), f"cache {n}"
