"""Shared test helpers: tolerance checks and running the CUDA path on seeded inputs."""
import numpy as np
import torch

from hybrid_attention_ssm_b200 import hymba as H
from hybrid_attention_ssm_b200 import synth

BF16_TOL = 2e-2      # max|err| <= 2e-2 * RMS(ref) for bf16 paths
SCAN_TOL = 1e-4      # ||err||_inf <= 1e-4 * ||ref||_inf for the fp32 scan state


def assert_rms(got, ref, tol=BF16_TOL, name=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{name}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    ratio = err / max(rms, 1e-300)
    print(f"[parity] {name}: max|err|/RMS = {ratio:.3e} (bound {tol})")
    assert err <= tol * rms, f"{name}: max|err| {err:.4e} > {tol} * RMS {rms:.4e} (ratio {ratio:.3e})"
    return ratio


def assert_elem(got, ref, rel=5e-3, abs_rms=1e-3, name=""):
    """Elementwise bound for a stored 16-bit stage computed from exact inputs:
    |got - ref| <= rel*|ref| + abs_rms*RMS(ref) (bf16 unit roundoff is 2^-8 = 3.9e-3)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{name}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = rel * np.abs(ref) + abs_rms * rms
    bad = np.abs(got - ref) > bound
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {bad.size} elements outside rel {rel} + {abs_rms}*RMS;"
                           f" worst excess {float(np.max(np.abs(got - ref) - bound)):.3e} (RMS {rms:.3e})")


def assert_rel_inf(got, ref, tol=SCAN_TOL, name=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    den = float(np.max(np.abs(ref)))
    err = float(np.max(np.abs(got - ref)))
    assert err <= tol * den, f"{name}: inf-norm err {err:.4e} > {tol} * {den:.4e}"
    return err / max(den, 1e-300)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device).to(torch.bfloat16)


def f32_dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def ws_view(ws, off, shape, dtype):
    """A typed view into the byte workspace at byte offset `off`."""
    n = int(np.prod(shape))
    es = torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + n * es].view(dtype).view(*shape)


class PrefillRun:
    """Runs hymba_mixer_prefill once on seeded inputs and keeps every buffer."""

    def __init__(self, dims, w, X, x_has_meta=0, cache=None, residual=None, max_tokens=None):
        self.dims, self.w = dims, w
        B, n = X.shape[0], X.shape[1]
        T = n if x_has_meta else dims.n_meta + n
        self.T = T
        self.dw = H.DeviceWeights(w)
        self.x = bf16_dev(X)
        self.cache = cache if cache is not None else H.Cache(dims, B, max_tokens or T)
        self.out = torch.zeros(B, T, dims.d_model, dtype=torch.bfloat16, device="cuda")
        self.ssm = torch.zeros(B, dims.d_inner, dims.d_state, dtype=torch.float32, device="cuda")
        self.conv = torch.zeros(B, dims.d_inner, dims.d_conv - 1, dtype=torch.float32, device="cuda")
        self.res = None if residual is None else bf16_dev(residual)
        nbytes = H.workspace_size(dims, B, n, x_has_meta)
        self.ws = H.alloc_workspace(nbytes)
        H.mixer_prefill(dims, self.dw, self.x, self.cache, self.out, self.ws, x_has_meta=x_has_meta,
                        ssm_state=self.ssm, conv_state=self.conv, residual=self.res)
        torch.cuda.synchronize()
        assert H.status_read(self.ws) == 0
        self.layout = H.stage_layout(dims, B, n, x_has_meta)
        self.B = B

    def stage(self, name, b=None):
        """A stage buffer as float64 [B, T, ...], or only sequence b's [T, ...] when b is given."""
        d, L, B, T = self.dims, self.layout, self.B, self.T
        shapes = {
            "q": (L.q, (B, T, d.n_q_heads, d.head_dim), torch.float16),
            "xz": (L.xz, (B, T, 2 * d.d_inner), torch.bfloat16),
            "xc": (L.xc, (B, T, d.d_inner), torch.bfloat16),
            "xbc": (L.xbc, (B, T, L.ld_xbc), torch.float32),
            "dt_pre": (L.dt_pre, (B, T, d.d_inner), torch.bfloat16),
            "y": (L.y, (B, T, d.d_inner), torch.bfloat16),
            "o": (L.o, (B, T, d.n_q_heads * d.head_dim), torch.float32),
            "u": (L.u, (B, T, d.attn_width + d.d_inner), torch.float16),
        }
        off, shape, dt = shapes[name]
        v = ws_view(self.ws, off, shape, dt)
        return to_np(v if b is None else v[b])

    def kv(self):
        T = self.T
        return to_np(self.cache.t["k"][:, :T]), to_np(self.cache.t["v"][:, :T])
