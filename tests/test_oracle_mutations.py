"""The pins catch plausible mistakes in the oracle.

Each case below plants one plausible mistake in the oracle on the CPU: a wrong sign, a
dropped term, a swapped operand, an off-by-one edge or a wrong index map. It then runs
every pin of tests/test_oracle_pins.py against the changed oracle. At least one pin must
fail for each planted mistake; otherwise the pins would let that mistake through, and the
GPU path would be checked against a wrong reference.

Two kinds of change are not planted:
- readings of silent passages (the RoPE pairing, the 1/2 of the average, the RMSNorm eps),
  which no passage fixes, so no pin can;
- layout conventions that the prefill and the decode of the oracle share by construction,
  such as the ring slot of a position. The mixer's outputs do not depend on them, and the
  GPU parity tests compare the caches slot by slot.
"""
import numpy as np
import pytest

from oracle import hymba_oracle as orc
from tests import test_oracle_pins as pins

ORIG = {name: getattr(orc, name) for name in
        ("selective_scan", "causal_conv1d_silu", "visibility_mask", "attention", "softplus", "ssm_params",
         "split_in_proj", "rmsnorm", "silu", "rope", "ffn_swiglu", "hymba_block")}


def _pin_calls(golden_dir):
    calls = [
        ("scan vs eq. (2) brute force", pins.test_scan_matches_bruteforce_eq2, {}),
        ("scan hand-derived", pins.test_scan_hand_derived, {"golden_dir": golden_dir}),
        ("scan state carry", pins.test_scan_state_carry_is_associative, {}),
        ("scan zero delta", pins.test_scan_zero_delta_keeps_state, {}),
        ("conv one-hot shift", pins.test_conv_one_hot_is_shift, {}),
        ("conv state carry", pins.test_conv_state_carry, {}),
        ("closed forms", pins.test_elementwise_closed_forms, {}),
        ("x_proj column layout", pins.test_x_proj_column_layout, {}),
        ("attention hand-derived", pins.test_attention_hand_derived, {"golden_dir": golden_dir}),
        ("window 1", pins.test_window_one_sees_meta_and_self, {}),
        ("rope", pins.test_rope_relative_position_and_norm, {}),
        ("window covering sequence", pins.test_window_covering_sequence_equals_global, {}),
        ("meta rows", pins.test_meta_rows_independent_of_input, {}),
        ("consumer reuses producer kv", pins.test_consumer_reuses_producer_kv, {}),
        ("norm invariances", pins.test_norm_scale_invariances, {}),
        ("tied out_proj", pins.test_tied_out_proj_reduces_to_printed_fusion, {}),
        ("consumer decode ring", pins.test_consumer_decode_reads_producer_ring, {}),
        ("kv share plan", pins.test_kv_share_plan_hymba_layout, {}),
        ("block residual", pins.test_block_residual_identity, {}),
        ("ffn hand-derived", pins.test_ffn_swiglu_hand_derived, {"golden_dir": golden_dir}),
        ("block = its sublayers in order", pins.test_block_is_its_two_sublayers_in_order, {}),
        ("block pre-norm", pins.test_block_sublayers_read_normalised_stream, {}),
    ]
    for args in [(1, 0, 3), (0, 4, 3), (0, 1, 2), (0, 7, 0)]:
        calls.append((f"attention vs SDPA {args}", pins.test_attention_matches_torch_sdpa,
                      dict(zip(("is_global", "W", "M"), args))))
    for g in (0, 1):
        calls.append((f"prefill then decode (global={g})", pins.test_prefill_then_decode_equals_longer_prefill,
                      {"is_global": g}))
    return calls


def _failing_pins(golden_dir):
    failed = []
    for name, fn, kw in _pin_calls(golden_dir):
        try:
            with np.errstate(all="ignore"):   # a planted mistake may well overflow
                fn(**kw)
        except Exception:  # noqa: BLE001  a pin that raises (assertion or otherwise) caught it
            failed.append(name)
    return failed


# ---------------------------------------------------------------------------------------
# the planted mistakes
# ---------------------------------------------------------------------------------------
def _scan_loop(xc, delta, A, Bm, Cm, z, h0=None, out_before_update=False, gate=True):
    xc, delta, A = (np.asarray(a, dtype=np.float64) for a in (xc, delta, A))
    Bm, Cm = np.asarray(Bm, dtype=np.float64), np.asarray(Cm, dtype=np.float64)
    h = np.zeros_like(A) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.zeros(xc.shape)
    for t in range(xc.shape[0]):
        if out_before_update:
            y[t] = h @ Cm[t]
        h = np.exp(delta[t][:, None] * A) * h + (delta[t] * xc[t])[:, None] * Bm[t][None, :]
        if not out_before_update:
            y[t] = h @ Cm[t]
    return (y * ORIG["silu"](z) if gate else y), h


def _attention_gqa_modulo(Q, K, V, q_pos, k_pos, n_meta, window, is_global):
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    Lq, Hq, D = Q.shape
    Hkv = K.shape[1]
    mask = orc.visibility_mask(q_pos, k_pos, n_meta, window, is_global)
    out = np.zeros((Lq, Hq, D))
    for h in range(Hq):
        g = h % Hkv
        s = np.where(mask, (Q[:, h] @ K[:, g].T) / np.sqrt(D), -np.inf)
        p = np.where(mask, np.exp(s - s.max(axis=1, keepdims=True)), 0.0)
        out[:, h] = (p / p.sum(axis=1, keepdims=True)) @ V[:, g]
    return out


def _conv_no_silu(x, w, b, x_prev=None):
    x, w = np.asarray(x, dtype=np.float64), np.asarray(w, dtype=np.float64)
    L, kc = x.shape[0], w.shape[1]
    head = np.zeros((kc - 1, x.shape[1])) if x_prev is None else np.asarray(x_prev, dtype=np.float64).T
    xp = np.concatenate([head, x], axis=0)
    acc = np.zeros(x.shape) + np.asarray(b, dtype=np.float64)[None, :]
    for k in range(kc):
        acc += w[None, :, k] * xp[k:k + L]
    return acc, xp[L:].T.copy()


def _swap_bc(*a, **k):
    delta, Bm, Cm, dt_low = ORIG["ssm_params"](*a, **k)
    return delta, Cm, Bm, dt_low


def _swap_kv(proj, dims):
    Q, K, V, xs, z = ORIG["split_in_proj"](proj, dims)
    return Q, V, K, xs, z


def _ffn_variant(v, bw, swap=False, silu_on_up=False, add=False):
    v = np.asarray(v, dtype=np.float64)
    g = v @ np.asarray(bw["w_gate"], dtype=np.float64).T
    u = v @ np.asarray(bw["w_up"], dtype=np.float64).T
    if swap:
        g, u = u, g
    if silu_on_up:
        act = g * ORIG["silu"](u)
    elif add:
        act = ORIG["silu"](g) + u
    else:
        act = ORIG["silu"](g) * u
    return act @ np.asarray(bw["w_down"], dtype=np.float64).T


def _block_variant(dims, w, bw, H, kv_in=None, norm2_on_input=False, no_ffn_residual=False, no_norm1=False):
    h_in = H if no_norm1 else orc.rmsnorm(H, bw["g_norm1"], dims.norm_eps)
    r = orc.mixer_prefill(dims, w, h_in, x_has_meta=True, kv_in=kv_in, residual=H)
    H1 = r["out"]
    f = orc.ffn_swiglu(orc.rmsnorm(H if norm2_on_input else H1, bw["g_norm2"], dims.norm_eps), bw)
    return (f if no_ffn_residual else H1 + f), r


MISTAKES = {
    "scan: exponent sign flipped": ("selective_scan",
                                    lambda xc, d, A, Bm, Cm, z, h0=None: ORIG["selective_scan"](xc, d, -np.asarray(A), Bm, Cm, z, h0)),
    "scan: x dropped from the input term": ("selective_scan",
                                            lambda xc, d, A, Bm, Cm, z, h0=None: _scan_loop(np.ones_like(np.asarray(xc, dtype=np.float64)), d, A, Bm, Cm, z, h0)),
    "scan: output read before the state update": ("selective_scan",
                                                  lambda *a, **k: _scan_loop(*a, out_before_update=True, **k)),
    "scan: output gate dropped": ("selective_scan", lambda *a, **k: _scan_loop(*a, gate=False, **k)),
    "conv: taps reversed": ("causal_conv1d_silu",
                            lambda x, w, b, x_prev=None: ORIG["causal_conv1d_silu"](x, np.asarray(w)[:, ::-1], b, x_prev)),
    "conv: SiLU dropped": ("causal_conv1d_silu", _conv_no_silu),
    "attention: window edge one step too wide": ("visibility_mask",
                                                 lambda q, k, M, W, g: ORIG["visibility_mask"](q, k, M, W + 1, g)),
    "attention: meta keys not kept visible": ("visibility_mask",
                                              lambda q, k, M, W, g: ORIG["visibility_mask"](q, k, 0, W, g)),
    "attention: causal mask dropped": ("visibility_mask",
                                       lambda q, k, M, W, g: np.ones((len(q), len(k)), dtype=bool)),
    "attention: 1/sqrt(D) scale dropped": ("attention",
                                           lambda Q, K, V, *r: ORIG["attention"](np.asarray(Q) * np.sqrt(np.shape(Q)[-1]), K, V, *r)),
    "attention: GQA head map h mod Hkv": ("attention", _attention_gqa_modulo),
    "softplus replaced by ReLU": ("softplus", lambda x: np.maximum(np.asarray(x, dtype=np.float64), 0.0)),
    "x_proj: B and C swapped": ("ssm_params", _swap_bc),
    "in_proj: K and V columns swapped": ("split_in_proj", _swap_kv),
    "RMSNorm: sum of squares instead of the mean": ("rmsnorm",
                                                    lambda v, gain, eps: np.asarray(v, dtype=np.float64) / np.sqrt(
                                                        np.sum(np.asarray(v, dtype=np.float64) ** 2, axis=-1, keepdims=True) + eps)
                                                    * np.asarray(gain, dtype=np.float64)),
    "RMSNorm: gain dropped": ("rmsnorm", lambda v, gain, eps: ORIG["rmsnorm"](v, np.ones_like(np.asarray(gain, dtype=np.float64)), eps)),
    "SiLU replaced by sigmoid": ("silu", lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))),
    "FFN: gate and up swapped": ("ffn_swiglu", lambda v, bw: _ffn_variant(v, bw, swap=True)),
    "FFN: SiLU applied to the up branch": ("ffn_swiglu", lambda v, bw: _ffn_variant(v, bw, silu_on_up=True)),
    "FFN: product replaced by a sum": ("ffn_swiglu", lambda v, bw: _ffn_variant(v, bw, add=True)),
    "block: second norm applied to the block input": (
        "hymba_block", lambda *a, **k: _block_variant(*a, norm2_on_input=True, **k)),
    "block: FFN residual dropped": ("hymba_block", lambda *a, **k: _block_variant(*a, no_ffn_residual=True, **k)),
    "block: mixer reads the un-normalised stream": (
        "hymba_block", lambda *a, **k: _block_variant(*a, no_norm1=True, **k)),
    "RoPE: angle sign flipped for every other position": (
        "rope", lambda x, positions, base: ORIG["rope"](x, np.asarray(positions) * np.where(np.arange(len(positions)) % 2, -1, 1), base)),
}


def test_pins_pass_on_the_oracle(golden_dir):
    assert _failing_pins(golden_dir) == []


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_planted_mistake_fails_a_pin(mistake, golden_dir, monkeypatch):
    name, fn = MISTAKES[mistake]
    monkeypatch.setattr(orc, name, fn)
    failed = _failing_pins(golden_dir)
    assert failed, f"no pin catches: {mistake}"
