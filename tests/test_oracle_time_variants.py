"""Pins of the oracle's two other time-conditioning variants: Pi0's concat
time MLP (reading R16) and DM0.5's per-layer time modulator (reading R17,
the adaLN-Zero form), against closed forms, a cross-variant identity and an
independent PyTorch statement.

A slip in either -- e(t) in the wrong half of the concatenation, a
modulation chunk taken in the wrong order, a gate applied to the residual
instead of the branch, a shift added before the scale -- fails one of these.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import expert as O
from synthetic import get_config, make_noise, make_prefix_kv, make_state, make_weights
from tests import torch_restatement as TR


def tiny(**kw):
    return get_config("tiny-fp32", **kw)


def _vel(W, cfg, t, seed=0):
    kv = make_prefix_kv(cfg, seed=seed)
    x = make_noise(cfg, seed=seed)[0]
    state = make_state(cfg, seed=seed)[0]
    return O.expert_velocity(W, cfg, x, state, t, kv[:, 0, 0], kv[:, 1, 0])


# ---------------------------------------------------------------------------
# Pi0 concat time MLP
# ---------------------------------------------------------------------------

def test_concat_zero_layers_closed_form():
    """Layer matrices 0: v = W_ao . RMSNorm_f(W_to . swish(W_ti . [a ; e(t)] + b_ti) + b_to) + b_ao."""
    cfg = tiny(time_cond="concat")
    W = O.to_f64(make_weights(cfg))
    for k in W:
        if k.startswith("layers.") and k.endswith(".w"):
            W[k][:] = 0.0
    t = 0.35
    v = _vel(W, cfg, t)
    x = make_noise(cfg)[0].astype(np.float64)
    a = x @ W["action_in_proj.w"].T + W["action_in_proj.b"]
    half = cfg.width // 2
    period = 4e-3 * (4.0 / 4e-3) ** (np.arange(half) / (half - 1))
    e = np.concatenate([np.sin(2 * math.pi * t / period), np.cos(2 * math.pi * t / period)])
    z = np.concatenate([a, np.tile(e, (a.shape[0], 1))], axis=1) @ W["time_mlp_in.w"].T + W["time_mlp_in.b"]
    tok = (z / (1 + np.exp(-z))) @ W["time_mlp_out.w"].T + W["time_mlp_out.b"]
    hn = F.rms_norm(torch.tensor(tok), (cfg.width,), weight=1.0 + torch.tensor(W["final_norm.g"]),
                    eps=cfg.rms_eps).numpy()
    np.testing.assert_allclose(v, hn @ W["action_out_proj.w"].T + W["action_out_proj.b"], rtol=1e-11, atol=1e-12)


def test_concat_time_half_zero_makes_the_velocity_time_free():
    cfg = tiny(time_cond="concat")
    W = O.to_f64(make_weights(cfg))
    W["time_mlp_in.w"][:, cfg.width:] = 0.0
    np.testing.assert_array_equal(_vel(W, cfg, 0.1), _vel(W, cfg, 0.9))
    W2 = O.to_f64(make_weights(cfg))
    assert np.max(np.abs(_vel(W2, cfg, 0.1) - _vel(W2, cfg, 0.9))) > 1e-6


# ---------------------------------------------------------------------------
# DM0.5 per-layer time modulator
# ---------------------------------------------------------------------------

def _modulator(W, cfg, scale_a, shift_a, gate_a, scale_m, shift_m, gate_m):
    w = cfg.width
    for l in range(cfg.n_layers):
        W[f"layers.{l}.time_mod.w"][:] = 0.0
        W[f"layers.{l}.time_mod.b"][:] = np.concatenate(
            [np.full(w, v) for v in (scale_a, shift_a, gate_a, scale_m, shift_m, gate_m)])


def test_adarms_unit_gates_equal_the_plain_expert_with_zero_gains():
    """time_mod.w = 0 and biases (scale 0, shift 0, gate 1): each layer is the
    plain layer with gains g = 0, and c(t) reaches nothing -- the velocity
    equals the "add" expert's with zero norm gains and a zero time MLP."""
    cfg = tiny(time_cond="adarms")
    W = O.to_f64(make_weights(cfg, seed=2))
    _modulator(W, cfg, 0.0, 0.0, 1.0, 0.0, 0.0, 1.0)
    plain = tiny()
    Wp = O.to_f64(make_weights(plain, seed=2))
    for k in list(W):
        if k in Wp and not k.startswith("time_mlp"):
            Wp[k] = W[k]
    for l in range(cfg.n_layers):
        Wp[f"layers.{l}.attn_norm.g"][:] = 0.0
        Wp[f"layers.{l}.mlp_norm.g"][:] = 0.0
    for k in ("time_mlp_in.w", "time_mlp_in.b", "time_mlp_out.w", "time_mlp_out.b"):
        Wp[k] = np.zeros_like(Wp[k])
    np.testing.assert_allclose(_vel(W, cfg, 0.6, seed=2), _vel(Wp, plain, 0.6, seed=2), rtol=1e-12, atol=1e-13)


def test_adarms_zero_gates_skip_every_layer():
    """Gates 0: no branch reaches the residual, so v is the head on the
    final norm of the action embeddings, whatever scale and shift are."""
    cfg = tiny(time_cond="adarms")
    W = O.to_f64(make_weights(cfg, seed=3))
    _modulator(W, cfg, 0.7, -0.3, 0.0, 0.2, 0.5, 0.0)
    v = _vel(W, cfg, 0.4, seed=3)
    x = make_noise(cfg, seed=3)[0].astype(np.float64)
    a = x @ W["action_in_proj.w"].T + W["action_in_proj.b"]
    hn = F.rms_norm(torch.tensor(a), (cfg.width,), weight=1.0 + torch.tensor(W["final_norm.g"]),
                    eps=cfg.rms_eps).numpy()
    np.testing.assert_allclose(v, hn @ W["action_out_proj.w"].T + W["action_out_proj.b"], rtol=1e-11, atol=1e-12)


def test_adarms_shift_is_added_after_the_scale():
    """With scale s and shift b on the attention norm only, a one-layer
    expert's q/k/v inputs are x/rms(x) (1 + s) + b: checked through the
    single-layer velocity against a hand composition in PyTorch."""
    cfg = tiny(time_cond="adarms", n_layers=1)
    W = O.to_f64(make_weights(cfg, seed=4))
    ref = TR.velocity(W, cfg, make_noise(cfg, seed=4), make_state(cfg, seed=4)[0], (0.3,),
                      make_prefix_kv(cfg, seed=4)[:, 0, 0], make_prefix_kv(cfg, seed=4)[:, 1, 0])
    np.testing.assert_allclose(_vel(W, cfg, 0.3, seed=4), ref[0], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("tc,mode", [("concat", "bidir"), ("adarms", "bidir"), ("adarms", "pi0_block"),
                                     ("concat", "pi0_block")])
def test_variants_match_independent_torch_statement(tc, mode):
    cfg = tiny(time_cond=tc, suffix_mask=mode)
    W = O.to_f64(make_weights(cfg, seed=5))
    kv = make_prefix_kv(cfg, seed=5)
    state = make_state(cfg, seed=5)[0]
    xs = np.stack([make_noise(cfg, seed=s)[0] for s in (5, 6)])
    ts = (0.8, 0.15)
    ref = TR.velocity(W, cfg, xs, state, ts, kv[:, 0, 0], kv[:, 1, 0])
    for g in range(2):
        v = O.expert_velocity(W, cfg, xs[g], state, ts[g], kv[:, 0, 0], kv[:, 1, 0])
        np.testing.assert_allclose(v, ref[g], rtol=1e-10, atol=1e-12)
