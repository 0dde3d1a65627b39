"""Pins of the oracle against what the pages and the mathematics fix.

Each test is chosen so that a plausible slip in the oracle (a wrong sign in
the Euler step, a dropped residual, a transposed operand, an off-by-one in
the accepted length, a wrong RoPE pairing) fails at least one of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import expert as O
from synthetic import get_config, make_draft, make_noise, make_prefix_kv, make_state, make_weights
from tests import torch_restatement as TR

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(**kw):
    return get_config("tiny-fp32", **kw)


def tiny_weights(cfg, seed=0):
    return O.to_f64(make_weights(cfg, seed))


# ---------------------------------------------------------------------------
# Euler integration   (DM0.5 guide, sec. 5.3)
# ---------------------------------------------------------------------------

def test_euler_lands_on_the_data_for_the_straight_path_field():
    """x_t = t*eps + (1-t)*a has velocity (x - a)/t = eps - a along the path;
    Euler from x_1 = eps must land exactly on a (any N)."""
    rng = np.random.default_rng(1)
    a = rng.standard_normal((5, 3))
    eps = rng.standard_normal((5, 3))
    for n in (1, 3, 10):
        x0 = O.euler_integrate(lambda x, t: (x - a) / t, eps, n)
        np.testing.assert_allclose(x0, a, rtol=0, atol=1e-12)


def test_euler_time_schedule_left_riemann_sum():
    """With v(x, t) = t*b the result is eps - b * sum_k t_k / N = eps - b (N+1)/(2N)."""
    b = np.array([0.3, -1.2])
    eps = np.array([1.0, 2.0])
    for n in (1, 2, 10):
        x0 = O.euler_integrate(lambda x, t: t * b, eps, n)
        np.testing.assert_allclose(x0, eps - b * (n + 1) / (2 * n), rtol=0, atol=1e-13)


def test_denoise_constant_velocity_expert_is_noise_minus_bias():
    """action_out_proj weights = 0 makes the expert's velocity the bias b for any
    input, so 10 Euler steps of dt = 0.1 give eps - b."""
    cfg = tiny()
    W = tiny_weights(cfg)
    W["action_out_proj.w"][:] = 0.0
    b = W["action_out_proj.b"]
    noise = make_noise(cfg, batch=2).astype(np.float64)
    x = O.denoise(W, cfg, noise, make_state(cfg, batch=2), make_prefix_kv(cfg, batch=2), 10)
    np.testing.assert_allclose(x, noise - b, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# FLASH endpoint reconstruction and decision   (FLASH, sec. 02, 03.2, 03.3)
# ---------------------------------------------------------------------------

def test_endpoint_recovers_draft_under_exact_velocity():
    """v = eps - D is the exact velocity of the straight path through D, so
    X_tau - tau*v = D at every tau: distances 0, whole chunk accepted."""
    cfg = tiny()
    rng = np.random.default_rng(2)
    d = make_draft(cfg).astype(np.float64)
    eps = rng.standard_normal(d.shape)
    n_acc, flags, dist = O.verify_with_velocity(lambda x, t: eps - d, d, eps, (0.0, 0.2, 0.5, 0.8, 1.0),
                                                0.05, cfg.gripper)
    assert np.max(dist) < 1e-12
    assert n_acc == cfg.chunk_len and flags == 0


def test_endpoint_distance_closed_form_for_constant_velocity_expert():
    """With the velocity fixed to b, A_hat - D = tau (eps - D - b)."""
    cfg = tiny()
    W = tiny_weights(cfg)
    W["action_out_proj.w"][:] = 0.0
    b = W["action_out_proj.b"]
    d = make_draft(cfg, n_switch=1).astype(np.float64)
    eps = make_noise(cfg, name="verify_noise")[0].astype(np.float64)
    taus = (0.0, 0.2, 0.5, 0.8)
    _, _, dist = O.verify(W, cfg, d, eps, make_state(cfg)[0], make_prefix_kv(cfg), taus, 0.05, cfg.gripper)
    for i, tau in enumerate(taus):
        np.testing.assert_allclose(dist[i], tau * np.linalg.norm(eps - d - b, axis=1), rtol=1e-12, atol=1e-14)


def test_constant_velocity_accept_length_closed_form():
    """With the velocity fixed to b and D = eps - b - z, the distances are
    d_i[h] = tau_i * |z_h|; rows 0-2 pass at every tau and row 3 fails at
    tau = 0.8, so exactly 3 rows are accepted."""
    cfg = tiny()
    W = tiny_weights(cfg)
    W["action_out_proj.w"][:] = 0.0
    b = W["action_out_proj.b"]
    eps = make_noise(cfg, name="verify_noise")[0].astype(np.float64)
    z = np.zeros((cfg.chunk_len, cfg.action_dim))
    z[:, 0] = [0.01, 0.02, 0.03, 0.07, 0.01, 0.01, 0.01, 0.01]
    d = eps - b - z
    taus = (0.2, 0.5, 0.8)
    n_acc, flags, dist = O.verify(W, cfg, d, eps, make_state(cfg)[0], make_prefix_kv(cfg), taus,
                                  0.05, cfg.gripper)
    for i, tau in enumerate(taus):
        np.testing.assert_allclose(dist[i], tau * np.abs(z[:, 0]), rtol=1e-9, atol=1e-14)
    assert n_acc == 3
    assert bool(flags & O.FLAG_SWITCH) == bool(O.gripper_switch_rows(d, cfg.gripper).size)


def test_decide_golden_cases():
    spec = json.load(open(os.path.join(GOLDEN, "flash_decide_cases.json")))
    for case in spec["cases"]:
        dist = np.array(case["dist"], dtype=np.float64)
        draft = np.zeros((dist.shape[1], 3))
        draft[:, 2] = case["gripper"]
        n_acc, flags = O.verify_decide(dist, draft, spec["delta"], 2)
        assert (n_acc, flags) == (case["accepted"], case["flags"]), case["name"]
        assert O.fallback(flags) == (case["accepted"] == 0 or bool(flags & 2))


def test_decide_bruteforce_all_small_patterns():
    """Every pass/fail pattern over T=2, H=4 and every gripper pattern over H=4."""
    delta = 0.05
    for bits in itertools.product([0, 1], repeat=8):
        dist = np.where(np.array(bits).reshape(2, 4) == 1, 0.01, 0.07)
        for g in itertools.product([-1.0, 1.0], repeat=4):
            draft = np.zeros((4, 2))
            draft[:, 1] = g
            n_acc, flags = O.verify_decide(dist, draft, delta, 1)
            passing = [L for L in range(5) if all(dist[i][h] < delta for i in range(2) for h in range(L))]
            assert n_acc == max(passing)
            sw = [h for h in range(1, 4) if (g[h] > 0) != (g[h - 1] > 0)]
            assert bool(flags & 1) == (n_acc == 0)
            assert bool(flags & 2) == bool(sw)
            assert bool(flags & 4) == any(h < n_acc for h in sw)


def test_gripper_switch_rows_zero_one_switch_drafts():
    cfg = tiny()
    d0 = make_draft(cfg, n_switch=0)
    d1 = make_draft(cfg, n_switch=1)
    assert O.gripper_switch_rows(d0, cfg.gripper).size == 0
    rows = O.gripper_switch_rows(d1, cfg.gripper)
    assert rows.size == 1 and 1 <= rows[0] < cfg.chunk_len


# ---------------------------------------------------------------------------
# attention   (DM0.5 guide, sec. 5.1-5.2 prefix KV access; reading R3)
# ---------------------------------------------------------------------------

def _brute_attention(q, k, v, visible):
    s_len, hq, d = q.shape
    hkv = k.shape[1]
    out = np.zeros_like(q)
    for r in range(s_len):
        for j in range(hq):
            kv = j // (hq // hkv)
            logits = [sum(q[r, j, e] * k[n, kv, e] for e in range(d)) / math.sqrt(d)
                      for n in range(k.shape[0])]
            mx = max(l for n, l in enumerate(logits) if visible[r, n])
            wts = [math.exp(l - mx) if visible[r, n] else 0.0 for n, l in enumerate(logits)]
            tot = sum(wts)
            for e in range(d):
                out[r, j, e] = sum(wts[n] * v[n, kv, e] for n in range(k.shape[0])) / tot
    return out


@pytest.mark.parametrize("p_len,s_len,hq,hkv,mode", [(1, 2, 2, 1, "bidir"), (3, 4, 4, 2, "bidir"),
                                                      (3, 4, 2, 1, "pi0_block"), (7, 9, 4, 1, "bidir")])
def test_attention_matches_bruteforce(p_len, s_len, hq, hkv, mode):
    rng = np.random.default_rng(p_len * 10 + s_len)
    d = 4
    q = rng.standard_normal((s_len, hq, d))
    k = rng.standard_normal((p_len + s_len, hkv, d))
    v = rng.standard_normal((p_len + s_len, hkv, d))
    vis = O.suffix_visibility(s_len, p_len, mode)
    np.testing.assert_allclose(O.attention(q, k, v, vis), _brute_attention(q, k, v, vis), rtol=1e-12, atol=1e-13)


def test_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(5)
    s_len, p_len, hq, hkv, d = 9, 64, 4, 1, 16
    q = rng.standard_normal((s_len, hq, d))
    k = rng.standard_normal((p_len + s_len, hkv, d))
    v = rng.standard_normal((p_len + s_len, hkv, d))
    for mode in ("bidir", "pi0_block"):
        vis = O.suffix_visibility(s_len, p_len, mode)
        ref = F.scaled_dot_product_attention(
            torch.tensor(q).transpose(0, 1), torch.tensor(k).transpose(0, 1).expand(hq, -1, -1),
            torch.tensor(v).transpose(0, 1).expand(hq, -1, -1), attn_mask=torch.tensor(vis)).transpose(0, 1)
        np.testing.assert_allclose(O.attention(q, k, v, vis), ref.numpy(), rtol=1e-12, atol=1e-13)


def test_attention_invariants():
    rng = np.random.default_rng(6)
    d = 8
    # a single key returns its value
    q = rng.standard_normal((1, 2, d))
    k = rng.standard_normal((1, 1, d))
    v = rng.standard_normal((1, 1, d))
    out = O.attention(q, k, v, np.ones((1, 1), bool))
    np.testing.assert_allclose(out[0, 0], v[0, 0], atol=1e-15)
    np.testing.assert_allclose(out[0, 1], v[0, 0], atol=1e-15)
    # equal keys average the values
    k = np.repeat(rng.standard_normal((1, 1, d)), 5, axis=0)
    v = rng.standard_normal((5, 1, d))
    out = O.attention(rng.standard_normal((3, 2, d)), k, v, np.ones((3, 5), bool))
    np.testing.assert_allclose(out[1, 1], v[:, 0].mean(axis=0), atol=1e-14)
    # permuting keys with their values changes nothing
    k = rng.standard_normal((6, 1, d))
    v = rng.standard_normal((6, 1, d))
    q = rng.standard_normal((3, 2, d))
    perm = rng.permutation(6)
    vis = np.ones((3, 6), bool)
    np.testing.assert_allclose(O.attention(q, k[perm], v[perm], vis), O.attention(q, k, v, vis), atol=1e-14)
    # GQA equals MHA with the kv head replicated
    q = rng.standard_normal((3, 4, d))
    k2 = rng.standard_normal((6, 2, d))
    v2 = rng.standard_normal((6, 2, d))
    mha = O.attention(q, np.repeat(k2, 2, axis=1), np.repeat(v2, 2, axis=1), vis)
    np.testing.assert_allclose(O.attention(q, k2, v2, vis), mha, atol=1e-14)


def test_suffix_mask_visibility():
    """bidir: perturbing an action row's key/value moves the state row's output;
    pi0_block: it does not, but it still moves the action rows."""
    rng = np.random.default_rng(7)
    p_len, s_len, d = 5, 4, 4
    q = rng.standard_normal((s_len, 1, d))
    k = rng.standard_normal((p_len + s_len, 1, d))
    v = rng.standard_normal((p_len + s_len, 1, d))
    k2, v2 = k.copy(), v.copy()
    k2[p_len + 2] += 1.0
    v2[p_len + 2] += 1.0
    for mode, state_changes in (("bidir", True), ("pi0_block", False)):
        vis = O.suffix_visibility(s_len, p_len, mode)
        a, b = O.attention(q, k, v, vis), O.attention(q, k2, v2, vis)
        assert (np.abs(a[0] - b[0]).max() > 1e-6) == state_changes
        assert np.abs(a[1] - b[1]).max() > 1e-6


# ---------------------------------------------------------------------------
# elementwise pieces against library routines and closed forms
# ---------------------------------------------------------------------------

def test_rms_norm_vs_torch_and_scale_invariance():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((5, 32))
    g = rng.standard_normal(32) * 0.1
    ref = F.rms_norm(torch.tensor(x), (32,), weight=1.0 + torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, g, 0.0), O.rms_norm(x, g, 0.0), rtol=1e-13)


def test_gelu_swish_vs_torch():
    z = np.linspace(-8, 8, 401)
    np.testing.assert_allclose(O.gelu_tanh(z), F.gelu(torch.tensor(z), approximate="tanh").numpy(),
                               rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.swish(z), F.silu(torch.tensor(z)).numpy(), rtol=1e-13, atol=1e-15)


def test_time_embedding_closed_forms():
    w = 64
    e0 = O.time_embedding(0.0, w)
    np.testing.assert_array_equal(e0[:32], 0.0)
    np.testing.assert_array_equal(e0[32:], 1.0)
    e1 = O.time_embedding(1.0, w)
    # first period 4e-3: angle 500*pi; last period 4.0: angle pi/2
    assert abs(e1[0]) < 1e-12 and abs(e1[32] - 1.0) < 1e-12
    assert abs(e1[31] - 1.0) < 1e-15 and abs(e1[63]) < 1e-15


def test_rope_closed_form_and_relative_position():
    d = 8
    theta = 10000.0
    e0 = np.zeros((1, 1, d))
    e0[0, 0, 1] = 1.0                       # pair (1, 1 + D/2)
    p = 3
    r = O.rope(e0, np.array([p]), theta)[0, 0]
    ang = p * theta ** (-2 * 1 / d)
    expect = np.zeros(d)
    expect[1], expect[1 + d // 2] = math.cos(ang), math.sin(ang)
    np.testing.assert_allclose(r, expect, atol=1e-15)
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    dots = [float(np.sum(O.rope(q, np.array([a + 5]), theta) * O.rope(k, np.array([a]), theta)))
            for a in (0, 7, 100)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(O.rope(q, np.array([11]), theta)), np.linalg.norm(q), rtol=1e-14)
    np.testing.assert_array_equal(O.rope(q, np.array([11]), 0.0), q)


# ---------------------------------------------------------------------------
# whole expert
# ---------------------------------------------------------------------------

def test_zero_layers_pass_the_embedding_through():
    """All layer matrices 0: every layer adds 0 to the residual stream, so
    v = W_ao . RMSNorm_f(W_ai x + b_ai + c(t)) + b_ao."""
    cfg = tiny()
    W = tiny_weights(cfg)
    for k in W:
        if k.startswith("layers.") and k.endswith(".w"):
            W[k][:] = 0.0
    x = make_noise(cfg)[0].astype(np.float64)
    t = 0.7
    kv = make_prefix_kv(cfg)
    v = O.expert_velocity(W, cfg, x, make_state(cfg)[0], t, kv[:, 0, 0], kv[:, 1, 0])
    c = TR.time_cond(W, t, cfg.width).numpy()
    h = x @ W["action_in_proj.w"].T + W["action_in_proj.b"] + c
    hn = F.rms_norm(torch.tensor(h), (cfg.width,), weight=1.0 + torch.tensor(W["final_norm.g"]), eps=cfg.rms_eps)
    expect = hn.numpy() @ W["action_out_proj.w"].T + W["action_out_proj.b"]
    np.testing.assert_allclose(v, expect, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mode,theta", [("bidir", 10000.0), ("pi0_block", 10000.0), ("bidir", 0.0)])
def test_expert_matches_independent_torch_statement(mode, theta):
    cfg = tiny(suffix_mask=mode, rope_theta=theta, n_kv_heads=1)
    W = tiny_weights(cfg, seed=3)
    kv = make_prefix_kv(cfg, seed=3)
    state = make_state(cfg, seed=3)[0]
    xs = np.stack([make_noise(cfg, seed=s)[0] for s in (3, 4)])
    ts = (0.9, 0.25)
    ref = TR.velocity(W, cfg, xs, state, ts, kv[:, 0, 0], kv[:, 1, 0])
    for g in range(2):
        v = O.expert_velocity(W, cfg, xs[g], state, ts[g], kv[:, 0, 0], kv[:, 1, 0])
        np.testing.assert_allclose(v, ref[g], rtol=1e-10, atol=1e-12)


def test_expert_gqa_two_kv_heads_matches_torch_statement():
    cfg = tiny(n_kv_heads=2)
    W = tiny_weights(cfg, seed=4)
    kv = make_prefix_kv(cfg, seed=4)
    state = make_state(cfg, seed=4)[0]
    x = make_noise(cfg, seed=4)
    ref = TR.velocity(W, cfg, x, state, (0.5,), kv[:, 0, 0], kv[:, 1, 0])
    v = O.expert_velocity(W, cfg, x[0], state, 0.5, kv[:, 0, 0], kv[:, 1, 0])
    np.testing.assert_allclose(v, ref[0], rtol=1e-10, atol=1e-12)


def test_batch_elements_are_independent():
    cfg = tiny()
    W = tiny_weights(cfg)
    noise, state, kv = make_noise(cfg, batch=2), make_state(cfg, batch=2), make_prefix_kv(cfg, batch=2)
    both = O.denoise(W, cfg, noise, state, kv, 3)
    one = O.denoise(W, cfg, noise[1:], state[1:], kv[:, :, 1:], 3)
    np.testing.assert_array_equal(both[1], one[0])


# ---------------------------------------------------------------------------
# FP8 E4M3 MLP weights
# ---------------------------------------------------------------------------

def test_e4m3_decode_fixed_codes():
    """Codes whose values the format fixes: zero, one, the extremes of both
    ranges, a subnormal, halves, and NaN."""
    codes = {0x00: 0.0, 0x38: 1.0, 0x30: 0.5, 0x3C: 1.5, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0,
             0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0xB8: -1.0, 0x77: 240.0}
    got = O.e4m3_decode(np.array(list(codes), dtype=np.uint8))
    assert np.array_equal(got, np.array(list(codes.values())))
    assert np.isnan(O.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    assert np.signbit(O.e4m3_decode(np.array([0x80], dtype=np.uint8)))[0]


def test_e4m3_decode_matches_torch_float8_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_fp8_mlp_weights_within_the_format_bound():
    """Decoded FP8 weights (decode x per-row scale) stay within E4M3's rounding
    bound of the draw they encode: relative 2^-4 for normal values, absolute
    scale * 2^-10 for subnormal ones; each row's largest magnitude is exact."""
    from synthetic.gen import _normal
    cfg = get_config("pi0-fp8mlp", n_layers=1, width=256, mlp_dim=512, n_q_heads=2, head_dim=128)
    raw = make_weights(cfg)
    W = O.to_f64(raw)
    for name in ("gate_proj", "up_proj", "down_proj"):
        key = f"layers.0.{name}.w"
        draw = _normal(cfg.seed, key, raw[key].shape, cfg.weight_std).astype(np.float64)
        scale = raw[f"layers.0.{name}.s"].astype(np.float64)[:, None]
        err = np.abs(W[key] - draw)
        normal = np.abs(draw) / scale >= 2.0 ** -6
        assert np.all(err[normal] <= 2.0 ** -4 * np.abs(draw)[normal] * (1 + 1e-6))
        assert np.all(err[~normal] <= (scale * 2.0 ** -10 * (1 + 1e-6) + 0 * err)[~normal])
        rows = np.arange(draw.shape[0])
        amax_idx = np.argmax(np.abs(draw), axis=1)
        assert np.allclose(W[key][rows, amax_idx], draw[rows, amax_idx], rtol=1e-6, atol=0)


# ---------------------------------------------------------------------------
# structure of the batched verification, and the GEMM primitive
# ---------------------------------------------------------------------------

def test_batched_verify_equals_separate_single_tau_calls():
    """Verification at several taus is the taus one at a time: the distance
    row of tau_i does not depend on the other taus, and the accepted length
    is the shortest of the single-tau lengths."""
    cfg = tiny()
    W = tiny_weights(cfg, seed=7)
    kv = make_prefix_kv(cfg, seed=7)
    state = make_state(cfg, seed=7)[0]
    draft = make_draft(cfg, seed=7)
    eps = make_noise(cfg, seed=7)[0]
    taus = (0.2, 0.5, 0.8)
    n_acc, _, dist = O.verify(W, cfg, draft, eps, state, kv, taus, 0.4, cfg.gripper)
    singles = [O.verify(W, cfg, draft, eps, state, kv, (t,), 0.4, cfg.gripper) for t in taus]
    for i, (_, _, d1) in enumerate(singles):
        np.testing.assert_array_equal(dist[i], d1[0])
    assert n_acc == min(s[0] for s in singles)


def test_linear_matches_a_naive_triple_loop():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 5))
    w = rng.standard_normal((4, 5))
    b = rng.standard_normal(4)
    y = np.zeros((3, 4))
    for i in range(3):
        for j in range(4):
            acc = 0.0
            for k in range(5):
                acc += x[i, k] * w[j, k]
            y[i, j] = acc + b[j]
    np.testing.assert_allclose(O.linear(x, w, b), y, rtol=1e-14, atol=1e-14)
