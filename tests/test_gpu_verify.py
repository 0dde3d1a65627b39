"""GPU parity of rtv_verify (FLASH parallel verification) against the oracle.

Distances are compared with the expert's tolerance; the accepted length and
the flags must match exactly whenever no distance lies within 1e-3 of
delta, and the oracle's decision rule applied to the device's own distances
must reproduce the device's decision bit for bit at any delta.
"""

import numpy as np
import pytest

from oracle import expert as O
from synthetic import get_config, make_draft, make_noise, make_state, make_weights
from tests.helpers import build_expert, rel_l2

pytestmark = pytest.mark.gpu


def pick_delta(dist, start=1, margin=2e-3):
    """A delta giving a non-trivial accepted length, with no distance within
    `margin` of it: delta sits between the running max of the per-row worst
    distance and the next row's worst distance (a later row first, so that
    the accepted prefix is as long as the distances allow)."""
    worst = dist.max(axis=0)
    allv = np.sort(dist.ravel())
    for j in range(len(worst) - 1, start - 1, -1):
        lo, hi = worst[:j].max(), worst[j]
        if hi - lo > 2 * margin:
            delta = 0.5 * (lo + hi)
            if np.min(np.abs(allv - delta)) > margin:
                return float(delta), j
    return None, None


def run_verify(cfg, taus, n_switch=0, weights=None, delta=None):
    ex, weights, kv = build_expert(cfg, weights=weights, max_taus=max(4, len(taus)))
    draft = make_draft(cfg, n_switch=n_switch)
    eps = make_noise(cfg, name="verify_noise")[0]
    state = make_state(cfg)[0]
    W = O.to_f64(weights)
    _, _, ref_dist = O.verify(W, cfg, draft, eps, state, kv, taus, 0.05, cfg.gripper)
    if delta is None:
        delta, _ = pick_delta(ref_dist)
        assert delta is not None
    ref_acc, ref_flags, _ = O.verify(W, cfg, draft, eps, state, kv, taus, delta, cfg.gripper)
    acc, flags, dist = ex.verify(draft, eps, state, taus, delta, cfg.gripper)
    s, bits = ex.status()
    assert s == 0 and bits == 0
    return ex, (acc, flags, dist), (ref_acc, ref_flags, ref_dist), (draft, eps, state, delta)


@pytest.mark.parametrize("n_switch", [0, 1])
def test_tiny_fp32_verify_matches_oracle(cuda_ok, n_switch):
    cfg = get_config("tiny-fp32")
    ex, got, ref, (draft, _, _, delta) = run_verify(cfg, (0.2, 0.5, 0.8), n_switch=n_switch)
    ex.close()
    assert np.max(np.abs(got[2] - ref[2])) <= 1e-4
    assert got[0] == ref[0] and got[1] == ref[1]
    assert bool(got[1] & 2) == bool(n_switch)


@pytest.mark.parametrize("n_switch", [0, 1])
def test_pi0_verify_three_taus_matches_oracle(cuda_ok, n_switch):
    # the draft of the FLASH verification workload has 0 or 1 gripper sign switch:
    # without one the fallback flag comes from the accepted length alone
    cfg = get_config("pi0-verify")
    ex, got, ref, (draft, _, _, delta) = run_verify(cfg, cfg.taus, n_switch=n_switch)
    ex.close()
    print("pi0-verify n_switch", n_switch, "rel_l2(dist) =", rel_l2(got[2], ref[2]), "accepted", got[0], ref[0],
          "delta", delta)
    assert rel_l2(got[2], ref[2]) <= 1e-2
    assert np.max(np.abs(got[2] - ref[2])) <= 3e-2
    assert got[0] == ref[0] and got[1] == ref[1]
    assert bool(got[1] & 2) == bool(n_switch)


def test_decision_rule_on_device_distances_is_bit_exact(cuda_ok):
    cfg = get_config("pi0-verify", n_layers=2)
    ex, got, ref, (draft, eps, state, _) = run_verify(cfg, (0.2, 0.5, 0.8), n_switch=1)
    dist = got[2]
    # delta at, just above and just below device distances, and at the extremes
    cands = [0.0, float(dist.max()) * 2, float(dist[1, 3]), float(np.nextafter(np.float32(dist[0, 5]), np.inf)),
             float(np.median(dist))]
    for delta in cands:
        # the decision of a call is the rule applied to that call's own distances
        # (repeated calls agree to fp32 rounding, not bit for bit)
        acc, flags, d2 = ex.verify(draft, eps, state, (0.2, 0.5, 0.8), delta, cfg.gripper)
        assert rel_l2(d2, dist) <= 1e-5
        assert (acc, flags) == O.verify_decide(d2, draft, delta, cfg.gripper)
    ex.close()


def test_verify_taus_are_independent_blocks(cuda_ok):
    """Batched taus see only their own suffix: each row of d equals the
    single-tau call's row, and the tau = 0 row is exactly 0."""
    cfg = get_config("pi0-verify", n_layers=2)
    ex, got, _, (draft, eps, state, delta) = run_verify(cfg, (0.0, 0.5, 0.8))
    for i, tau in enumerate((0.0, 0.5, 0.8)):
        _, _, d1 = ex.verify(draft, eps, state, (tau,), delta, cfg.gripper)
        np.testing.assert_allclose(d1[0], got[2][i], rtol=2e-3, atol=1e-5)
    assert np.all(got[2][0] == 0.0)
    ex.close()


def test_constant_velocity_expert_closed_form_distances(cuda_ok):
    """Zero action_out weights: d_i[h] = tau_i * ||eps_h - D_h - b||."""
    cfg = get_config("tiny-fp32")
    w = make_weights(cfg)
    w["action_out_proj.w"] = np.zeros_like(w["action_out_proj.w"])
    taus = (0.2, 0.5, 0.8)
    ex, got, _, (draft, eps, _, _) = run_verify(cfg, taus, weights=w, delta=0.05)
    ex.close()
    b = w["action_out_proj.b"].astype(np.float64)
    for i, tau in enumerate(taus):
        expect = tau * np.linalg.norm(eps.astype(np.float64) - draft - b, axis=1)
        np.testing.assert_allclose(got[2][i], expect, rtol=1e-5, atol=1e-6)


def test_verify_argument_errors(cuda_ok):
    from flow_matching_action_dm0_b200 import RtvError
    cfg = get_config("tiny-fp32")
    ex, _, _ = build_expert(cfg)
    d = make_draft(cfg)
    e = make_noise(cfg, name="verify_noise")[0]
    s = make_state(cfg)[0]
    for taus, gd in (((1.5,), cfg.gripper), ((0.5,), cfg.action_dim), ((0.1,) * 9, cfg.gripper)):
        with pytest.raises(RtvError):
            ex.verify(d, e, s, taus, 0.05, gd)
    ex.close()
