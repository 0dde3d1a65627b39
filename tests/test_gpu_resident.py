"""GPU parity of the resident (persistent) chunk kernel against the oracle.

The resident kernel runs a whole chunk -- every Euler step, every layer --
in one launch of one CTA per SM (RTV_PATH=resident selects it for the bf16
experts whose shapes it serves).  Its split-K partial sums meet in fp32 in
L2 in arrival order, so repeated calls agree to rounding, not bit for bit.
"""

import numpy as np
import pytest

from oracle import expert as O
from synthetic import get_config, make_draft, make_noise, make_state, make_weights
from tests.helpers import bf16_tolerance_ok, build_expert, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture
def resident(monkeypatch):
    monkeypatch.setenv("RTV_PATH", "resident")
    yield


def _denoise(cfg, n_steps=None, batch=None):
    n = cfg.n_steps if n_steps is None else n_steps
    ex, weights, kv = build_expert(cfg, batch=batch)
    noise, state = make_noise(cfg, batch=batch), make_state(cfg, batch=batch)
    got = ex.denoise(noise, state, n)
    s, bits = ex.status()
    assert s == 0 and bits == 0, bits
    launches = ex.kernels_per_call(n)
    ex.close()
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, kv, n)
    return got, ref, launches


def test_resident_full_chunk_matches_oracle(cuda_ok, resident):
    cfg = get_config("pi0-bf16")
    got, ref, launches = _denoise(cfg)
    print("resident pi0-bf16 rel_l2", rel_l2(got, ref), "max_abs", np.max(np.abs(got - ref)), "kernels", launches)
    assert launches == 1
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("prefix_len", [37, 64, 960])
def test_resident_prefix_tiling_edges(cuda_ok, resident, prefix_len):
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=prefix_len)
    got, ref, _ = _denoise(cfg, n_steps=3)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("variant", [dict(suffix_mask="pi0_block"), dict(rope_theta=0.0), dict(n_kv_heads=2)])
def test_resident_attention_variants(cuda_ok, resident, variant):
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=200, **variant)
    got, ref, _ = _denoise(cfg, n_steps=3)
    assert bf16_tolerance_ok(got, ref), (variant, rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_resident_batch_two_matches_oracle(cuda_ok, resident):
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=300)
    got, ref, _ = _denoise(cfg, n_steps=2, batch=2)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_resident_repeat_calls_agree_to_rounding(cuda_ok, resident):
    """The split-K sums meet in arrival order: the last bits of a sum differ
    between calls, and through the bf16 roundings of every operand that
    follows, the two calls' rounding noise decorrelates.  Repeated calls then
    differ at the bf16 level (not more), and each stays within the oracle's
    tolerance."""
    cfg = get_config("pi0-bf16", n_layers=2)
    ex, weights, kv = build_expert(cfg)
    noise, state = make_noise(cfg), make_state(cfg)
    a = ex.denoise(noise, state, 5)
    b = ex.denoise(noise, state, 5)
    ex.close()
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, kv, 5)
    assert bf16_tolerance_ok(b, a), rel_l2(b, a)
    assert bf16_tolerance_ok(a, ref) and bf16_tolerance_ok(b, ref)


@pytest.mark.parametrize("n_switch", [0, 1])
def test_resident_verify_three_taus_matches_oracle(cuda_ok, resident, n_switch):
    cfg = get_config("pi0-verify", n_layers=4)
    ex, weights, kv = build_expert(cfg, max_taus=4)
    draft = make_draft(cfg, n_switch=n_switch)
    eps = make_noise(cfg, name="verify_noise")[0]
    state = make_state(cfg)[0]
    W = O.to_f64(weights)
    _, _, ref_d = O.verify(W, cfg, draft, eps, state, kv, cfg.taus, 0.05, cfg.gripper)
    acc, flags, dist = ex.verify(draft, eps, state, cfg.taus, 0.05, cfg.gripper)
    s, bits = ex.status()
    ex.close()
    assert s == 0 and bits == 0
    assert rel_l2(dist, ref_d) <= 1e-2 and np.max(np.abs(dist - ref_d)) <= 3e-2, rel_l2(dist, ref_d)
    # the decision is the rule applied to the device's own distances
    assert (acc, flags) == O.verify_decide(dist, draft, 0.05, cfg.gripper)
