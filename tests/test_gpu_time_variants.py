"""GPU parity of the time-conditioning variants against the oracle: Pi0's
concat time MLP (RTV_TIME_CONCAT) and DM0.5's per-layer time modulator
(RTV_TIME_ADARMS), on the SIMT path (fp32: max-abs <= 1e-4) and the
tensor-core path (bf16: relative L2 <= 1e-2, max-abs <= 3e-2), denoising
and verification (accepted length and flags exact).
"""

import numpy as np
import pytest

from oracle import expert as O
from synthetic import get_config, make_draft, make_noise, make_state
from tests.helpers import bf16_tolerance_ok, build_expert, rel_l2

pytestmark = pytest.mark.gpu


def _denoise(cfg, n_steps, batch=1):
    ex, weights, kv = build_expert(cfg, batch=batch)
    noise, state = make_noise(cfg, batch=batch), make_state(cfg, batch=batch)
    got = ex.denoise(noise, state, n_steps)
    s, bits = ex.status()
    assert s == 0 and bits == 0
    path = ex.path
    ex.close()
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, kv, n_steps)
    return got, ref, path


def _verify(cfg, delta):
    ex, weights, kv = build_expert(cfg, batch=1)
    draft, eps, state = make_draft(cfg), make_noise(cfg)[0], make_state(cfg)[0]
    acc, flags, dist = ex.verify(draft, eps, state, cfg.taus, delta, cfg.gripper)
    s, bits = ex.status()
    assert s == 0 and bits == 0
    ex.close()
    r_acc, r_flags, r_dist = O.verify(O.to_f64(weights), cfg, draft, eps, state, kv, cfg.taus, delta, cfg.gripper)
    return (acc, flags, dist), (r_acc, r_flags, r_dist)


@pytest.mark.parametrize("tc", ["concat", "adarms"])
@pytest.mark.parametrize("batch", [1, 2])
def test_fp32_variant_denoise_matches_oracle(cuda_ok, tc, batch):
    cfg = get_config("tiny-fp32", time_cond=tc)
    got, ref, path = _denoise(cfg, 10, batch)
    assert path == "simt"
    assert np.max(np.abs(got - ref)) <= 1e-4, np.max(np.abs(got - ref))


@pytest.mark.parametrize("tc", ["concat", "adarms"])
def test_fp32_variant_verify_matches_oracle(cuda_ok, tc):
    cfg = get_config("tiny-fp32", time_cond=tc)
    (acc, flags, dist), (r_acc, r_flags, r_dist) = _verify(cfg, 0.5)
    assert np.max(np.abs(dist - r_dist)) <= 1e-4
    assert (acc, flags) == (r_acc, r_flags)


@pytest.mark.parametrize("name", ["pi0-concat", "dm05-adarms"])
@pytest.mark.parametrize("batch", [1, 3])
def test_bf16_variant_two_layers_matches_oracle(cuda_ok, name, batch):
    cfg = get_config(name, n_layers=2)
    got, ref, path = _denoise(cfg, 3, batch)
    assert path == "tcgen05"
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("name", ["pi0-concat", "dm05-adarms"])
def test_bf16_variant_verify_matches_oracle(cuda_ok, name):
    cfg = get_config(name, n_layers=2)
    (acc, flags, dist), (r_acc, r_flags, r_dist) = _verify(cfg, 0.3)
    assert rel_l2(dist, r_dist) <= 1e-2
    near = np.abs(np.asarray(r_dist, np.float64) - 0.3) < 1e-3
    if not near.any():
        assert (acc, flags) == (r_acc, r_flags)


def test_bf16_adarms_simt_path_matches_oracle(cuda_ok, monkeypatch):
    monkeypatch.setenv("RTV_PATH", "simt")
    cfg = get_config("dm05-adarms", n_layers=2)
    got, ref, path = _denoise(cfg, 2)
    assert path == "simt"
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("name", ["dm05-adarms", "pi0-concat"])
def test_variant_full_chunk_matches_oracle(cuda_ok, name):
    """The full 18-layer, 816-prefix, 10-step chunk."""
    cfg = get_config(name)
    got, ref, _ = _denoise(cfg, 10)
    err_rel, err_abs = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    print(f"{name} rel_l2={err_rel:.3e} max_abs={err_abs:.3e}")
    assert err_rel <= 1e-2 and err_abs <= 3e-2
