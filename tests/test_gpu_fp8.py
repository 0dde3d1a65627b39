"""GPU parity of the FP8 E4M3 MLP configuration against the oracle.

Gate/up/down are given as E4M3 codes with one fp32 scale per output row; the
oracle decodes them by the format's definition and multiplies by the scale in
fp64, the device widens the codes to bf16 exactly and applies the scale after
its fp32 accumulation.  Same bf16 tolerances as the bf16 expert (relative L2
<= 1e-2, max-abs <= 3e-2).
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
    assert ex.path == "tcgen05"
    ex.close()
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, kv, n_steps)
    return got, ref


def test_fp8_mlp_two_layers_matches_oracle(cuda_ok):
    cfg = get_config("pi0-fp8mlp", n_layers=2)
    got, ref = _denoise(cfg, 3)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_fp8_mlp_full_chunk_matches_oracle(cuda_ok):
    """The full 18-layer, 560-prefix, 10-step chunk."""
    cfg = get_config("pi0-fp8mlp")
    got, ref = _denoise(cfg, 10)
    err_rel, err_abs = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    print(f"pi0-fp8mlp rel_l2={err_rel:.3e} max_abs={err_abs:.3e}")
    assert err_rel <= 1e-2 and err_abs <= 3e-2


def test_fp8_mlp_batch_four_matches_oracle(cuda_ok):
    cfg = get_config("pi0-fp8mlp", n_layers=2, batch=4)
    got, ref = _denoise(cfg, 2, batch=4)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_fp8_mlp_batch_sixteen_matches_oracle(cuda_ok):
    cfg = get_config("pi0-fp8mlp", n_layers=2, batch=16)
    got, ref = _denoise(cfg, 2, batch=16)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_fp8_mlp_verify_distances_match_oracle(cuda_ok):
    cfg = get_config("pi0-fp8mlp", n_layers=2)
    ex, weights, kv = build_expert(cfg)
    draft, eps, state = make_draft(cfg), make_noise(cfg)[0], make_state(cfg)[0]
    taus = (0.2, 0.5, 0.8)
    _, _, dist = ex.verify(draft, eps, state, taus, 0.05, cfg.gripper)
    ex.close()
    _, _, ref = O.verify(O.to_f64(weights), cfg, draft, eps, state, kv, taus, 0.05, cfg.gripper)
    assert rel_l2(dist, ref) <= 1e-2


def test_fp8_mlp_refused_on_the_simt_path(cuda_ok, monkeypatch):
    from flow_matching_action_dm0_b200 import ActionExpert, RtvError
    monkeypatch.setenv("RTV_PATH", "simt")
    with pytest.raises(RtvError) as e:
        ActionExpert(get_config("pi0-fp8mlp", n_layers=1))
    assert e.value.status == 8   # RTV_ERR_UNSUPPORTED
