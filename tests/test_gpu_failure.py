"""Failure detection on the GPU, without a GPU fault.

* A non-finite input (a NaN in the noise) propagates to the action chunk; the
  output head records RTV_DEV_NUMERIC, rtv_device_status reports
  RTV_ERR_NUMERIC, and the next clean call on the same context is correct
  (no state of the context keeps the NaN).
* A device-side wait that runs out: the layered kernels given a wait limit of
  one nanosecond, and the resident kernel given two microseconds (it cannot
  pass its first grid barrier in time).  Every CTA stops issuing work, waits
  for the copies and MMAs it already issued, frees its tensor memory and
  returns; the status word reports RTV_DEV_TIMEOUT and the context stays
  usable (a second call reports the same, no CUDA error), and a context with
  the default limit then computes the chunk correctly.
"""

import numpy as np
import pytest

from flow_matching_action_dm0_b200 import ActionExpert
from flow_matching_action_dm0_b200 import _lib as L
from oracle import expert as O
from synthetic import f32_to_bf16_bits, get_config, make_noise, make_prefix_kv, make_state, make_weights
from tests.helpers import bf16_tolerance_ok, build_expert, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("path", ["layered", "resident"])
def test_nan_input_is_reported_and_the_next_call_is_clean(cuda_ok, monkeypatch, path):
    monkeypatch.setenv("RTV_PATH", path)
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=100)
    ex, weights, kv = build_expert(cfg)
    noise, state = make_noise(cfg), make_state(cfg)
    bad = noise.copy()
    bad[0, 3, 5] = np.nan
    out = ex.denoise(bad, state, 3)
    assert not np.all(np.isfinite(out))
    s, bits = L.rtv_device_status(ex.h)
    assert s == L.RTV_ERR_NUMERIC and (bits & L.RTV_DEV_NUMERIC), (s, bits)
    got = ex.denoise(noise, state, 3)
    s, bits = ex.status()
    assert s == 0 and bits == 0
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, kv, 3)
    assert bf16_tolerance_ok(got, ref), rel_l2(got, ref)
    ex.close()


# Wait limits that run out on every launch: the layered kernels' first wait on
# a copy (a weight box is ~1 us away when the MMA thread first looks) at 1 ns;
# the resident kernel's first grid barrier at 2 us.
@pytest.mark.parametrize("path,limit_ns", [("layered", 1), ("resident", 2000)])
def test_wait_that_runs_out_is_reported_and_the_context_stays_usable(cuda_ok, monkeypatch, path, limit_ns):
    monkeypatch.setenv("RTV_PATH", path)
    cfg = get_config("pi0-bf16", n_layers=1, prefix_len=64)
    weights = make_weights(cfg)
    kv = np.ascontiguousarray(f32_to_bf16_bits(make_prefix_kv(cfg)))
    noise, state = make_noise(cfg), make_state(cfg)
    ex = ActionExpert(cfg, barrier_timeout_ns=limit_ns)
    ex.load(weights)
    ex.set_prefix_kv(kv)
    for _ in range(2):
        ex.denoise(noise, state, 2)
        s, bits = L.rtv_device_status(ex.h)
        assert s == L.RTV_ERR_TIMEOUT and (bits & L.RTV_DEV_TIMEOUT), (s, bits)
    ex.close()
    ok = ActionExpert(cfg)
    ok.load(weights)
    ok.set_prefix_kv(kv)
    got = ok.denoise(noise, state, 2)
    s, bits = ok.status()
    assert s == 0 and bits == 0
    ok.close()
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, make_prefix_kv(cfg), 2)
    assert bf16_tolerance_ok(got, ref), rel_l2(got, ref)
