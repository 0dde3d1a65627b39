"""Shared test helpers: build a library context from seeded synthetic inputs."""

from __future__ import annotations

import numpy as np

from synthetic import make_prefix_kv, make_weights


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def build_expert(cfg, weights=None, kv=None, batch=None, max_taus=4, device=0, prefix_len=None):
    """ActionExpert with the config's seeded weights and prefix KV installed."""
    from flow_matching_action_dm0_b200 import ActionExpert
    batch = cfg.batch if batch is None else batch
    weights = make_weights(cfg) if weights is None else weights
    kv = make_prefix_kv(cfg, batch=batch, prefix_len=prefix_len) if kv is None else kv
    ex = ActionExpert(cfg, device=device, max_batch=max(batch, 1), max_taus=max_taus,
                      max_prefix_len=max(cfg.prefix_len, kv.shape[3]))
    ex.load(weights)
    ex.set_prefix_kv(np.ascontiguousarray(kv))
    ex.synchronize()
    return ex, weights, kv


def bf16_tolerance_ok(got, ref, rel=1e-2, abs_=3e-2):
    return rel_l2(got, ref) <= rel and float(np.max(np.abs(np.asarray(got, np.float64) - ref))) <= abs_
